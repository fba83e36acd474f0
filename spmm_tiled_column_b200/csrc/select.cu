// select.cu -- input-adaptive column selection.
//
// "Reduced Matrix Multiplication" (hotelren.com article): §4.1 step 2 picks the channel
// indices to keep from per-channel scores; §4.2 multiplies only on that subset; §5.1
// ranks channels by mean |activation| and keeps a top-k sorted by index; §7.3 shares one
// index set across a block of tokens.  Two rules are provided:
//   threshold: column k is active iff some batch row has x != 0 and not |x| < t;
//   top-k:     the k columns with the largest sum over the batch of |x| (exact), ties
//              to the lower index, listed in ascending order.
#include "spw_internal.cuh"

namespace spw {
namespace {

constexpr int kSelThreads = 1024;
constexpr int kTopkMaxK = 24576;
constexpr int kKeyIndexBits = 19;  // K <= 2^19 keeps (score << 19 | index part) in 64 bits

__global__ void __launch_bounds__(kSelThreads)
threshold_kernel(const uint16_t* __restrict__ x, int B, int K, int ldx, float t,
                 uint32_t* __restrict__ act_bits, uint32_t* __restrict__ count) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint32_t mine = 0;
    for (int base = 0; base < K; base += kSelThreads) {
        const int k = base + tid;
        bool active = false;
        if (k < K)
            for (int b = 0; b < B; b++) active |= passes_threshold(x[(size_t)b * ldx + k], t);
        const uint32_t word = __ballot_sync(0xffffffffu, active);
        if (lane == 0 && k < K) act_bits[k >> 5] = word;
        if (lane == 0) mine += __popc(word);
    }
    __shared__ uint32_t s_cnt[kSelThreads / 32];
    if (lane == 0) s_cnt[warp] = mine;
    __syncthreads();
    if (warp == 0) {
        uint32_t v = s_cnt[lane];
#pragma unroll
        for (int d = 16; d > 0; d >>= 1) v += __shfl_xor_sync(0xffffffffu, v, d);
        if (lane == 0) *count = v;
    }
}

// |x| of an fp16 value as an exact integer multiple of 2^-24; non-finite -> 2^44, above
// any sum of at most 16 finite magnitudes (16 * 65504 * 2^24 < 2^44).
__device__ inline unsigned long long magnitude_units(uint16_t h, bool* nonfinite) {
    const uint32_t e = (h >> 10) & 0x1f, f = h & 0x3ff;
    if (e == 31) {
        *nonfinite = true;
        return 0;
    }
    if (e == 0) return f;
    return (unsigned long long)(1024 + f) << (e - 1);
}

__global__ void __launch_bounds__(kSelThreads)
topk_kernel(const uint16_t* __restrict__ x, int B, int K, int ldx, int kk,
            uint32_t* __restrict__ act_bits, uint32_t* __restrict__ idx) {
    extern __shared__ unsigned long long s_key[];  // K keys
    __shared__ uint32_t s_hist[256];
    __shared__ unsigned long long s_prefix;
    __shared__ uint32_t s_remaining;
    __shared__ uint32_t s_warp_count[kSelThreads / 32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const unsigned long long index_mask = (1ull << kKeyIndexBits) - 1;

    for (int k = tid; k < K; k += kSelThreads) {
        unsigned long long score = 0;
        bool nonfinite = false;
        for (int b = 0; b < B; b++) score += magnitude_units(x[(size_t)b * ldx + k], &nonfinite);
        if (nonfinite) score = 1ull << 44;
        s_key[k] = (score << kKeyIndexBits) | (index_mask - (unsigned long long)k);
    }
    if (tid == 0) {
        s_prefix = 0;
        s_remaining = (uint32_t)kk;
    }
    __syncthreads();

    // Radix select of the kk-th largest key, 8 bits at a time from the top.  Keys are
    // unique (they embed the index), so the selected set {key >= kth} has kk members.
    unsigned long long prefix_mask = 0;
    for (int pass = 0; pass < 8 && kk > 0; pass++) {
        const int shift = 56 - 8 * pass;
        for (int d = tid; d < 256; d += kSelThreads) s_hist[d] = 0;
        __syncthreads();
        const unsigned long long prefix = s_prefix;
        for (int k = tid; k < K; k += kSelThreads) {
            const unsigned long long key = s_key[k];
            if ((key & prefix_mask) == prefix) atomicAdd(&s_hist[(key >> shift) & 255], 1u);
        }
        __syncthreads();
        if (warp == 0) {
            // lane owns digits 255-8*lane .. 248-8*lane (descending)
            uint32_t c[8], sum = 0;
#pragma unroll
            for (int i = 0; i < 8; i++) {
                c[i] = s_hist[255 - 8 * lane - i];
                sum += c[i];
            }
            uint32_t incl = sum;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                uint32_t u = __shfl_up_sync(0xffffffffu, incl, d);
                if (lane >= d) incl += u;
            }
            const uint32_t before = incl - sum;  // keys in higher digits than this lane's
            const uint32_t rem = s_remaining;
            const bool here = before < rem && rem <= incl;
            if (here) {
                uint32_t cum = before;
                for (int i = 0; i < 8; i++) {
                    if (cum + c[i] >= rem) {
                        const unsigned long long digit = (unsigned long long)(255 - 8 * lane - i);
                        s_prefix = prefix | (digit << shift);
                        s_remaining = rem - cum;
                        break;
                    }
                    cum += c[i];
                }
            }
        }
        prefix_mask |= 255ull << shift;
        __syncthreads();
    }
    const unsigned long long kth = s_prefix;

    // Bitmap and ascending index list.
    uint32_t base = 0;
    for (int chunk = 0; chunk < K; chunk += kSelThreads) {
        const int k = chunk + tid;
        const bool sel = kk > 0 && k < K && s_key[k] >= kth;
        const uint32_t word = __ballot_sync(0xffffffffu, sel);
        if (lane == 0 && k < K) act_bits[k >> 5] = word;
        if (lane == 0) s_warp_count[warp] = __popc(word);
        __syncthreads();
        uint32_t warp_base = 0, total = 0;
        for (int w = 0; w < kSelThreads / 32; w++) {
            const uint32_t c = s_warp_count[w];
            if (w < warp) warp_base += c;
            total += c;
        }
        if (sel && idx) idx[base + warp_base + __popc(word & lanemask_lt())] = (uint32_t)k;
        base += total;
        __syncthreads();
    }
}

int check_x(const uint16_t* d_x, int B, int K, int ldx) {
    if (!d_x || B < 1 || B > 16 || K < 1 || ldx < K) return SPW_ERR_INVALID_ARG;
    if (!aligned16(d_x)) return SPW_ERR_ALIGNMENT;
    return SPW_OK;
}

}  // namespace
}  // namespace spw

using namespace spw;

extern "C" {

int spw_select_threshold(const uint16_t* d_x, int B, int K, int ldx, float t,
                         uint32_t* d_act_bits, uint32_t* d_count, void* stream) {
    int rc = check_x(d_x, B, K, ldx);
    if (rc != SPW_OK) return rc;
    if (!d_act_bits || !d_count || !(t >= 0.0f) || isinf(t)) return SPW_ERR_INVALID_ARG;
    if (!aligned16(d_act_bits) || ((uintptr_t)d_count & 3u)) return SPW_ERR_ALIGNMENT;
    threshold_kernel<<<1, kSelThreads, 0, (cudaStream_t)stream>>>(d_x, B, K, ldx, t, d_act_bits,
                                                                  d_count);
    SPW_LAUNCH_CHECK();
    return SPW_OK;
}

int spw_select_topk(const uint16_t* d_x, int B, int K, int ldx, int k, uint32_t* d_act_bits,
                    uint32_t* d_idx, void* stream) {
    int rc = check_x(d_x, B, K, ldx);
    if (rc != SPW_OK) return rc;
    if (!d_act_bits || k < 0 || k > K) return SPW_ERR_INVALID_ARG;
    if (!aligned16(d_act_bits) || ((uintptr_t)d_idx & 3u)) return SPW_ERR_ALIGNMENT;
    if (K > kTopkMaxK) return SPW_ERR_UNSUPPORTED;
    const size_t smem = (size_t)K * sizeof(unsigned long long);
    static bool attr_set[kMaxDevices];
    int dev = 0;
    SPW_CUDA_TRY(cudaGetDevice(&dev));
    if (dev >= 0 && dev < 64 && !attr_set[dev]) {
        SPW_CUDA_TRY(cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          kTopkMaxK * (int)sizeof(unsigned long long)));
        attr_set[dev] = true;
    }
    topk_kernel<<<1, kSelThreads, smem, (cudaStream_t)stream>>>(d_x, B, K, ldx, k, d_act_bits, d_idx);
    SPW_LAUNCH_CHECK();
    return SPW_OK;
}

}  // extern "C"
