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

// Threshold rule, one CTA: each thread tests 8 consecutive columns of every batch row
// with one 16-byte load per row (plain 16-bit loads where a row's 8 columns are not
// 16-byte aligned or run past K), then the 8-bit results of lanes 4w..4w+3 are combined
// into the warp's 32-column word w.
__global__ void __launch_bounds__(kSelThreads)
threshold_kernel(const uint16_t* __restrict__ x, int B, int K, int ldx, float t,
                 uint32_t* __restrict__ act_bits, uint32_t* __restrict__ count) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const bool zero_t = t == 0.0f;
    uint32_t mine = 0;
    for (int base = 0; base < K; base += 8 * kSelThreads) {
        const int k0 = base + 8 * tid;  // this thread's 8 columns
        uint32_t bits = 0;
        if (k0 < K) {
            const bool vec = k0 + 8 <= K && (((uintptr_t)(x + k0) & 15u) == 0) && (ldx % 8 == 0 || B == 1);
            // all rows' loads first (up to 16, independent), then the tests
            uint4 w[16];
#pragma unroll
            for (int b = 0; b < 16; b++) {
                w[b] = make_uint4(0u, 0u, 0u, 0u);
                if (b < B) {
                    const uint16_t* row = x + (size_t)b * ldx + k0;
                    if (vec) {
                        w[b] = __ldg((const uint4*)row);
                    } else {
                        uint16_t v[8];
#pragma unroll
                        for (int e = 0; e < 8; e++) v[e] = k0 + e < K ? row[e] : (uint16_t)0;
                        w[b] = make_uint4((uint32_t)v[0] | ((uint32_t)v[1] << 16), (uint32_t)v[2] | ((uint32_t)v[3] << 16),
                                          (uint32_t)v[4] | ((uint32_t)v[5] << 16), (uint32_t)v[6] | ((uint32_t)v[7] << 16));
                    }
                }
            }
#pragma unroll
            for (int b = 0; b < 16; b++) {
                if (b >= B) break;
                const uint32_t ws[4] = {w[b].x, w[b].y, w[b].z, w[b].w};
#pragma unroll
                for (int e = 0; e < 8; e++) {
                    const uint16_t v = (uint16_t)(ws[e >> 1] >> (16 * (e & 1)));
                    if (zero_t ? (v & 0x7fffu) != 0u : passes_threshold(v, t)) bits |= 1u << e;
                }
            }
        }
        // word w of this warp's 256 columns = the bits of lanes 4w .. 4w+3
        uint32_t word = bits << (8 * (lane & 3));
        word |= __shfl_xor_sync(0xffffffffu, word, 1);
        word |= __shfl_xor_sync(0xffffffffu, word, 2);
        const int kw = base + 256 * warp + 32 * (lane >> 2);  // first column of word lane/4
        if ((lane & 3) == 0 && kw < K) {
            act_bits[kw >> 5] = word;
            mine += __popc(word);
        }
    }
    mine = __reduce_add_sync(0xffffffffu, mine);
    __shared__ uint32_t s_cnt[kSelThreads / 32];
    if (lane == 0) s_cnt[warp] = mine;
    __syncthreads();
    if (warp == 0) {
        const uint32_t v = __reduce_add_sync(0xffffffffu, s_cnt[lane]);
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

// Exclusive prefix over the CTA of one value per thread (kSelThreads threads), in thread
// order; *total receives the sum.  Uses s_warp (kSelThreads / 32 words).
__device__ inline uint32_t block_exclusive_scan(uint32_t v, uint32_t* s_warp, uint32_t* total) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t incl = (uint32_t)warp_inclusive_scan((int)v, lane);
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const uint32_t w = s_warp[lane];
        const uint32_t wi = (uint32_t)warp_inclusive_scan((int)w, lane);
        s_warp[lane] = wi - w;  // exclusive prefix of the warp sums
        if (lane == 31) s_warp[kSelThreads / 32] = wi;
    }
    __syncthreads();
    const uint32_t r = s_warp[warp] + incl - v;
    *total = s_warp[kSelThreads / 32];
    __syncthreads();  // s_warp is reused by the next call
    return r;
}

// Exact top-k, one CTA.  Keys score * 2^19 + (2^19 - 1 - index) are unique and order the
// columns by score, ties to the lower index.  A radix select finds the kk-th largest key:
// it starts at the highest bit any key has set (the keys' top bits are mostly zero), takes
// 11 bits per pass (2048 bins, a CTA-wide scan from the top bin down), and stops as soon
// as the kk-th key's bin is selected whole.  The selected set is {key >= threshold}.
// (Measured on B200 at K = 11008: 16.7 us; per-warp-pair 256-bin histograms and warp-
// aggregated histogram updates were both slower.)
constexpr int kDigitBits = 11;
constexpr int kBins = 1 << kDigitBits;
static_assert(kBins == 2 * kSelThreads, "the scan gives each thread two bins");

__global__ void __launch_bounds__(kSelThreads)
topk_kernel(const uint16_t* __restrict__ x, int B, int K, int ldx, int kk,
            uint32_t* __restrict__ act_bits, uint32_t* __restrict__ idx) {
    extern __shared__ unsigned long long s_key[];  // K keys, then the word offsets
    __shared__ uint32_t s_hist[kBins];
    __shared__ uint32_t s_warp[kSelThreads / 32 + 1];
    __shared__ unsigned long long s_thresh;
    __shared__ uint32_t s_remaining, s_done, s_or_lo, s_or_hi;
    const int tid = threadIdx.x, lane = tid & 31;
    const unsigned long long index_mask = (1ull << kKeyIndexBits) - 1;

    if (tid == 0) {
        s_thresh = 0;
        s_remaining = (uint32_t)kk;
        s_done = kk <= 0 ? 1u : 0u;
        s_or_lo = s_or_hi = 0;
    }
    __syncthreads();
    unsigned long long orv = 0;
    for (int k = tid; k < K; k += kSelThreads) {
        uint16_t v[16];  // all rows' loads first (independent), then the exact sum
#pragma unroll
        for (int b = 0; b < 16; b++) v[b] = b < B ? x[(size_t)b * ldx + k] : (uint16_t)0;
        unsigned long long score = 0;
        bool nonfinite = false;
#pragma unroll
        for (int b = 0; b < 16; b++) score += magnitude_units(v[b], &nonfinite);
        if (nonfinite) score = 1ull << 44;
        const unsigned long long key = (score << kKeyIndexBits) | (index_mask - (unsigned long long)k);
        s_key[k] = key;
        orv |= key;
    }
    const uint32_t lo = __reduce_or_sync(0xffffffffu, (uint32_t)orv);
    const uint32_t hi = __reduce_or_sync(0xffffffffu, (uint32_t)(orv >> 32));
    if (lane == 0) {
        atomicOr(&s_or_lo, lo);
        atomicOr(&s_or_hi, hi);
    }
    __syncthreads();
    const unsigned long long all_or = ((unsigned long long)s_or_hi << 32) | s_or_lo;
    int top = 63 - __clzll(all_or);  // highest bit any key has set (keys are nonzero)

    // Bits above `top` are zero in every key; `known` marks the bits already decided.
    unsigned long long known = top < 63 ? ~((2ull << top) - 1) : 0ull;
    while (!s_done && top >= 0) {
        const int width = top + 1 < kDigitBits ? top + 1 : kDigitBits;
        const int shift = top + 1 - width;
        const unsigned long long thresh = s_thresh;
        for (int d = tid; d < kBins; d += kSelThreads) s_hist[d] = 0;
        __syncthreads();
        for (int k = tid; k < K; k += kSelThreads) {
            const unsigned long long key = s_key[k];
            if ((key & known) == thresh) atomicAdd(&s_hist[(uint32_t)(key >> shift) & (kBins - 1)], 1u);
        }
        __syncthreads();
        // bins from the top down: thread t holds digits kBins-1-2t and kBins-2-2t
        const int d0 = kBins - 1 - 2 * tid, d1 = d0 - 1;
        const uint32_t c0 = s_hist[d0], c1 = s_hist[d1];
        uint32_t total;
        const uint32_t before = block_exclusive_scan(c0 + c1, s_warp, &total);
        const uint32_t rem = s_remaining;
        __syncthreads();  // every thread has read s_remaining
        if (before < rem && rem <= before + c0 + c1) {
            const bool first = rem <= before + c0;
            const int dg = first ? d0 : d1;
            const uint32_t above = first ? before : before + c0;
            const uint32_t inbin = first ? c0 : c1;
            s_thresh = thresh | ((unsigned long long)dg << shift);
            s_remaining = rem - above;
            if (rem - above == inbin) s_done = 1u;  // the whole bin is selected
        }
        known |= ((1ull << width) - 1) << shift;
        top = shift - 1;
        __syncthreads();
    }
    // Selected: the keys >= s_thresh (exactly kk of them; none when kk == 0).
    const unsigned long long thresh = s_thresh;
    const bool none = kk <= 0;
    const int n_words = (K + 31) / 32;
    uint32_t* s_wofs = (uint32_t*)(s_key + K);  // prefix of selected counts per word
    for (int w0 = 0; w0 < n_words; w0 += kSelThreads / 32) {
        const int w = w0 + (tid >> 5), k = 32 * w + lane;
        const bool sel = !none && w < n_words && k < K && s_key[k] >= thresh;
        const uint32_t word = __ballot_sync(0xffffffffu, sel);
        if (lane == 0 && w < n_words) {
            act_bits[w] = word;
            s_wofs[w] = __popc(word);
        }
    }
    __syncthreads();
    if (idx && !none) {
        // word offsets: a CTA-wide exclusive scan, words in blocks of kSelThreads
        uint32_t carry = 0;
        for (int w0 = 0; w0 < n_words; w0 += kSelThreads) {
            const int w = w0 + tid;
            const uint32_t c = w < n_words ? s_wofs[w] : 0u;
            uint32_t total;
            const uint32_t ex = block_exclusive_scan(c, s_warp, &total);
            if (w < n_words) s_wofs[w] = carry + ex;
            carry += total;
        }
        __syncthreads();
        for (int w0 = 0; w0 < n_words; w0 += kSelThreads / 32) {
            const int w = w0 + (tid >> 5), k = 32 * w + lane;
            const bool sel = w < n_words && k < K && s_key[k] >= thresh;
            const uint32_t word = __ballot_sync(0xffffffffu, sel);
            if (sel) idx[s_wofs[w] + __popc(word & lanemask_lt())] = (uint32_t)k;
        }
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
    // keys, then one word offset per 32 columns
    const size_t smem = (size_t)K * sizeof(unsigned long long) + 4 * (size_t)((K + 31) / 32);
    static bool attr_set[kMaxDevices];
    int dev = 0;
    SPW_CUDA_TRY(cudaGetDevice(&dev));
    if (dev >= 0 && dev < kMaxDevices && !attr_set[dev]) {
        SPW_CUDA_TRY(cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          kTopkMaxK * (int)sizeof(unsigned long long) + 4 * (kTopkMaxK / 32)));
        attr_set[dev] = true;
    }
    topk_kernel<<<1, kSelThreads, smem, (cudaStream_t)stream>>>(d_x, B, K, ldx, k, d_act_bits, d_idx);
    SPW_LAUNCH_CHECK();
    return SPW_OK;
}

}  // extern "C"
