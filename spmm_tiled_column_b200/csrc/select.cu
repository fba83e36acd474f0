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
// Used for B > 1 (about 40 us at K = 11008 on B200, graph-timed; per-warp-pair 256-bin
// histograms and warp-aggregated histogram updates were both slower); one row takes
// topk1_kernel below.
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

// Writes act_bits and, when idx is not NULL, the ascending index list from the selected
// words s_selw[n_words] (s_wofs: n_words words of scratch).  Whole CTA.
__device__ inline void emit_selection(const uint32_t* s_selw, uint32_t* s_wofs, uint32_t* s_warp,
                                      int K, uint32_t* act_bits, uint32_t* idx) {
    const int tid = threadIdx.x, lane = tid & 31;
    const int n_words = (K + 31) / 32;
    uint32_t carry = 0;
    for (int w0 = 0; w0 < n_words; w0 += kSelThreads) {
        const int w = w0 + tid;
        const uint32_t word = w < n_words ? s_selw[w] : 0u;
        if (w < n_words) act_bits[w] = word;
        uint32_t total;
        const uint32_t ex = block_exclusive_scan((uint32_t)__popc(word), s_warp, &total);
        if (w < n_words) s_wofs[w] = carry + ex;
        carry += total;
    }
    if (!idx) return;
    __syncthreads();
    for (int w0 = 0; w0 < n_words; w0 += kSelThreads / 32) {
        const int w = w0 + (tid >> 5);
        if (w >= n_words) continue;
        const uint32_t word = s_selw[w];
        if ((word >> lane) & 1u) idx[s_wofs[w] + __popc(word & lanemask_lt())] = (uint32_t)(32 * w + lane);
    }
}

// In warp 0: bins hist[nb-1] .. hist[0] from the top, nb / 32 per lane; finds the bin
// holding the kk-th largest element (1 <= kk <= the histogram's total) and how many
// elements lie in higher bins, returned to every lane.
__device__ inline void find_bin_from_top(const uint32_t* hist, int nb, uint32_t kk, int lane,
                                         uint32_t* bin, uint32_t* above) {
    const int per = nb / 32;
    uint32_t sum = 0;
    for (int j = 0; j < per; j++) sum += hist[nb - 1 - per * lane - j];
    const uint32_t incl = (uint32_t)warp_inclusive_scan((int)sum, lane);
    const uint32_t excl = incl - sum;
    uint32_t b = 0, a = 0;
    bool found = false;
    if (excl < kk && kk <= incl) {
        uint32_t run = excl;
        for (int j = 0; j < per; j++) {
            const uint32_t c = hist[nb - 1 - per * lane - j];
            if (run + c >= kk) {
                b = (uint32_t)(nb - 1 - per * lane - j);
                a = run;
                found = true;
                break;
            }
            run += c;
        }
    }
    const uint32_t m = __ballot_sync(0xffffffffu, found);
    const int src = m ? __ffs(m) - 1 : 0;
    *bin = __shfl_sync(0xffffffffu, b, src);
    *above = __shfl_sync(0xffffffffu, a, src);
}

// Top-k of one row (B = 1).  The score is |x| itself, so the fp16 magnitude bits (15
// bits; Inf and NaN clamped to 0x7C00, tying above every finite value) order the columns
// exactly.  Two histogram passes -- the top 7 bits, then the low 8 bits within the chosen
// top bin -- give the threshold magnitude T and how many columns of magnitude T to keep;
// those are the lowest-index ones (ties to the lower index), found with one CTA-wide scan
// over the columns in index order (thread t owns a contiguous run of columns).
constexpr int kT1Hi = 128, kT1Lo = 256;

__global__ void __launch_bounds__(kSelThreads)
topk1_kernel(const uint16_t* __restrict__ x, int K, int kk, uint32_t* __restrict__ act_bits,
             uint32_t* __restrict__ idx) {
    extern __shared__ uint32_t s_dyn[];  // K magnitudes (u16), selected words, word offsets
    const int n_words = (K + 31) / 32;
    uint16_t* s_mag = (uint16_t*)s_dyn;
    uint32_t* s_selw = s_dyn + (K + 1) / 2;
    uint32_t* s_wofs = s_selw + n_words;
    __shared__ uint32_t s_hist[kT1Lo];
    __shared__ uint32_t s_warp[kSelThreads / 32 + 1];
    __shared__ uint32_t s_bin, s_rem;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int k = tid; k < K; k += kSelThreads) {
        const uint32_t m = (uint32_t)__ldg(x + k) & 0x7fffu;
        s_mag[k] = (uint16_t)(m > 0x7c00u ? 0x7c00u : m);
    }
    for (int w = tid; w < n_words; w += kSelThreads) s_selw[w] = 0u;
    if (tid < kT1Lo) s_hist[tid] = 0u;
    __syncthreads();
    if (kk > 0) {
        for (int k = tid; k < K; k += kSelThreads) atomicAdd(&s_hist[s_mag[k] >> 8], 1u);
        __syncthreads();
        if (warp == 0) {
            uint32_t b, a;
            find_bin_from_top(s_hist, kT1Hi, (uint32_t)kk, lane, &b, &a);
            if (lane == 0) {
                s_bin = b;
                s_rem = (uint32_t)kk - a;
            }
        }
        __syncthreads();
        const uint32_t hb = s_bin, rem = s_rem;
        __syncthreads();  // every thread has read s_bin and s_rem
        if (tid < kT1Lo) s_hist[tid] = 0u;
        __syncthreads();
        for (int k = tid; k < K; k += kSelThreads) {
            const uint32_t m = s_mag[k];
            if ((m >> 8) == hb) atomicAdd(&s_hist[m & 0xffu], 1u);
        }
        __syncthreads();
        if (warp == 0) {
            uint32_t b, a;
            find_bin_from_top(s_hist, kT1Lo, rem, lane, &b, &a);
            if (lane == 0) {
                s_bin = (hb << 8) | b;
                s_rem = rem - a;  // columns of magnitude T to keep, the lowest indices first
            }
        }
        __syncthreads();
        const uint32_t T = s_bin, take = s_rem;
        const int c = (K + kSelThreads - 1) / kSelThreads;
        const int k0 = tid * c, k1 = min(k0 + c, K);
        uint32_t ties = 0;
        for (int k = k0; k < k1; k++) ties += s_mag[k] == T ? 1u : 0u;
        uint32_t total;
        uint32_t rank = block_exclusive_scan(ties, s_warp, &total);
        for (int k = k0; k < k1; k++) {
            const uint32_t m = s_mag[k];
            bool sel = m > T;
            if (m == T) sel = rank++ < take;
            if (sel) atomicOr(&s_selw[k >> 5], 1u << (k & 31));
        }
    }
    __syncthreads();
    emit_selection(s_selw, s_wofs, s_warp, K, act_bits, kk > 0 ? idx : nullptr);
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
    if (B == 1) {
        // magnitudes (u16, rounded up to whole words), selected words, word offsets
        const size_t smem1 = 4 * (size_t)((K + 1) / 2) + 8 * (size_t)((K + 31) / 32);
        static bool attr1_set[kMaxDevices];
        int dev1 = 0;
        SPW_CUDA_TRY(cudaGetDevice(&dev1));
        if (dev1 >= 0 && dev1 < kMaxDevices && !attr1_set[dev1]) {
            SPW_CUDA_TRY(cudaFuncSetAttribute(topk1_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                              4 * ((kTopkMaxK + 1) / 2) + 8 * (kTopkMaxK / 32)));
            attr1_set[dev1] = true;
        }
        topk1_kernel<<<1, kSelThreads, smem1, (cudaStream_t)stream>>>(d_x, K, k, d_act_bits, d_idx);
        SPW_LAUNCH_CHECK();
        return SPW_OK;
    }
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
