// tokens.cu -- per-token index sets with token grouping for prefill.
//
// "Reduced Matrix Multiplication" §4.2 multiplies each token only over the channels it
// keeps; §6.1 notes that with a different channel set per token a plain GEMM no longer
// applies, and that tokens with the same or alike channel sets are grouped so that each
// group runs its own dense product; §6.2 adds that the groups must stay large enough to
// keep the matrix units busy.  This library's reading, at the granularity of its stored
// tiles (64 columns):
//   1. token_sig_kernel: the signature of token m has bit kt set iff the threshold rule
//      keeps some X[m,k] in k-tile kt (64 kt <= k < 64 kt + 64); up to 4 words.
//   2. token_rank_kernel: the position of each token in the order (signature, token
//      index) -- words compared from word 0 as unsigned integers -- by counting the
//      tokens before it; a grid of (token block, key block) pairs adds partial counts.
//   3. token_gather_kernel: token i moves to position r = rank[i]: perm[r] = i, row r of
//      the grouped input holds x~ (the rule applied) of token i, and the signature of
//      token i is ORed into that of its token tile r / T.
// The prefill product (spmm.cu) then runs every token tile over the k-tiles of its tile
// signature only -- a k-tile outside it holds no kept entry of any of the tile's tokens,
// so skipping it changes no sum -- and writes row r of its result to row perm[r] of Y.
#include "spw_internal.cuh"

namespace spw {
namespace {

constexpr int kSigThreads = 256;
constexpr int kRowChunks = 8;     // 16-byte chunks per thread: 256 x 8 x 8 halves = 16384 columns
constexpr int kRankTokens = 128;  // tokens per rank block (one per thread)
constexpr int kRankKeys = 64;     // keys per rank block, staged in shared memory

// True when the rule keeps either fp16 half of w.
__device__ inline bool keeps_pair(uint32_t w, float t) {
    return passes_threshold((uint16_t)(w & 0xffffu), t) || passes_threshold((uint16_t)(w >> 16), t);
}

// One CTA per token: a thread's 16-byte chunks (8 columns each) are all loaded before any
// is tested, so the row is in flight at once; a warp's 32 consecutive chunks = 4 k-tiles,
// whose flags come out of one ballot.  Block 0 also clears the tile signatures; every
// block clears its token's rank counter.
__global__ void __launch_bounds__(kSigThreads)
token_sig_kernel(const uint16_t* __restrict__ X, int ldx, int K, float t, int words,
                 uint64_t* __restrict__ sig, uint32_t* __restrict__ rank,
                 uint64_t* __restrict__ tile_sig, int tile_words) {
    __shared__ unsigned long long w[kMaxTokenWords];
    const int m = blockIdx.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (threadIdx.x < kMaxTokenWords) w[threadIdx.x] = 0ull;
    if (threadIdx.x == 0) rank[m] = 0u;
    if (m == 0)
        for (int i = threadIdx.x; i < tile_words; i += kSigThreads) tile_sig[i] = 0ull;
    __syncthreads();
    const uint16_t* row = X + (size_t)m * ldx;
    const int chunks = (K + 7) / 8;  // <= kSigThreads * kRowChunks
    uint4 v[kRowChunks];
#pragma unroll
    for (int u = 0; u < kRowChunks; u++) {
        const int c = 32 * warp + kSigThreads * u + lane;
        v[u] = (8 * c + 8 <= K) ? __ldg((const uint4*)(row + 8 * c)) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < kRowChunks; u++) {
        const int base = 32 * warp + kSigThreads * u;  // the warp's first chunk this round
        if (base >= chunks) break;                       // warp-uniform
        const int c = base + lane;
        bool any = false;
        if (8 * c + 8 <= K) {
            any = keeps_pair(v[u].x, t) || keeps_pair(v[u].y, t) || keeps_pair(v[u].z, t) || keeps_pair(v[u].w, t);
        } else {
            for (int k = 8 * c; k < K; k++) any = any || passes_threshold(__ldg(row + k), t);
        }
        const uint32_t b = __ballot_sync(0xffffffffu, any);
        if (lane < 4 && ((b >> (8 * lane)) & 0xffu) != 0u) {
            const int kt = base / 8 + lane;
            atomicOr(&w[kt >> 6], 1ull << (kt & 63));
        }
    }
    __syncthreads();
    if (threadIdx.x < words) sig[(size_t)m * words + threadIdx.x] = w[threadIdx.x];
}

// Block (bx, by): tokens bx*128 .. +127 (one per thread) against keys by*64 .. +63;
// each thread counts the keys ordered before its token and adds the count to its rank.
template <int WORDS>
__global__ void __launch_bounds__(kRankTokens)
token_rank_kernel(const uint64_t* __restrict__ sig, int M, uint32_t* __restrict__ rank) {
    __shared__ unsigned long long keys[kRankKeys * WORDS];
    const int i = blockIdx.x * kRankTokens + threadIdx.x;
    const int j0 = blockIdx.y * kRankKeys;
    const int nj = min(kRankKeys, M - j0);
    for (int e = threadIdx.x; e < nj * WORDS; e += kRankTokens) keys[e] = __ldg(sig + (size_t)j0 * WORDS + e);
    __syncthreads();
    if (i >= M) return;
    uint64_t a[WORDS];
#pragma unroll
    for (int w = 0; w < WORDS; w++) a[w] = __ldg(sig + (size_t)i * WORDS + w);
    uint32_t cnt = 0;
    for (int j = 0; j < nj; j++) {
        int ord = 0;  // -1: key j before token i's key, +1 after, 0 equal
#pragma unroll
        for (int w = 0; w < WORDS; w++) {
            const uint64_t kw = keys[j * WORDS + w];
            if (ord == 0 && kw != a[w]) ord = kw < a[w] ? -1 : 1;
        }
        cnt += (ord < 0 || (ord == 0 && j0 + j < i)) ? 1u : 0u;
    }
    if (cnt) atomicAdd(rank + i, cnt);
}

// One CTA per token i: moves it to position rank[i] (row of the grouped input, entry of
// perm) with the rule applied, and ORs its signature into its token tile's.  Columns K
// .. ldg-1 of the grouped row are written as zeros.
__global__ void __launch_bounds__(kSigThreads)
token_gather_kernel(const uint16_t* __restrict__ X, int ldx, int K, float t, int words,
                    const uint64_t* __restrict__ sig, const uint32_t* __restrict__ rank, int T,
                    uint16_t* __restrict__ Xg, int ldg, uint32_t* __restrict__ perm,
                    uint64_t* __restrict__ tile_sig) {
    const int i = blockIdx.x;
    const uint32_t r = __ldg(rank + i);
    if (threadIdx.x == 0) perm[r] = (uint32_t)i;
    if (threadIdx.x < words)
        atomicOr((unsigned long long*)tile_sig + (size_t)(r / (uint32_t)T) * words + threadIdx.x,
                 (unsigned long long)__ldg(sig + (size_t)i * words + threadIdx.x));
    const uint16_t* src = X + (size_t)i * ldx;
    uint16_t* dst = Xg + (size_t)r * ldg;
    // all of this thread's chunks loaded first (the row in flight at once), then stored
    uint4 q[kRowChunks];
#pragma unroll
    for (int u = 0; u < kRowChunks; u++) {
        const int k0 = 8 * (threadIdx.x + kSigThreads * u);
        q[u] = make_uint4(0u, 0u, 0u, 0u);
        if (k0 + 8 <= K) {
            q[u] = __ldg((const uint4*)(src + k0));
        } else if (k0 < K) {
            uint32_t w4[4] = {0u, 0u, 0u, 0u};
            for (int e = 0; e < 8 && k0 + e < K; e++)
                w4[e >> 1] |= (uint32_t)__ldg(src + k0 + e) << (16 * (e & 1));
            q[u] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
    }
#pragma unroll
    for (int u = 0; u < kRowChunks; u++) {
        const int k0 = 8 * (threadIdx.x + kSigThreads * u);
        if (k0 >= ldg) break;
        uint32_t v[4] = {q[u].x, q[u].y, q[u].z, q[u].w};
#pragma unroll
        for (int e = 0; e < 4; e++) {
            const uint16_t lo = (uint16_t)(v[e] & 0xffffu), hi = (uint16_t)(v[e] >> 16);
            v[e] = (passes_threshold(lo, t) ? lo : 0u) | ((passes_threshold(hi, t) ? (uint32_t)hi : 0u) << 16);
        }
        *(uint4*)(dst + k0) = make_uint4(v[0], v[1], v[2], v[3]);
    }
}

}  // namespace

uint64_t token_groups_scratch_bytes(int M, int K) {
    const int words = token_sig_words(K);
    return round_up_u64(8ull * (uint64_t)M * words, 256) + round_up_u64(4ull * (uint64_t)M, 256);
}

int group_tokens_launch(const uint16_t* X, int M, int K, int ldx, float t, int T, uint16_t* Xg,
                        int ldg, uint32_t* perm, uint64_t* tile_sig, void* scratch,
                        cudaStream_t stream) {
    const int words = token_sig_words(K);
    uint64_t* sig = (uint64_t*)scratch;
    uint32_t* rank = (uint32_t*)((uint8_t*)scratch + round_up_u64(8ull * (uint64_t)M * words, 256));
    const int tiles = (M + T - 1) / T;
    token_sig_kernel<<<M, kSigThreads, 0, stream>>>(X, ldx, K, t, words, sig, rank, tile_sig,
                                                    tiles * words);
    SPW_LAUNCH_CHECK();
    const dim3 grid((unsigned)((M + kRankTokens - 1) / kRankTokens), (unsigned)((M + kRankKeys - 1) / kRankKeys));
    switch (words) {
        case 1: token_rank_kernel<1><<<grid, kRankTokens, 0, stream>>>(sig, M, rank); break;
        case 2: token_rank_kernel<2><<<grid, kRankTokens, 0, stream>>>(sig, M, rank); break;
        case 3: token_rank_kernel<3><<<grid, kRankTokens, 0, stream>>>(sig, M, rank); break;
        default: token_rank_kernel<4><<<grid, kRankTokens, 0, stream>>>(sig, M, rank); break;
    }
    SPW_LAUNCH_CHECK();
    token_gather_kernel<<<M, kSigThreads, 0, stream>>>(X, ldx, K, t, words, sig, rank, T, Xg, ldg,
                                                       perm, tile_sig);
    SPW_LAUNCH_CHECK();
    return SPW_OK;
}

}  // namespace spw

using namespace spw;

extern "C" {

uint64_t spw_group_tokens_workspace_bytes(int M, int K) {
    if (M < 1 || M > kMaxGroupTokens || K < 1 || K > kMaxTokenK) return 0;
    return token_groups_scratch_bytes(M, K);
}

int spw_group_tokens(const uint16_t* d_X, int M, int K, int ldx, float t, int token_tile,
                     uint16_t* d_Xg, int ldxg, uint32_t* d_perm, uint64_t* d_tile_sig, void* d_ws,
                     uint64_t ws_bytes, void* stream) {
    if (M < 1 || K < 1 || token_tile < 1 || !d_X || !d_Xg || !d_perm || !d_tile_sig || !d_ws)
        return SPW_ERR_INVALID_ARG;
    if (M > kMaxGroupTokens || K > kMaxTokenK) return SPW_ERR_UNSUPPORTED;
    if (!(t >= 0.0f) || isinf(t)) return SPW_ERR_INVALID_ARG;
    if (!ld_ok(ldx, K, M) || ldxg < K || ldxg % 8 != 0) return SPW_ERR_INVALID_ARG;
    if (!aligned16(d_X) || !aligned16(d_Xg) || !aligned16(d_perm) || !aligned16(d_tile_sig) ||
        !aligned16(d_ws))
        return SPW_ERR_ALIGNMENT;
    if (ws_bytes < token_groups_scratch_bytes(M, K)) return SPW_ERR_BUFFER_TOO_SMALL;
    return group_tokens_launch(d_X, M, K, ldx, t, token_tile, d_Xg, ldxg, d_perm, d_tile_sig, d_ws,
                               (cudaStream_t)stream);
}

}  // extern "C"
