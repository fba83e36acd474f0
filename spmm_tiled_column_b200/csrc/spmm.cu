// spmm.cu -- products on tcgen05 tensor cores with the compressed weight as the A operand:
//   prefill  Y = X . W_masked^T            (spw_spmm, M tokens)
//   decode   y_b = W_masked . x~_b         (spw_spmv_tc, B <= 16 rows, threshold rule)
//   prefill with per-token index sets      (spw_spmm_tokens: token-list mode)
//   prefill on the 2:4 + residual split    (spw_spmm24: 2:4 mode)
//
// Method: "Unified Static-Dynamic Pruning for Efficient LLM Inference" (abstract) pairs
// its bitmap format with a Tensor-Core SpMM for prefill.  Dense tensor cores take only
// 2:4 structured sparsity ("Accelerating LLM GPU inference with moderately unstructured
// sparse weight matrices", §1, challenge 1), so unstructured tiles are decoded to dense
// in shared memory and fed to dense MMA; the weight crosses HBM compressed.
//
// This library's design for B200 (one output tile, or one K part of one, per CTA):
//   * Output tile = 128 weight rows (two 64-row TCB strips; the MMA's M) by MT tokens or
//     batch rows (the MMA's N: MT <= 256 in one MMA, 512 as two), K stepped by 64 (one
//     TCB k-tile).  The fp32 accumulator, 128 lanes x MT columns, lives in TMEM.  Each
//     decoded 64-column weight tile feeds up to 512 tokens.  For narrow tiles (decode
//     batches, MT <= 32) the 16-wide k-slices rotate over 4 accumulators, so the MMAs
//     form 4 independent chains instead of one; the epilogue adds them.
//   * When output tiles are fewer than the SMs can hold, K is split across CTAs: each
//     stores its fp32 partial tile; the last CTA of a tile (counted with an atomic) sums
//     the partials in K order -- deterministic -- and writes fp16.  When the tiles need
//     more than one wave but fewer than two, only the last tiles are split, and their
//     parts fill the SMs as the whole tiles finish.  Each CTA walks its k-steps from a
//     start rotated by its weight-row tile, so CTAs sharing an X tile read different
//     parts of it at any moment.
//   * warp 0, lane 0 (X producer): TMA-loads the X tiles (MT rows x 64, fp16, 128-byte
//     swizzle, no multicast).  The last warp, lane 0 (TCB producer): 1-D bulk-copies the
//     two TCB tiles (bitmaps + packed values) of each k-step.  Two warps, not two lanes
//     of one: divergent lanes of a warp run one path at a time, so one ring's wait
//     (a suspended mbarrier try_wait) would hold up the other ring's issue.
//   * warp 1 (MMA): allocates TMEM; one thread issues tcgen05.mma.kind::f16 (A = decoded
//     W, B = X, both K-major 128B-swizzled shared memory) and commits stage releases.
//   * Decode (spw_spmv_tc) with a threshold above zero or a column set first writes x~ to
//     the workspace with a small kernel (rule_kernel); with threshold 0 and no column set
//     x~ differs from x only in dropping exact zeros, which contribute nothing, and X is
//     read as given.
//   * warps 2..17 (decoders, then epilogue): warp d decodes strip d/8, columns
//     8 (d%8) .. 8 (d%8) + 7, one 16-byte chunk of each of its rows; it needs only those
//     8 columns' value starts (one reduction over the columns before them plus a 4-lane
//     scan).  Lane l owns rows 2l and 2l+1 at bits q, q+1 (q = 2l mod 32) of one half of
//     each column's bitmap word; the kept rows from 2l+1 upward are the
//     last c = popc(bits >> (q+1)) values of that half, so row 2l+1's value is at end - 2c
//     and row 2l's just before it.  Dense rows are written as 16-byte chunks in the
//     swizzled layout the MMA reads.  After the K loop the same warps read the fp32
//     accumulators (tcgen05.ld) and write Y (or the split-K partials).
//   * Every mbarrier wait is bounded and also polls a CTA-wide abort flag; on a timeout
//     the kernel raises SPW_ERR_TIMEOUT, drains outstanding copies and MMAs (bounded),
//     frees TMEM and returns.
//   * Token-list mode ("Reduced Matrix Multiplication" §6.1): X holds the grouped rows
//     (tokens.cu); warp 2 turns the token tile's k-tile signature into an ascending list
//     in shared memory, every role walks that list instead of 0 .. n_ktiles-1, a tile
//     with an empty list writes zeros, and the epilogue writes row r to row perm[r].
//   * 2:4 mode ("Accelerating LLM GPU inference ..." §1, layers (i) and (iii)): each X
//     stage also carries the k-step's 2:4 values (64-byte swizzle) and metadata
//     (split24.cu layout); the MMA thread moves the metadata into tensor memory with
//     tcgen05.cp and issues two tcgen05.mma.sp (K = 32), then the dense MMAs of the
//     decoded residual tile only when the k-tile holds residual weights (the W ring
//     advances on those k-steps only); token tiles <= 256 (accumulators + metadata).
//   * SM-pair mode (opt-in, SPW_SPMM_PAIR=1): see the kernel's comment.
// A decoded tile holds explicit zeros where the mask drops a weight, so a non-finite
// activation reaches every row through the MMA (0 * Inf = NaN, as in a dense product);
// the CUDA-core decode (spmv.cu) skips dropped weights instead.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <stdlib.h>
#include <string.h>

#include <mutex>

#include "spw_internal.cuh"

namespace spw {
namespace {

constexpr int kTileRows = 128;          // weight rows per CTA tile (the MMA's M, or half of it)
constexpr int kPeerSlots = 8;           // pair mode: the peer's stage-ready ring (on the leader)
constexpr uint32_t kRecBytesPerWarp = 160;  // a decoder warp's column records (see the decoders)
constexpr int kTileStrips = kTileRows / kStripRows;
constexpr int kBK = 64;                 // one TCB k-tile
constexpr int kMaxTokens = 512;         // tokens per CTA tile (TMEM columns)
constexpr int kDecoderWarps = 16;
constexpr int kTcbWarp = 2 + kDecoderWarps;             // the TCB producer's warp (the last)
constexpr int kThreads = 32 * (3 + kDecoderWarps);      // X producer, MMA, decoders, TCB producer
constexpr uint32_t kWStageBytes = kTileRows * kBK * 2;  // 16 KB
constexpr int kSmemLimit = 227 * 1024;
// 2:4 mode (spw_spmm24): per k-step S area = the 2:4 values of both strips (2 x 4 KB, the
// 64-byte-swizzled K-major layout of split24.cu) and their metadata (2 x 1 KB: 128 lanes
// x 16 bytes, the source matrix of one tcgen05.cp), held in the X stage right after the
// token tile.
constexpr uint32_t kS24ValBytes = 4096;
constexpr uint32_t kS24MetaBytes = 1024;
constexpr uint32_t kSStageBytes = kTileStrips * (kS24ValBytes + kS24MetaBytes);  // 9 KB
constexpr int kMaxTokens24 = 256;  // accumulators <= 256 columns: the metadata slots fit

struct SpmmParams {
    const uint64_t* bitmaps;
    const uint32_t* tileptr;
    const uint16_t* values;
    uint64_t values_units;      // the values section, in 16-byte units
    uint16_t* Y;
    uint32_t* counters;         // split-K arrivals per output tile (ksplit > 1)
    float* partials;            // split-K fp32 partial tiles
    int* status;
    int M, N, K, ldy;
    int n_strips, n_ktiles;
    int MT, nh;                 // tokens per tile; MMAs per k-slice (MT / nh each)
    int n_acc;                  // independent accumulators (32 columns apart) for MT <= 32
    int ksplit;                 // K parts of each split tile (1: no split tiles)
    int n_whole;                // tiles 0 .. n_whole-1 run whole; the rest are split
    int m_tiles;                // token tiles (tile t: token tile t % m_tiles, weight rows t / m_tiles)
    int sx, sr, sw;             // X, raw-tile and decoded-weight stage counts
    uint32_t x_stage_bytes;     // MT * 128 (2:4 mode: + the S area)
    uint32_t raw_stage_bytes;   // 1024 + 2 * val_slot
    uint32_t val_slot;          // bytes per strip's values slot (incl. 16 bytes of slack)
    uint32_t tmem_cols;
    uint32_t off_w, off_raw, off_rec, off_tptr, off_bar;  // dynamic smem offsets
    long long wait_limit;       // pipeline waits, in SM cycles (drains use the fixed limit)
    // Token grouping (spw_spmm_tokens): X rows are in grouped order; token tile mt visits
    // only the k-tiles set in tile_sig[mt * sig_words ..] and its row r is row perm[r] of
    // Y.  Null tile_sig: every k-tile, rows in place.
    const uint64_t* tile_sig;
    const uint32_t* perm;
    int sig_words;
    uint32_t off_klist;         // dynamic smem: the visited k-tile count, then the list
    // 2:4 + residual (spw_spmm24): the structured part (split24.cu layout); the TCB
    // sections above then describe the residual.  Each X stage holds the k-step's S area
    // at byte off_s; the MMA thread copies its metadata into tensor-memory columns
    // e_col + 4 s .. e_col + 4 s + 3 (two used) before the stage's sparse MMAs.
    const uint8_t* s24_vals;
    const uint8_t* s24_meta;
    uint32_t off_s, e_col;
};

// ------------------------------------------------------------------ tcgen05 helpers
__device__ inline uint64_t umma_desc_sw128(uint32_t saddr) {
    // K-major, 128-byte swizzle: 8-row atoms of 1024 bytes (stride byte offset 1024),
    // leading byte offset 16 (unused for swizzled K-major), version 1, layout type 2.
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFF);
    d |= (uint64_t)(16 >> 4) << 16;
    d |= (uint64_t)(1024 >> 4) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

// kind::f16 instruction descriptor: fp32 accumulator, fp16 A and B, both K-major.
// K-major, 64-byte swizzle: 8-row atoms of 512 bytes (the 2:4 values, 64 bytes per row).
__device__ inline uint64_t umma_desc_sw64(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFF);
    d |= (uint64_t)(16 >> 4) << 16;
    d |= (uint64_t)(512 >> 4) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)4 << 61;
    return d;
}

// Sparse MMA (2:4 A): A holds two of every four K positions (16 halves per row for K =
// 32), the metadata selecting them sits in tensor memory at e_tmem (an even column;
// idesc bits 0-1 pick the column pair's half), idesc bit 2 marks the MMA sparse.
__device__ inline void umma_f16_sp(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                   uint32_t e_tmem, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.sp.cta_group::1.kind::f16 [%0], %1, %2, [%5], %3, {%6, %6, %6, %6}, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(e_tmem), "r"(0u)
        : "memory");
}

// Shared -> tensor memory copy of a 128-row x 16-byte matrix (row r to lane r, four
// 32-bit columns), issued by the MMA thread: it runs in order with that thread's later
// tcgen05.mma, so the MMAs that read the columns need no other synchronisation.  The
// source is one K-major, unswizzled matrix: 8-row core matrices of 128 contiguous bytes.
__device__ inline void tmem_cp_128x128b(uint32_t taddr, uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFF);
    d |= (uint64_t)(128 >> 4) << 16;  // between core matrices along K (one here)
    d |= (uint64_t)(128 >> 4) << 32;  // between 8-row core matrices
    d |= (uint64_t)1 << 46;           // descriptor version; layout type 0: no swizzle
    asm volatile("tcgen05.cp.cta_group::1.128x128b [%0], %1;" ::"r"(taddr), "l"(d) : "memory");
}

__host__ __device__ constexpr uint32_t idesc_f16(int M, int N) {
    return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ inline void umma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ inline void umma_commit(uint32_t bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
        : "memory");
}

__device__ inline void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ inline void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

// ---- SM-pair (cta_group::2) helpers: a cluster of two CTAs computes one 256-row tile;
// CTA rank 0 issues the MMAs for both.
__device__ inline uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ inline uint32_t map_to_rank(uint32_t saddr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}

// Every thread of both CTAs (no thread may leave early): orders everything before it in
// either CTA before everything after it in both.
__device__ inline void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ inline void mbar_arrive_cluster(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// Waits with cluster-scope acquire (for arrivals made by the other CTA of the pair).
__device__ inline bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
    return done != 0;
}
__device__ inline bool mbar_test_wait_cluster(uint32_t bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
    return done != 0;
}

__device__ inline void umma_f16_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                     uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive on the barrier at this shared-memory address (this CTA's, or the other CTA's
// through its cluster address) once the MMAs issued so far have completed.
__device__ inline void umma_commit_pair_local(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}
// The same barrier in both CTAs of the pair (issued by rank 0): two commits, one to each
// CTA's copy of the barrier, both completing with the same MMAs.
__device__ inline void umma_commit_pair_both(uint32_t bar) {
    umma_commit_pair_local(bar);
    umma_commit_pair_local(map_to_rank(bar, 1u));
}

__device__ inline void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr)
        : "memory");
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ inline void tma_load_2d(uint32_t dst, const CUtensorMap* map, int c0, int c1,
                                   uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"((uint64_t)map), "r"(c0), "r"(c1), "r"(bar)
        : "memory");
}

// Bounded wait that also gives up when another warp has flagged an abort.
// A limit shorter than the default polls with the non-blocking test (see mbar_wait).
__device__ inline bool wait_or_abort(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                     long long limit) {
    const bool blocking = limit >= kWaitLimitCycles;
    if (blocking && mbar_try_wait(bar, parity)) return true;
    const long long start = clock64();
    while (!(blocking ? mbar_try_wait(bar, parity) : mbar_test_wait(bar, parity))) {
        if (*abort_flag) return false;
        if (clock64() - start > limit) return false;
    }
    return true;
}

// The same for a barrier the other CTA of a pair arrives on (cluster-scope acquire).
__device__ inline bool wait_or_abort_cluster(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                             long long limit) {
    const bool blocking = limit >= kWaitLimitCycles;
    if (blocking && mbar_try_wait_cluster(bar, parity)) return true;
    const long long start = clock64();
    while (!(blocking ? mbar_try_wait_cluster(bar, parity) : mbar_test_wait_cluster(bar, parity))) {
        if (*abort_flag) return false;
        if (clock64() - start > limit) return false;
    }
    return true;
}

__device__ inline void flag_abort(volatile int* abort_flag, int* status) {
    *abort_flag = 1;
    raise_status(status, SPW_ERR_TIMEOUT);
}



// Decode's x~ for the tensor-core path: the threshold rule and the caller's column set
// applied once per call, into the workspace (B rows of ld halves), 8 halves per thread.
__global__ void __launch_bounds__(256) rule_kernel(const uint16_t* __restrict__ x, int ldx, int B, int K,
                                                   float t, const uint32_t* __restrict__ act_bits,
                                                   uint16_t* __restrict__ xt, int ld) {
    const int per_row = (K + 7) / 8;
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= B * per_row) return;
    const int b = i / per_row, k0 = 8 * (i % per_row);
    uint16_t out[8];
#pragma unroll
    for (int e = 0; e < 8; e++) {
        const int k = k0 + e;
        uint16_t v = 0;
        if (k < K) {
            v = x[(size_t)b * ldx + k];
            bool keep = passes_threshold(v, t);
            if (act_bits && keep) keep = (act_bits[k >> 5] >> (k & 31)) & 1u;
            if (!keep) v = 0;
        }
        out[e] = v;
    }
    uint4 w;
    w.x = (uint32_t)out[0] | ((uint32_t)out[1] << 16);
    w.y = (uint32_t)out[2] | ((uint32_t)out[3] << 16);
    w.z = (uint32_t)out[4] | ((uint32_t)out[5] << 16);
    w.w = (uint32_t)out[6] | ((uint32_t)out[7] << 16);
    *(uint4*)(xt + (size_t)b * ld + k0) = w;
}

// PAIR: a cluster of two CTAs on an SM pair computes one 256-weight-row tile.  Each CTA
// decodes its own 128 rows (the MMA's A, split by rows) and TMA-loads its own half of the
// token tile (the MMA's B, split by tokens); CTA rank 0 issues tcgen05.mma.cta_group::2
// for both, whose accumulator halves land in each CTA's own tensor memory.  The other
// CTA's MMA warp relays "my X and W stages are ready" to rank 0 with a cluster-scope
// arrive; rank 0's commits release the stages in both CTAs.  Per output element the X
// tile crosses L2 half as often as with one CTA per 128-row tile.
template <bool PAIR, bool SP24 = false>
__global__ void __launch_bounds__(kThreads, 1)
spmm_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ SpmmParams p) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    // 1024-byte alignment for the swizzled operand tiles
    unsigned char* smem = (unsigned char*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // This CTA's output tile and K range: CTA c < n_whole computes tile c whole; the others
    // compute part (c - n_whole) % ksplit of split tile n_whole + (c - n_whole) / ksplit.
    const uint32_t rank = PAIR ? cluster_rank() : 0u;  // 0: issues the pair's MMAs
    const int cta = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;  // the (pair's) tile slot
    const bool split = cta >= p.n_whole;
    const int tile = split ? p.n_whole + (cta - p.n_whole) / p.ksplit : cta;
    const int parts = split ? p.ksplit : 1;
    const int kz = split ? (cta - p.n_whole) % p.ksplit : 0;
    // index of this CTA's 128-row output half among the split ones (when split)
    const int stile = PAIR ? 2 * (tile - p.n_whole) + (int)rank : tile - p.n_whole;
    const int mt = tile % p.m_tiles, ntile = tile / p.m_tiles;
    const int m0 = mt * p.MT;
    const int n0 = ntile * (PAIR ? 2 * kTileRows : kTileRows) + kTileRows * (int)rank;
    const int s0 = n0 / kStripRows;
    const int nk = p.n_ktiles;
    const int SX = p.sx, SR = p.sr;

    uint64_t* bars = (uint64_t*)(smem + p.off_bar);
    uint64_t* x_full = bars;
    uint64_t* x_empty = x_full + SX;
    uint64_t* r_full = x_empty + SX;
    uint64_t* r_empty = r_full + SR;
    const int SW = p.sw;
    uint64_t* w_full = r_empty + SR;
    uint64_t* w_empty = w_full + SW;
    uint64_t* acc_full = w_empty + SW;
    uint64_t* drain = acc_full + 1;
    uint64_t* peer_ready = drain + 1;  // PAIR, on rank 0: the other CTA's stages are ready
    uint32_t* tmem_slot = (uint32_t*)(peer_ready + kPeerSlots);
    volatile int* abort_flag = (volatile int*)(tmem_slot + 1);
    volatile uint32_t* last_flag = (volatile uint32_t*)(tmem_slot + 2);
    uint32_t* tptr = (uint32_t*)(smem + p.off_tptr);
    volatile int* klist_n = (volatile int*)(smem + p.off_klist);
    uint16_t* klist = (uint16_t*)(smem + p.off_klist + 16);

    if (threadIdx.x == 0) {
        for (int i = 0; i < SX; i++) {
            mbar_init(smem_u32(&x_full[i]), 1);
            mbar_init(smem_u32(&x_empty[i]), 1);
        }
        for (int i = 0; i < SR; i++) {
            mbar_init(smem_u32(&r_full[i]), 1);
            mbar_init(smem_u32(&r_empty[i]), kDecoderWarps);
        }
        for (int i = 0; i < SW; i++) {
            mbar_init(smem_u32(&w_full[i]), kDecoderWarps);
            mbar_init(smem_u32(&w_empty[i]), 1);
        }
        mbar_init(smem_u32(acc_full), 1);
        mbar_init(smem_u32(drain), 1);
        for (int i = 0; i < kPeerSlots; i++) mbar_init(smem_u32(&peer_ready[i]), 1);
        *abort_flag = 0;
        *last_flag = 0;
        fence_mbar_init();
    }
    // tile pointers of the CTA's strips, for every k-tile (row j = strip s0 + j)
    for (int i = threadIdx.x; i < kTileStrips * (nk + 1); i += kThreads) {
        const int j = i / (nk + 1), kt = i % (nk + 1);
        const int s = s0 + j;
        tptr[i] = (s < p.n_strips) ? __ldg(p.tileptr + (size_t)s * nk + kt) : 0u;
    }
    if (p.tile_sig && warp == 2) {
        // Token grouping: the k-tiles of this token tile's signature, ascending.
        const uint64_t* ts = p.tile_sig + (size_t)mt * p.sig_words;
        int count = 0;
        for (int base = 0; base < nk; base += 32) {
            const int kt = base + lane;
            const bool on = kt < nk && ((__ldg(ts + (kt >> 6)) >> (kt & 63)) & 1ull);
            const uint32_t b = __ballot_sync(0xffffffffu, on);
            if (on) klist[count + __popc(b & lanemask_lt())] = (uint16_t)kt;
            count += __popc(b);
        }
        if (lane == 0) *klist_n = count;
    }
    if (warp == 1) {  // TMEM allocation (whole warp; in pair mode warp 1 of both CTAs)
        if constexpr (PAIR) {
            asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                             smem_u32(tmem_slot)),
                         "r"(p.tmem_cols)
                         : "memory");
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
        } else {
            asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                             smem_u32(tmem_slot)),
                         "r"(p.tmem_cols)
                         : "memory");
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
        }
    }
    tc_fence_before();
    __syncthreads();
    if constexpr (PAIR) cluster_sync_all();  // both CTAs' barriers exist before any remote arrive
    tc_fence_after();
    // Pair mode: an abort in either CTA stops both (the flag is also set in the other CTA).
    const uint32_t peer_abort = PAIR ? map_to_rank(smem_u32((const void*)abort_flag), rank ^ 1u) : 0u;
    auto abort_both = [&]() {
        flag_abort(abort_flag, p.status);
        if constexpr (PAIR) asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(peer_abort), "r"(1) : "memory");
    };
    const uint32_t tmem = *tmem_slot;
    // The k-tiles this CTA visits: its part of 0 .. nk-1, or of the token tile's list.
    // Every role walks them from a start rotated by the weight-row tile: the CTAs that
    // share an X tile then read different k-columns of it at any moment instead of all
    // hitting the same L2 lines together.
    const int n_list = p.tile_sig ? *klist_n : nk;
    const int k_begin = (int)((long long)kz * n_list / parts);
    const int k_end = (int)((long long)(kz + 1) * n_list / parts);
    const int n_kc = k_end - k_begin;
    const int k_rot = n_kc > 0 ? ntile % n_kc : 0;
    auto kstep = [&](int i) {
        const int j = k_begin + (i + k_rot < n_kc ? i + k_rot : i + k_rot - n_kc);
        return p.tile_sig ? (int)klist[j] : j;
    };
    // 2:4 mode: k-tile kt holds no residual weight in either strip (no decode, no dense MMA)
    auto residual_empty = [&](int kt) {
        bool e = true;
#pragma unroll
        for (int q = 0; q < kTileStrips; q++)
            if (s0 + q < p.n_strips && tptr[q * (nk + 1) + kt + 1] != tptr[q * (nk + 1) + kt]) e = false;
        return e;
    };

    int x_issued = 0, r_issued = 0;  // lane 0 of warp 0 (X) and of the TCB warp: stages armed
    if (warp == 0 || warp == kTcbWarp) {
        // ------------------------------------------------------------ producer
        if (warp == 0 && lane == 0) {  // X ring
            asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&tmap_x) : "memory");
            // Per MMA h the token rows m0 + h rows .. +rows; in pair mode this CTA loads
            // its half of them (the MMA's B is split by tokens across the pair).
            const int rows = p.MT / p.nh;
            const int crows = PAIR ? rows / 2 : rows;  // TMA box height
            int xs = 0;
            uint32_t xph = 0;
            for (int i = 0; i < n_kc; i++) {
                const int kt = kstep(i);
                // X tile: rows m0..m0+MT-1, columns 64 kt.. (zero fill outside X)
                if (i >= SX && !wait_or_abort(smem_u32(&x_empty[xs]), xph ^ 1u, abort_flag, p.wait_limit)) {
                    abort_both();
                    break;
                }
                const uint32_t xbar = smem_u32(&x_full[xs]);
                const uint32_t xst = sbase + (uint32_t)xs * p.x_stage_bytes;
                uint32_t xbytes = p.x_stage_bytes;
                if constexpr (SP24) {  // the token tile, then the 2:4 values and metadata
                    xbytes = p.off_s;
                    for (int j = 0; j < kTileStrips; j++)
                        xbytes += (s0 + j < p.n_strips ? kS24ValBytes : 0u) + kS24MetaBytes;
                }
                mbar_arrive_expect_tx(xbar, xbytes);
                for (int h = 0; h < p.nh; h++)
                    tma_load_2d(xst + (uint32_t)(h * crows * 128), &tmap_x, kt * kBK,
                                m0 + h * rows + (int)rank * crows, xbar);
                if constexpr (SP24) {
                    // a missing second strip (odd strip count) takes the padding metadata
                    // block (valid groups, no kept weight); its values are never stored
                    const size_t pad = (size_t)p.n_strips * nk;
                    for (int j = 0; j < kTileStrips; j++) {
                        const bool has = s0 + j < p.n_strips;
                        const size_t t = has ? (size_t)(s0 + j) * nk + kt : pad;
                        if (has)
                            bulk_g2s(xst + p.off_s + kS24ValBytes * j, p.s24_vals + t * kS24ValBytes,
                                     kS24ValBytes, xbar);
                        bulk_g2s(xst + p.off_s + kTileStrips * kS24ValBytes + kS24MetaBytes * j,
                                 p.s24_meta + t * kS24MetaBytes, kS24MetaBytes, xbar);
                    }
                }
                x_issued++;
                if (++xs == SX) { xs = 0; xph ^= 1u; }
            }
        } else if (warp == kTcbWarp && lane == 0) {  // TCB ring: the two tiles of each k-step
            int rs = 0;
            uint32_t rph = 0;
            for (int i = 0; i < n_kc; i++) {
                const int kt = kstep(i);
                if (i >= SR && !wait_or_abort(smem_u32(&r_empty[rs]), rph ^ 1u, abort_flag, p.wait_limit)) {
                    abort_both();
                    break;
                }
                const uint32_t rbar = smem_u32(&r_full[rs]);
                const uint32_t rst = sbase + p.off_raw + (uint32_t)rs * p.raw_stage_bytes;
                uint32_t total = 0, vb[kTileStrips], u0[kTileStrips];
                for (int j = 0; j < kTileStrips; j++) {
                    vb[j] = 0;
                    u0[j] = 0;
                    if (s0 + j >= p.n_strips) continue;
                    u0[j] = tptr[j * (nk + 1) + kt];
                    const uint32_t u1 = tptr[j * (nk + 1) + kt + 1];
                    vb[j] = u1 >= u0[j] && u1 <= p.values_units ? (u1 - u0[j]) * 16u : 0xFFFFFFFFu;
                    if (vb[j] > p.val_slot - 16u) {  // outside the section or larger than the header allows
                        raise_status(p.status, SPW_ERR_FORMAT);
                        vb[j] = 0;
                    }
                    total += 512u + vb[j];
                }
                mbar_arrive_expect_tx(rbar, total);
                for (int j = 0; j < kTileStrips; j++) {
                    if (s0 + j >= p.n_strips) continue;
                    const size_t t = (size_t)(s0 + j) * nk + kt;
                    bulk_g2s(rst + 512u * j, p.bitmaps + t * kTileCols, 512u, rbar);
                    if (vb[j])
                        bulk_g2s(rst + 1024u + (uint32_t)j * p.val_slot, p.values + (size_t)u0[j] * 8,
                                 vb[j], rbar);
                }
                r_issued++;
                if (++rs == SR) { rs = 0; rph ^= 1u; }
            }
        }
    } else if (warp == 1 && (!PAIR || rank == 0)) {
        // ------------------------------------------------------------ MMA issuer
        // (pair mode: rank 0, for both CTAs: M = 256, A and B halves in each CTA)
        const uint32_t idesc = idesc_f16(PAIR ? 2 * kTileRows : kTileRows, p.MT / p.nh);
        const uint32_t half_cols = (uint32_t)(p.MT / p.nh);           // the MMA's N per h
        const uint32_t brows = PAIR ? half_cols / 2 : half_cols;       // this CTA's B rows per h
        int xs = 0, ws = 0;
        uint32_t xph = 0, wph = 0;
        bool ok = true;
        for (int i = 0; i < n_kc && ok; i++) {
            // 2:4 mode: the W ring advances only on k-steps with residual weights
            const bool dense = !SP24 || !residual_empty(kstep(i));
            ok = __all_sync(0xffffffffu, wait_or_abort(smem_u32(&x_full[xs]), xph, abort_flag, p.wait_limit));
            if (dense)
                ok = ok && __all_sync(0xffffffffu, wait_or_abort(smem_u32(&w_full[ws]), wph, abort_flag, p.wait_limit));
            if constexpr (PAIR)
                ok = ok && __all_sync(0xffffffffu,
                                      wait_or_abort_cluster(smem_u32(&peer_ready[i % kPeerSlots]),
                                                            (uint32_t)((i / kPeerSlots) & 1), abort_flag,
                                                            p.wait_limit));
            if (!ok) {
                if (lane == 0) abort_both();
                break;
            }
            if (lane == 0) {
                tc_fence_after();
                const uint32_t xa = sbase + (uint32_t)xs * p.x_stage_bytes;
                const uint32_t wa = sbase + p.off_w + (uint32_t)ws * kWStageBytes;
                if constexpr (SP24) {
                    // The stage's metadata into its four tensor-memory columns, then two
                    // sparse MMAs (K = 32 each: 16 stored halves = 32 bytes of the S rows,
                    // 64 bytes of X's; metadata column e + j of the even column e), then the
                    // residual's dense MMAs when the k-tile holds any residual weight.
                    const uint32_t sa = xa + p.off_s;
                    const uint32_t e = tmem + p.e_col + 4u * (uint32_t)xs;
                    tmem_cp_128x128b(e, sa + kTileStrips * kS24ValBytes);
                    const uint32_t idesc_sp = idesc | (1u << 2);
#pragma unroll
                    for (int j = 0; j < 2; j++) {
                        const uint64_t adesc = umma_desc_sw64(sa + 32u * j);
                        const uint64_t bdesc = umma_desc_sw128(xa + 64u * j);
                        umma_f16_sp(tmem, adesc, bdesc, idesc_sp | (uint32_t)j, e, (i > 0 || j > 0) ? 1u : 0u);
                    }
                }
#pragma unroll
                for (int j = 0; j < kBK / 16; j++) {
                    if (!dense) break;
                    const uint64_t adesc = umma_desc_sw128(wa + 32u * j);
                    const int slice = i * (kBK / 16) + j;
                    const uint32_t acc = p.n_acc > 1 ? 32u * (uint32_t)(slice % p.n_acc) : 0u;
                    const uint32_t first = SP24 ? 0u
                                                : p.n_acc > 1 ? (uint32_t)(slice < p.n_acc) : (uint32_t)(slice == 0);
                    for (int h = 0; h < p.nh; h++) {
                        const uint64_t bdesc = umma_desc_sw128(xa + brows * 128u * h + 32u * j);
                        if constexpr (PAIR)
                            umma_f16_pair(tmem + acc + half_cols * h, adesc, bdesc, idesc, first ? 0u : 1u);
                        else
                            umma_f16(tmem + acc + half_cols * h, adesc, bdesc, idesc, first ? 0u : 1u);
                    }
                }
                if constexpr (PAIR) {
                    umma_commit_pair_both(smem_u32(&x_empty[xs]));
                    umma_commit_pair_both(smem_u32(&w_empty[ws]));
                } else {
                    umma_commit(smem_u32(&x_empty[xs]));
                    if (dense) umma_commit(smem_u32(&w_empty[ws]));
                }
            }
            __syncwarp();
            if (++xs == SX) { xs = 0; xph ^= 1u; }
            if (dense && ++ws == SW) { ws = 0; wph ^= 1u; }
        }
        if (lane == 0) {
            if constexpr (PAIR) {
                umma_commit_pair_both(smem_u32(acc_full));
                umma_commit_pair_local(smem_u32(drain));
            } else {
                umma_commit(smem_u32(acc_full));
                umma_commit(smem_u32(drain));
            }
            (void)mbar_drain(smem_u32(drain), 0);  // every issued MMA has completed
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ pair relay (rank 1)
        // Once this CTA's X stage has landed and its decoders have filled the W stage of a
        // k-step, tell rank 0 (cluster-scope release); rank 0's commits free both stages.
        const uint32_t ready0 = map_to_rank(smem_u32(&peer_ready[0]), 0u);
        int xs = 0, ws = 0;
        uint32_t xph = 0, wph = 0;
        for (int i = 0; i < n_kc; i++) {
            bool ok = __all_sync(0xffffffffu, wait_or_abort(smem_u32(&x_full[xs]), xph, abort_flag, p.wait_limit));
            ok = ok && __all_sync(0xffffffffu, wait_or_abort(smem_u32(&w_full[ws]), wph, abort_flag, p.wait_limit));
            if (!ok) {
                if (lane == 0) abort_both();
                break;
            }
            if (lane == 0) mbar_arrive_cluster(ready0 + 8u * (uint32_t)(i % kPeerSlots));
            __syncwarp();
            if (++xs == SX) { xs = 0; xph ^= 1u; }
            if (++ws == SW) { ws = 0; wph ^= 1u; }
        }
    } else {
        // ------------------------------------------------------------ decoders
        const int d = warp - 2;          // 0..15
        const int q = d >> 3;            // strip within the tile
        const int g = d & 7;             // 8-column group: one 16-byte chunk per row
        const bool strip_ok = s0 + q < p.n_strips;
        // The warp's 8 column records, 8 bytes per half-column {bits, end of the half's
        // values}: the low halves (rows 0-31) at kRecLo, the high halves at kRecHi, so the
        // 16 bytes at pair p hold columns 2p and 2p+1; the high block sits 16 bytes off so
        // that the two half-warps' reads of one pair fall in different banks.
        constexpr uint32_t kRecLo = 0, kRecHi = 80;
        unsigned char* rec = smem + p.off_rec + kRecBytesPerWarp * d;
        const int qb = 2 * (lane & 15);  // this lane's rows sit at bits qb, qb+1 of one half
        const int sh = qb + 1;
        const uint32_t bit0 = 1u << qb, bit1 = 2u << qb;
        const uint4* recp = (const uint4*)(rec + (lane < 16 ? kRecLo : kRecHi));
        const uint32_t nl0 = 64u * q + 2u * lane;  // local W rows nl0, nl0 + 1
        // Stores of the dense rows: the first store of lanes 4m..4m+3 writes their even row
        // when m is even and their odd row when m is odd (the second store the other), so
        // the 8 lanes of each quarter-warp write 8 distinct swizzled chunk positions.
        const uint32_t swap = ((uint32_t)lane >> 2) & 1u;
        const uint32_t rowA = nl0 + swap, rowB = nl0 + 1u - swap;
        int rs = 0, ws = 0, wi = 0;  // wi: W stages filled so far
        uint32_t rph = 0, wph = 0;
        for (int i = 0; i < n_kc; i++) {
            // every lane waits; __all_sync keeps the outcome warp-uniform
            if (!__all_sync(0xffffffffu, wait_or_abort(smem_u32(&r_full[rs]), rph, abort_flag, p.wait_limit))) {
                abort_both();
                break;
            }
            const uint32_t rst_s = sbase + p.off_raw + (uint32_t)rs * p.raw_stage_bytes;
            // 2:4 mode: a k-tile without residual weights needs no dense W stage (the MMA
            // warp skips its dense MMAs), so its decode is only the check that the strip's
            // residual bitmaps are empty too; the W ring (w_full / w_empty, the stage
            // index) advances only on k-steps with residual weights, on both sides alike.
            const bool skip = SP24 && residual_empty(kstep(i));
            bool dec = strip_ok && !skip;  // warp-uniform
            if (skip && strip_ok) {
                const uint4 bw = *(const uint4*)(smem + p.off_raw + (size_t)rs * p.raw_stage_bytes +
                                                 512u * q + 16u * lane);
                if (__any_sync(0xffffffffu, (bw.x | bw.y | bw.z | bw.w) != 0u) && lane == 0)
                    raise_status(p.status, SPW_ERR_FORMAT);
            }
            if (dec) {
                // columns 2l and 2l+1 of the strip: counts, starts, and the records of the
                // warp's 8 columns (lanes 4g .. 4g+3 hold them).  Only those 8 starts are
                // needed: the kept count of the columns before them (one reduction) plus a
                // scan within the 4 lanes.
                const uint4 bw = *(const uint4*)(smem + p.off_raw + (size_t)rs * p.raw_stage_bytes +
                                                 512u * q + 16u * lane);
                const int cl0 = __popc(bw.x), c0 = cl0 + __popc(bw.y);
                const int cl1 = __popc(bw.z), c1 = cl1 + __popc(bw.w);
                const int cnt = c0 + c1;
                const int before = (int)__reduce_add_sync(0xffffffffu, (lane >> 2) < g ? (uint32_t)cnt : 0u);
                int loc = cnt;
                const int l1 = __shfl_up_sync(0xffffffffu, loc, 1);
                if ((lane & 3) >= 1) loc += l1;
                const int l2 = __shfl_up_sync(0xffffffffu, loc, 2);
                if ((lane & 3) >= 2) loc += l2;
                const int incl = before + loc;  // exact for lanes 4g .. 4g+3
                const uint32_t vb = rst_s + 1024u + (uint32_t)q * p.val_slot;
                const uint32_t a0 = vb + 2u * (uint32_t)(incl - c0 - c1);
                const uint32_t a1 = a0 + 2u * (uint32_t)c0;
                // The tile's packed values fill u1 - u0 16-byte units (0 when the producer
                // rejected the range), so its bitmaps must count between 8 (u1 - u0) - 7
                // and 8 (u1 - u0) kept weights.  Anything else means the bitmaps and the
                // tile pointers disagree: report it and decode the tile as empty rather
                // than read values that belong to no column.
                const int kt = kstep(i);
                const uint32_t u0 = tptr[q * (nk + 1) + kt], u1 = tptr[q * (nk + 1) + kt + 1];
                const uint32_t units = u1 >= u0 && u1 <= p.values_units &&
                                               (uint64_t)(u1 - u0) * 16u <= p.val_slot - 16u
                                           ? u1 - u0
                                           : 0u;
                const uint32_t total = __reduce_add_sync(0xffffffffu, (uint32_t)cnt);
                if ((total + 7u) >> 3 != units) {
                    if (lane == 0) raise_status(p.status, SPW_ERR_FORMAT);
                    dec = false;
                } else if ((lane >> 2) == g) {
                    const uint32_t pp = 16u * (uint32_t)(lane & 3);  // pair: columns 2(l&3), +1
                    *(uint4*)(rec + kRecLo + pp) =
                        make_uint4(bw.x, a0 + 2u * (uint32_t)cl0, bw.z, a1 + 2u * (uint32_t)cl1);
                    *(uint4*)(rec + kRecHi + pp) = make_uint4(bw.y, a1, bw.w, a1 + 2u * (uint32_t)c1);
                }
            }
            __syncwarp();
            if (!skip && wi >= SW &&
                !__all_sync(0xffffffffu, wait_or_abort(smem_u32(&w_empty[ws]), wph ^ 1u, abort_flag, p.wait_limit))) {
                abort_both();
                break;
            }
            unsigned char* wst = smem + p.off_w + (uint32_t)ws * kWStageBytes;
            if (!skip) {  // 8 columns -> one 16-byte chunk per row
                uint32_t o0[4] = {0u, 0u, 0u, 0u}, o1[4] = {0u, 0u, 0u, 0u};
                if (dec) {
#pragma unroll
                    for (int pr = 0; pr < 4; pr++) {
                        const uint4 r = recp[pr];
                        const uint32_t bits[2] = {r.x, r.z}, end[2] = {r.y, r.w};
#pragma unroll
                        for (int e = 0; e < 2; e++) {
                            uint32_t a;
                            asm("mad.lo.s32 %0, %1, -2, %2;" : "=r"(a) : "r"(__popc(bits[e] >> sh)), "r"(end[e]));
                            const uint32_t v1 = lds_u16(a), v0 = lds_u16(a - 2u);
                            const uint32_t sft = 16u * (uint32_t)e;
                            o0[pr] |= ((bits[e] & bit0) ? v0 : 0u) << sft;
                            o1[pr] |= ((bits[e] & bit1) ? v1 : 0u) << sft;
                        }
                    }
                }
                const uint4 wA = swap ? make_uint4(o1[0], o1[1], o1[2], o1[3]) : make_uint4(o0[0], o0[1], o0[2], o0[3]);
                const uint4 wB = swap ? make_uint4(o0[0], o0[1], o0[2], o0[3]) : make_uint4(o1[0], o1[1], o1[2], o1[3]);
                const uint32_t chunk = (uint32_t)g;
                *(uint4*)(wst + rowA * 128u + ((chunk ^ (rowA & 7u)) << 4)) = wA;
                *(uint4*)(wst + rowB * 128u + ((chunk ^ (rowB & 7u)) << 4)) = wB;
            }
            fence_proxy_async_smem();  // generic-proxy stores -> tensor-core reads
            __syncwarp();
            if (lane == 0) {
                if (!skip) mbar_arrive(smem_u32(&w_full[ws]));
                mbar_arrive(smem_u32(&r_empty[rs]));
            }
            if (++rs == SR) { rs = 0; rph ^= 1u; }
            if (!skip) {
                wi++;
                if (++ws == SW) { ws = 0; wph ^= 1u; }
            }
        }

        // ------------------------------------------------------------ epilogue
        const bool acc_ready =
            __all_sync(0xffffffffu, !*abort_flag && wait_or_abort(smem_u32(acc_full), 0, abort_flag, p.wait_limit));
        if (acc_ready) {
            tc_fence_after();
            const int quarter = warp & 3;       // TMEM lanes this warp may access
            const int part_of = (warp - 2) >> 2;  // which 32-column chunks: j % 4 == part_of
            const int row = 32 * quarter + lane;
            const int n = n0 + row;
            float* part = split ? p.partials + ((size_t)stile * p.ksplit + kz) * (size_t)p.MT * kTileRows
                                : nullptr;
            // 32 accumulator columns per load; the allocation is a power of two >= 32, so a
            // tile of 16 tokens reads 16 valid columns and 16 unused ones.
            // accumulators written by this CTA's k-slices (each k-slice writes one of them)
            const int n_used = min(p.n_acc, (k_end - k_begin) * (kBK / 16));
            for (int j = part_of; j < (p.MT + 31) / 32; j += 4) {
                uint32_t r[32];
                if (n_kc > 0) {
                    tmem_ld32(tmem + ((uint32_t)(32 * quarter) << 16) + 32u * j, r);
                } else {  // no k-step (a token tile with an empty list): no MMA wrote TMEM
#pragma unroll
                    for (int c = 0; c < 32; c++) r[c] = 0u;
                }
                for (int a = 1; a < n_used; a++) {  // narrow tiles: add the other chains
                    uint32_t r2[32];
                    tmem_ld32(tmem + ((uint32_t)(32 * quarter) << 16) + 32u * (uint32_t)a, r2);
#pragma unroll
                    for (int c = 0; c < 32; c++) r[c] = __float_as_uint(__uint_as_float(r[c]) + __uint_as_float(r2[c]));
                }
                const int lim = min(32, p.MT - 32 * j);
                if (split) {
#pragma unroll
                    for (int c = 0; c < 32; c++)
                        if (c < lim) part[(size_t)(32 * j + c) * kTileRows + row] = __uint_as_float(r[c]);
                } else if (n < p.N) {
#pragma unroll
                    for (int c = 0; c < 32; c++) {
                        const int m = m0 + 32 * j + c;
                        if (c < lim && m < p.M) {
                            const int ym = p.perm ? (int)__ldg(p.perm + m) : m;
                            p.Y[(size_t)ym * p.ldy + n] = __half_as_ushort(__float2half_rn(__uint_as_float(r[c])));
                        }
                    }
                }
            }
            if (split) __threadfence();  // partials before the arrival below
        } else {
            abort_both();
        }
    }

    tc_fence_before();
    __syncthreads();
    // One decision for the whole CTA: in pair mode the other CTA may raise the flag at
    // any moment, and every thread must take the same side of the barriers below.
    volatile int* aborted = (volatile int*)(tmem_slot + 3);
    if (threadIdx.x == 0) *aborted = *abort_flag;
    __syncthreads();
    if (split && !*aborted) {
        // Split-K: the last CTA of this output tile sums every partial in K order.
        if (threadIdx.x == 0) {
            const uint32_t old = atom_add_release_gpu(&p.counters[stile], 1u);
            *last_flag = old == (uint32_t)(p.ksplit - 1) ? 1u : 0u;
            if (*last_flag) p.counters[stile] = 0u;
        }
        __syncthreads();
        if (*last_flag) {
            __threadfence();
            // Four consecutive rows of one token per thread (16-byte loads), four such
            // groups, two partials at a time: 8 loads in flight per thread.  The partials
            // are summed in split order (deterministic).
            const float4* base = (const float4*)(p.partials + (size_t)stile * p.ksplit * (size_t)p.MT * kTileRows);
            const int n4 = p.MT * kTileRows / 4, stride4 = p.MT * kTileRows / 4;
            for (int i0 = threadIdx.x; i0 < n4; i0 += 4 * kThreads) {
                float4 acc[4];
#pragma unroll
                for (int u = 0; u < 4; u++) acc[u] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                for (int z0 = 0; z0 < p.ksplit; z0 += 2) {
                    float4 v[2][4];
#pragma unroll
                    for (int dz = 0; dz < 2; dz++)
#pragma unroll
                        for (int u = 0; u < 4; u++) {
                            const int i = i0 + u * kThreads;
                            v[dz][u] = (z0 + dz < p.ksplit && i < n4)
                                           ? __ldcg(base + (size_t)(z0 + dz) * stride4 + i)
                                           : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                        }
#pragma unroll
                    for (int dz = 0; dz < 2; dz++)
#pragma unroll
                        for (int u = 0; u < 4; u++) {
                            acc[u].x += v[dz][u].x;
                            acc[u].y += v[dz][u].y;
                            acc[u].z += v[dz][u].z;
                            acc[u].w += v[dz][u].w;
                        }
                }
#pragma unroll
                for (int u = 0; u < 4; u++) {
                    const int i = i0 + u * kThreads;
                    if (i >= n4) continue;
                    const int tok = (4 * i) / kTileRows, row = (4 * i) % kTileRows;
                    const int m = m0 + tok;
                    if (m >= p.M) continue;
                    const int ym = p.perm ? (int)__ldg(p.perm + m) : m;
                    const float v[4] = {acc[u].x, acc[u].y, acc[u].z, acc[u].w};
#pragma unroll
                    for (int e = 0; e < 4; e++)
                        if (n0 + row + e < p.N)
                            p.Y[(size_t)ym * p.ldy + n0 + row + e] = __half_as_ushort(__float2half_rn(v[e]));
                }
            }
        }
    }
    if ((warp == 0 || warp == kTcbWarp) && *abort_flag) {
        // Drain the copies this CTA armed (bounded), each producer its own ring: for each
        // slot, the phase of its last issue.  Phases a consumer already waited for return
        // at once.
        for (int i = 0; warp == 0 && lane == 0 && i < SX && i < x_issued; i++) {
            const int last = i + ((x_issued - 1 - i) / SX) * SX;
            (void)mbar_drain(smem_u32(&x_full[i]), (uint32_t)((last / SX) & 1));
        }
        for (int i = 0; warp == kTcbWarp && lane == 0 && i < SR && i < r_issued; i++) {
            const int last = i + ((r_issued - 1 - i) / SR) * SR;
            (void)mbar_drain(smem_u32(&r_full[i]), (uint32_t)((last / SR) & 1));
        }
    }
    __syncthreads();
    // Pair mode: rank 0's MMAs read both CTAs' shared memory and write both tensor
    // memories; neither CTA frees either until both are past this point (rank 0 has
    // drained its MMAs by then, rank 1 has read its accumulator or given up).
    if constexpr (PAIR) cluster_sync_all();
    if (warp == 1) {
        tc_fence_after();
        if constexpr (PAIR)
            asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                         "r"(p.tmem_cols)
                         : "memory");
        else
            asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                         "r"(p.tmem_cols)
                         : "memory");
    }
}

}  // namespace

// ------------------------------------------------------------------ host side
namespace {

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::mutex g_encode_mutex;

int get_encoder() {
    std::lock_guard<std::mutex> lock(g_encode_mutex);
    if (g_encode) return SPW_OK;
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn)
        return SPW_ERR_CUDA;
    g_encode = (PFN_cuTensorMapEncodeTiled_v12000)fn;
    return SPW_OK;
}

struct SpmmPlan {
    bool pair;  // 256-row tiles on SM pairs (tcgen05 cta_group::2)
    bool sp24;  // 2:4 + residual: S areas in the X stages, metadata columns, <= 256 tokens
    uint32_t off_s, e_col;
    int MT, nh, n_acc, m_tiles, n_tiles, ksplit, n_whole, sx, sr, sw, ctas_per_sm;
    uint32_t x_stage_bytes, val_slot, raw_stage_bytes, tmem_cols;
    uint32_t off_w, off_raw, off_rec, off_tptr, off_klist, off_bar;
    size_t smem;
    uint64_t ws_counters, ws_bytes;
    uint64_t ws_xt;  // decode with a rule: offset of x~ (B rows of K rounded up to 8)
};

// Clusters of two CTAs (one per SM, the most shared memory) that can be resident at once
// on the current device: the SM pairs available to pair-mode tiles.  0 when the query
// fails (pair mode is then not used).
int device_pair_slots() {
    static int cache[kMaxDevices];
    static bool done[kMaxDevices];
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
    std::lock_guard<std::mutex> lock(mu);
    if (!done[dev]) {
        int n = 0;
        if (cudaFuncSetAttribute(spmm_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kSmemLimit) == cudaSuccess) {
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3(2);
            cfg.blockDim = dim3(kThreads);
            cfg.dynamicSmemBytes = kSmemLimit;
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = 2;
            attr[0].val.clusterDim.y = 1;
            attr[0].val.clusterDim.z = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            if (cudaOccupancyMaxActiveClusters(&n, spmm_kernel<true>, &cfg) != cudaSuccess) n = 0;
        }
        (void)cudaGetLastError();
        cache[dev] = n;
        done[dev] = true;
    }
    return cache[dev];
}

// Token tile, split-K factor, stage counts and shared-memory layout for M rows of X.
// sm_count > 0 plans for that many SMs (spw_spmm_plan; pair mode then assumes sm_count / 2
// SM pairs); 0 asks the current device.  allow_pair: the prefill may use 256-row tiles on
// SM pairs (not the tensor-core decode, whose batches are too narrow for X traffic to
// matter).  Pair mode is off unless SPW_SPMM_PAIR=1: on B200 it measured 5-9 % slower
// than one CTA per 128-row tile at M = 2048 (q 102.7 vs 95.3 us), since the kernel is
// bound by shared-memory bandwidth (decoder traffic, X writes, MMA operand reads) rather
// than by the L2 traffic of X that it halves.
int make_spmm_plan(const spw_format* h, int M, bool rule, SpmmPlan* pl, int sm_count = 0,
                   bool allow_pair = false, bool tokens = false, bool sp24 = false) {
    const int sms = sm_count > 0 ? sm_count : device_sm_count();
    if (sms <= 0) return SPW_ERR_CUDA;
    pl->pair = false;
    pl->sp24 = sp24;
    pl->off_s = 0;
    pl->e_col = 0;
    if (allow_pair && !rule && !tokens && !sp24 && M >= 256 && h->N > (uint32_t)kTileRows) {
        const char* e = getenv("SPW_SPMM_PAIR");
        const bool env_on = e && e[0] == '1';
        const int pairs = env_on ? (sm_count > 0 ? sm_count / 2 : device_pair_slots()) : 0;
        pl->pair = pairs > 0;
    }
    const int tile_rows = pl->pair ? 2 * kTileRows : kTileRows;
    // Token tile (512, 256 or 128 tokens, or all M when smaller) and split-K from a small
    // cost model in microseconds: k-steps x max(decode ~0.7, MMA ~0.76 x MT / 512) per CTA,
    // plus, when K is split, the fp32 partial tile written and summed (~0.1 GB/ms per
    // CTA).  One CTA per SM.  Two shapes of split: every tile in k parts (whole waves), or
    // -- when the tiles need more than one wave but fewer than two -- the first F tiles
    // whole and the rest in k parts that fill the SMs as the whole tiles finish (the span
    // estimated as in-order list scheduling).
    pl->n_tiles = (int)((h->N + tile_rows - 1) / tile_rows);
    const long long slots = pl->pair ? (sm_count > 0 ? sm_count / 2 : device_pair_slots()) : sms;
    const long long nk_all = h->n_ktiles;
    const long long kcap = nk_all / 2 > 0 ? (nk_all / 2 < 16 ? nk_all / 2 : 16) : 1;
    double best = 1e300;
    const int tok_cap = sp24 ? kMaxTokens24 : kMaxTokens;
    int best_mt_max = tok_cap, best_ks = 1;
    long long best_whole = -1;  // -1: every tile in best_ks parts (or whole when best_ks == 1)
    for (int tok_max = tok_cap; tok_max >= 128; tok_max /= 2) {
        const int mt = (M + tok_max - 1) / tok_max;
        const int per_t = (M + mt - 1) / mt;
        const int nh_t = per_t > 256 ? 2 : 1;
        const double MTd = (double)round_up_u64((uint64_t)per_t, 16u * nh_t);
        const long long tiles_t = (long long)mt * pl->n_tiles;
        for (long long k = 1; k <= kcap; k++) {
            const double waves = (double)((tiles_t * k + slots - 1) / slots);
            const double step = MTd * 0.76 / 512.0 > 0.7 ? MTd * 0.76 / 512.0 : 0.7;
            const double split = k > 1 ? MTd * 512.0 * (double)(k + 1) / 1e5 : 0.0;
            const double cost = waves * ((double)nk_all / (double)k * step + split);
            if (cost < best * 0.98) {
                best = cost;
                best_mt_max = tok_max;
                best_ks = (int)k;
                best_whole = -1;
            }
        }
        if (tiles_t > slots && tiles_t < 2 * slots) {
            const double step = MTd * 0.76 / 512.0 > 0.7 ? MTd * 0.76 / 512.0 : 0.7;
            const double whole = (double)nk_all * step;     // one whole tile
            const double wr = MTd * 512.0 / 1e5;            // one part's partial tile, written
            for (long long mult = 1; mult <= 2; mult++) {
                const long long S = (tiles_t - slots) * mult;  // split tiles
                if (S > tiles_t) break;
                const long long F = tiles_t - S;               // <= slots
                const long long idle = slots - F;              // SMs free from the start
                for (long long k = 2; k <= kcap && k <= 8; k++) {
                    const double part = (double)nk_all / (double)k * step + wr;
                    const long long Q = S * k;
                    const long long early = idle * (long long)(whole / part);  // parts done by then
                    double span;
                    if (Q > early) span = whole + (double)((Q - early + slots - 1) / slots) * part;
                    else span = idle > 0 ? (double)((Q + idle - 1) / idle) * part : whole;
                    if (span < whole) span = whole;
                    span += (double)k * wr;                    // the last part sums k partials
                    if (span < best * 0.98) {
                        best = span;
                        best_mt_max = tok_max;
                        best_ks = (int)k;
                        best_whole = F;
                    }
                }
            }
        }
        if (M <= tok_max / 2) continue;  // smaller token caps change nothing more for small M
    }
    pl->m_tiles = (M + best_mt_max - 1) / best_mt_max;
    const int per = (M + pl->m_tiles - 1) / pl->m_tiles;
    pl->nh = per > 256 ? 2 : 1;
    pl->MT = (int)round_up_u64((uint64_t)per, 16u * pl->nh);  // each MMA's N a multiple of 16
    pl->x_stage_bytes = (uint32_t)pl->MT * (pl->pair ? 64u : 128u);  // this CTA's share of X
    if (sp24) {  // the k-step's 2:4 values and metadata follow the token tile
        pl->off_s = pl->x_stage_bytes;
        pl->x_stage_bytes += kSStageBytes;
    }
    pl->n_acc = (pl->MT <= 32 && !sp24) ? 4 : 1;
    uint32_t cols = 32;
    while (cols < (uint32_t)(pl->n_acc > 1 ? 32 * pl->n_acc : pl->MT)) cols <<= 1;
    pl->tmem_cols = cols;
    if (sp24) {  // accumulators in columns 0 .. MT-1 (MT <= 256), metadata from column 256
        pl->tmem_cols = 512;
        pl->e_col = 256;
    }
    pl->val_slot = (uint32_t)round_up_u64(16ull * h->max_tile_units + 16, 16);
    pl->raw_stage_bytes = 1024u + (uint32_t)kTileStrips * pl->val_slot;
    const uint32_t tptr_bytes = (uint32_t)round_up_u64(4ull * kTileStrips * (h->n_ktiles + 1), 16);
    // token grouping: the visited k-tile count (16 bytes) and list (2 bytes each)
    const uint32_t klist_bytes = tokens ? 16u + (uint32_t)round_up_u64(2ull * h->n_ktiles, 16) : 0u;
    // {X, TCB, decoded-weight, 2:4} stages, deepest first
    const int options[][4] = {{4, 4, 4, 0}, {3, 4, 4, 0}, {2, 4, 4, 0}, {2, 4, 3, 0}, {2, 3, 3, 0},
                              {2, 3, 2, 0}, {2, 2, 2, 0}};
    const int options24[][4] = {{4, 3, 2, 0}, {3, 3, 2, 0}, {3, 2, 2, 0}, {2, 2, 2, 0}};
    bool found = false;
    const int n_opt = sp24 ? (int)(sizeof(options24) / sizeof(options24[0]))
                           : (int)(sizeof(options) / sizeof(options[0]));
    for (int oi = 0; oi < n_opt; oi++) {
        const int* o = sp24 ? options24[oi] : options[oi];
        const int sx = o[0], sr = o[1], sw = o[2], ss = o[3];
        const uint32_t off_w = (uint32_t)sx * pl->x_stage_bytes;
        const uint32_t off_raw = off_w + (uint32_t)sw * kWStageBytes;
        (void)ss;
        const uint32_t off_rec = off_raw + (uint32_t)sr * pl->raw_stage_bytes;
        const uint32_t off_tptr = off_rec + kRecBytesPerWarp * kDecoderWarps;
        const uint32_t off_klist = off_tptr + tptr_bytes;
        const uint32_t off_bar = (uint32_t)round_up_u64(off_klist + klist_bytes, 8);
        const uint32_t bar_bytes = 8u * (2 * sx + 2 * sr + 2 * sw + 2 + kPeerSlots) + 16u;
        const size_t total = (size_t)off_bar + bar_bytes + 1024;  // + base alignment slack
        if (total <= (size_t)kSmemLimit) {
            pl->sx = sx;
            pl->sr = sr;
            pl->sw = sw;
            pl->off_w = off_w;
            pl->off_raw = off_raw;
            pl->off_rec = off_rec;
            pl->off_tptr = off_tptr;
            pl->off_klist = off_klist;
            pl->off_bar = off_bar;
            pl->smem = total;
            found = true;
            break;
        }
    }
    if (!found) return SPW_ERR_UNSUPPORTED;
    pl->ctas_per_sm = 1;  // 576 threads: one CTA per SM
    const long long tiles = (long long)pl->m_tiles * pl->n_tiles;
    pl->ksplit = best_ks;
    // the hybrid was costed for this token tile's tile count; the uniform plans split all
    // tiles (or none)
    pl->n_whole = best_whole >= 0 ? (int)best_whole : (best_ks > 1 ? 0 : (int)tiles);
    // split-K counters and partial tiles per 128-row output half (two per pair tile)
    const long long n_split = (tiles - pl->n_whole) * (pl->pair ? 2 : 1);
    pl->ws_counters = n_split > 0 ? round_up_u64(4ull * (uint64_t)n_split, 256) : 0;
    pl->ws_bytes = n_split > 0
                       ? pl->ws_counters + 4ull * (uint64_t)n_split * pl->ksplit * pl->MT * kTileRows
                       : 0;
    pl->ws_xt = round_up_u64(pl->ws_bytes, 256);
    if (rule) pl->ws_bytes = pl->ws_xt + 2ull * (uint64_t)M * round_up_u64(h->K, 8);
    return SPW_OK;
}

// Shared by spw_spmm and spw_spmv_tc: checks, tensor map, launch.
// Token grouping (tile_sig not null): X is the grouped input, perm and tile_sig as
// group_tokens_launch wrote them for the plan's token tile.
int tc_product(const spw_format* hdr, const void* d_buf, const uint16_t* d_X, int M, int ldx,
               uint16_t* d_Y, int ldy, int rule, float t, const uint32_t* act_bits, void* d_ws,
               uint64_t ws_bytes, cudaStream_t stream, const uint32_t* perm = nullptr,
               const uint64_t* tile_sig = nullptr, int sig_words = 0, const uint8_t* s24 = nullptr) {
    const bool needs_rule = rule && (t > 0.0f || act_bits);
    const bool tokens = tile_sig != nullptr;
    const bool sp24 = s24 != nullptr;
    SpmmPlan pl;
    int rc = make_spmm_plan(hdr, M, needs_rule, &pl, 0, !rule && !tokens && !sp24, tokens, sp24);
    if (rc != SPW_OK) return rc;
    if (pl.ws_bytes) {
        if (!d_ws) return SPW_ERR_INVALID_ARG;
        if (ws_bytes < pl.ws_bytes) return SPW_ERR_BUFFER_TOO_SMALL;
        if (!aligned16(d_ws)) return SPW_ERR_ALIGNMENT;
    }
    rc = get_encoder();
    if (rc != SPW_OK) return rc;
    int* status = device_status_ptr();
    if (!status) return SPW_ERR_CUDA;

    if (needs_rule) {  // x~ into the workspace; the product reads it instead of X
        const int ld = (int)round_up_u64(hdr->K, 8);
        uint16_t* xt = (uint16_t*)((uint8_t*)d_ws + pl.ws_xt);
        const int n = M * ((int)(hdr->K + 7) / 8);
        rule_kernel<<<(n + 255) / 256, 256, 0, stream>>>(d_X, ldx, M, (int)hdr->K, t, act_bits, xt, ld);
        SPW_LAUNCH_CHECK();
        d_X = xt;
        ldx = ld;
    }
    // X as a 2-D tensor map: dim 0 = K (contiguous), dim 1 = M rows at ldx elements.
    CUtensorMap tmap;
    const cuuint64_t dims[2] = {(cuuint64_t)hdr->K, (cuuint64_t)M};
    const cuuint64_t ld_bytes = (cuuint64_t)((M > 1 ? ldx : ((ldx + 7) / 8 * 8)) * 2);
    const cuuint64_t strides[1] = {ld_bytes};
    const cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)(pl.MT / pl.nh / (pl.pair ? 2 : 1))};
    const cuuint32_t estr[2] = {1, 1};
    CUresult cr = g_encode(&tmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, (void*)d_X, dims, strides, box,
                           estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (cr != CUDA_SUCCESS) return SPW_ERR_CUDA;

    const uint8_t* buf = (const uint8_t*)d_buf;
    SpmmParams prm;
    memset(&prm, 0, sizeof(prm));
    prm.bitmaps = (const uint64_t*)(buf + hdr->off_bitmaps);
    prm.tileptr = (const uint32_t*)(buf + hdr->off_tileptr);
    prm.values = (const uint16_t*)(buf + hdr->off_values);
    prm.values_units = (hdr->bytes_total - hdr->off_values) / 16;
    prm.Y = d_Y;
    prm.counters = pl.ws_bytes ? (uint32_t*)d_ws : nullptr;
    prm.partials = pl.ws_bytes ? (float*)((uint8_t*)d_ws + pl.ws_counters) : nullptr;
    prm.status = status;
    prm.M = M;
    prm.N = (int)hdr->N;
    prm.K = (int)hdr->K;
    prm.ldy = ldy;
    prm.n_strips = (int)hdr->n_strips;
    prm.n_ktiles = (int)hdr->n_ktiles;
    prm.MT = pl.MT;
    prm.nh = pl.nh;
    prm.n_acc = pl.n_acc;
    prm.ksplit = pl.ksplit;
    prm.n_whole = pl.n_whole;
    prm.m_tiles = pl.m_tiles;
    prm.sx = pl.sx;
    prm.sr = pl.sr;
    prm.sw = pl.sw;
    prm.x_stage_bytes = pl.x_stage_bytes;
    prm.raw_stage_bytes = pl.raw_stage_bytes;
    prm.val_slot = pl.val_slot;
    prm.tmem_cols = pl.tmem_cols;
    prm.off_w = pl.off_w;
    prm.off_raw = pl.off_raw;
    prm.off_rec = pl.off_rec;
    prm.off_tptr = pl.off_tptr;
    prm.off_klist = pl.off_klist;
    prm.off_bar = pl.off_bar;
    prm.tile_sig = tile_sig;
    prm.perm = perm;
    prm.sig_words = sig_words;
    if (sp24) {
        const uint64_t n_tiles = (uint64_t)hdr->n_strips * hdr->n_ktiles;
        prm.s24_vals = s24;
        prm.s24_meta = s24 + n_tiles * kS24ValBytes;
        prm.off_s = pl.off_s;
        prm.e_col = pl.e_col;
    }
    prm.wait_limit = wait_limit_cycles();

    static size_t attr_smem[3][kMaxDevices];
    int dev = 0;
    SPW_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= kMaxDevices) return SPW_ERR_CUDA;
    const int variant = pl.pair ? 1 : sp24 ? 2 : 0;
    if (attr_smem[variant][dev] < pl.smem) {
        SPW_CUDA_TRY(cudaFuncSetAttribute(pl.pair ? spmm_kernel<true>
                                                  : sp24 ? spmm_kernel<false, true> : spmm_kernel<false>,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize, (int)pl.smem));
        attr_smem[variant][dev] = pl.smem;
    }
    const long long tiles = (long long)pl.m_tiles * pl.n_tiles;
    const long long slots = pl.n_whole + (tiles - pl.n_whole) * pl.ksplit;  // tiles or parts
    const long long ctas = slots * (pl.pair ? 2 : 1);
    if (ctas > 0x7fffffffll) return SPW_ERR_UNSUPPORTED;
    if (pl.pair) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)ctas);
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = pl.smem;
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        SPW_CUDA_TRY(cudaLaunchKernelEx(&cfg, spmm_kernel<true>, tmap, prm));
    } else if (sp24) {
        spmm_kernel<false, true><<<dim3((unsigned)ctas), kThreads, pl.smem, stream>>>(tmap, prm);
    } else {
        spmm_kernel<false><<<dim3((unsigned)ctas), kThreads, pl.smem, stream>>>(tmap, prm);
    }
    SPW_LAUNCH_CHECK();
    return SPW_OK;
}

}  // namespace
}  // namespace spw

using namespace spw;

extern "C" {

int spw_spmm_plan(const spw_format* hdr, int M, int sm_count, spw_spmm_plan_info* out) {
    if (!out || M < 1) return SPW_ERR_INVALID_ARG;
    const int rc = check_header(hdr);
    if (rc != SPW_OK) return rc;
    SpmmPlan pl;
    const int prc = make_spmm_plan(hdr, M, false, &pl, sm_count, true);
    if (prc != SPW_OK) return prc;
    const long long tiles = (long long)pl.m_tiles * pl.n_tiles;
    out->token_tile = pl.MT;
    out->token_tiles = pl.m_tiles;
    out->weight_tiles = pl.n_tiles;
    out->k_parts = pl.ksplit;
    out->whole_tiles = pl.n_whole;
    out->ctas = (int32_t)((pl.n_whole + (tiles - pl.n_whole) * pl.ksplit) * (pl.pair ? 2 : 1));
    out->cta_pair = pl.pair ? 1 : 0;
    out->reserved = 0;
    out->workspace_bytes = pl.ws_bytes;
    return SPW_OK;
}

uint64_t spw_spmm_workspace_bytes(const spw_format* hdr, int M) {
    if (check_header(hdr) != SPW_OK || M < 1) return 0;
    SpmmPlan pl;
    if (make_spmm_plan(hdr, M, false, &pl, 0, true) != SPW_OK) return 0;
    return pl.ws_bytes;
}

int spw_spmm(const spw_format* hdr, const void* d_buf, const uint16_t* d_X, int M, int ldx,
             uint16_t* d_Y, int ldy, void* d_ws, uint64_t ws_bytes, void* stream) {
    int rc = check_header(hdr);
    if (rc != SPW_OK) return rc;
    if (M < 0) return SPW_ERR_INVALID_ARG;
    if (M == 0) return SPW_OK;  // nothing to compute; X and Y may be NULL
    if (!d_buf || !d_X || !d_Y) return SPW_ERR_INVALID_ARG;
    if (!ld_ok(ldx, (int)hdr->K, M) || ldy < (int)hdr->N) return SPW_ERR_INVALID_ARG;
    if (!aligned16(d_buf) || !aligned16(d_X) || !aligned16(d_Y)) return SPW_ERR_ALIGNMENT;
    return tc_product(hdr, d_buf, d_X, M, ldx, d_Y, ldy, 0, 0.0f, nullptr, d_ws, ws_bytes,
                      (cudaStream_t)stream);
}

// Token grouping: workspace sections after the product's own (split-K) bytes.
struct TokensLayout {
    SpmmPlan pl;
    int ldg, words;
    uint64_t off_xg, off_perm, off_tsig, off_scratch, total;
};

static int tokens_layout(const spw_format* hdr, int M, int sm_count, TokensLayout* L) {
    const int rc = make_spmm_plan(hdr, M, false, &L->pl, sm_count, false, true);
    if (rc != SPW_OK) return rc;
    const int K = (int)hdr->K;
    L->ldg = (int)round_up_u64((uint64_t)K, 8);
    L->words = token_sig_words(K);
    L->off_xg = round_up_u64(L->pl.ws_bytes, 256);
    L->off_perm = L->off_xg + round_up_u64(2ull * (uint64_t)M * L->ldg, 256);
    L->off_tsig = L->off_perm + round_up_u64(4ull * (uint64_t)M, 256);
    L->off_scratch = L->off_tsig + round_up_u64(8ull * (uint64_t)L->pl.m_tiles * L->words, 256);
    L->total = L->off_scratch + token_groups_scratch_bytes(M, K);
    return SPW_OK;
}

uint64_t spw_spmm_tokens_workspace_bytes(const spw_format* hdr, int M) {
    if (check_header(hdr) != SPW_OK || M < 1 || M > kMaxGroupTokens || hdr->K > (uint32_t)kMaxTokenK)
        return 0;
    TokensLayout L;
    if (tokens_layout(hdr, M, 0, &L) != SPW_OK) return 0;
    return L.total;
}

int spw_spmm_tokens_plan(const spw_format* hdr, int M, int sm_count, spw_spmm_plan_info* out) {
    if (!out || M < 1) return SPW_ERR_INVALID_ARG;
    const int rc = check_header(hdr);
    if (rc != SPW_OK) return rc;
    if (M > kMaxGroupTokens || hdr->K > (uint32_t)kMaxTokenK) return SPW_ERR_UNSUPPORTED;
    TokensLayout L;
    const int prc = tokens_layout(hdr, M, sm_count, &L);
    if (prc != SPW_OK) return prc;
    const SpmmPlan& pl = L.pl;
    const long long tiles = (long long)pl.m_tiles * pl.n_tiles;
    out->token_tile = pl.MT;
    out->token_tiles = pl.m_tiles;
    out->weight_tiles = pl.n_tiles;
    out->k_parts = pl.ksplit;
    out->whole_tiles = pl.n_whole;
    out->ctas = (int32_t)(pl.n_whole + (tiles - pl.n_whole) * pl.ksplit);
    out->cta_pair = 0;
    out->reserved = 0;
    out->workspace_bytes = L.total;
    return SPW_OK;
}

int spw_spmm_tokens(const spw_format* hdr, const void* d_buf, const uint16_t* d_X, int M, int ldx,
                    float threshold, uint16_t* d_Y, int ldy, void* d_ws, uint64_t ws_bytes,
                    void* stream) {
    int rc = check_header(hdr);
    if (rc != SPW_OK) return rc;
    if (M < 0) return SPW_ERR_INVALID_ARG;
    if (M == 0) return SPW_OK;
    if (!d_buf || !d_X || !d_Y || !d_ws) return SPW_ERR_INVALID_ARG;
    if (!(threshold >= 0.0f) || isinf(threshold)) return SPW_ERR_INVALID_ARG;
    if (!ld_ok(ldx, (int)hdr->K, M) || ldy < (int)hdr->N) return SPW_ERR_INVALID_ARG;
    if (!aligned16(d_buf) || !aligned16(d_X) || !aligned16(d_Y) || !aligned16(d_ws))
        return SPW_ERR_ALIGNMENT;
    if (M > kMaxGroupTokens || hdr->K > (uint32_t)kMaxTokenK) return SPW_ERR_UNSUPPORTED;
    TokensLayout L;
    rc = tokens_layout(hdr, M, 0, &L);
    if (rc != SPW_OK) return rc;
    if (ws_bytes < L.total) return SPW_ERR_BUFFER_TOO_SMALL;
    uint8_t* ws = (uint8_t*)d_ws;
    uint16_t* xg = (uint16_t*)(ws + L.off_xg);
    uint32_t* perm = (uint32_t*)(ws + L.off_perm);
    uint64_t* tsig = (uint64_t*)(ws + L.off_tsig);
    cudaStream_t st = (cudaStream_t)stream;
    rc = group_tokens_launch(d_X, M, (int)hdr->K, ldx, threshold, L.pl.MT, xg, L.ldg, perm, tsig,
                             ws + L.off_scratch, st);
    if (rc != SPW_OK) return rc;
    return tc_product(hdr, d_buf, xg, M, L.ldg, d_Y, ldy, 0, 0.0f, nullptr, d_ws, L.pl.ws_bytes, st,
                      perm, tsig, L.words);
}

uint64_t spw_spmm24_workspace_bytes(const spw_format* hdr_r, int M) {
    if (check_header(hdr_r) != SPW_OK || M < 1) return 0;
    SpmmPlan pl;
    if (make_spmm_plan(hdr_r, M, false, &pl, 0, false, false, true) != SPW_OK) return 0;
    return pl.ws_bytes;
}

int spw_spmm24_plan(const spw_format* hdr_r, int M, int sm_count, spw_spmm_plan_info* out) {
    if (!out || M < 1) return SPW_ERR_INVALID_ARG;
    const int rc = check_header(hdr_r);
    if (rc != SPW_OK) return rc;
    SpmmPlan pl;
    const int prc = make_spmm_plan(hdr_r, M, false, &pl, sm_count, false, false, true);
    if (prc != SPW_OK) return prc;
    const long long tiles = (long long)pl.m_tiles * pl.n_tiles;
    out->token_tile = pl.MT;
    out->token_tiles = pl.m_tiles;
    out->weight_tiles = pl.n_tiles;
    out->k_parts = pl.ksplit;
    out->whole_tiles = pl.n_whole;
    out->ctas = (int32_t)(pl.n_whole + (tiles - pl.n_whole) * pl.ksplit);
    out->cta_pair = 0;
    out->reserved = 0;
    out->workspace_bytes = pl.ws_bytes;
    return SPW_OK;
}

int spw_spmm24(const spw_format* hdr_r, const void* d_buf_r, const void* d_s24, uint64_t s24_bytes,
               const uint16_t* d_X, int M, int ldx, uint16_t* d_Y, int ldy, void* d_ws,
               uint64_t ws_bytes, void* stream) {
    int rc = check_header(hdr_r);
    if (rc != SPW_OK) return rc;
    if (M < 0) return SPW_ERR_INVALID_ARG;
    if (M == 0) return SPW_OK;
    if (!d_buf_r || !d_s24 || !d_X || !d_Y) return SPW_ERR_INVALID_ARG;
    if (!ld_ok(ldx, (int)hdr_r->K, M) || ldy < (int)hdr_r->N) return SPW_ERR_INVALID_ARG;
    if (!aligned16(d_buf_r) || !aligned16(d_s24) || !aligned16(d_X) || !aligned16(d_Y))
        return SPW_ERR_ALIGNMENT;
    const uint64_t need = (uint64_t)hdr_r->n_strips * hdr_r->n_ktiles * (kS24ValBytes + kS24MetaBytes) +
                          kS24MetaBytes;  // + the padding metadata block
    if (s24_bytes < need) return SPW_ERR_BUFFER_TOO_SMALL;
    return tc_product(hdr_r, d_buf_r, d_X, M, ldx, d_Y, ldy, 0, 0.0f, nullptr, d_ws, ws_bytes,
                      (cudaStream_t)stream, nullptr, nullptr, 0, (const uint8_t*)d_s24);
}

uint64_t spw_spmv_tc_workspace_bytes(const spw_format* hdr, int B) {
    if (B < 1 || B > 16 || check_header(hdr) != SPW_OK) return 0;
    SpmmPlan pl;
    if (make_spmm_plan(hdr, B, true, &pl) != SPW_OK) return 0;
    return pl.ws_bytes;  // room for x~ whatever the threshold and column set
}

int spw_spmv_tc(const spw_format* hdr, const void* d_buf, const uint16_t* d_x, int B, int ldx,
                float threshold, const uint32_t* d_act_bits, uint16_t* d_y, int ldy, void* d_ws,
                uint64_t ws_bytes, void* stream) {
    int rc = check_header(hdr);
    if (rc != SPW_OK) return rc;
    if (B < 1 || B > 16 || !d_buf || !d_x || !d_y) return SPW_ERR_INVALID_ARG;
    if (!(threshold >= 0.0f) || isinf(threshold)) return SPW_ERR_INVALID_ARG;
    if (!ld_ok(ldx, (int)hdr->K, B) || ldy < (int)hdr->N) return SPW_ERR_INVALID_ARG;
    if (!aligned16(d_buf) || !aligned16(d_x) || !aligned16(d_y) || !aligned16(d_act_bits))
        return SPW_ERR_ALIGNMENT;
    return tc_product(hdr, d_buf, d_x, B, ldx, d_y, ldy, 1, threshold, d_act_bits, d_ws, ws_bytes,
                      (cudaStream_t)stream);
}

}  // extern "C"
