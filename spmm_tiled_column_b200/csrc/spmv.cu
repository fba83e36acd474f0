// spmv.cu -- decode spMspV on CUDA cores: y_b = W_masked . x~_b for 1 <= B <= 16.
//
// Method: "Unified Static-Dynamic Pruning for Efficient LLM Inference" (abstract and
// method notes) pairs its bitmap weight format with a CUDA-core spMspV kernel that skips
// activations at run time and decodes bitmaps in shared memory; "Reduced Matrix
// Multiplication" §4.2 computes only the reduced product over the selected input columns
// (§3.1: decode is bound by reading the weight).  The kernel below is this library's
// design for B200:
//
//   * Work split: the tiles of the TCB buffers of a group, in storage order (layer, strip,
//     then k), are cut into one contiguous, equal-count range per consumer warp of a
//     persistent grid (a multiple of the SM count).  A range covers a piece of one or two
//     strips.
//   * Data movement: each CTA has one producer warp and up to eight consumer warps.  Lane
//     k of the producer streams consumer k's tiles -- the 64 bitmap words and the packed
//     values, two 1-D bulk copies (cp.async.bulk, no multicast) -- into that consumer's
//     S-stage ring, one "full" mbarrier per stage counting the bytes and one "empty"
//     mbarrier per stage released by the consumer.  Consumers read activations (and the
//     caller's column-set words) with plain loads, one tile ahead.
//   * Activation skipping: the consumer applies the threshold rule to the tile's 64 x B
//     activations; a ballot gives the active columns (some row's entry survives and the
//     column holds a kept weight).  Inactive columns cost nothing further.
//   * Bitmap decode: lane l owns rows 2l and 2l+1 of the strip, both in one 32-bit half of
//     each column's bitmap word, at bits q and q+1 (q = 2l mod 32).  The kept rows from
//     2l+1 upward hold the last c values of that half's packed segment, c = popc(bits >>
//     (q+1)); row 2l+1's value, if kept, is the first of them and row 2l's, if kept, the one
//     just before.  One popcount, one multiply-add for the
//     address and two 16-bit loads per column; fp16 x fp16 is fused into fp32 accumulators
//     (fma.rn.f32.f16) under a predicate per row.  A column's record {low bits, end of the
//     low half, high bits, end of the high half} is read with one 64-bit load per lane
//     (each half-warp reads its own 8 bytes of the same 16).
//   * Split-K combine: a warp writes its fp32 partial for each strip piece into the
//     workspace; the last contributor of a strip (counted with an atomic) sums all pieces
//     in a fixed order (even pieces, odd pieces, then the two sums), so results are
//     deterministic, rounds to fp16 and resets the counter.  A strip with a single
//     contributor is written directly.  No warp waits for another CTA.
//   * Tile checks: a tile whose pointers leave the values section or whose bitmaps index
//     more values than a stage holds is skipped and reported (SPW_ERR_FORMAT).
//   * FFN mode (spw_spmv_ffn, "Reduced Matrix Multiplication" §4.2): the gate and up
//     layers form one group; once both layers' rows of a strip are final, the warp that
//     finished second computes h = SiLU(g) * u for those rows and the strip's column-set
//     words of h.
#include <stdlib.h>
#include <string.h>

#include "spw_internal.cuh"

namespace spw {
namespace {

constexpr int kMaxConsumers = 8;  // consumer warps per CTA (plus one producer warp)
constexpr int kMaxGroup = 8;      // layers per grouped launch
constexpr int kDefaultConsumers = 8;
constexpr int kDefaultCtasPerSm = 2;
constexpr int kMaxStages = 4;
constexpr int kMinStages = 2;
constexpr int kCtaHeader = 128;  // CTA-wide words before the consumer regions
// Per-consumer header: full mbarriers at 0, empty mbarriers at 32, each stage's tile size
// (16-byte units, written by the producer) at 64, then the column records and x~.  A
// record is 8 bytes per half-column: {the half's 32 bitmap bits, the shared-memory
// address just past that half's packed values}.  The low halves (rows 0-31) sit at
// kRecLoOff, the high halves at kRecHiOff, both in column-position order, so the 16 bytes
// at position 2j are the records of columns 2j and 2j+1; the high block is offset by 16
// bytes so that the two half-warps' 16-byte reads of one pair fall in different banks.
constexpr int kFullOff = 0;
constexpr int kEmptyOff = 32;
constexpr int kUnitsOff = 64;
constexpr int kRecLoOff = 128;
constexpr int kRecHiOff = kRecLoOff + 64 * 8 + 16;
constexpr int kXtOff = kRecHiOff + 64 * 8;  // 64 columns x xt_stride(B) halves
// Column-fetch mode: two record sets and two x~ sets (tiles alternate), then two value
// buffers of sparse_vbuf bytes, each with 16 bytes of slack on both sides of the values.
constexpr int kSpRecOff = 128;
constexpr int kSpRecSet = 1056;  // one set: low block, 16-byte gap, high block (rounded)
constexpr int kSpXtOff = kSpRecOff + 2 * kSpRecSet;
constexpr int kSmemPerSm = 227 * 1024;
constexpr uint32_t kStageValsOff = 512;  // stage: 64 bitmap words, then packed values

// One layer of a decode group: its TCB buffer sections, activations, outputs, workspace
// sections, and its range in the group's concatenated tile space.
struct SpmvLayer {
    const uint64_t* bitmaps;
    const uint32_t* tileptr;
    const uint16_t* values;
    const uint16_t* x;
    const uint32_t* act_bits;
    uint16_t* y;
    uint32_t* counters;
    float* partials;
    int N, K, ldx, ldy;
    int n_ktiles;
    int maxc;
    int tile_begin, n_tiles;
    uint64_t values_units;  // the values section, in 16-byte units
};

struct SpmvParams {
    SpmvLayer L[kMaxGroup];
    int n_layers;
    int* status;
    long long wait_limit;  // pipeline waits, in SM cycles (drains use the fixed limit)
    // Column fetch (the caller passed a column set or a threshold above zero): no producer;
    // each consumer copies only its active columns' values (sparse_vbuf bytes per buffer).
    int sparse_fetch;
    uint32_t sparse_vbuf;
    int n_tiles;      // all layers
    int total_warps;  // working consumer warps
    int stages;
    uint32_t stage_bytes;
    uint32_t warp_smem;
    float t;
    int neg2;  // -2, passed at run time so the address step stays a multiply-add
    // FFN mode (spw_spmv_ffn): layers 0 and 1 are gate and up of one FFN; h = SiLU(g) * u
    // and its column-set bits are written once both layers' rows of a strip are final.
    uint16_t* ffn_h;      // null: not FFN mode
    int ffn_ldh;
    uint32_t* ffn_bits;   // ceil(N / 32) words
    uint32_t* ffn_pairs;  // per strip: finished layers (0, 1 or 2; left at 0)
    float ffn_t;
};

__host__ __device__ constexpr int xt_stride(int B) {
    return B <= 1 ? 1 : B <= 2 ? 2 : B <= 4 ? 4 : B <= 8 ? 8 : 16;
}

__host__ __device__ constexpr uint32_t warp_header_bytes(int B) {
    return (uint32_t)((kXtOff + 64 * 2 * xt_stride(B) + 127) / 128 * 128);
}

__host__ __device__ constexpr uint32_t sparse_header_bytes(int B) {
    return (uint32_t)((kSpXtOff + 2 * 64 * 2 * xt_stride(B) + 127) / 128 * 128);
}

// Column pairs decoded per group: the loads of a group are issued before its
// multiply-adds (x~ of a group is 16 to 64 bytes, read with 16-byte loads).
__host__ __device__ constexpr int pair_group(int B) { return B <= 2 ? 4 : B <= 4 ? 2 : 1; }

__host__ __device__ inline long long warp_of_tile(long long t, long long total_warps,
                                                  long long n_tiles) {
    return ((t + 1) * total_warps - 1) / n_tiles;
}

// Split a 32-bit word into its two fp16 halves (register halves, no shifts).
__device__ inline void split_halves(uint32_t w, uint16_t& lo, uint16_t& hi) {
    asm("mov.b32 {%0, %1}, %2;" : "=h"(lo), "=h"(hi) : "r"(w));
}

// acc[b] += a * x[b] for N batch rows when bits & bit != 0: one lop3 that writes the
// predicate directly, then N predicated fused multiply-adds (fp16 inputs, fp32
// accumulator, one rounding).  A skipped product never touches acc, so a value that
// belongs to another row (possibly Inf/NaN) cannot leak in.
template <int N>
__device__ inline void fma_rows_chunk(uint32_t bits, uint32_t bit, uint16_t a, const uint16_t* x,
                                      float* acc);

template <>
__device__ inline void fma_rows_chunk<1>(uint32_t bits, uint32_t bit, uint16_t a, const uint16_t* x,
                                         float* acc) {
    asm("{\n\t.reg .pred p, q;\n\t.reg .b32 t;\n\t"
        "setp.ne.b32 q, 1, 0;\n\t"
        "lop3.and.b32 t|p, %2, %3, 0, 0xc0, q;\n\t"
        "@p fma.rn.f32.f16 %0, %4, %1, %0;\n\t}"
        : "+f"(acc[0])
        : "h"(x[0]), "r"(bits), "r"(bit), "h"(a));
}

template <>
__device__ inline void fma_rows_chunk<2>(uint32_t bits, uint32_t bit, uint16_t a, const uint16_t* x,
                                         float* acc) {
    asm("{\n\t.reg .pred p, q;\n\t.reg .b32 t;\n\t"
        "setp.ne.b32 q, 1, 0;\n\t"
        "lop3.and.b32 t|p, %4, %5, 0, 0xc0, q;\n\t"
        "@p fma.rn.f32.f16 %0, %6, %2, %0;\n\t"
        "@p fma.rn.f32.f16 %1, %6, %3, %1;\n\t}"
        : "+f"(acc[0]), "+f"(acc[1])
        : "h"(x[0]), "h"(x[1]), "r"(bits), "r"(bit), "h"(a));
}

template <>
__device__ inline void fma_rows_chunk<4>(uint32_t bits, uint32_t bit, uint16_t a, const uint16_t* x,
                                         float* acc) {
    asm("{\n\t.reg .pred p, q;\n\t.reg .b32 t;\n\t"
        "setp.ne.b32 q, 1, 0;\n\t"
        "lop3.and.b32 t|p, %8, %9, 0, 0xc0, q;\n\t"
        "@p fma.rn.f32.f16 %0, %10, %4, %0;\n\t"
        "@p fma.rn.f32.f16 %1, %10, %5, %1;\n\t"
        "@p fma.rn.f32.f16 %2, %10, %6, %2;\n\t"
        "@p fma.rn.f32.f16 %3, %10, %7, %3;\n\t}"
        : "+f"(acc[0]), "+f"(acc[1]), "+f"(acc[2]), "+f"(acc[3])
        : "h"(x[0]), "h"(x[1]), "h"(x[2]), "h"(x[3]), "r"(bits), "r"(bit), "h"(a));
}

template <>
__device__ inline void fma_rows_chunk<8>(uint32_t bits, uint32_t bit, uint16_t a, const uint16_t* x,
                                         float* acc) {
    asm("{\n\t.reg .pred p, q;\n\t.reg .b32 t;\n\t"
        "setp.ne.b32 q, 1, 0;\n\t"
        "lop3.and.b32 t|p, %16, %17, 0, 0xc0, q;\n\t"
        "@p fma.rn.f32.f16 %0, %18, %8, %0;\n\t"
        "@p fma.rn.f32.f16 %1, %18, %9, %1;\n\t"
        "@p fma.rn.f32.f16 %2, %18, %10, %2;\n\t"
        "@p fma.rn.f32.f16 %3, %18, %11, %3;\n\t"
        "@p fma.rn.f32.f16 %4, %18, %12, %4;\n\t"
        "@p fma.rn.f32.f16 %5, %18, %13, %5;\n\t"
        "@p fma.rn.f32.f16 %6, %18, %14, %6;\n\t"
        "@p fma.rn.f32.f16 %7, %18, %15, %7;\n\t}"
        : "+f"(acc[0]), "+f"(acc[1]), "+f"(acc[2]), "+f"(acc[3]), "+f"(acc[4]), "+f"(acc[5]), "+f"(acc[6]), "+f"(acc[7])
        : "h"(x[0]), "h"(x[1]), "h"(x[2]), "h"(x[3]), "h"(x[4]), "h"(x[5]), "h"(x[6]), "h"(x[7]), "r"(bits), "r"(bit), "h"(a));
}


// Any batch width as chunks of 8, 4, 2 and 1 rows.
template <int B>
__device__ inline void fma_rows(uint32_t bits, uint32_t bit, uint16_t a, const uint16_t* x,
                                float* acc) {
    if constexpr (B >= 8) {
        fma_rows_chunk<8>(bits, bit, a, x, acc);
        if constexpr (B > 8) fma_rows<B - 8>(bits, bit, a, x + 8, acc + 8);
    } else if constexpr (B >= 4) {
        fma_rows_chunk<4>(bits, bit, a, x, acc);
        if constexpr (B > 4) fma_rows<B - 4>(bits, bit, a, x + 4, acc + 4);
    } else if constexpr (B >= 2) {
        fma_rows_chunk<2>(bits, bit, a, x, acc);
        if constexpr (B > 2) fma_rows<B - 2>(bits, bit, a, x + 2, acc + 2);
    } else {
        fma_rows_chunk<1>(bits, bit, a, x, acc);
    }
}

// x~ for G consecutive compacted columns (stride XS halves per column).
template <int B, int G>
__device__ inline void load_xg(const uint16_t* xt, int j, uint16_t (&xv)[G][B]) {
    constexpr int XS = xt_stride(B);
    constexpr int WORDS = G * XS / 2;  // 32-bit words covering G columns
    static_assert(WORDS >= 1 && (WORDS < 4 || WORDS % 4 == 0), "x~ slice must be 4, 8 or 16k bytes");
    uint32_t w[WORDS];
    if constexpr (WORDS >= 4) {  // 16-byte loads
        const uint4* p = (const uint4*)(xt + j * XS);
#pragma unroll
        for (int q = 0; q < WORDS / 4; q++) {
            const uint4 v = p[q];
            w[4 * q] = v.x;
            w[4 * q + 1] = v.y;
            w[4 * q + 2] = v.z;
            w[4 * q + 3] = v.w;
        }
    } else if constexpr (WORDS == 2) {  // 8 bytes
        const uint2 v = *(const uint2*)(xt + j * XS);
        w[0] = v.x;
        w[1] = v.y;
    } else {  // 4 bytes
        w[0] = *(const uint32_t*)(xt + j * XS);
    }
    uint16_t h[2 * WORDS];
#pragma unroll
    for (int q = 0; q < WORDS; q++) split_halves(w[q], h[2 * q], h[2 * q + 1]);
#pragma unroll
    for (int c = 0; c < G; c++)
#pragma unroll
        for (int b = 0; b < B; b++) xv[c][b] = h[c * XS + b];
}

// 2 PG column positions of one tile, branch-free.  recp points at this lane's half of
// the records (low or high block): the 16 bytes at position 2j hold columns 2j and 2j+1.
// Every lane loads its two candidate values whether or not its bits are set (both
// addresses stay inside the stage: the lowest is 2 bytes below the tile's first value,
// in the bitmap block, the highest the tile's last value), and the predicated
// multiply-adds keep only the products of kept rows.
template <int B, int PG>
__device__ inline void decode_pairs(const uint4* recp, const uint16_t* xt, int j, int sh, int neg2,
                                    uint32_t bit0, uint32_t bit1, float* acc0, float* acc1) {
    constexpr int G = 2 * PG;
    uint4 r[PG];
    uint16_t xv[G][B];
#pragma unroll
    for (int g = 0; g < PG; g++) r[g] = recp[(j >> 1) + g];
    load_xg<B, G>(xt, j, xv);
    uint32_t bits[G], end[G];
#pragma unroll
    for (int g = 0; g < PG; g++) {
        bits[2 * g] = r[g].x;
        end[2 * g] = r[g].y;
        bits[2 * g + 1] = r[g].z;
        end[2 * g + 1] = r[g].w;
    }
    uint16_t v0[G], v1[G];
#pragma unroll
    for (int c = 0; c < G; c++) {
        const int above = __popc(bits[c] >> sh);  // kept rows from 2l+1 up in this half
        uint32_t a;                               // row 2l+1's value: end - 2 * above
        asm("mad.lo.s32 %0, %1, %2, %3;" : "=r"(a) : "r"(above), "r"(neg2), "r"(end[c]));
        v1[c] = lds_u16(a);
        v0[c] = lds_u16(a - 2u);
    }
#pragma unroll
    for (int c = 0; c < G; c++) {
        fma_rows<B>(bits[c], bit0, v0[c], xv[c], acc0);
        fma_rows<B>(bits[c], bit1, v1[c], xv[c], acc1);
    }
}

// 16-byte global -> shared copy through L2 only (cp.async.cg), and its group fences.
__device__ inline void cp_async16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ inline void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ inline void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Position of a cursor in the group's tile space: layer, tile within the layer, its k-tile
// and strip.
struct Cursor {
    int l, t, kt, s;
};

__device__ inline Cursor cursor_at(const SpmvParams& p, int tg) {
    int l = 0;
    while (l + 1 < p.n_layers && tg >= p.L[l + 1].tile_begin) l++;
    const int t = tg - p.L[l].tile_begin;
    const int nk = p.L[l].n_ktiles;
    return Cursor{l, t, t % nk, t / nk};
}

__device__ inline void cursor_next(const SpmvParams& p, Cursor& c) {
    c.t++;
    if (++c.kt == p.L[c.l].n_ktiles) {
        c.kt = 0;
        c.s++;
    }
    if (c.t == p.L[c.l].n_tiles && c.l + 1 < p.n_layers) {
        c.l++;
        c.t = 0;
        c.kt = 0;
        c.s = 0;
    }
}

// Keeps the accumulators' producing instructions (and so the shared-memory loads they
// depend on) ahead of the stage release that follows.
template <int B>
__device__ inline void pin_acc(float* acc0, float* acc1) {
#pragma unroll
    for (int b = 0; b < B; b++) asm volatile("" : "+f"(acc0[b]), "+f"(acc1[b]));
}

// Producer warp: lane k streams consumer k's tiles (bitmap words and packed values) into
// its ring.  Weights only, so it may run before the previous kernel on the stream is
// complete (programmatic dependent launch).  Before it exits, every copy it issued has
// landed, so no copy can write shared memory after the CTA is gone.
template <int B>
__device__ void produce(const SpmvParams& p, unsigned char* regions, int W, int lane) {
    constexpr uint32_t HDR = warp_header_bytes(B);
    const int T = p.n_tiles, PW = p.total_warps, S = p.stages;
    const int gw = blockIdx.x * W + lane;
    const bool has = lane < W && gw < PW;
    int n = 0;
    Cursor c{0, 0, 0, 0};
    if (has) {
        const int tb = (int)((long long)gw * T / PW);
        n = (int)((long long)(gw + 1) * T / PW) - tb;
        c = cursor_at(p, tb);
    }
    const int nmax = __reduce_max_sync(0xffffffffu, n);
    const uint32_t reg_s = smem_u32(regions + (size_t)(has ? lane : 0) * p.warp_smem);
    const uint64_t pol = policy_evict_first();
    uint32_t u0 = 0, u1 = 0;  // the current tile's value range, in 16-byte units
    if (has) {
        const uint32_t* tp = p.L[c.l].tileptr + c.t;
        u0 = __ldg(tp);
        u1 = __ldg(tp + 1);
    }
    int issued = 0;
    bool ok = has;
    for (int r = 0; r < nmax; r++) {
        if (!ok || r >= n) continue;
        Cursor nc = c;
        cursor_next(p, nc);
        uint32_t nu0 = 0, nu1 = 0;  // next tile's range, fetched a round ahead
        if (r + 1 < n) {
            const uint32_t* tp = p.L[nc.l].tileptr + nc.t;
            nu0 = nc.l == c.l ? u1 : __ldg(tp);
            nu1 = __ldg(tp + 1);
        }
        const int slot = r % S;
        if (r >= S && !mbar_wait(reg_s + kEmptyOff + 8 * slot, (uint32_t)((r / S - 1) & 1), p.wait_limit)) {
            raise_status(p.status, SPW_ERR_TIMEOUT);
            ok = false;
            continue;
        }
        const SpmvLayer& L = p.L[c.l];
        uint64_t vbytes = u1 >= u0 && u1 <= L.values_units ? 16ull * (u1 - u0) : ~0ull;
        if (vbytes > p.stage_bytes - kStageValsOff - 16u) {  // outside the section or larger than the header allows
            raise_status(p.status, SPW_ERR_FORMAT);
            vbytes = 0;
        }
        // The tile's size for the consumer's bitmap check (published by the arrive below).
        *(volatile uint32_t*)(regions + (size_t)lane * p.warp_smem + kUnitsOff + 4 * slot) =
            (uint32_t)(vbytes >> 4);
        const uint32_t bar = reg_s + kFullOff + 8 * slot;
        const uint32_t st = reg_s + HDR + (uint32_t)slot * p.stage_bytes;
        mbar_arrive_expect_tx(bar, 512u + (uint32_t)vbytes);
        bulk_g2s_hint(st, L.bitmaps + (size_t)c.t * kTileCols, 512u, bar, pol);
        if (vbytes) bulk_g2s_hint(st + kStageValsOff, L.values + (size_t)u0 * 8, (uint32_t)vbytes, bar, pol);
        issued = r + 1;
        c = nc;
        u0 = nu0;
        u1 = nu1;
    }
    for (int r = issued > S ? issued - S : 0; r < issued; r++)
        (void)mbar_drain(reg_s + kFullOff + 8 * (r % S), (uint32_t)((r / S) & 1));
}

// Activations of tile columns 2l and 2l+1 for every batch row (one 32-bit load per row
// when both columns exist) and the caller's two column-set bits.
template <int B>
__device__ inline void load_act(const SpmvParams& p, const Cursor& c, int lane, uint32_t (&xw)[B],
                                uint32_t& aw) {
    const SpmvLayer& L = p.L[c.l];
    const int col = c.kt * kTileCols + 2 * lane;
    const uint16_t* xp = L.x + col;
    if (col + 1 < L.K) {
#pragma unroll
        for (int b = 0; b < B; b++) xw[b] = __ldg((const unsigned int*)(xp + (size_t)b * L.ldx));
    } else if (col < L.K) {
#pragma unroll
        for (int b = 0; b < B; b++) xw[b] = __ldg((const unsigned short*)(xp + (size_t)b * L.ldx));
    } else {
#pragma unroll
        for (int b = 0; b < B; b++) xw[b] = 0u;
    }
    aw = 3u;
    if (L.act_bits && col < L.K) aw = (__ldg(L.act_bits + (col >> 5)) >> (col & 31)) & 3u;
}

// FFN mode, after a warp wrote the final fp16 outputs of strip s of the gate or the up
// layer: the second of the two to finish computes, for the strip's rows r and every
// batch row b, h[b][r] = fp16(SiLU(g[b][r]) * u[b][r]) in fp32 from the fp16 outputs
// (SiLU(v) = v / (1 + e^-v)), and the strip's two column-set words: bit r is set when the
// threshold rule keeps h[b][r] for some b.  The outputs are read back from L2 after the
// pair counter's acquire; the counter is reset for the next call.
template <int B>
__device__ void ffn_strip(const SpmvParams& p, int s, int lane) {
    __syncwarp();  // this warp's output stores before the count (release below)
    uint32_t old = 0;
    if (lane == 0) old = atom_add_acq_rel_gpu(p.ffn_pairs + s, 1u);
    old = __shfl_sync(0xffffffffu, old, 0);
    if (old != 1u) return;
    __syncwarp();  // every lane's loads below after lane 0's acquire
    __threadfence();
    const SpmvLayer& G = p.L[0];
    const SpmvLayer& U = p.L[1];
    const int r0 = s * kStripRows + 2 * lane;
    bool keep0 = false, keep1 = false;
#pragma unroll 1
    for (int b = 0; b < B; b++) {
#pragma unroll
        for (int e = 0; e < 2; e++) {
            const int r = r0 + e;
            if (r >= G.N) continue;
            const float g = __half2float(__ushort_as_half(__ldcg(G.y + (size_t)b * G.ldy + r)));
            const float u = __half2float(__ushort_as_half(__ldcg(U.y + (size_t)b * U.ldy + r)));
            const uint16_t h = __half_as_ushort(__float2half_rn(g / (1.0f + expf(-g)) * u));
            p.ffn_h[(size_t)b * p.ffn_ldh + r] = h;
            const bool k = passes_threshold(h, p.ffn_t);
            if (e == 0) keep0 |= k; else keep1 |= k;
        }
    }
    const uint32_t m0 = __ballot_sync(0xffffffffu, keep0), m1 = __ballot_sync(0xffffffffu, keep1);
    if (lane == 0) {
        uint32_t w0 = 0u, w1 = 0u;  // rows 64 s .. 64 s + 31 and 64 s + 32 .. 64 s + 63
#pragma unroll
        for (int l = 0; l < 16; l++) {
            w0 |= (((m0 >> l) & 1u) << (2 * l)) | (((m1 >> l) & 1u) << (2 * l + 1));
            w1 |= (((m0 >> (l + 16)) & 1u) << (2 * l)) | (((m1 >> (l + 16)) & 1u) << (2 * l + 1));
        }
        const int nw = (G.N + 31) / 32;
        if (2 * s < nw) p.ffn_bits[2 * s] = w0;
        if (2 * s + 1 < nw) p.ffn_bits[2 * s + 1] = w1;
        p.ffn_pairs[s] = 0u;
    }
}

// End of tile i of a warp's range: when it closes the warp's piece of strip cur.s (the
// strip's last k-tile, or the warp's last tile), write the piece's rows directly (a
// strip held by one warp) or publish the fp32 partials and let the strip's last
// contributor sum every piece in a fixed order (deterministic), then run the FFN step;
// the accumulators restart at zero.
template <int B>
__device__ inline void finish_piece(const SpmvParams& p, const SpmvLayer& L, const Cursor& cur, int i,
                                    int ntiles, int gw, int lane, float* acc0, float* acc1) {
    const int T = p.n_tiles, PW = p.total_warps;
    const int nk = L.n_ktiles;
    if (cur.kt != nk - 1 && i + 1 != ntiles) return;
    const int s = cur.s;
    const int first = L.tile_begin + s * nk;
    const int g_first = (int)warp_of_tile(first, PW, T);
    const int g_last = (int)warp_of_tile((long long)first + nk - 1, PW, T);
    const int count = g_last - g_first + 1;
    const int r0 = s * kStripRows + 2 * lane;
    bool finished = false;  // this warp wrote the strip's final outputs (warp-uniform)
    if (count == 1) {
#pragma unroll
        for (int b = 0; b < B; b++) {
            if (r0 < L.N) L.y[(size_t)b * L.ldy + r0] = __half_as_ushort(__float2half_rn(acc0[b]));
            if (r0 + 1 < L.N)
                L.y[(size_t)b * L.ldy + r0 + 1] = __half_as_ushort(__float2half_rn(acc1[b]));
        }
        finished = true;
    } else {
        // Publish this piece: store the partials, then one release atomic per warp.
        const int idx = gw - g_first;
        float2* mine = (float2*)(L.partials + ((size_t)s * L.maxc + idx) * B * 64);
#pragma unroll
        for (int b = 0; b < B; b++) mine[b * 32 + lane] = make_float2(acc0[b], acc1[b]);
        __syncwarp();
        uint32_t old = 0;
        if (lane == 0) old = atom_add_release_gpu(&L.counters[s], 1u);
        old = __shfl_sync(0xffffffffu, old, 0);
        if ((int)old == count - 1) {
            // Last contributor: sum every piece in a fixed order (deterministic).  Lanes
            // l and l+16 read rows 4(l mod 16)..+3 of the even and odd pieces with 16-byte
            // loads, 32 pieces in flight per round; the two halves then add up.
            __threadfence();
            const float* base = L.partials + (size_t)s * L.maxc * B * 64;
            const int half = lane >> 4, r4 = 4 * (lane & 15);
#pragma unroll 1
            for (int b = 0; b < B; b++) {
                float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll 1
                for (int j0 = half; j0 < count; j0 += 32) {
                    float4 v[16];
#pragma unroll
                    for (int u = 0; u < 16; u++) {
                        const int j = j0 + 2 * u;
                        v[u] = j < count ? __ldcg((const float4*)(base + ((size_t)j * B + b) * 64 + r4))
                                         : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                    }
#pragma unroll
                    for (int u = 0; u < 16; u++) {
                        acc.x += v[u].x;
                        acc.y += v[u].y;
                        acc.z += v[u].z;
                        acc.w += v[u].w;
                    }
                }
                acc.x += __shfl_xor_sync(0xffffffffu, acc.x, 16);
                acc.y += __shfl_xor_sync(0xffffffffu, acc.y, 16);
                acc.z += __shfl_xor_sync(0xffffffffu, acc.z, 16);
                acc.w += __shfl_xor_sync(0xffffffffu, acc.w, 16);
                const int r = s * kStripRows + r4;
                uint16_t* yb = L.y + (size_t)b * L.ldy;
                if (half == 0) {
                    if (r < L.N) yb[r] = __half_as_ushort(__float2half_rn(acc.x));
                    if (r + 1 < L.N) yb[r + 1] = __half_as_ushort(__float2half_rn(acc.y));
                    if (r + 2 < L.N) yb[r + 2] = __half_as_ushort(__float2half_rn(acc.z));
                    if (r + 3 < L.N) yb[r + 3] = __half_as_ushort(__float2half_rn(acc.w));
                }
            }
            if (lane == 0) L.counters[s] = 0u;
            finished = true;
        }
    }
    if (p.ffn_h && finished) ffn_strip<B>(p, s, lane);
#pragma unroll
    for (int b = 0; b < B; b++) acc0[b] = acc1[b] = 0.0f;
}

// Consumer warp gw: its tile range, decoded from its ring; partial sums flushed per strip.
template <int B>
__device__ void consume(const SpmvParams& p, unsigned char* reg, int gw, int lane) {
    constexpr int XS = xt_stride(B);
    constexpr int PG = pair_group(B);
    constexpr uint32_t HDR = warp_header_bytes(B);
    const int T = p.n_tiles, PW = p.total_warps, S = p.stages;
    if (gw >= PW) return;  // warps are independent: no block-wide barrier follows
    const int t_begin = (int)((long long)gw * T / PW);
    const int ntiles = (int)((long long)(gw + 1) * T / PW) - t_begin;
    const uint32_t reg_s = smem_u32(reg);
    uint2* rec_lo = (uint2*)(reg + kRecLoOff);
    uint2* rec_hi = (uint2*)(reg + kRecHiOff);
    const uint4* recp = (const uint4*)(reg + (lane < 16 ? kRecLoOff : kRecHiOff));
    uint16_t* xt = (uint16_t*)(reg + kXtOff);
    const uint32_t ltmask = lanemask_lt();
    // This lane's rows 2l and 2l+1 sit at bits q and q+1 of the low (lanes 0-15) or high
    // (lanes 16-31) 32 bits of a column's bitmap word.
    const int q = 2 * (lane & 15);
    const int sh = q + 1;
    const uint32_t bit0 = 1u << q, bit1 = 2u << q;
    const int neg2 = p.neg2;
    const bool zero_t = p.t == 0.0f;  // the rule is then "v != 0": one test on the bits

    // Activations, column sets, outputs and the workspace only after the previous kernel
    // on the stream is complete.
    pdl_wait();
    pdl_launch_dependents();

    float acc0[B], acc1[B];
#pragma unroll
    for (int b = 0; b < B; b++) acc0[b] = acc1[b] = 0.0f;
    Cursor cc = cursor_at(p, t_begin);
    uint32_t xw[B], aw;
    load_act<B>(p, cc, lane, xw, aw);
    int slot = 0;
    uint32_t phase = 0;

    for (int i = 0; i < ntiles; i++) {
        const Cursor cur = cc;
        uint32_t xc[B];
#pragma unroll
        for (int b = 0; b < B; b++) xc[b] = xw[b];
        const uint32_t ac = aw;
        cursor_next(p, cc);
        if (i + 1 < ntiles) load_act<B>(p, cc, lane, xw, aw);  // one tile ahead
        const SpmvLayer& L = p.L[cur.l];
        const uint32_t st_s = reg_s + HDR + (uint32_t)slot * p.stage_bytes;
        // Warp-uniform outcome: the ballots below need every lane.
        if (!__all_sync(0xffffffffu, mbar_wait(reg_s + kFullOff + 8 * slot, phase, p.wait_limit))) {
            raise_status(p.status, SPW_ERR_TIMEOUT);
            return;  // the producer drains the copies still in flight
        }

        const uint4 bw = *(const uint4*)(reg + HDR + (size_t)slot * p.stage_bytes + 16 * lane);
        const uint32_t units = *(const volatile uint32_t*)(reg + kUnitsOff + 4 * slot);
        // Column starts within the tile's values (all 64 columns, in column order).
        const int cl0 = __popc(bw.x), c0 = cl0 + __popc(bw.y);
        const int cl1 = __popc(bw.z), c1 = cl1 + __popc(bw.w);
        const int incl = warp_inclusive_scan(c0 + c1, lane);
        // The tile's packed values fill `units` 16-byte units, so its bitmaps must count
        // between 8 units - 7 and 8 units kept weights (the padding is under 8 halves).
        // Anything else means the bitmaps and the tile pointers disagree: report it and
        // decode the tile as empty rather than read values that belong to no column.
        const int total = __shfl_sync(0xffffffffu, incl, 31);
        const bool ok = (uint32_t)(total + 7) >> 3 == units;  // warp-uniform
        if (!ok && lane == 0) raise_status(p.status, SPW_ERR_FORMAT);

        // Threshold rule and column set for columns 2l and 2l+1.
        const int col = cur.kt * kTileCols + 2 * lane;
        const bool in0 = ok && col < L.K && (ac & 1u), in1 = ok && col + 1 < L.K && (ac & 2u);
        uint16_t xa[B], xb[B];
        bool any0 = false, any1 = false;
#pragma unroll
        for (int b = 0; b < B; b++) {
            uint16_t lo, hi;
            split_halves(xc[b], lo, hi);
            const bool p0 = in0 && (zero_t ? (lo & 0x7fffu) != 0u : passes_threshold(lo, p.t));
            const bool p1 = in1 && (zero_t ? (hi & 0x7fffu) != 0u : passes_threshold(hi, p.t));
            xa[b] = p0 ? lo : (uint16_t)0;
            xb[b] = p1 ? hi : (uint16_t)0;
            any0 |= p0;
            any1 |= p1;
        }
        any0 = any0 && (bw.x | bw.y) != 0u;
        any1 = any1 && (bw.z | bw.w) != 0u;
        const uint32_t m0 = __ballot_sync(0xffffffffu, any0);
        const uint32_t m1 = __ballot_sync(0xffffffffu, any1);
        const int n_act = __popc(m0) + __popc(m1);

        if (n_act > 0) {
            const uint32_t vb = st_s + kStageValsOff;
            const uint32_t a0 = vb + 2u * (uint32_t)(incl - c0 - c1);
            const uint32_t a1 = a0 + 2u * (uint32_t)c0;
            const uint2 lo0 = make_uint2(bw.x, a0 + 2u * (uint32_t)cl0);
            const uint2 hi0 = make_uint2(bw.y, a0 + 2u * (uint32_t)c0);
            const uint2 lo1 = make_uint2(bw.z, a1 + 2u * (uint32_t)cl1);
            const uint2 hi1 = make_uint2(bw.w, a1 + 2u * (uint32_t)c1);
            if (B <= 4 && n_act == 64) {
                // Every column active: records in column order (lane l writes the pair
                // 2l, 2l+1 of each half with one 16-byte store) and a fully unrolled decode.
                *(uint4*)(rec_lo + 2 * lane) = make_uint4(lo0.x, lo0.y, lo1.x, lo1.y);
                *(uint4*)(rec_hi + 2 * lane) = make_uint4(hi0.x, hi0.y, hi1.x, hi1.y);
                if constexpr (B == 1) {
                    *(uint32_t*)(xt + 2 * lane) = (uint32_t)xa[0] | ((uint32_t)xb[0] << 16);
                } else {
#pragma unroll
                    for (int b = 0; b < B; b++) {
                        xt[(2 * lane) * XS + b] = xa[b];
                        xt[(2 * lane + 1) * XS + b] = xb[b];
                    }
                }
                __syncwarp();
                if constexpr (B <= 4) {
#pragma unroll
                    for (int j = 0; j < 64; j += 2 * PG)
                        decode_pairs<B, PG>(recp, xt, j, sh, neg2, bit0, bit1, acc0, acc1);
                }
            } else {
                // Active columns compacted in column order; an odd count is padded with an
                // empty column (no bits: its multiply-adds never fire).
                const int pos0 = __popc(m0 & ltmask) + __popc(m1 & ltmask);
                const int pos1 = pos0 + (any0 ? 1 : 0);
                if (any0) {
                    rec_lo[pos0] = lo0;
                    rec_hi[pos0] = hi0;
#pragma unroll
                    for (int b = 0; b < B; b++) xt[pos0 * XS + b] = xa[b];
                }
                if (any1) {
                    rec_lo[pos1] = lo1;
                    rec_hi[pos1] = hi1;
#pragma unroll
                    for (int b = 0; b < B; b++) xt[pos1 * XS + b] = xb[b];
                }
                if ((n_act & 1) && lane == 0) {
                    rec_lo[n_act] = make_uint2(0u, vb);
                    rec_hi[n_act] = make_uint2(0u, vb);
                }
                __syncwarp();
                const int n_cols = (n_act + 1) & ~1;
                int j = 0;
                for (; j + 2 * PG <= n_cols; j += 2 * PG)
                    decode_pairs<B, PG>(recp, xt, j, sh, neg2, bit0, bit1, acc0, acc1);
                if constexpr (PG > 1) {
                    for (; j < n_cols; j += 2)
                        decode_pairs<B, 1>(recp, xt, j, sh, neg2, bit0, bit1, acc0, acc1);
                }
            }
        }
        pin_acc<B>(acc0, acc1);
        __syncwarp();
        if (lane == 0) mbar_arrive(reg_s + kEmptyOff + 8 * slot);  // stage back to the producer
        if (++slot == S) {
            slot = 0;
            phase ^= 1u;
        }

        finish_piece<B>(p, L, cur, i, ntiles, gw, lane, acc0, acc1);
    }
}

// ---------------------------------------------------------------- column-fetch consumer
// Used when the caller passes a column set or a threshold above zero: the bytes of
// inactive columns are never read ("Reduced Matrix Multiplication" §4.2: only W[:, I]
// takes part in the product).  There is no producer: each consumer warp loads a tile's
// bitmap words and tile pointers with plain 16-byte loads two tiles ahead of its decode;
// one tile ahead it applies the threshold rule and column set, builds the records and
// copies, with per-lane 16-byte cp.async, only the 16-byte chunks that hold an active
// column's values; tiles alternate between two record / x~ / value sets.
template <int B>
struct SpTile {  // one tile before its preparation
    Cursor c;
    uint32_t xw[B], aw;
    uint4 bw;  // this lane's two columns' bitmap words
    uint32_t u0, u1;
};

template <int B>
__device__ inline void sp_load(const SpmvParams& p, const Cursor& c, int lane, SpTile<B>& d) {
    d.c = c;
    load_act<B>(p, c, lane, d.xw, d.aw);
    const SpmvLayer& L = p.L[c.l];
    d.bw = __ldg((const uint4*)(L.bitmaps + (size_t)c.t * kTileCols) + lane);
    d.u0 = __ldg(L.tileptr + c.t);
    d.u1 = __ldg(L.tileptr + c.t + 1);
}

// Prepares tile d into set `set` (records, x~, value copies as one cp.async group, which
// is committed even when empty).  Returns the tile's active column count; *all64 when
// every column is active and B <= 4 (records then in column order, fully unrolled decode).
template <int B>
__device__ inline int sp_prepare(const SpmvParams& p, unsigned char* reg, uint32_t reg_s, int set,
                                 const SpTile<B>& d, int lane, uint32_t ltmask, bool zero_t,
                                 bool* all64) {
    constexpr int XS = xt_stride(B);
    const SpmvLayer& L = p.L[d.c.l];
    unsigned char* rset = reg + kSpRecOff + set * kSpRecSet;
    uint2* rec_lo = (uint2*)rset;
    uint2* rec_hi = (uint2*)(rset + (kRecHiOff - kRecLoOff));
    uint16_t* xt = (uint16_t*)(reg + kSpXtOff + set * 128 * XS);
    const uint32_t vb = reg_s + sparse_header_bytes(B) + (uint32_t)set * p.sparse_vbuf + 16u;
    const uint4 bw = d.bw;
    const int cl0 = __popc(bw.x), c0 = cl0 + __popc(bw.y);
    const int cl1 = __popc(bw.z), c1 = cl1 + __popc(bw.w);
    const int incl = warp_inclusive_scan(c0 + c1, lane);
    const int total = __shfl_sync(0xffffffffu, incl, 31);
    // The tile's value range inside the section and the buffer, and the bitmaps' count
    // consistent with it (the checks of the whole-tile path); a tile that fails is decoded
    // as empty and reported.
    const bool range_ok = d.u1 >= d.u0 && d.u1 <= L.values_units &&
                          16ull * (d.u1 - d.u0) + 32ull <= (uint64_t)p.sparse_vbuf;
    const bool ok = range_ok && (uint32_t)(total + 7) >> 3 == d.u1 - d.u0;  // warp-uniform
    if (!ok && lane == 0) raise_status(p.status, SPW_ERR_FORMAT);
    const int col = d.c.kt * kTileCols + 2 * lane;
    const bool in0 = ok && col < L.K && (d.aw & 1u), in1 = ok && col + 1 < L.K && (d.aw & 2u);
    uint16_t xa[B], xb[B];
    bool any0 = false, any1 = false;
#pragma unroll
    for (int b = 0; b < B; b++) {
        uint16_t lo, hi;
        split_halves(d.xw[b], lo, hi);
        const bool p0 = in0 && (zero_t ? (lo & 0x7fffu) != 0u : passes_threshold(lo, p.t));
        const bool p1 = in1 && (zero_t ? (hi & 0x7fffu) != 0u : passes_threshold(hi, p.t));
        xa[b] = p0 ? lo : (uint16_t)0;
        xb[b] = p1 ? hi : (uint16_t)0;
        any0 |= p0;
        any1 |= p1;
    }
    any0 = any0 && (bw.x | bw.y) != 0u;
    any1 = any1 && (bw.z | bw.w) != 0u;
    const uint32_t m0 = __ballot_sync(0xffffffffu, any0);
    const uint32_t m1 = __ballot_sync(0xffffffffu, any1);
    const int n_act = __popc(m0) + __popc(m1);
    *all64 = B <= 4 && n_act == 64;
    __syncwarp();  // the tile that used this set two tiles back is fully decoded
    if (n_act > 0) {
        const int st0 = incl - c0 - c1;  // index of column 2l's first value in the tile
        const uint32_t a0 = vb + 2u * (uint32_t)st0;
        const uint32_t a1 = a0 + 2u * (uint32_t)c0;
        const uint2 lo0 = make_uint2(bw.x, a0 + 2u * (uint32_t)cl0);
        const uint2 hi0 = make_uint2(bw.y, a0 + 2u * (uint32_t)c0);
        const uint2 lo1 = make_uint2(bw.z, a1 + 2u * (uint32_t)cl1);
        const uint2 hi1 = make_uint2(bw.w, a1 + 2u * (uint32_t)c1);
        if (*all64) {
            *(uint4*)(rec_lo + 2 * lane) = make_uint4(lo0.x, lo0.y, lo1.x, lo1.y);
            *(uint4*)(rec_hi + 2 * lane) = make_uint4(hi0.x, hi0.y, hi1.x, hi1.y);
#pragma unroll
            for (int b = 0; b < B; b++) {
                xt[(2 * lane) * XS + b] = xa[b];
                xt[(2 * lane + 1) * XS + b] = xb[b];
            }
        } else {
            const int pos0 = __popc(m0 & ltmask) + __popc(m1 & ltmask);
            const int pos1 = pos0 + (any0 ? 1 : 0);
            if (any0) {
                rec_lo[pos0] = lo0;
                rec_hi[pos0] = hi0;
#pragma unroll
                for (int b = 0; b < B; b++) xt[pos0 * XS + b] = xa[b];
            }
            if (any1) {
                rec_lo[pos1] = lo1;
                rec_hi[pos1] = hi1;
#pragma unroll
                for (int b = 0; b < B; b++) xt[pos1 * XS + b] = xb[b];
            }
            if ((n_act & 1) && lane == 0) {
                rec_lo[n_act] = make_uint2(0u, vb);
                rec_hi[n_act] = make_uint2(0u, vb);
            }
        }
        // The 16-byte chunks that hold this lane's active columns' values (the two
        // columns' values are adjacent, so one range covers both when both are active).
        int lo = 0, hi = -1;
        if (any0) {
            lo = st0 >> 3;
            hi = (st0 + c0 - 1) >> 3;
        }
        if (any1) {
            if (!any0) lo = (st0 + c0) >> 3;
            hi = (st0 + c0 + c1 - 1) >> 3;
        }
        const uint16_t* src = L.values + (size_t)d.u0 * 8;
        for (int ch = lo; ch <= hi; ch++) cp_async16(vb + 16u * (uint32_t)ch, src + 8 * ch);
    }
    cp_async_commit();
    return n_act;
}

template <int B>
__device__ void consume_sparse(const SpmvParams& p, unsigned char* reg, int gw, int lane) {
    constexpr int XS = xt_stride(B);
    constexpr int PG = pair_group(B);
    const int T = p.n_tiles, PW = p.total_warps;
    if (gw >= PW) return;
    const int t_begin = (int)((long long)gw * T / PW);
    const int ntiles = (int)((long long)(gw + 1) * T / PW) - t_begin;
    const uint32_t reg_s = smem_u32(reg);
    const uint32_t ltmask = lanemask_lt();
    const int q = 2 * (lane & 15);
    const int sh = q + 1;
    const uint32_t bit0 = 1u << q, bit1 = 2u << q;
    const int neg2 = p.neg2;
    const bool zero_t = p.t == 0.0f;

    pdl_wait();
    pdl_launch_dependents();

    float acc0[B], acc1[B];
#pragma unroll
    for (int b = 0; b < B; b++) acc0[b] = acc1[b] = 0.0f;
    Cursor cc = cursor_at(p, t_begin);
    SpTile<B> d0, d1;
    sp_load<B>(p, cc, lane, d0);
    cursor_next(p, cc);
    if (ntiles > 1) sp_load<B>(p, cc, lane, d1);
    bool all_cur = false;
    int n_cur = sp_prepare<B>(p, reg, reg_s, 0, d0, lane, ltmask, zero_t, &all_cur);
    Cursor cur = d0.c;
    for (int i = 0; i < ntiles; i++) {
        bool all_next = false;
        int n_next = 0;
        SpTile<B> d2;
        if (i + 1 < ntiles) {
            cursor_next(p, cc);  // tile i + 2
            if (i + 2 < ntiles) sp_load<B>(p, cc, lane, d2);
            n_next = sp_prepare<B>(p, reg, reg_s, (i + 1) & 1, d1, lane, ltmask, zero_t, &all_next);
            cp_async_wait<1>();  // tile i's copies (the older group) have landed
        } else {
            cp_async_wait<0>();
        }
        __syncwarp();  // and every lane's copies are visible to the whole warp
        if (n_cur > 0) {
            unsigned char* rset = reg + kSpRecOff + (i & 1) * kSpRecSet;
            const uint4* recp = (const uint4*)(rset + (lane < 16 ? 0 : (kRecHiOff - kRecLoOff)));
            const uint16_t* xt = (const uint16_t*)(reg + kSpXtOff + (i & 1) * 128 * XS);
            if constexpr (B <= 4) {
                if (all_cur) {
#pragma unroll
                    for (int j = 0; j < 64; j += 2 * PG)
                        decode_pairs<B, PG>(recp, xt, j, sh, neg2, bit0, bit1, acc0, acc1);
                }
            }
            if (!all_cur) {
                const int n_cols = (n_cur + 1) & ~1;
                int j = 0;
                for (; j + 2 * PG <= n_cols; j += 2 * PG)
                    decode_pairs<B, PG>(recp, xt, j, sh, neg2, bit0, bit1, acc0, acc1);
                if constexpr (PG > 1) {
                    for (; j < n_cols; j += 2)
                        decode_pairs<B, 1>(recp, xt, j, sh, neg2, bit0, bit1, acc0, acc1);
                }
            }
        }
        pin_acc<B>(acc0, acc1);
        __syncwarp();
        finish_piece<B>(p, p.L[cur.l], cur, i, ntiles, gw, lane, acc0, acc1);
        cur = d1.c;
        n_cur = n_next;
        all_cur = all_next;
        d1 = d2;
    }
}

template <int B>
__global__ void __launch_bounds__((kMaxConsumers + 1) * 32, B <= 8 ? 2 : 1)
spmv_kernel(const __grid_constant__ SpmvParams p) {
    extern __shared__ __align__(1024) unsigned char smem[];
    const int W = (int)(blockDim.x >> 5) - 1;  // consumer warps; the last warp produces
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    unsigned char* regions = smem + kCtaHeader;
    if (threadIdx.x == 0) {
        for (int k = 0; k < W; k++) {
            const uint32_t r = smem_u32(regions + (size_t)k * p.warp_smem);
            for (int s = 0; s < p.stages; s++) {
                mbar_init(r + kFullOff + 8 * s, 1);
                mbar_init(r + kEmptyOff + 8 * s, 1);
            }
        }
        fence_mbar_init();
    }
    __syncthreads();
    if (warp == W) {
        if (!p.sparse_fetch) produce<B>(p, regions, W, lane);
        pdl_launch_dependents();
        return;
    }
    if (p.sparse_fetch)
        consume_sparse<B>(p, regions + (size_t)warp * p.warp_smem, blockIdx.x * W + warp, lane);
    else
        consume<B>(p, regions + (size_t)warp * p.warp_smem, blockIdx.x * W + warp, lane);
}

struct Plan {
    bool sparse;            // column fetch (consume_sparse)
    uint32_t sparse_vbuf;   // its value buffer bytes
    int grid, warps, ctas_per_sm, stages;  // warps = consumer warps per CTA
    uint32_t stage_bytes, warp_smem;
    size_t smem;
    long long n_tiles, total_warps;
    int maxc[kMaxGroup];
    uint64_t ws_off[kMaxGroup];       // each layer's workspace section (counters first)
    uint64_t ws_counters[kMaxGroup];  // bytes of that section's counter block
    uint64_t ws_bytes;
};

// Occupancy knobs: consumer warps per CTA, CTAs per SM and stages per warp.
// SPW_SPMV_WARPS, SPW_SPMV_CTAS_PER_SM and SPW_SPMV_STAGES override the defaults (a
// tuning aid; they change only the launch shape, never the work done).
int env_int(const char* name, int dflt, int lo, int hi) {
    const char* v = getenv(name);
    if (!v || !*v) return dflt;
    const int x = atoi(v);
    return (x < lo || x > hi) ? dflt : x;
}

// Launch plan for a group of n layers decoded in one launch (n = 1 for spw_spmv).
// want_sparse: fetch only active columns when their buffers fit the same launch shape
// (the work partition, and so the workspace and the results, do not depend on the mode).
int make_plan(int n, const spw_format* h, int B, Plan* pl, bool want_sparse = false) {
    const int sms = device_sm_count();
    if (sms <= 0) return SPW_ERR_CUDA;
    long long T = 0;
    uint32_t max_units = 0;
    for (int l = 0; l < n; l++) {
        T += (long long)h[l].n_strips * h[l].n_ktiles;
        max_units = h[l].max_tile_units > max_units ? h[l].max_tile_units : max_units;
    }
    if (T > 0x7fffffffll) return SPW_ERR_UNSUPPORTED;
    pl->n_tiles = T;
    // stage: bitmap words, values, and 16 bytes of slack for the branch-free loads one
    // past a column's last value
    pl->stage_bytes = (uint32_t)round_up_u64(kStageValsOff + 16ull * max_units + 16, 128);
    // Preferred launch shape first; fall back to fewer warps per SM when the stages of
    // wide batches or dense formats do not fit two per warp.
    const int want_warps = env_int("SPW_SPMV_WARPS", kDefaultConsumers, 1, kMaxConsumers);
    const int want_ctas = env_int("SPW_SPMV_CTAS_PER_SM", kDefaultCtasPerSm, 1, 32);
    const int shapes[][2] = {{want_warps, want_ctas}, {4, 2}, {4, 1}, {2, 1}, {1, 1}};
    int stages = 0;
    for (const auto& sh : shapes) {
        pl->warps = sh[0];
        pl->ctas_per_sm = B > 8 && sh[1] > 1 ? 1 : sh[1];  // wide batches: one CTA per SM
        const long long budget = kSmemPerSm / pl->ctas_per_sm - 1024 - kCtaHeader;
        const long long per_warp = budget / pl->warps - warp_header_bytes(B);
        stages = per_warp > 0 ? (int)(per_warp / pl->stage_bytes) : 0;
        if (stages >= kMinStages) break;
    }
    if (stages < kMinStages) return SPW_ERR_UNSUPPORTED;
    const int max_stages = env_int("SPW_SPMV_STAGES", kMaxStages, kMinStages, kMaxStages);
    if (stages > max_stages) stages = max_stages;
    pl->grid = sms * pl->ctas_per_sm;
    pl->total_warps = (long long)pl->grid * pl->warps;
    if (pl->total_warps > T) pl->total_warps = T;  // one tile or more per working warp
    pl->stages = stages;
    pl->warp_smem = warp_header_bytes(B) + (uint32_t)stages * pl->stage_bytes;
    pl->smem = kCtaHeader + (size_t)pl->warps * pl->warp_smem;
    pl->sparse = false;
    pl->sparse_vbuf = 0;
    if (want_sparse) {
        const uint32_t vbuf = (uint32_t)round_up_u64(16ull * max_units + 32, 128);
        const uint32_t sp_warp = sparse_header_bytes(B) + 2u * vbuf;
        const long long budget = kSmemPerSm / pl->ctas_per_sm - 1024 - kCtaHeader;
        if ((long long)pl->warps * sp_warp <= budget) {
            pl->sparse = true;
            pl->sparse_vbuf = vbuf;
            pl->warp_smem = sp_warp;
            pl->smem = kCtaHeader + (size_t)pl->warps * sp_warp;
        }
    }
    // Per layer: the most warps that share one strip under this partition, and the
    // layer's workspace section (arrival counters, then fp32 partial sums).
    uint64_t off = 0;
    long long begin = 0;
    for (int l = 0; l < n; l++) {
        int maxc = 1;
        for (long long st = 0; st < h[l].n_strips; st++) {
            const long long first = begin + st * h[l].n_ktiles;
            const long long c = warp_of_tile(first + h[l].n_ktiles - 1, pl->total_warps, T) -
                                warp_of_tile(first, pl->total_warps, T) + 1;
            if (c > maxc) maxc = (int)c;
        }
        pl->maxc[l] = maxc;
        pl->ws_off[l] = off;
        pl->ws_counters[l] = round_up_u64(4ull * h[l].n_strips, 256);
        off += pl->ws_counters[l] +
               round_up_u64((uint64_t)h[l].n_strips * maxc * B * 64 * sizeof(float), 256);
        begin += (long long)h[l].n_strips * h[l].n_ktiles;
    }
    pl->ws_bytes = off;
    return SPW_OK;
}

template <int B>
int launch(const Plan& pl, const SpmvParams& prm, cudaStream_t s) {
    static size_t attr_smem[kMaxDevices];
    int dev = 0;
    SPW_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= kMaxDevices) return SPW_ERR_CUDA;
    if (attr_smem[dev] < pl.smem) {
        SPW_CUDA_TRY(cudaFuncSetAttribute(spmv_kernel<B>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          (int)pl.smem));
        // The grid is sized for this many CTAs per SM; ask for the full shared-memory
        // carveout so small per-CTA footprints do not lower the residency.
        SPW_CUDA_TRY(cudaFuncSetAttribute(spmv_kernel<B>,
                                          cudaFuncAttributePreferredSharedMemoryCarveout,
                                          (int)cudaSharedmemCarveoutMaxShared));
        attr_smem[dev] = pl.smem;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(pl.grid);
    cfg.blockDim = dim3((pl.warps + 1) * 32);
    cfg.dynamicSmemBytes = pl.smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = launch_overlap() ? 1 : 0;
    SPW_CUDA_TRY(cudaLaunchKernelEx(&cfg, spmv_kernel<B>, prm));
    SPW_LAUNCH_CHECK();
    return SPW_OK;
}

// Checks shared by spw_spmv and spw_spmv_group, and the launch.
// FFN mode outputs (spw_spmv_ffn): h, its column-set words, the per-strip pair counters
// and the threshold applied to h.
struct FfnOut {
    uint16_t* h;
    int ldh;
    uint32_t* bits;
    uint32_t* pairs;
    float t;
};

int decode_group_launch(int n, const spw_format* hdrs, const void* const* bufs,
                        const uint16_t* const* xs, const int* ldxs,
                        const uint32_t* const* act_bits, uint16_t* const* ys, const int* ldys,
                        int B, float threshold, void* d_ws, uint64_t ws_bytes, cudaStream_t s,
                        const FfnOut* ffn = nullptr) {
    if (n < 1 || n > kMaxGroup || !hdrs || !bufs || !xs || !ldxs || !ys || !ldys)
        return SPW_ERR_INVALID_ARG;
    if (!d_ws) return SPW_ERR_INVALID_ARG;
    for (int l = 0; l < n; l++) {
        const int rc = check_decode_args(&hdrs[l], bufs[l], xs[l], B, ldxs[l], threshold,
                                         act_bits ? act_bits[l] : nullptr, ys[l], ldys[l]);
        if (rc != SPW_OK) return rc;
    }
    if (!aligned16(d_ws)) return SPW_ERR_ALIGNMENT;
    // Column fetch (spw_set_column_fetch): never, when the caller signals activation
    // sparsity (a column set or a threshold above zero), or always.  The mode changes
    // which bytes are read, never the result.
    const int fetch = column_fetch_mode();
    bool want_sparse = fetch == 2;
    if (fetch == 1) {
        want_sparse = threshold > 0.0f;
        for (int l = 0; l < n; l++) want_sparse = want_sparse || (act_bits && act_bits[l]);
    }
    Plan pl;
    int rc = make_plan(n, hdrs, B, &pl, want_sparse && !ffn);
    if (rc != SPW_OK) return rc;
    if (ws_bytes < pl.ws_bytes) return SPW_ERR_BUFFER_TOO_SMALL;
    int* status = device_status_ptr();
    if (!status) return SPW_ERR_CUDA;
    SpmvParams prm;
    memset(&prm, 0, sizeof(prm));
    long long begin = 0;
    for (int l = 0; l < n; l++) {
        const spw_format& h = hdrs[l];
        const uint8_t* buf = (const uint8_t*)bufs[l];
        SpmvLayer& L = prm.L[l];
        L.bitmaps = (const uint64_t*)(buf + h.off_bitmaps);
        L.tileptr = (const uint32_t*)(buf + h.off_tileptr);
        L.values = (const uint16_t*)(buf + h.off_values);
        L.x = xs[l];
        L.act_bits = act_bits ? act_bits[l] : nullptr;
        L.y = ys[l];
        L.counters = (uint32_t*)((uint8_t*)d_ws + pl.ws_off[l]);
        L.partials = (float*)((uint8_t*)d_ws + pl.ws_off[l] + pl.ws_counters[l]);
        L.N = (int)h.N;
        L.K = (int)h.K;
        L.ldx = ldxs[l];
        L.ldy = ldys[l];
        L.n_ktiles = (int)h.n_ktiles;
        L.maxc = pl.maxc[l];
        L.tile_begin = (int)begin;
        L.n_tiles = (int)((long long)h.n_strips * h.n_ktiles);
        L.values_units = (h.bytes_total - h.off_values) / 16;
        begin += L.n_tiles;
    }
    prm.n_layers = n;
    prm.status = status;
    prm.n_tiles = (int)pl.n_tiles;
    prm.total_warps = (int)pl.total_warps;
    prm.stages = pl.stages;
    prm.stage_bytes = pl.stage_bytes;
    prm.warp_smem = pl.warp_smem;
    prm.t = threshold;
    prm.neg2 = -2;
    prm.wait_limit = wait_limit_cycles();
    prm.sparse_fetch = pl.sparse ? 1 : 0;
    prm.sparse_vbuf = pl.sparse_vbuf;
    if (ffn) {
        prm.ffn_h = ffn->h;
        prm.ffn_ldh = ffn->ldh;
        prm.ffn_bits = ffn->bits;
        prm.ffn_pairs = ffn->pairs;
        prm.ffn_t = ffn->t;
    }
    switch (B) {
#define SPW_CASE(b) \
    case b: return launch<b>(pl, prm, s);
        SPW_CASE(1) SPW_CASE(2) SPW_CASE(3) SPW_CASE(4) SPW_CASE(5) SPW_CASE(6) SPW_CASE(7)
        SPW_CASE(8) SPW_CASE(9) SPW_CASE(10) SPW_CASE(11) SPW_CASE(12) SPW_CASE(13)
        SPW_CASE(14) SPW_CASE(15) SPW_CASE(16)
#undef SPW_CASE
    }
    return SPW_ERR_INVALID_ARG;
}

// Workspace of spw_spmv_ffn: the two-layer decode group's section, the per-strip pair
// counters, then the fp16 gate and up outputs (B rows of ld halves each).
struct FfnWorkspace {
    uint64_t group, pairs, g, u, total;
    int ld;
};

int ffn_workspace(const spw_format* hdr_gate, const spw_format* hdr_up, int B, FfnWorkspace* w) {
    if (!hdr_gate || !hdr_up || B < 1 || B > 16) return SPW_ERR_INVALID_ARG;
    int rc = check_header(hdr_gate);
    if (rc == SPW_OK) rc = check_header(hdr_up);
    if (rc != SPW_OK) return rc;
    if (hdr_gate->N != hdr_up->N || hdr_gate->K != hdr_up->K) return SPW_ERR_INVALID_ARG;
    const spw_format hd[2] = {*hdr_gate, *hdr_up};
    Plan pl;
    rc = make_plan(2, hd, B, &pl);
    if (rc != SPW_OK) return rc;
    w->ld = (int)round_up_u64(hdr_gate->N, 8);
    w->group = round_up_u64(pl.ws_bytes, 256);
    w->pairs = round_up_u64(4ull * hdr_gate->n_strips, 256);
    const uint64_t out = round_up_u64(2ull * (uint64_t)B * (uint64_t)w->ld, 256);
    w->g = w->group + w->pairs;
    w->u = w->g + out;
    w->total = w->u + out;
    return SPW_OK;
}

}  // namespace

int check_decode_args(const spw_format* hdr, const void* buf, const uint16_t* x, int B, int ldx,
                      float threshold, const uint32_t* act_bits, const uint16_t* y, int ldy) {
    const int rc = check_header(hdr);
    if (rc != SPW_OK) return rc;
    if (B < 1 || B > 16) return SPW_ERR_INVALID_ARG;
    if (!(threshold >= 0.0f) || isinf(threshold)) return SPW_ERR_INVALID_ARG;
    if (!buf || !x || !y) return SPW_ERR_INVALID_ARG;
    if (!ld_ok(ldx, (int)hdr->K, B) || ldy < (int)hdr->N) return SPW_ERR_INVALID_ARG;
    if (!aligned16(buf) || !aligned16(x) || !aligned16(y) || !aligned16(act_bits))
        return SPW_ERR_ALIGNMENT;
    return SPW_OK;
}

}  // namespace spw

using namespace spw;

extern "C" {

uint64_t spw_spmv_ffn_workspace_bytes(const spw_format* hdr_gate, const spw_format* hdr_up, int B) {
    FfnWorkspace w;
    return ffn_workspace(hdr_gate, hdr_up, B, &w) == SPW_OK ? w.total : 0;
}

int spw_spmv_ffn(const spw_format* hdr_gate, const void* d_buf_gate, const spw_format* hdr_up,
                 const void* d_buf_up, const uint16_t* d_x, int B, int ldx, float threshold,
                 uint16_t* d_h, int ldh, uint32_t* d_act_bits, void* d_ws, uint64_t ws_bytes,
                 void* stream) {
    FfnWorkspace w;
    const int rc = ffn_workspace(hdr_gate, hdr_up, B, &w);
    if (rc != SPW_OK) return rc;
    if (!d_h || !d_act_bits || !d_ws || ldh < (int)hdr_gate->N) return SPW_ERR_INVALID_ARG;
    if (!(threshold >= 0.0f) || isinf(threshold)) return SPW_ERR_INVALID_ARG;
    if (!aligned16(d_h) || !aligned16(d_act_bits) || !aligned16(d_ws)) return SPW_ERR_ALIGNMENT;
    if (ws_bytes < w.total) return SPW_ERR_BUFFER_TOO_SMALL;
    uint8_t* ws = (uint8_t*)d_ws;
    const spw_format hd[2] = {*hdr_gate, *hdr_up};
    const void* bufs[2] = {d_buf_gate, d_buf_up};
    const uint16_t* xs[2] = {d_x, d_x};
    const int ldxs[2] = {ldx, ldx};
    uint16_t* ys[2] = {(uint16_t*)(ws + w.g), (uint16_t*)(ws + w.u)};
    const int ldys[2] = {w.ld, w.ld};
    const FfnOut ffn = {d_h, ldh, d_act_bits, (uint32_t*)(ws + w.group), threshold};
    return decode_group_launch(2, hd, bufs, xs, ldxs, nullptr, ys, ldys, B, 0.0f, d_ws, w.group,
                               (cudaStream_t)stream, &ffn);
}

uint64_t spw_spmv_workspace_bytes(const spw_format* hdr, int B) {
    return spw_spmv_group_workspace_bytes(1, hdr, B);
}

uint64_t spw_spmv_group_workspace_bytes(int n, const spw_format* hdrs, int B) {
    if (n < 1 || n > kMaxGroup || !hdrs || B < 1 || B > 16) return 0;
    for (int l = 0; l < n; l++)
        if (check_header(&hdrs[l]) != SPW_OK) return 0;
    Plan pl;
    if (make_plan(n, hdrs, B, &pl) != SPW_OK) return 0;
    return pl.ws_bytes;
}

int spw_spmv(const spw_format* hdr, const void* d_buf, const uint16_t* d_x, int B, int ldx,
             float threshold, const uint32_t* d_act_bits, uint16_t* d_y, int ldy, void* d_ws,
             uint64_t ws_bytes, void* stream) {
    if (!hdr) return SPW_ERR_INVALID_ARG;
    return decode_group_launch(1, hdr, &d_buf, &d_x, &ldx, &d_act_bits, &d_y, &ldy, B, threshold,
                               d_ws, ws_bytes, (cudaStream_t)stream);
}

int spw_spmv_group(int n, const spw_format* hdrs, const void* const* d_bufs,
                   const uint16_t* const* d_xs, const int* ldxs, const uint32_t* const* d_act_bits,
                   uint16_t* const* d_ys, const int* ldys, int B, float threshold, void* d_ws,
                   uint64_t ws_bytes, void* stream) {
    return decode_group_launch(n, hdrs, d_bufs, d_xs, ldxs, d_act_bits, d_ys, ldys, B, threshold,
                               d_ws, ws_bytes, (cudaStream_t)stream);
}

}  // extern "C"
