// spmv.cu -- decode spMspV on CUDA cores: y_b = W_masked . x~_b for 1 <= B <= 16.
//
// Method: "Unified Static-Dynamic Pruning for Efficient LLM Inference" (abstract and
// method notes) pairs its bitmap weight format with a CUDA-core spMspV kernel that skips
// activations at run time and decodes bitmaps in shared memory; "Reduced Matrix
// Multiplication" §4.2 computes only the reduced product over the selected input columns
// (§3.1: decode is bound by reading the weight).  The kernel below is this library's
// design for B200:
//
//   * Work split: the tiles of the TCB buffer, in storage order (strip-major, then k),
//     are cut into one contiguous, equal-count range per warp of a persistent grid
//     (a multiple of the SM count).  A range covers a piece of one or two strips.
//   * Data movement: each warp runs its own S-stage pipeline in shared memory.  One lane
//     issues 1-D bulk copies (cp.async.bulk, no multicast) of a tile's 64 bitmap words,
//     its packed values, the tile's 64 activations of every batch row and, if given,
//     the caller's column-set words; a single mbarrier per stage counts the bytes.
//   * Activation skipping: after a stage lands, the warp applies the threshold rule to
//     its 64 x B activations, and a ballot gives the tile's active columns (some row's
//     entry survives and the column holds a kept weight).  Inactive columns cost nothing
//     further.
//   * Bitmap decode: lane l owns rows l and l+32 of the strip.  For an active column
//     with bitmap words (lo, hi) the lane's value sits at position
//     colstart + popc(lo & lanes_below) in the column's segment (hi rows start after
//     popc(lo) values); column starts are a warp prefix sum of popcounts.  fp16 x fp16 is
//     fused into an fp32 accumulator (fma.rn.f32.f16).
//   * Split-K combine: a warp writes its fp32 partial for each strip piece into the
//     workspace; the last contributor of a strip (counted with an atomic) sums all pieces
//     in warp order -- a fixed order, so results are deterministic -- rounds to fp16 and
//     resets the counter.  A strip with a single contributor is written directly.
#include <stdlib.h>
#include <string.h>

#include "spw_internal.cuh"

namespace spw {
namespace {

constexpr int kMaxWarpsPerCta = 8;
constexpr int kMaxGroup = 8;  // layers per grouped launch
constexpr int kDefaultWarpsPerCta = 8;
constexpr int kDefaultCtasPerSm = 2;
constexpr int kMaxStages = 4;
constexpr int kMinStages = 2;
// Per-warp header: mbarriers at 0, tileptr cache at 64, column records at 512, x~ at 1536
// (64 columns x xt_stride(B) halves).
constexpr int kTptrCacheOff = 64;
constexpr int kTptrCacheEntries = 65;
constexpr int kRecOff = 512;
constexpr int kXtOff = 1536;
constexpr int kSmemPerSm = 227 * 1024;

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
};

struct SpmvParams {
    SpmvLayer L[kMaxGroup];
    int n_layers;
    int* status;
    int n_tiles;       // all layers
    int total_warps;
    int stages;
    uint32_t stage_bytes;
    uint32_t warp_smem;
    float t;
};

__host__ __device__ constexpr int xt_stride(int B) {
    return B <= 1 ? 1 : B <= 2 ? 2 : B <= 4 ? 4 : B <= 8 ? 8 : 16;
}
__host__ __device__ constexpr uint32_t stage_vals_off(int B) { return 512u + 128u * B + 16u; }

__host__ __device__ inline long long warp_of_tile(long long t, long long total_warps,
                                                  long long n_tiles) {
    return ((t + 1) * total_warps - 1) / n_tiles;
}

// Columns decoded per group: loads for the whole group are issued before any
// multiply-add, so a warp has 2 * kGroup independent load chains in flight.
constexpr int kGroup = 4;

// Split a 32-bit word into its two fp16 halves (register halves, no shifts).
__device__ inline void split_halves(uint32_t w, uint16_t& lo, uint16_t& hi) {
    asm("mov.b32 {%0, %1}, %2;" : "=h"(lo), "=h"(hi) : "r"(w));
}

// Load x~ for G consecutive compacted columns (stride XS halves per column).
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

// G compacted active columns of one tile, branch-free: every lane loads the value at
// its rank position for both of its rows whether or not its bit is set (the position is
// always inside the stage), and a predicated fused multiply-add keeps the product only
// where the bit is set, so a value of another row (possibly Inf/NaN) never leaks in.
template <int B, int G>
__device__ inline void decode_group(const uint4* rec, const uint16_t* xt, int j, uint32_t lanebit,
                                    uint32_t ltmask, float* acc0, float* acc1) {
    uint4 r[G];
    uint16_t xv[G][B];
#pragma unroll
    for (int c = 0; c < G; c++) r[c] = rec[j + c];
    load_xg<B, G>(xt, j, xv);
    uint16_t w0[G], w1[G];
#pragma unroll
    for (int c = 0; c < G; c++) {
        w0[c] = lds_u16(r[c].z + 2u * __popc(r[c].x & ltmask));
        w1[c] = lds_u16(r[c].w + 2u * __popc(r[c].y & ltmask));
    }
#pragma unroll
    for (int c = 0; c < G; c++)
#pragma unroll
        for (int b = 0; b < B; b++) {
            acc0[b] = fma_f16_f32_if(r[c].x, lanebit, w0[c], xv[c][b], acc0[b]);
            acc1[b] = fma_f16_f32_if(r[c].y, lanebit, w1[c], xv[c][b], acc1[b]);
        }
}

__host__ __device__ constexpr uint32_t warp_header_bytes(int B) {
    return (uint32_t)((kXtOff + 64 * 2 * xt_stride(B) + 127) / 128 * 128);
}

// Position of a warp's cursor in the group's tile space: layer, tile within the layer,
// its k-tile and strip.
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

template <int B>
__global__ void __launch_bounds__(kMaxWarpsPerCta * 32, B <= 9 ? 2 : 1)
spmv_kernel(const __grid_constant__ SpmvParams p) {
    extern __shared__ __align__(1024) unsigned char smem[];
    constexpr int XS = xt_stride(B);
    constexpr uint32_t VOFF = stage_vals_off(B);
    constexpr uint32_t HDR = warp_header_bytes(B);
    const int warps_per_cta = blockDim.x >> 5;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    unsigned char* wsm = smem + (size_t)warp * p.warp_smem;
    const int gw = blockIdx.x * warps_per_cta + warp;
    // PW <= T (host side), so every working warp's range is nonempty and the warps
    // touching a strip are consecutive.
    const int T = p.n_tiles, PW = p.total_warps;
    if (gw >= PW) return;  // warps are independent: no block-wide barrier follows
    const int t_begin = (int)((long long)gw * T / PW);
    const int t_end = (int)((long long)(gw + 1) * T / PW);
    const int ntiles = t_end - t_begin;
    const int S = p.stages;

    uint64_t* mbar = (uint64_t*)wsm;
    uint32_t* tpc = (uint32_t*)(wsm + kTptrCacheOff);
    uint4* rec = (uint4*)(wsm + kRecOff);
    uint16_t* xt = (uint16_t*)(wsm + kXtOff);
    const uint32_t wsm_s = smem_u32(wsm);

    if (lane == 0) {
        for (int s = 0; s < S; s++) mbar_init(smem_u32(&mbar[s]), 1);
        fence_mbar_init();
    }
    __syncwarp();

    const uint64_t evict_first = policy_evict_first();
    int tpc_layer = -1, tpc_base = 0;  // tileptr cache: layer and first local tile
    Cursor ic = cursor_at(p, t_begin);  // next tile to issue
    // Copies for one tile.  Weights (bitmaps, values) may be fetched before the previous
    // kernel on the stream has finished; activations and column-set words only after
    // pdl_wait(), so the prologue issues them separately (issue_x).  The stage's expected
    // byte count always includes them, so the stage cannot complete early.
    auto issue_x = [&](int slot, const Cursor& c) {  // lane 0 only
        const SpmvLayer& L = p.L[c.l];
        const uint32_t bar = smem_u32(&mbar[slot]);
        const uint32_t st = wsm_s + HDR + (uint32_t)slot * p.stage_bytes;
        const int kcols = min(kTileCols, L.K - c.kt * kTileCols);
        const uint32_t xbytes = (uint32_t)((kcols * 2 + 15) & ~15);
        const uint16_t* xsrc = L.x + (size_t)c.kt * kTileCols;
#pragma unroll
        for (int b = 0; b < B; b++) bulk_g2s(st + 512u + 128u * b, xsrc + (size_t)b * L.ldx, xbytes, bar);
        if (L.act_bits) bulk_g2s(st + 512u + 128u * B, L.act_bits + ((c.kt * 2) & ~3), 16u, bar);
    };
    auto issue_next = [&](int slot, bool with_x) {  // warp-collective; lane 0 issues
        const SpmvLayer& L = p.L[ic.l];
        if (ic.l != tpc_layer || ic.t + 1 - tpc_base >= kTptrCacheEntries) {  // refill cache
            for (int j = lane; j < kTptrCacheEntries; j += 32)
                if (ic.t + j <= L.n_tiles) tpc[j] = __ldg(L.tileptr + ic.t + j);
            __syncwarp();
            tpc_layer = ic.l;
            tpc_base = ic.t;
        }
        if (lane == 0) {
            const uint32_t bar = smem_u32(&mbar[slot]);
            const uint32_t st = wsm_s + HDR + (uint32_t)slot * p.stage_bytes;
            const uint32_t u0 = tpc[ic.t - tpc_base], u1 = tpc[ic.t + 1 - tpc_base];
            uint32_t vbytes = (u1 - u0) * 16u;
            if (vbytes + VOFF + 16u > p.stage_bytes) {  // tile larger than the header allows
                raise_status(p.status, SPW_ERR_FORMAT);
                vbytes = 0;
            }
            const int kcols = min(kTileCols, L.K - ic.kt * kTileCols);
            const uint32_t xbytes = (uint32_t)((kcols * 2 + 15) & ~15);
            const uint32_t total = 512u + vbytes + (uint32_t)B * xbytes + (L.act_bits ? 16u : 0u);
            fence_proxy_async_smem();
            mbar_arrive_expect_tx(bar, total);
            bulk_g2s_hint(st, L.bitmaps + (size_t)ic.t * kTileCols, 512u, bar, evict_first);
            if (vbytes) bulk_g2s_hint(st + VOFF, L.values + (size_t)u0 * 8, vbytes, bar, evict_first);
            if (with_x) issue_x(slot, ic);
        }
        cursor_next(p, ic);
    };

    // Prologue: weights of the first S - 1 tiles, then (once the previous kernel on the
    // stream is complete) their activations.
    const int n_pro = min(S - 1, ntiles);
    for (int i = 0; i < n_pro; i++) issue_next(i, false);
    pdl_wait();
    if (lane == 0) {
        Cursor c = cursor_at(p, t_begin);
        for (int i = 0; i < n_pro; i++) {
            issue_x(i, c);
            cursor_next(p, c);
        }
    }
    pdl_launch_dependents();

    const uint32_t lanebit = 1u << lane, ltmask = lanebit - 1u;
    float acc0[B], acc1[B];
#pragma unroll
    for (int b = 0; b < B; b++) acc0[b] = acc1[b] = 0.0f;
    Cursor cc = cursor_at(p, t_begin);  // tile being consumed
    int slot = 0;
    uint32_t phase = 0;

    for (int i = 0; i < ntiles; i++) {
        if (i + S - 1 < ntiles) issue_next(slot == 0 ? S - 1 : slot - 1, true);
        if (!mbar_wait(smem_u32(&mbar[slot]), phase)) {
            raise_status(p.status, SPW_ERR_TIMEOUT);
            for (int j = i + 1; j < ntiles && j < i + S; j++)  // drain (bounded)
                (void)mbar_wait(smem_u32(&mbar[j % S]), (uint32_t)((j / S) & 1));
            return;
        }
        const SpmvLayer& L = p.L[cc.l];
        const unsigned char* st = wsm + HDR + (uint32_t)slot * p.stage_bytes;
        const uint64_t* bm = (const uint64_t*)st;
        const uint16_t* xr = (const uint16_t*)(st + 512);

        // Activations of the lane's two columns, threshold rule, column set.
        const int k0 = cc.kt * kTileCols + lane;
        bool ok0 = k0 < L.K, ok1 = k0 + 32 < L.K;
        if (L.act_bits) {
            const uint32_t* aw = (const uint32_t*)(st + 512 + 128 * B);
            const int w = (cc.kt * 2) & 3;
            ok0 = ok0 && ((aw[w] >> lane) & 1u);
            ok1 = ok1 && ((aw[w + 1] >> lane) & 1u);
        }
        uint16_t xa[B], xb[B];
        bool any0 = false, any1 = false;
#pragma unroll
        for (int b = 0; b < B; b++) {
            const uint16_t a0 = xr[b * 64 + lane], a1 = xr[b * 64 + lane + 32];
            const bool p0 = ok0 && passes_threshold(a0, p.t);
            const bool p1 = ok1 && passes_threshold(a1, p.t);
            xa[b] = p0 ? a0 : (uint16_t)0;
            xb[b] = p1 ? a1 : (uint16_t)0;
            any0 |= p0;
            any1 |= p1;
        }
        const uint64_t w0 = bm[lane], w1 = bm[lane + 32];
        any0 = any0 && w0 != 0;
        any1 = any1 && w1 != 0;
        const uint32_t act_lo = __ballot_sync(0xffffffffu, any0);
        const uint32_t act_hi = __ballot_sync(0xffffffffu, any1);
        const int n_act = __popc(act_lo) + __popc(act_hi);

        if (n_act > 0) {
            // Column starts within the tile's values (all 64 columns, in column order):
            // one warp scan of both counts packed as 16-bit halves (sums stay <= 2048).
            const int c0 = __popcll(w0), c1 = __popcll(w1);
            const int sp = warp_inclusive_scan(c0 | (c1 << 16), lane);
            const int tot0 = __shfl_sync(0xffffffffu, sp, 31) & 0xffff;
            const int s0 = sp & 0xffff, s1 = sp >> 16;
            const uint32_t vb = wsm_s + HDR + (uint32_t)slot * p.stage_bytes + VOFF;
            const uint32_t a0 = vb + 2u * (uint32_t)(s0 - c0);
            const uint32_t a1 = vb + 2u * (uint32_t)(tot0 + s1 - c1);
            // Records {lo bits, hi bits, address of the lo rows' first value, address of
            // the hi rows' first value}.  When every column is active they sit at their
            // column positions and the decode is fully unrolled; otherwise the active
            // columns are compacted and padded with empty records to a group multiple.
            const bool all = B <= 4 && n_act == 64;  // wider batches keep the loop (registers)
            const int pos0 = all ? lane : __popc(act_lo & ltmask);
            const int pos1 = all ? lane + 32 : __popc(act_lo) + __popc(act_hi & ltmask);
            if (any0) {
                rec[pos0] = make_uint4((uint32_t)w0, (uint32_t)(w0 >> 32), a0,
                                       a0 + 2u * __popc((uint32_t)w0));
#pragma unroll
                for (int b = 0; b < B; b++) xt[pos0 * XS + b] = xa[b];
            }
            if (any1) {
                rec[pos1] = make_uint4((uint32_t)w1, (uint32_t)(w1 >> 32), a1,
                                       a1 + 2u * __popc((uint32_t)w1));
#pragma unroll
                for (int b = 0; b < B; b++) xt[pos1 * XS + b] = xb[b];
            }
            if constexpr (B <= 4) {
                if (all) {
                    __syncwarp();
#pragma unroll
                    for (int j = 0; j < 64; j += kGroup)
                        decode_group<B, kGroup>(rec, xt, j, lanebit, ltmask, acc0, acc1);
                }
            }
            if (!all) {
                const int n_pad = (n_act + kGroup - 1) & ~(kGroup - 1);
                if (lane < n_pad - n_act) {
                    rec[n_act + lane] = make_uint4(0u, 0u, vb, vb);
#pragma unroll
                    for (int b = 0; b < B; b++) xt[(n_act + lane) * XS + b] = 0;
                }
                __syncwarp();
                for (int j = 0; j < n_pad; j += kGroup)
                    decode_group<B, kGroup>(rec, xt, j, lanebit, ltmask, acc0, acc1);
            }
        }
        __syncwarp();
        if (++slot == S) {
            slot = 0;
            phase ^= 1u;
        }

        // End of this warp's piece of strip s: write or combine the partial sums.
        const bool strip_end = (cc.kt == L.n_ktiles - 1) || (i + 1 == ntiles);
        const int s = cc.s;
        const int nk = L.n_ktiles;
        const int first = L.tile_begin + s * nk;
        cursor_next(p, cc);
        if (!strip_end) continue;
        const int g_first = (int)warp_of_tile(first, PW, T);
        const int g_last = (int)warp_of_tile((long long)first + nk - 1, PW, T);
        const int count = g_last - g_first + 1;
        const int r0 = s * kStripRows + lane, r1 = r0 + 32;
        if (count == 1) {
#pragma unroll
            for (int b = 0; b < B; b++) {
                if (r0 < L.N) L.y[(size_t)b * L.ldy + r0] = __half_as_ushort(__float2half_rn(acc0[b]));
                if (r1 < L.N) L.y[(size_t)b * L.ldy + r1] = __half_as_ushort(__float2half_rn(acc1[b]));
            }
        } else {
            // Publish this piece: store the partials, then one release atomic per warp.
            const int idx = gw - g_first;
            float* mine = L.partials + ((size_t)s * L.maxc + idx) * B * 64;
#pragma unroll
            for (int b = 0; b < B; b++) {
                mine[b * 64 + lane] = acc0[b];
                mine[b * 64 + lane + 32] = acc1[b];
            }
            __syncwarp();
            uint32_t old = 0;
            if (lane == 0) old = atom_add_release_gpu(&L.counters[s], 1u);
            old = __shfl_sync(0xffffffffu, old, 0);
            if ((int)old == count - 1) {
                // Last contributor: sum every piece in contributor order (deterministic).
                // Lane l owns rows 2l and 2l+1; eight pieces' loads are in flight at once.
                __threadfence();
                const float* base = L.partials + (size_t)s * L.maxc * B * 64;
                const int row = s * kStripRows + 2 * lane;
#pragma unroll 1
                for (int b = 0; b < B; b++) {
                    float sx = 0.0f, sy = 0.0f;
#pragma unroll 1
                    for (int j0 = 0; j0 < count; j0 += 8) {
                        float2 v[8];
#pragma unroll
                        for (int u = 0; u < 8; u++)
                            v[u] = (j0 + u < count)
                                       ? __ldcg((const float2*)(base + ((size_t)(j0 + u) * B + b) * 64) + lane)
                                       : make_float2(0.0f, 0.0f);
#pragma unroll
                        for (int u = 0; u < 8; u++) {
                            sx += v[u].x;
                            sy += v[u].y;
                        }
                    }
                    if (row < L.N) L.y[(size_t)b * L.ldy + row] = __half_as_ushort(__float2half_rn(sx));
                    if (row + 1 < L.N)
                        L.y[(size_t)b * L.ldy + row + 1] = __half_as_ushort(__float2half_rn(sy));
                }
                if (lane == 0) L.counters[s] = 0u;
            }
        }
#pragma unroll
        for (int b = 0; b < B; b++) acc0[b] = acc1[b] = 0.0f;
    }
}

struct Plan {
    int grid, warps, ctas_per_sm, stages;
    uint32_t stage_bytes, warp_smem;
    size_t smem;
    long long n_tiles, total_warps;
    int maxc[kMaxGroup];
    uint64_t ws_off[kMaxGroup];       // each layer's workspace section (counters first)
    uint64_t ws_counters[kMaxGroup];  // bytes of that section's counter block
    uint64_t ws_bytes;
};

// Occupancy knobs: warps per CTA and CTAs per SM.  SPW_SPMV_WARPS and
// SPW_SPMV_CTAS_PER_SM override the defaults (a tuning aid; both change only the launch
// shape, never the work done).
int env_int(const char* name, int dflt, int lo, int hi) {
    const char* v = getenv(name);
    if (!v || !*v) return dflt;
    const int x = atoi(v);
    return (x < lo || x > hi) ? dflt : x;
}

// Launch plan for a group of n layers decoded in one launch (n = 1 for spw_spmv).
int make_plan(int n, const spw_format* h, int B, Plan* pl) {
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
    // stage: bitmaps, x rows, column-set words, values, and 16 bytes of slack for the
    // branch-free loads one past a column's last value
    pl->stage_bytes = (uint32_t)round_up_u64(stage_vals_off(B) + 16ull * max_units + 16, 128);
    // Preferred launch shape first; fall back to fewer warps per SM when the stages of
    // wide batches or dense formats do not fit two per warp.
    const int want_warps = env_int("SPW_SPMV_WARPS", kDefaultWarpsPerCta, 1, kMaxWarpsPerCta);
    const int want_ctas = env_int("SPW_SPMV_CTAS_PER_SM", kDefaultCtasPerSm, 1, 32);
    const int shapes[][2] = {{want_warps, want_ctas}, {4, 2}, {4, 1}, {2, 1}, {1, 1}};
    int stages = 0;
    for (const auto& sh : shapes) {
        pl->warps = sh[0];
        pl->ctas_per_sm = sh[1];
        const long long budget = kSmemPerSm / pl->ctas_per_sm - 1024;
        const long long per_warp = budget / pl->warps - warp_header_bytes(B);
        stages = per_warp > 0 ? (int)(per_warp / pl->stage_bytes) : 0;
        if (stages >= kMinStages) break;
    }
    if (stages < kMinStages) return SPW_ERR_UNSUPPORTED;
    if (stages > kMaxStages) stages = kMaxStages;
    pl->grid = sms * pl->ctas_per_sm;
    pl->total_warps = (long long)pl->grid * pl->warps;
    if (pl->total_warps > T) pl->total_warps = T;  // one tile or more per working warp
    pl->stages = stages;
    pl->warp_smem = warp_header_bytes(B) + (uint32_t)stages * pl->stage_bytes;
    pl->smem = (size_t)pl->warps * pl->warp_smem;
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
    static size_t attr_smem[64];
    int dev = 0;
    SPW_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= 64) return SPW_ERR_CUDA;
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
    cfg.blockDim = dim3(pl.warps * 32);
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
int decode_group_launch(int n, const spw_format* hdrs, const void* const* bufs,
                        const uint16_t* const* xs, const int* ldxs,
                        const uint32_t* const* act_bits, uint16_t* const* ys, const int* ldys,
                        int B, float threshold, void* d_ws, uint64_t ws_bytes, cudaStream_t s) {
    if (n < 1 || n > kMaxGroup || !hdrs || !bufs || !xs || !ldxs || !ys || !ldys)
        return SPW_ERR_INVALID_ARG;
    if (!d_ws || B < 1 || B > 16) return SPW_ERR_INVALID_ARG;
    if (!(threshold >= 0.0f) || isinf(threshold)) return SPW_ERR_INVALID_ARG;
    for (int l = 0; l < n; l++) {
        const int rc = check_header(&hdrs[l]);
        if (rc != SPW_OK) return rc;
        if (!bufs[l] || !xs[l] || !ys[l]) return SPW_ERR_INVALID_ARG;
        if (!ld_ok(ldxs[l], (int)hdrs[l].K, B) || ldys[l] < (int)hdrs[l].N) return SPW_ERR_INVALID_ARG;
        const uint32_t* ab = act_bits ? act_bits[l] : nullptr;
        if (!aligned16(bufs[l]) || !aligned16(xs[l]) || !aligned16(ys[l]) || !aligned16(ab))
            return SPW_ERR_ALIGNMENT;
    }
    if (!aligned16(d_ws)) return SPW_ERR_ALIGNMENT;
    Plan pl;
    int rc = make_plan(n, hdrs, B, &pl);
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

}  // namespace
}  // namespace spw

using namespace spw;

extern "C" {

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
