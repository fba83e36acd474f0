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

#include "spw_internal.cuh"

namespace spw {
namespace {

constexpr int kMaxWarpsPerCta = 8;
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

struct SpmvParams {
    const uint64_t* bitmaps;
    const uint32_t* tileptr;
    const uint16_t* values;
    const uint16_t* x;
    const uint32_t* act_bits;
    uint16_t* y;
    uint32_t* counters;
    float* partials;
    int* status;
    int n_tiles;
    int total_warps;
    int N, K, ldx, ldy;
    int n_ktiles;
    int maxc;
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

// Load x~ for eight consecutive compacted columns (stride XS halves per column).
template <int B>
__device__ inline void load_x8(const uint16_t* xt, int j, uint16_t (&xv)[8][B]) {
    constexpr int XS = xt_stride(B);
    constexpr int WORDS = 8 * XS / 2;  // 32-bit words covering 8 columns
    uint32_t w[WORDS];
    const uint4* p = (const uint4*)(xt + j * XS);
#pragma unroll
    for (int q = 0; q < WORDS / 4; q++) {
        const uint4 v = p[q];
        w[4 * q] = v.x;
        w[4 * q + 1] = v.y;
        w[4 * q + 2] = v.z;
        w[4 * q + 3] = v.w;
    }
#pragma unroll
    for (int c = 0; c < 8; c++)
#pragma unroll
        for (int b = 0; b < B; b++) {
            const int h = c * XS + b;  // half index
            xv[c][b] = (uint16_t)(w[h >> 1] >> (16 * (h & 1)));
        }
}

// Eight compacted active columns of one tile, branch-free: every lane loads the value at
// its rank position for both of its rows whether or not its bit is set (the position is
// always inside the stage), and a predicated fused multiply-add keeps the product only
// where the bit is set, so a value of another row (possibly Inf/NaN) never leaks in.
template <int B>
__device__ inline void decode8(const uint4* rec, const uint16_t* xt, int j, uint32_t lanebit,
                               uint32_t ltmask, float* acc0, float* acc1) {
    uint4 r[8];
    uint16_t xv[8][B];
#pragma unroll
    for (int c = 0; c < 8; c++) r[c] = rec[j + c];
    load_x8<B>(xt, j, xv);
    uint16_t w0[8], w1[8];
#pragma unroll
    for (int c = 0; c < 8; c++) {
        w0[c] = lds_u16(r[c].z + 2u * __popc(r[c].x & ltmask));
        w1[c] = lds_u16(r[c].w + 2u * __popc(r[c].y & ltmask));
    }
#pragma unroll
    for (int c = 0; c < 8; c++)
#pragma unroll
        for (int b = 0; b < B; b++) {
            acc0[b] = fma_f16_f32_if(r[c].x, lanebit, w0[c], xv[c][b], acc0[b]);
            acc1[b] = fma_f16_f32_if(r[c].y, lanebit, w1[c], xv[c][b], acc1[b]);
        }
}

__host__ __device__ constexpr uint32_t warp_header_bytes(int B) {
    return (uint32_t)((kXtOff + 64 * 2 * xt_stride(B) + 127) / 128 * 128);
}

template <int B>
__global__ void __launch_bounds__(kMaxWarpsPerCta * 32)
spmv_kernel(const SpmvParams p) {
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
    const int nk = p.n_ktiles;

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
    int tpc_base = -(1 << 30);
    // Tile coordinates of the next tile to issue, advanced incrementally.
    int issue_t = t_begin;
    int issue_kt = t_begin % nk;
    // Copies for the next tile.  Weights (bitmaps, values) may be fetched before the
    // previous kernel has finished; activations and column-set words only after
    // pdl_wait(), so the prologue issues them separately (issue_x).  The stage's
    // expected byte count always includes them, so the stage cannot complete early.
    auto issue_x = [&](int slot, int kt_of_tile) {  // lane 0 only
        const uint32_t bar = smem_u32(&mbar[slot]);
        const uint32_t st = wsm_s + HDR + (uint32_t)slot * p.stage_bytes;
        const int kcols = min(kTileCols, p.K - kt_of_tile * kTileCols);
        const uint32_t xbytes = (uint32_t)((kcols * 2 + 15) & ~15);
        const uint16_t* xsrc = p.x + (size_t)kt_of_tile * kTileCols;
#pragma unroll
        for (int b = 0; b < B; b++) bulk_g2s(st + 512u + 128u * b, xsrc + (size_t)b * p.ldx, xbytes, bar);
        if (p.act_bits)
            bulk_g2s(st + 512u + 128u * B, p.act_bits + ((kt_of_tile * 2) & ~3), 16u, bar);
    };
    auto issue_next = [&](int slot, bool with_x) {  // warp-collective; lane 0 issues
        if (issue_t + 1 - tpc_base >= kTptrCacheEntries) {  // refill the tileptr cache
            for (int j = lane; j < kTptrCacheEntries; j += 32)
                if (issue_t + j <= T) tpc[j] = __ldg(p.tileptr + issue_t + j);
            __syncwarp();
            tpc_base = issue_t;
        }
        if (lane == 0) {
            const uint32_t bar = smem_u32(&mbar[slot]);
            const uint32_t st = wsm_s + HDR + (uint32_t)slot * p.stage_bytes;
            const uint32_t u0 = tpc[issue_t - tpc_base], u1 = tpc[issue_t + 1 - tpc_base];
            uint32_t vbytes = (u1 - u0) * 16u;
            if (vbytes + VOFF + 16u > p.stage_bytes) {  // tile larger than the header allows
                raise_status(p.status, SPW_ERR_FORMAT);
                vbytes = 0;
            }
            const int kcols = min(kTileCols, p.K - issue_kt * kTileCols);
            const uint32_t xbytes = (uint32_t)((kcols * 2 + 15) & ~15);
            const uint32_t total = 512u + vbytes + (uint32_t)B * xbytes + (p.act_bits ? 16u : 0u);
            fence_proxy_async_smem();
            mbar_arrive_expect_tx(bar, total);
            bulk_g2s_hint(st, p.bitmaps + (size_t)issue_t * kTileCols, 512u, bar, evict_first);
            if (vbytes)
                bulk_g2s_hint(st + VOFF, p.values + (size_t)u0 * 8, vbytes, bar, evict_first);
            if (with_x) issue_x(slot, issue_kt);
        }
        issue_t++;
        if (++issue_kt == nk) issue_kt = 0;
    };

    // Prologue: weights of the first S - 1 tiles, then (once the previous kernel on the
    // stream is complete) their activations.
    const int n_pro = min(S - 1, ntiles);
    for (int i = 0; i < n_pro; i++) issue_next(i, false);
    pdl_wait();
    if (lane == 0)
        for (int i = 0; i < n_pro; i++) issue_x(i, (t_begin + i) % nk);
    pdl_launch_dependents();

    const uint32_t lanebit = 1u << lane, ltmask = lanebit - 1u;
    float acc0[B], acc1[B];
#pragma unroll
    for (int b = 0; b < B; b++) acc0[b] = acc1[b] = 0.0f;
    int s_cur = t_begin / nk;
    int kt = t_begin % nk;
    int slot = 0;
    uint32_t phase = 0;

    for (int i = 0; i < ntiles; i++) {
        const int t = t_begin + i;
        if (i + S - 1 < ntiles) issue_next(slot == 0 ? S - 1 : slot - 1, true);
        if (!mbar_wait(smem_u32(&mbar[slot]), phase)) {
            raise_status(p.status, SPW_ERR_TIMEOUT);
            for (int j = i + 1; j < ntiles && j < i + S; j++)  // drain (bounded)
                (void)mbar_wait(smem_u32(&mbar[j % S]), (uint32_t)((j / S) & 1));
            return;
        }
        const unsigned char* st = wsm + HDR + (uint32_t)slot * p.stage_bytes;
        const uint64_t* bm = (const uint64_t*)st;
        const uint16_t* xr = (const uint16_t*)(st + 512);

        // Activations of the lane's two columns, threshold rule, column set.
        const int k0 = kt * kTileCols + lane;
        bool ok0 = k0 < p.K, ok1 = k0 + 32 < p.K;
        if (p.act_bits) {
            const uint32_t* aw = (const uint32_t*)(st + 512 + 128 * B);
            const int w = (kt * 2) & 3;
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
            // Column starts within the tile's values (all 64 columns, in column order).
            const int c0 = __popcll(w0), c1 = __popcll(w1);
            const int s0 = warp_inclusive_scan(c0, lane);
            const int tot0 = __shfl_sync(0xffffffffu, s0, 31);
            const int s1 = warp_inclusive_scan(c1, lane);
            const uint32_t vb = wsm_s + HDR + (uint32_t)slot * p.stage_bytes + VOFF;
            const uint32_t a0 = vb + 2u * (uint32_t)(s0 - c0);
            const uint32_t a1 = vb + 2u * (uint32_t)(tot0 + s1 - c1);
            // Compacted records of the active columns, padded with empty ones to a
            // multiple of 8: {lo bits, hi bits, address of the lo rows' first value,
            // address of the hi rows' first value}.
            const int pos0 = __popc(act_lo & ltmask);
            const int pos1 = __popc(act_lo) + __popc(act_hi & ltmask);
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
            const int n_pad = (n_act + 7) & ~7;
            if (lane < n_pad - n_act) {
                rec[n_act + lane] = make_uint4(0u, 0u, vb, vb);
#pragma unroll
                for (int b = 0; b < B; b++) xt[(n_act + lane) * XS + b] = 0;
            }
            __syncwarp();
            for (int j = 0; j < n_pad; j += 8) decode8<B>(rec, xt, j, lanebit, ltmask, acc0, acc1);
        }
        __syncwarp();
        if (++slot == S) {
            slot = 0;
            phase ^= 1u;
        }

        // End of this warp's piece of strip s: write or combine the partial sums.
        const bool strip_end = (kt == nk - 1) || (t + 1 == t_end);
        const int s = s_cur;
        if (++kt == nk) {
            kt = 0;
            s_cur++;
        }
        if (!strip_end) continue;
        const int g_first = (int)warp_of_tile((long long)s * nk, PW, T);
        const int g_last = (int)warp_of_tile((long long)(s + 1) * nk - 1, PW, T);
        const int count = g_last - g_first + 1;
        const int r0 = s * kStripRows + lane, r1 = r0 + 32;
        if (count == 1) {
#pragma unroll
            for (int b = 0; b < B; b++) {
                if (r0 < p.N) p.y[(size_t)b * p.ldy + r0] = __half_as_ushort(__float2half_rn(acc0[b]));
                if (r1 < p.N) p.y[(size_t)b * p.ldy + r1] = __half_as_ushort(__float2half_rn(acc1[b]));
            }
        } else {
            // Publish this piece: store the partials, then one release atomic per warp.
            const int idx = gw - g_first;
            float* mine = p.partials + ((size_t)s * p.maxc + idx) * B * 64;
#pragma unroll
            for (int b = 0; b < B; b++) {
                mine[b * 64 + lane] = acc0[b];
                mine[b * 64 + lane + 32] = acc1[b];
            }
            __syncwarp();
            uint32_t old = 0;
            if (lane == 0) old = atom_add_release_gpu(&p.counters[s], 1u);
            old = __shfl_sync(0xffffffffu, old, 0);
            if ((int)old == count - 1) {
                // Last contributor: sum every piece in contributor order (deterministic).
                // Lane l owns rows 2l and 2l+1; eight pieces' loads are in flight at once.
                __threadfence();
                const float* base = p.partials + (size_t)s * p.maxc * B * 64;
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
                    if (row < p.N) p.y[(size_t)b * p.ldy + row] = __half_as_ushort(__float2half_rn(sx));
                    if (row + 1 < p.N)
                        p.y[(size_t)b * p.ldy + row + 1] = __half_as_ushort(__float2half_rn(sy));
                }
                if (lane == 0) p.counters[s] = 0u;
            }
        }
#pragma unroll
        for (int b = 0; b < B; b++) acc0[b] = acc1[b] = 0.0f;
    }
}

struct Plan {
    int grid, warps, ctas_per_sm, stages, maxc;
    uint32_t stage_bytes, warp_smem;
    size_t smem;
    long long total_warps;
    uint64_t ws_counters, ws_bytes;
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

int make_plan(const spw_format* h, int B, Plan* pl) {
    const int sms = device_sm_count();
    if (sms <= 0) return SPW_ERR_CUDA;
    const long long T = (long long)h->n_strips * h->n_ktiles;
    // stage: bitmaps, x rows, column-set words, values, and 16 bytes of slack for the
    // branch-free loads one past a column's last value
    pl->stage_bytes =
        (uint32_t)round_up_u64(stage_vals_off(B) + 16ull * h->max_tile_units + 16, 128);
    // Preferred launch shape first; fall back to fewer warps per SM when the stages of
    // wide batches or dense formats do not fit two per warp.
    const int want_warps = env_int("SPW_SPMV_WARPS", kDefaultWarpsPerCta, 1, kMaxWarpsPerCta);
    const int want_ctas = env_int("SPW_SPMV_CTAS_PER_SM", kDefaultCtasPerSm, 1, 8);
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
    int maxc = 1;
    for (long long s = 0; s < h->n_strips; s++) {
        const long long c = warp_of_tile((s + 1) * h->n_ktiles - 1, pl->total_warps, T) -
                            warp_of_tile(s * h->n_ktiles, pl->total_warps, T) + 1;
        if (c > maxc) maxc = (int)c;
    }
    pl->maxc = maxc;
    pl->ws_counters = round_up_u64(4ull * h->n_strips, 256);
    pl->ws_bytes = pl->ws_counters + (uint64_t)h->n_strips * maxc * B * 64 * sizeof(float);
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

}  // namespace
}  // namespace spw

using namespace spw;

extern "C" {

uint64_t spw_spmv_workspace_bytes(const spw_format* hdr, int B) {
    if (check_header(hdr) != SPW_OK || B < 1 || B > 16) return 0;
    Plan pl;
    if (make_plan(hdr, B, &pl) != SPW_OK) return 0;
    return pl.ws_bytes;
}

int spw_spmv(const spw_format* hdr, const void* d_buf, const uint16_t* d_x, int B, int ldx,
             float threshold, const uint32_t* d_act_bits, uint16_t* d_y, int ldy, void* d_ws,
             uint64_t ws_bytes, void* stream) {
    int rc = check_header(hdr);
    if (rc != SPW_OK) return rc;
    if (!d_buf || !d_x || !d_y || !d_ws || B < 1 || B > 16) return SPW_ERR_INVALID_ARG;
    if (!(threshold >= 0.0f) || isinf(threshold)) return SPW_ERR_INVALID_ARG;
    if (!ld_ok(ldx, (int)hdr->K, B) || ldy < (int)hdr->N) return SPW_ERR_INVALID_ARG;
    if (!aligned16(d_buf) || !aligned16(d_x) || !aligned16(d_y) || !aligned16(d_ws) ||
        !aligned16(d_act_bits))
        return SPW_ERR_ALIGNMENT;
    Plan pl;
    rc = make_plan(hdr, B, &pl);
    if (rc != SPW_OK) return rc;
    if (ws_bytes < pl.ws_bytes) return SPW_ERR_BUFFER_TOO_SMALL;
    int* status = device_status_ptr();
    if (!status) return SPW_ERR_CUDA;
    const uint8_t* buf = (const uint8_t*)d_buf;
    SpmvParams prm;
    prm.bitmaps = (const uint64_t*)(buf + hdr->off_bitmaps);
    prm.tileptr = (const uint32_t*)(buf + hdr->off_tileptr);
    prm.values = (const uint16_t*)(buf + hdr->off_values);
    prm.x = d_x;
    prm.act_bits = d_act_bits;
    prm.y = d_y;
    prm.counters = (uint32_t*)d_ws;
    prm.partials = (float*)((uint8_t*)d_ws + pl.ws_counters);
    prm.status = status;
    if ((long long)hdr->n_strips * hdr->n_ktiles > 0x7fffffffll) return SPW_ERR_UNSUPPORTED;
    prm.n_tiles = (int)((long long)hdr->n_strips * hdr->n_ktiles);
    prm.total_warps = (int)pl.total_warps;
    prm.N = (int)hdr->N;
    prm.K = (int)hdr->K;
    prm.ldx = ldx;
    prm.ldy = ldy;
    prm.n_ktiles = (int)hdr->n_ktiles;
    prm.maxc = pl.maxc;
    prm.stages = pl.stages;
    prm.stage_bytes = pl.stage_bytes;
    prm.warp_smem = pl.warp_smem;
    prm.t = threshold;
    cudaStream_t s = (cudaStream_t)stream;
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

}  // extern "C"
