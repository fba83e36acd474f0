// spmm.cu -- prefill SpMM on tcgen05 tensor cores: Y = X . W_masked^T.
//
// Method: "Unified Static-Dynamic Pruning for Efficient LLM Inference" (abstract) pairs
// its bitmap format with a Tensor-Core SpMM for prefill.  Dense tensor cores take only
// 2:4 structured sparsity ("Accelerating LLM GPU inference with moderately unstructured
// sparse weight matrices", §1, challenge 1), so unstructured tiles are decoded to dense
// in shared memory and fed to dense MMA; the weight crosses HBM compressed.
//
// This library's design for B200 (one CTA per SM, one 256 x 256 output tile per CTA):
//   * Y tile = 256 tokens (two M = 128 accumulators, 2 x 256 fp32 TMEM columns = all 512)
//     by 256 weight rows (four 64-row TCB strips), K stepped by 64 (one TCB k-tile).
//   * warp 0 (producer): TMA loads the X tile (256 x 64 fp16, 128-byte swizzle, no
//     multicast) and 1-D bulk copies the four TCB tiles (bitmaps + packed values).
//   * warp 1 (MMA): allocates TMEM; one thread issues tcgen05.mma.kind::f16 (A = X,
//     B = decoded W, both K-major 128B-swizzled shared memory) and commits stage releases.
//   * warps 2..9 (decoders, then epilogue): each owns one strip and 32 of its 64 columns;
//     lane l produces rows l and l+32: the value of a kept weight sits at
//     colstart + popc(bitmap & lanes_below); dense rows are written as 16-byte chunks in
//     the swizzled layout the MMA reads.  After the K loop the same warps read the fp32
//     accumulators (tcgen05.ld), round to fp16 and store Y.
//   * Every mbarrier wait is bounded and also polls a CTA-wide abort flag; on a timeout
//     the kernel raises SPW_ERR_TIMEOUT, drains outstanding copies and MMAs (bounded),
//     frees TMEM and returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "spw_internal.cuh"

namespace spw {
namespace {

constexpr int kBM = 256;                // tokens per CTA tile (two M = 128 MMAs)
constexpr int kBN = 256;                // weight rows per CTA tile (four strips)
constexpr int kBK = 64;                 // one TCB k-tile
constexpr int kStrips = kBN / kStripRows;
constexpr int kThreads = 320;           // 10 warps
constexpr int kDecoderWarps = 8;
constexpr uint32_t kXStageBytes = kBM * kBK * 2;  // 32 KB
constexpr uint32_t kWStageBytes = kBN * kBK * 2;  // 32 KB
constexpr int kWStages = 2;
constexpr int kSmemLimit = 227 * 1024;
constexpr uint32_t kTmemCols = 512;

struct SpmmParams {
    const uint64_t* bitmaps;
    const uint32_t* tileptr;
    const uint16_t* values;
    uint16_t* Y;
    int* status;
    int M, N, K, ldy;
    int n_strips, n_ktiles;
    int sx, sr;                 // X and raw-tile stage counts
    uint32_t raw_stage_bytes;   // 2048 + 4 * val_slot
    uint32_t val_slot;          // bytes per strip's values slot (incl. 16 bytes of slack)
    uint32_t off_w, off_raw, off_rec, off_tptr, off_bar;  // dynamic smem offsets
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
__device__ inline bool wait_or_abort(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long start = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (*abort_flag) return false;
        if (clock64() - start > kWaitLimitCycles) return false;
    }
    return true;
}

__device__ inline void flag_abort(volatile int* abort_flag, int* status) {
    *abort_flag = 1;
    raise_status(status, SPW_ERR_TIMEOUT);
}

__device__ inline uint32_t pack2(uint16_t lo, uint16_t hi) {
    return (uint32_t)lo | ((uint32_t)hi << 16);
}

__global__ void __launch_bounds__(kThreads, 1)
spmm_kernel(const __grid_constant__ CUtensorMap tmap_x, const SpmmParams p) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    // 1024-byte alignment for the swizzled operand tiles
    unsigned char* smem = (unsigned char*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m0 = blockIdx.x * kBM;
    const int n0 = blockIdx.y * kBN;
    const int s0 = n0 / kStripRows;
    const int nk = p.n_ktiles;
    const int SX = p.sx, SR = p.sr;

    uint64_t* bars = (uint64_t*)(smem + p.off_bar);
    uint64_t* x_full = bars;
    uint64_t* x_empty = x_full + SX;
    uint64_t* r_full = x_empty + SX;
    uint64_t* r_empty = r_full + SR;
    uint64_t* w_full = r_empty + SR;
    uint64_t* w_empty = w_full + kWStages;
    uint64_t* acc_full = w_empty + kWStages;
    uint64_t* drain = acc_full + 1;
    uint32_t* tmem_slot = (uint32_t*)(drain + 1);
    volatile int* abort_flag = (volatile int*)(tmem_slot + 1);
    uint32_t* tptr = (uint32_t*)(smem + p.off_tptr);

    if (threadIdx.x == 0) {
        for (int i = 0; i < SX; i++) {
            mbar_init(smem_u32(&x_full[i]), 1);
            mbar_init(smem_u32(&x_empty[i]), 1);
        }
        for (int i = 0; i < SR; i++) {
            mbar_init(smem_u32(&r_full[i]), 1);
            mbar_init(smem_u32(&r_empty[i]), kDecoderWarps);
        }
        for (int i = 0; i < kWStages; i++) {
            mbar_init(smem_u32(&w_full[i]), kDecoderWarps);
            mbar_init(smem_u32(&w_empty[i]), 1);
        }
        mbar_init(smem_u32(acc_full), 1);
        mbar_init(smem_u32(drain), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    // tile pointers of the CTA's strips, for every k-tile (row j = strip s0 + j)
    for (int i = threadIdx.x; i < kStrips * (nk + 1); i += kThreads) {
        const int j = i / (nk + 1), kt = i % (nk + 1);
        const int s = s0 + j;
        tptr[i] = (s < p.n_strips) ? __ldg(p.tileptr + (size_t)s * nk + kt) : 0u;
    }
    if (warp == 1) {  // TMEM allocation (whole warp)
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    int x_issued = 0, r_issued = 0;  // producer lane 0: stages armed on each ring
    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&tmap_x) : "memory");
            int xs = 0, rs = 0;
            uint32_t xph = 0, rph = 0;
            for (int kt = 0; kt < nk; kt++) {
                // X tile: rows m0..m0+255, columns 64 kt.. (zero fill outside X)
                if (kt >= SX && !wait_or_abort(smem_u32(&x_empty[xs]), xph ^ 1u, abort_flag)) {
                    flag_abort(abort_flag, p.status);
                    break;
                }
                const uint32_t xbar = smem_u32(&x_full[xs]);
                mbar_arrive_expect_tx(xbar, kXStageBytes);
                tma_load_2d(sbase + (uint32_t)xs * kXStageBytes, &tmap_x, kt * kBK, m0, xbar);
                x_issued++;
                if (++xs == SX) { xs = 0; xph ^= 1u; }
                // the four TCB tiles of this k-step
                if (kt >= SR && !wait_or_abort(smem_u32(&r_empty[rs]), rph ^ 1u, abort_flag)) {
                    flag_abort(abort_flag, p.status);
                    break;
                }
                const uint32_t rbar = smem_u32(&r_full[rs]);
                const uint32_t rst = sbase + p.off_raw + (uint32_t)rs * p.raw_stage_bytes;
                uint32_t total = 0, vb[kStrips], u0[kStrips];
                for (int j = 0; j < kStrips; j++) {
                    vb[j] = 0;
                    u0[j] = 0;
                    if (s0 + j >= p.n_strips) continue;
                    u0[j] = tptr[j * (nk + 1) + kt];
                    vb[j] = (tptr[j * (nk + 1) + kt + 1] - u0[j]) * 16u;
                    if (vb[j] + 16u > p.val_slot) {  // larger than the header allows
                        raise_status(p.status, SPW_ERR_FORMAT);
                        vb[j] = 0;
                    }
                    total += 512u + vb[j];
                }
                fence_proxy_async_smem();
                mbar_arrive_expect_tx(rbar, total);
                for (int j = 0; j < kStrips; j++) {
                    if (s0 + j >= p.n_strips) continue;
                    const size_t t = (size_t)(s0 + j) * nk + kt;
                    bulk_g2s(rst + 512u * j, p.bitmaps + t * kTileCols, 512u, rbar);
                    if (vb[j])
                        bulk_g2s(rst + 2048u + (uint32_t)j * p.val_slot, p.values + (size_t)u0[j] * 8,
                                 vb[j], rbar);
                }
                r_issued++;
                if (++rs == SR) { rs = 0; rph ^= 1u; }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc = idesc_f16(128, kBN);
            int xs = 0, ws = 0;
            uint32_t xph = 0, wph = 0;
            for (int kt = 0; kt < nk; kt++) {
                if (!wait_or_abort(smem_u32(&x_full[xs]), xph, abort_flag) ||
                    !wait_or_abort(smem_u32(&w_full[ws]), wph, abort_flag)) {
                    flag_abort(abort_flag, p.status);
                    break;
                }
                tc_fence_after();
                const uint32_t xa = sbase + (uint32_t)xs * kXStageBytes;
                const uint32_t wa = sbase + p.off_w + (uint32_t)ws * kWStageBytes;
#pragma unroll
                for (int j = 0; j < kBK / 16; j++) {
                    const uint64_t bdesc = umma_desc_sw128(wa + 32u * j);
#pragma unroll
                    for (int h = 0; h < 2; h++) {
                        const uint64_t adesc = umma_desc_sw128(xa + 16384u * h + 32u * j);
                        umma_f16(tmem + 256u * h, adesc, bdesc, idesc, (kt > 0 || j > 0) ? 1u : 0u);
                    }
                }
                umma_commit(smem_u32(&x_empty[xs]));
                umma_commit(smem_u32(&w_empty[ws]));
                if (++xs == SX) { xs = 0; xph ^= 1u; }
                if (++ws == kWStages) { ws = 0; wph ^= 1u; }
            }
            umma_commit(smem_u32(acc_full));
            umma_commit(smem_u32(drain));
            (void)mbar_wait(smem_u32(drain), 0);  // every issued MMA has completed
        }
    } else {
        // ------------------------------------------------------------ decoders
        const int d = warp - 2;          // 0..7
        const int q = d & 3;             // strip within the tile
        const int h = d >> 2;            // column half
        const bool strip_ok = s0 + q < p.n_strips;
        uint4* rec = (uint4*)(smem + p.off_rec + 512u * d);
        const uint32_t lanebit = 1u << lane, ltmask = lanebit - 1u;
        const uint32_t nl0 = 64u * q + lane, nl1 = nl0 + 32u;  // local W rows
        int rs = 0, ws = 0;
        uint32_t rph = 0, wph = 0;
        bool ok = true;
        for (int kt = 0; kt < nk && ok; kt++) {
            // every lane waits; __all_sync keeps the outcome warp-uniform
            if (!__all_sync(0xffffffffu, wait_or_abort(smem_u32(&r_full[rs]), rph, abort_flag))) {
                flag_abort(abort_flag, p.status);
                break;
            }
            const unsigned char* rst = smem + p.off_raw + (uint32_t)rs * p.raw_stage_bytes;
            if (strip_ok) {
                const uint64_t* bm = (const uint64_t*)(rst + 512u * q);
                const uint64_t wa = bm[lane], wb = bm[lane + 32];
                const int ca = __popcll(wa), cb = __popcll(wb);
                const int sa = warp_inclusive_scan(ca, lane);
                const int tot = __shfl_sync(0xffffffffu, sa, 31);
                const int sb = warp_inclusive_scan(cb, lane);
                const uint64_t w = h ? wb : wa;
                const uint32_t start = (uint32_t)(h ? tot + sb - cb : sa - ca);
                const uint32_t va = sbase + p.off_raw + (uint32_t)rs * p.raw_stage_bytes + 2048u +
                                    (uint32_t)q * p.val_slot + 2u * start;
                rec[lane] = make_uint4((uint32_t)w, (uint32_t)(w >> 32), va,
                                       va + 2u * __popc((uint32_t)w));
            }
            __syncwarp();
            if (kt >= kWStages &&
                !__all_sync(0xffffffffu, wait_or_abort(smem_u32(&w_empty[ws]), wph ^ 1u, abort_flag))) {
                flag_abort(abort_flag, p.status);
                break;
            }
            unsigned char* wst = smem + p.off_w + (uint32_t)ws * kWStageBytes;
#pragma unroll
            for (int g = 0; g < 4; g++) {  // 8 columns -> one 16-byte chunk per row
                uint32_t o0[4], o1[4];
                if (strip_ok) {
                    uint16_t v0[8], v1[8];
#pragma unroll
                    for (int c = 0; c < 8; c++) {
                        const uint4 r = rec[8 * g + c];
                        const uint16_t a = lds_u16(r.z + 2u * __popc(r.x & ltmask));
                        const uint16_t b = lds_u16(r.w + 2u * __popc(r.y & ltmask));
                        v0[c] = (r.x & lanebit) ? a : (uint16_t)0;
                        v1[c] = (r.y & lanebit) ? b : (uint16_t)0;
                    }
#pragma unroll
                    for (int c = 0; c < 4; c++) {
                        o0[c] = pack2(v0[2 * c], v0[2 * c + 1]);
                        o1[c] = pack2(v1[2 * c], v1[2 * c + 1]);
                    }
                } else {
#pragma unroll
                    for (int c = 0; c < 4; c++) o0[c] = o1[c] = 0u;
                }
                const uint32_t chunk = 4u * h + g;
                *(uint4*)(wst + nl0 * 128u + ((chunk ^ (nl0 & 7u)) << 4)) =
                    make_uint4(o0[0], o0[1], o0[2], o0[3]);
                *(uint4*)(wst + nl1 * 128u + ((chunk ^ (nl1 & 7u)) << 4)) =
                    make_uint4(o1[0], o1[1], o1[2], o1[3]);
            }
            fence_proxy_async_smem();  // generic-proxy stores -> tensor-core reads
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(smem_u32(&w_full[ws]));
                mbar_arrive(smem_u32(&r_empty[rs]));
            }
            if (++rs == SR) { rs = 0; rph ^= 1u; }
            if (++ws == kWStages) { ws = 0; wph ^= 1u; }
        }

        // ------------------------------------------------------------ epilogue
        const bool acc_ready =
            __all_sync(0xffffffffu, !*abort_flag && wait_or_abort(smem_u32(acc_full), 0, abort_flag));
        if (acc_ready) {
            tc_fence_after();
            const int quarter = warp & 3;           // TMEM lanes this warp may access
            const int acc = (warp - 2) >> 2;        // accumulator 0 (warps 2-5) or 1 (6-9)
            const int m = m0 + 128 * acc + 32 * quarter + lane;
            const bool vec = (p.ldy % 8) == 0;
            for (int j = 0; j < kBN / 32; j++) {
                uint32_t r[32];
                tmem_ld32(tmem + ((uint32_t)(32 * quarter) << 16) + 256u * acc + 32u * j, r);
                const int n = n0 + 32 * j;
                if (m >= p.M || n >= p.N) continue;
                uint16_t* yrow = p.Y + (size_t)m * p.ldy + n;
                uint32_t packed[16];
#pragma unroll
                for (int c = 0; c < 16; c++)
                    packed[c] = pack2(__half_as_ushort(__float2half_rn(__uint_as_float(r[2 * c]))),
                                      __half_as_ushort(__float2half_rn(__uint_as_float(r[2 * c + 1]))));
                if (vec && n + 32 <= p.N) {
#pragma unroll
                    for (int c = 0; c < 4; c++)
                        *(uint4*)(yrow + 8 * c) = make_uint4(packed[4 * c], packed[4 * c + 1],
                                                             packed[4 * c + 2], packed[4 * c + 3]);
                } else {
                    const int lim = min(32, p.N - n);
                    for (int c = 0; c < lim; c++) yrow[c] = (uint16_t)(packed[c >> 1] >> (16 * (c & 1)));
                }
            }
        } else {
            flag_abort(abort_flag, p.status);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0 && lane == 0 && *abort_flag) {
        // Drain the copies this CTA armed (bounded): for each slot, the phase of its
        // last issue.  Phases a consumer already waited for return at once.
        for (int i = 0; i < SX && i < x_issued; i++) {
            const int last = i + ((x_issued - 1 - i) / SX) * SX;
            (void)mbar_wait(smem_u32(&x_full[i]), (uint32_t)((last / SX) & 1));
        }
        for (int i = 0; i < SR && i < r_issued; i++) {
            const int last = i + ((r_issued - 1 - i) / SR) * SR;
            (void)mbar_wait(smem_u32(&r_full[i]), (uint32_t)((last / SR) & 1));
        }
    }
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(kTmemCols)
                     : "memory");
    }
}

// ------------------------------------------------------------------ host side
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
    int sx, sr;
    uint32_t val_slot, raw_stage_bytes, off_w, off_raw, off_rec, off_tptr, off_bar;
    size_t smem;
};

int make_spmm_plan(const spw_format* h, SpmmPlan* pl) {
    pl->val_slot = (uint32_t)round_up_u64(16ull * h->max_tile_units + 16, 16);
    pl->raw_stage_bytes = 2048u + (uint32_t)kStrips * pl->val_slot;
    const uint32_t tptr_bytes = (uint32_t)round_up_u64(4ull * kStrips * (h->n_ktiles + 1), 16);
    const int options[][2] = {{4, 4}, {4, 3}, {3, 3}, {3, 2}, {2, 3}, {2, 2}};
    for (const auto& o : options) {
        const int sx = o[0], sr = o[1];
        const uint32_t off_w = (uint32_t)sx * kXStageBytes;
        const uint32_t off_raw = off_w + (uint32_t)kWStages * kWStageBytes;
        const uint32_t off_rec = off_raw + (uint32_t)sr * pl->raw_stage_bytes;
        const uint32_t off_tptr = off_rec + 512u * kDecoderWarps;
        const uint32_t off_bar = (uint32_t)round_up_u64(off_tptr + tptr_bytes, 8);
        const uint32_t bar_bytes = 8u * (2 * sx + 2 * sr + 2 * kWStages + 2) + 16u;
        const size_t total = (size_t)off_bar + bar_bytes + 1024;  // + base alignment slack
        if (total <= (size_t)kSmemLimit) {
            pl->sx = sx;
            pl->sr = sr;
            pl->off_w = off_w;
            pl->off_raw = off_raw;
            pl->off_rec = off_rec;
            pl->off_tptr = off_tptr;
            pl->off_bar = off_bar;
            pl->smem = total;
            return SPW_OK;
        }
    }
    return SPW_ERR_UNSUPPORTED;
}

}  // namespace
}  // namespace spw

using namespace spw;

extern "C" {

uint64_t spw_spmm_workspace_bytes(const spw_format* hdr, int M) {
    (void)hdr;
    (void)M;
    return 0;
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
    (void)d_ws;
    (void)ws_bytes;
    SpmmPlan pl;
    rc = make_spmm_plan(hdr, &pl);
    if (rc != SPW_OK) return rc;
    rc = get_encoder();
    if (rc != SPW_OK) return rc;
    int* status = device_status_ptr();
    if (!status) return SPW_ERR_CUDA;

    // X as a 2-D tensor map: dim 0 = K (contiguous), dim 1 = M rows at ldx elements.
    CUtensorMap tmap;
    const cuuint64_t dims[2] = {(cuuint64_t)hdr->K, (cuuint64_t)M};
    const cuuint64_t ld_bytes = (cuuint64_t)((M > 1 ? ldx : ((ldx + 7) / 8 * 8)) * 2);
    const cuuint64_t strides[1] = {ld_bytes};
    const cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)kBM};
    const cuuint32_t estr[2] = {1, 1};
    CUresult cr = g_encode(&tmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, (void*)d_X, dims, strides, box,
                           estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (cr != CUDA_SUCCESS) return SPW_ERR_CUDA;

    const uint8_t* buf = (const uint8_t*)d_buf;
    SpmmParams prm;
    prm.bitmaps = (const uint64_t*)(buf + hdr->off_bitmaps);
    prm.tileptr = (const uint32_t*)(buf + hdr->off_tileptr);
    prm.values = (const uint16_t*)(buf + hdr->off_values);
    prm.Y = d_Y;
    prm.status = status;
    prm.M = M;
    prm.N = (int)hdr->N;
    prm.K = (int)hdr->K;
    prm.ldy = ldy;
    prm.n_strips = (int)hdr->n_strips;
    prm.n_ktiles = (int)hdr->n_ktiles;
    prm.sx = pl.sx;
    prm.sr = pl.sr;
    prm.raw_stage_bytes = pl.raw_stage_bytes;
    prm.val_slot = pl.val_slot;
    prm.off_w = pl.off_w;
    prm.off_raw = pl.off_raw;
    prm.off_rec = pl.off_rec;
    prm.off_tptr = pl.off_tptr;
    prm.off_bar = pl.off_bar;

    static size_t attr_smem[64];
    int dev = 0;
    SPW_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= 64) return SPW_ERR_CUDA;
    if (attr_smem[dev] < pl.smem) {
        SPW_CUDA_TRY(cudaFuncSetAttribute(spmm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          (int)pl.smem));
        attr_smem[dev] = pl.smem;
    }
    const dim3 grid((M + kBM - 1) / kBM, (hdr->N + kBN - 1) / kBN);
    if (grid.y > 65535u) return SPW_ERR_UNSUPPORTED;
    spmm_kernel<<<grid, kThreads, pl.smem, (cudaStream_t)stream>>>(tmap, prm);
    SPW_LAUNCH_CHECK();
    return SPW_OK;
}

}  // extern "C"
