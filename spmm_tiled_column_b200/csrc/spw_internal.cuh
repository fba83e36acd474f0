// spw_internal.cuh -- shared device and host helpers of the spw CUDA library (sm_100a).
//
// Everything here belongs to the product path.  It declares the TCB v1 geometry for the
// kernels, the asynchronous-copy and mbarrier primitives (inline PTX, no multicast
// anywhere), bounded waits that report SPW_ERR_TIMEOUT through a device status word,
// and host-side argument checks.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "spw.h"

namespace spw {

// ------------------------------------------------------------------ TCB v1 geometry
constexpr uint32_t kMagic = 0x31424354u;  // "TCB1"
constexpr uint32_t kFormatVersion = 1u;
constexpr int kStripRows = 64;  // TN: rows per strip (one u64 bitmap word per column)
constexpr int kTileCols = 64;   // TK: columns per tile
constexpr int kHeaderBytes = 256;
constexpr int kSectionAlign = 256;

struct Geometry {
    uint32_t n_strips, n_ktiles;
    uint64_t n_tiles, off_bitmaps, off_tileptr, off_values;
};

__host__ __device__ inline uint64_t round_up_u64(uint64_t v, uint64_t a) {
    return (v + a - 1) / a * a;
}

__host__ __device__ inline Geometry geometry(int N, int K) {
    Geometry g;
    g.n_strips = (uint32_t)((N + kStripRows - 1) / kStripRows);
    g.n_ktiles = (uint32_t)((K + kTileCols - 1) / kTileCols);
    g.n_tiles = (uint64_t)g.n_strips * g.n_ktiles;
    g.off_bitmaps = kHeaderBytes;
    g.off_tileptr = round_up_u64(g.off_bitmaps + 8ull * g.n_tiles * kTileCols, kSectionAlign);
    g.off_values = round_up_u64(g.off_tileptr + 4ull * (g.n_tiles + 1), kSectionAlign);
    return g;
}

// ------------------------------------------------------------------ device status word
// One int per device (file-scope __device__ in api.cu); kernels receive its address.
// Device code only ever raises it to a nonzero spw_status with atomicCAS from 0.
__device__ inline void raise_status(int* status, int code) {
    if (status) atomicCAS(status, 0, code);
}

// Upper bound, in SM clock cycles, on the spin-waits of the library's kernels: about one
// second at the B200's 1.9 GHz clock; normal waits end within microseconds.  Kernels take
// the limit of their pipeline waits as a launch parameter (spw_set_wait_limit_cycles can
// shorten it to exercise the timeout path); the waits that drain copies and MMAs after an
// abort always use this fixed limit, so that no asynchronous copy can still be writing
// shared memory when a CTA exits.
constexpr long long kWaitLimitCycles = 2000000000ll;

// ------------------------------------------------------------------ PTX primitives
__device__ inline uint32_t smem_u32(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ inline void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

// Make mbarrier initialisation visible to the async proxy (bulk copies, tcgen05).
__device__ inline void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Order this thread's earlier generic-proxy shared-memory accesses before later
// async-proxy accesses (bulk copies writing into a buffer that was just read).
__device__ inline void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ inline void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ inline void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ inline bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
    return done != 0;
}

// Non-blocking test of the same phase condition.
__device__ inline bool mbar_test_wait(uint32_t bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
    return done != 0;
}

// Wait for the phase with the given parity to complete, giving up after `limit` cycles.
// Returns false on timeout (the caller reports it and unwinds).  try_wait may suspend the
// thread until the phase completes (up to a hardware time window), which is the cheap way
// to wait but would let a short wait finish whatever the limit; a limit shorter than the
// default (set only to exercise the timeout path) therefore polls with test_wait.
__device__ inline bool mbar_wait(uint32_t bar, uint32_t parity, long long limit) {
    if (limit >= kWaitLimitCycles) {
        if (mbar_try_wait(bar, parity)) return true;
        const long long start = clock64();
        while (!mbar_try_wait(bar, parity)) {
            if (clock64() - start > limit) return false;
        }
        return true;
    }
    const long long start = clock64();
    while (!mbar_test_wait(bar, parity)) {
        if (clock64() - start > limit) return false;
    }
    return true;
}

// Drain wait after an abort (or at exit): always the fixed limit.
__device__ inline bool mbar_drain(uint32_t bar, uint32_t parity) {
    return mbar_wait(bar, parity, kWaitLimitCycles);
}

// One-dimensional bulk copy global -> shared (this CTA), completing on an mbarrier.
// dst, src and bytes must be multiples of 16.  No multicast.
__device__ inline void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

// Same, with an L2 eviction-priority hint (createpolicy) for streamed-once data.
__device__ inline uint64_t policy_evict_first() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

__device__ inline void bulk_g2s_hint(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar,
                                     uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint "
        "[%0], [%1], %2, [%3], %4;" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar), "l"(policy)
        : "memory");
}

// Shared-memory load without volatile, so the compiler may schedule it freely.  Only use
// it with an address computed from data loaded after the barrier that publishes the
// location (the data dependency keeps it after that barrier).
__device__ inline uint16_t lds_u16(uint32_t addr) {
    uint16_t v;
    asm("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr));
    return v;
}

// acc = (bits & lanebit) ? a * b + acc : acc, with fp16 a, b and an fp32 accumulator, as a
// predicated fused multiply-add (the skipped product never touches acc, so a stored
// Inf/NaN elsewhere in the column cannot leak in).
__device__ inline float fma_f16_f32_if(uint32_t bits, uint32_t lanebit, uint16_t a, uint16_t b,
                                       float acc) {
    asm("{\n\t.reg .pred p;\n\t.reg .b32 t;\n\t"
        "and.b32 t, %1, %2;\n\t"
        "setp.ne.b32 p, t, 0;\n\t"
        "@p fma.rn.f32.f16 %0, %3, %4, %0;\n\t}"
        : "+f"(acc)
        : "r"(bits), "r"(lanebit), "h"(a), "h"(b));
    return acc;
}

// d = a * b + c with fp16 a, b and fp32 c, d (one rounding; the fp16 product is exact).
__device__ inline float fma_f16_f32(uint16_t a, uint16_t b, float c) {
    float d;
    asm("fma.rn.f32.f16 %0, %1, %2, %3;" : "=f"(d) : "h"(a), "h"(b), "f"(c));
    return d;
}

// Device-scope atomic add with release semantics (orders this thread's earlier writes,
// and by cumulativity those of threads it synchronised with, before the add).
__device__ inline uint32_t atom_add_release_gpu(uint32_t* p, uint32_t v) {
    uint32_t old;
    asm volatile("atom.release.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v)
                 : "memory");
    return old;
}

// Device-scope add with acquire and release semantics; returns the old value.
__device__ inline uint32_t atom_add_acq_rel_gpu(uint32_t* p, uint32_t v) {
    uint32_t old;
    asm volatile("atom.add.acq_rel.gpu.global.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}

// Programmatic dependent launch: wait until the previous kernel on the stream has
// completed and its memory is visible / allow the next kernel to begin launching.
// Both are no-ops for a kernel launched without the programmatic attribute.
__device__ inline void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ inline void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ inline uint32_t lanemask_lt() {
    uint32_t m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// Threshold rule on one fp16 activation: takes part iff v != 0 and not |v| < t.
// NaN takes part (it is not zero and not below t).
__device__ inline bool passes_threshold(uint16_t bits, float t) {
    const float v = __half2float(__ushort_as_half(bits));
    return v != 0.0f && !(fabsf(v) < t);
}

__device__ inline int warp_inclusive_scan(int v, int lane) {
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        int u = __shfl_up_sync(0xffffffffu, v, d);
        if (lane >= d) v += u;
    }
    return v;
}

}  // namespace spw

// ------------------------------------------------------------------ host helpers
namespace spw {

// Per-device host state (status-word address, SM count, kernel attributes) is kept for
// device ordinals below this.
constexpr int kMaxDevices = 64;

inline bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

// Row stride rule for fp16 operands: multiple of 8 elements unless the operand has a
// single row.
inline bool ld_ok(int ld, int row_len, int rows) {
    if (ld < row_len) return false;
    return rows <= 1 || (ld % 8) == 0;
}

// Checks a host header against the TCB v1 geometry it claims.
int check_header(const spw_format* h);

// Address of this device's status word (looked up once per device).
int* device_status_ptr();

// Number of SMs of the current device (cached per device).
int device_sm_count();

// Host-side checks of a decode call's arguments, shared by every decode entry point:
// header, batch, null pointers, alignment, leading dimensions and threshold.  Returns
// SPW_OK or the status the call must return; touches no device state.
int check_decode_args(const spw_format* hdr, const void* buf, const uint16_t* x, int B, int ldx,
                      float threshold, const uint32_t* act_bits, const uint16_t* y, int ldy);

// Process-wide switch set by spw_set_launch_overlap.
bool launch_overlap();

// Limit of the kernels' pipeline waits, in SM cycles (spw_set_wait_limit_cycles).
long long wait_limit_cycles();

// Decode column-fetch mode set by spw_set_column_fetch (0, 1 or 2).
int column_fetch_mode();

// Token grouping for prefill (tokens.cu): signatures of up to 4 words of k-tile bits.
constexpr int kMaxTokenWords = 4;
constexpr int kMaxTokenK = 64 * 64 * kMaxTokenWords;  // 16384 columns
constexpr int kMaxGroupTokens = 16384;
inline int token_sig_words(int K) { return ((K + 63) / 64 + 63) / 64; }
// Scratch bytes (per-token signatures and rank counters) of group_tokens_launch.
uint64_t token_groups_scratch_bytes(int M, int K);
// Launches the three grouping kernels on stream: X (M x K at ldx) -> Xg (M x ldg, the
// rule applied, rows in grouped order), perm[M] (row r of Xg is token perm[r]) and
// tile_sig[ceil(M / T) * words] (k-tiles each token tile of T rows visits).
int group_tokens_launch(const uint16_t* X, int M, int K, int ldx, float t, int T, uint16_t* Xg,
                        int ldg, uint32_t* perm, uint64_t* tile_sig, void* scratch,
                        cudaStream_t stream);

}  // namespace spw

#define SPW_CUDA_TRY(expr)                         \
    do {                                           \
        cudaError_t _e = (expr);                   \
        if (_e != cudaSuccess) return SPW_ERR_CUDA; \
    } while (0)

#define SPW_LAUNCH_CHECK()                                        \
    do {                                                          \
        if (cudaPeekAtLastError() != cudaSuccess) {               \
            (void)cudaGetLastError();                             \
            return SPW_ERR_CUDA;                                  \
        }                                                         \
    } while (0)
