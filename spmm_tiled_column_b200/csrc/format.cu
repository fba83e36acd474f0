// format.cu -- TCB v1 compression and decompression kernels.
//
// The Tiled-Column-wise Bitmap Compressed format is named in "Unified Static-Dynamic
// Pruning for Efficient LLM Inference" (abstract) without a byte layout; TCB v1 is this
// library's layout (documented in include/spw.h).  Compression runs once, offline ("the
// pattern is precomputed and stored in a dedicated format", "Accelerating LLM GPU
// inference with moderately unstructured sparse weight matrices", §2.1):
//   1. census:  one block per tile builds the 64 column bitmaps (one u64 per column,
//               bit r = row 64 s + r kept) and counts the tile's kept weights;
//   2. scan:    one block turns the counts into 16-byte-unit tile pointers and writes
//               the header (nnz, bytes_total, max_tile_units);
//   3. scatter: one block per tile writes the kept values column by column in row
//               order (the order of the set bits), each tile padded to 16 bytes.
// The host reads the header back between 2 and 3 to check the caller's buffer size.
#include "spw_internal.cuh"

namespace spw {
namespace {

constexpr int kScanThreads = 1024;

// Thread c of block (kt, s) owns column k = 64 kt + c of strip s.
__global__ void __launch_bounds__(64)
census_kernel(const uint8_t* __restrict__ mask, int ld_mask, int N, int K, uint32_t n_ktiles,
              uint64_t* __restrict__ bitmaps, uint32_t* __restrict__ counts) {
    const uint32_t kt = blockIdx.x, s = blockIdx.y;
    const int c = threadIdx.x;
    const int k = (int)kt * kTileCols + c;
    const int row0 = (int)s * kStripRows;
    const int rows = min(kStripRows, N - row0);
    uint64_t word = 0;
    if (k < K) {
        const uint8_t* p = mask + (size_t)row0 * ld_mask + k;
        for (int r = 0; r < rows; r++)
            if (p[(size_t)r * ld_mask]) word |= 1ull << r;
    }
    const uint64_t t = (uint64_t)s * n_ktiles + kt;
    bitmaps[t * kTileCols + c] = word;
    int cnt = __popcll(word);
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, d);
    __shared__ int half_count[2];
    if ((c & 31) == 0) half_count[c >> 5] = cnt;
    __syncthreads();
    if (c == 0) counts[t] = (uint32_t)(half_count[0] + half_count[1]);
}

// Single block: exclusive scan of per-tile 16-byte units in place, plus the header.
__global__ void __launch_bounds__(kScanThreads)
scan_kernel(uint8_t* __restrict__ buf, uint64_t n_tiles, uint32_t N, uint32_t K, Geometry g) {
    uint32_t* tileptr = (uint32_t*)(buf + g.off_tileptr);
    const int tid = threadIdx.x;
    const uint64_t per = (n_tiles + kScanThreads - 1) / kScanThreads;
    const uint64_t lo = min(n_tiles, per * tid), hi = min(n_tiles, lo + per);
    uint64_t units = 0, nnz = 0;
    uint32_t mx = 0;
    for (uint64_t t = lo; t < hi; t++) {
        const uint32_t c = tileptr[t];
        const uint32_t u = (c + 7) / 8;
        units += u;
        nnz += c;
        mx = max(mx, u);
    }
    __shared__ unsigned long long s_units[kScanThreads];
    __shared__ unsigned long long s_nnz[kScanThreads];
    __shared__ uint32_t s_max[kScanThreads];
    s_units[tid] = units;
    s_nnz[tid] = nnz;
    s_max[tid] = mx;
    __syncthreads();
    // Hillis-Steele inclusive scan of units; tree reductions of nnz and max.
    for (int d = 1; d < kScanThreads; d <<= 1) {
        unsigned long long v = tid >= d ? s_units[tid - d] : 0ull;
        __syncthreads();
        s_units[tid] += v;
        __syncthreads();
    }
    for (int d = kScanThreads / 2; d > 0; d >>= 1) {
        if (tid < d) {
            s_nnz[tid] += s_nnz[tid + d];
            s_max[tid] = max(s_max[tid], s_max[tid + d]);
        }
        __syncthreads();
    }
    uint64_t run = s_units[tid] - units;  // exclusive prefix
    for (uint64_t t = lo; t < hi; t++) {
        const uint32_t c = tileptr[t];
        tileptr[t] = (uint32_t)run;
        run += (c + 7) / 8;
    }
    if (tid == kScanThreads - 1) {
        const uint64_t total = s_units[tid];
        tileptr[n_tiles] = (uint32_t)total;
        spw_format h;
        h.magic = kMagic;
        h.version = kFormatVersion;
        h.N = N;
        h.K = K;
        h.TN = kStripRows;
        h.TK = kTileCols;
        h.n_strips = g.n_strips;
        h.n_ktiles = g.n_ktiles;
        h.nnz = s_nnz[0];
        h.bytes_total = g.off_values + 16 * total;
        h.off_bitmaps = g.off_bitmaps;
        h.off_tileptr = g.off_tileptr;
        h.off_values = g.off_values;
        h.max_tile_units = s_max[0];
        h.reserved = 0;
        *(spw_format*)buf = h;
    }
}

// Exclusive prefix over the 64 columns of a tile (two warps), from each column's count.
__device__ inline int tile_column_offset(int cnt, int c, int* s_warp_total) {
    const int lane = c & 31;
    const int incl = warp_inclusive_scan(cnt, lane);
    if (lane == 31) s_warp_total[c >> 5] = incl;
    __syncthreads();
    return incl - cnt + (c >= 32 ? s_warp_total[0] : 0);
}

__global__ void __launch_bounds__(64)
scatter_kernel(const uint16_t* __restrict__ W, int ldw, int N, int K, uint32_t n_ktiles,
               const uint64_t* __restrict__ bitmaps, const uint32_t* __restrict__ tileptr,
               uint16_t* __restrict__ values) {
    const uint32_t kt = blockIdx.x, s = blockIdx.y;
    const int c = threadIdx.x;
    const int k = (int)kt * kTileCols + c;
    const uint64_t t = (uint64_t)s * n_ktiles + kt;
    const uint64_t word = bitmaps[t * kTileCols + c];
    __shared__ int s_tot[2];
    const int off = tile_column_offset(__popcll(word), c, s_tot);
    uint16_t* out = values + (size_t)tileptr[t] * 8 + off;
    const int row0 = (int)s * kStripRows;
    const int rows = min(kStripRows, N - row0);
    int j = 0;
    for (int r = 0; r < rows; r++)  // lockstep over rows: reads of W are coalesced
        if ((word >> r) & 1ull) out[j++] = W[(size_t)(row0 + r) * ldw + k];
    (void)K;
}

__global__ void __launch_bounds__(64)
decompress_kernel(int N, int K, uint32_t n_ktiles, const uint64_t* __restrict__ bitmaps,
                  const uint32_t* __restrict__ tileptr, const uint16_t* __restrict__ values,
                  uint16_t* __restrict__ out, int ldw) {
    const uint32_t kt = blockIdx.x, s = blockIdx.y;
    const int c = threadIdx.x;
    const int k = (int)kt * kTileCols + c;
    const uint64_t t = (uint64_t)s * n_ktiles + kt;
    const uint64_t word = bitmaps[t * kTileCols + c];
    __shared__ int s_tot[2];
    const int off = tile_column_offset(__popcll(word), c, s_tot);
    if (k >= K) return;
    const uint16_t* in = values + (size_t)tileptr[t] * 8 + off;
    const int row0 = (int)s * kStripRows;
    const int rows = min(kStripRows, N - row0);
    int j = 0;
    for (int r = 0; r < rows; r++) {  // lockstep over rows: writes are coalesced
        uint16_t v = 0;
        if ((word >> r) & 1ull) v = in[j++];
        out[(size_t)(row0 + r) * ldw + k] = v;
    }
}

// Counts for spw_format_query: total 16-byte units and nnz, accumulated with atomics.
__global__ void __launch_bounds__(64)
query_kernel(const uint8_t* __restrict__ mask, int ld_mask, int N, int K,
             unsigned long long* __restrict__ totals) {
    const uint32_t kt = blockIdx.x, s = blockIdx.y;
    const int c = threadIdx.x;
    const int k = (int)kt * kTileCols + c;
    const int row0 = (int)s * kStripRows;
    const int rows = min(kStripRows, N - row0);
    int cnt = 0;
    if (k < K) {
        const uint8_t* p = mask + (size_t)row0 * ld_mask + k;
        for (int r = 0; r < rows; r++) cnt += p[(size_t)r * ld_mask] != 0;
    }
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, d);
    __shared__ int half_count[2];
    if ((c & 31) == 0) half_count[c >> 5] = cnt;
    __syncthreads();
    if (c == 0) {
        const unsigned long long tile = (unsigned long long)(half_count[0] + half_count[1]);
        atomicAdd(&totals[0], (tile + 7) / 8);
        atomicAdd(&totals[1], tile);
    }
}

int check_mask_args(const uint8_t* d_mask, int N, int K, int ld_mask) {
    if (!d_mask || N < 1 || K < 1 || ld_mask < K) return SPW_ERR_INVALID_ARG;
    if (!aligned16(d_mask)) return SPW_ERR_ALIGNMENT;
    Geometry g = geometry(N, K);
    if (g.n_ktiles > 0x7fffffffu || g.n_strips > 65535u) return SPW_ERR_UNSUPPORTED;
    return SPW_OK;
}

}  // namespace
}  // namespace spw

using namespace spw;

extern "C" {

int spw_format_query(const uint8_t* d_mask, int N, int K, int ld_mask, uint64_t* bytes_total,
                     uint64_t* nnz, void* stream) {
    if (!bytes_total || !nnz) return SPW_ERR_INVALID_ARG;
    int rc = check_mask_args(d_mask, N, K, ld_mask);
    if (rc != SPW_OK) return rc;
    cudaStream_t s = (cudaStream_t)stream;
    Geometry g = geometry(N, K);
    unsigned long long* d_totals = nullptr;
    SPW_CUDA_TRY(cudaMallocAsync((void**)&d_totals, 2 * sizeof(unsigned long long), s));
    unsigned long long h[2] = {0, 0};
    int out = SPW_OK;
    if (cudaMemsetAsync(d_totals, 0, sizeof(h), s) != cudaSuccess) out = SPW_ERR_CUDA;
    if (out == SPW_OK) {
        query_kernel<<<dim3(g.n_ktiles, g.n_strips), 64, 0, s>>>(d_mask, ld_mask, N, K, d_totals);
        if (cudaGetLastError() != cudaSuccess) out = SPW_ERR_CUDA;
    }
    if (out == SPW_OK &&
        cudaMemcpyAsync(h, d_totals, sizeof(h), cudaMemcpyDeviceToHost, s) != cudaSuccess)
        out = SPW_ERR_CUDA;
    if (cudaFreeAsync(d_totals, s) != cudaSuccess) out = SPW_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) out = SPW_ERR_CUDA;
    if (out != SPW_OK) return out;
    *bytes_total = g.off_values + 16ull * h[0];
    *nnz = h[1];
    return SPW_OK;
}

int spw_compress(const uint16_t* d_W, int ldw, const uint8_t* d_mask, int ld_mask, int N, int K,
                 void* d_buf, uint64_t buf_bytes, spw_format* hdr_out, void* stream) {
    int rc = check_mask_args(d_mask, N, K, ld_mask);
    if (rc != SPW_OK) return rc;
    if (!d_W || !d_buf || ldw < K) return SPW_ERR_INVALID_ARG;
    if (!aligned16(d_W) || !aligned16(d_buf)) return SPW_ERR_ALIGNMENT;
    Geometry g = geometry(N, K);
    if (buf_bytes < g.off_values) return SPW_ERR_BUFFER_TOO_SMALL;
    cudaStream_t s = (cudaStream_t)stream;
    uint8_t* buf = (uint8_t*)d_buf;
    uint64_t* bitmaps = (uint64_t*)(buf + g.off_bitmaps);
    uint32_t* tileptr = (uint32_t*)(buf + g.off_tileptr);

    SPW_CUDA_TRY(cudaMemsetAsync(buf, 0, g.off_values, s));
    census_kernel<<<dim3(g.n_ktiles, g.n_strips), 64, 0, s>>>(d_mask, ld_mask, N, K, g.n_ktiles,
                                                             bitmaps, tileptr);
    SPW_LAUNCH_CHECK();
    scan_kernel<<<1, kScanThreads, 0, s>>>(buf, g.n_tiles, (uint32_t)N, (uint32_t)K, g);
    SPW_LAUNCH_CHECK();
    spw_format h;
    SPW_CUDA_TRY(cudaMemcpyAsync(&h, buf, sizeof(h), cudaMemcpyDeviceToHost, s));
    SPW_CUDA_TRY(cudaStreamSynchronize(s));
    if (h.bytes_total > buf_bytes) return SPW_ERR_BUFFER_TOO_SMALL;
    SPW_CUDA_TRY(cudaMemsetAsync(buf + g.off_values, 0, h.bytes_total - g.off_values, s));
    scatter_kernel<<<dim3(g.n_ktiles, g.n_strips), 64, 0, s>>>(
        d_W, ldw, N, K, g.n_ktiles, bitmaps, tileptr, (uint16_t*)(buf + g.off_values));
    SPW_LAUNCH_CHECK();
    if (hdr_out) {
        SPW_CUDA_TRY(cudaStreamSynchronize(s));
        *hdr_out = h;
    }
    return SPW_OK;
}

int spw_decompress(const spw_format* hdr, const void* d_buf, uint16_t* d_W_out, int ldw,
                   void* stream) {
    int rc = check_header(hdr);
    if (rc != SPW_OK) return rc;
    if (!d_buf || !d_W_out || ldw < (int)hdr->K) return SPW_ERR_INVALID_ARG;
    if (!aligned16(d_buf) || !aligned16(d_W_out)) return SPW_ERR_ALIGNMENT;
    if (hdr->n_strips > 65535u) return SPW_ERR_UNSUPPORTED;
    cudaStream_t s = (cudaStream_t)stream;
    const uint8_t* buf = (const uint8_t*)d_buf;
    decompress_kernel<<<dim3(hdr->n_ktiles, hdr->n_strips), 64, 0, s>>>(
        (int)hdr->N, (int)hdr->K, hdr->n_ktiles, (const uint64_t*)(buf + hdr->off_bitmaps),
        (const uint32_t*)(buf + hdr->off_tileptr), (const uint16_t*)(buf + hdr->off_values), d_W_out,
        ldw);
    SPW_LAUNCH_CHECK();
    return SPW_OK;
}

}  // extern "C"
