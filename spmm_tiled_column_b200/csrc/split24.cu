// split24.cu -- the 2:4 + residual split of a pruned weight for the sparse tensor cores.
//
// "Accelerating LLM GPU inference with moderately unstructured sparse weight matrices"
// (abstract, §1; its related-work paragraph describes the same split for SparTA): tensor
// cores accelerate only 2:4 structured sparsity, so the weight is stored as a 2:4 part
// for sparse MMA plus a residual that keeps the product exact.  Within every group of
// four columns of a row the first two kept weights (column order) form the 2:4 part;
// any further kept weights go to the residual, which this library stores as an ordinary
// TCB v1 buffer (compressed from the residual mask this kernel writes).
//
// The 2:4 part, per 64 x 64 tile t = strip * n_ktiles + k-tile, is laid out as the
// prefill kernel's shared memory wants it, so that one bulk copy per strip lands it:
//   values:   4096 bytes per tile at t * 4096: row r's 32 kept-or-padding halves (two
//             per group of four columns, in column order) fill 64 bytes at 64 r; its four
//             16-byte chunks (groups 4c .. 4c+3) sit at chunk position c ^ ((r >> 1) & 3)
//             (the 64-byte swizzle of the MMA's K-major operand layout).
//   metadata: 1024 bytes per tile at n_tiles * 4096 + t * 1024: 16 bytes per tensor
//             memory lane L of the tile's row block (64 lanes), {word for the tile's
//             columns 0-31, word for columns 32-63, 0, 0} -- one row of the 128 x 16-byte
//             matrix that tcgen05.cp moves into four tensor-memory columns.  A word holds
//             rows 16 (L / 16) + L % 8 (bits 0-15) and that row + 8 (bits 16-31), columns
//             32 j + 16 ((L / 8) % 2) .. +15 of its half j as four 4-bit groups (group g
//             at bits 4 g of its half), each group {first index, second index} in bits
//             {0-1, 2-3}, first < second.
//   padding:  1024 bytes at n_tiles * 5120: the metadata of a tile with no kept weight
//             (every group {0, 1}), copied for the missing second strip of a weight with
//             an odd strip count.
// A group with fewer than two kept weights is padded with the lowest free positions and
// zero values; rows past N and columns past K hold no kept weight.
#include "spw_internal.cuh"

namespace spw {
namespace {

constexpr int kS24ValBytes = 4096;
constexpr int kS24MetaBytes = 1024;

__global__ void __launch_bounds__(64)
split24_kernel(const uint16_t* __restrict__ W, int ldw, const uint8_t* __restrict__ mask,
               int ld_mask, int N, int K, int n_ktiles, int n_tiles, uint8_t* __restrict__ s24,
               uint8_t* __restrict__ mask_r, int ld_r) {
    __shared__ uint16_t meta16[2][64][2];  // [MMA half j][lane][row half]
    const int t = blockIdx.x;
    const int s = t / n_ktiles, kt = t % n_ktiles;
    const int r = threadIdx.x;  // row within the strip
    const int n = 64 * s + r;
    uint32_t vals[16];           // this row's 32 stored halves, two per 32-bit word
    uint32_t nib[2] = {0u, 0u};  // 4 bits per group: groups 0-7 in nib[0], 8-15 in nib[1]
#pragma unroll
    for (int G = 0; G < 16; G++) {
        const int k0 = 64 * kt + 4 * G;
        int pos[4], cnt = 0;
        uint16_t w[4] = {0, 0, 0, 0};
#pragma unroll
        for (int e = 0; e < 4; e++) {
            const int k = k0 + e;
            const bool kept = n < N && k < K && mask[(size_t)n * ld_mask + k] != 0;
            if (kept) {
                w[e] = W[(size_t)n * ldw + k];
                if (cnt < 2) pos[cnt] = e;
                cnt++;
            }
            if (n < N && k < K) mask_r[(size_t)n * ld_r + k] = (kept && cnt > 2) ? 1 : 0;
        }
        int i0, i1;
        uint16_t v0 = 0, v1 = 0;
        if (cnt >= 2) {
            i0 = pos[0];
            i1 = pos[1];
            v0 = w[i0];
            v1 = w[i1];
        } else if (cnt == 1) {
            if (pos[0] == 0) {
                i0 = 0;
                i1 = 1;
                v0 = w[0];
            } else {
                i0 = 0;
                i1 = pos[0];
                v1 = w[i1];
            }
        } else {
            i0 = 0;
            i1 = 1;
        }
        vals[G] = (uint32_t)v0 | ((uint32_t)v1 << 16);
        nib[G >> 3] |= (uint32_t)(i0 | (i1 << 2)) << (4 * (G & 7));
    }
    // values: four 16-byte chunks, swizzled
    uint8_t* vrow = s24 + (size_t)t * kS24ValBytes + 64 * r;
#pragma unroll
    for (int c = 0; c < 4; c++)
        *(uint4*)(vrow + 16 * (c ^ ((r >> 1) & 3))) =
            make_uint4(vals[4 * c], vals[4 * c + 1], vals[4 * c + 2], vals[4 * c + 3]);
    // metadata: row r = 16 b + 8 h + i feeds lanes 16 b + 8 k1 + i, half h, for both k1
    const int b = r >> 4, h = (r >> 3) & 1, i = r & 7;
#pragma unroll
    for (int j = 0; j < 2; j++)
#pragma unroll
        for (int k1 = 0; k1 < 2; k1++)
            meta16[j][16 * b + 8 * k1 + i][h] = (uint16_t)((nib[j] >> (16 * k1)) & 0xffffu);
    __syncthreads();
    uint32_t* meta = (uint32_t*)(s24 + (size_t)n_tiles * kS24ValBytes + (size_t)t * kS24MetaBytes);
    *(uint4*)(meta + 4 * r) = make_uint4((uint32_t)meta16[0][r][0] | ((uint32_t)meta16[0][r][1] << 16),
                                         (uint32_t)meta16[1][r][0] | ((uint32_t)meta16[1][r][1] << 16), 0u, 0u);
    if (t == 0) {  // the padding block after the last tile
        uint32_t* pad = (uint32_t*)(s24 + (size_t)n_tiles * (kS24ValBytes + kS24MetaBytes));
        *(uint4*)(pad + 4 * r) = make_uint4(0x44444444u, 0x44444444u, 0u, 0u);
    }
}

}  // namespace
}  // namespace spw

using namespace spw;

extern "C" {

uint64_t spw_s24_bytes(int N, int K) {
    if (N < 1 || K < 1) return 0;
    const uint64_t tiles = (uint64_t)((N + 63) / 64) * (uint64_t)((K + 63) / 64);
    return tiles * (kS24ValBytes + kS24MetaBytes) + kS24MetaBytes;  // + the padding block
}

int spw_split24(const uint16_t* d_W, int ldw, const uint8_t* d_mask, int ld_mask, int N, int K,
                void* d_s24, uint64_t s24_bytes, uint8_t* d_mask_r, int ld_mask_r, void* stream) {
    if (N < 1 || K < 1 || !d_W || !d_mask || !d_s24 || !d_mask_r) return SPW_ERR_INVALID_ARG;
    if (ldw < K || ld_mask < K || ld_mask_r < K) return SPW_ERR_INVALID_ARG;
    if (!aligned16(d_s24)) return SPW_ERR_ALIGNMENT;
    const int n_ktiles = (K + 63) / 64, n_strips = (N + 63) / 64;
    if ((long long)n_ktiles * n_strips > 0x7fffffffll) return SPW_ERR_UNSUPPORTED;
    if (s24_bytes < spw_s24_bytes(N, K)) return SPW_ERR_BUFFER_TOO_SMALL;
    const int tiles = n_ktiles * n_strips;
    split24_kernel<<<tiles, 64, 0, (cudaStream_t)stream>>>(d_W, ldw, d_mask, ld_mask, N, K, n_ktiles,
                                                           tiles, (uint8_t*)d_s24, d_mask_r,
                                                           ld_mask_r);
    SPW_LAUNCH_CHECK();
    return SPW_OK;
}

}  // extern "C"
