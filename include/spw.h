/*
 * spw.h -- C ABI of the sparse-weight SpMV / SpMM library for NVIDIA B200 (sm_100a).
 *
 * The library multiplies a pruned LLM linear-layer weight (fp16, moderate unstructured
 * sparsity) by activations:
 *   decode  (spMspV): y_b = W_masked . x~_b  for a batch of 1..16 activation vectors,
 *                     skipping the K-columns whose activation is zero or below a threshold;
 *   prefill (SpMM):   Y = X . W_masked^T     for M token rows, on tcgen05 tensor cores.
 * The weight is stored once, offline, in the TCB v1 tiled column-bitmap format.
 *
 * Sources (web pages, cited by title and section):
 *   [SPDP] "Unified Static-Dynamic Pruning for Efficient LLM Inference", abstract: static
 *          unstructured weight pruning unified with input-adaptive dynamic pruning, a
 *          Tiled-Column-wise Bitmap Compressed (Tiled-CBC) format, a CUDA-core spMspV
 *          decode kernel with activation skipping, a Tensor-Core SpMM prefill kernel.
 *   [RMM]  "Reduced Matrix Multiplication" (hotelren.com article), §4.1 (score, select,
 *          multiply on the subset, map back), §4.2 (Y[:, I] = X @ W[:, I]; FFN channel
 *          selection), §5.1 (top-k by |activation|, ascending indices), §7.3 (one index
 *          set shared across a block of tokens).
 *   [3LF]  "Accelerating LLM GPU inference with moderately unstructured sparse weight
 *          matrices", §1 (tensor cores take only 2:4 sparsity; the stored format must give
 *          the exact product; bitmap decoding cost on CUDA cores), §2.1 (prefill [BL, H]
 *          and decode [B, H] shapes; the pattern is precomputed and stored offline).
 *
 * Conventions for every call
 *   - Device pointers are global-memory addresses on the current CUDA device.  The
 *     caller allocates and owns every buffer; the library allocates nothing on the
 *     decode / prefill path (spw_format_query allocates 16 bytes of scratch, offline).
 *   - fp16 data is passed as uint16_t bit patterns (IEEE binary16).
 *   - Matrices are row-major with a leading dimension ("ld") in elements between rows.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls are
 *     asynchronous on `stream` unless their comment says they synchronise.
 *   - Arguments are validated on the host before any launch.  A bad argument returns a
 *     status code and launches nothing.  No call aborts, traps or prints.
 *   - Alignment: every device pointer must be 16-byte aligned (d_count and d_idx: 4).
 *     Leading dimensions only need to cover a row, except where a call copies rows
 *     with 16-byte bulk or tensor copies: the ldx of every decode and prefill call
 *     (spw_spmv and its group, FFN, no-alloc, tensor-core and auto forms; spw_spmm,
 *     spw_spmm_tokens, spw_spmm24, spw_group_tokens) must be a multiple of 8 fp16
 *     elements unless that operand has a single row.  Such copies
 *     may read an activation row up to the next 16-byte boundary past its last
 *     element (never across it, so never outside the row's allocation granule).
 *   - Buffer contents: the header is checked on the host.  The product kernels check each
 *     tile they read against it -- its tile pointers inside the values section and at
 *     most max_tile_units apart, its bitmaps' kept count within what max_tile_units
 *     allows -- and decode a tile that fails as empty, reporting SPW_ERR_FORMAT through
 *     spw_last_device_status.  Other disagreements between a buffer's sections give
 *     undefined numbers but no access outside the buffer.  spw_compress writes
 *     consistent buffers.
 *
 * The TCB v1 layout (this project's reading of Tiled-CBC; the page names the format but
 * gives no layout).  All integers little-endian.  A strip is 64 consecutive weight rows,
 * a tile is one strip times 64 consecutive columns; n_strips = ceil(N/64),
 * n_ktiles = ceil(K/64), tile t = s * n_ktiles + kt.
 *   [0, 256)      header: the spw_format struct below, then zero bytes.
 *   off_bitmaps   uint64 bitmap[n_strips][n_ktiles*64]; bit r of bitmap[s][k] is set iff
 *                 mask[64 s + r][k] != 0 (bits for rows >= N and columns >= K are 0).
 *   off_tileptr   uint32 tileptr[n_strips*n_ktiles + 1]: start of tile t's values in
 *                 16-byte units from off_values; the last entry is the total.
 *   off_values    uint16 values: per tile, the kept weights column by column (ascending
 *                 k), within a column by ascending row (the order of the set bits),
 *                 fp16 bits unchanged; each tile padded with 0x0000 to 16 bytes.
 *   Sections start at multiples of 256.  bytes_total = off_values + 16*tileptr[last].
 *   Every other byte is zero, so a buffer is a pure function of (W, mask).
 */
#ifndef SPW_H
#define SPW_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes returned by every call (0 = success). */
typedef enum {
    SPW_OK = 0,
    SPW_ERR_INVALID_ARG = 1,      /* null pointer, bad size or leading dimension, bad t  */
    SPW_ERR_ALIGNMENT = 2,        /* pointer or leading dimension breaks the 16-B rule   */
    SPW_ERR_BUFFER_TOO_SMALL = 3, /* format buffer or workspace smaller than required    */
    SPW_ERR_FORMAT = 4,           /* header magic/version/geometry does not match TCB v1 */
    SPW_ERR_UNSUPPORTED = 5,      /* valid request the library does not handle           */
    SPW_ERR_CUDA = 6,             /* a CUDA runtime call failed (launch, copy, device)   */
    SPW_ERR_TIMEOUT = 7           /* a bounded device-side wait ran out (see below)      */
} spw_status;

/* Host copy of the TCB v1 header; byte-identical to the first 80 bytes of a buffer. */
typedef struct {
    uint32_t magic;          /* 0x31424354 ("TCB1")                                   */
    uint32_t version;        /* 1                                                     */
    uint32_t N, K;           /* weight rows (outputs) and columns (inputs)            */
    uint32_t TN, TK;         /* 64, 64                                                */
    uint32_t n_strips;       /* ceil(N / 64)                                          */
    uint32_t n_ktiles;       /* ceil(K / 64)                                          */
    uint64_t nnz;            /* kept weights                                          */
    uint64_t bytes_total;    /* buffer length in bytes                                */
    uint64_t off_bitmaps, off_tileptr, off_values; /* section offsets in bytes        */
    uint32_t max_tile_units; /* largest tile, in 16-byte units                        */
    uint32_t reserved;       /* 0                                                     */
} spw_format;

/* Text for a status code (static storage; never NULL). */
const char* spw_status_string(int status);

/* Library version: 100 * major + minor.  The TCB format version is separate (1). */
int spw_version(void);

/* Launch overlap between consecutive decode calls (process-wide; off by default).
 * When enabled, spw_spmv launches with programmatic dependent launch: its CTAs may start
 * while the previous kernel on the stream is still finishing, and begin streaming the
 * compressed weight (the TCB buffer) before that kernel's writes are visible.  It also
 * lets the next kernel start early.  Activations, column sets, outputs and the
 * workspace are only touched after the previous kernel has completed, so chaining
 * layers stays correct; the one requirement is that the kernel immediately before
 * spw_spmv on the stream does not write the TCB buffer being read (true for weights
 * compressed at load time and left alone).  Returns the previous setting. */
int spw_set_launch_overlap(int enable);

/* Column fetch for the CUDA-core decode (process-wide; mode 0 by default).  With a column
 * set or a threshold the decode skips the work of inactive columns ("Reduced Matrix
 * Multiplication" §4.2: only W[:, I] takes part); whether it also skips their bytes is
 * this switch:
 *   0  whole tiles: each tile's bitmaps and packed values are streamed with bulk copies,
 *      inactive columns included (their work is skipped, their bytes are read);
 *   1  column fetch when a call carries a column set or a threshold above zero: each
 *      decode warp reads a tile's bitmaps, applies the rule, and copies only the 16-byte
 *      chunks that hold an active column's values (about 60-75 % of a tile's bytes at
 *      50 % random activation sparsity, falling with sparsity);
 *   2  column fetch for every call (for tests and measurement).
 * Results are identical in every mode (same work split and summation order).  On B200
 * the down projection at 50 % activation sparsity ran slower with column fetch (whole
 * tiles keep the weight stream ahead of the decode; column fetch can only start a tile's
 * copies once the activations are known), hence the default.  Returns the previous mode,
 * or -1 for a mode outside 0..2 (the setting is then unchanged). */
int spw_set_column_fetch(int mode);

/* Limit of the product kernels' bounded pipeline waits, in SM clock cycles (process-wide).
 * The default, about one second (2e9 cycles), is far above any normal wait, which ends
 * within microseconds; a wait that runs out makes the kernel stop, drain the copies and
 * tensor-core operations it has in flight, free its tensor memory, report SPW_ERR_TIMEOUT
 * through spw_last_device_status and return.  A smaller limit exists so that tests can
 * drive that path on purpose: a few hundred cycles is shorter than a weight copy from
 * HBM, so the first wait of the next call gives up.  The drain waits keep the default
 * limit whatever is set here.  cycles = 0 (or above the default) restores the default.
 * Takes effect at the next launch.  Returns the previous limit in cycles.  No page has a
 * counterpart; it serves failure detection only. */
uint64_t spw_set_wait_limit_cycles(uint64_t cycles);

/* Size of the TCB v1 buffer for an N x K mask (device uint8, row stride ld_mask bytes,
 * nonzero = kept).  [SPDP] format; layout above.  Writes bytes_total and nnz (host
 * pointers).  Synchronises `stream`.  Allocates 16 bytes of device scratch (offline).
 * Errors: INVALID_ARG (null pointer, N or K < 1, ld_mask < K), ALIGNMENT, CUDA. */
int spw_format_query(const uint8_t* d_mask, int N, int K, int ld_mask, uint64_t* bytes_total,
                     uint64_t* nnz, void* stream);

/* Compress a masked weight into a TCB v1 buffer ([SPDP] Tiled-CBC; [3LF] §2.1: done once,
 * offline).  d_W: N x K fp16 bits, row stride ldw; d_mask: N x K uint8, row stride
 * ld_mask.  Kept values are copied bit-exactly (a kept -0.0 stays 0x8000); masked-out
 * values are ignored.  d_buf receives exactly bytes_total bytes (spw_format_query); the
 * result is byte-identical to the oracle encoder.  When hdr_out is not NULL the header
 * is copied back into it.  Synchronises `stream` (the size check needs the tile counts).
 * Errors: INVALID_ARG, ALIGNMENT, BUFFER_TOO_SMALL (nothing past the header sections is
 * written then), CUDA. */
int spw_compress(const uint16_t* d_W, int ldw, const uint8_t* d_mask, int ld_mask, int N, int K,
                 void* d_buf, uint64_t buf_bytes, spw_format* hdr_out, void* stream);

/* Copy the header of a device TCB buffer into *hdr_out and check it (magic, version,
 * geometry, section offsets, bytes_total <= buf_bytes).  Synchronises `stream`.
 * Errors: INVALID_ARG, FORMAT, CUDA. */
int spw_format_read(const void* d_buf, uint64_t buf_bytes, spw_format* hdr_out, void* stream);

/* Decompress a TCB buffer into the dense masked weight W_masked (N x K fp16 bits, row
 * stride ldw): kept positions get their stored bits, all others 0x0000.  The inverse of
 * spw_compress ([3LF] §2.1: the stored pattern must reproduce the weight exactly).
 * Asynchronous.  Errors: INVALID_ARG, ALIGNMENT, FORMAT, CUDA. */
int spw_decompress(const spw_format* hdr, const void* d_buf, uint16_t* d_W_out, int ldw,
                   void* stream);

/* Threshold selection ([RMM] §4.1 step 2, §7.3).  For x (B x K fp16, row stride ldx) an
 * entry v takes part iff v != 0 and not |v| < t (compared exactly in fp32); |v| == t and
 * NaN take part.  Column k is active iff some row's entry takes part.  Writes the
 * active-column bitmap d_act_bits[ceil(K/32)] (bit k%32 of word k/32; bits >= K are 0)
 * and the number of active columns to d_count (one uint32).  1 <= B <= 16; t finite and
 * >= 0.  Asynchronous.  Errors: INVALID_ARG, ALIGNMENT, CUDA. */
int spw_select_threshold(const uint16_t* d_x, int B, int K, int ldx, float t,
                         uint32_t* d_act_bits, uint32_t* d_count, void* stream);

/* Top-k selection ([RMM] §5.1).  Score of column k = sum over the B rows of |x_b[k]|,
 * computed exactly (in units of 2^-24); a column holding Inf or NaN scores above every
 * finite score.  The k highest-scoring columns are kept, ties going to the lower index.
 * Writes the bitmap d_act_bits[ceil(K/32)] and, if d_idx is not NULL, the kept indices
 * in ascending order to d_idx[k].  0 <= k <= K, 1 <= B <= 16, K <= 24576.
 * Asynchronous.  Errors: INVALID_ARG, ALIGNMENT, UNSUPPORTED (K too large), CUDA. */
int spw_select_topk(const uint16_t* d_x, int B, int K, int ldx, int k, uint32_t* d_act_bits,
                    uint32_t* d_idx, void* stream);

/* Workspace bytes spw_spmv needs for this format and batch on the current device. */
uint64_t spw_spmv_workspace_bytes(const spw_format* hdr, int B);

/* Decode spMspV ([SPDP] CUDA-core spMspV with activation skipping; [RMM] §4.2 reduced
 * product over the reduction dimension):
 *   y_b[n] = sum_k W[n,k] mask[n,k] x~_b[k],  b < B, n < N,
 *   x~_b[k] = x_b[k] if k is in I, x_b[k] != 0 and not |x_b[k]| < threshold, else 0,
 * with I = the columns set in d_act_bits, or every column when d_act_bits is NULL.
 * Columns with no surviving entry in any row cost no decode work (their weight bytes
 * are still read with the tile's whole-tile copy).  fp32 accumulation, one
 * round-to-nearest-even to fp16 at the end.  x: B x K fp16 (row stride ldx); y: B x N
 * fp16 (row stride ldy).  1 <= B <= 16; threshold finite and >= 0.
 * Workspace: d_ws of at least spw_spmv_workspace_bytes(hdr, B) bytes.  Its first
 * 4 * n_strips bytes are split-K arrival counters: they must be zero before the first
 * call, and every call that completes with device status SPW_OK leaves them zero
 * again; the rest is scratch for fp32 partial sums.  Concurrent calls must not share a
 * workspace.  Results are deterministic (a fixed summation order).  Asynchronous.
 * Errors: INVALID_ARG, ALIGNMENT, FORMAT, BUFFER_TOO_SMALL (workspace), CUDA; a device
 * wait that runs out is reported by spw_last_device_status (SPW_ERR_TIMEOUT), after
 * which y is undefined and the workspace counters must be zeroed again. */
int spw_spmv(const spw_format* hdr, const void* d_buf, const uint16_t* d_x, int B, int ldx,
             float threshold, const uint32_t* d_act_bits, uint16_t* d_y, int ldy, void* d_ws,
             uint64_t ws_bytes, void* stream);

/* Grouped decode: up to SPW_GROUP_MAX (8) independent layers in one launch, e.g. the
 * q/k/v projections that share an input, or gate/up.  Layer l computes exactly what
 * spw_spmv(&hdrs[l], d_bufs[l], d_xs[l], B, ldxs[l], threshold, d_act_bits[l], d_ys[l],
 * ldys[l], ...) computes; all layers share B and the threshold.  One launch has one
 * ramp-up and one tail instead of one per layer: the group's tiles form one
 * concatenated work list split evenly across the persistent grid.  hdrs, d_bufs, d_xs,
 * ldxs, d_act_bits (may itself be NULL: no column sets), d_ys and ldys are host arrays
 * of n entries.  The workspace (spw_spmv_group_workspace_bytes) holds every layer's
 * split-K counters and partial sums, with the counter rules of spw_spmv (all zero before
 * the first call, left zero after each call that completes).  Asynchronous.
 * Errors: as spw_spmv, plus INVALID_ARG for n outside 1..SPW_GROUP_MAX. */
#define SPW_GROUP_MAX 8
uint64_t spw_spmv_group_workspace_bytes(int n, const spw_format* hdrs, int B);
int spw_spmv_group(int n, const spw_format* hdrs, const void* const* d_bufs,
                   const uint16_t* const* d_xs, const int* ldxs,
                   const uint32_t* const* d_act_bits, uint16_t* const* d_ys, const int* ldys,
                   int B, float threshold, void* d_ws, uint64_t ws_bytes, void* stream);

/* Workspace bytes spw_spmv_ffn needs for this gate/up pair and batch (0 if the headers
 * are invalid or their shapes differ). */
uint64_t spw_spmv_ffn_workspace_bytes(const spw_format* hdr_gate, const spw_format* hdr_up, int B);

/* Fused FFN activation for decode ("Reduced Matrix Multiplication" §4.2: H = act(X W_up),
 * keep the high-response channels of H, multiply with the matching rows of W_down; §3.2:
 * SiLU's saturation is where the zeros come from), in the gated form of Llama's FFN:
 *   g_b = fp16(W_gate . x_b), u_b = fp16(W_up . x_b)   (as spw_spmv with threshold 0)
 *   h_b[r] = fp16(SiLU(g_b[r]) * u_b[r]),  SiLU(v) = v / (1 + e^-v), computed in fp32
 *   act bit r set iff the threshold rule keeps h_b[r] for some b (as spw_select_threshold)
 * in one launch: the gate and up layers are one decode group, and once both layers' rows
 * of a 64-row strip are final the warp that finished second computes that strip's h and
 * its two column-set words.  The outputs feed the down projection directly:
 * spw_spmv(down, h, threshold, act_bits) computes only the kept columns.
 *   hdr_gate, hdr_up: same N (intermediate size) and K (hidden size).
 *   d_x:  B x K fp16 input rows at ldx, used as given (no input threshold).
 *   d_h:  B x N fp16 output at ldh >= N (written).  d_act_bits: ceil(N/32) words (written).
 *   d_ws: spw_spmv_ffn_workspace_bytes(...) bytes, zero before the first call and left so
 *         (split-K and pair counters); it also holds g and u.  Concurrent calls must not
 *         share a workspace.
 * Deterministic.  Asynchronous.  Errors: INVALID_ARG (shapes differ, bad B, null
 * pointer, ldh < N, threshold negative, NaN or Inf), ALIGNMENT, FORMAT, BUFFER_TOO_SMALL,
 * CUDA; device-side waits and tile checks as spw_spmv. */
int spw_spmv_ffn(const spw_format* hdr_gate, const void* d_buf_gate, const spw_format* hdr_up,
                 const void* d_buf_up, const uint16_t* d_x, int B, int ldx, float threshold,
                 uint16_t* d_h, int ldh, uint32_t* d_act_bits, void* d_ws, uint64_t ws_bytes,
                 void* stream);

/* Allocation-free decode.  The pages have no counterpart to this call; it exists for
 * callers that cannot call cudaMalloc, for example code running inside a framework that
 * reserved all device memory up front and forbids further allocation, or a path that may
 * not take the device-wide synchronisation an allocation can imply.  It computes exactly
 * what spw_spmv computes (same arguments minus the workspace), using as its split-K
 * workspace a fixed 8 MiB array inside the library's device image instead of caller
 * memory.  It calls no cudaMalloc/cudaFree and no allocating library routine.
 *   - Every GPU that loads the library holds the 8 MiB array until the process exits.
 *   - Requests whose workspace (spw_spmv_workspace_bytes) exceeds
 *     spw_spmv_noalloc_max_scratch_bytes() return SPW_ERR_UNSUPPORTED and launch nothing;
 *     use spw_spmv with a caller workspace for those.
 *   - The first call on a device looks up the array's device address (once per device,
 *     with that device current); make that first call before any stream capture.
 *   - All calls share the one array and each call clears its counters first: calls whose
 *     executions overlap on the GPU (other streams, other threads) race and give wrong
 *     results.  Serialise them.
 * Errors: as spw_spmv, plus UNSUPPORTED for the size limit. */
uint64_t spw_spmv_noalloc_max_scratch_bytes(void);
int spw_spmv_noalloc(const spw_format* hdr, const void* d_buf, const uint16_t* d_x, int B,
                     int ldx, float threshold, const uint32_t* d_act_bits, uint16_t* d_y, int ldy,
                     void* stream);

/* Workspace bytes spw_spmm needs for M rows of X on the current device: 0 when no output
 * tile is split along K (d_ws may then be NULL); otherwise the workspace holds an arrival
 * counter per split tile (its first bytes: zero before the first call, left zero by every
 * call that completes) and fp32 partial tiles.  Tiles are split when the output tiles
 * would leave SMs idle: all of them when they fill less than a wave, the last ones when
 * they need more than one wave but fewer than two (see spw_spmm_plan).  0 for an invalid
 * header or M < 1. */
uint64_t spw_spmm_workspace_bytes(const spw_format* hdr, int M);

/* The launch plan spw_spmm uses for this format and M on a device with sm_count SMs
 * (sm_count <= 0: the current device).  token_tile tokens (a multiple of 16) per output
 * tile, token_tiles x weight_tiles output tiles of 128 weight rows -- or, when cta_pair
 * is 1, of 256 weight rows each computed by a cluster of two CTAs on an SM pair (one
 * tcgen05 cta_group::2 MMA: each CTA decodes its 128 rows and loads half the token
 * tile, so X crosses L2 half as often); the first whole_tiles tiles run whole and the
 * others in k_parts parts along K (k_parts = 1: no split); ctas = (whole_tiles + (tiles
 * - whole_tiles) * k_parts) * (cta_pair ? 2 : 1); workspace_bytes as
 * spw_spmm_workspace_bytes.  Pair mode is used only when the environment sets
 * SPW_SPMM_PAIR=1, and then for M >= 256 and N > 128 (with sm_count > 0 it assumes
 * sm_count / 2 SM pairs).  Host only, no launch.
 * Errors: INVALID_ARG, FORMAT, CUDA (no device and sm_count <= 0). */
typedef struct {
    int32_t token_tile, token_tiles, weight_tiles, k_parts, whole_tiles, ctas;
    int32_t cta_pair;  /* 1: each tile is 256 weight rows on an SM pair (two CTAs) */
    int32_t reserved;  /* 0 */
    uint64_t workspace_bytes;
} spw_spmm_plan_info;
int spw_spmm_plan(const spw_format* hdr, int M, int sm_count, spw_spmm_plan_info* out);

/* Prefill SpMM ([SPDP] Tensor-Core SpMM; [3LF] §1: tensor cores take only 2:4 sparsity,
 * so unstructured tiles are decoded to dense in shared memory and fed to dense MMA):
 *   Y[m,n] = sum_k X[m,k] W[n,k] mask[n,k],  m < M, n < N.
 * X: M x K fp16 (row stride ldx); Y: M x N fp16 (row stride ldy).  tcgen05 MMA with
 * fp32 accumulation in tensor memory, one round-to-nearest-even to fp16.  M >= 0
 * (M == 0 does nothing and then X and Y may be NULL).  The decoded weight tile is the MMA's
 * A operand (128 rows), X its B operand (up to 512 tokens per tile).  A dropped weight is
 * an explicit zero in the product, so a non-finite X entry reaches every output row
 * (0 * Inf = NaN, as in a dense product).  Deterministic.  Asynchronous.
 * Errors: INVALID_ARG, ALIGNMENT, FORMAT, BUFFER_TOO_SMALL (workspace), CUDA; device
 * timeouts as for spw_spmv. */
int spw_spmm(const spw_format* hdr, const void* d_buf, const uint16_t* d_X, int M, int ldx,
             uint16_t* d_Y, int ldy, void* d_ws, uint64_t ws_bytes, void* stream);

/* Token grouping ("Reduced Matrix Multiplication" §6.1: tokens whose channel sets are the
 * same or alike are grouped, each group running its own dense product; the pages leave
 * the similarity open, and this is the plainest reading at the stored tile width):
 *   signature of token m: bit kt (bit kt % 64 of word kt / 64, words = ceil(ceil(K/64)
 *     / 64)) is set iff the threshold rule keeps some X[m,k], 64 kt <= k < 64 kt + 64;
 *   order: tokens sorted by signature (words compared from word 0 as unsigned 64-bit
 *     integers), equal signatures by lower token index;
 *   outputs: d_perm[r] = the token at position r (M words); row r of d_Xg (M rows at
 *     ldxg >= K, a multiple of 8) = x~ of that token (entries the rule drops written as
 *     +0, columns K..ldxg-1 as 0); d_tile_sig[j * words + w] = OR of the signatures of
 *     positions j T .. min((j+1) T, M) - 1 (T = token_tile), i.e. the k-tiles token tile
 *     j has to visit.
 * 1 <= M <= 16384, 1 <= K <= 16384, token_tile >= 1, t finite and >= 0.  d_ws: scratch of
 * spw_group_tokens_workspace_bytes(M, K) bytes (no state kept between calls).
 * Deterministic.  Asynchronous.  Errors: INVALID_ARG, ALIGNMENT (any pointer not 16-byte
 * aligned), UNSUPPORTED (M or K too large), BUFFER_TOO_SMALL, CUDA. */
uint64_t spw_group_tokens_workspace_bytes(int M, int K);
int spw_group_tokens(const uint16_t* d_X, int M, int K, int ldx, float t, int token_tile,
                     uint16_t* d_Xg, int ldxg, uint32_t* d_perm, uint64_t* d_tile_sig, void* d_ws,
                     uint64_t ws_bytes, void* stream);

/* Workspace bytes of spw_spmm_tokens for M tokens (0 for an invalid header, M < 1, or
 * M or K above 16384). */
uint64_t spw_spmm_tokens_workspace_bytes(const spw_format* hdr, int M);

/* The launch plan of spw_spmm_tokens, as spw_spmm_plan reports it for spw_spmm (never
 * SM-pair tiles); workspace_bytes is spw_spmm_tokens_workspace_bytes.  token_tile is the
 * T of its token grouping.  Errors: as spw_spmm_plan, plus UNSUPPORTED (M or K too
 * large). */
int spw_spmm_tokens_plan(const spw_format* hdr, int M, int sm_count, spw_spmm_plan_info* out);

/* Prefill with a per-token index set ("Reduced Matrix Multiplication" §4.2, each token
 * keeping its own channels; §6.1-§6.2, token grouping):
 *   Y[m,n] = sum_k x~[m,k] W[n,k] mask[n,k],
 *   x~[m,k] = X[m,k] if X[m,k] != 0 and not |X[m,k]| < threshold, else 0,
 * i.e. row m is what spw_spmv computes for token m alone.  The call groups the tokens
 * as spw_group_tokens does, with T = the token tile of spw_spmm_tokens_plan, into the
 * workspace, then runs the prefill product (as spw_spmm) on the grouped rows, where
 * every token tile visits only the k-tiles of its tile signature (a skipped k-tile holds
 * no kept entry of the tile's tokens) and its rows are written back to their tokens' rows
 * of Y.  Without a shared zero pattern among the tokens of a tile nothing is skipped
 * and the call costs spw_spmm plus the grouping (a read of X, a write of x~).
 * Non-finite kept entries reach every output row, as in spw_spmm.  M >= 0 (M == 0 does
 * nothing), M and K <= 16384, threshold finite and >= 0.  d_ws: at least
 * spw_spmm_tokens_workspace_bytes(hdr, M) bytes; its first bytes are the split-K
 * counters of spw_spmm (zero before the first call, left zero by each call that
 * completes), then the grouped input, perm, tile signatures and grouping scratch.
 * Deterministic.  Asynchronous.  Errors: as spw_spmm, plus UNSUPPORTED (M or K too
 * large) and INVALID_ARG for a bad threshold or a NULL workspace. */
int spw_spmm_tokens(const spw_format* hdr, const void* d_buf, const uint16_t* d_X, int M, int ldx,
                    float threshold, uint16_t* d_Y, int ldy, void* d_ws, uint64_t ws_bytes,
                    void* stream);

/* 2:4 + residual split ("Accelerating LLM GPU inference with moderately unstructured
 * sparse weight matrices", abstract and §1: a 2:4 layer for the sparse tensor cores and a
 * residual layer that keeps the SpMM exact; the pages' slot-filling middle layer is not
 * built).  In every group of four columns 4g .. 4g+3 of a row, the first two kept
 * weights (mask != 0, column order) form the 2:4 part; every further kept weight of the
 * group is set in the residual mask d_mask_r (N x K u8 at ld_mask_r, written: 1 for a
 * residual weight, 0 elsewhere), which the caller compresses into an ordinary TCB v1
 * buffer (spw_format_query / spw_compress with the same W) for spw_spmm24.
 * d_s24 (spw_s24_bytes(N, K) bytes, written) holds the 2:4 part per 64 x 64 tile t =
 * strip * n_ktiles + k-tile:
 *   values at t * 4096: row r's 32 halves -- for each group of four columns, the values
 *     at its two selected positions, lower position first -- fill bytes 64 r .. 64 r +
 *     63, the 16-byte chunk c (groups 4c .. 4c+3) at position c ^ ((r >> 1) & 3);
 *   metadata at n_tiles * 4096 + t * 1024: 16 bytes per lane L (0..63) = {word for the
 *     tile's columns 0-31, word for columns 32-63, 0, 0}; a word holds row 16 (L/16) +
 *     L%8 in bits 0-15 and that row + 8 in bits 16-31, for columns 32 j + 16 ((L/8) % 2)
 *     .. +15 of its half j as four 4-bit groups (group g at bits 4g of the half: the
 *     first selected position in bits 0-1, the second in bits 2-3, first < second);
 *   padding at n_tiles * 5120: 1024 bytes of metadata for a tile with no kept weight.
 * A group with fewer than two kept weights selects the lowest free positions with value
 * 0; rows past N and columns past K keep nothing.  W: N x K fp16 at ldw; mask: N x K u8
 * at ld_mask.  Asynchronous.  Errors: INVALID_ARG, ALIGNMENT (d_s24), BUFFER_TOO_SMALL,
 * UNSUPPORTED (too many tiles), CUDA. */
uint64_t spw_s24_bytes(int N, int K);
int spw_split24(const uint16_t* d_W, int ldw, const uint8_t* d_mask, int ld_mask, int N, int K,
                void* d_s24, uint64_t s24_bytes, uint8_t* d_mask_r, int ld_mask_r, void* stream);

/* Workspace bytes and launch plan of spw_spmm24 (as spw_spmm's, with at most 256 tokens
 * per tile and no SM-pair tiles); hdr_r is the residual's TCB header. */
uint64_t spw_spmm24_workspace_bytes(const spw_format* hdr_r, int M);
int spw_spmm24_plan(const spw_format* hdr_r, int M, int sm_count, spw_spmm_plan_info* out);

/* Prefill on the 2:4 + residual split ([3LF] layers (i) and (iii)):
 *   Y[m,n] = sum_k X[m,k] (S[n,k] + R[n,k]),  S + R = W masked (spw_split24),
 * where S (d_s24) runs on the sparse tensor cores (tcgen05.mma.sp, K = 32 per
 * instruction, metadata in tensor memory) and R (hdr_r / d_buf_r, a TCB v1 buffer of the
 * residual) is decoded in shared memory and runs as dense MMA into the same fp32
 * accumulator; a k-tile whose residual tiles are empty costs no decode and no dense MMA.
 * X, Y, M, ldx, ldy, workspace, determinism and errors as spw_spmm; d_s24 must be the
 * buffer spw_split24 wrote for the same weight and mask (same N and K as hdr_r; only its
 * size, spw_s24_bytes(N, K) bytes, can be checked: BUFFER_TOO_SMALL otherwise) and be
 * 16-byte aligned. */
int spw_spmm24(const spw_format* hdr_r, const void* d_buf_r, const void* d_s24, uint64_t s24_bytes,
               const uint16_t* d_X, int M, int ldx, uint16_t* d_Y, int ldy, void* d_ws,
               uint64_t ws_bytes, void* stream);

/* Workspace bytes spw_spmv_tc needs (the rules of spw_spmm_workspace_bytes with M = B);
 * 0 for B outside 1..16. */
uint64_t spw_spmv_tc_workspace_bytes(const spw_format* hdr, int B);

/* Decode on tensor cores ([SPDP] reads "hybrid" as a runtime choice of decode path;
 * [RMM] §4.2 reduced product): computes what spw_spmv computes -- same arguments, the
 * threshold rule and column set applied to x in shared memory -- with the decoded weight
 * tiles as the A operand of tcgen05 MMA (M = 128 weight rows, N = B rounded up to 16).
 * Its time hardly changes with B, while spw_spmv's per-row multiply-adds grow with B:
 * measured faster than spw_spmv from 14 rows on the Llama-7B shapes (from 8 on the
 * 4096 x 4096 one); spw_spmv_auto makes that choice.  As in spw_spmm, a non-finite x~ entry reaches every row, including rows whose weight
 * in that column is dropped.  Workspace: spw_spmv_tc_workspace_bytes (zero-initialised
 * counters, left zero).  Inactive columns are decoded but contribute zeros.  Deterministic.
 * Asynchronous.  Errors: as spw_spmv. */
int spw_spmv_tc(const spw_format* hdr, const void* d_buf, const uint16_t* d_x, int B, int ldx,
                float threshold, const uint32_t* d_act_bits, uint16_t* d_y, int ldy, void* d_ws,
                uint64_t ws_bytes, void* stream);

/* Decode with the path chosen by batch size ([SPDP] abstract: "hybrid" decoding, read as
 * a runtime choice between the decode paths): spw_spmv_tc for batches of
 * spw_spmv_auto_path(B) == 1, spw_spmv otherwise, with the same arguments.  The tensor-core
 * path is taken from the batch where it measured faster on every Llama-7B shape at 50 %
 * sparsity (14 rows); the choice depends on B alone, is made on the host and costs no
 * device read.  The result is that of the path taken: what spw_spmv computes,
 * deterministic, except that on the tensor-core path a non-finite x~ entry reaches every
 * row (see spw_spmv_tc).
 *   spw_spmv_auto_path(B): 0 (CUDA cores), 1 (tensor cores), -1 for B outside 1..16.
 *   spw_spmv_auto_workspace_bytes(hdr, B): the workspace of the path taken, with that
 *   path's counter rules (zero before the first call, left zero); 0 for B outside 1..16.
 * Asynchronous.  Errors: those of the path taken; INVALID_ARG for B outside 1..16. */
int spw_spmv_auto_path(int B);
uint64_t spw_spmv_auto_workspace_bytes(const spw_format* hdr, int B);
int spw_spmv_auto(const spw_format* hdr, const void* d_buf, const uint16_t* d_x, int B, int ldx,
                  float threshold, const uint32_t* d_act_bits, uint16_t* d_y, int ldy, void* d_ws,
                  uint64_t ws_bytes, void* stream);

/* Synchronise `stream`, then read and clear the library's device status word for the
 * current device: *code = SPW_OK, SPW_ERR_TIMEOUT if a bounded device wait ran out, or
 * SPW_ERR_FORMAT if a product kernel met a tile that disagrees with its header (see
 * "Buffer contents"), since the last read.  Errors: INVALID_ARG, CUDA. */
int spw_last_device_status(void* stream, int* code);

#ifdef __cplusplus
}
#endif

#endif /* SPW_H */
