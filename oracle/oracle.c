/*
 * oracle.c -- reference CPU implementation of the sparse-weight SpMV / SpMM path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the CPU-baseline
 * leg of the benchmark load this file (as liboracle.so through oracle/__init__.py).
 * The CUDA library never links, loads or calls it, and the two share no code, header,
 * table or constant: this file declares everything it uses itself.
 *
 * It is plain, single-threaded C.  Floating point is fp64.  Loops follow the
 * definitions directly, with no blocking, fusion or reordering.
 *
 * Sources (web pages, cited by title and section):
 *   [SPDP] "Unified Static-Dynamic Pruning for Efficient LLM Inference" (summary of
 *          arXiv 2607.21985), abstract and method notes.  Unstructured static weight
 *          pruning is combined with input-adaptive dynamic pruning.  The weight is held in
 *          a Tiled-Column-wise Bitmap Compressed (Tiled-CBC) format.  A CUDA-core spMspV
 *          kernel skips activations at run time, and a Tensor-Core SpMM kernel serves
 *          prefill.  The page names the format but gives no byte layout.
 *   [RMM]  "Reduced Matrix Multiplication" article (hotelren.com/news/4430107; its
 *          printed title line is an extraction artefact).  Section 4.1 gives the four
 *          steps (score, select, multiply on the subset, map back).  Section 4.2 gives
 *          the reduced product Y[:, I] = X @ W[:, I] and, for an FFN, keeping only the
 *          high-response channels of H and the matching rows of W_down.  Section 5.1
 *          ranks channels by mean |activation| and keeps a top-k, sorted by index.
 *   [3LF]  "Accelerating LLM GPU inference with moderately unstructured sparse weight
 *          matrices" (translation of arXiv 2607.08786).  Section 1 requires the stored
 *          format to give a correct SpMM, i.e. the product with the masked dense weight.
 *          Section 2.1 gives the prefill [BL, H] and decode [B, H] activation shapes,
 *          and says the sparsity pattern is precomputed and stored in a dedicated format.
 *
 * Functions and the passage each follows:
 *   orc_half_to_double   IEEE-754 binary16 decoding (the weights and activations are fp16).
 *   orc_tcb_query        size of the TCB v1 buffer for a mask            [SPDP] format.
 *   orc_tcb_encode       reference TCB v1 encoder (the layout's definition) [SPDP] format.
 *   orc_tcb_decode       reference TCB v1 decoder (inverse of the above)  [3LF] §2.1.
 *   orc_select_threshold active-column set for the threshold rule       [RMM] §4.1-4.2.
 *   orc_select_topk      active-column set for top-k by summed |x|       [RMM] §5.1.
 *   orc_spmv             y_b = W_masked . x~_b in fp64                   [RMM] §4.2, [3LF] §1.
 *   orc_spmm             Y = X . W_masked^T in fp64 (optionally some rows) [3LF] §1, §2.1.
 *   orc_double_to_half   IEEE-754 binary16 encoding, round to nearest, ties to even
 *   orc_round_to_half    (and its element-wise form).
 *   orc_silu_mul         h = fp16(SiLU(g) * u) for the gated FFN    [RMM] §4.2, §3.2.
 *   orc_spmm_tokens      Y = X~ . W_masked^T, each token its own index set [RMM] §4.2, §6.1.
 *   orc_token_groups     token order and token-tile k-tile sets      [RMM] §6.1.
 *   orc_split24          2:4 part and residual of a mask             [3LF] abstract, §1.
 *
 * Pins: tests/test_oracle_*.py check every function against things fixed outside this
 * file: numpy's binary16 decoder over all 65536 bit patterns, hand-derived TCB buffers
 * (tests/golden/), exact rational arithmetic on small products, brute force selection,
 * and closed forms (identity, diagonal, all-zero, one nonzero per row).
 *
 * ---------------------------------------------------------------------------------------
 * TCB v1 -- the tiled column-bitmap layout.  The pages only name the format, so this
 * layout is this project's reading of it.  All integers are little-endian.
 *
 *   The weight W is N x K, row-major (row n = output feature, column k = input feature).
 *   A strip is 64 consecutive rows, and a tile is one strip times 64 consecutive
 *   columns.  n_strips = ceil(N / 64) and n_ktiles = ceil(K / 64).  Tile t = s *
 *   n_ktiles + kt covers rows [64 s, 64 s + 64) and columns [64 kt, 64 kt + 64).
 *
 *   [header, 256 B]  u32 magic 0x31424354, u32 version 1, u32 N, u32 K, u32 TN = 64,
 *                    u32 TK = 64, u32 n_strips, u32 n_ktiles, u64 nnz, u64 bytes_total,
 *                    u64 off_bitmaps, u64 off_tileptr, u64 off_values,
 *                    u32 max_tile_units, u32 0.  Bytes 80..255 are zero.
 *   [bitmaps]        u64 bitmap[n_strips][n_ktiles * 64] at off_bitmaps = 256.  Bit r of
 *                    bitmap[s][k] is set iff row 64 s + r exists, column k exists and
 *                    mask[64 s + r][k] != 0.
 *   [tileptr]        u32 tileptr[n_strips * n_ktiles + 1] at off_tileptr, the first
 *                    multiple of 256 after the bitmaps.  tileptr[t] is where tile t's
 *                    values start, in 16-byte units counted from off_values;
 *                    tileptr[n_strips * n_ktiles] is the total.
 *   [values]         u16 at off_values, the first multiple of 256 after tileptr.
 *                    Tile t holds the kept weights of its columns in ascending column
 *                    order, and within a column in ascending row order (the order of the
 *                    set bits).  The weight's fp16 bits are copied unchanged.  The tile
 *                    is then padded with 0x0000 to a multiple of 8 values (16 bytes).
 *   bytes_total = off_values + 16 * tileptr[n_strips * n_ktiles].
 *   max_tile_units = the largest tileptr[t + 1] - tileptr[t].
 *   Every byte not named above, up to bytes_total, is zero.
 * ---------------------------------------------------------------------------------------
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_ERR_ARG 1
#define ORC_ERR_BUFFER_TOO_SMALL 3
#define ORC_ERR_FORMAT 4

#define TCB_MAGIC 0x31424354u /* the bytes "TCB1" */
#define TCB_VERSION 1u
#define TCB_ROWS 64    /* rows per strip */
#define TCB_COLS 64    /* columns per tile */
#define TCB_HEADER 256 /* header bytes */

/* ---------------------------------------------------------------- binary16 decoding */

/* Value of an IEEE-754 binary16 bit pattern: 1 sign bit, 5 exponent bits (bias 15),
 * 10 fraction bits.  Exponent 0 gives zero or a subnormal (fraction * 2^-24); exponent
 * 31 gives infinity or NaN; otherwise (1024 + fraction) * 2^(exponent - 25). */
double orc_half_to_double(uint16_t h) {
    int negative = (h >> 15) & 1;
    int exponent = (h >> 10) & 0x1f;
    int fraction = h & 0x3ff;
    double magnitude;
    if (exponent == 0)
        magnitude = ldexp((double)fraction, -24);
    else if (exponent == 31)
        magnitude = fraction ? NAN : INFINITY;
    else
        magnitude = ldexp((double)(1024 + fraction), exponent - 25);
    return negative ? -magnitude : magnitude;
}

/* ---------------------------------------------------------------- little-endian I/O */

static void put_u32(uint8_t* p, uint32_t v) {
    for (int i = 0; i < 4; i++) p[i] = (uint8_t)(v >> (8 * i));
}
static void put_u64(uint8_t* p, uint64_t v) {
    for (int i = 0; i < 8; i++) p[i] = (uint8_t)(v >> (8 * i));
}
static uint32_t get_u32(const uint8_t* p) {
    uint32_t v = 0;
    for (int i = 0; i < 4; i++) v |= (uint32_t)p[i] << (8 * i);
    return v;
}
static uint64_t get_u64(const uint8_t* p) {
    uint64_t v = 0;
    for (int i = 0; i < 8; i++) v |= (uint64_t)p[i] << (8 * i);
    return v;
}

static uint64_t round_up(uint64_t v, uint64_t a) { return (v + a - 1) / a * a; }

/* ---------------------------------------------------------------- TCB v1 geometry */

typedef struct {
    uint32_t n_strips, n_ktiles;
    uint64_t off_bitmaps, off_tileptr, off_values;
} tcb_sections;

static tcb_sections tcb_geometry(int N, int K) {
    tcb_sections g;
    g.n_strips = (uint32_t)((N + TCB_ROWS - 1) / TCB_ROWS);
    g.n_ktiles = (uint32_t)((K + TCB_COLS - 1) / TCB_COLS);
    uint64_t n_tiles = (uint64_t)g.n_strips * g.n_ktiles;
    g.off_bitmaps = TCB_HEADER;
    g.off_tileptr = round_up(g.off_bitmaps + 8 * n_tiles * TCB_COLS, 256);
    g.off_values = round_up(g.off_tileptr + 4 * (n_tiles + 1), 256);
    return g;
}

static int kept(const uint8_t* mask, int ld_mask, int N, int K, int n, int k) {
    return n < N && k < K && mask[(size_t)n * ld_mask + k] != 0;
}

/* Number of kept weights in tile (s, kt). */
static uint64_t tile_count(const uint8_t* mask, int ld_mask, int N, int K, int s, int kt) {
    uint64_t c = 0;
    for (int k = kt * TCB_COLS; k < (kt + 1) * TCB_COLS; k++)
        for (int r = 0; r < TCB_ROWS; r++) c += kept(mask, ld_mask, N, K, s * TCB_ROWS + r, k);
    return c;
}

static int check_dims(int N, int K, int ld, int ld_mask) {
    if (N < 1 || K < 1 || ld < K || ld_mask < K) return ORC_ERR_ARG;
    return ORC_OK;
}

int orc_tcb_query(const uint8_t* mask, int N, int K, int ld_mask, uint64_t* bytes_total,
                  uint64_t* nnz) {
    if (!mask || !bytes_total || !nnz || check_dims(N, K, K, ld_mask)) return ORC_ERR_ARG;
    tcb_sections g = tcb_geometry(N, K);
    uint64_t units = 0, count = 0;
    for (uint32_t s = 0; s < g.n_strips; s++)
        for (uint32_t kt = 0; kt < g.n_ktiles; kt++) {
            uint64_t c = tile_count(mask, ld_mask, N, K, (int)s, (int)kt);
            count += c;
            units += (c + 7) / 8;
        }
    *bytes_total = g.off_values + 16 * units;
    *nnz = count;
    return ORC_OK;
}

int orc_tcb_encode(const uint16_t* W, int ldw, const uint8_t* mask, int ld_mask, int N, int K,
                   uint8_t* buf, uint64_t buf_bytes) {
    if (!W || !mask || !buf || check_dims(N, K, ldw, ld_mask)) return ORC_ERR_ARG;
    uint64_t bytes_total, nnz;
    orc_tcb_query(mask, N, K, ld_mask, &bytes_total, &nnz);
    if (buf_bytes < bytes_total) return ORC_ERR_BUFFER_TOO_SMALL;
    tcb_sections g = tcb_geometry(N, K);
    uint64_t n_tiles = (uint64_t)g.n_strips * g.n_ktiles;
    memset(buf, 0, bytes_total);

    /* bitmaps */
    for (uint32_t s = 0; s < g.n_strips; s++)
        for (uint64_t k = 0; k < (uint64_t)g.n_ktiles * TCB_COLS; k++) {
            uint64_t word = 0;
            for (int r = 0; r < TCB_ROWS; r++)
                if (kept(mask, ld_mask, N, K, (int)(s * TCB_ROWS + r), (int)k)) word |= 1ull << r;
            put_u64(buf + g.off_bitmaps + 8 * (s * (uint64_t)g.n_ktiles * TCB_COLS + k), word);
        }

    /* tile pointers and values */
    uint64_t unit = 0;
    uint32_t max_units = 0;
    for (uint32_t s = 0; s < g.n_strips; s++)
        for (uint32_t kt = 0; kt < g.n_ktiles; kt++) {
            uint64_t t = (uint64_t)s * g.n_ktiles + kt;
            put_u32(buf + g.off_tileptr + 4 * t, (uint32_t)unit);
            uint8_t* out = buf + g.off_values + 16 * unit;
            uint64_t j = 0;
            for (int k = (int)kt * TCB_COLS; k < ((int)kt + 1) * TCB_COLS; k++)
                for (int r = 0; r < TCB_ROWS; r++) {
                    int n = (int)s * TCB_ROWS + r;
                    if (!kept(mask, ld_mask, N, K, n, k)) continue;
                    uint16_t bits = W[(size_t)n * ldw + k];
                    out[2 * j] = (uint8_t)(bits & 0xff);
                    out[2 * j + 1] = (uint8_t)(bits >> 8);
                    j++;
                }
            uint64_t tile_units = (j + 7) / 8; /* the padding is already zero */
            if (tile_units > max_units) max_units = (uint32_t)tile_units;
            unit += tile_units;
        }
    put_u32(buf + g.off_tileptr + 4 * n_tiles, (uint32_t)unit);

    /* header */
    put_u32(buf + 0, TCB_MAGIC);
    put_u32(buf + 4, TCB_VERSION);
    put_u32(buf + 8, (uint32_t)N);
    put_u32(buf + 12, (uint32_t)K);
    put_u32(buf + 16, TCB_ROWS);
    put_u32(buf + 20, TCB_COLS);
    put_u32(buf + 24, g.n_strips);
    put_u32(buf + 28, g.n_ktiles);
    put_u64(buf + 32, nnz);
    put_u64(buf + 40, bytes_total);
    put_u64(buf + 48, g.off_bitmaps);
    put_u64(buf + 56, g.off_tileptr);
    put_u64(buf + 64, g.off_values);
    put_u32(buf + 72, max_units);
    return ORC_OK;
}

/* Decode a TCB v1 buffer into the dense masked weight: kept positions get their stored
 * fp16 bits, dropped positions get 0x0000.  W_out is N x K with row stride ldw. */
int orc_tcb_decode(const uint8_t* buf, uint64_t buf_bytes, uint16_t* W_out, int ldw) {
    if (!buf || !W_out || buf_bytes < TCB_HEADER) return ORC_ERR_ARG;
    if (get_u32(buf) != TCB_MAGIC || get_u32(buf + 4) != TCB_VERSION) return ORC_ERR_FORMAT;
    int N = (int)get_u32(buf + 8), K = (int)get_u32(buf + 12);
    if (N < 1 || K < 1 || ldw < K) return ORC_ERR_ARG;
    if (get_u32(buf + 16) != TCB_ROWS || get_u32(buf + 20) != TCB_COLS) return ORC_ERR_FORMAT;
    tcb_sections g = tcb_geometry(N, K);
    if (get_u32(buf + 24) != g.n_strips || get_u32(buf + 28) != g.n_ktiles ||
        get_u64(buf + 48) != g.off_bitmaps || get_u64(buf + 56) != g.off_tileptr ||
        get_u64(buf + 64) != g.off_values)
        return ORC_ERR_FORMAT;
    uint64_t bytes_total = get_u64(buf + 40);
    if (bytes_total > buf_bytes || bytes_total < g.off_values) return ORC_ERR_FORMAT;
    uint64_t n_tiles = (uint64_t)g.n_strips * g.n_ktiles;

    for (int n = 0; n < N; n++)
        for (int k = 0; k < K; k++) W_out[(size_t)n * ldw + k] = 0;

    for (uint32_t s = 0; s < g.n_strips; s++)
        for (uint32_t kt = 0; kt < g.n_ktiles; kt++) {
            uint64_t t = (uint64_t)s * g.n_ktiles + kt;
            uint64_t start = get_u32(buf + g.off_tileptr + 4 * t);
            uint64_t end = get_u32(buf + g.off_tileptr + 4 * (t + 1));
            if (end < start || g.off_values + 16 * end > bytes_total) return ORC_ERR_FORMAT;
            const uint8_t* in = buf + g.off_values + 16 * start;
            uint64_t j = 0;
            for (int k = (int)kt * TCB_COLS; k < ((int)kt + 1) * TCB_COLS; k++) {
                uint64_t word = get_u64(buf + g.off_bitmaps +
                                        8 * ((uint64_t)s * g.n_ktiles * TCB_COLS + (uint64_t)k));
                for (int r = 0; r < TCB_ROWS; r++) {
                    if (!((word >> r) & 1)) continue;
                    int n = (int)s * TCB_ROWS + r;
                    if (n >= N || k >= K) return ORC_ERR_FORMAT;
                    if (j >= 8 * (end - start)) return ORC_ERR_FORMAT;
                    W_out[(size_t)n * ldw + k] = (uint16_t)(in[2 * j] | (in[2 * j + 1] << 8));
                    j++;
                }
            }
            if ((j + 7) / 8 != end - start) return ORC_ERR_FORMAT;
        }
    (void)n_tiles;
    return ORC_OK;
}

/* ---------------------------------------------------------------- selection */

/* The per-entry rule for the threshold t: an activation v takes part iff it is not zero
 * and |v| is not below t.  |v| == t takes part; NaN takes part (it is not zero and not
 * below t), so it propagates as it would in a dense product. */
static int passes_threshold(double v, double t) { return v != 0.0 && !(fabs(v) < t); }

static int valid_threshold(float t) { return t >= 0.0f && !isinf(t); } /* NaN fails t >= 0 */

/* Column k is active iff some batch row's entry passes the threshold (the union over
 * the batch; [RMM] §7.3 shares one channel set across a block of tokens). */
int orc_select_threshold(const uint16_t* x, int B, int K, int ldx, float t, uint32_t* act_bits,
                         uint32_t* count) {
    if (!x || !act_bits || !count || B < 1 || K < 1 || ldx < K || !valid_threshold(t))
        return ORC_ERR_ARG;
    int words = (K + 31) / 32;
    for (int w = 0; w < words; w++) act_bits[w] = 0;
    uint32_t c = 0;
    for (int k = 0; k < K; k++) {
        int active = 0;
        for (int b = 0; b < B; b++)
            if (passes_threshold(orc_half_to_double(x[(size_t)b * ldx + k]), (double)t)) active = 1;
        if (active) {
            act_bits[k / 32] |= 1u << (k % 32);
            c++;
        }
    }
    *count = c;
    return ORC_OK;
}

/* Top-k by channel importance, [RMM] §5.1: the score of column k is the sum over the
 * batch of |x_b[k]| (the page uses the mean; the mean ranks the same).  Every fp16 value
 * is a multiple of 2^-24 below 2^16, so a sum of up to 2^20 of them is exact in fp64.
 * A column with a non-finite entry scores +infinity.  Columns are ranked by score,
 * highest first, ties by lower index; the first k are kept and listed in ascending
 * index order, as on the page. */
typedef struct {
    double score;
    int index;
} scored_column;

static int by_rank(const void* a, const void* b) {
    const scored_column* p = (const scored_column*)a;
    const scored_column* q = (const scored_column*)b;
    if (p->score > q->score) return -1;
    if (p->score < q->score) return 1;
    return (p->index > q->index) - (p->index < q->index);
}

int orc_select_topk(const uint16_t* x, int B, int K, int ldx, int k, uint32_t* act_bits,
                    uint32_t* idx) {
    if (!x || !act_bits || B < 1 || K < 1 || ldx < K || k < 0 || k > K) return ORC_ERR_ARG;
    scored_column* cols = (scored_column*)malloc(sizeof(scored_column) * (size_t)K);
    if (!cols) return ORC_ERR_ARG;
    for (int c = 0; c < K; c++) {
        double s = 0.0;
        int finite = 1;
        for (int b = 0; b < B; b++) {
            double v = orc_half_to_double(x[(size_t)b * ldx + c]);
            if (!isfinite(v)) finite = 0;
            s += fabs(v);
        }
        cols[c].score = finite ? s : INFINITY;
        cols[c].index = c;
    }
    qsort(cols, (size_t)K, sizeof(scored_column), by_rank);
    int words = (K + 31) / 32;
    for (int w = 0; w < words; w++) act_bits[w] = 0;
    for (int i = 0; i < k; i++) act_bits[cols[i].index / 32] |= 1u << (cols[i].index % 32);
    free(cols);
    if (idx) {
        int j = 0;
        for (int c = 0; c < K; c++)
            if ((act_bits[c / 32] >> (c % 32)) & 1) idx[j++] = (uint32_t)c;
    }
    return ORC_OK;
}

/* ---------------------------------------------------------------- products */

/* Decode: y_b[n] = sum over k of W[n,k] * mask[n,k] * x~_b[k], where x~_b[k] = x_b[k] if
 * column k is in the set I, x_b[k] != 0 and |x_b[k]| is not below t, and 0 otherwise.
 * I is the caller's column set act_bits, or every column when act_bits is NULL.  This
 * is the reduced product of [RMM] §4.2 over the reduction dimension, which must equal
 * the masked dense product ([3LF] §1).  y is B x N, row b at y + b * N. */
int orc_spmv(const uint16_t* W, int ldw, const uint8_t* mask, int ld_mask, int N, int K,
             const uint16_t* x, int B, int ldx, float t, const uint32_t* act_bits, double* y) {
    if (!W || !mask || !x || !y || check_dims(N, K, ldw, ld_mask) || B < 1 || ldx < K ||
        !valid_threshold(t))
        return ORC_ERR_ARG;
    for (int b = 0; b < B; b++)
        for (int n = 0; n < N; n++) {
            double acc = 0.0;
            for (int k = 0; k < K; k++) {
                if (!mask[(size_t)n * ld_mask + k]) continue;
                if (act_bits && !((act_bits[k / 32] >> (k % 32)) & 1)) continue;
                double v = orc_half_to_double(x[(size_t)b * ldx + k]);
                if (!passes_threshold(v, (double)t)) continue;
                acc += orc_half_to_double(W[(size_t)n * ldw + k]) * v;
            }
            y[(size_t)b * N + n] = acc;
        }
    return ORC_OK;
}

/* Prefill: Y[m,n] = sum over k of X[m,k] * W[n,k] * mask[n,k] ([3LF] §1 and §2.1).
 * When rows is not NULL only the listed rows of X are computed, and Y holds n_rows x N
 * results in the listed order; otherwise Y is M x N (n_rows is then M). */
int orc_spmm(const uint16_t* W, int ldw, const uint8_t* mask, int ld_mask, int N, int K,
             const uint16_t* X, int M, int ldx, const int* rows, int n_rows, double* Y) {
    if (!W || !mask || !X || !Y || check_dims(N, K, ldw, ld_mask) || M < 0 || ldx < K)
        return ORC_ERR_ARG;
    int count = rows ? n_rows : M;
    for (int i = 0; i < count; i++) {
        int m = rows ? rows[i] : i;
        if (m < 0 || m >= M) return ORC_ERR_ARG;
        for (int n = 0; n < N; n++) {
            double acc = 0.0;
            for (int k = 0; k < K; k++)
                if (mask[(size_t)n * ld_mask + k])
                    acc += orc_half_to_double(X[(size_t)m * ldx + k]) *
                           orc_half_to_double(W[(size_t)n * ldw + k]);
            Y[(size_t)i * N + n] = acc;
        }
    }
    return ORC_OK;
}

/* IEEE-754 binary16 encoding of v: round to nearest, ties to even; overflow to infinity,
 * NaN to a quiet NaN with the sign kept, gradual underflow to subnormals and zero. */
uint16_t orc_double_to_half(double v) {
    uint16_t sign = signbit(v) ? 0x8000u : 0u;
    if (isnan(v)) return (uint16_t)(sign | 0x7E00u);
    double a = fabs(v);
    if (isinf(a)) return (uint16_t)(sign | 0x7C00u);
    /* a = m * 2^e with m in [0.5, 1); the binary16 exponent of a is e - 1 */
    int e;
    double m = frexp(a, &e);
    if (a == 0.0) return sign;
    int exp16 = e - 1;                      /* a in [2^exp16, 2^(exp16+1)) */
    double q;                               /* a in units of the target's last place */
    if (exp16 < -14) q = ldexp(a, 24);      /* subnormal: units of 2^-24 */
    else q = ldexp(m, 11);                  /* normal: 11 significant bits, in [1024, 2048) */
    double r = floor(q);
    double frac = q - r;
    if (frac > 0.5 || (frac == 0.5 && fmod(r, 2.0) != 0.0)) r += 1.0;
    if (exp16 < -14) {
        /* r counts 2^-24 units; 1024 of them is the smallest normal, which the bit pattern
         * below also encodes correctly (exponent field 1, fraction 0) */
        return (uint16_t)(sign | (uint16_t)r);
    }
    if (r == 2048.0) {                      /* rounding carried into the next binade */
        r = 1024.0;
        exp16 += 1;
    }
    if (exp16 > 15) return (uint16_t)(sign | 0x7C00u);
    return (uint16_t)(sign | (uint16_t)((exp16 + 15) << 10) | (uint16_t)((int)r - 1024));
}

/* Element-wise orc_double_to_half over n values. */
int orc_round_to_half(const double* v, int64_t n, uint16_t* out) {
    if ((!v || !out) && n > 0) return ORC_ERR_ARG;
    for (int64_t i = 0; i < n; i++) out[i] = orc_double_to_half(v[i]);
    return ORC_OK;
}

/* Gated FFN activation ("Reduced Matrix Multiplication" §4.2: H = act(X W_up), then keep
 * the high-response channels of H; §3.2: SiLU's saturation makes many of them near zero),
 * in Llama's gated form: h[b][r] = fp16(SiLU(g[b][r]) * u[b][r]) with SiLU(v) = v / (1 +
 * e^-v), from fp16 gate and up outputs g and u, computed in fp64 and rounded once.
 * g, u and h are B x N at leading dimension ld. */
int orc_silu_mul(const uint16_t* g, const uint16_t* u, int B, int N, int ld, uint16_t* h) {
    if (!g || !u || !h || B < 0 || N < 0 || ld < N) return ORC_ERR_ARG;
    for (int b = 0; b < B; b++)
        for (int r = 0; r < N; r++) {
            double gv = orc_half_to_double(g[(size_t)b * ld + r]);
            double uv = orc_half_to_double(u[(size_t)b * ld + r]);
            double silu = gv / (1.0 + exp(-gv));
            h[(size_t)b * ld + r] = orc_double_to_half(silu * uv);
        }
    return ORC_OK;
}

/* Prefill with a per-token index set ([RMM] §4.2: the reduced product over the columns a
 * token keeps; §6.1: every token of a batch has its own index set):
 *   Y[m,n] = sum over k of x~[m,k] * W[n,k] * mask[n,k],
 *   x~[m,k] = X[m,k] if the threshold rule keeps it (X[m,k] != 0 and not |X[m,k]| < t),
 *             else 0,
 * i.e. row m is the decode result of token m alone (orc_spmv with B = 1).  When rows is
 * not NULL only the listed rows are computed, in the listed order. */
int orc_spmm_tokens(const uint16_t* W, int ldw, const uint8_t* mask, int ld_mask, int N, int K,
                    const uint16_t* X, int M, int ldx, float t, const int* rows, int n_rows,
                    double* Y) {
    if (!W || !mask || !X || !Y || check_dims(N, K, ldw, ld_mask) || M < 0 || ldx < K ||
        !valid_threshold(t))
        return ORC_ERR_ARG;
    int count = rows ? n_rows : M;
    for (int i = 0; i < count; i++) {
        int m = rows ? rows[i] : i;
        if (m < 0 || m >= M) return ORC_ERR_ARG;
        for (int n = 0; n < N; n++) {
            double acc = 0.0;
            for (int k = 0; k < K; k++) {
                if (mask[(size_t)n * ld_mask + k] == 0) continue;
                double xv = orc_half_to_double(X[(size_t)m * ldx + k]);
                if (!passes_threshold(xv, (double)t)) continue; /* k is not in token m's set */
                acc += xv * orc_half_to_double(W[(size_t)n * ldw + k]);
            }
            Y[(size_t)i * N + n] = acc;
        }
    }
    return ORC_OK;
}

/* Token grouping ([RMM] §6.1: tokens whose index sets are the same or alike go into one
 * group, and each group runs its own dense product over the columns it uses).  The
 * pages leave the similarity measure open; this is the plainest reading at the
 * granularity of the stored tiles (64 columns):
 *   - signature of token m: bit kt (bit kt % 64 of word kt / 64, words = ceil(K / 4096))
 *     is set iff the threshold rule keeps some X[m,k] with 64 kt <= k < 64 kt + 64;
 *   - order: tokens sorted by signature, the words compared one after another from word
 *     0 as unsigned 64-bit integers, equal signatures by lower token index; perm[r] is the
 *     token at position r (identical signatures end up next to each other);
 *   - token tiles: positions [j T, min((j + 1) T, M)) form tile j; its signature
 *     tile_sig[j * words + w] is the OR of its tokens' signatures -- the k-tiles that
 *     tile's product has to visit.
 * K <= 16384 (at most 4 words). */
typedef struct {
    uint64_t sig[4];
    int words;
    int token;
} token_key;

static int cmp_token_key(const void* a, const void* b) {
    const token_key* x = (const token_key*)a;
    const token_key* y = (const token_key*)b;
    for (int w = 0; w < x->words; w++)
        if (x->sig[w] != y->sig[w]) return x->sig[w] < y->sig[w] ? -1 : 1;
    return (x->token > y->token) - (x->token < y->token);
}

int orc_token_groups(const uint16_t* X, int M, int K, int ldx, float t, int T, uint32_t* perm,
                     uint64_t* tile_sig) {
    if (!X || !perm || !tile_sig || M < 1 || K < 1 || K > 16384 || ldx < K || T < 1 ||
        !valid_threshold(t))
        return ORC_ERR_ARG;
    int n_ktiles = (K + 63) / 64;
    int words = (n_ktiles + 63) / 64;
    token_key* keys = (token_key*)calloc((size_t)M, sizeof(token_key));
    if (!keys) return ORC_ERR_ARG;
    for (int m = 0; m < M; m++) {
        keys[m].words = words;
        keys[m].token = m;
        for (int k = 0; k < K; k++)
            if (passes_threshold(orc_half_to_double(X[(size_t)m * ldx + k]), (double)t)) {
                int kt = k / 64;
                keys[m].sig[kt / 64] |= (uint64_t)1 << (kt % 64);
            }
    }
    qsort(keys, (size_t)M, sizeof(token_key), cmp_token_key);
    int tiles = (M + T - 1) / T;
    for (int j = 0; j < tiles * words; j++) tile_sig[j] = 0;
    for (int r = 0; r < M; r++) {
        perm[r] = (uint32_t)keys[r].token;
        for (int w = 0; w < words; w++) tile_sig[(size_t)(r / T) * words + w] |= keys[r].sig[w];
    }
    free(keys);
    return ORC_OK;
}

/* 2:4 + residual split ("Accelerating LLM GPU inference with moderately unstructured
 * sparse weight matrices": abstract and §1, layers (i) and (iii) of its three-layer
 * format -- a structured part for the sparse tensor cores and a residual that keeps the
 * product exact; the related-work paragraph on SparTA describes the same two-way split).
 * The pages do not say which kept weights of a group go to the structured part; this
 * reading takes the first two in column order:
 *   for every row n and every group of four columns 4g .. 4g+3 (the last group of a
 *   ragged K is shorter), the kept weights (mask != 0) at the two lowest columns go to
 *   the 2:4 part (mask_s), every further kept weight of the group to the residual
 *   (mask_r).  mask_s and mask_r are disjoint and their union is mask. */
int orc_split24(const uint8_t* mask, int ld_mask, int N, int K, uint8_t* mask_s,
                uint8_t* mask_r) {
    if (!mask || !mask_s || !mask_r || N < 0 || K < 0 || ld_mask < K) return ORC_ERR_ARG;
    for (int n = 0; n < N; n++)
        for (int g = 0; g < K; g += 4) {
            int taken = 0;
            for (int k = g; k < g + 4 && k < K; k++) {
                size_t i = (size_t)n * K + k;
                mask_s[i] = 0;
                mask_r[i] = 0;
                if (mask[(size_t)n * ld_mask + k] == 0) continue; /* not kept */
                if (taken < 2) {
                    mask_s[i] = 1;
                    taken++;
                } else {
                    mask_r[i] = 1;
                }
            }
        }
    return ORC_OK;
}
