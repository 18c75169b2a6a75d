/*
 * sherry_oracle.c -- plain CPU oracle for the Sherry 1.25-bit ternary format.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or
 * load this file: only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg use it.  It shares no code, header, table or constant with
 * the CUDA library; it restates the format from its written definition.
 *
 * What it computes (source: "Sherry: Hardware-Efficient 1.25-Bit Ternary
 * Quantization via Fine-grained Sparsification", arXiv 2601.07892, abstract
 * and Figure 2 caption): weights are ternary {-1, 0, +1}; every block of four
 * consecutive weights along K holds exactly one zero (3:4 sparsity) and is
 * coded in five bits (4 zero positions x 2^3 sign patterns = 32 states).
 * The product computed is y = s (.) (W_ternary . x_int8) with one fp32 scale
 * per output row.
 *
 * Readings where the pages are silent (each is restated in the design notes):
 *  - prune: in each block the weight of smallest |w| becomes the zero; ties go
 *    to the lowest index (strict '<' while scanning i = 0..3);
 *  - sign: a kept weight is -1 when w < 0, else +1 (so a kept -0.0 is +1);
 *  - scale: the mean |w| over the kept weights of the row, summed in double
 *    in ascending k, divided by the kept count 3K/4, rounded once to fp32;
 *  - layout: a row is cut into tiles of 128 weights (32 blocks); a tile is
 *    five 32-bit words Z0, Z1, S0, S1, S2 (plane 0 = Z0, 1 = Z1, 2 = S0,
 *    3 = S1, 4 = S2).  Rows are taken in groups of 32; within a group the
 *    tiles follow each other and, within a tile, each plane holds the 32 rows
 *    of the group:
 *        word(plane, n, t) = codes[((n / 32) * T + t) * 160 + plane * 32 + n % 32],
 *    T = K / 128.  Rows past N in the last group are padding and hold zeros;
 *    block j (j = 0..31, weights k = 128 t + 4 j + i, i = 0..3) keeps its
 *    2-bit zero position p in bits [2*(j/2), 2*(j/2)+1] of Z_(j mod 2);
 *    the r-th kept weight of block j (r = 0, 1, 2 in ascending i) has its
 *    sign in bit j of S_r, 1 meaning -1.
 *  - logical 5-bit code of one block: c = p | s0 << 2 | s1 << 3 | s2 << 4.
 *
 * Arithmetic: unpack to int8 {-1, 0, +1}; dot products in int64; the output
 * is y = (double) s_n * (double) acc, which is exact in double here.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <math.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORC_OK = 0, ORC_BAD_ARG = 1, ORC_NO_MEM = 2 };

#define ORC_TILE 128   /* weights per tile            */
#define ORC_NBLK 32    /* 4-weight blocks per tile    */
#define ORC_NPLANE 5   /* 32-bit words per tile       */

#define ORC_GROUP 32    /* rows per group in the layout */

static int64_t orc_word(int64_t plane, int64_t n, int64_t t, int64_t T)
{
    return ((n / ORC_GROUP) * T + t) * (ORC_NPLANE * ORC_GROUP) + plane * ORC_GROUP + n % ORC_GROUP;
}

static int64_t orc_padded_rows(int64_t N)
{
    return (N + ORC_GROUP - 1) / ORC_GROUP * ORC_GROUP;
}

/* Number of bytes of packed codes for an N x K matrix (scales excluded),
 * rows padded to a whole group. */
int64_t oracle_packed_bytes(int64_t N, int64_t K)
{
    if (N < 0 || K < 0 || K % ORC_TILE) return -1;
    return orc_padded_rows(N) * (K / ORC_TILE) * ORC_NPLANE * 4;
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* 3:4 prune of one block: zero position (argmin |w|, lowest index on ties)
 * and the three kept signs in ascending position (1 = negative). */
void oracle_prune_block(const float *w, int32_t *zero_pos, int32_t *neg)
{
    int p = 0;
    for (int i = 1; i < 4; i++)
        if (fabsf(w[i]) < fabsf(w[p])) p = i;
    int r = 0;
    for (int i = 0; i < 4; i++) {
        if (i == p) continue;
        neg[r++] = (w[i] < 0.0f) ? 1 : 0;
    }
    *zero_pos = p;
}

/* Logical 5-bit code of a block from its zero position and kept signs. */
int32_t oracle_block_code(int32_t zero_pos, const int32_t *neg)
{
    return (zero_pos & 3) | (neg[0] & 1) << 2 | (neg[1] & 1) << 3 | (neg[2] & 1) << 4;
}

/* Ternary values of the four weights of a block given its 5-bit code. */
void oracle_code_weights(int32_t code, int8_t *w)
{
    int p = code & 3, r = 0;
    for (int i = 0; i < 4; i++) {
        if (i == p) { w[i] = 0; continue; }
        w[i] = ((code >> (2 + r)) & 1) ? -1 : 1;
        r++;
    }
}

/* Pack fp32 latent weights W[N][K] (row-major) into codes + per-row scales. */
int oracle_pack(const float *w, int64_t N, int64_t K, uint32_t *codes, float *scales)
{
    if (!w || !codes || !scales || N < 1 || K < ORC_TILE || K % ORC_TILE) return ORC_BAD_ARG;
    const int64_t T = K / ORC_TILE;
    #pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; n++) {
        double sum_abs = 0.0;
        for (int64_t t = 0; t < T; t++) {
            uint32_t z[2] = {0, 0}, s[3] = {0, 0, 0};
            for (int j = 0; j < ORC_NBLK; j++) {
                const float *blk = w + n * K + t * ORC_TILE + 4 * j;
                int32_t p, neg[3];
                oracle_prune_block(blk, &p, neg);
                z[j & 1] |= (uint32_t)p << (2 * (j >> 1));
                for (int r = 0; r < 3; r++) s[r] |= (uint32_t)neg[r] << j;
                for (int i = 0; i < 4; i++)
                    if (i != p) sum_abs += fabs((double)blk[i]);
            }
            codes[orc_word(0, n, t, T)] = z[0];
            codes[orc_word(1, n, t, T)] = z[1];
            codes[orc_word(2, n, t, T)] = s[0];
            codes[orc_word(3, n, t, T)] = s[1];
            codes[orc_word(4, n, t, T)] = s[2];
        }
        scales[n] = (float)(sum_abs / (0.75 * (double)K));
    }
    for (int64_t n = N; n < orc_padded_rows(N); n++)
        for (int64_t t = 0; t < T; t++)
            for (int p = 0; p < ORC_NPLANE; p++) codes[orc_word(p, n, t, T)] = 0u;
    return ORC_OK;
}

/* Ternary row n (K int8 values) from the packed codes. */
static void orc_unpack_row(const uint32_t *codes, int64_t n, int64_t K, int8_t *row)
{
    const int64_t T = K / ORC_TILE;
    for (int64_t t = 0; t < T; t++) {
        uint32_t z[2] = {codes[orc_word(0, n, t, T)], codes[orc_word(1, n, t, T)]};
        uint32_t s[3] = {codes[orc_word(2, n, t, T)], codes[orc_word(3, n, t, T)],
                         codes[orc_word(4, n, t, T)]};
        for (int j = 0; j < ORC_NBLK; j++) {
            int p = (int)((z[j & 1] >> (2 * (j >> 1))) & 3u);
            int r = 0;
            for (int i = 0; i < 4; i++) {
                int8_t v = 0;
                if (i != p) {
                    v = ((s[r] >> j) & 1u) ? -1 : 1;
                    r++;
                }
                row[t * ORC_TILE + 4 * j + i] = v;
            }
        }
    }
}

/* Unpack the whole matrix to int8 Wt[N][K] in {-1, 0, +1}. */
int oracle_unpack(const uint32_t *codes, int64_t N, int64_t K, int8_t *wt)
{
    if (!codes || !wt || N < 1 || K < ORC_TILE || K % ORC_TILE) return ORC_BAD_ARG;
    #pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; n++) orc_unpack_row(codes, n, K, wt + n * K);
    return ORC_OK;
}

/* acc[m][n] = sum_k Wt[n][k] * x[m][k] in int64, for M activation rows x[M][K].
 * The decode GEMV (M = batch) and the prefill GEMM (M = tokens) are the same
 * definition; both entry points below call this loop. */
static int orc_matmul_acc(const uint32_t *codes, const int8_t *x, int64_t M, int64_t N,
                          int64_t K, int64_t *acc)
{
    if (!codes || !x || !acc || M < 1 || N < 1 || K < ORC_TILE || K % ORC_TILE) return ORC_BAD_ARG;
    int err = 0;
    #pragma omp parallel
    {
        int8_t *row = (int8_t *)malloc((size_t)K);
        if (!row) {
            #pragma omp atomic write
            err = 1;
        }
        #pragma omp for schedule(static)
        for (int64_t n = 0; n < N; n++) {
            if (!row) continue;
            orc_unpack_row(codes, n, K, row);
            for (int64_t m = 0; m < M; m++) {
                const int8_t *xm = x + m * K;
                int64_t a = 0;
                for (int64_t k = 0; k < K; k++) a += (int64_t)row[k] * (int64_t)xm[k];
                acc[m * N + n] = a;
            }
        }
        free(row);
    }
    return err ? ORC_NO_MEM : ORC_OK;
}

static int orc_matmul(const uint32_t *codes, const float *scales, const int8_t *x, int64_t M,
                      int64_t N, int64_t K, double *y)
{
    if (!scales || !y) return ORC_BAD_ARG;
    int64_t *acc = (int64_t *)malloc((size_t)(M * N) * sizeof(int64_t));
    if (!acc) return ORC_NO_MEM;
    int rc = orc_matmul_acc(codes, x, M, N, K, acc);
    if (rc == ORC_OK)
        for (int64_t m = 0; m < M; m++)
            for (int64_t n = 0; n < N; n++)
                y[m * N + n] = (double)scales[n] * (double)acc[m * N + n];
    free(acc);
    return rc;
}

/* Decode GEMV: x[B][K] int8, acc/y[B][N]. */
int oracle_gemv_acc(const uint32_t *codes, const int8_t *x, int64_t N, int64_t K, int64_t B,
                    int64_t *acc)
{
    return orc_matmul_acc(codes, x, B, N, K, acc);
}

int oracle_gemv(const uint32_t *codes, const float *scales, const int8_t *x, int64_t N,
                int64_t K, int64_t B, double *y)
{
    return orc_matmul(codes, scales, x, B, N, K, y);
}

/* Prefill GEMM: x[M][K] int8 (tokens), acc/y[M][N]. */
int oracle_gemm_acc(const uint32_t *codes, const int8_t *x, int64_t M, int64_t N, int64_t K,
                    int64_t *acc)
{
    return orc_matmul_acc(codes, x, M, N, K, acc);
}

int oracle_gemm(const uint32_t *codes, const float *scales, const int8_t *x, int64_t M,
                int64_t N, int64_t K, double *y)
{
    return orc_matmul(codes, scales, x, M, N, K, y);
}

/*
 * Activation front-end.  The setting the method is served in is W1.25A8
 * (int8 activations); the pages do not say how the int8 activations are made.
 * Reading taken (restated in the design notes): per token b,
 *     amax_b = max_k |x[b][k]|,   s_b = amax_b / 127,
 *     q[b][k] = clamp(rint(x[b][k] * (127 / amax_b)), -127, 127),
 * every operation in IEEE single precision, rounding to nearest even (the
 * default mode); an all-zero row gives s_b = 0 and q = 0.  x holds bf16 bit
 * patterns: the upper 16 bits of an fp32 value.
 */
static float orc_bf16(uint16_t h)
{
    const uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* The rule above on one token row of fp32 values. */
static void orc_quantize_row(const float *xr, int64_t K, int8_t *q, float *s)
{
    float amax = 0.0f;
    for (int64_t k = 0; k < K; k++) {
        const float a = fabsf(xr[k]);
        if (a > amax) amax = a;
    }
    if (amax == 0.0f) {
        *s = 0.0f;
        memset(q, 0, (size_t)K);
        return;
    }
    const float inv = 127.0f / amax;
    *s = amax / 127.0f;
    for (int64_t k = 0; k < K; k++) {
        const float v = xr[k] * inv;
        float r = nearbyintf(v);
        if (r > 127.0f) r = 127.0f;
        if (r < -127.0f) r = -127.0f;
        q[k] = (int8_t)r;
    }
}

int oracle_quantize_act(const uint16_t *x, int64_t B, int64_t K, int8_t *q, float *s)
{
    if (!x || !q || !s || B < 1 || K < 1) return ORC_BAD_ARG;
    float *row = (float *)malloc(sizeof(float) * (size_t)K);
    if (!row) return ORC_NO_MEM;
    for (int64_t b = 0; b < B; b++) {
        for (int64_t k = 0; k < K; k++) row[k] = orc_bf16(x[b * K + k]);
        orc_quantize_row(row, K, q + b * K, s + b);
    }
    free(row);
    return ORC_OK;
}

/*
 * Re-quantization of fp32 activations (for example the y of a previous GEMV,
 * feeding the next layer): the same per-token rule, read from fp32 values.
 */
int oracle_quantize_f32(const float *x, int64_t B, int64_t K, int8_t *q, float *s)
{
    if (!x || !q || !s || B < 1 || K < 1) return ORC_BAD_ARG;
    for (int64_t b = 0; b < B; b++) orc_quantize_row(x + b * K, K, q + b * K, s + b);
    return ORC_OK;
}

/*
 * SwiGLU, the gated activation of the LLaMA MLP (the models the method is
 * evaluated on are LLaMA-3.2 1B and 3B): the down projection's input is
 *     h = silu(g) * u,   silu(g) = g / (1 + e^(-g)),
 * with g and u the gate and up projections' outputs.  Evaluated in double
 * and rounded once to fp32.
 */
int oracle_swiglu(const float *g, const float *u, int64_t n, float *h)
{
    if (!g || !u || !h || n < 1) return ORC_BAD_ARG;
    for (int64_t i = 0; i < n; i++) {
        const double gd = (double)g[i];
        h[i] = (float)(gd / (1.0 + exp(-gd)) * (double)u[i]);
    }
    return ORC_OK;
}

/* GEMV on quantized activations: y[b][n] = s[n] * sx[b] * acc[b][n], in double. */
int oracle_gemv_act(const uint32_t *codes, const float *scales, const int8_t *q, const float *sx,
                    int64_t N, int64_t K, int64_t B, double *y)
{
    if (!sx) return ORC_BAD_ARG;
    int64_t *acc = (int64_t *)malloc(sizeof(int64_t) * (size_t)(B * N > 0 ? B * N : 1));
    if (!acc) return ORC_NO_MEM;
    int rc = orc_matmul_acc(codes, q, B, N, K, acc);
    if (rc == ORC_OK)
        for (int64_t b = 0; b < B; b++)
            for (int64_t n = 0; n < N; n++)
                y[b * N + n] = (double)scales[n] * (double)sx[b] * (double)acc[b * N + n];
    free(acc);
    return rc;
}

/*
 * Comparison formats.  The pages set Sherry's 1.25 bits per weight against
 * the two ternary packings they call the state of the art (arXiv 2601.07892,
 * abstract; Figure 2 caption): a 2-bit aligned packing, which wastes a quarter
 * of its code space, and a 1.67-bit packing of three weights in five bits,
 * whose 3-way grouping does not match power-of-two lanes.  Neither layout is
 * printed; the readings below are this build's own (restated in the design
 * notes).  Both hold any ternary matrix; for comparison they are filled from
 * the same ternary values as a Sherry matrix (via oracle_unpack).
 *
 * Format 1, "I2" (2 bits per weight, aligned):
 *   - code of one weight: 0 -> 0, 1 -> +1, 3 -> -1 (bit 0 = nonzero, bit 1 =
 *     negative); the unused code 2 decodes to 0;
 *   - a tile is 128 weights of a row in eight 32-bit words; word q holds
 *     weights k = 128 t + 16 q + m (m = 0..15): weight m sits at bits
 *     [4 (m mod 8) + 2 (m / 8), +1], so nibble n of the word holds weights n
 *     (low two bits) and n + 8 (high two bits);
 *   - rows in groups of 32 as for Sherry: word(q, n, t) =
 *     codes[((n / 32) * T + t) * 256 + 32 q + n % 32], T = K / 128, K a
 *     multiple of 128; rows past N are zero.
 * Format 2, "T3" (three weights in five bits, 1.67 bits per weight):
 *   - code of a triple (w0, w1, w2): c = (w0 + 1) + 3 (w1 + 1) + 9 (w2 + 1),
 *     0..26; codes 27..31 are never written and decode to three zeros;
 *   - a tile is 32 triples = 96 weights of a row in five 32-bit words: triple
 *     j covers k = 96 t + 3 j + {0, 1, 2} and its code is bits [5 j, 5 j + 4]
 *     of the 160-bit little-endian string of words 0..4 (string bit b is bit
 *     b mod 32 of word b / 32), so triples 6, 12, 19 and 25 straddle words;
 *   - a row of K weights (K a multiple of 128) is padded with zero weights to
 *     an even number of tiles, T3 = 2 * ceil(K / 192) (the GPU streams tiles
 *     in pairs); rows in groups of 32: word(p, n, t) =
 *     codes[((n / 32) * T3 + t) * 160 + 32 p + n % 32]; rows past N hold
 *     zero words (as in both other layouts).
 */
enum { ORC_FMT_I2 = 1, ORC_FMT_T3 = 2 };

/* Tiles per row of a comparison format (0 for a bad format or K). */
int64_t oracle_cmp_tiles(int32_t fmt, int64_t K)
{
    if (K < ORC_TILE || K % ORC_TILE) return 0;
    if (fmt == ORC_FMT_I2) return K / ORC_TILE;
    if (fmt == ORC_FMT_T3) return 2 * ((K + 191) / 192);
    return 0;
}

/* Words per tile per row of a comparison format. */
static int64_t orc_cmp_tile_words(int32_t fmt) { return fmt == ORC_FMT_I2 ? 8 : 5; }

/* Bytes of codes of an N x K matrix in a comparison format (-1 if invalid). */
int64_t oracle_cmp_packed_bytes(int32_t fmt, int64_t N, int64_t K)
{
    const int64_t T = oracle_cmp_tiles(fmt, K);
    if (T == 0 || N < 1) return -1;
    return orc_padded_rows(N) * T * orc_cmp_tile_words(fmt) * 4;
}

static int64_t orc_cmp_word(int32_t fmt, int64_t q, int64_t n, int64_t t, int64_t T)
{
    const int64_t tw = orc_cmp_tile_words(fmt);
    return ((n / ORC_GROUP) * T + t) * (tw * ORC_GROUP) + q * ORC_GROUP + n % ORC_GROUP;
}

/* 2-bit code of one ternary value, and back. */
static uint32_t orc_i2_code(int8_t w) { return w == 0 ? 0u : (w > 0 ? 1u : 3u); }
static int8_t orc_i2_weight(uint32_t c) { return (c & 1u) ? ((c & 2u) ? -1 : 1) : 0; }

/* Base-3 code of a triple, and back (codes past 26 give zeros). */
int32_t oracle_t3_code(const int8_t *w)
{
    return (w[0] + 1) + 3 * (w[1] + 1) + 9 * (w[2] + 1);
}

void oracle_t3_weights(int32_t code, int8_t *w)
{
    if (code < 0 || code > 26) {
        w[0] = w[1] = w[2] = 0;
        return;
    }
    w[0] = (int8_t)(code % 3 - 1);
    w[1] = (int8_t)((code / 3) % 3 - 1);
    w[2] = (int8_t)(code / 9 - 1);
}

/* Ternary weight k of row `row` (K values), zero past K. */
static int8_t orc_row_at(const int8_t *row, int64_t K, int64_t k) { return k < K ? row[k] : 0; }

/* Encode a ternary matrix Wt[N][K] (values in {-1, 0, +1}) in format fmt. */
int oracle_cmp_encode(int32_t fmt, const int8_t *wt, int64_t N, int64_t K, uint32_t *codes)
{
    const int64_t T = oracle_cmp_tiles(fmt, K);
    if (!wt || !codes || N < 1 || T == 0) return ORC_BAD_ARG;
    const int64_t tw = orc_cmp_tile_words(fmt);
    memset(codes, 0, (size_t)oracle_cmp_packed_bytes(fmt, N, K));
    for (int64_t n = 0; n < N; n++) {
        const int8_t *row = wt + n * K;
        for (int64_t t = 0; t < T; t++) {
            uint32_t w[8] = {0, 0, 0, 0, 0, 0, 0, 0};
            if (fmt == ORC_FMT_I2) {
                for (int q = 0; q < 8; q++)
                    for (int m = 0; m < 16; m++) {
                        const uint32_t c = orc_i2_code(row[t * ORC_TILE + 16 * q + m]);
                        w[q] |= c << (4 * (m % 8) + 2 * (m / 8));
                    }
            } else {
                for (int j = 0; j < 32; j++) {
                    int8_t tri[3];
                    for (int i = 0; i < 3; i++) tri[i] = orc_row_at(row, K, 96 * t + 3 * j + i);
                    const uint32_t c = (uint32_t)oracle_t3_code(tri);
                    for (int b = 0; b < 5; b++) {
                        const int bit = 5 * j + b;
                        w[bit / 32] |= ((c >> b) & 1u) << (bit % 32);
                    }
                }
            }
            for (int q = 0; q < tw; q++) codes[orc_cmp_word(fmt, q, n, t, T)] = w[q];
        }
    }
    return ORC_OK;
}

/* Ternary row n (K values) of a comparison-format matrix. */
static void orc_cmp_unpack_row(int32_t fmt, const uint32_t *codes, int64_t n, int64_t K, int8_t *row)
{
    const int64_t T = oracle_cmp_tiles(fmt, K);
    const int64_t tw = orc_cmp_tile_words(fmt);
    for (int64_t t = 0; t < T; t++) {
        uint32_t w[8];
        for (int q = 0; q < tw; q++) w[q] = codes[orc_cmp_word(fmt, q, n, t, T)];
        if (fmt == ORC_FMT_I2) {
            for (int q = 0; q < 8; q++)
                for (int m = 0; m < 16; m++)
                    row[t * ORC_TILE + 16 * q + m] =
                        orc_i2_weight(w[q] >> (4 * (m % 8) + 2 * (m / 8)));
        } else {
            for (int j = 0; j < 32; j++) {
                uint32_t c = 0;
                for (int b = 0; b < 5; b++) {
                    const int bit = 5 * j + b;
                    c |= ((w[bit / 32] >> (bit % 32)) & 1u) << b;
                }
                int8_t tri[3];
                oracle_t3_weights((int32_t)c, tri);
                for (int i = 0; i < 3; i++) {
                    const int64_t k = 96 * t + 3 * j + i;
                    if (k < K) row[k] = tri[i];
                }
            }
        }
    }
}

int oracle_cmp_unpack(int32_t fmt, const uint32_t *codes, int64_t N, int64_t K, int8_t *wt)
{
    if (!codes || !wt || N < 1 || oracle_cmp_tiles(fmt, K) == 0) return ORC_BAD_ARG;
    #pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; n++) orc_cmp_unpack_row(fmt, codes, n, K, wt + n * K);
    return ORC_OK;
}

/* acc[b][n] = sum_k Wt[n][k] * x[b][k] in int64 for a comparison-format matrix. */
int oracle_cmp_gemv_acc(int32_t fmt, const uint32_t *codes, const int8_t *x, int64_t N, int64_t K,
                        int64_t B, int64_t *acc)
{
    if (!codes || !x || !acc || N < 1 || B < 1 || oracle_cmp_tiles(fmt, K) == 0) return ORC_BAD_ARG;
    int err = 0;
    #pragma omp parallel
    {
        int8_t *row = (int8_t *)malloc((size_t)K);
        if (!row) {
            #pragma omp atomic write
            err = 1;
        }
        #pragma omp for schedule(static)
        for (int64_t n = 0; n < N; n++) {
            if (!row) continue;
            orc_cmp_unpack_row(fmt, codes, n, K, row);
            for (int64_t b = 0; b < B; b++) {
                int64_t a = 0;
                for (int64_t k = 0; k < K; k++) a += (int64_t)row[k] * (int64_t)x[b * K + k];
                acc[b * N + n] = a;
            }
        }
        free(row);
    }
    return err ? ORC_NO_MEM : ORC_OK;
}
