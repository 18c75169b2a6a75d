/*
 * sherry.h -- C ABI of libsherry.so: the Sherry 1.25-bit ternary weight format
 * on NVIDIA B200 (sm_100a).
 *
 * The method ("Sherry: Hardware-Efficient 1.25-Bit Ternary Quantization via
 * Fine-grained Sparsification", arXiv 2601.07892, abstract; Figure 2 caption)
 * keeps weights in {-1, 0, +1} with 3:4 sparsity -- every block of
 * four consecutive weights along K holds exactly one zero -- and codes each
 * block in five bits (4 zero positions x 2^3 signs = 32 states), a regular
 * 1.25 bits per weight.  The product it serves is
 *
 *     y[b][n] = s[n] * sum_k W[n][k] * x[b][k],    W ternary, x int8, s fp32.
 *
 * ---------------------------------------------------------------------------
 * Packed layout (the pages fix only the code size, five bits per four weights; this layout is
 * the library's reading, chosen so that 32 blocks decode with 32-bit SWAR
 * logic and a GEMV work chunk is one contiguous block of memory):
 *   - a row of K weights (K a multiple of 128) is cut into T = K / 128 tiles of
 *     128 weights = 32 blocks; weight k = 128 t + 4 j + i is position i of
 *     block j of tile t;
 *   - a tile is five uint32 words Z0, Z1, S0, S1, S2 (planes 0..4; 20 bytes per
 *     128 weights, exactly 1.25 bits per weight);
 *   - rows are taken in groups of 32; within a group the tiles follow each
 *     other and within a tile each plane holds the 32 rows of the group:
 *         codes[((n / 32) * T + t) * 160 + plane * 32 + n % 32],
 *     i.e. a [ceil(N/32)][T][5][32] array of uint32; rows past N in the last
 *     group are padding and hold zeros;
 *   - block j's zero position p (0..3) is the 2-bit field at bits
 *     [2*(j/2), 2*(j/2)+1] of Z_(j mod 2) (Z0 holds the even blocks, Z1 the
 *     odd ones);
 *   - the r-th kept weight of block j (r = 0, 1, 2, in ascending position)
 *     has its sign at bit j of S_r, 1 meaning -1.
 *   - scales[n] is one fp32 per output row.
 * Pack rule (not on the pages; the library's reading): in each block the
 * weight of smallest |w| is zeroed (ties go to the lowest index), a kept
 * weight becomes -1 if w < 0 and +1 otherwise, and scales[n] is the mean |w|
 * of the row's kept weights (3K/4 of them), accumulated in double and rounded
 * once to fp32.
 *
 * ---------------------------------------------------------------------------
 * Conventions shared by every call
 *   - Every pointer argument is a DEVICE pointer unless stated otherwise; the
 *     caller allocates and owns every buffer.  The library keeps no device
 *     allocation between calls.
 *   - Calls are asynchronous on `stream` (NULL = legacy default stream).  The
 *     checks listed under each call run on the host before any launch and
 *     return an error without touching the GPU.  A launch failure returns
 *     SHERRY_ERR_CUDA; the CUDA error text is then available from
 *     sherry_last_error().  Errors inside a running kernel surface as CUDA
 *     errors at the caller's next synchronisation.
 *   - No C++ exception crosses this interface.  Calls are thread-safe; two
 *     calls that share an output or a workspace must not overlap on the GPU.
 *   - Calls run on the current device.  What a call sets up there once (the
 *     kernels' shared-memory attributes, the static scratch's device address)
 *     is kept per device together with the CUDA context it was made in, and
 *     made again when another context is current, e.g. after cudaDeviceReset.
 *   - Integer results are exact: the dot products are accumulated in int32,
 *     which cannot overflow for K <= SHERRY_MAX_K, and converted to fp32
 *     exactly (|acc| <= 3K/4 * 128 < 2^24), so y = fl32(s * acc) with one
 *     rounding.
 */
#ifndef SHERRY_H
#define SHERRY_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Opaque CUDA stream handle; identical to cudaStream_t / CUstream. */
struct CUstream_st;
typedef struct CUstream_st *sherry_stream_t;

typedef enum {
    SHERRY_OK = 0,
    SHERRY_ERR_NULL = 1,        /* a required pointer is NULL                          */
    SHERRY_ERR_SHAPE = 2,       /* N, M or B < 1, K < 128 or K % 128 != 0, K too large */
    SHERRY_ERR_ALIGN = 3,       /* a pointer is not aligned as the call requires        */
    SHERRY_ERR_UNSUPPORTED = 4, /* a size beyond what the kernels support (e.g. B > 16) */
    SHERRY_ERR_CUDA = 5,        /* a CUDA call or launch failed                         */
    SHERRY_ERR_TIMEOUT = 6,     /* a bounded device-side wait ran out (see below)       */
    SHERRY_ERR_WORKSPACE = 7    /* workspace missing or smaller than required           */
} sherry_status;

#define SHERRY_TILE_K 128         /* weights per tile                     */
#define SHERRY_WORDS_PER_TILE 5   /* uint32 words per tile                */
#define SHERRY_ROW_GROUP 32       /* rows per group of the code layout    */
#define SHERRY_MAX_K 131072       /* keeps |acc| < 2^24                   */
#define SHERRY_MAX_GEMV_BATCH 16  /* activation rows per GEMV call        */
#define SHERRY_MAX_GROUP 128      /* GEMVs per grouped call               */
#define SHERRY_STATIC_SCRATCH_BYTES (4u << 20)  /* scratch of sherry_gemv_static */

/* Bytes of packed codes for an N x K matrix: ceil(N/32)*32 * K * 5 / 32
 * (N * K * 5 / 32 when N is a multiple of 32; scales excluded).  The count
 * is the abstract's five bits per block of four weights, 1.25 bits per weight
 * (arXiv 2601.07892, abstract); the rounding of N up to whole 32-row groups
 * is this layout's own.
 * Returns 0 when K is not a positive multiple of 128 or N < 1. */
size_t sherry_packed_bytes(int64_t N, int64_t K);

/*
 * sherry_pack -- 3:4 prune, ternarise, encode and scale (arXiv 2601.07892,
 * abstract: blocks of four weights, five bits each).
 *   w       [N][K] fp32, row-major, finite values (NaN/Inf give an unspecified
 *           but deterministic code); 16-byte aligned.
 *   codes   output, sherry_packed_bytes(N, K) bytes, layout above (padding rows
 *           are written as zeros); 16-byte aligned.
 *   scales  output, N fp32.
 * Errors: NULL, SHAPE (N < 1, K not a positive multiple of 128, K > SHERRY_MAX_K),
 * ALIGN, CUDA.
 */
sherry_status sherry_pack(const float *w, int64_t N, int64_t K, uint32_t *codes,
                          float *scales, sherry_stream_t stream);

/* One matrix of a grouped pack call (pointers and rules as for sherry_pack). */
typedef struct {
    const float *w;    /* [N][K] fp32, 16-byte aligned */
    uint32_t *codes;   /* sherry_packed_bytes(N, K) bytes, 16-byte aligned */
    float *scales;     /* [N] */
    int64_t N;
    int64_t K;
} sherry_pack_desc;

/*
 * sherry_pack_grouped -- sherry_pack of `count` matrices (count <=
 * SHERRY_MAX_GROUP) in one launch, e.g. every projection of a model at load
 * time.  The results are those of one sherry_pack call per matrix, bit for bit.
 *   descs  HOST array of `count` descriptors (copied into the launch
 *          parameters; may be reused as soon as the call returns).
 * Errors: NULL (descs or a pointer), SHAPE (count < 1 or a matrix's N, K),
 * UNSUPPORTED (count > SHERRY_MAX_GROUP), ALIGN, CUDA.  Every descriptor is
 * checked before anything is launched.
 */
sherry_status sherry_pack_grouped(const sherry_pack_desc *descs, int count,
                                  sherry_stream_t stream);

/*
 * Workspace of the GEMV calls.  A call re-orders its activations once into
 * the order in which the decoded weights meet the multiply-accumulate, and
 * long rows are processed as several K-parts whose int32 partial sums meet in
 * the workspace.  sherry_gemv_workspace_bytes(N, K, B) is the size one GEMV
 * needs; a grouped call needs the sum over its GEMVs, laid out in descriptor
 * order.  Int8 calls with B <= 2, K a multiple of 512 and at most 8192, and
 * 16-byte aligned activations re-order inside the GEMV kernel and leave the
 * workspace untouched, as do bf16 calls of that kind with at most 64 chunks
 * of 32 rows x 512 weights per SM (which also quantize there); the size asked
 * is the same.  The workspace is a device buffer, 256-byte
 * aligned, owned by the caller; its contents are scratch: every call that
 * prepares activations (sherry_gemv, sherry_gemv_acc, sherry_gemv_grouped,
 * sherry_gemv_prepare) may rewrite it, and a run leaves its partial-sum area
 * cleared.  Calls that overlap on the GPU must not share a workspace.
 */
size_t sherry_gemv_workspace_bytes(int64_t N, int64_t K, int B);

/*
 * sherry_gemv -- decode GEMV, y = s (.) (W_ternary . x_int8) for B <= 16
 * activation rows (arXiv 2601.07892, abstract: ternary weights served by
 * hardware-aligned packing; the batch-1 case is the decode step).
 *   codes   [ceil(N/32)][K/128][5][32] uint32 from sherry_pack; 4-byte aligned
 *           (16-byte aligned and K a multiple of 512 select the pipelined kernel).
 *   scales  [N] fp32.
 *   x       [B][K] int8, row-major, any value in [-128, 127]; 4-byte aligned.
 *   y       [B][N] fp32 output, row-major.
 *   workspace / workspace_bytes: see sherry_gemv_workspace_bytes.
 * Errors: NULL, SHAPE, ALIGN, UNSUPPORTED (B > 16), WORKSPACE, CUDA.
 */
sherry_status sherry_gemv(const uint32_t *codes, const float *scales, const int8_t *x,
                          float *y, int64_t N, int64_t K, int B, void *workspace,
                          size_t workspace_bytes, sherry_stream_t stream);

/* As sherry_gemv, but writes the exact integer accumulators acc[B][N] (int32,
 * row-major) instead of scaled outputs; no scales are read.  For bit-exact
 * checks of the decode and the dot products. */
sherry_status sherry_gemv_acc(const uint32_t *codes, const int8_t *x, int32_t *acc,
                              int64_t N, int64_t K, int B, void *workspace,
                              size_t workspace_bytes, sherry_stream_t stream);

/*
 * Activation front-end.  The method is served as W1.25A8 (1.25-bit weights,
 * int8 activations: arXiv 2601.07892, abstract); the pages do not say how the
 * int8 activations are produced.  Reading taken here: per token (batch row) b
 *     amax_b = max_k |x[b][k]|,   s_b = amax_b / 127,
 *     q[b][k] = clamp(rint(x[b][k] * (127 / amax_b)), -127, 127),
 * every operation in fp32 with round-to-nearest-even; amax_b = 0 gives s_b = 0
 * and q = 0.  x is bf16 (uint16 bit patterns: the upper half of an fp32).
 *
 * sherry_quantize_act -- the front-end alone.
 *   x  [B][K] bf16, row-major, device, 16-byte aligned, K a multiple of 8.
 *   q  [B][K] int8 output, 4-byte aligned.   s  [B] fp32 output.
 * Errors: NULL, SHAPE, ALIGN, UNSUPPORTED, CUDA.
 */
sherry_status sherry_quantize_act(const uint16_t *x, int64_t B, int64_t K, int8_t *q, float *s,
                                  sherry_stream_t stream);

/*
 * sherry_gemv_bf16 -- the decode GEMV on bf16 activations: each token is
 * quantized as sherry_quantize_act does (in the re-order launch, keeping s_b in
 * the workspace; for small calls inside the GEMV kernel) and the GEMV scales
 * by both the weight and the activation scale:
 *   y[b][n] = fl32(fl32(s[n] * s_b) * acc[b][n]),  acc = W . q^T exactly.
 *   x  [B][K] bf16, 16-byte aligned; other arguments as sherry_gemv.
 *   workspace: sherry_gemv_bf16_workspace_bytes(N, K, B) bytes (a grouped call:
 *   the sum over its GEMVs, in descriptor order), 256-byte aligned.
 * Errors: as sherry_gemv.
 */
size_t sherry_gemv_bf16_workspace_bytes(int64_t N, int64_t K, int B);
sherry_status sherry_gemv_bf16(const uint32_t *codes, const float *scales, const uint16_t *x,
                               float *y, int64_t N, int64_t K, int B, void *workspace,
                               size_t workspace_bytes, sherry_stream_t stream);

/* One GEMV of a grouped bf16 call (device pointers). */
typedef struct {
    const uint32_t *codes;
    const float *scales;
    const uint16_t *x;  /* [B][K] bf16 */
    float *y;           /* [B][N] */
    int64_t N;
    int64_t K;
} sherry_gemv_bf16_desc;

/* sherry_gemv_bf16 over `count` GEMVs with the same B in one pass (one
 * re-order launch and one GEMV launch), as sherry_gemv_grouped. */
sherry_status sherry_gemv_bf16_grouped(const sherry_gemv_bf16_desc *descs, int count, int B,
                                       void *workspace, size_t workspace_bytes,
                                       sherry_stream_t stream);

/*
 * Front-end on fp32 activations, for chaining layers: the fp32 y of one GEMV
 * becomes the next GEMV's input without leaving the library.  Two forms:
 *   plain   the activations are x itself (e.g. the y of the previous layer);
 *   SwiGLU  the activations are h = silu(g) * u, silu(g) = g / (1 + e^-g),
 *           with g and u the outputs of the gate and up projections: the
 *           gated MLP of the LLaMA models the method is evaluated on
 *           (LLaMA-3.2 1B and 3B, arXiv 2601.07892, abstract).  h is formed in
 *           fp32, each operation rounded once, e^-g by CUDA's expf (within
 *           2 ulp); a g so negative that e^-g overflows gives h = -0 * u.
 * Each token row is then quantized by the rule of sherry_quantize_act, read
 * from the fp32 values.  The plain form is exact; in the SwiGLU form h differs
 * from the exactly rounded silu(g) * u by a few ulp, so a q whose scaled value
 * lies within ~1e-4 of a rounding tie may differ by one.
 * The rows are handled by one cluster of 8 CTAs each, which exchange their
 * maxima through distributed shared memory; NaN and Inf inputs are not
 * supported (the result is unspecified).
 *
 * sherry_quantize_f32 / sherry_quantize_swiglu -- the front-end alone.
 *   x, g, u  [B][K] fp32, row-major, device, 16-byte aligned; K a positive
 *            multiple of 128, at most SHERRY_MAX_K; B at most 65536.
 *   q  [B][K] int8 output, natural order, 4-byte aligned.   s  [B] fp32 output.
 * Errors: NULL, SHAPE, ALIGN, UNSUPPORTED, CUDA.
 */
sherry_status sherry_quantize_f32(const float *x, int64_t B, int64_t K, int8_t *q, float *s,
                                  sherry_stream_t stream);
sherry_status sherry_quantize_swiglu(const float *g, const float *u, int64_t B, int64_t K, int8_t *q,
                                     float *s, sherry_stream_t stream);

/*
 * sherry_gemv_f32 / sherry_gemv_swiglu -- the decode GEMV on fp32 activations
 * (plain, or the SwiGLU h of g and u), quantized per token in the re-order
 * launch as above, and scaled by both scales as sherry_gemv_bf16 is:
 *   y[b][n] = fl32(fl32(s[n] * s_b) * acc[b][n]),  acc = W . q^T exactly.
 *   x, g, u  [B][K] fp32, 16-byte aligned; other arguments as sherry_gemv.
 *   workspace: sherry_gemv_f32_workspace_bytes(N, K, B) bytes (equal to the
 *   bf16 size; a grouped call: the sum over its GEMVs, in descriptor order),
 *   256-byte aligned.
 * Errors: as sherry_gemv.
 */
size_t sherry_gemv_f32_workspace_bytes(int64_t N, int64_t K, int B);
sherry_status sherry_gemv_f32(const uint32_t *codes, const float *scales, const float *x, float *y,
                              int64_t N, int64_t K, int B, void *workspace, size_t workspace_bytes,
                              sherry_stream_t stream);
sherry_status sherry_gemv_swiglu(const uint32_t *codes, const float *scales, const float *g,
                                 const float *u, float *y, int64_t N, int64_t K, int B,
                                 void *workspace, size_t workspace_bytes, sherry_stream_t stream);

/* One GEMV of a grouped fp32 call (device pointers); u NULL: plain, else SwiGLU. */
typedef struct {
    const uint32_t *codes;
    const float *scales;
    const float *x;  /* [B][K] fp32 activations; SwiGLU: the gate outputs g */
    const float *u;  /* [B][K] up outputs (SwiGLU), or NULL */
    float *y;        /* [B][N] */
    int64_t N;
    int64_t K;
} sherry_gemv_f32_desc;

/* sherry_gemv_f32 / _swiglu over `count` GEMVs with the same B in one pass
 * (one front-end launch and one GEMV launch), as sherry_gemv_grouped. */
sherry_status sherry_gemv_f32_grouped(const sherry_gemv_f32_desc *descs, int count, int B,
                                      void *workspace, size_t workspace_bytes,
                                      sherry_stream_t stream);

/*
 * sherry_gemv_static -- sherry_gemv without a caller workspace: the call
 * allocates nothing.  The paper has no counterpart; this entry point exists
 * for callers that may not allocate device memory on their decode path.
 * Its scratch (re-ordered activations, split-K partial sums and counters) is
 * one device array of SHERRY_STATIC_SCRATCH_BYTES (4 MiB) per device, inside
 * this library.
 *   Arguments, layouts and the result are those of sherry_gemv.
 *   Size limit: sherry_gemv_workspace_bytes(N, K, B) must not exceed
 *   SHERRY_STATIC_SCRATCH_BYTES, otherwise the call returns
 *   SHERRY_ERR_WORKSPACE with the two sizes in sherry_last_error().
 *   Set-up: the first call on a device (with that device current) looks up
 *   the array's device address (cudaGetSymbolAddress) and caches it for the
 *   device's current context (looked up again in a new context, e.g. after
 *   cudaDeviceReset); make that first call before any stream capture.
 *   Sharing: every call on a device uses the same array.  Each call re-writes
 *   the activations and zeroes the partial sums and counters it needs before
 *   its GEMV kernel reads them, so consecutive calls are independent; calls
 *   that overlap on the GPU (other streams, other host threads) race on the
 *   array and give undefined results.
 *   No cudaMalloc, cudaFree or other allocating routine is called.
 * Errors: as sherry_gemv; WORKSPACE for sizes beyond the limit; CUDA if the
 * set-up fails.
 */
sherry_status sherry_gemv_static(const uint32_t *codes, const float *scales, const int8_t *x,
                                 float *y, int64_t N, int64_t K, int B, sherry_stream_t stream);

/* One GEMV of a grouped call.  All pointers are device pointers with the
 * alignment sherry_gemv requires. */
typedef struct {
    const uint32_t *codes;
    const float *scales;
    const int8_t *x;   /* [B][K] */
    float *y;          /* [B][N] */
    int64_t N;
    int64_t K;
} sherry_gemv_desc;

/*
 * sherry_gemv_grouped -- `count` independent GEMVs (count <= SHERRY_MAX_GROUP),
 * all with the same batch B, in one pass: one activation re-ordering launch
 * and one GEMV launch whose warps stream the codes of every GEMV.  This is the
 * decode step of a whole stack of layers whose inputs are already known.  The
 * pages define no grouping; each GEMV is the product of sherry_gemv, and the
 * stack is the batch-1 decode workload of LLaMA-3.2-1B-shaped layers that the
 * method is evaluated on (arXiv 2601.07892, abstract: LLaMA-3.2 1B and 3B).
 *   descs  HOST array of `count` descriptors (copied into the launch
 *          parameters; may be reused as soon as the call returns).
 *   workspace: at least the sum over the group of
 *          sherry_gemv_workspace_bytes(N_i, K_i, B) bytes.
 * Errors: as sherry_gemv, per descriptor; UNSUPPORTED if count > SHERRY_MAX_GROUP.
 */
sherry_status sherry_gemv_grouped(const sherry_gemv_desc *descs, int count, int B,
                                  void *workspace, size_t workspace_bytes,
                                  sherry_stream_t stream);

/*
 * The two halves of sherry_gemv_grouped, for callers that reuse one input
 * across several GEMVs or time the GEMV kernel alone:
 *   sherry_gemv_prepare  re-orders each descriptor's x into the workspace
 *                        (reads descs[i].x, N, K; codes, scales, y unused);
 *   sherry_gemv_run      runs the GEMVs on a workspace prepared by a previous
 *                        sherry_gemv_prepare with the same descriptors' K and
 *                        order and the same B, on the same stream (descs[i].x
 *                        is not read).
 * sherry_gemv_grouped(d, n, B, ws) == prepare(d, n, B, ws) then run(d, n, B, ws).
 * Errors: as sherry_gemv_grouped, each for the fields it reads.
 */
sherry_status sherry_gemv_prepare(const sherry_gemv_desc *descs, int count, int B,
                                  void *workspace, size_t workspace_bytes,
                                  sherry_stream_t stream);
sherry_status sherry_gemv_run(const sherry_gemv_desc *descs, int count, int B,
                              const void *workspace, size_t workspace_bytes,
                              sherry_stream_t stream);

/*
 * Comparison formats.  The pages set Sherry's 1.25 bits per weight against two
 * ternary packings (arXiv 2601.07892, abstract; Figure 2 caption): a 2-bit
 * aligned one and a 1.67-bit one of three weights in five bits.  These calls
 * hold the same ternary matrix in those formats and run the same decode GEMV
 * machinery on them, so that the three can be measured side by side.  Layouts
 * (the pages print none; these are the library's readings):
 *   SHERRY_CMP_I2  2 bits per weight: code 0 -> 0, 1 -> +1, 3 -> -1 (2 -> 0);
 *                  a tile is 128 weights of a row in 8 words; word q holds
 *                  weights 16 q + n at bits [4 n, 4 n + 1] and 16 q + 8 + n at
 *                  bits [4 n + 2, 4 n + 3], n = 0..7; rows in groups of 32:
 *                  codes[((n / 32) * T + t) * 256 + 32 q + n % 32], T = K / 128.
 *   SHERRY_CMP_T3  three weights in five bits: triple (w0, w1, w2) has code
 *                  (w0 + 1) + 3 (w1 + 1) + 9 (w2 + 1); a tile is 32 triples = 96
 *                  weights in 5 words, triple j at bits [5 j, 5 j + 4] of the
 *                  160-bit little-endian string of the words; a row is padded
 *                  with zero weights to T3 = 2 * ceil(K / 192) tiles; rows in
 *                  groups of 32: codes[((n / 32) * T3 + t) * 160 + 32 p + n % 32].
 * The GEMV takes B <= 2 rows of int8 activations (row-major [B][K]) and writes
 * y = s (.) (W . x^T) as sherry_gemv does; it is not tuned beyond the decode
 * kernel it shares with Sherry.
 */
#define SHERRY_CMP_I2 1
#define SHERRY_CMP_T3 2

/* Bytes of codes of an N x K matrix in a comparison format (0 if invalid). */
size_t sherry_cmp_packed_bytes(int fmt, int64_t N, int64_t K);

/* Workspace of a comparison GEMV (the sum over a grouped call's GEMVs):
 * T3 expands each activation triple to a 32-bit word; I2 reads x in place (0). */
size_t sherry_cmp_workspace_bytes(int fmt, int64_t N, int64_t K, int B);

/*
 * sherry_cmp_transcode -- the matrix of Sherry `codes` (N x K, layout above)
 * written in comparison format `fmt` to `out` (sherry_cmp_packed_bytes bytes;
 * T3's padding weights past K are zero weights; padding rows past N hold zero
 * words).  Device pointers, 4-byte aligned.
 * Errors: NULL, SHAPE, ALIGN, UNSUPPORTED (unknown fmt), CUDA.
 */
sherry_status sherry_cmp_transcode(int fmt, const uint32_t *codes, int64_t N, int64_t K,
                                   uint32_t *out, sherry_stream_t stream);

/*
 * sherry_cmp_gemv_grouped -- sherry_gemv_grouped on matrices in comparison
 * format `fmt` (descs[i].codes in that format), B <= 2.  Codes 16-byte
 * aligned; I2 also needs K a multiple of 512 and x 16-byte aligned.
 *   workspace: at least the sum of sherry_cmp_workspace_bytes over the group,
 *   256-byte aligned (may be NULL when that sum is 0).
 * Errors: NULL, SHAPE, ALIGN, UNSUPPORTED (fmt, B > 2, count), WORKSPACE, CUDA.
 */
sherry_status sherry_cmp_gemv_grouped(int fmt, const sherry_gemv_desc *descs, int count, int B,
                                      void *workspace, size_t workspace_bytes,
                                      sherry_stream_t stream);

/* One comparison GEMV writing the exact int32 accumulators acc[B][N]. */
sherry_status sherry_cmp_gemv_acc(int fmt, const uint32_t *codes, const int8_t *x, int32_t *acc,
                                  int64_t N, int64_t K, int B, void *workspace,
                                  size_t workspace_bytes, sherry_stream_t stream);

/*
 * sherry_gemm -- prefill GEMM, Y = X . W^T scaled per output column,
 *   Y[m][n] = s[n] * sum_k X[m][k] * W[n][k]   (the same product for M tokens).
 * The pages define no GEMM: this is the product the abstract serves
 * (arXiv 2601.07892, abstract: ternary weights with int8 activations) taken
 * over M tokens at once, the prefill step of the same decoder layers; at
 * M >= 64 it is a dense contraction and runs on the tensor cores.
 * The kernel decodes weight tiles to int8 in shared memory and runs them on
 * the tcgen05 int8 tensor-core path with int32 accumulators in tensor memory.
 *   codes   [ceil(N/32)][K/128][5][32] uint32; 4-byte aligned.
 *   scales  [N] fp32.
 *   x       [M][K] int8 row-major; 16-byte aligned (tensor-memory-access copies).
 *   y       [M][N] fp32 output, row-major.
 * Errors: NULL, SHAPE, ALIGN, CUDA, TIMEOUT (only through sherry_device_error).
 */
sherry_status sherry_gemm(const uint32_t *codes, const float *scales, const int8_t *x,
                          float *y, int64_t M, int64_t N, int64_t K, sherry_stream_t stream);

/* As sherry_gemm, writing exact int32 accumulators acc[M][N]. */
sherry_status sherry_gemm_acc(const uint32_t *codes, const int8_t *x, int32_t *acc,
                              int64_t M, int64_t N, int64_t K, sherry_stream_t stream);

/*
 * Device-side error word.  Kernels that wait on barriers bound every wait;
 * when one runs out the kernel records SHERRY_ERR_TIMEOUT here, releases what
 * it holds and returns instead of hanging.  sherry_device_error() synchronises
 * the current device, returns the recorded status (SHERRY_OK if none) and
 * clears it.
 */
sherry_status sherry_device_error(void);

/*
 * sherry_set_wait_limit -- limit, in SM clock cycles, of the bounded waits of
 * kernels launched after this call by any thread of the process (the GEMM's
 * operand and accumulator barriers).  0 restores the default of 4e9 cycles
 * (about 2 s at 1.9 GHz).  Meant for tests and failure drills: with a small
 * limit the waits give up, the kernel records SHERRY_ERR_TIMEOUT (read and
 * cleared by sherry_device_error), lets the copies and MMAs it already issued
 * finish (those drains keep their own long limit), releases its tensor memory
 * and returns; its output is then undefined.  The setting is process-wide.
 * Errors: SHAPE if cycles < 0.
 */
sherry_status sherry_set_wait_limit(int64_t cycles);

/*
 * sherry_probe_mma_i8 -- measurement aid, not part of the product: one CTA
 * per SM (their number written to *ctas) issues `iters` x 4 back-to-back
 * tcgen05.mma.cta_group::1.kind::i8 of the GEMM's shape (M = 128 weight rows,
 * N = 256 tokens, K = 32, operands in 128-byte-swizzled shared memory) on
 * zeroed operands.  Timing the launch gives the int8 tensor-core rate the
 * GEMM's MMAs can reach on this device: *ctas * iters * 4 * 128 * 256 * 32
 * multiply-accumulates (twice that in ops).  Asynchronous on `stream`.
 * Errors: NULL, SHAPE (iters < 1), CUDA.
 */
sherry_status sherry_probe_mma_i8(int iters, int *ctas, sherry_stream_t stream);

/* Text of a status code (static string). */
const char *sherry_status_string(sherry_status status);

/* Text of the last CUDA error seen by this thread in a library call. */
const char *sherry_last_error(void);

/* Library version as MAJOR * 10000 + MINOR * 100 + PATCH. */
int sherry_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SHERRY_H */
