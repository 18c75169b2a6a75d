// gemv.cu -- decode GEMV on Sherry codes: y = s (.) (W_ternary . x_int8), B <= 16,
// and the activation front-ends that feed it.
//
// The product is the one the pages state for ternary weights with 3:4 blocks
// coded in five bits (arXiv 2601.07892, abstract; Figure 2 caption, which
// presents the block patterns as suited to SIMD).  On B200 a batch-1 GEMV is bound by HBM reads of
// the codes (0.15625 bytes per weight) only if the decode costs a few
// instructions per 4-weight block.  Every kernel here decodes the same way:
//
//   * a thread decodes whole 128-weight tiles with 32-bit SWAR logic: for a
//     (position i, block group beta) pair one selector word holds, per nibble,
//     (zero position | sign << 2) of one block, and one byte permute (PRMT)
//     against an 8-byte table per position turns four nibbles into four
//     ternary bytes; shifts that move left run as IMAD on the FMA pipe, so the
//     ALU pipe carries only the permutes, the selector merges and a few shifts;
//   * the activations are re-ordered into the order in which the decoded
//     bytes meet the multiply-accumulate.
//
// Kernels:
//   gemv_dot_kernel   B <= 2 (the decode path): per-warp rings of 4-tile
//                     chunks filled by bulk copies (cp.async.bulk completing
//                     on one mbarrier per stage), dp4a against broadcast
//                     activation words, chunk-balanced warp ranges, items cut
//                     between warps summed in shared memory.  Small int8 calls
//                     copy raw x and re-order it in the kernel (no re-order
//                     launch).
//   gemv_pipe_kernel  B >= 3: per-warp 3-stage cp.async rings of code chunks;
//                     the int8 MMA m16n8k32 takes the decoded weights as its A
//                     fragment from registers and one batch row per column, so
//                     batches up to 8 cost the same MMA count as one.  Its
//                     activation fragments come from a layout in fragment
//                     order (xw_word), so that each warp load covers whole
//                     128-byte lines.
//   gemv_kernel       the general fallback (K not a multiple of 512, or code
//                     rows not 16-byte aligned), MMA from registers.
//   xprep_kernel      re-orders int8 activations, or quantizes bf16 ones per
//                     token first; clears the K-part sums of split rows.
//   xprep_f32_kernel  the fp32 / SwiGLU front-end: one thread-block cluster
//                     per token row, maxima exchanged through distributed
//                     shared memory.
// Rows longer than 8192 are split into K-parts, summed exactly with integer
// atomics.  Consecutive launches use programmatic dependent launch.
#include <algorithm>
#include <cstdio>
#include <cstring>
#include <mutex>

#include <cooperative_groups.h>

#include "common.cuh"

namespace sherry {
namespace {

// ---------------------------------------------------------------------------
// Launch parameters
// ---------------------------------------------------------------------------
struct GemvDesc {
    const uint32_t *codes;
    const float *scales;
    const float *xscale;  // per batch row activation scales (bf16 front-end), else null
    const uint4 *xw;      // re-ordered activations (layout: see xw_word)
    const int8_t *x;      // raw int8 activations [B][K] (re-ordered inside the dot kernel)
    const uint16_t *xbf;  // raw bf16 activations [B][K] (quantized inside the dot kernel)
    void *out;            // float y[B][N] or int32 acc[B][N]
    int32_t *part_acc;    // K-part partial sums [B][N] (pipelined kernel, kparts > 1)
    uint32_t *part_cnt;   // K-parts finished per unit (pipelined kernel, kparts > 1)
    int N;
    int T;                // tiles per row (K / 128)
    int Tp;               // tile stride of xw (T rounded up to a whole chunk)
    int unit_begin16;     // register kernel: first 16-row unit in the group
    int units;            // pipelined kernels: items per K-part column (32-row units, or
                          // groups of 1 or 2 units for the dot kernel)
    int units32;          // 32-row units of the GEMV (ceil(N / 32))
    int nchunk;           // pipelined kernel: 4-tile chunks per row
    int kparts;           // pipelined kernel: K-parts per unit
    int cpp;              // pipelined kernel: chunks per K-part
    int chunk_begin;      // pipelined kernel: first 4-tile chunk of the group (all groups' rows
                          // in order, each row's K-parts in order)
};

struct GemvParams {
    int count;
    int B;
    // 1: this launch follows the call's own re-order launch, whose grid writes
    // no codes and started only after every earlier ordinary launch completed,
    // so the first code copies may be issued before griddepcontrol.wait.  0:
    // the kernel before may be the caller's (e.g. the one that wrote the
    // codes), so nothing is read before the wait.
    int prefetch_codes;
    int pad0;
    int total_units16;    // register kernel
    int total_chunks;     // pipelined kernel: chunks of all groups (the balancing space)
    // Constants passed at run time so that they live in registers instead of
    // being re-created per use, and so that left shifts by a power of two stay
    // multiplications (IMAD on the FMA pipe) instead of ALU shifts.
    uint32_t mul4, mul2;          // 4, 2
    uint32_t m33, m55, m44;       // masks
    uint32_t tlo[4], thi[4];      // PRMT byte tables of the four positions
    uint32_t f16one, f16negz;     // fp16x2 1.0 and -0.0 (high-half copy, see hi_half)
    GemvDesc d[SHERRY_MAX_GROUP];
};

struct XprepDesc {
    const int8_t *x;
    const uint16_t *xbf;  // bf16 activations to quantize (xprep_bf16_kernel), else null
    float *xscale;        // bf16: per batch row activation scales written here
    uint32_t *xw;         // first word of this GEMV's workspace region
    uint32_t *zero;       // split-K partial sums and counters to clear
    int K;
    int Tp;
    int unit_begin;       // first work unit of this GEMV
    int xunits;           // int8: (batch row, 4 tiles) warp units, B * Tp / 4; bf16: rows
    int zero_words;       // words at `zero` (0 if the rows are not split)
};

struct XprepParams {
    int count;
    int B;
    int total_units;
    int xrows;            // layout of the re-ordered activations (see xw_word)
    XprepDesc d[SHERRY_MAX_GROUP];
};

// Front-end on fp32 activations: the y of a previous GEMV, or (u set) the
// SwiGLU h = silu(g) * u of a gate and an up projection.
struct XprepF32Desc {
    const float *x;       // [B][K] activations; SwiGLU: the gate outputs g
    const float *u;       // SwiGLU: the up outputs [B][K]; null for plain fp32
    float *xscale;        // per batch row activation scales written here
    uint32_t *xw;         // re-ordered activations (see xw_word), or null
    int8_t *q;            // natural-order int8 output [B][K] (front-end alone), or null
    uint32_t *zero;       // split-K partial sums and counters to clear
    int K;
    int Tp;
    int cluster_begin;    // first cluster (= token row) of this GEMV
    int zero_words;
};

struct XprepF32Params {
    int count;
    int B;
    int total_clusters;
    int xrows;            // layout of the re-ordered activations (see xw_word)
    XprepF32Desc d[SHERRY_MAX_GROUP];
};

constexpr int kGemvThreads = 256;
constexpr int kGemvWarps = kGemvThreads / 32;

constexpr int kUnitRows = 32;      // pipelined kernel: rows per unit (two m16 blocks)
constexpr int kChunkTiles = 4;     // tiles per K-chunk = per ring stage
// longest K-part: 16 chunks = 8192 weights per row, so rows up to K = 8192 are
// never split.  A split row's K-parts meet through integer atomics and a
// memory fence per part, which cost far more than the balance they buy:
// measured on the 16-layer stacks, 4-chunk parts ran the 3B stack at B = 4 in
// 245 us and the 1B stack in 54.4 us, 16-chunk parts in 107 us and 52.4 us.
// Long rows (K > 8192) still split; an item cut between the warps of a CTA
// is summed in shared memory instead.
constexpr int kMaxPartChunks = 16;
constexpr int kRing = 3;           // stages per warp
// A stage holds one chunk: 4 tile blocks of 5 planes x 32 rows (160 words, a
// contiguous 2560 bytes in global memory), each block padded to 168 words in
// shared memory so that a read of (tile t, plane p, rows g + 8 rb) by lanes
// (g, t) hits 32 distinct banks.
constexpr int kTileWords = 5 * kUnitRows;            // 160
constexpr int kTileWordsPadded = kTileWords + 8;     // 168
constexpr int kStageWords = kChunkTiles * kTileWordsPadded;
constexpr int kPipeThreads = 512;  // one CTA of 16 warps per SM (see PipeShape)
constexpr int kPipeWarps = kPipeThreads / 32;
constexpr size_t kPipeSmem = (size_t)kPipeWarps * kRing * kStageWords * 4;

int64_t padded_tiles(int64_t K) {
    const int64_t T = K / SHERRY_TILE_K;
    return (T + kChunkTiles - 1) / kChunkTiles * kChunkTiles;
}
int64_t round_words(int64_t w) { return (w + 63) / 64 * 64; }  // 256-byte regions

// Layout of a call's re-ordered activations, fixed by the batch B alone so
// that a prepared workspace and the run that reads it always agree.
//   B <= 2 (the small-batch kernel): [b][Tp][32 words], tile by tile.
//   B >= 3 (the MMA kernels): batch rows in groups of R = xgroup_rows(B) rows
//   (4 for B <= 4, else 8; the last group padded), laid out as
//   [group][chunk c][uint4 j][row r][tile t of the chunk][word e]: uint4 j of
//   tile 4c + t of row r holds the tile's re-ordered words 4j .. 4j+3.  A
//   warp's fragment load j of a chunk (lane (g, t) reads row g of the group,
//   tile t) then covers 64 R contiguous bytes, i.e. 2 or 4 whole 128-byte
//   lines, where the tile-by-tile layout spread it over 16 or 32 lines.
__host__ __device__ __forceinline__ int xgroup_rows(int B) { return B <= 2 ? 0 : (B <= 4 ? 4 : 8); }
// rows of the region: B, or B padded to whole groups
int64_t xw_rows(int B) {
    const int R = xgroup_rows(B);
    return R ? (int64_t)(B + R - 1) / R * R : (int64_t)B;
}
// word index of re-ordered word l (0..31) of tile t of batch row b; R =
// xgroup_rows(B), Tp a multiple of 4
__device__ __forceinline__ size_t xw_word(int R, int Tp, int b, int t, int l) {
    if (R == 0) return ((size_t)b * Tp + t) * 32 + l;
    const int grp = b / R, r = b - grp * R;
    return (((((size_t)grp * (Tp >> 2) + (t >> 2)) * 8 + (l >> 2)) * R + r) * 4 + (t & 3)) * 4 + (l & 3);
}

// K-parts per 32-row unit in the pipelined kernel.
int64_t kparts_for(int64_t K) {
    const int64_t nchunk = padded_tiles(K) / kChunkTiles;
    return (nchunk + kMaxPartChunks - 1) / kMaxPartChunks;
}

// Split-K words of one GEMV: partial sums [B][N] and per-unit counters, only
// when the rows are split into several K-parts.
int64_t split_words(int64_t N, int64_t K, int B) {
    if (kparts_for(K) <= 1) return 0;
    return round_words((int64_t)B * N + (N + kUnitRows - 1) / kUnitRows);
}

// Workspace words of one GEMV: re-ordered activations, then the split-K words.
int64_t ws_words(int64_t N, int64_t K, int B) {
    return round_words(xw_rows(B) * padded_tiles(K) * 32) + split_words(N, K, B);
}

// ---------------------------------------------------------------------------
// Activation re-order
// ---------------------------------------------------------------------------
// Word q (of 32) of tile t (t < Tp) of batch row b, stored at xw_word(b, t, q):
// q = 2 (4 i + beta) + h holds the activations met
// by char4(i, beta, h) of tile t: bytes x[b][128 t + 16 k' + 64 h + 4 beta + i],
// k' = 0..3; tiles t >= K/128 are zero so that padded chunks contribute
// nothing.  The split-K partial sums and counters are cleared.
//
// One warp per work unit: a (batch row, tile) unit -- lane l loads raw word l
// of the tile (128 contiguous bytes per warp); the bytes of output word q are
// byte i of raw words 4 k' + 16 h + beta, fetched with four shuffles and
// merged with three byte permutes -- or a unit of 32 words to clear.
__device__ __forceinline__ uint32_t reorder_word(uint32_t raw, int lane) {
    const int i = lane >> 3, beta = (lane >> 1) & 3, h = lane & 1;
    const uint32_t pick2 = (uint32_t)i | ((uint32_t)(4 + i) << 4);  // byte i of a, byte i of b
    const uint32_t v0 = __shfl_sync(0xFFFFFFFFu, raw, 0 + 16 * h + beta);
    const uint32_t v1 = __shfl_sync(0xFFFFFFFFu, raw, 4 + 16 * h + beta);
    const uint32_t v2 = __shfl_sync(0xFFFFFFFFu, raw, 8 + 16 * h + beta);
    const uint32_t v3 = __shfl_sync(0xFFFFFFFFu, raw, 12 + 16 * h + beta);
    return prmt(prmt(v0, v1, pick2), prmt(v2, v3, pick2), 0x5410u);
}

// Programmatic dependent launch: the re-order and GEMV kernels are launched so
// that they may start while the kernel before them in the stream still runs.
// Each waits for it (griddepcontrol.wait: the prior grid completed and its
// writes are visible) before reading or writing anything that grid may touch;
// without a prior grid the wait returns.  Each lets its own dependents be
// scheduled from its start (griddepcontrol.launch_dependents), which only
// moves their launch work under this grid's tail: they still wait for its
// completion.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_allow_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Activation front-end (int8 activations of the W1.25A8 setting; the pages
// do not say how they are made): per token, amax = max |x|, s = amax / 127,
// q = clamp(rint(x * (127 / amax)), -127, 127), all in fp32 with round-to-
// nearest-even; amax = 0 gives s = 0, q = 0.  x is bf16 (the upper half of an
// fp32).
__device__ __forceinline__ float bf16_lo(uint32_t two) { return __uint_as_float(two << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t two) { return __uint_as_float(two & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t quant_byte(float x, float inv) {
    int q = __float2int_rn(__fmul_rn(x, inv));
    q = max(-127, min(127, q));
    return (uint32_t)(q & 0xFF);
}
// four consecutive bf16 values (two words) -> four int8 in one word, k order
__device__ __forceinline__ uint32_t quant_word(uint2 v, float inv) {
    return quant_byte(bf16_lo(v.x), inv) | (quant_byte(bf16_hi(v.x), inv) << 8) |
           (quant_byte(bf16_lo(v.y), inv) << 16) | (quant_byte(bf16_hi(v.y), inv) << 24);
}
// max |x| over one bf16 row, reduced over the warp (all lanes get it)
__device__ __forceinline__ float row_absmax_bf16(const uint16_t *row, int K, int lane) {
    float m = 0.0f;
    const uint4 *r4 = reinterpret_cast<const uint4 *>(row);  // 8 values per uint4
    // eight loads in flight per lane: the row comes from L2, one load at a time
    // would expose its latency K / 256 times
#pragma unroll 8
    for (int i = lane; i < K / 8; i += 32) {
        const uint4 v = __ldg(r4 + i);
        m = fmaxf(m, fmaxf(fmaxf(fabsf(bf16_lo(v.x)), fabsf(bf16_hi(v.x))),
                           fmaxf(fabsf(bf16_lo(v.y)), fabsf(bf16_hi(v.y)))));
        m = fmaxf(m, fmaxf(fmaxf(fabsf(bf16_lo(v.z)), fabsf(bf16_hi(v.z))),
                           fmaxf(fabsf(bf16_lo(v.w)), fabsf(bf16_hi(v.w)))));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    return m;
}

constexpr int kXqTiles = 4;  // tiles per re-order unit (one chunk of one batch row)

// bf16 front-end: one CTA per (GEMV, batch row), its warps taking the row's
// tiles in turn.  Each warp loads its tiles once (rows up to kBfKeep tiles per
// warp, K <= 8192, stay in registers between the passes), the CTA reduces the
// token's absmax through shared memory, and each warp quantizes and re-orders
// its tiles: one round trip to L2 per row instead of one per tile group.
constexpr int kBfWarps = 8;
constexpr int kBfKeep = 8;

__device__ __forceinline__ float absmax4_bf16(uint2 v) {
    return fmaxf(fmaxf(fabsf(bf16_lo(v.x)), fabsf(bf16_hi(v.x))),
                 fmaxf(fabsf(bf16_lo(v.y)), fabsf(bf16_hi(v.y))));
}

__global__ void __launch_bounds__(kBfWarps * 32) xprep_bf16_kernel(const __grid_constant__ XprepParams P) {
    pdl_allow_dependents();
    pdl_wait();  // x may come from the kernel before; the last GEMV may still read xw
    __shared__ float wmax[kBfWarps];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int u = blockIdx.x; u < P.total_units; u += gridDim.x) {
        int lo = 0, hi = P.count - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (P.d[mid].unit_begin <= u) lo = mid; else hi = mid - 1;
        }
        const XprepDesc &D = P.d[lo];
        const int local = u - D.unit_begin;
        if (local < D.xunits) {
            const int b = local;
            const int T = D.K / SHERRY_TILE_K;
            // four bf16 values per uint2: tile t, lane l at t * 32 + l
            const uint2 *row = reinterpret_cast<const uint2 *>(D.xbf + (size_t)b * D.K);
            uint2 keep[kBfKeep];
            float m = 0.0f;
#pragma unroll
            for (int j = 0; j < kBfKeep; j++) {
                const int t = warp + kBfWarps * j;
                keep[j] = t < T ? __ldg(row + (size_t)t * 32 + lane) : make_uint2(0u, 0u);
                m = fmaxf(m, absmax4_bf16(keep[j]));
            }
            for (int t = warp + kBfWarps * kBfKeep; t < T; t += kBfWarps)
                m = fmaxf(m, absmax4_bf16(__ldg(row + (size_t)t * 32 + lane)));
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
            if (lane == 0) wmax[warp] = m;
            __syncthreads();
            float amax = wmax[0];
#pragma unroll
            for (int w = 1; w < kBfWarps; w++) amax = fmaxf(amax, wmax[w]);
            const float inv = amax > 0.0f ? __fdiv_rn(127.0f, amax) : 0.0f;
            if (threadIdx.x == 0) D.xscale[b] = amax > 0.0f ? __fdiv_rn(amax, 127.0f) : 0.0f;
#pragma unroll
            for (int j = 0; j < kBfKeep; j++) {
                const int t = warp + kBfWarps * j;
                if (t < D.Tp)
                    D.xw[xw_word(P.xrows, D.Tp, b, t, lane)] =
                        reorder_word(t < T ? quant_word(keep[j], inv) : 0u, lane);
            }
            for (int t = warp + kBfWarps * kBfKeep; t < D.Tp; t += kBfWarps)
                D.xw[xw_word(P.xrows, D.Tp, b, t, lane)] =
                    reorder_word(t < T ? quant_word(__ldg(row + (size_t)t * 32 + lane), inv) : 0u, lane);
            __syncthreads();  // wmax is rewritten for the CTA's next row
        } else {
            const int w = (local - D.xunits) * (kBfWarps * 32) + (int)threadIdx.x;
            if (w < D.zero_words) D.zero[w] = 0u;
        }
    }
}

__global__ void __launch_bounds__(256) xprep_kernel(const __grid_constant__ XprepParams P) {
    pdl_allow_dependents();
    pdl_wait();  // x may come from the kernel before; the last GEMV may still read xw
    const int lane = threadIdx.x & 31;
    const int nw = gridDim.x * (blockDim.x >> 5);
    for (int u = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); u < P.total_units; u += nw) {
        int lo = 0, hi = P.count - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (P.d[mid].unit_begin <= u) lo = mid; else hi = mid - 1;
        }
        const XprepDesc &D = P.d[lo];
        const int local = u - D.unit_begin;
        if (local < D.xunits) {
            // int8: unit = (row b, 4 tiles); the four tiles' loads are issued together
            const int per_row = D.Tp / kXqTiles;
            const int b = local / per_row, t0 = (local - b * per_row) * kXqTiles;
            const int T = D.K / SHERRY_TILE_K;
            // x rows are 4-byte aligned (x is, and K is a multiple of 128)
            const uint32_t *row = reinterpret_cast<const uint32_t *>(D.x + (size_t)b * D.K);
            uint32_t raw[kXqTiles];
#pragma unroll
            for (int q = 0; q < kXqTiles; q++)
                raw[q] = t0 + q < T ? __ldg(row + (size_t)(t0 + q) * (SHERRY_TILE_K / 4) + lane) : 0u;
#pragma unroll
            for (int q = 0; q < kXqTiles; q++)
                D.xw[xw_word(P.xrows, D.Tp, b, t0 + q, lane)] = reorder_word(raw[q], lane);
        } else {
            const int w = (local - D.xunits) * 32 + lane;
            if (w < D.zero_words) D.zero[w] = 0u;
        }
    }
}

// SwiGLU of the LLaMA MLP: silu(g) * u = g / (1 + e^-g) * u, each operation
// rounded once (IEEE single precision; expf is CUDA's, within 2 ulp).  A g so
// negative that e^-g overflows gives g / inf = -0.
__device__ __forceinline__ float swiglu_f32(float g, float u) {
    return __fmul_rn(__fdiv_rn(g, __fadd_rn(1.0f, expf(-g))), u);
}

// Four consecutive activations of a token row from offset `off`.
__device__ __forceinline__ float4 act4(const XprepF32Desc &D, size_t off) {
    float4 a = __ldg(reinterpret_cast<const float4 *>(D.x + off));
    if (D.u) {
        const float4 v = __ldg(reinterpret_cast<const float4 *>(D.u + off));
        a.x = swiglu_f32(a.x, v.x);
        a.y = swiglu_f32(a.y, v.y);
        a.z = swiglu_f32(a.z, v.z);
        a.w = swiglu_f32(a.w, v.w);
    }
    return a;
}

constexpr int kF32Cluster = 8;                  // CTAs per token row (one cluster)
constexpr int kF32Threads = 256;
constexpr int kF32Warps = kF32Threads / 32;
constexpr int kF32ClusterWarps = kF32Cluster * kF32Warps;

// One thread-block cluster per (GEMV, token row).  Its 64 warps take the
// row's 128-element tiles in turn: the first pass forms the activations and
// their absolute maximum, the CTAs exchange their maxima through distributed
// shared memory at a cluster barrier, and the second pass quantizes them with
// the per-token rule of the bf16 front-end and re-orders them (or writes them
// in natural order).  A warp keeps the activations of its first two tiles in
// registers between the passes (every tile of rows up to K = 16384) and forms
// those of later tiles again.
__global__ void __launch_bounds__(kF32Threads) xprep_f32_kernel(const __grid_constant__ XprepF32Params P) {
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    __shared__ float warp_max[kF32Warps];
    __shared__ float cta_max, row_max;
    pdl_allow_dependents();
    pdl_wait();  // x and u may come from the kernel before; the last GEMV may still read xw
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int rank = (int)cluster.block_rank();
    const int ci = (int)(blockIdx.x / kF32Cluster);
    int lo = 0, hi = P.count - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (P.d[mid].cluster_begin <= ci) lo = mid; else hi = mid - 1;
    }
    const XprepF32Desc &D = P.d[lo];
    const int b = ci - D.cluster_begin;
    const int T = D.K / SHERRY_TILE_K;
    const int cw = rank * kF32Warps + warp;  // warp index within the cluster
    const size_t row = (size_t)b * D.K;

    auto absmax4 = [](float m, const float4 &a) {
        return fmaxf(m, fmaxf(fmaxf(fabsf(a.x), fabsf(a.y)), fmaxf(fabsf(a.z), fabsf(a.w))));
    };
    float m = 0.0f;
    float4 h0 = make_float4(0.0f, 0.0f, 0.0f, 0.0f), h1 = h0;  // tiles cw and cw + 64
    if (cw < T) h0 = act4(D, row + (size_t)cw * SHERRY_TILE_K + 4 * lane);
    if (cw + kF32ClusterWarps < T)
        h1 = act4(D, row + (size_t)(cw + kF32ClusterWarps) * SHERRY_TILE_K + 4 * lane);
    m = absmax4(absmax4(m, h0), h1);
    for (int t = cw + 2 * kF32ClusterWarps; t < T; t += kF32ClusterWarps)
        m = absmax4(m, act4(D, row + (size_t)t * SHERRY_TILE_K + 4 * lane));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    if (lane == 0) warp_max[warp] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        float c = 0.0f;
        for (int w = 0; w < kF32Warps; w++) c = fmaxf(c, warp_max[w]);
        cta_max = c;
    }
    cluster.sync();  // every CTA's maximum is in its shared memory
    if (warp == 0) {
        float r = lane < kF32Cluster ? *cluster.map_shared_rank(&cta_max, (unsigned)lane) : 0.0f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) r = fmaxf(r, __shfl_xor_sync(0xFFFFFFFFu, r, o));
        if (lane == 0) row_max = r;
    }
    __syncthreads();
    const float amax = row_max;
    const float inv = amax > 0.0f ? __fdiv_rn(127.0f, amax) : 0.0f;
    if (rank == 0 && threadIdx.x == 0) D.xscale[b] = amax > 0.0f ? __fdiv_rn(amax, 127.0f) : 0.0f;

    const int t_end = D.q ? T : D.Tp;
    for (int t = cw, j = 0; t < t_end; t += kF32ClusterWarps, j++) {
        uint32_t raw = 0u;
        if (t < T) {
            const float4 a = j == 0 ? h0 : j == 1 ? h1 : act4(D, row + (size_t)t * SHERRY_TILE_K + 4 * lane);
            raw = quant_byte(a.x, inv) | (quant_byte(a.y, inv) << 8) | (quant_byte(a.z, inv) << 16) |
                  (quant_byte(a.w, inv) << 24);
        }
        if (D.q)
            reinterpret_cast<uint32_t *>(D.q + row + (size_t)t * SHERRY_TILE_K)[lane] = raw;
        else
            D.xw[xw_word(P.xrows, D.Tp, b, t, lane)] = reorder_word(raw, lane);
    }
    // the GEMV's split-K words, cleared by its clusters together
    const int stride = P.B * kF32Cluster * kF32Threads;
    for (int w = (b * kF32Cluster + rank) * kF32Threads + (int)threadIdx.x; w < D.zero_words; w += stride)
        D.zero[w] = 0u;
    cluster.sync();  // no CTA leaves while another may still read its maximum
}

// ---------------------------------------------------------------------------
// Device helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mma_s8(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                       uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t ld_code(const uint32_t *p) {
    uint32_t v;
    asm volatile("ld.global.nc.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}

__device__ __forceinline__ uint4 ld_x(const uint4 *p) {
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t pick(const uint4 &v, int j) {
    return j == 0 ? v.x : j == 1 ? v.y : j == 2 ? v.z : v.w;
}

__device__ __forceinline__ uint32_t lop_mux(uint32_t m, uint32_t a, uint32_t b) {  // m ? a : b
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xCA;" : "=r"(d) : "r"(m), "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ uint32_t lop_merge(uint32_t a, uint32_t b, uint32_t m) {  // (a&m)|(b&~m)
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xE4;" : "=r"(d) : "r"(a), "r"(b), "r"(m));
    return d;
}
__device__ __forceinline__ uint32_t lop_or_masked(uint32_t x, uint32_t m, uint32_t z) {  // (x&m)|z
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(x), "r"(m), "r"(z));
    return d;
}
// Multiplication by a power of two passed at run time, so that the compiler
// keeps it on the FMA pipe instead of turning it into an ALU shift.
__device__ __forceinline__ uint32_t imul(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.lo.u32 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}


// Scale of output (row, batch row b): s[row], times the activation scale of b
// when the activations came through the bf16 front-end (one fp32 rounding).
__device__ __forceinline__ float out_scale(const GemvDesc &D, int row, int b) {
    const float s = __ldg(D.scales + row);
    return D.xscale ? __fmul_rn(s, __ldg(D.xscale + b)) : s;
}

struct Consts {
    uint32_t mul4, mul2, m33, m55, m44;
    uint32_t tlo[4], thi[4];
    uint32_t f16one, f16negz;
};

__device__ __forceinline__ void load_consts(const GemvParams &P, Consts &C) {
    C.mul4 = P.mul4;
    C.mul2 = P.mul2;
    C.m33 = P.m33;
    C.m55 = P.m55;
    C.m44 = P.m44;
#pragma unroll
    for (int i = 0; i < 4; i++) {
        C.tlo[i] = P.tlo[i];
        C.thi[i] = P.thi[i];
    }
    C.f16one = P.f16one;
    C.f16negz = P.f16negz;
}

// High half of a selector word, moved to the low half for the next PRMT (which
// reads selector bits 0..15 only).  Done as one fp16x2 FMA whose first operand
// takes the high half in both lanes: h * 1.0 + (-0.0) = h exactly for every
// finite h, subnormals included (no .ftz).  A selector nibble never has bit 3
// set, so bit 11 of the half is clear, its exponent field is never all ones,
// and h is never NaN or Inf.  The FMA runs on the FMA-lite pipe, which the
// rest of the decode leaves idle, instead of taking an ALU shift or a two-
// instruction mul.hi on the heavy FMA pipe.
__device__ __forceinline__ uint32_t hi_half(const Consts &C, uint32_t sel) {
    uint32_t d;
    asm("{\n\t.reg .b16 l, h;\n\t.reg .b32 t;\n\t"
        "mov.b32 {l, h}, %1;\n\tmov.b32 t, {h, h};\n\t"
        "fma.rn.f16x2 %0, t, %2, %3;\n\t}"
        : "=r"(d)
        : "r"(sel), "r"(C.f16one), "r"(C.f16negz));
    return d;
}

// Per-row tile state of the pipelined kernel: zero-position nibbles per block
// group and the four per-position sign planes.  Selector of (i, beta):
//   zm[beta] | (sign plane i moved so block 4k+beta's bit lands at 4k+2) & 0x44444444.
// Work split: masks, merges, permutes and right shifts on the ALU pipe (2
// cycles per warp instruction); left shifts on the heavy FMA pipe as IMAD (2
// cycles); the selectors' high halves on the FMA-lite pipe (hi_half).
struct TileDecoder6 {
    uint32_t zm[4];
    uint32_t sg[4];

    __device__ __forceinline__ void load(const Consts &C, uint32_t z0, uint32_t z1, uint32_t s0,
                                         uint32_t s1, uint32_t s2) {
        zm[0] = z0 & C.m33;
        zm[1] = z1 & C.m33;
        zm[2] = (z0 >> 2) & C.m33;
        zm[3] = (z1 >> 2) & C.m33;
        // bit-sliced zero positions: lo bit (L) and hi bit (H) of p_j at bit j
        const uint32_t L = lop_merge(z0, imul(z1, C.mul2), C.m55);
        const uint32_t H = lop_merge(z0 >> 1, z1, C.m55);
        // sign of position i when kept: rank 0; rank 0 if p == 0 else 1;
        // rank 1 if p <= 1 else 2; rank 2
        sg[0] = s0;
        sg[1] = lop_mux(L | H, s1, s0);
        sg[2] = lop_mux(H, s2, s1);
        sg[3] = s2;
    }
    __device__ __forceinline__ uint32_t sel(const Consts &C, int i, int beta) const {
        const uint32_t v = beta == 0 ? imul(sg[i], C.mul4)
                         : beta == 1 ? imul(sg[i], C.mul2)
                         : beta == 2 ? sg[i] : (sg[i] >> 1);
        return lop_or_masked(v, C.m44, zm[beta]);
    }
};

// ---------------------------------------------------------------------------
// Register kernel (general fallback): each warp owns 16 rows x all of K; a
// thread decodes rows g and g+8 of tile 4s + t and keeps the next slice's code
// words in registers.
// ---------------------------------------------------------------------------
// NB = number of 8-row batch groups (1: B <= 8, 2: B <= 16).
template <int NB, bool ACC_OUT>
__global__ void __launch_bounds__(kGemvThreads) gemv_kernel(const __grid_constant__ GemvParams P) {
    pdl_allow_dependents();
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int nwarps = gridDim.x * kGemvWarps;
    for (int u = blockIdx.x * kGemvWarps + (threadIdx.x >> 5); u < P.total_units16; u += nwarps) {
        int lo = 0, hi = P.count - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (P.d[mid].unit_begin16 <= u) lo = mid; else hi = mid - 1;
        }
        const GemvDesc &D = P.d[lo];
        const int N = D.N, T = D.T;
        const int r0 = (u - D.unit_begin16) * 16 + g, r1 = r0 + 8;
        const bool v0 = r0 < N, v1 = r1 < N;
        // word (p, row, tile) = ((row / 32) * T + tile) * 160 + 32 p + row % 32;
        // rows past N inside the last group are zero padding, so loads need no row test
        const uint32_t *c0 = D.codes + (size_t)(r0 / 32) * T * 160 + (r0 % 32);
        const uint32_t *c1 = D.codes + (size_t)(r1 / 32) * T * 160 + (r1 % 32);

        int acc[NB][4];
#pragma unroll
        for (int nb = 0; nb < NB; nb++) acc[nb][0] = acc[nb][1] = acc[nb][2] = acc[nb][3] = 0;

        const int nslices = (T + 3) >> 2;
        uint32_t w0[5], w1[5];
        {
            const int tile = t;
            const bool tv = tile < T;
#pragma unroll
            for (int p = 0; p < 5; p++) {
                w0[p] = tv ? ld_code(c0 + (size_t)tile * 160 + p * 32) : 0u;
                w1[p] = tv ? ld_code(c1 + (size_t)tile * 160 + p * 32) : 0u;
            }
        }
        for (int s = 0; s < nslices; s++) {
            const int tile = s * 4 + t;
            const bool tv = tile < T;
            TileDecoder d0, d1;
            d0.load(w0[0], w0[1], w0[2], w0[3], w0[4]);
            d1.load(w1[0], w1[1], w1[2], w1[3], w1[4]);
            uint4 xv[NB][8];
#pragma unroll
            for (int nb = 0; nb < NB; nb++) {
                const int b = nb * 8 + g;
                const bool xvld = tv && b < P.B;
                const int R = xgroup_rows(P.B);
#pragma unroll
                for (int k = 0; k < 8; k++)
                    xv[nb][k] = xvld ? ld_x(D.xw + xw_word(R, D.Tp, b, tile, 4 * k) / 4) : make_uint4(0, 0, 0, 0);
            }
            if (s + 1 < nslices) {  // prefetch the next slice's code words
                const int nt = tile + 4;
                const bool ntv = nt < T;
#pragma unroll
                for (int p = 0; p < 5; p++) {
                    w0[p] = ntv ? ld_code(c0 + (size_t)nt * 160 + p * 32) : 0u;
                    w1[p] = ntv ? ld_code(c1 + (size_t)nt * 160 + p * 32) : 0u;
                }
            }
#pragma unroll
            for (int i = 0; i < 4; i++) {
                const uint32_t tlo = table_lo(i), thi = table_hi(i);
#pragma unroll
                for (int beta = 0; beta < 4; beta++) {
                    const uint32_t s0 = d0.sel(i, beta), s1 = d1.sel(i, beta);
                    const uint32_t a0 = prmt(tlo, thi, s0);
                    const uint32_t a2 = prmt(tlo, thi, s0 >> 16);
                    const uint32_t a1 = prmt(tlo, thi, s1);
                    const uint32_t a3 = prmt(tlo, thi, s1 >> 16);
                    const int m = 4 * i + beta;
#pragma unroll
                    for (int nb = 0; nb < NB; nb++) {
                        const uint4 &xq = xv[nb][m >> 1];
                        mma_s8(acc[nb], a0, a1, a2, a3, pick(xq, (m & 1) * 2),
                               pick(xq, (m & 1) * 2 + 1));
                    }
                }
            }
        }
        // epilogue: c0 = (row g, col 2t), c1 = (row g, col 2t+1), c2/c3 = row g+8
#pragma unroll
        for (int nb = 0; nb < NB; nb++) {
#pragma unroll
            for (int e = 0; e < 4; e++) {
                const int row = (e < 2) ? r0 : r1;
                const bool rv = (e < 2) ? v0 : v1;
                const int b = nb * 8 + 2 * t + (e & 1);
                if (rv && b < P.B) {
                    if (ACC_OUT)
                        static_cast<int32_t *>(D.out)[(size_t)b * N + row] = acc[nb][e];
                    else
                        static_cast<float *>(D.out)[(size_t)b * N + row] =
                            out_scale(D, row, b) * (float)acc[nb][e];
                }
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Pipelined kernel (K % 512 == 0, codes 16-byte aligned).
//
//   * work item = (32-row unit, K-part of at most kMaxPartChunks chunks = 8192
//     weights per row); thread (g, t) decodes rows g, g+8, g+16, g+24 of the
//     unit for tile 4c + t of chunk c, so the activation fragments it loads
//     feed 32 MMAs;
//   * a chunk of a unit (32 rows x 4 tiles) is one contiguous 2560-byte block
//     of the code layout; each warp streams its items' chunks through a
//     private ring of kRing shared-memory stages filled by cp.async with
//     consecutive lanes on consecutive 16 bytes, so an SM (one CTA of 16
//     warps) keeps ~80 KB of fully coalesced HBM reads in flight;
//   * each CTA takes a run of whole items (in GEMV order) of about 1/gridDim
//     of the chunks, its ends rounded to the nearer item boundary, and its
//     warps split the run into equal chunk ranges; an
//     item cut by a warp boundary is summed in shared memory by the warp that
//     holds its first chunk, after one CTA barrier;
//   * a unit with several K-parts adds its partial int32 sums into part_acc
//     with atomics; the warp that completes the last part (per-unit counter)
//     scales, writes y and clears its part_acc entries and the counter, so
//     the workspace is ready for the next launch.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
                 "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}


// Chunk space: the 4-tile chunks of all groups, group by group, each group's
// 32-row units in order and each unit's chunks in K order.  An item (unit,
// K-part kp) holds chunks kp*cpp .. min(nchunk, kp*cpp + cpp) - 1 of its unit.
__device__ __forceinline__ int desc_by_chunk(const GemvParams &P, int c) {
    int lo = 0, hi = P.count - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (P.d[mid].chunk_begin <= c) lo = mid; else hi = mid - 1;
    }
    return lo;
}


// (GEMV, unit, K-part) of an item, advanced item by item without searches or
// divisions.
struct ItemCursor {
    int id, unit, kp;
};
// The item holding chunk c (c < total_chunks), and the chunk it starts at.
__device__ __forceinline__ ItemCursor cursor_at_chunk(const GemvParams &P, int c, int &start) {
    ItemCursor r;
    r.id = desc_by_chunk(P, c);
    const GemvDesc &D = P.d[r.id];
    const int rc = c - D.chunk_begin;
    r.unit = rc / D.nchunk;
    r.kp = (rc - r.unit * D.nchunk) / D.cpp;
    start = D.chunk_begin + r.unit * D.nchunk + r.kp * D.cpp;
    return r;
}
// The item boundary nearest to chunk c (c <= total_chunks): the start of the
// item holding c, or the start of the next one if that is nearer.  Monotone in
// c, so consecutive CTAs get valid ranges; rounding to the nearer end keeps a
// CTA's range within half an item of its share.
__device__ __forceinline__ int item_boundary_near(const GemvParams &P, int c) {
    if (c >= P.total_chunks) return P.total_chunks;
    int start;
    const ItemCursor r = cursor_at_chunk(P, c, start);
    const GemvDesc &D = P.d[r.id];
    const int end = start + min(D.cpp, D.nchunk - r.kp * D.cpp);
    return (c - start <= end - c) ? start : end;
}
__device__ __forceinline__ void cursor_next(const GemvParams &P, ItemCursor &c) {
    if (++c.kp == P.d[c.id].kparts) {
        c.kp = 0;
        if (++c.unit == P.d[c.id].units) {
            c.unit = 0;
            ++c.id;
        }
    }
}

// A stage's copies read ordinary device memory and always complete; the bound
// only keeps a warp from spinning for good after a fault elsewhere.
constexpr long long kStageWaitLimit = 4000000000LL;

// First error recorded by a GEMV kernel (see sherry_device_error).
__device__ unsigned int g_gemv_device_error = 0;

// Bounded wait of all lanes on a stage's mbarrier phase; false (on every lane)
// if it did not complete within kStageWaitLimit cycles on some lane.
__device__ __forceinline__ bool stage_wait(uint64_t *bar, uint32_t parity) {
    bool ok = mbar_try_wait(bar, parity);
    if (!ok) {
        const long long t0 = clock64();
        while (!(ok = mbar_try_wait(bar, parity)))
            if (clock64() - t0 > kStageWaitLimit) break;
    }
    return __all_sync(0xFFFFFFFFu, ok);
}

#ifndef SHERRY_PIPE_MIN_BLOCKS
#define SHERRY_PIPE_MIN_BLOCKS 1
#endif
// Shared memory of the MMA kernel: the warps' rings, then per warp the
// fragments of a later piece of a cut item [warp][2 * NB * 4][32] (the
// chunk split and the cut items are those of the small-batch kernel below).
// One CTA of 16 warps per SM (142 KB at NB = 1, 158 KB at NB = 2): measured on
// the 16-layer 3B stack against two CTAs of 8 warps, 96.0 -> 90.9 us at B = 4
// and 128.7 -> 125.7 us at B = 16.
template <int NB>
struct PipeShape {
    static constexpr int kCutWords = 2 * NB * 4 * 32;
    static constexpr size_t kSmem = kPipeSmem + (size_t)kPipeWarps * kCutWords * 4;
};

// Finishes an item of the MMA kernel: per row block rb, fragment e holds
// (row g + 8 [e >= 2], batch column 2t + (e & 1)) of the unit.
template <int NB, bool ACC_OUT>
__device__ __forceinline__ void pipe_finish(const GemvDesc &D, int unit, int B, int lane,
                                            int (&acc)[2][NB][4]) {
    const int g = lane >> 2, t = lane & 3;
    const int N = D.N;
    const int rbase = unit * kUnitRows;
    bool finish = true;
    if (D.kparts > 1) {
#pragma unroll
        for (int rb = 0; rb < 2; rb++)
#pragma unroll
            for (int nb = 0; nb < NB; nb++)
#pragma unroll
                for (int e = 0; e < 4; e++) {
                    const int row = rbase + rb * 16 + g + ((e & 2) ? 8 : 0);
                    const int b = nb * 8 + 2 * t + (e & 1);
                    if (row < N && b < B) atomicAdd(D.part_acc + (size_t)b * N + row, acc[rb][nb][e]);
                }
        __threadfence();
        __syncwarp();
        uint32_t done = 0;
        if (lane == 0) done = atomicAdd(D.part_cnt + unit, 1u);
        finish = __shfl_sync(0xFFFFFFFFu, done, 0) == (uint32_t)(D.kparts - 1);
        if (finish) {
            __threadfence();
#pragma unroll
            for (int rb = 0; rb < 2; rb++)
#pragma unroll
                for (int nb = 0; nb < NB; nb++)
#pragma unroll
                    for (int e = 0; e < 4; e++) {
                        const int row = rbase + rb * 16 + g + ((e & 2) ? 8 : 0);
                        const int b = nb * 8 + 2 * t + (e & 1);
                        if (row < N && b < B) {
                            int32_t *pa = D.part_acc + (size_t)b * N + row;
                            acc[rb][nb][e] = __ldcg(pa);
                            *pa = 0;
                        }
                    }
            if (lane == 0) D.part_cnt[unit] = 0u;
        }
    }
    if (finish) {
#pragma unroll
        for (int rb = 0; rb < 2; rb++)
#pragma unroll
            for (int nb = 0; nb < NB; nb++)
#pragma unroll
                for (int e = 0; e < 4; e++) {
                    const int row = rbase + rb * 16 + g + ((e & 2) ? 8 : 0);
                    const int b = nb * 8 + 2 * t + (e & 1);
                    if (row < N && b < B) {
                        if (ACC_OUT)
                            static_cast<int32_t *>(D.out)[(size_t)b * N + row] = acc[rb][nb][e];
                        else
                            static_cast<float *>(D.out)[(size_t)b * N + row] =
                                out_scale(D, row, b) * (float)acc[rb][nb][e];
                    }
                }
    }
}

// XR: rows per activation group of the fragment-order layout, xgroup_rows(B)
// (a template parameter so that every fragment load has a constant offset).
template <int NB, bool ACC_OUT, int XR>
__global__ void __launch_bounds__(kPipeThreads, SHERRY_PIPE_MIN_BLOCKS)
    gemv_pipe_kernel(const __grid_constant__ GemvParams P) {
    pdl_allow_dependents();
    extern __shared__ __align__(16) uint32_t pipe_smem[];
    int *cut_sum = reinterpret_cast<int *>(pipe_smem + kPipeSmem / 4);
    __shared__ int cut_start[kPipeWarps];
    __shared__ int cta_bound[2];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    // chunk range [b0, b1) of this warp: the CTA takes whole items of about
    // 1/gridDim of the chunks, its warps equal chunk shares of them
    if (threadIdx.x < 2) {
        const long long tc = P.total_chunks, nb = gridDim.x;
        cta_bound[threadIdx.x] = item_boundary_near(P, (int)((blockIdx.x + threadIdx.x) * tc / nb));
    }
    __syncthreads();
    const int cta_lo = cta_bound[0];
    const long long len = cta_bound[1] - cta_lo;
    const int b0 = cta_lo + (int)(warp * len / kPipeWarps);
    const int b1 = cta_lo + (int)((warp + 1) * len / kPipeWarps);
    // -1: no cut item starts before b0; -2: empty range (skipped when summing)
    if (lane == 0) cut_start[warp] = b0 < b1 ? -1 : -2;
    uint32_t *ring = pipe_smem + (size_t)warp * kRing * kStageWords;
    Consts C;
    load_consts(P, C);
    const int B = P.B;
    constexpr int xstride = 4 * XR;     // uint4 between a tile's uint4 j and j + 1

    int start = b1;
    ItemCursor cur = {0, 0, 0};
    if (b0 < b1) cur = cursor_at_chunk(P, b0, start);

    // ---- producer side: the issue cursor runs kRing-1 stages ahead ----
    // lane l copies 16-byte pieces l + 32 j (j = 0..4) of the 2560-byte chunk;
    // piece words 4i..4i+3 belong to tile block 4i / 160.  Codes only (and
    // only when P.prefetch_codes allows it before pdl_wait()): the activations
    // are read from global memory after pdl_wait().
    ItemCursor icur = cur;
    int istart = start, ic = 0, ic_end = 0;
    const uint32_t *isrc = nullptr;  // first word of the current unit's group
    auto set_issue_item = [&]() {
        const GemvDesc &D = P.d[icur.id];
        isrc = D.codes + (size_t)icur.unit * D.T * kTileWords + 4 * lane;
        const int first = icur.kp * D.cpp;
        ic = first + max(b0 - istart, 0);
        ic_end = first + min(b1 - istart, min(D.cpp, D.nchunk - first));
    };
    if (istart < b1) set_issue_item();
    uint32_t dst_piece[5];
#pragma unroll
    for (int j = 0; j < 5; j++) {
        const int wd = 4 * (lane + 32 * j);
        const int tb = wd / kTileWords;
        dst_piece[j] = smem_u32(ring) + 4u * (uint32_t)(tb * kTileWordsPadded + (wd - tb * kTileWords));
    }
    auto issue = [&](int slot) {
        if (istart < b1) {
            const uint32_t *src = isrc + (size_t)ic * kChunkTiles * kTileWords;
            const uint32_t sofs = (uint32_t)slot * kStageWords * 4;
#pragma unroll
            for (int j = 0; j < 5; j++) cp_async16(dst_piece[j] + sofs, src + 128 * j, 16u);
            if (++ic == ic_end) {
                const GemvDesc &D = P.d[icur.id];
                istart += min(D.cpp, D.nchunk - icur.kp * D.cpp);
                if (istart < b1) {
                    cursor_next(P, icur);
                    set_issue_item();
                }
            }
        }
        cp_async_commit();
    };
    if (!P.prefetch_codes) pdl_wait();
#pragma unroll
    for (int s = 0; s < kRing - 1; s++) issue(s);
    if (P.prefetch_codes) pdl_wait();

    // ---- consumer side ----
    int slot = 0;
    int acc[2][NB][4];  // [row block][batch group][fragment]
    bool own_cut = false;  // the last item continues in later warps of the CTA
    while (start < b1) {
        const GemvDesc &D = P.d[cur.id];
        const int first = cur.kp * D.cpp;
        const int nreal = min(D.cpp, D.nchunk - first);
        const int c_begin = first + max(b0 - start, 0);
        const int c_end = first + min(b1 - start, nreal);
        // lane (g, t) reads row g of each group (rows past the batch are padding
        // whose columns are never stored; with 4-row groups lanes g >= 4 re-read
        // rows g - 4), tile t of the chunk: chunk c at xstride * 8 uint4, uint4 j
        // of the tile at xstride * j
        const uint4 *xrow[NB];
#pragma unroll
        for (int nb = 0; nb < NB; nb++)
            xrow[nb] = D.xw + xw_word(XR, D.Tp, nb * XR + (g & (XR - 1)), t, 0) / 4;
#pragma unroll
        for (int a = 0; a < 2; a++)
#pragma unroll
            for (int nb = 0; nb < NB; nb++) acc[a][nb][0] = acc[a][nb][1] = acc[a][nb][2] = acc[a][nb][3] = 0;
        for (int c = c_begin; c < c_end; c++) {
            cp_async_wait<kRing - 2>();
            __syncwarp();
            // tile t of the chunk, plane p, row g + 8 r: word t * 168 + 32 p + g + 8 r
            const uint32_t *st = ring + slot * kStageWords + t * kTileWordsPadded + g;
            // padded tiles hold zero activations, so no load is predicated
            const size_t xoff = (size_t)c * 8 * xstride;
            // the four rows of this lane (g, g + 8 of row block 0, g + 16, g + 24 of row
            // block 1) are decoded together, so each activation fragment is loaded once
            // for both row blocks, and the next position's fragments are loaded while
            // the current position's MMAs run
            TileDecoder6 d[4];
#pragma unroll
            for (int r = 0; r < 4; r++)
                d[r].load(C, st[0 * 32 + 8 * r], st[1 * 32 + 8 * r], st[2 * 32 + 8 * r],
                          st[3 * 32 + 8 * r], st[4 * 32 + 8 * r]);
            __syncwarp();  // every lane has its words: the stage can be refilled
            issue(slot == 0 ? kRing - 1 : slot - 1);
            slot = (slot + 1 == kRing) ? 0 : slot + 1;
            uint4 xq[NB][2], xn[NB][2];
#pragma unroll
            for (int nb = 0; nb < NB; nb++) {
                xq[nb][0] = ld_x(xrow[nb] + xoff);
                xq[nb][1] = ld_x(xrow[nb] + xoff + xstride);
            }
#pragma unroll
            for (int i = 0; i < 4; i++) {
                if (i < 3) {
#pragma unroll
                    for (int nb = 0; nb < NB; nb++) {
                        xn[nb][0] = ld_x(xrow[nb] + xoff + (2 * i + 2) * xstride);
                        xn[nb][1] = ld_x(xrow[nb] + xoff + (2 * i + 3) * xstride);
                    }
                }
                const uint32_t tlo = C.tlo[i], thi = C.thi[i];
#pragma unroll
                for (int beta = 0; beta < 4; beta++) {
                    const int m = 4 * i + beta;  // MMA index: activation words 2m, 2m+1
#pragma unroll
                    for (int rb = 0; rb < 2; rb++) {  // row block rb: rows g + 16 rb, g + 8 + 16 rb
                        const uint32_t s0 = d[2 * rb].sel(C, i, beta);
                        const uint32_t s1 = d[2 * rb + 1].sel(C, i, beta);
                        const uint32_t a0 = prmt(tlo, thi, s0);
                        const uint32_t a2 = prmt(tlo, thi, hi_half(C, s0));
                        const uint32_t a1 = prmt(tlo, thi, s1);
                        const uint32_t a3 = prmt(tlo, thi, hi_half(C, s1));
#pragma unroll
                        for (int nb = 0; nb < NB; nb++) {
                            const uint4 &xx = xq[nb][(m >> 1) & 1];
                            mma_s8(acc[rb][nb], a0, a1, a2, a3, pick(xx, (m & 1) * 2),
                                   pick(xx, (m & 1) * 2 + 1));
                        }
                    }
                }
                if (i < 3) {
#pragma unroll
                    for (int nb = 0; nb < NB; nb++) {
                        xq[nb][0] = xn[nb][0];
                        xq[nb][1] = xn[nb][1];
                    }
                }
            }
        }
        if (start < b0) {
            // a later piece of an item cut at b0: hand the fragments to its first warp
            int *cs = cut_sum + warp * PipeShape<NB>::kCutWords + lane;
#pragma unroll
            for (int rb = 0; rb < 2; rb++)
#pragma unroll
                for (int nb = 0; nb < NB; nb++)
#pragma unroll
                    for (int e = 0; e < 4; e++) cs[((rb * NB + nb) * 4 + e) * 32] = acc[rb][nb][e];
            if (lane == 0) cut_start[warp] = start;
        } else if (b1 - start < nreal) {
            own_cut = true;  // first piece of an item cut at b1: finished after the barrier
        } else {
            pipe_finish<NB, ACC_OUT>(D, cur.unit, B, lane, acc);
        }
        start += nreal;
        if (start < b1) cursor_next(P, cur);
    }
    cp_async_wait<0>();
    __syncthreads();  // the later pieces' fragments are in shared memory
    if (own_cut) {
        const GemvDesc &D = P.d[cur.id];
        const int mine = D.chunk_begin + cur.unit * D.nchunk + cur.kp * D.cpp;  // the cut item
        for (int w = warp + 1; w < kPipeWarps; w++) {
            const int cs = cut_start[w];
            if (cs == -2) continue;
            if (cs != mine) break;
            const int *src = cut_sum + w * PipeShape<NB>::kCutWords + lane;
#pragma unroll
            for (int rb = 0; rb < 2; rb++)
#pragma unroll
                for (int nb = 0; nb < NB; nb++)
#pragma unroll
                    for (int e = 0; e < 4; e++) acc[rb][nb][e] += src[((rb * NB + nb) * 4 + e) * 32];
        }
        pipe_finish<NB, ACC_OUT>(D, cur.unit, B, lane, acc);
    }
}

// ---------------------------------------------------------------------------
// Small-batch kernel (B <= 2): dot products on the ALU/FMA pipes, no MMA.
//   * an item is (unit group, K-part), a unit group being NU (1 or 2)
//     consecutive 32-row units.  Lane l owns row l of each unit of the group,
//     so a tile's five words of one unit are five conflict-free shared loads,
//     each lane ends with its rows' sums (no reduction across lanes), and the
//     activation words of a tile, read once per warp (broadcast loads), feed
//     NU rows per lane;
//   * work is split by chunk count, a chunk being 4 tiles of every unit of a
//     group.  Each CTA takes a run of whole items holding about 1/gridDim of
//     the chunks (its ends rounded to the nearer item boundary) and its warps
//     split the run into equal chunk ranges, so no
//     warp ends the launch with a whole extra item to do.  An item cut by a
//     warp boundary is summed by the warps holding its pieces: later pieces
//     leave their row sums in shared memory, and after one CTA barrier the
//     warp holding the item's first chunk adds them and finishes the item;
//   * each warp streams its chunks through a private 2-stage ring in shared
//     memory.  One lane fills a stage with bulk copies (cp.async.bulk): one
//     per unit of the group (a unit's chunk is a contiguous 2,560 bytes of the
//     code layout) and one per batch row for the chunk's activations, all
//     completing on the stage's mbarrier.  The next chunk is requested before
//     the current one is waited for, so a warp has two chunks in flight;
//   * each decoded word (four ternary bytes) meets its activation word in one
//     dp4a: for B <= 2 this is cheaper than an m16n8k32 MMA whose 8 columns
//     would mostly be empty.
// K-parts and the split-K completion are those of the pipelined kernel, with
// one counter per unit group.
// ---------------------------------------------------------------------------
// 32-row units per item of the dot kernel: 2 for calls of more than
// kDotPairMinChunksPerSM 32-row chunks per SM (the broadcast activation loads
// and the in-kernel re-order are shared by two rows per lane), else 1 (twice
// the items, so a small call spreads over twice the SMs).  Measured on the
// 16-layer 1B stack with in-kernel re-order: 54.5 us per step with 2, 58.9
// with 1; a 2048 x 8192 GEMV: 7.3 us with 1, 9.1 with 2.
constexpr int kDotMaxUnits = 2;
constexpr int kDotPairMinChunksPerSM = 64;
// Stages per warp.  Measured on the 1B stack with two-unit items: 16 warps x
// 2 stages of 4-tile chunks 52.5 us; deeper rings with fewer warps (the same
// shared memory) 54.5 us (12 x 3) and 62.3 us (8 x 4); 16 warps x 4 stages
// of 2-tile chunks 58.8 us.
constexpr int kDotRing = 2;
// bf16 calls up to this many 32-row chunks per SM quantize and re-order x in
// the dot kernel (each warp takes the token's absmax from the row itself, so
// large calls keep the front-end launch); int8 calls of any size re-order x
// in the kernel (measured on the 16-layer 1B stack: 54.5 us per step against
// 56.6 us with the re-order launch).
constexpr int kRawBfMaxChunksPerSM = 64;
// Weight formats the small-batch kernel streams: Sherry, and the two ternary
// packings the pages compare it against (arXiv 2601.07892, abstract; Figure 2
// caption): 2 bits per weight, aligned ("I2"), and three weights in five bits
// ("T3").  Per format: 32-bit words per tile of one row (a tile is 128
// weights, or 96 for T3) and tiles per chunk.  Every format's chunk carries
// 32 activation words per tile and batch row.
enum DotFormat { kFmtSherry = 0, kFmtI2 = 1, kFmtT3 = 2 };
template <int FMT>
struct FmtTraits {
    static constexpr int kTileWords = FMT == kFmtI2 ? 8 : 5;
    static constexpr int kChunkTiles = FMT == kFmtT3 ? 2 : 4;
    static constexpr int kUnitChunkWords = kChunkTiles * kTileWords * kUnitRows;
};

// Shared memory of a CTA of the small-batch kernel with `warps` warps: the
// rings, the stages' mbarriers, the cut-item sums and starts.
constexpr size_t dot_smem_bytes(int warps, int ring, int stage_words, int cut_words) {
    return (size_t)warps * ((size_t)ring * stage_words * 4 + ring * 8 + (size_t)cut_words * 4 + 4);
}

// 8 or 16 warps per CTA (see kWarps).  B = 1 with two units per item: one CTA
// of 16 warps per SM, 180 KB of shared memory, up to 128 registers per thread.
// XMODE 2 adds to each stage the chunk's raw bf16 activations (1 KB per batch row).
template <int NBX, int XMODE = 0, int FMT = kFmtSherry, int NU_ = kDotMaxUnits>
struct DotShape {
    static constexpr int NU = NU_;
    static constexpr int kChunkTilesF = FmtTraits<FMT>::kChunkTiles;
    static constexpr int kCodeWords = NU * FmtTraits<FMT>::kUnitChunkWords;
    static constexpr int kXWords = NBX * kChunkTilesF * 32;                     // int8, decode order
    static constexpr int kBfWords = XMODE == 2 ? NBX * kChunkTilesF * 64 : 0;   // raw bf16
    static constexpr int kStageWords = kCodeWords + kXWords + kBfWords;
    static constexpr int kCutWords = NU * NBX * 32;
    // Two-unit items (large calls) run one CTA of 16 warps per SM where its
    // rings fit: a CTA's chunk range is rounded to whole items once per SM
    // instead of once per half, which halves the spread of work between SMs
    // (items of 16 chunks against ~200 chunks per SM on the 1B stack).
    static constexpr int kRing = kDotRing;  // stages per warp
    static constexpr bool kPair =
        NU == 2 && dot_smem_bytes(16, kRing, kStageWords, kCutWords) + 1024 <= 227u * 1024u;
    static constexpr int kWarps = kPair ? 16 : 8;
    static constexpr int kThreads = kWarps * 32;
    static constexpr int kRingWords = kWarps * kRing * kStageWords;
    // after the rings: the stages' mbarriers [warp][stage], then per warp the
    // row sums of a later piece of a cut item [NU][NBX][32] and that item's
    // first chunk
    static constexpr size_t kBarOffset = (size_t)kRingWords * 4;
    static constexpr size_t kCutOffset = kBarOffset + (size_t)kWarps * kRing * 8;
    static constexpr size_t kSmem = kCutOffset + ((size_t)kWarps * kCutWords + kWarps) * 4;
    // CTAs per SM that fit the 227 KB of shared memory (1 KB reserved per CTA)
    static constexpr int kFit = (int)((227u * 1024u) / (kSmem + 1024u));
    static constexpr int kMinBlocks = kFit < 1 ? 1 : (kFit > 4 ? 4 : kFit);
    static_assert(kStageWords % 4 == 0, "stages must stay 16-byte aligned for bulk copies");
};

// Finishes an item: lane = row of each unit of the group, v = the item's row
// sums.  A K-part of a split row adds into the K-part sums; the last K-part to
// finish scales, stores and clears them.
// sx: the activation scales, when the kernel quantized the activations itself.
template <int NBX, int NU, bool ACC_OUT, bool SX_REG>
__device__ __forceinline__ void dot_finish(const GemvDesc &D, int group, int B, int lane,
                                           int (&v)[NU][NBX], const float (&sx)[NBX]) {
    const int N = D.N;
    bool finish = true;
    if (D.kparts > 1) {
#pragma unroll
        for (int u = 0; u < NU; u++) {
            const int row = (group * NU + u) * kUnitRows + lane;
            if (row < N) {
#pragma unroll
                for (int b = 0; b < NBX; b++)
                    if (b < B) atomicAdd(D.part_acc + (size_t)b * N + row, v[u][b]);
            }
        }
        __threadfence();
        __syncwarp();
        uint32_t done = 0;
        if (lane == 0) done = atomicAdd(D.part_cnt + group, 1u);
        finish = __shfl_sync(0xFFFFFFFFu, done, 0) == (uint32_t)(D.kparts - 1);
        if (finish) {
            __threadfence();
#pragma unroll
            for (int u = 0; u < NU; u++) {
                const int row = (group * NU + u) * kUnitRows + lane;
                if (row < N) {
#pragma unroll
                    for (int b = 0; b < NBX; b++) {
                        if (b < B) {
                            int32_t *pa = D.part_acc + (size_t)b * N + row;
                            v[u][b] = __ldcg(pa);
                            *pa = 0;
                        }
                    }
                }
            }
            if (lane == 0) D.part_cnt[group] = 0u;
        }
    }
    if (!finish) return;
#pragma unroll
    for (int u = 0; u < NU; u++) {
        const int row = (group * NU + u) * kUnitRows + lane;
        if (row >= N) continue;
#pragma unroll
        for (int b = 0; b < NBX; b++) {
            if (b >= B) continue;
            if (ACC_OUT) {
                static_cast<int32_t *>(D.out)[(size_t)b * N + row] = v[u][b];
            } else {
                const float sc = SX_REG ? __fmul_rn(__ldg(D.scales + row), sx[b]) : out_scale(D, row, b);
                static_cast<float *>(D.out)[(size_t)b * N + row] = sc * (float)v[u][b];
            }
        }
    }
}

// One chunk of the 2-bit format: 4 tiles x 8 words per unit.  Word q of a
// tile holds weights 16 q + n (low two bits of nibble n) and 16 q + 8 + n
// (high two bits); code 1 is +1, 3 is -1, 0 and 2 are 0.  Masking the low (or,
// after a shift, the high) two bits of every nibble gives a PRMT selector
// whose halves decode four consecutive weights each, so the activations stay
// in natural order: x word 4 q + r of the tile meets decoded word r.
template <int NBX, int NU>
__device__ __forceinline__ void dot_chunk_i2(const uint32_t *st, int code_words, int lane,
                                             const Consts &C, int (&acc)[NU][NBX][2]) {
    // table: byte c = weight of code c (0, +1, 0, -1)
    const uint32_t tab = 0xFF000100u;
#pragma unroll
    for (int tt = 0; tt < 4; tt++) {
        const uint4 *xs = reinterpret_cast<const uint4 *>(st + code_words + tt * 32);
#pragma unroll
        for (int q = 0; q < 8; q++) {
            uint4 xv[NBX];
#pragma unroll
            for (int b = 0; b < NBX; b++) xv[b] = xs[b * 32 + q];
#pragma unroll
            for (int u = 0; u < NU; u++) {
                const uint32_t w = st[u * FmtTraits<kFmtI2>::kUnitChunkWords + tt * 256 + q * 32 + lane];
                const uint32_t s0 = w & C.m33, s1 = (w >> 2) & C.m33;
                const int d0 = (int)prmt(tab, 0u, s0), d1 = (int)prmt(tab, 0u, hi_half(C, s0));
                const int d2 = (int)prmt(tab, 0u, s1), d3 = (int)prmt(tab, 0u, hi_half(C, s1));
#pragma unroll
                for (int b = 0; b < NBX; b++) {
                    acc[u][b][0] = __dp4a(d0, (int)xv[b].x, acc[u][b][0]);
                    acc[u][b][1] = __dp4a(d1, (int)xv[b].y, acc[u][b][1]);
                    acc[u][b][0] = __dp4a(d2, (int)xv[b].z, acc[u][b][0]);
                    acc[u][b][1] = __dp4a(d3, (int)xv[b].w, acc[u][b][1]);
                }
            }
        }
    }
}

// Field j (bits 5 j .. 5 j + 4) of a T3 tile's 160-bit string, times 4 (its
// table entry's byte offset).  j is a constant after unrolling, so only one
// branch remains: one shift (or funnel shift, for the fields that straddle
// two words) and one mask.
__device__ __forceinline__ uint32_t t3_field_x4(const uint32_t (&w)[5], int j) {
    const int b = 5 * j, wi = b >> 5, sh = b & 31;
    if (sh >= 2 && sh <= 27) return (w[wi] >> (sh - 2)) & 0x7Cu;
    if (sh < 2) return (w[wi] << (2 - sh)) & 0x7Cu;
    return __funnelshift_r(w[wi], w[wi + 1], sh - 2) & 0x7Cu;
}

// One chunk of the three-in-five format: 2 tiles x 5 words per unit; triple
// j's code indexes a 32-entry table of packed ternary bytes in shared memory
// (lane = row, so a lookup of 32 rows is one conflict-free access), and the
// entry meets activation word j = (x[3j], x[3j+1], x[3j+2], 0) in one dp4a.
template <int NBX, int NU>
__device__ __forceinline__ void dot_chunk_t3(const uint32_t *st, int code_words, int lane,
                                             const uint32_t *lut, int (&acc)[NU][NBX][2]) {
    const uint8_t *lut_b = reinterpret_cast<const uint8_t *>(lut);
#pragma unroll
    for (int tt = 0; tt < 2; tt++) {
        uint32_t w[NU][5];
#pragma unroll
        for (int u = 0; u < NU; u++)
#pragma unroll
            for (int p = 0; p < 5; p++)
                w[u][p] = st[u * FmtTraits<kFmtT3>::kUnitChunkWords + tt * 160 + p * 32 + lane];
        const uint4 *xs = reinterpret_cast<const uint4 *>(st + code_words + tt * 32);
#pragma unroll
        for (int q = 0; q < 8; q++) {
            uint4 xv[NBX];
#pragma unroll
            for (int b = 0; b < NBX; b++) xv[b] = xs[b * 16 + q];  // 64 words per batch row
#pragma unroll
            for (int u = 0; u < NU; u++) {
                int e[4];
                e[0] = *reinterpret_cast<const int *>(lut_b + t3_field_x4(w[u], 4 * q + 0));
                e[1] = *reinterpret_cast<const int *>(lut_b + t3_field_x4(w[u], 4 * q + 1));
                e[2] = *reinterpret_cast<const int *>(lut_b + t3_field_x4(w[u], 4 * q + 2));
                e[3] = *reinterpret_cast<const int *>(lut_b + t3_field_x4(w[u], 4 * q + 3));
#pragma unroll
                for (int b = 0; b < NBX; b++) {
                    acc[u][b][0] = __dp4a(e[0], (int)xv[b].x, acc[u][b][0]);
                    acc[u][b][1] = __dp4a(e[1], (int)xv[b].y, acc[u][b][1]);
                    acc[u][b][0] = __dp4a(e[2], (int)xv[b].z, acc[u][b][0]);
                    acc[u][b][1] = __dp4a(e[3], (int)xv[b].w, acc[u][b][1]);
                }
            }
        }
    }
}

// XMODE: where the activations come from.
//   0  re-ordered words in the workspace (written by the re-order launch);
//   1  raw int8 from D.x (16-byte aligned rows): each warp re-orders its
//      chunk's 4 tiles in shared memory (four shuffles and three byte permutes
//      per word, as the re-order launch does);
//   2  raw bf16 from D.xbf: each warp takes the token's absmax from the row
//      (once per activation pointer), then quantizes and re-orders its chunk's
//      tiles by the rule of the bf16 front-end.
// Modes 1 and 2 need no re-order launch.  They are used for calls of few
// chunks, where that launch and its wait cost more than the per-chunk work.
// FMT: the weight format (Sherry, or a comparison format with XMODE 0).
template <int NBX, bool ACC_OUT, int XMODE, int FMT = kFmtSherry, int NU_ = kDotMaxUnits>
__global__ void __launch_bounds__(DotShape<NBX, XMODE, FMT, NU_>::kThreads,
                                  DotShape<NBX, XMODE, FMT, NU_>::kMinBlocks)
    gemv_dot_kernel(const __grid_constant__ GemvParams P) {
    constexpr bool XRAW = XMODE == 1;
    constexpr bool XBF = XMODE == 2;
    static_assert(FMT == kFmtSherry || XMODE == 0, "comparison formats read prepared activations");
    using Shape = DotShape<NBX, XMODE, FMT, NU_>;
    using F = FmtTraits<FMT>;
    constexpr int CT = F::kChunkTiles;
    constexpr int UCW = F::kUnitChunkWords;
    constexpr int NU = Shape::NU;
    constexpr int SW = Shape::kStageWords;
    constexpr int kWarps = Shape::kWarps;
    pdl_allow_dependents();
    extern __shared__ __align__(128) uint32_t dot_smem[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint8_t *smem_bytes = reinterpret_cast<uint8_t *>(dot_smem);
    constexpr int RING = Shape::kRing;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem_bytes + Shape::kBarOffset) + warp * RING;
    int *cut_sum = reinterpret_cast<int *>(smem_bytes + Shape::kCutOffset);
    int *cut_start = cut_sum + kWarps * Shape::kCutWords;
    // chunk range [b0, b1) of this warp; threads 0 and 1 find the CTA's bounds
    __shared__ int cta_bound[2];
    if (threadIdx.x < 2) {
        const long long tc = P.total_chunks, nb = gridDim.x;
        cta_bound[threadIdx.x] = item_boundary_near(P, (int)((blockIdx.x + threadIdx.x) * tc / nb));
    }
    if (lane == 0) {
#pragma unroll
        for (int s = 0; s < RING; s++) mbar_init(&bars[s], 1);
        fence_mbar_init();
    }
    // T3: entry c of the table = the triple of code c as three ternary bytes
    // (byte 3 zero), codes past 26 zero
    __shared__ uint32_t t3_lut[32];
    if (FMT == kFmtT3 && threadIdx.x < 32) {
        const int c = (int)threadIdx.x;
        t3_lut[c] = c > 26 ? 0u
                           : ((uint32_t)(c % 3 - 1) & 0xFFu) | (((uint32_t)((c / 3) % 3 - 1) & 0xFFu) << 8) |
                                 (((uint32_t)(c / 9 - 1) & 0xFFu) << 16);
    }
    __syncthreads();
    const int cta_lo = cta_bound[0], cta_hi = cta_bound[1];
    const long long len = cta_hi - cta_lo;
    const int b0 = cta_lo + (int)(warp * len / kWarps);
    const int b1 = cta_lo + (int)((warp + 1) * len / kWarps);
    // -1: no cut item starts before b0; -2: empty range (skipped when summing)
    if (lane == 0) cut_start[warp] = b0 < b1 ? -1 : -2;
    uint32_t *ring = dot_smem + (size_t)warp * RING * SW;
    const uint32_t ring_addr = smem_u32(ring);
    Consts C;
    load_consts(P, C);
    const int B = P.B;

    // the warp's items: from the one holding chunk b0, while they start before b1
    int start = b1;
    ItemCursor cur = {0, 0, 0};
    if (b0 < b1) cur = cursor_at_chunk(P, b0, start);

    // ---- producer side: runs one chunk ahead of the consumer ----
    // Lane 0 arms the stage's mbarrier with the byte count and issues the bulk
    // copies; every lane advances the cursor.  Until pdl_wait() only codes are
    // read, and only when P.prefetch_codes says the kernel before is this
    // call's re-order launch: the activation words and the K-part sums belong
    // to that kernel.
    ItemCursor icur = cur;
    int istart = start, ic = 0, ic_end = 0;
    auto set_issue_item = [&]() {
        const GemvDesc &D = P.d[icur.id];
        const int first = icur.kp * D.cpp;
        ic = first + max(b0 - istart, 0);
        ic_end = first + min(b1 - istart, min(D.cpp, D.nchunk - first));
    };
    if (istart < b1) set_issue_item();
    // activation bytes per chunk and batch row: 32 words per tile (raw bf16: twice that)
    constexpr uint32_t kXBytes = XBF ? CT * 128 * 2 : CT * 128;
    auto issue_codes = [&](int slot) {
        const GemvDesc &D = P.d[icur.id];
        if (lane == 0) {
            const int unit0 = icur.unit * NU;
            const int present = min(NU, D.units32 - unit0);
            const uint32_t dst = ring_addr + (uint32_t)slot * SW * 4;
            fence_proxy_async_smem();  // the warp's reads of the stage's previous chunk come first
            mbar_arrive_expect_tx(&bars[slot], (uint32_t)present * UCW * 4 + (uint32_t)B * kXBytes);
            const uint32_t *src =
                D.codes + ((size_t)unit0 * D.T + (size_t)ic * CT) * (F::kTileWords * kUnitRows);
#pragma unroll
            for (int u = 0; u < NU; u++)
                if (u < present)
                    bulk_load(dst + (uint32_t)u * UCW * 4,
                              src + (size_t)u * D.T * (F::kTileWords * kUnitRows), UCW * 4, &bars[slot]);
        }
    };
    auto issue_x_and_advance = [&](int slot) {
        const GemvDesc &D = P.d[icur.id];
        if (lane == 0) {
            const uint32_t dst = ring_addr + (uint32_t)slot * SW * 4 + (uint32_t)Shape::kCodeWords * 4;
#pragma unroll
            for (int b = 0; b < NBX; b++) {
                if (b < B) {
                    if (XBF)
                        bulk_load(dst + (uint32_t)Shape::kXWords * 4 + (uint32_t)b * kXBytes,
                                  D.xbf + ((size_t)b * D.T + (size_t)ic * CT) * SHERRY_TILE_K,
                                  kXBytes, &bars[slot]);
                    else if (XRAW)
                        bulk_load(dst + (uint32_t)b * kXBytes,
                                  D.x + ((size_t)b * D.T + (size_t)ic * CT) * SHERRY_TILE_K,
                                  kXBytes, &bars[slot]);
                    else  // 32 words (8 uint4) per tile
                        bulk_load(dst + (uint32_t)b * kXBytes,
                                  D.xw + ((size_t)b * D.Tp + (size_t)ic * CT) * 8, kXBytes,
                                  &bars[slot]);
                }
            }
        }
        if (++ic == ic_end) {
            istart += min(D.cpp, D.nchunk - icur.kp * D.cpp);
            if (istart < b1) {
                cursor_next(P, icur);
                set_issue_item();
            }
        }
    };
    uint32_t inflight = 0;  // stages whose copies were issued and not yet waited for
    auto issue = [&](int slot) {
        if (istart < b1) {
            issue_codes(slot);
            issue_x_and_advance(slot);
            inflight |= 1u << slot;
        }
    };
    const bool first_copy = istart < b1;
    if (first_copy && P.prefetch_codes) {
        issue_codes(0);
    } else if (first_copy && lane == 0) {
        // the kernel before may have written the codes: only warm L2 with the
        // first chunk's codes before the wait (L2 is where every write lands,
        // so the copy after the wait reads the final data from it)
        const GemvDesc &D = P.d[icur.id];
        const int unit0 = icur.unit * NU;
        const int present = min(NU, D.units32 - unit0);
        const uint32_t *src = D.codes + ((size_t)unit0 * D.T + (size_t)ic * CT) * (F::kTileWords * kUnitRows);
        for (int u = 0; u < present; u++)
            bulk_prefetch_l2(src + (size_t)u * D.T * (F::kTileWords * kUnitRows), UCW * 4);
    }
    pdl_wait();
    if (first_copy && !P.prefetch_codes) issue_codes(0);
    if (first_copy) {
        issue_x_and_advance(0);
        inflight = 1u;
    }
    // stages 1 .. RING - 2: later chunks in flight before the first is waited for
#pragma unroll
    for (int s = 1; s + 1 < RING; s++) issue(s);

    // ---- consumer side ----
    int slot = 0;
    uint32_t phase = 0;  // bit s: parity of stage s's next phase
    bool failed = false;
    int v[NU][NBX];
    bool own_cut = false;  // the last item continues in later warps of the CTA
    // XMODE 2: per-token quantization of the activations the warp works on
    const uint16_t *sx_of = nullptr;  // the activations (and row length) sx belongs to
    int sx_T = 0;
    float sx[NBX], sx_inv[NBX];
#pragma unroll
    for (int b = 0; b < NBX; b++) sx[b] = sx_inv[b] = 0.0f;
    while (start < b1) {
        const GemvDesc &D = P.d[cur.id];
        if (XBF && (D.xbf != sx_of || D.T != sx_T)) {  // after pdl_wait(): x may come from the kernel before
            sx_of = D.xbf;
            sx_T = D.T;
#pragma unroll
            for (int b = 0; b < NBX; b++) {
                if (b < B) {
                    const float amax = row_absmax_bf16(D.xbf + (size_t)b * D.T * SHERRY_TILE_K,
                                                       D.T * SHERRY_TILE_K, lane);
                    sx_inv[b] = amax > 0.0f ? __fdiv_rn(127.0f, amax) : 0.0f;
                    sx[b] = amax > 0.0f ? __fdiv_rn(amax, 127.0f) : 0.0f;
                }
            }
        }
        const int first = cur.kp * D.cpp;
        const int nreal = min(D.cpp, D.nchunk - first);
        const int c_begin = first + max(b0 - start, 0);
        const int c_end = first + min(b1 - start, nreal);
        int acc[NU][NBX][2];
#pragma unroll
        for (int u = 0; u < NU; u++)
#pragma unroll
            for (int b = 0; b < NBX; b++) acc[u][b][0] = acc[u][b][1] = 0;
        for (int c = c_begin; c < c_end; c++) {
            issue(slot == 0 ? RING - 1 : slot - 1);  // the stage the previous chunk used
            if (!stage_wait(&bars[slot], (phase >> slot) & 1u)) {
                failed = true;
                break;
            }
            inflight &= ~(1u << slot);
            phase ^= 1u << slot;
            uint32_t *st = ring + slot * SW;
            if (XRAW) {  // raw words of the chunk's tiles -> the decode order, in place
                uint32_t *xr = st + Shape::kCodeWords;
                uint32_t w[NBX][CT];
#pragma unroll
                for (int b = 0; b < NBX; b++)
#pragma unroll
                    for (int tt = 0; tt < CT; tt++)
                        w[b][tt] = b < B ? reorder_word(xr[(b * CT + tt) * 32 + lane], lane) : 0u;
                __syncwarp();
#pragma unroll
                for (int b = 0; b < NBX; b++)
#pragma unroll
                    for (int tt = 0; tt < CT; tt++)
                        if (b < B) xr[(b * CT + tt) * 32 + lane] = w[b][tt];
                __syncwarp();
            }
            if (XBF) {  // bf16 of the chunk's tiles -> quantized words in the decode order
                uint32_t *xq = st + Shape::kCodeWords;
                const uint2 *xb = reinterpret_cast<const uint2 *>(st + Shape::kCodeWords + Shape::kXWords);
#pragma unroll
                for (int b = 0; b < NBX; b++)
#pragma unroll
                    for (int tt = 0; tt < CT; tt++)
                        if (b < B)
                            xq[(b * CT + tt) * 32 + lane] =
                                reorder_word(quant_word(xb[(b * CT + tt) * 32 + lane], sx_inv[b]), lane);
                __syncwarp();
            }
            if (FMT == kFmtI2) {
                dot_chunk_i2<NBX, NU>(st, Shape::kCodeWords, lane, C, acc);
            } else if (FMT == kFmtT3) {
                dot_chunk_t3<NBX, NU>(st, Shape::kCodeWords, lane, t3_lut, acc);
            } else {
#pragma unroll
            for (int tt = 0; tt < CT; tt++) {
                TileDecoder6 d[NU];
#pragma unroll
                for (int u = 0; u < NU; u++) {
                    const uint32_t *cw = st + u * UCW + tt * kTileWords + lane;
                    d[u].load(C, cw[0], cw[32], cw[64], cw[96], cw[128]);
                }
                // activation words of tile tt: batch row b at b * 128, word q at q
                const uint4 *xs = reinterpret_cast<const uint4 *>(st + Shape::kCodeWords + tt * 32);
#pragma unroll
                for (int i = 0; i < 4; i++) {
                    uint4 xa[NBX], xb[NBX];  // words 8i..8i+3 (beta 0, 1) and 8i+4..8i+7 (beta 2, 3)
#pragma unroll
                    for (int b = 0; b < NBX; b++) {
                        xa[b] = xs[b * 32 + 2 * i];
                        xb[b] = xs[b * 32 + 2 * i + 1];
                    }
#pragma unroll
                    for (int beta = 0; beta < 4; beta++) {
#pragma unroll
                        for (int u = 0; u < NU; u++) {
                            const uint32_t sl = d[u].sel(C, i, beta);
                            const int lo = (int)prmt(C.tlo[i], C.thi[i], sl);
                            const int hi = (int)prmt(C.tlo[i], C.thi[i], hi_half(C, sl));
#pragma unroll
                            for (int b = 0; b < NBX; b++) {
                                const uint4 &xv = beta < 2 ? xa[b] : xb[b];
                                int &a = acc[u][b][beta & 1];
                                a = __dp4a(lo, (int)pick(xv, 2 * (beta & 1)), a);
                                a = __dp4a(hi, (int)pick(xv, 2 * (beta & 1) + 1), a);
                            }
                        }
                    }
                }
            }
            }
            __syncwarp();  // every lane is done with this stage before it is refilled
            slot = slot + 1 == RING ? 0 : slot + 1;
        }
        if (failed) break;
#pragma unroll
        for (int u = 0; u < NU; u++)
#pragma unroll
            for (int b = 0; b < NBX; b++) v[u][b] = acc[u][b][0] + acc[u][b][1];
        if (start < b0) {
            // a later piece of an item cut at b0: hand the sums to its first warp
#pragma unroll
            for (int u = 0; u < NU; u++)
#pragma unroll
                for (int b = 0; b < NBX; b++) cut_sum[((warp * NU + u) * NBX + b) * 32 + lane] = v[u][b];
            if (lane == 0) cut_start[warp] = start;
        } else if (b1 - start < nreal) {
            own_cut = true;  // first piece of an item cut at b1: finished after the barrier
        } else {
            dot_finish<NBX, NU, ACC_OUT, XBF>(D, cur.unit, B, lane, v, sx);
        }
        start += nreal;
        if (start < b1) cursor_next(P, cur);
    }
    if (failed) {
        // a stage never completed: record it, let the copies still in flight
        // land (bounded) and leave the CTA's item summing alone
        if (lane == 0) atomicCAS(&g_gemv_device_error, 0u, (unsigned int)SHERRY_ERR_TIMEOUT);
#pragma unroll
        for (int s = 0; s < RING; s++)
            if (inflight & (1u << s)) stage_wait(&bars[s], (phase >> s) & 1u);
        own_cut = false;
    }
    __syncthreads();  // the later pieces' sums are in shared memory
    if (own_cut) {
        const GemvDesc &D = P.d[cur.id];
        const int mine = D.chunk_begin + cur.unit * D.nchunk + cur.kp * D.cpp;  // the cut item
        for (int w = warp + 1; w < kWarps; w++) {
            const int cs = cut_start[w];
            if (cs == -2) continue;
            if (cs != mine) break;
#pragma unroll
            for (int u = 0; u < NU; u++)
#pragma unroll
                for (int b = 0; b < NBX; b++) v[u][b] += cut_sum[((w * NU + u) * NBX + b) * 32 + lane];
        }
        dot_finish<NBX, NU, ACC_OUT, XBF>(P.d[cur.id], cur.unit, B, lane, v, sx);
    }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
// Launch with the programmatic-stream-serialization attribute (see pdl_wait).
template <typename KernelT, typename ParamsT>
void launch_pdl(KernelT kernel, int grid, int threads, size_t smem, cudaStream_t stream,
                const ParamsT &gp) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3((unsigned)threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaLaunchKernelEx(&cfg, kernel, gp);
}

// The fp32 front-end: one cluster of kF32Cluster CTAs per (GEMV, token row),
// launched like the others with programmatic stream serialization.
void launch_xprep_f32(const XprepF32Params &p, cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(p.total_clusters * kF32Cluster));
    cfg.blockDim = dim3((unsigned)kF32Threads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kF32Cluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    cudaLaunchKernelEx(&cfg, xprep_f32_kernel, p);
}

template <typename KernelT>
int grid_for(KernelT kernel, int threads, size_t smem, int want, OccupancyCache &cache) {
    int dev = 0;
    cudaGetDevice(&dev);
    const int d = dev & 63;
    const unsigned long long now = context_id();
    int bps = cache.bps[d].load(std::memory_order_acquire);
    if (bps == 0 || now == 0 || cache.ctx[d].load(std::memory_order_acquire) != now) {
        if (smem > 48 * 1024)
            cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        bps = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&bps, kernel, threads, smem) != cudaSuccess ||
            bps < 1)
            bps = 1;
        cache.bps[d].store(bps, std::memory_order_release);
        cache.ctx[d].store(context_id(), std::memory_order_release);  // current now, if it was not
    }
    return std::max(1, std::min(want, bps * sm_count()));
}

template <int NB, bool ACC, int XR>
void launch_pipe(const GemvParams &gp, cudaStream_t stream) {
    static OccupancyCache cache;
    // one chunk per warp at most (items cut between warps are summed in shared memory)
    const size_t smem = PipeShape<NB>::kSmem;
    const int want = (gp.total_chunks + kPipeWarps - 1) / kPipeWarps;
    const int grid = grid_for(gemv_pipe_kernel<NB, ACC, XR>, kPipeThreads, smem, want, cache);
    launch_pdl(gemv_pipe_kernel<NB, ACC, XR>, grid, kPipeThreads, smem, stream, gp);
}

template <int NBX, bool ACC, int XMODE, int NU>
void launch_dot_nu(const GemvParams &gp, cudaStream_t stream) {
    static OccupancyCache cache;
    using Shape = DotShape<NBX, XMODE, kFmtSherry, NU>;
    // one chunk (of a unit group) per warp at most: a small GEMV spreads over as
    // many SMs as it has chunks (items cut between warps are summed in shared memory)
    const int want = (gp.total_chunks + Shape::kWarps - 1) / Shape::kWarps;
    const int grid = grid_for(gemv_dot_kernel<NBX, ACC, XMODE, kFmtSherry, NU>, Shape::kThreads,
                              Shape::kSmem, want, cache);
    launch_pdl(gemv_dot_kernel<NBX, ACC, XMODE, kFmtSherry, NU>, grid, Shape::kThreads, Shape::kSmem,
               stream, gp);
}
template <int NBX, bool ACC, int XMODE>
void launch_dot(const GemvParams &gp, int nu, cudaStream_t stream) {
    if (nu == 2) launch_dot_nu<NBX, ACC, XMODE, 2>(gp, stream);
    else launch_dot_nu<NBX, ACC, XMODE, 1>(gp, stream);
}

template <int NB, bool ACC>
void launch_regs(const GemvParams &gp, cudaStream_t stream) {
    static OccupancyCache cache;
    const int want = (gp.total_units16 + kGemvWarps - 1) / kGemvWarps;
    const int grid = grid_for(gemv_kernel<NB, ACC>, kGemvThreads, 0, want, cache);
    launch_pdl(gemv_kernel<NB, ACC>, grid, kGemvThreads, 0, stream, gp);
}

struct GemvCall {
    const uint32_t *codes;
    const float *scales;
    const int8_t *x;        // int8 activations, or null when xbf is given
    void *out;
    int64_t N, K;
    const uint16_t *xbf;    // bf16 activations (quantized per token), or null
    const float *xf = nullptr;  // fp32 activations (quantized per token), or null
    const float *xu = nullptr;  // with xf: SwiGLU up outputs, the activations being silu(xf) * xu
};

// First GEMV of a call that uses an activation pointer with a given K: a
// small open-addressing table (SHERRY_MAX_GROUP entries at most).  A slot is
// live only if it carries the current call's stamp, so starting a call costs
// one increment instead of clearing the table.
struct ActivationIndex {
    static constexpr int kSlots = 4 * SHERRY_MAX_GROUP;
    const void *ptr[kSlots];
    int64_t k[kSlots];
    int first[kSlots];
    uint32_t stamp[kSlots] = {};
    uint32_t now = 0;
    void start_call() {
        if (++now == 0) {  // the stamps wrapped: clear them once
            std::memset(stamp, 0, sizeof(stamp));
            now = 1;
        }
    }
    // the GEMV that first used (p, K) in this call, registering gemv i if none did
    int find_or_add(const void *p, int64_t K, int i) {
        const uint64_t h = (reinterpret_cast<uintptr_t>(p) >> 4) * 0x9E3779B97F4A7C15ull ^ (uint64_t)K;
        for (int n = 0; n < kSlots; n++) {
            const int s = (int)((h + (uint64_t)n) % kSlots);
            if (stamp[s] != now) {
                stamp[s] = now;
                ptr[s] = p;
                k[s] = K;
                first[s] = i;
                return i;
            }
            if (ptr[s] == p && k[s] == K) return first[s];
        }
        return i;
    }
};

// Words after a GEMV's region for the activation scales of the bf16 front-end.
constexpr int64_t kActScaleWords = 64;  // >= SHERRY_MAX_GEMV_BATCH, 256-byte region

enum Phase { kPrepare = 1, kRun = 2, kBoth = 3 };

sherry_status gemv_launch(const GemvCall *calls, int count, int B, bool acc_out, void *workspace,
                          size_t workspace_bytes, cudaStream_t stream, int phase) {
    if (count < 1) return SHERRY_ERR_SHAPE;
    if (count > SHERRY_MAX_GROUP) return SHERRY_ERR_UNSUPPORTED;
    if (B < 1) return SHERRY_ERR_SHAPE;
    if (B > SHERRY_MAX_GEMV_BATCH) return SHERRY_ERR_UNSUPPORTED;
    if (!workspace) return SHERRY_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return SHERRY_ERR_ALIGN;
    int64_t words = 0, units16 = 0, items = 0, chunks = 0;
    for (int i = 0; i < count; i++) {
        const GemvCall &c = calls[i];
        const bool need_x = (phase & kPrepare) != 0, need_out = (phase & kRun) != 0;
        if ((need_x && !c.x && !c.xbf && !c.xf) ||
            (need_out && (!c.codes || !c.out || (!acc_out && !c.scales))))
            return SHERRY_ERR_NULL;
        if (c.N < 1 || !valid_k(c.K)) return SHERRY_ERR_SHAPE;
        if ((need_x && c.x && !aligned(c.x, 4)) || (need_x && c.xbf && !aligned(c.xbf, 16)) ||
            (need_x && c.xf && !aligned(c.xf, 16)) || (need_x && c.xu && !aligned(c.xu, 16)) ||
            (need_out && (!aligned(c.codes, 4) || !aligned(c.out, 4) ||
                          (c.scales && !aligned(c.scales, 4)))))
            return SHERRY_ERR_ALIGN;
        if (c.N > (int64_t)1 << 28) return SHERRY_ERR_UNSUPPORTED;
        words += ws_words(c.N, c.K, B) + ((c.xbf || c.xf) ? kActScaleWords : 0);
        units16 += (c.N + 15) / 16;
        const int64_t nchunk = padded_tiles(c.K) / kChunkTiles;
        const int64_t kparts = kparts_for(c.K);
        items += (c.N + kUnitRows - 1) / kUnitRows * kparts;
        chunks += (c.N + kUnitRows - 1) / kUnitRows * nchunk;
    }
    if (workspace_bytes < (size_t)words * 4) return SHERRY_ERR_WORKSPACE;
    if (words > 0x7FFFFFFF || units16 > 0x7FFFFFFF || items > 0x7FFFFFFF || chunks > 0x7FFFFFFF)
        return SHERRY_ERR_UNSUPPORTED;

    // the pipelined kernel needs whole 4-tile chunks and 16-byte aligned code rows
    bool pipelined = true;
    for (int i = 0; i < count; i++)
        if ((calls[i].K / SHERRY_TILE_K) % kChunkTiles != 0 ||
            ((phase & kRun) && !aligned(calls[i].codes, 16)))
            pipelined = false;

    // one front-end per call: the fp32 one runs as its own cluster launch
    int nf32 = 0;
    for (int i = 0; i < count; i++) nf32 += calls[i].xf != nullptr;
    if (nf32 != 0 && nf32 != count) return SHERRY_ERR_UNSUPPORTED;
    const bool f32 = nf32 == count;

    // Launch parameters live in thread-local storage (they are too large for the
    // stack frame of every call).  Each is reached once through a reference, so
    // the loops below do not pay a thread-local address lookup per access, and
    // only the header and the descriptors in use are cleared (the kernels read
    // no descriptor past `count`).
    static thread_local XprepParams xp_tls;
    static thread_local XprepF32Params fp_tls;
    static thread_local GemvParams gp_tls;
    static thread_local ActivationIndex index_tls;
    XprepParams &xp = xp_tls;
    XprepF32Params &fp = fp_tls;
    GemvParams &gp = gp_tls;
    ActivationIndex &first_user = index_tls;
    std::memset(&xp, 0, offsetof(XprepParams, d) + (size_t)count * sizeof(XprepDesc));
    std::memset(&gp, 0, offsetof(GemvParams, d) + (size_t)count * sizeof(GemvDesc));
    if (f32) std::memset(&fp, 0, offsetof(XprepF32Params, d) + (size_t)count * sizeof(XprepF32Desc));
    xp.count = gp.count = fp.count = count;
    xp.B = gp.B = fp.B = B;
    xp.xrows = fp.xrows = xgroup_rows(B);
    fp.total_clusters = count * B;
    gp.mul4 = 4u;
    gp.mul2 = 2u;
    gp.f16one = 0x3C003C00u;
    gp.f16negz = 0x80008000u;
    gp.m33 = 0x33333333u;
    gp.m55 = 0x55555555u;
    gp.m44 = 0x44444444u;
    {
        const uint32_t lo[4] = {0x01010100u, 0x01010001u, 0x01000101u, 0x00010101u};
        const uint32_t hi[4] = {0xFFFFFF00u, 0xFFFF00FFu, 0xFF00FFFFu, 0x00FFFFFFu};
        for (int i = 0; i < 4; i++) {
            gp.tlo[i] = lo[i];
            gp.thi[i] = hi[i];
        }
    }
    first_user.start_call();
    // items of the dot kernel (B <= 2) hold one or two 32-row units, the MMA kernel's one
    const bool dot = pipelined && B <= 2;
    const int nu = dot && chunks > (int64_t)kDotPairMinChunksPerSM * sm_count() ? 2 : 1;
    int64_t off = 0;
    int wb = 0, ub16 = 0, cb = 0, cb32 = 0;
    for (int i = 0; i < count; i++) {
        const GemvCall &c = calls[i];
        uint32_t *region = static_cast<uint32_t *>(workspace) + off;
        const int Tp = (int)padded_tiles(c.K);
        const int xw_words = (int)round_words(xw_rows(B) * Tp * 32);
        const int units32 = (int)((c.N + kUnitRows - 1) / kUnitRows);
        const int units = (units32 + nu - 1) / nu;
        const int nchunk = Tp / kChunkTiles;
        const int kparts = (int)kparts_for(c.K);
        const int cpp = (nchunk + kparts - 1) / kparts;
        const bool bf = c.xbf != nullptr || c.xf != nullptr;
        // activation scales of the bf16 or fp32 front-end follow the GEMV's regular words
        float *act_scale = bf ? reinterpret_cast<float *>(region + ws_words(c.N, c.K, B)) : nullptr;
        XprepDesc &X = xp.d[i];
        X.x = c.x;
        X.xbf = c.xbf;
        X.xscale = act_scale;
        X.xw = region;
        X.zero = region + xw_words;
        X.K = (int)c.K;
        X.Tp = Tp;
        X.unit_begin = wb;
        X.xunits = bf ? B : B * (Tp / kXqTiles);
        X.zero_words = (int)split_words(c.N, c.K, B);
        if (f32) {
            XprepF32Desc &F = fp.d[i];
            F.x = c.xf;
            F.u = c.xu;
            F.xscale = act_scale;
            F.xw = region;
            F.q = nullptr;
            F.zero = X.zero;
            F.K = (int)c.K;
            F.Tp = Tp;
            F.cluster_begin = i * B;
            F.zero_words = X.zero_words;
        }
        GemvDesc &D = gp.d[i];
        D.codes = c.codes;
        D.scales = c.scales;
        D.xscale = act_scale;
        D.xw = reinterpret_cast<const uint4 *>(region);
        D.x = c.x;
        D.xbf = c.xbf;
        D.out = c.out;
        D.part_acc = kparts > 1 ? reinterpret_cast<int32_t *>(region + xw_words) : nullptr;
        D.part_cnt = kparts > 1 ? region + xw_words + (int64_t)B * c.N : nullptr;
        D.N = (int)c.N;
        D.T = (int)(c.K / SHERRY_TILE_K);
        D.Tp = Tp;
        D.unit_begin16 = ub16;
        D.units = units;
        D.units32 = units32;
        D.nchunk = nchunk;
        D.kparts = kparts;
        D.cpp = cpp;
        D.chunk_begin = cb;
        // A GEMV whose activations an earlier GEMV of the call already prepares
        // (same int8 or bf16 pointer, same K) reads that GEMV's region instead of
        // re-ordering them again: q, k and v, or gate and up, share one copy.
        // Only a call that prepares and runs (the run phase alone may not see x).
        if (phase == kBoth && !f32) {
            const int j = first_user.find_or_add(c.x ? (const void *)c.x : (const void *)c.xbf, c.K, i);
            if (j != i) {
                D.xw = gp.d[j].xw;
                D.xscale = gp.d[j].xscale;
                X.xunits = 0;
            }
        }
        off += ws_words(c.N, c.K, B) + (bf ? kActScaleWords : 0);
        // zero units: 32 words per warp (int8), 256 per CTA (bf16)
        wb += X.xunits + (X.zero_words + (c.xbf ? kBfWarps * 32 : 32) - 1) / (c.xbf ? kBfWarps * 32 : 32);
        ub16 += (int)((c.N + 15) / 16);
        cb += units * nchunk;
        cb32 += units32 * nchunk;
    }
    xp.total_units = wb;
    gp.total_units16 = ub16;
    gp.total_chunks = cb;
    // An int8 call at B <= 2 skips the re-order launch: the dot kernel re-orders
    // each chunk's activations itself (four shuffles and three byte permutes
    // per word, shared by the unit group's rows; rows are not split, so there
    // are no K-part sums to clear).
    bool raw_x = phase == kBoth && dot;
    bool raw_bf = raw_x && !acc_out && cb32 <= kRawBfMaxChunksPerSM * sm_count();
    for (int i = 0; i < count && raw_x; i++)
        raw_x = calls[i].x && !calls[i].xbf && !calls[i].xf && aligned(calls[i].x, 16) &&
                kparts_for(calls[i].K) == 1;
    // likewise a small bf16 call: each warp quantizes the tokens it reads
    for (int i = 0; i < count && raw_bf; i++)
        raw_bf = calls[i].xbf && kparts_for(calls[i].K) == 1;
    gp.prefetch_codes = (phase & kPrepare) && !raw_x && !raw_bf;
    if ((phase & kPrepare) && !raw_x && !raw_bf) {
        if (f32) {
            launch_xprep_f32(fp, stream);
        } else if (calls[0].xbf) {  // a call's GEMVs are all bf16 or all int8
            launch_pdl(xprep_bf16_kernel, std::max(1, std::min(wb, sm_count() * 8)), kBfWarps * 32, 0,
                       stream, xp);
        } else {
            const int blocks = std::max(1, std::min((wb + 7) / 8, sm_count() * 8));
            launch_pdl(xprep_kernel, blocks, 256, 0, stream, xp);
        }
        const sherry_status st = launch_status("sherry_gemv (activation re-order)");
        if (st != SHERRY_OK) return st;
    }
    if (!(phase & kRun)) return SHERRY_OK;
    // B <= 2: dp4a kernel; B >= 3: the MMA kernel (its 8 batch columns cost the
    // same as one, while dp4a work grows with B) -- measured on the decode stack
    if (dot) {
        if (raw_bf) {  // bf16 calls have no accumulator form
            if (B == 1) launch_dot<1, false, 2>(gp, nu, stream); else launch_dot<2, false, 2>(gp, nu, stream);
        } else if (raw_x) {
            if (B == 1) {
                if (acc_out) launch_dot<1, true, 1>(gp, nu, stream); else launch_dot<1, false, 1>(gp, nu, stream);
            } else {
                if (acc_out) launch_dot<2, true, 1>(gp, nu, stream); else launch_dot<2, false, 1>(gp, nu, stream);
            }
        } else if (B == 1) {
            if (acc_out) launch_dot<1, true, 0>(gp, nu, stream); else launch_dot<1, false, 0>(gp, nu, stream);
        } else {
            if (acc_out) launch_dot<2, true, 0>(gp, nu, stream); else launch_dot<2, false, 0>(gp, nu, stream);
        }
    } else if (pipelined) {
        if (B <= 4) {
            if (acc_out) launch_pipe<1, true, 4>(gp, stream); else launch_pipe<1, false, 4>(gp, stream);
        } else if (B <= 8) {
            if (acc_out) launch_pipe<1, true, 8>(gp, stream); else launch_pipe<1, false, 8>(gp, stream);
        } else {
            if (acc_out) launch_pipe<2, true, 8>(gp, stream); else launch_pipe<2, false, 8>(gp, stream);
        }
    } else {
        if (B <= 8) {
            if (acc_out) launch_regs<1, true>(gp, stream); else launch_regs<1, false>(gp, stream);
        } else {
            if (acc_out) launch_regs<2, true>(gp, stream); else launch_regs<2, false>(gp, stream);
        }
    }
    return launch_status("sherry_gemv");
}

sherry_status grouped(const sherry_gemv_desc *descs, int count, int B, void *workspace,
                      size_t workspace_bytes, cudaStream_t stream, int phase) {
    if (!descs) return SHERRY_ERR_NULL;
    if (count < 1) return SHERRY_ERR_SHAPE;
    if (count > SHERRY_MAX_GROUP) return SHERRY_ERR_UNSUPPORTED;
    GemvCall calls[SHERRY_MAX_GROUP];
    for (int i = 0; i < count; i++)
        calls[i] = GemvCall{descs[i].codes, descs[i].scales, descs[i].x, descs[i].y, descs[i].N,
                            descs[i].K, nullptr};
    return gemv_launch(calls, count, B, false, workspace, workspace_bytes, stream, phase);
}

sherry_status grouped_bf16(const sherry_gemv_bf16_desc *descs, int count, int B, void *workspace,
                           size_t workspace_bytes, cudaStream_t stream) {
    if (!descs) return SHERRY_ERR_NULL;
    if (count < 1) return SHERRY_ERR_SHAPE;
    if (count > SHERRY_MAX_GROUP) return SHERRY_ERR_UNSUPPORTED;
    GemvCall calls[SHERRY_MAX_GROUP];
    for (int i = 0; i < count; i++) {
        if (!descs[i].x) return SHERRY_ERR_NULL;
        calls[i] = GemvCall{descs[i].codes, descs[i].scales, nullptr, descs[i].y, descs[i].N,
                            descs[i].K, descs[i].x};
    }
    return gemv_launch(calls, count, B, false, workspace, workspace_bytes, stream, kBoth);
}

sherry_status grouped_f32(const sherry_gemv_f32_desc *descs, int count, int B, void *workspace,
                          size_t workspace_bytes, cudaStream_t stream) {
    if (!descs) return SHERRY_ERR_NULL;
    if (count < 1) return SHERRY_ERR_SHAPE;
    if (count > SHERRY_MAX_GROUP) return SHERRY_ERR_UNSUPPORTED;
    GemvCall calls[SHERRY_MAX_GROUP];
    for (int i = 0; i < count; i++) {
        if (!descs[i].x) return SHERRY_ERR_NULL;
        calls[i] = GemvCall{descs[i].codes, descs[i].scales, nullptr, descs[i].y, descs[i].N,
                            descs[i].K, nullptr, descs[i].x, descs[i].u};
    }
    return gemv_launch(calls, count, B, false, workspace, workspace_bytes, stream, kBoth);
}

// The fp32 front-end alone: q and s in natural order (one cluster per row).
sherry_status quantize_f32(const float *x, const float *u, int64_t B, int64_t K, int8_t *q, float *s,
                           cudaStream_t stream) {
    if (!x || !q || !s) return SHERRY_ERR_NULL;
    if (B < 1 || !valid_k(K)) return SHERRY_ERR_SHAPE;
    if (B > 65536) return SHERRY_ERR_UNSUPPORTED;
    if (!aligned(x, 16) || (u && !aligned(u, 16)) || !aligned(q, 4) || !aligned(s, 4))
        return SHERRY_ERR_ALIGN;
    static thread_local XprepF32Params fp;
    std::memset(&fp, 0, sizeof(fp));
    fp.count = 1;
    fp.B = (int)B;
    fp.total_clusters = (int)B;
    XprepF32Desc &F = fp.d[0];
    F.x = x;
    F.u = u;
    F.xscale = s;
    F.q = q;
    F.K = (int)K;
    F.Tp = (int)(K / SHERRY_TILE_K);
    launch_xprep_f32(fp, stream);
    return launch_status(u ? "sherry_quantize_swiglu" : "sherry_quantize_f32");
}

// ---------------------------------------------------------------------------
// Comparison formats: the 2-bit aligned and the three-in-five ternary
// packings the pages set Sherry against, streamed by the same small-batch
// kernel (gemv_dot_kernel with FMT = kFmtI2 / kFmtT3) for a like-for-like
// measurement.  Their codes are made from Sherry codes (the same ternary
// matrix) by a transcode kernel.
// ---------------------------------------------------------------------------
int64_t cmp_tiles(int fmt, int64_t K) {
    if (!valid_k(K)) return 0;
    if (fmt == kFmtI2) return K / SHERRY_TILE_K;
    if (fmt == kFmtT3) return 2 * ((K + 191) / 192);
    return 0;
}
int64_t cmp_tile_words(int fmt) { return fmt == kFmtI2 ? 8 : 5; }

// Ternary weight k of row n from Sherry codes (T tiles per row).
__device__ __forceinline__ int sherry_weight(const uint32_t *codes, int n, int k, int T) {
    const int t = k >> 7, j = (k >> 2) & 31, i = k & 3;
    const uint32_t *tile = codes + ((size_t)(n >> 5) * T + t) * kTileWords + (n & 31);
    const int p = (int)((__ldg(tile + 32 * (j & 1)) >> (2 * (j >> 1))) & 3u);
    if (i == p) return 0;
    const int r = i - (i > p ? 1 : 0);
    return ((__ldg(tile + 32 * (2 + r)) >> j) & 1u) ? -1 : 1;
}

// One thread per (row, comparison tile): decode the tile's weights from the
// Sherry codes and write its words; rows past N (the last group's padding)
// hold zero words, as in the Sherry layout.
__global__ void __launch_bounds__(256) transcode_kernel(const uint32_t *__restrict__ codes,
                                                        uint32_t *__restrict__ out, int N, int K,
                                                        int T, int Tc, int rows, int fmt) {
    const long long id = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (id >= (long long)rows * Tc) return;
    const int n = (int)(id % rows), t = (int)(id / rows);
    const bool real = n < N;
    if (fmt == kFmtI2) {
        uint32_t *dst = out + ((size_t)(n >> 5) * Tc + t) * 256 + (n & 31);
        for (int q = 0; q < 8; q++) {
            uint32_t w = 0;
            for (int m = 0; m < 16; m++) {
                const int v = real ? sherry_weight(codes, n, 128 * t + 16 * q + m, T) : 0;
                const uint32_t c = v == 0 ? 0u : (v > 0 ? 1u : 3u);
                w |= c << (4 * (m & 7) + 2 * (m >> 3));
            }
            dst[32 * q] = w;
        }
    } else {
        uint32_t w[5] = {0u, 0u, 0u, 0u, 0u};
        for (int j = 0; j < 32; j++) {
            int d[3];
            for (int e = 0; e < 3; e++) {
                const int k = 96 * t + 3 * j + e;
                d[e] = (real && k < K) ? sherry_weight(codes, n, k, T) : 0;
            }
            const uint32_t c = (uint32_t)((d[0] + 1) + 3 * (d[1] + 1) + 9 * (d[2] + 1));
            const int b = 5 * j;
            w[b >> 5] |= c << (b & 31);
            if ((b & 31) > 27) w[(b >> 5) + 1] |= c >> (32 - (b & 31));
        }
        uint32_t *dst = out + ((size_t)(n >> 5) * Tc + t) * 160 + (n & 31);
        for (int p = 0; p < 5; p++) dst[32 * p] = real ? w[p] : 0u;
    }
}

// T3 activations: word j of tile t = (x[96t+3j], x[96t+3j+1], x[96t+3j+2], 0)
// (zero past K), [B][Tc][32] per GEMV.  One thread per word.
struct CmpXDesc {
    const int8_t *x;
    uint32_t *xw;
    int K, Tc, word_begin, words;
};
struct CmpXParams {
    int count;
    int total_words;
    CmpXDesc d[SHERRY_MAX_GROUP];
};

__global__ void __launch_bounds__(256) t3_expand_kernel(const __grid_constant__ CmpXParams P) {
    pdl_allow_dependents();
    pdl_wait();  // x may come from the kernel before; the last GEMV may still read xw
    for (int g = blockIdx.x * blockDim.x + threadIdx.x; g < P.total_words; g += gridDim.x * blockDim.x) {
        int lo = 0, hi = P.count - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (P.d[mid].word_begin <= g) lo = mid; else hi = mid - 1;
        }
        const CmpXDesc &D = P.d[lo];
        const int w = g - D.word_begin;
        const int b = w / (D.Tc * 32), r = w - b * D.Tc * 32;  // r = tile * 32 + j
        const int k0 = 3 * (r & 31) + 96 * (r >> 5);
        const int8_t *xr = D.x + (size_t)b * D.K;
        uint32_t v = 0;
        for (int e = 0; e < 3; e++)
            if (k0 + e < D.K) v |= (uint32_t)(uint8_t)xr[k0 + e] << (8 * e);
        D.xw[w] = v;
    }
}

int64_t cmp_ws_words(int fmt, int64_t K, int B) {
    return fmt == kFmtT3 ? round_words((int64_t)B * cmp_tiles(fmt, K) * 32) : 0;
}

template <int NBX, bool ACC, int FMT, int NU>
void launch_dot_fmt_nu(const GemvParams &gp, cudaStream_t stream) {
    static OccupancyCache cache;
    using Shape = DotShape<NBX, 0, FMT, NU>;
    const size_t smem = Shape::kSmem;
    const int want = (gp.total_chunks + Shape::kWarps - 1) / Shape::kWarps;
    const int grid = grid_for(gemv_dot_kernel<NBX, ACC, 0, FMT, NU>, Shape::kThreads, smem, want, cache);
    launch_pdl(gemv_dot_kernel<NBX, ACC, 0, FMT, NU>, grid, Shape::kThreads, smem, stream, gp);
}
template <int NBX, bool ACC, int FMT>
void launch_dot_fmt(const GemvParams &gp, int nu, cudaStream_t stream) {
    if (nu == 2) launch_dot_fmt_nu<NBX, ACC, FMT, 2>(gp, stream);
    else launch_dot_fmt_nu<NBX, ACC, FMT, 1>(gp, stream);
}

sherry_status cmp_launch(int fmt, const GemvCall *calls, int count, int B, bool acc_out,
                         void *workspace, size_t workspace_bytes, cudaStream_t stream) {
    if (fmt != kFmtI2 && fmt != kFmtT3) return SHERRY_ERR_UNSUPPORTED;
    if (count < 1) return SHERRY_ERR_SHAPE;
    if (count > SHERRY_MAX_GROUP) return SHERRY_ERR_UNSUPPORTED;
    if (B < 1) return SHERRY_ERR_SHAPE;
    if (B > 2) return SHERRY_ERR_UNSUPPORTED;  // the comparison runs the decode kernel (B <= 2)
    int64_t words = 0, chunks = 0;
    for (int i = 0; i < count; i++) {
        const GemvCall &c = calls[i];
        if (!c.codes || !c.x || !c.out || (!acc_out && !c.scales)) return SHERRY_ERR_NULL;
        if (c.N < 1 || !valid_k(c.K)) return SHERRY_ERR_SHAPE;
        if (fmt == kFmtI2 && c.K % (4 * SHERRY_TILE_K) != 0) return SHERRY_ERR_SHAPE;
        if (!aligned(c.codes, 16) || !aligned(c.out, 4) || (c.scales && !aligned(c.scales, 4)) ||
            !aligned(c.x, fmt == kFmtI2 ? 16 : 1))
            return SHERRY_ERR_ALIGN;
        if (c.N > (int64_t)1 << 28) return SHERRY_ERR_UNSUPPORTED;
        words += cmp_ws_words(fmt, c.K, B);
        chunks += (c.N + kUnitRows - 1) / kUnitRows * (cmp_tiles(fmt, c.K) / (fmt == kFmtT3 ? 2 : 4));
    }
    if (words > 0 && (!workspace || !aligned(workspace, 256))) return workspace ? SHERRY_ERR_ALIGN
                                                                                : SHERRY_ERR_WORKSPACE;
    if (workspace_bytes < (size_t)words * 4) return SHERRY_ERR_WORKSPACE;
    if (words > 0x7FFFFFFF || chunks > 0x7FFFFFFF) return SHERRY_ERR_UNSUPPORTED;

    // one or two 32-row units per item, as for Sherry calls
    const int nu = chunks > (int64_t)kDotPairMinChunksPerSM * sm_count() ? 2 : 1;
    static thread_local GemvParams gp;
    static thread_local CmpXParams xp;
    std::memset(&gp, 0, sizeof(gp));
    std::memset(&xp, 0, sizeof(xp));
    gp.count = xp.count = count;
    gp.B = B;
    gp.m33 = 0x33333333u;
    gp.f16one = 0x3C003C00u;
    gp.f16negz = 0x80008000u;
    int64_t off = 0;
    int cb = 0, xb = 0;
    for (int i = 0; i < count; i++) {
        const GemvCall &c = calls[i];
        const int Tc = (int)cmp_tiles(fmt, c.K);
        const int ct = fmt == kFmtT3 ? 2 : 4;
        GemvDesc &D = gp.d[i];
        D.codes = c.codes;
        D.scales = c.scales;
        D.out = c.out;
        D.N = (int)c.N;
        D.T = Tc;
        D.units32 = (int)((c.N + kUnitRows - 1) / kUnitRows);
        D.units = (D.units32 + nu - 1) / nu;
        D.nchunk = Tc / ct;
        D.kparts = 1;
        D.cpp = D.nchunk;
        D.chunk_begin = cb;
        cb += D.units * D.nchunk;
        if (fmt == kFmtI2) {  // natural-order activations, read in place
            D.xw = reinterpret_cast<const uint4 *>(c.x);
            D.Tp = Tc;
        } else {
            uint32_t *region = static_cast<uint32_t *>(workspace) + off;
            D.xw = reinterpret_cast<const uint4 *>(region);
            D.Tp = Tc;
            CmpXDesc &X = xp.d[i];
            X.x = c.x;
            X.xw = region;
            X.K = (int)c.K;
            X.Tc = Tc;
            X.word_begin = xb;
            X.words = B * Tc * 32;
            xb += X.words;
            off += cmp_ws_words(fmt, c.K, B);
        }
    }
    gp.total_chunks = cb;
    xp.total_words = xb;
    if (fmt == kFmtT3) {
        const int blocks = std::max(1, std::min((xb + 255) / 256, sm_count() * 8));
        launch_pdl(t3_expand_kernel, blocks, 256, 0, stream, xp);
        const sherry_status st = launch_status("sherry_cmp_gemv (activation expansion)");
        if (st != SHERRY_OK) return st;
        gp.prefetch_codes = 1;  // follows this call's own expansion launch
    }
    if (fmt == kFmtI2) {
        if (B == 1) {
            if (acc_out) launch_dot_fmt<1, true, kFmtI2>(gp, nu, stream); else launch_dot_fmt<1, false, kFmtI2>(gp, nu, stream);
        } else {
            if (acc_out) launch_dot_fmt<2, true, kFmtI2>(gp, nu, stream); else launch_dot_fmt<2, false, kFmtI2>(gp, nu, stream);
        }
    } else {
        if (B == 1) {
            if (acc_out) launch_dot_fmt<1, true, kFmtT3>(gp, nu, stream); else launch_dot_fmt<1, false, kFmtT3>(gp, nu, stream);
        } else {
            if (acc_out) launch_dot_fmt<2, true, kFmtT3>(gp, nu, stream); else launch_dot_fmt<2, false, kFmtT3>(gp, nu, stream);
        }
    }
    return launch_status("sherry_cmp_gemv");
}

// Per-token quantization of bf16 activations, natural order (one warp per row).
__global__ void __launch_bounds__(256) quantize_act_kernel(const uint16_t *__restrict__ x, int B, int K,
                                                           int8_t *__restrict__ q, float *__restrict__ s) {
    const int lane = threadIdx.x & 31;
    const int b = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (b >= B) return;
    const uint16_t *row = x + (size_t)b * K;
    const float amax = row_absmax_bf16(row, K, lane);
    const float inv = amax > 0.0f ? __fdiv_rn(127.0f, amax) : 0.0f;
    if (lane == 0) s[b] = amax > 0.0f ? __fdiv_rn(amax, 127.0f) : 0.0f;
    const uint2 *r2 = reinterpret_cast<const uint2 *>(row);
    uint32_t *qw = reinterpret_cast<uint32_t *>(q + (size_t)b * K);
    for (int i = lane; i < K / 4; i += 32) qw[i] = quant_word(__ldg(r2 + i), inv);
}

}  // namespace

// Reads and clears the GEMV kernels' error word (SHERRY_OK if none); the
// caller has synchronised the device.
sherry_status gemv_device_error() {
    unsigned int v = 0;
    cudaError_t err = cudaMemcpyFromSymbol(&v, g_gemv_device_error, sizeof(v));
    if (err != cudaSuccess) {
        set_last_error("sherry_device_error (read)", err);
        return SHERRY_ERR_CUDA;
    }
    if (v != 0) {
        const unsigned int zero = 0;
        err = cudaMemcpyToSymbol(g_gemv_device_error, &zero, sizeof(zero));
        if (err != cudaSuccess) {
            set_last_error("sherry_device_error (clear)", err);
            return SHERRY_ERR_CUDA;
        }
    }
    return static_cast<sherry_status>(v);
}

}  // namespace sherry

extern "C" size_t sherry_gemv_workspace_bytes(int64_t N, int64_t K, int B) {
    if (B < 1 || N < 1 || K < 1) return 0;
    return (size_t)sherry::ws_words(N, K, B) * 4;
}

extern "C" sherry_status sherry_gemv(const uint32_t *codes, const float *scales, const int8_t *x,
                                     float *y, int64_t N, int64_t K, int B, void *workspace,
                                     size_t workspace_bytes, sherry_stream_t stream) {
    if (!scales) return SHERRY_ERR_NULL;
    const sherry::GemvCall c{codes, scales, x, y, N, K, nullptr};
    return sherry::gemv_launch(&c, 1, B, false, workspace, workspace_bytes,
                               reinterpret_cast<cudaStream_t>(stream), sherry::kBoth);
}

extern "C" sherry_status sherry_gemv_acc(const uint32_t *codes, const int8_t *x, int32_t *acc,
                                         int64_t N, int64_t K, int B, void *workspace,
                                         size_t workspace_bytes, sherry_stream_t stream) {
    const sherry::GemvCall c{codes, nullptr, x, acc, N, K, nullptr};
    return sherry::gemv_launch(&c, 1, B, true, workspace, workspace_bytes,
                               reinterpret_cast<cudaStream_t>(stream), sherry::kBoth);
}

extern "C" sherry_status sherry_gemv_grouped(const sherry_gemv_desc *descs, int count, int B,
                                             void *workspace, size_t workspace_bytes,
                                             sherry_stream_t stream) {
    return sherry::grouped(descs, count, B, workspace, workspace_bytes,
                           reinterpret_cast<cudaStream_t>(stream), sherry::kBoth);
}

extern "C" sherry_status sherry_gemv_prepare(const sherry_gemv_desc *descs, int count, int B,
                                             void *workspace, size_t workspace_bytes,
                                             sherry_stream_t stream) {
    return sherry::grouped(descs, count, B, workspace, workspace_bytes,
                           reinterpret_cast<cudaStream_t>(stream), sherry::kPrepare);
}

extern "C" sherry_status sherry_gemv_run(const sherry_gemv_desc *descs, int count, int B,
                                         const void *workspace, size_t workspace_bytes,
                                         sherry_stream_t stream) {
    return sherry::grouped(descs, count, B, const_cast<void *>(workspace), workspace_bytes,
                           reinterpret_cast<cudaStream_t>(stream), sherry::kRun);
}

extern "C" size_t sherry_gemv_bf16_workspace_bytes(int64_t N, int64_t K, int B) {
    if (B < 1 || N < 1 || K < 1) return 0;
    return (size_t)(sherry::ws_words(N, K, B) + sherry::kActScaleWords) * 4;
}

extern "C" sherry_status sherry_gemv_bf16(const uint32_t *codes, const float *scales,
                                          const uint16_t *x, float *y, int64_t N, int64_t K, int B,
                                          void *workspace, size_t workspace_bytes,
                                          sherry_stream_t stream) {
    if (!scales || !x) return SHERRY_ERR_NULL;
    const sherry::GemvCall c{codes, scales, nullptr, y, N, K, x};
    return sherry::gemv_launch(&c, 1, B, false, workspace, workspace_bytes,
                               reinterpret_cast<cudaStream_t>(stream), sherry::kBoth);
}

extern "C" sherry_status sherry_gemv_bf16_grouped(const sherry_gemv_bf16_desc *descs, int count,
                                                  int B, void *workspace, size_t workspace_bytes,
                                                  sherry_stream_t stream) {
    return sherry::grouped_bf16(descs, count, B, workspace, workspace_bytes,
                                reinterpret_cast<cudaStream_t>(stream));
}

extern "C" sherry_status sherry_quantize_act(const uint16_t *x, int64_t B, int64_t K, int8_t *q,
                                             float *s, sherry_stream_t stream) {
    using namespace sherry;
    if (!x || !q || !s) return SHERRY_ERR_NULL;
    if (B < 1 || K < 8 || K % 8 != 0) return SHERRY_ERR_SHAPE;
    if (B > 0x7FFFFFFF || K > 0x7FFFFFFF) return SHERRY_ERR_UNSUPPORTED;
    if (!aligned(x, 16) || !aligned(q, 4) || !aligned(s, 4)) return SHERRY_ERR_ALIGN;
    const int blocks = (int)((B + 7) / 8);
    quantize_act_kernel<<<blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(x, (int)B, (int)K,
                                                                                    q, s);
    return launch_status("sherry_quantize_act");
}

extern "C" size_t sherry_gemv_f32_workspace_bytes(int64_t N, int64_t K, int B) {
    return sherry_gemv_bf16_workspace_bytes(N, K, B);
}

extern "C" sherry_status sherry_gemv_f32(const uint32_t *codes, const float *scales, const float *x,
                                         float *y, int64_t N, int64_t K, int B, void *workspace,
                                         size_t workspace_bytes, sherry_stream_t stream) {
    if (!scales || !x) return SHERRY_ERR_NULL;
    const sherry::GemvCall c{codes, scales, nullptr, y, N, K, nullptr, x, nullptr};
    return sherry::gemv_launch(&c, 1, B, false, workspace, workspace_bytes,
                               reinterpret_cast<cudaStream_t>(stream), sherry::kBoth);
}

extern "C" sherry_status sherry_gemv_swiglu(const uint32_t *codes, const float *scales,
                                            const float *g, const float *u, float *y, int64_t N,
                                            int64_t K, int B, void *workspace,
                                            size_t workspace_bytes, sherry_stream_t stream) {
    if (!scales || !g || !u) return SHERRY_ERR_NULL;
    const sherry::GemvCall c{codes, scales, nullptr, y, N, K, nullptr, g, u};
    return sherry::gemv_launch(&c, 1, B, false, workspace, workspace_bytes,
                               reinterpret_cast<cudaStream_t>(stream), sherry::kBoth);
}

extern "C" sherry_status sherry_gemv_f32_grouped(const sherry_gemv_f32_desc *descs, int count, int B,
                                                 void *workspace, size_t workspace_bytes,
                                                 sherry_stream_t stream) {
    return sherry::grouped_f32(descs, count, B, workspace, workspace_bytes,
                               reinterpret_cast<cudaStream_t>(stream));
}

extern "C" sherry_status sherry_quantize_f32(const float *x, int64_t B, int64_t K, int8_t *q, float *s,
                                             sherry_stream_t stream) {
    return sherry::quantize_f32(x, nullptr, B, K, q, s, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" sherry_status sherry_quantize_swiglu(const float *g, const float *u, int64_t B, int64_t K,
                                                int8_t *q, float *s, sherry_stream_t stream) {
    if (!u) return SHERRY_ERR_NULL;
    return sherry::quantize_f32(g, u, B, K, q, s, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" size_t sherry_cmp_packed_bytes(int fmt, int64_t N, int64_t K) {
    const int64_t T = sherry::cmp_tiles(fmt, K);
    if (T == 0 || N < 1) return 0;
    return (size_t)((N + SHERRY_ROW_GROUP - 1) / SHERRY_ROW_GROUP) * SHERRY_ROW_GROUP * (size_t)T *
           (size_t)sherry::cmp_tile_words(fmt) * 4;
}

extern "C" size_t sherry_cmp_workspace_bytes(int fmt, int64_t N, int64_t K, int B) {
    if (N < 1 || B < 1 || sherry::cmp_tiles(fmt, K) == 0) return 0;
    return (size_t)sherry::cmp_ws_words(fmt, K, B) * 4;
}

extern "C" sherry_status sherry_cmp_transcode(int fmt, const uint32_t *codes, int64_t N, int64_t K,
                                              uint32_t *out, sherry_stream_t stream) {
    using namespace sherry;
    if (fmt != kFmtI2 && fmt != kFmtT3) return SHERRY_ERR_UNSUPPORTED;
    if (!codes || !out) return SHERRY_ERR_NULL;
    if (N < 1 || !valid_k(K)) return SHERRY_ERR_SHAPE;
    if (N > (int64_t)1 << 28) return SHERRY_ERR_UNSUPPORTED;
    if (!aligned(codes, 4) || !aligned(out, 4)) return SHERRY_ERR_ALIGN;
    const int64_t rows = (N + kUnitRows - 1) / kUnitRows * kUnitRows;
    const int64_t Tc = cmp_tiles(fmt, K);
    const int64_t threads = rows * Tc;
    if (threads > 0x7FFFFFFFLL * 256) return SHERRY_ERR_UNSUPPORTED;
    transcode_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        codes, out, (int)N, (int)K, (int)(K / SHERRY_TILE_K), (int)Tc, (int)rows, fmt);
    return launch_status("sherry_cmp_transcode");
}

extern "C" sherry_status sherry_cmp_gemv_grouped(int fmt, const sherry_gemv_desc *descs, int count,
                                                 int B, void *workspace, size_t workspace_bytes,
                                                 sherry_stream_t stream) {
    using namespace sherry;
    if (!descs) return SHERRY_ERR_NULL;
    if (count < 1) return SHERRY_ERR_SHAPE;
    if (count > SHERRY_MAX_GROUP) return SHERRY_ERR_UNSUPPORTED;
    GemvCall calls[SHERRY_MAX_GROUP];
    for (int i = 0; i < count; i++)
        calls[i] = GemvCall{descs[i].codes, descs[i].scales, descs[i].x, descs[i].y, descs[i].N,
                            descs[i].K, nullptr};
    return cmp_launch(fmt, calls, count, B, false, workspace, workspace_bytes,
                      reinterpret_cast<cudaStream_t>(stream));
}

extern "C" sherry_status sherry_cmp_gemv_acc(int fmt, const uint32_t *codes, const int8_t *x,
                                             int32_t *acc, int64_t N, int64_t K, int B,
                                             void *workspace, size_t workspace_bytes,
                                             sherry_stream_t stream) {
    const sherry::GemvCall c{codes, nullptr, x, acc, N, K, nullptr};
    return sherry::cmp_launch(fmt, &c, 1, B, true, workspace, workspace_bytes,
                              reinterpret_cast<cudaStream_t>(stream));
}

// ---------------------------------------------------------------------------
// sherry_gemv_static: the GEMV above with its scratch in a fixed device array.
// ---------------------------------------------------------------------------
namespace sherry {
namespace {

static __device__ __align__(256) uint32_t g_gemv_static_scratch[SHERRY_STATIC_SCRATCH_BYTES / 4];

constexpr int kStaticMaxDevices = 64;
std::mutex g_static_mu;
void *g_static_ptr[kStaticMaxDevices] = {};
unsigned long long g_static_ctx[kStaticMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once
// per device and context.
sherry_status static_scratch(void **out) {
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) {
        set_last_error("sherry_gemv_static (cudaGetDevice)", err);
        return SHERRY_ERR_CUDA;
    }
    if (dev < 0 || dev >= kStaticMaxDevices) return SHERRY_ERR_UNSUPPORTED;
    const unsigned long long now = context_id();
    std::lock_guard<std::mutex> lock(g_static_mu);
    if (g_static_ptr[dev] == nullptr || now == 0 || g_static_ctx[dev] != now) {
        void *p = nullptr;
        err = cudaGetSymbolAddress(&p, g_gemv_static_scratch);
        if (err != cudaSuccess || p == nullptr) {
            g_static_ptr[dev] = nullptr;
            set_last_error("sherry_gemv_static (cudaGetSymbolAddress)",
                           err != cudaSuccess ? err : cudaErrorInvalidSymbol);
            return SHERRY_ERR_CUDA;
        }
        g_static_ptr[dev] = p;
        g_static_ctx[dev] = context_id();  // the lookup made the context current if it was not
    }
    *out = g_static_ptr[dev];
    return SHERRY_OK;
}

}  // namespace
}  // namespace sherry

extern "C" sherry_status sherry_gemv_static(const uint32_t *codes, const float *scales,
                                            const int8_t *x, float *y, int64_t N, int64_t K, int B,
                                            sherry_stream_t stream) {
    using namespace sherry;
    if (!codes || !scales || !x || !y) return SHERRY_ERR_NULL;
    if (N < 1 || !valid_k(K) || B < 1) return SHERRY_ERR_SHAPE;
    if (B > SHERRY_MAX_GEMV_BATCH || N > (int64_t)1 << 28) return SHERRY_ERR_UNSUPPORTED;
    const size_t need = (size_t)ws_words(N, K, B) * 4;
    if (need > (size_t)SHERRY_STATIC_SCRATCH_BYTES) {
        char msg[200];
        std::snprintf(msg, sizeof(msg),
                      "sherry_gemv_static: N=%lld K=%lld B=%d needs %zu bytes of scratch; the "
                      "static scratch holds %zu",
                      (long long)N, (long long)K, B, need, (size_t)SHERRY_STATIC_SCRATCH_BYTES);
        set_last_error_text(msg);
        return SHERRY_ERR_WORKSPACE;
    }
    void *scratch = nullptr;
    const sherry_status st = static_scratch(&scratch);
    if (st != SHERRY_OK) return st;
    const GemvCall c{codes, scales, x, y, N, K, nullptr};
    return gemv_launch(&c, 1, B, false, scratch, SHERRY_STATIC_SCRATCH_BYTES,
                       reinterpret_cast<cudaStream_t>(stream), kBoth);
}
