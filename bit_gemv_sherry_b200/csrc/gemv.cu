// gemv.cu -- decode GEMV on Sherry codes: y = s (.) (W_ternary . x_int8), B <= 16.
//
// The product is the one the pages state for ternary weights with 3:4 blocks
// coded in five bits (arXiv 2601.07892, abstract; Figure 2 caption: "SIMD-
// friendly 4-way patterns").  On B200 the batch-1 GEMV is bound by HBM reads of
// the codes (0.15625 bytes per weight) only if the decode costs a few
// instructions per 4-weight block, so:
//
//   * each warp owns 16 output rows (the M of an int8 m16n8k32 tensor-core
//     MMA) and walks K four tiles at a time, one tile per thread of a quad;
//   * a thread decodes its tile for two rows with 32-bit SWAR logic: per
//     (position i, block group beta) one selector word whose nibbles are
//     (zero position | sign << 2) of eight blocks, and one byte permute
//     (PRMT) per four weights against an 8-byte table -- ~2.8 instructions
//     per 4-weight block, no shared memory, no lookup loads;
//   * the int8 words go straight from registers into mma.sync as the A
//     fragment; the activations, re-ordered once per call into the same
//     order (xprep_kernel), are the B fragment, one batch row per column, so
//     batches up to 8 cost the same MMA count as batch 1;
//   * accumulation is exact int32; the epilogue applies the row scale once.
//
// The MMA replaces the per-block dp4a of a plain SIMT kernel (one tensor-core
// instruction per 128 blocks instead of 128 dp4a), leaving the issue slots to
// the decode.
#include <algorithm>
#include <cstring>

#include "common.cuh"

namespace sherry {
namespace {

constexpr int kGemvThreads = 256;
constexpr int kGemvWarps = kGemvThreads / 32;

struct GemvDesc {
    const uint32_t *codes;
    const float *scales;
    const uint4 *xw;   // re-ordered activations [B][T][32 words]
    void *out;         // float y[B][N] or int32 acc[B][N]
    int N;
    int T;
    int unit_begin;    // first 16-row unit of this GEMV in the group
    int pad;
};

struct GemvParams {
    int count;
    int B;
    int total_units;
    int pad;
    GemvDesc d[SHERRY_MAX_GROUP];
};

struct XprepDesc {
    const int8_t *x;
    uint32_t *xw;
    int K;
    int word_begin;  // first output word of this GEMV
};

struct XprepParams {
    int count;
    int B;
    int total_words;
    int pad;
    XprepDesc d[SHERRY_MAX_GROUP];
};

// xw[b][t][q]: word q = 2 (4 i + beta) + h holds the activations met by
// char4(i, beta, h) of tile t: bytes x[b][128 t + 16 k' + 64 h + 4 beta + i], k' = 0..3.
__global__ void __launch_bounds__(256) xprep_kernel(const __grid_constant__ XprepParams P) {
    const int w = blockIdx.x * blockDim.x + threadIdx.x;
    if (w >= P.total_words) return;
    int lo = 0, hi = P.count - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (P.d[mid].word_begin <= w) lo = mid; else hi = mid - 1;
    }
    const XprepDesc &D = P.d[lo];
    const int local = w - D.word_begin;
    const int T = D.K / SHERRY_TILE_K;
    const int q = local & 31;
    const int t = (local >> 5) % T;
    const int b = (local >> 5) / T;
    const int m = q >> 1, h = q & 1, i = m >> 2, beta = m & 3;
    const uint8_t *src = reinterpret_cast<const uint8_t *>(D.x) + (size_t)b * D.K +
                         (size_t)t * SHERRY_TILE_K + 64 * h + 4 * beta + i;
    const uint32_t v = (uint32_t)src[0] | ((uint32_t)src[16] << 8) | ((uint32_t)src[32] << 16) |
                       ((uint32_t)src[48] << 24);
    D.xw[local] = v;
}

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

// NB = number of 8-row batch groups (1: B <= 8, 2: B <= 16).
template <int NB, bool ACC_OUT>
__global__ void __launch_bounds__(kGemvThreads) gemv_kernel(const __grid_constant__ GemvParams P) {
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int nwarps = gridDim.x * kGemvWarps;
    for (int u = blockIdx.x * kGemvWarps + (threadIdx.x >> 5); u < P.total_units; u += nwarps) {
        int lo = 0, hi = P.count - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (P.d[mid].unit_begin <= u) lo = mid; else hi = mid - 1;
        }
        const GemvDesc &D = P.d[lo];
        const int N = D.N, T = D.T;
        const int r0 = (u - D.unit_begin) * 16 + g, r1 = r0 + 8;
        const bool v0 = r0 < N, v1 = r1 < N;
        const size_t plane = (size_t)N * T;
        const uint32_t *c0 = D.codes + (size_t)r0 * T;
        const uint32_t *c1 = D.codes + (size_t)r1 * T;

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
                w0[p] = (tv && v0) ? ld_code(c0 + p * plane + tile) : 0u;
                w1[p] = (tv && v1) ? ld_code(c1 + p * plane + tile) : 0u;
            }
        }
        for (int s = 0; s < nslices; s++) {
            const int tile = s * 4 + t;
            const bool tv = tile < T;
            TileDecoder d0, d1;
            d0.load(w0[0], w0[1], w0[2], w0[3], w0[4]);
            d1.load(w1[0], w1[1], w1[2], w1[3], w1[4]);
            // activations of this tile for batch rows g (+8)
            uint4 xv[NB][8];
#pragma unroll
            for (int nb = 0; nb < NB; nb++) {
                const int b = nb * 8 + g;
                const bool xvld = tv && b < P.B;
                const uint4 *xp = D.xw + ((size_t)b * T + tile) * 8;
#pragma unroll
                for (int k = 0; k < 8; k++) xv[nb][k] = xvld ? ld_x(xp + k) : make_uint4(0, 0, 0, 0);
            }
            // prefetch the next slice's code words
            if (s + 1 < nslices) {
                const int nt = tile + 4;
                const bool ntv = nt < T;
#pragma unroll
                for (int p = 0; p < 5; p++) {
                    w0[p] = (ntv && v0) ? ld_code(c0 + p * plane + nt) : 0u;
                    w1[p] = (ntv && v1) ? ld_code(c1 + p * plane + nt) : 0u;
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
                        const uint32_t b0 = pick(xq, (m & 1) * 2), b1 = pick(xq, (m & 1) * 2 + 1);
                        mma_s8(acc[nb], a0, a1, a2, a3, b0, b1);
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
                    if (ACC_OUT) {
                        static_cast<int32_t *>(D.out)[(size_t)b * N + row] = acc[nb][e];
                    } else {
                        static_cast<float *>(D.out)[(size_t)b * N + row] =
                            __ldg(D.scales + row) * (float)acc[nb][e];
                    }
                }
            }
        }
    }
}

size_t ws_bytes(int64_t K, int B) { return (size_t)((B * K + 255) / 256) * 256; }

template <int NB, bool ACC>
int gemv_grid(int units) {
    static int blocks_per_sm[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    int &bps = blocks_per_sm[dev & 63];
    if (bps == 0) {
        int n = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, gemv_kernel<NB, ACC>, kGemvThreads, 0) !=
                cudaSuccess ||
            n < 1)
            n = 1;
        bps = n;
    }
    const int want = (units + kGemvWarps - 1) / kGemvWarps;
    return std::max(1, std::min(want, bps * sm_count()));
}

struct GemvCall {
    const uint32_t *codes;
    const float *scales;
    const int8_t *x;
    void *out;
    int64_t N, K;
};

sherry_status gemv_launch(const GemvCall *calls, int count, int B, bool acc_out, void *workspace,
                          size_t workspace_bytes, cudaStream_t stream) {
    if (count < 1) return SHERRY_ERR_SHAPE;
    if (count > SHERRY_MAX_GROUP) return SHERRY_ERR_UNSUPPORTED;
    if (B < 1) return SHERRY_ERR_SHAPE;
    if (B > SHERRY_MAX_GEMV_BATCH) return SHERRY_ERR_UNSUPPORTED;
    if (!workspace) return SHERRY_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return SHERRY_ERR_ALIGN;
    size_t need = 0;
    int64_t units = 0, words = 0;
    for (int i = 0; i < count; i++) {
        const GemvCall &c = calls[i];
        if (!c.codes || !c.x || !c.out || (!acc_out && !c.scales)) return SHERRY_ERR_NULL;
        if (c.N < 1 || !valid_k(c.K)) return SHERRY_ERR_SHAPE;
        if (!aligned(c.codes, 4) || !aligned(c.x, 4) || !aligned(c.out, 4) ||
            (c.scales && !aligned(c.scales, 4)))
            return SHERRY_ERR_ALIGN;
        if (c.N > (int64_t)1 << 30) return SHERRY_ERR_UNSUPPORTED;
        need += ws_bytes(c.K, B);
        units += (c.N + 15) / 16;
        words += (int64_t)B * c.K / 4;
    }
    if (workspace_bytes < need) return SHERRY_ERR_WORKSPACE;
    if (units > 0x7FFFFFFF || words > 0x7FFFFFFF) return SHERRY_ERR_UNSUPPORTED;

    static thread_local XprepParams xp;
    static thread_local GemvParams gp;
    std::memset(&xp, 0, sizeof(xp));
    std::memset(&gp, 0, sizeof(gp));
    xp.count = gp.count = count;
    xp.B = gp.B = B;
    size_t off = 0;
    int ub = 0, wb = 0;
    for (int i = 0; i < count; i++) {
        const GemvCall &c = calls[i];
        uint32_t *xw = reinterpret_cast<uint32_t *>(static_cast<char *>(workspace) + off);
        xp.d[i].x = c.x;
        xp.d[i].xw = xw;
        xp.d[i].K = (int)c.K;
        xp.d[i].word_begin = wb;
        gp.d[i].codes = c.codes;
        gp.d[i].scales = c.scales;
        gp.d[i].xw = reinterpret_cast<const uint4 *>(xw);
        gp.d[i].out = c.out;
        gp.d[i].N = (int)c.N;
        gp.d[i].T = (int)(c.K / SHERRY_TILE_K);
        gp.d[i].unit_begin = ub;
        off += ws_bytes(c.K, B);
        ub += (int)((c.N + 15) / 16);
        wb += (int)((int64_t)B * c.K / 4);
    }
    xp.total_words = wb;
    gp.total_units = ub;
    xprep_kernel<<<(wb + 255) / 256, 256, 0, stream>>>(xp);
    sherry_status st = launch_status("sherry_gemv (activation re-order)");
    if (st != SHERRY_OK) return st;
    if (B <= 8) {
        if (acc_out)
            gemv_kernel<1, true><<<gemv_grid<1, true>(ub), kGemvThreads, 0, stream>>>(gp);
        else
            gemv_kernel<1, false><<<gemv_grid<1, false>(ub), kGemvThreads, 0, stream>>>(gp);
    } else {
        if (acc_out)
            gemv_kernel<2, true><<<gemv_grid<2, true>(ub), kGemvThreads, 0, stream>>>(gp);
        else
            gemv_kernel<2, false><<<gemv_grid<2, false>(ub), kGemvThreads, 0, stream>>>(gp);
    }
    return launch_status("sherry_gemv");
}

}  // namespace
}  // namespace sherry

extern "C" size_t sherry_gemv_workspace_bytes(int64_t K, int B) {
    if (B < 1 || K < 1) return 0;
    return sherry::ws_bytes(K, B);
}

extern "C" sherry_status sherry_gemv(const uint32_t *codes, const float *scales, const int8_t *x,
                                     float *y, int64_t N, int64_t K, int B, void *workspace,
                                     size_t workspace_bytes, sherry_stream_t stream) {
    const sherry::GemvCall c{codes, scales, x, y, N, K};
    if (!scales) return SHERRY_ERR_NULL;
    return sherry::gemv_launch(&c, 1, B, false, workspace, workspace_bytes,
                               reinterpret_cast<cudaStream_t>(stream));
}

extern "C" sherry_status sherry_gemv_acc(const uint32_t *codes, const int8_t *x, int32_t *acc,
                                         int64_t N, int64_t K, int B, void *workspace,
                                         size_t workspace_bytes, sherry_stream_t stream) {
    const sherry::GemvCall c{codes, nullptr, x, acc, N, K};
    return sherry::gemv_launch(&c, 1, B, true, workspace, workspace_bytes,
                               reinterpret_cast<cudaStream_t>(stream));
}

extern "C" sherry_status sherry_gemv_grouped(const sherry_gemv_desc *descs, int count, int B,
                                             void *workspace, size_t workspace_bytes,
                                             sherry_stream_t stream) {
    if (!descs) return SHERRY_ERR_NULL;
    if (count < 1) return SHERRY_ERR_SHAPE;
    if (count > SHERRY_MAX_GROUP) return SHERRY_ERR_UNSUPPORTED;
    sherry::GemvCall calls[SHERRY_MAX_GROUP];
    for (int i = 0; i < count; i++) {
        calls[i] = sherry::GemvCall{descs[i].codes, descs[i].scales, descs[i].x, descs[i].y,
                                    descs[i].N, descs[i].K};
        if (!descs[i].scales) return SHERRY_ERR_NULL;
    }
    return sherry::gemv_launch(calls, count, B, false, workspace, workspace_bytes,
                               reinterpret_cast<cudaStream_t>(stream));
}
