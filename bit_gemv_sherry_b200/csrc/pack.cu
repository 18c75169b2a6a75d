// pack.cu -- sherry_pack: fp32 latent weights -> Sherry 1.25-bit codes + row scales.
//
// The step the pages call "packing blocks of four weights into five bits" under
// "3:4 fine-grained sparsity" (arXiv 2601.07892, abstract).  One warp handles a
// 128-weight tile: lane j loads block j as a float4 (one coalesced 512-byte
// row segment per warp), picks its zero (smallest |w|, lowest index on ties),
// and the warp assembles the five words with ballots -- bit j of a ballot is
// block j, which is exactly the bit-sliced sign layout.  Kept |w| are summed
// in double per lane, reduced over the warp, then over the warps of the row in
// a fixed order, so the scale is deterministic.  HBM-bound: 4 bytes read and
// 0.16 bytes written per weight.
#include "common.cuh"

namespace sherry {
namespace {

constexpr int kPackThreads = 256;
constexpr int kPackWarps = kPackThreads / 32;
constexpr int kPackUnroll = 4;

struct TileBits {
    uint32_t z0, z1, s0, s1, s2;
    double sum;
};

__device__ __forceinline__ float4 ld_stream(const float4 *p) {
    float4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ TileBits pack_tile(float4 v) {
    const float a0 = fabsf(v.x), a1 = fabsf(v.y), a2 = fabsf(v.z), a3 = fabsf(v.w);
    int p = 0;
    float m = a0;
    if (a1 < m) { p = 1; m = a1; }
    if (a2 < m) { p = 2; m = a2; }
    if (a3 < m) { p = 3; m = a3; }
    const bool f0 = v.x < 0.0f, f1 = v.y < 0.0f, f2 = v.z < 0.0f, f3 = v.w < 0.0f;
    // kept weights in ascending position -> ranks 0, 1, 2
    const bool r0 = (p == 0) ? f1 : f0;
    const bool r1 = (p <= 1) ? f2 : f1;
    const bool r2 = (p <= 2) ? f3 : f2;
    const float k0 = (p == 0) ? a1 : a0;
    const float k1 = (p <= 1) ? a2 : a1;
    const float k2 = (p <= 2) ? a3 : a2;
    TileBits tb;
    const uint32_t L = __ballot_sync(0xFFFFFFFFu, p & 1);
    const uint32_t H = __ballot_sync(0xFFFFFFFFu, p & 2);
    tb.s0 = __ballot_sync(0xFFFFFFFFu, r0);
    tb.s1 = __ballot_sync(0xFFFFFFFFu, r1);
    tb.s2 = __ballot_sync(0xFFFFFFFFu, r2);
    // Z0: fields of the even blocks, Z1: fields of the odd blocks.
    tb.z0 = (L & 0x55555555u) | ((H & 0x55555555u) << 1);
    tb.z1 = ((L >> 1) & 0x55555555u) | (H & 0xAAAAAAAAu);
    double s = (double)k0 + (double)k1 + (double)k2;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
    tb.sum = s;
    return tb;
}

// CTA = 8 warps; `wpr` warps share one row (tiles strided by wpr), the CTA
// covers 8 / wpr rows.  Rows N..Npad-1 (padding of the last 32-row group) are
// written as zero words.
__global__ void __launch_bounds__(kPackThreads) pack_kernel(const float *__restrict__ w, int64_t N,
                                                            int64_t Npad, int64_t K, int wpr,
                                                            uint32_t *__restrict__ codes,
                                                            float *__restrict__ scales) {
    __shared__ double partial[kPackWarps];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int rpc = kPackWarps / wpr;
    const int64_t n = (int64_t)blockIdx.x * rpc + warp / wpr;
    const int sub = warp % wpr;
    const int64_t T = K / SHERRY_TILE_K;
    double row_sum = 0.0;
    // word (p, n, t) = ((n / 32) * T + t) * 160 + 32 p + n % 32
    uint32_t *out = codes + (n / SHERRY_ROW_GROUP) * T * (5 * SHERRY_ROW_GROUP) + n % SHERRY_ROW_GROUP;
    if (n < N) {
        const float4 *row = reinterpret_cast<const float4 *>(w + n * K);
        for (int64_t t0 = sub; t0 < T; t0 += (int64_t)wpr * kPackUnroll) {
            float4 v[kPackUnroll];
#pragma unroll
            for (int u = 0; u < kPackUnroll; u++) {
                const int64_t t = t0 + (int64_t)u * wpr;
                v[u] = (t < T) ? ld_stream(row + t * 32 + lane) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int u = 0; u < kPackUnroll; u++) {
                const int64_t t = t0 + (int64_t)u * wpr;
                if (t >= T) break;  // warp-uniform
                const TileBits tb = pack_tile(v[u]);
                row_sum += tb.sum;
                if (lane < 5) {
                    const uint32_t word = lane == 0 ? tb.z0 : lane == 1 ? tb.z1 : lane == 2 ? tb.s0
                                          : lane == 3 ? tb.s1 : tb.s2;
                    out[t * (5 * SHERRY_ROW_GROUP) + lane * SHERRY_ROW_GROUP] = word;
                }
            }
        }
    } else if (n < Npad) {
        for (int64_t t = sub; t < T; t += wpr)
            if (lane < 5) out[t * (5 * SHERRY_ROW_GROUP) + lane * SHERRY_ROW_GROUP] = 0u;
    }
    if (lane == 0) partial[warp] = row_sum;
    __syncthreads();
    if (threadIdx.x < rpc) {
        const int64_t rn = (int64_t)blockIdx.x * rpc + threadIdx.x;
        if (rn < N) {
            double s = 0.0;
            for (int k = 0; k < wpr; k++) s += partial[threadIdx.x * wpr + k];
            scales[rn] = (float)(s / (0.75 * (double)K));
        }
    }
}

}  // namespace
}  // namespace sherry

extern "C" sherry_status sherry_pack(const float *w, int64_t N, int64_t K, uint32_t *codes,
                                     float *scales, sherry_stream_t stream) {
    using namespace sherry;
    if (!w || !codes || !scales) return SHERRY_ERR_NULL;
    if (N < 1 || !valid_k(K)) return SHERRY_ERR_SHAPE;
    if (!aligned(w, 16) || !aligned(codes, 16) || !aligned(scales, 4)) return SHERRY_ERR_ALIGN;
    const int64_t T = K / SHERRY_TILE_K;
    const int64_t Npad = (N + SHERRY_ROW_GROUP - 1) / SHERRY_ROW_GROUP * SHERRY_ROW_GROUP;
    int wpr = 1;
    while (wpr < kPackWarps && wpr * 2 <= T) wpr *= 2;
    const int rpc = kPackWarps / wpr;
    const int64_t grid = (Npad + rpc - 1) / rpc;
    if (grid > 0x7FFFFFFF) return SHERRY_ERR_UNSUPPORTED;
    pack_kernel<<<(unsigned)grid, kPackThreads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        w, N, Npad, K, wpr, codes, scales);
    return launch_status("sherry_pack");
}
