// pack.cu -- sherry_pack: fp32 latent weights -> Sherry 1.25-bit codes + row scales.
//
// The format's packing step: every block of four weights keeps one zero (3:4
// sparsity) and is coded in five bits (arXiv 2601.07892, abstract).  One warp handles a
// 128-weight tile at a time: lane j loads block j as a float4 (one coalesced
// 512-byte row segment per warp), picks its zero (smallest |w|, lowest index
// on ties), and the warp assembles the five words with ballots -- bit j of a
// ballot is block j, which is exactly the bit-sliced sign layout.  A warp
// takes a run of tiles of one row and keeps eight tile loads in flight.  Kept
// |w| are summed in double per lane, reduced over the warp once, then over the
// warps of the row in a fixed order, so the scale is deterministic.  One
// launch serves one matrix (sherry_pack) or a group of matrices
// (sherry_pack_grouped: a model's projections at load time, without a launch
// per matrix).  HBM-bound: 4 bytes read and 0.16 bytes written per weight.
#include <algorithm>
#include <cstring>

#include "common.cuh"

namespace sherry {
namespace {

constexpr int kPackThreads = 128;  // 4 warps: 0.83 ms for the 1B stack's latents against 0.85 with 8, 0.86 with 16
constexpr int kPackWarps = kPackThreads / 32;
constexpr int kPackBatch = 8;      // tiles loaded per batch
// fewest tiles a warp of a multi-warp row takes: rows up to K = 8192 get one
// warp (measured on the 1B stack's 3.9 GB of latents: 0.98 ms with 8, 0.85 ms
// with 64; 16 loads per batch instead of 8 ran slower at any split)
constexpr int64_t kPackMinTiles = 64;

struct TileBits {
    uint32_t z0, z1, s0, s1, s2;
};

__device__ __forceinline__ float4 ld_stream(const float4 *p) {
    float4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "l"(p));
    return v;
}

// Zero position, kept signs and the five words of one tile (lane j = block j);
// `kept` receives this lane's sum of kept |w| (not reduced over the warp).
__device__ __forceinline__ TileBits pack_tile(float4 v, double &kept) {
    const float a0 = fabsf(v.x), a1 = fabsf(v.y), a2 = fabsf(v.z), a3 = fabsf(v.w);
    // argmin with the lowest index on ties, as selects (no branches)
    const bool b1 = a1 < a0;
    const float m01 = b1 ? a1 : a0;
    const int p01 = b1 ? 1 : 0;
    const bool b2 = a2 < m01;
    const float m02 = b2 ? a2 : m01;
    const int p02 = b2 ? 2 : p01;
    const int p = (a3 < m02) ? 3 : p02;
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
    kept += (double)k0 + (double)k1 + (double)k2;
    return tb;
}

// Lanes 0..4 store words Z0, Z1, S0, S1, S2 of a tile at plane offsets 32 p.
__device__ __forceinline__ void store_words(uint32_t *tile_out, const TileBits &tb, int lane) {
    const uint32_t lo = (lane & 1) ? tb.z1 : tb.z0;
    const uint32_t sg = (lane & 1) ? tb.s1 : tb.s0;
    const uint32_t word = (lane & 4) ? tb.s2 : ((lane & 2) ? sg : lo);
    if (lane < 5) tile_out[lane * SHERRY_ROW_GROUP] = word;
}

// One launch packs a group of matrices; matrix i owns CTAs cta_begin[i] ..
// cta_begin[i+1]-1.  CTA = 4 warps; `wpr` warps share one row, warp `sub` of
// a row takes the `tpw` consecutive tiles sub * tpw .. and loads them
// kPackBatch at a time (all loads of a batch in flight before the first tile
// is packed).  Each lane sums its kept |w| in double over all its tiles; the
// lanes are reduced once per warp and the warps of a row in a fixed order, so
// the scale is deterministic.  Rows N..Npad-1 (padding of the last 32-row
// group) are written as zero words.
struct PackDesc {
    const float *w;
    uint32_t *codes;
    float *scales;
    int64_t N, Npad, K, tpw;
    int wpr;
    int cta_begin;
};
struct PackParams {
    int count;
    int pad;
    PackDesc d[SHERRY_MAX_GROUP];
};

__global__ void __launch_bounds__(kPackThreads) pack_kernel(const __grid_constant__ PackParams P) {
    __shared__ double partial[kPackWarps];
    int lo = 0, hi = P.count - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (P.d[mid].cta_begin <= (int)blockIdx.x) lo = mid; else hi = mid - 1;
    }
    const PackDesc &D = P.d[lo];
    const float *__restrict__ w = D.w;
    uint32_t *__restrict__ codes = D.codes;
    float *__restrict__ scales = D.scales;
    const int64_t N = D.N, Npad = D.Npad, K = D.K, tpw = D.tpw;
    const int wpr = D.wpr;
    const int64_t cta = (int64_t)blockIdx.x - D.cta_begin;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int rpc = kPackWarps / wpr;
    const int64_t n = cta * rpc + warp / wpr;
    const int sub = warp % wpr;
    const int64_t T = K / SHERRY_TILE_K;
    const int64_t t_begin = sub * tpw;
    const int64_t t_end = t_begin + tpw < T ? t_begin + tpw : T;
    double kept = 0.0;
    // word (p, n, t) = ((n / 32) * T + t) * 160 + 32 p + n % 32
    uint32_t *out = codes + (n / SHERRY_ROW_GROUP) * T * (5 * SHERRY_ROW_GROUP) + n % SHERRY_ROW_GROUP;
    if (n < N) {
        const float4 *row = reinterpret_cast<const float4 *>(w + n * K);
        for (int64_t t0 = t_begin; t0 < t_end; t0 += kPackBatch) {
            if (t0 + kPackBatch <= t_end) {  // full batch: no per-tile bounds tests
                float4 v[kPackBatch];
#pragma unroll
                for (int u = 0; u < kPackBatch; u++) v[u] = ld_stream(row + (t0 + u) * 32 + lane);
#pragma unroll
                for (int u = 0; u < kPackBatch; u++) {
                    const TileBits tb = pack_tile(v[u], kept);
                    store_words(out + (t0 + u) * (5 * SHERRY_ROW_GROUP), tb, lane);
                }
            } else {
                for (int64_t t = t0; t < t_end; t++) {
                    const TileBits tb = pack_tile(ld_stream(row + t * 32 + lane), kept);
                    store_words(out + t * (5 * SHERRY_ROW_GROUP), tb, lane);
                }
            }
        }
    } else if (n < Npad) {
        for (int64_t t = t_begin; t < t_end; t++)
            if (lane < 5) out[t * (5 * SHERRY_ROW_GROUP) + lane * SHERRY_ROW_GROUP] = 0u;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) kept += __shfl_xor_sync(0xFFFFFFFFu, kept, o);
    if (lane == 0) partial[warp] = kept;
    __syncthreads();
    if (threadIdx.x < rpc) {
        const int64_t rn = cta * rpc + threadIdx.x;
        if (rn < N) {
            double s = 0.0;
            for (int k = 0; k < wpr; k++) s += partial[threadIdx.x * wpr + k];
            scales[rn] = (float)(s / (0.75 * (double)K));
        }
    }
}

}  // namespace

// Checks one matrix of a pack call.
sherry_status pack_check(const float *w, int64_t N, int64_t K, const uint32_t *codes,
                         const float *scales) {
    if (!w || !codes || !scales) return SHERRY_ERR_NULL;
    if (N < 1 || !valid_k(K)) return SHERRY_ERR_SHAPE;
    if (!aligned(w, 16) || !aligned(codes, 16) || !aligned(scales, 4)) return SHERRY_ERR_ALIGN;
    return SHERRY_OK;
}

// One launch over `count` checked matrices (w, codes, scales, N, K filled in).
sherry_status pack_launch(PackDesc *descs, int count, cudaStream_t stream) {
    static thread_local PackParams pp;
    std::memset(&pp, 0, sizeof(pp));
    pp.count = count;
    int64_t ctas = 0;
    for (int i = 0; i < count; i++) {
        PackDesc &d = descs[i];
        const int64_t T = d.K / SHERRY_TILE_K;
        d.Npad = (d.N + SHERRY_ROW_GROUP - 1) / SHERRY_ROW_GROUP * SHERRY_ROW_GROUP;
        // warps per row: as many as keep at least kPackMinTiles tiles each (up to 4)
        int wpr = 1;
        while (wpr < kPackWarps && (int64_t)wpr * 2 * kPackMinTiles <= T) wpr *= 2;
        d.wpr = wpr;
        d.tpw = (T + wpr - 1) / wpr;
        const int rpc = kPackWarps / wpr;
        d.cta_begin = (int)ctas;
        ctas += (d.Npad + rpc - 1) / rpc;
        if (ctas > 0x7FFFFFFF) return SHERRY_ERR_UNSUPPORTED;
        pp.d[i] = d;
    }
    pack_kernel<<<(unsigned)ctas, kPackThreads, 0, stream>>>(pp);
    return launch_status("sherry_pack");
}

}  // namespace sherry

extern "C" sherry_status sherry_pack(const float *w, int64_t N, int64_t K, uint32_t *codes,
                                     float *scales, sherry_stream_t stream) {
    using namespace sherry;
    const sherry_status st = pack_check(w, N, K, codes, scales);
    if (st != SHERRY_OK) return st;
    PackDesc d = {};
    d.w = w;
    d.codes = codes;
    d.scales = scales;
    d.N = N;
    d.K = K;
    return pack_launch(&d, 1, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" sherry_status sherry_pack_grouped(const sherry_pack_desc *descs, int count,
                                             sherry_stream_t stream) {
    using namespace sherry;
    if (!descs) return SHERRY_ERR_NULL;
    if (count < 1) return SHERRY_ERR_SHAPE;
    if (count > SHERRY_MAX_GROUP) return SHERRY_ERR_UNSUPPORTED;
    PackDesc d[SHERRY_MAX_GROUP] = {};
    for (int i = 0; i < count; i++) {
        const sherry_status st = pack_check(descs[i].w, descs[i].N, descs[i].K, descs[i].codes,
                                            descs[i].scales);
        if (st != SHERRY_OK) return st;
        d[i].w = descs[i].w;
        d[i].codes = descs[i].codes;
        d[i].scales = descs[i].scales;
        d[i].N = descs[i].N;
        d[i].K = descs[i].K;
    }
    return pack_launch(d, count, reinterpret_cast<cudaStream_t>(stream));
}
