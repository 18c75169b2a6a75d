// gemm.cu -- prefill GEMM on Sherry codes with tcgen05 int8 tensor cores.
//
//   Y[m][n] = s[n] * sum_k X[m][k] * W[n][k],  X int8 [M][K], W ternary from codes.
//
// The pages give only the format (arXiv 2601.07892, abstract: ternary weights,
// 3:4 sparsity, four weights in five bits).  At M >= 64 tokens the product is a
// dense contraction, so the weights are decoded to int8 in shared memory and
// fed to the 5th-generation tensor cores:
//
//   warp 0      TMA producer: 256-token x 128-byte X tiles, 128-byte swizzle,
//               into a 4-stage ring (completion via mbarrier transaction count);
//   warp 1      allocates 512 TMEM columns (two 128 x 256 int32 accumulators)
//               and, from one thread, issues tcgen05.mma.kind::i8 (M=128,
//               N=256, K=32) four times per stage, committing every second
//               stage back to its producers (a commit frees a pair of stages)
//               and each finished tile to the epilogue;
//   warps 2-9   decoders, two groups of four taking alternate stages: thread r
//               of a group loads weight row r's five code words (two of its
//               stages ahead), decodes them (SWAR + PRMT, as in the GEMV),
//               re-orders the bytes to natural K order with 4x4 byte
//               transposes and writes the row's 128 bytes into the swizzled
//               K-major operand layout;
//   warps 10-13 epilogue: tcgen05.ld of their 32-lane quarter of the finished
//               accumulator, y = s * (float) acc, coalesced fp32 stores;
//               double-buffered TMEM lets tile i's epilogue overlap tile i+1's MMAs.
//
// Weights are the A operand (M = 128 output features per tile), tokens the B
// operand (N = 256), so each decoded weight feeds 256 tokens.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>

#include "common.cuh"

namespace sherry {

// First error recorded by a kernel of this file (see sherry_device_error).
__device__ unsigned int g_gemm_device_error = 0;

namespace {

constexpr int kBM = 128;            // weight rows per tile (UMMA M)
constexpr int kBN = 256;            // tokens per tile (UMMA N)
constexpr int kBK = 128;            // K per stage = one Sherry tile
constexpr int kStages = 4;
constexpr int kABytes = kBM * kBK;  // 16 KB
constexpr int kBBytes = kBN * kBK;  // 32 KB
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kDecGroups = 2;                   // decoder groups, taking alternate stages
constexpr int kThreads = 32 * (2 + 4 * kDecGroups + 4);
constexpr int kTmemCols = 512;
constexpr uint32_t kIdesc = (2u << 4)                  // D = s32
                            | (1u << 7) | (1u << 10)   // A, B = signed int8
                            | ((uint32_t)(kBN >> 3) << 17) | ((uint32_t)(kBM >> 4) << 24);
constexpr size_t kSmemBytes = (size_t)kStages * kStageBytes + 1024 + 512;
constexpr int kMaxDevices = 64;  // devices whose kernel attributes are tracked
// Bounded waits, in SM clock cycles: the operand and accumulator barriers
// (settable through sherry_set_wait_limit) and the drains of copies and MMAs
// already in flight, which keep their own long limit.
constexpr long long kDefaultWaitLimit = 4000000000LL;  // ~2 s at 1.9 GHz
constexpr long long kDrainWaitLimit = 1000000000LL;
std::atomic<long long> g_wait_limit{0};  // 0: kDefaultWaitLimit

struct __align__(8) Barriers {
    uint64_t full_a[kStages];         // A tile written: 128 decoder threads
    uint64_t full_b[kStages];         // X tile landed: 1 arrival + bytes
    uint64_t empty[kStages / 2];      // stage pair (2p, 2p+1) read by the MMAs: 1 commit
    uint64_t tmem_full[2];
    uint64_t tmem_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

__device__ __forceinline__ uint32_t ld_code(const uint32_t *p) {
    uint32_t v;
    asm volatile("ld.global.nc.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}

// 4x4 byte transpose: out[k] byte i = in[i] byte k.
__device__ __forceinline__ void transpose4(const uint32_t (&in)[4], uint32_t (&out)[4]) {
    const uint32_t t0 = prmt(in[0], in[1], 0x5140u), t1 = prmt(in[0], in[1], 0x7362u);
    const uint32_t t2 = prmt(in[2], in[3], 0x5140u), t3 = prmt(in[2], in[3], 0x7362u);
    out[0] = prmt(t0, t2, 0x5410u);
    out[1] = prmt(t0, t2, 0x7632u);
    out[2] = prmt(t1, t3, 0x5410u);
    out[3] = prmt(t1, t3, 0x7632u);
}

template <bool ACC_OUT>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmap_x, const uint32_t *__restrict__ codes,
                const float *__restrict__ scales, void *__restrict__ out, int M, int N, int T,
                long long wait_limit) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + ((1024 - (raw_addr & 1023)) & 1023);
    Barriers *bar = reinterpret_cast<Barriers *>(smem + (size_t)kStages * kStageBytes);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tiles_n = (N + kBM - 1) / kBM, tiles_m = (M + kBN - 1) / kBN;
    const int num_tiles = tiles_n * tiles_m;
    volatile int *abort = &bar->abort;
    unsigned int *err = &g_gemm_device_error;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; s++) {
            mbar_init(&bar->full_a[s], 128);
            mbar_init(&bar->full_b[s], 1);
            if (s % 2 == 0) mbar_init(&bar->empty[s / 2], 1);
        }
        for (int a = 0; a < 2; a++) {
            mbar_init(&bar->tmem_full[a], 1);
            mbar_init(&bar->tmem_empty[a], 128);
        }
        mbar_init(&bar->drain, 1);
        bar->abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&bar->tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = bar->tmem_base;

    if (warp == 0) {
        // ---------------- TMA producer: X tiles ----------------
        if (lane == 0) {
            uint32_t it = 0;
            for (int tile = blockIdx.x; tile < num_tiles && !*abort; tile += gridDim.x) {
                const int xb = tile / tiles_n;
                for (int kt = 0; kt < T; kt++, it++) {
                    const int s = it % kStages;
                    const uint32_t ph = (it / kStages) & 1;
                    if (!mbar_wait(&bar->empty[s >> 1], ph ^ 1, abort, err, wait_limit)) break;
                    uint8_t *b_smem = smem + (size_t)s * kStageBytes + kABytes;
                    mbar_arrive_expect_tx(&bar->full_b[s], kBBytes);
                    tma_load_2d(b_smem, &tmap_x, &bar->full_b[s], kt * kBK, xb * kBN);
                }
            }
            // Let every issued copy land before the CTA's shared memory is released,
            // whether or not a role gave up later: the last copy of each stage
            // (earlier ones were consumed through the stage's barrier phases).
            const uint32_t n = it < (uint32_t)kStages ? it : (uint32_t)kStages;
            for (uint32_t j = 1; j <= n; j++) {
                const uint32_t k = it - j;
                volatile int no_abort = 0;
                mbar_wait(&bar->full_b[k % kStages], (k / kStages) & 1, &no_abort, err,
                          kDrainWaitLimit);
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            uint32_t it = 0, acc_it = 0;
            bool issued = false;
            for (int tile = blockIdx.x; tile < num_tiles && !*abort; tile += gridDim.x, acc_it++) {
                const uint32_t a = acc_it & 1, aph = (acc_it >> 1) & 1;
                if (!mbar_wait(&bar->tmem_empty[a], aph ^ 1, abort, err, wait_limit)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + a * kBN;
                bool ok = true;
                for (int kt = 0; kt < T; kt++, it++) {
                    const int s = it % kStages;
                    const uint32_t ph = (it / kStages) & 1;
                    if (!mbar_wait(&bar->full_a[s], ph, abort, err, wait_limit) ||
                        !mbar_wait(&bar->full_b[s], ph, abort, err, wait_limit)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(smem + (size_t)s * kStageBytes);
                    const uint32_t b_addr = a_addr + kABytes;
#pragma unroll
                    for (int k = 0; k < kBK / 32; k++) {
                        umma_i8(d_tmem, smem_desc_sw128(a_addr + 32 * k),
                                smem_desc_sw128(b_addr + 32 * k), kIdesc, (kt | k) != 0);
                    }
                    issued = true;
                    // one commit frees a pair of stages: half the commits of the issuing thread
                    if (s & 1) umma_commit(&bar->empty[s >> 1]);
                }
                if (!ok) break;
                umma_commit(&bar->tmem_full[a]);
            }
            // Wait for every issued MMA before TMEM and the operand stages are
            // released, whether or not a role gave up after this loop ended.
            if (issued) {
                umma_commit(&bar->drain);
                volatile int no_abort = 0;
                mbar_wait(&bar->drain, 0, &no_abort, err, kDrainWaitLimit);
            }
        }
    } else if (warp < 2 + 4 * kDecGroups) {
        // ------- decoders: group g takes stages j = g mod kDecGroups, one row per thread -------
        // Stage j of this CTA is (tile blockIdx.x + (j / T) * gridDim.x, K tile j % T).  A
        // thread loads its row's five code words itself (a warp reads 128 contiguous bytes
        // per plane) two of its group's stages ahead, so the loads overlap the decode.
        const int g = (warp - 2) >> 2;
        const int r = threadIdx.x - 64 - 128 * g;
        const int my_tiles = num_tiles > (int)blockIdx.x
                                 ? (num_tiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
        const uint32_t total = (uint32_t)my_tiles * (uint32_t)T;
        auto load_stage = [&](uint32_t j, uint32_t (&w)[5]) {
            const int tile = (int)blockIdx.x + (int)(j / T) * (int)gridDim.x;
            const int row = (tile % tiles_n) * kBM + r;
            if (j < total && row < N) {
                // word (p, row, kt) = ((row / 32) * T + kt) * 160 + 32 p + row % 32
                const uint32_t *c = codes + ((size_t)(row / 32) * T + j % T) * 160 + (row % 32);
#pragma unroll
                for (int p = 0; p < 5; p++) w[p] = ld_code(c + 32 * p);
            } else {
#pragma unroll
                for (int p = 0; p < 5; p++) w[p] = 0u;
            }
        };
        uint32_t wa[5], wb[5];
        load_stage(g, wa);
        load_stage(g + kDecGroups, wb);
        for (uint32_t j = g; j < total; j += kDecGroups) {
            uint32_t w[5];
#pragma unroll
            for (int p = 0; p < 5; p++) {
                w[p] = wa[p];
                wa[p] = wb[p];
            }
            load_stage(j + 2 * kDecGroups, wb);
            const int s = j % kStages;
            const uint32_t ph = (j / kStages) & 1;
            // the A slot's previous tile has been consumed by the MMAs
            if (!__all_sync(0xFFFFFFFFu, mbar_wait(&bar->empty[s >> 1], ph ^ 1, abort, err, wait_limit)))
                break;
            const int tile = (int)blockIdx.x + (int)(j / T) * (int)gridDim.x;
            const bool valid = (tile % tiles_n) * kBM + r < N;
            TileDecoder dec;
            dec.load(w[0], w[1], w[2], w[3], w[4]);
            uint8_t *a_row = smem + (size_t)s * kStageBytes + (size_t)r * kBK;
#pragma unroll
            for (int h = 0; h < 2; h++) {
                uint32_t nat[4][4];  // [beta][k'] natural-order words of block 4(k'+4h)+beta
#pragma unroll
                for (int beta = 0; beta < 4; beta++) {
                    uint32_t byi[4];
#pragma unroll
                    for (int i = 0; i < 4; i++) {
                        const uint32_t sel = dec.sel(i, beta);
                        byi[i] = valid ? prmt(table_lo(i), table_hi(i), h ? (sel >> 16) : sel) : 0u;
                    }
                    transpose4(byi, nat[beta]);
                }
#pragma unroll
                for (int kp = 0; kp < 4; kp++) {
                    const int c = 4 * h + kp;  // 16-byte chunk = blocks 4c..4c+3
                    const uint4 v = make_uint4(nat[0][kp], nat[1][kp], nat[2][kp], nat[3][kp]);
                    *reinterpret_cast<uint4 *>(a_row + ((c ^ (r & 7)) << 4)) = v;
                }
            }
            fence_proxy_async_smem();
            mbar_arrive(&bar->full_a[s]);
        }
    } else {
        // ---------------- epilogue ----------------
        const int q = warp & 3;  // TMEM lane quarter this warp may access
        uint32_t acc_it = 0;
        for (int tile = blockIdx.x; tile < num_tiles && !*abort; tile += gridDim.x, acc_it++) {
            const int wb = tile % tiles_n, xb = tile / tiles_n;
            const uint32_t a = acc_it & 1, aph = (acc_it >> 1) & 1;
            // every lane waits; the warp leaves together if any lane's wait gave up
            if (!__all_sync(0xFFFFFFFFu, mbar_wait(&bar->tmem_full[a], aph, abort, err, wait_limit)))
                break;
            tc_fence_after();
            const int row = wb * kBM + q * 32 + lane;
            const bool rv = row < N;
            const float sc = (!ACC_OUT && rv) ? __ldg(scales + row) : 0.0f;
            const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + a * kBN;
            for (int c0 = 0; c0 < kBN; c0 += 16) {
                uint32_t v[16];
                tmem_ld16(taddr + c0, v);
                tmem_ld_wait();
                const int tok0 = xb * kBN + c0;
#pragma unroll
                for (int j = 0; j < 16; j++) {
                    const int tok = tok0 + j;
                    if (rv && tok < M) {
                        if (ACC_OUT)
                            static_cast<int32_t *>(out)[(size_t)tok * N + row] = (int32_t)v[j];
                        else
                            static_cast<float *>(out)[(size_t)tok * N + row] = sc * (float)(int32_t)v[j];
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(&bar->tmem_empty[a]);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

// Tensor-core peak probe: one CTA per SM issues back-to-back
// tcgen05.mma.cta_group::1.kind::i8 of the GEMM's shape (M = 128, N = 256,
// K = 32, A and B from 128-byte-swizzled shared memory, int32 accumulator in
// tensor memory) on zeroed operands, with no data movement and no barrier
// between them: the int8 rate the GEMM's MMAs can reach on this device.
constexpr int kProbeThreads = 128;
constexpr int kProbeN = 256;                                  // widest UMMA N
constexpr size_t kProbeSmem = (size_t)kABytes + kProbeN * kBK + 1024;
constexpr uint32_t kProbeIdesc = (2u << 4) | (1u << 7) | (1u << 10) |
                                 ((uint32_t)(kProbeN >> 3) << 17) | ((uint32_t)(kBM >> 4) << 24);

__global__ void __launch_bounds__(kProbeThreads, 1) mma_probe_kernel(int iters) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + ((1024 - (raw_addr & 1023)) & 1023);
    __shared__ __align__(8) uint64_t done;
    __shared__ uint32_t tmem_base;
    for (int i = threadIdx.x; i < (kABytes + kProbeN * kBK) / 16; i += blockDim.x)
        reinterpret_cast<uint4 *>(smem)[i] = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async_smem();  // the zeroed operands, to the tensor core's view
    if (threadIdx.x == 0) {
        mbar_init(&done, 1);
        fence_mbar_init();
    }
    if (threadIdx.x < 32) {
        tmem_alloc(&tmem_base, kProbeN);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (threadIdx.x == 0) {
        const uint32_t a_addr = smem_u32(smem), b_addr = a_addr + kABytes;
        for (int it = 0; it < iters; it++) {
#pragma unroll
            for (int k = 0; k < kBK / 32; k++)
                umma_i8(tmem_base, smem_desc_sw128(a_addr + 32 * k), smem_desc_sw128(b_addr + 32 * k),
                        kProbeIdesc, (it | k) != 0);
        }
        umma_commit(&done);
        volatile int no_abort = 0;
        mbar_wait(&done, 0, &no_abort, &g_gemm_device_error, kDrainWaitLimit);
    }
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x < 32) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kProbeN);
    }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

template <bool ACC>
sherry_status gemm_launch(const uint32_t *codes, const float *scales, const int8_t *x, void *out,
                          int64_t M, int64_t N, int64_t K, cudaStream_t stream) {
    if (!codes || !x || !out || (!ACC && !scales)) return SHERRY_ERR_NULL;
    if (M < 1 || N < 1 || !valid_k(K)) return SHERRY_ERR_SHAPE;
    if (M > 0x7FFFFFFF || N > 0x7FFFFFFF) return SHERRY_ERR_UNSUPPORTED;
    if (!aligned(codes, 4) || !aligned(x, 16) || !aligned(out, 4) || (scales && !aligned(scales, 4)))
        return SHERRY_ERR_ALIGN;
    auto encode = encode_fn();
    if (!encode) {
        set_last_error("cuTensorMapEncodeTiled unavailable", cudaErrorNotSupported);
        return SHERRY_ERR_CUDA;
    }
    CUtensorMap tmap;
    const cuuint64_t gdim[2] = {(cuuint64_t)K, (cuuint64_t)M};
    const cuuint64_t gstride[1] = {(cuuint64_t)K};
    const cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)kBN};
    const cuuint32_t estride[2] = {1, 1};
    const CUresult cr = encode(&tmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t *>(x), gdim,
                               gstride, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (cr != CUDA_SUCCESS) {
        set_last_error("cuTensorMapEncodeTiled", cudaErrorInvalidValue);
        return SHERRY_ERR_CUDA;
    }
    // the shared-memory attribute lives in the device's context: set it once
    // per device and context this kernel runs in
    static std::atomic<unsigned long long> attr_ctx[kMaxDevices];
    int dev = 0;
    {
        const cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) {
            set_last_error("sherry_gemm (cudaGetDevice)", e);
            return SHERRY_ERR_CUDA;
        }
    }
    if (dev < 0 || dev >= kMaxDevices) return SHERRY_ERR_UNSUPPORTED;
    const unsigned long long ctx = context_id();
    if (ctx == 0 || attr_ctx[dev].load(std::memory_order_acquire) != ctx) {
        const cudaError_t e = cudaFuncSetAttribute(gemm_kernel<ACC>,
                                                   cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   (int)kSmemBytes);
        if (e != cudaSuccess) {
            set_last_error("sherry_gemm (shared memory attribute)", e);
            return SHERRY_ERR_CUDA;
        }
        attr_ctx[dev].store(context_id(), std::memory_order_release);
    }
    const int64_t tiles = ((N + kBM - 1) / kBM) * ((M + kBN - 1) / kBN);
    if (tiles > 0x7FFFFFFF) return SHERRY_ERR_UNSUPPORTED;
    const int grid = (int)std::min<int64_t>(tiles, sm_count());
    const long long lim = g_wait_limit.load(std::memory_order_relaxed);
    gemm_kernel<ACC><<<grid, kThreads, kSmemBytes, stream>>>(tmap, codes, scales, out, (int)M,
                                                             (int)N, (int)(K / kBK),
                                                             lim > 0 ? lim : kDefaultWaitLimit);
    return launch_status("sherry_gemm");
}

}  // namespace
}  // namespace sherry

extern "C" sherry_status sherry_gemm(const uint32_t *codes, const float *scales, const int8_t *x,
                                     float *y, int64_t M, int64_t N, int64_t K,
                                     sherry_stream_t stream) {
    return sherry::gemm_launch<false>(codes, scales, x, y, M, N, K,
                                      reinterpret_cast<cudaStream_t>(stream));
}

extern "C" sherry_status sherry_gemm_acc(const uint32_t *codes, const int8_t *x, int32_t *acc,
                                         int64_t M, int64_t N, int64_t K, sherry_stream_t stream) {
    return sherry::gemm_launch<true>(codes, nullptr, x, acc, M, N, K,
                                     reinterpret_cast<cudaStream_t>(stream));
}

extern "C" sherry_status sherry_probe_mma_i8(int iters, int *ctas, sherry_stream_t stream) {
    using namespace sherry;
    if (!ctas) return SHERRY_ERR_NULL;
    if (iters < 1) return SHERRY_ERR_SHAPE;
    static std::atomic<unsigned long long> attr_ctx[kMaxDevices];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        set_last_error("sherry_probe_mma_i8 (cudaGetDevice)", e);
        return SHERRY_ERR_CUDA;
    }
    if (dev < 0 || dev >= kMaxDevices) return SHERRY_ERR_UNSUPPORTED;
    const unsigned long long ctx = context_id();
    if (ctx == 0 || attr_ctx[dev].load(std::memory_order_acquire) != ctx) {
        e = cudaFuncSetAttribute(mma_probe_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kProbeSmem);
        if (e != cudaSuccess) {
            set_last_error("sherry_probe_mma_i8 (shared memory attribute)", e);
            return SHERRY_ERR_CUDA;
        }
        attr_ctx[dev].store(context_id(), std::memory_order_release);
    }
    *ctas = sm_count();
    mma_probe_kernel<<<*ctas, kProbeThreads, kProbeSmem, reinterpret_cast<cudaStream_t>(stream)>>>(iters);
    return launch_status("sherry_probe_mma_i8");
}

extern "C" sherry_status sherry_set_wait_limit(int64_t cycles) {
    if (cycles < 0) return SHERRY_ERR_SHAPE;
    sherry::g_wait_limit.store((long long)cycles, std::memory_order_relaxed);
    return SHERRY_OK;
}

extern "C" sherry_status sherry_device_error(void) {
    cudaError_t err = cudaDeviceSynchronize();
    if (err != cudaSuccess) {
        sherry::set_last_error("sherry_device_error (synchronize)", err);
        return SHERRY_ERR_CUDA;
    }
    unsigned int v = 0;
    err = cudaMemcpyFromSymbol(&v, sherry::g_gemm_device_error, sizeof(v));
    if (err != cudaSuccess) {
        sherry::set_last_error("sherry_device_error (read)", err);
        return SHERRY_ERR_CUDA;
    }
    if (v != 0) {
        const unsigned int zero = 0;
        err = cudaMemcpyToSymbol(sherry::g_gemm_device_error, &zero, sizeof(zero));
        if (err != cudaSuccess) {
            sherry::set_last_error("sherry_device_error (clear)", err);
            return SHERRY_ERR_CUDA;
        }
    }
    // the GEMV kernels keep their own word; both are read and cleared
    const sherry_status g = sherry::gemv_device_error();
    if (v == 0) return g;
    return static_cast<sherry_status>(v);
}
