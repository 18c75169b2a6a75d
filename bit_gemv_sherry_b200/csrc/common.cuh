// common.cuh -- internal helpers of libsherry (not part of the public ABI).
//
// Host: argument checks and the thread-local CUDA error text.
// Device: the Sherry tile decode (SWAR over the five words of a 128-weight
// tile), and thin inline-PTX wrappers for mbarriers, bulk tensor copies and
// the tcgen05 tensor-core instructions used by the GEMM.
#pragma once

#include <atomic>
#include <cstdint>
#include <cuda_runtime.h>

#include "sherry.h"

namespace sherry {

// ---------------------------------------------------------------------------
// Host-side helpers
// ---------------------------------------------------------------------------
void set_last_error(const char *what, cudaError_t err);
void set_last_error_text(const char *text);
sherry_status launch_status(const char *what);

inline bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

inline bool valid_k(int64_t K) { return K >= SHERRY_TILE_K && K % SHERRY_TILE_K == 0 && K <= SHERRY_MAX_K; }

// Number of SMs of the current device (cached per device).
int sm_count();

// Identifier of the CUDA context current on this thread, unique over the
// process's lifetime (cuCtxGetId), or 0 if none is current or the driver
// does not provide it.  Per-device set-up that lives in a context (kernel
// attributes, the device address of a module variable) is cached with the
// identifier of the context it was made in and made again when the current
// context differs: a cudaDeviceReset ends the device's primary context, and
// the next one starts with default attributes and a new module image.
unsigned long long context_id();

// Blocks per SM of a kernel launch shape, kept per device with the context
// it was measured in (the shared-memory attribute is set in that context).
struct OccupancyCache {
    std::atomic<unsigned long long> ctx[64];
    std::atomic<int> bps[64];
};

// Reads and clears the error word of the GEMV kernels (after a device sync).
sherry_status gemv_device_error();

// ---------------------------------------------------------------------------
// Tile decode
// ---------------------------------------------------------------------------
// A tile is five words Z0, Z1, S0, S1, S2.  Block j (0..31) has its zero
// position p_j in bits [2*(j/2), 2*(j/2)+1] of Z_(j&1); the r-th kept weight
// of block j has its sign (1 = negative) at bit j of S_r.
//
// The decoder groups the 32 blocks by j mod 4 ("beta") and produces int8x4
// words ("char4") holding position i of four blocks:
//   char4(i, beta, h) byte k' = weight (block 4 (k' + 4 h) + beta, position i)
//                             = K offset 16 k' + 64 h + 4 beta + i within the tile,
// for i, beta in 0..3, h in 0..1 -- 32 char4 per tile.
//
// For a group beta, (Z_(beta&1) >> 2*(beta>>1)) & 0x33333333 puts p of block
// 4k + beta in bits [4k, 4k+1] (k = 0..7).  Bit 4k+2 receives the sign that
// position i of that block would carry if kept ("SG_i", a per-position sign
// plane derived from S0..S2 and the zero positions).  That nibble (p | sign<<2)
// indexes an 8-byte table per position i with a byte permute:
//   T_i[p | s<<2] = 0 if p == i, else (s ? -1 : +1),
// so one PRMT turns four nibbles into four ternary bytes.
struct TileDecoder {
    uint32_t zm[4];   // zero-position nibbles per group beta
    uint32_t sg[4];   // sign plane per position i (bit j = block j)

    __device__ __forceinline__ void load(uint32_t z0, uint32_t z1, uint32_t s0, uint32_t s1,
                                         uint32_t s2) {
        zm[0] = z0 & 0x33333333u;
        zm[1] = z1 & 0x33333333u;
        zm[2] = (z0 >> 2) & 0x33333333u;
        zm[3] = (z1 >> 2) & 0x33333333u;
        // bit-sliced zero positions: lo bit (L) and hi bit (H) of p_j at bit j
        const uint32_t L = (z0 & 0x55555555u) | ((z1 << 1) & 0xAAAAAAAAu);
        const uint32_t H = ((z0 >> 1) & 0x55555555u) | (z1 & 0xAAAAAAAAu);
        // Sign of position i when kept (ranks counted in ascending position):
        //   i = 0: rank 0;  i = 1: rank 0 if p == 0 else rank 1;
        //   i = 2: rank 1 if p <= 1 else rank 2;  i = 3: rank 2.
        sg[0] = s0;
        sg[1] = ((L | H) & s1) | (~(L | H) & s0);
        sg[2] = (H & s2) | (~H & s1);
        sg[3] = s2;
    }

    // Selector word of (position i, group beta): nibble k = p | sign << 2 for
    // block 4k + beta, k = 0..7.  The low half serves h = 0, the high half h = 1.
    __device__ __forceinline__ uint32_t sel(int i, int beta) const {
        uint32_t s = sg[i];
        uint32_t sh;
        switch (beta) {  // move bit 4k+beta to bit 4k+2
            case 0: sh = s << 2; break;
            case 1: sh = s << 1; break;
            case 2: sh = s; break;
            default: sh = s >> 1; break;
        }
        return zm[beta] | (sh & 0x44444444u);
    }
};

// Byte tables T_i (low word = sign 0, high word = sign 1), byte p of each word.
__device__ __forceinline__ uint32_t table_lo(int i) {
    return i == 0 ? 0x01010100u : i == 1 ? 0x01010001u : i == 2 ? 0x01000101u : 0x00010101u;
}
__device__ __forceinline__ uint32_t table_hi(int i) {
    return i == 0 ? 0xFFFFFF00u : i == 1 ? 0xFFFF00FFu : i == 2 ? 0xFF00FFFFu : 0x00FFFFFFu;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// ---------------------------------------------------------------------------
// mbarrier / bulk tensor copy / tcgen05 wrappers (sm_100a)
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile(
        "{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
            smem_u32(bar)),
        "r"(bytes)
        : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait: returns false when the phase does not complete within
// ~`limit_cycles` SM clocks (then SHERRY_ERR_TIMEOUT goes to *err_word and
// *abort is raised for the other roles of the CTA), or when *abort is set.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, volatile int *abort,
                                          unsigned int *err_word,
                                          long long limit_cycles = 4000000000LL) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort) return false;
        if (clock64() - t0 > limit_cycles) {
            *abort = 1;
            atomicCAS(err_word, 0u, (unsigned int)SHERRY_ERR_TIMEOUT);
            return false;
        }
    }
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 2-D tiled bulk tensor copy global -> shared (no multicast), completion on mbarrier.
__device__ __forceinline__ void tma_load_2d(void *dst, const void *tmap, uint64_t *bar, int x,
                                            int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(smem_u32(bar)), "r"(x), "r"(y)
        : "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t *dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc], int8 x int8 -> int32.
__device__ __forceinline__ void umma_i8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                        uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc], int8 x int8 -> int32.  A is M rows in
// tensor-memory lanes 0..M-1, four K-consecutive int8 per 32-bit column.
__device__ __forceinline__ void umma_i8_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                               uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// 1-D bulk copy global -> shared (no multicast), completion on mbarrier.  dst,
// src and bytes are multiples of 16.
__device__ __forceinline__ void bulk_load(uint32_t dst_smem, const void *src, uint32_t bytes,
                                          uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(dst_smem),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}
// Warm L2 with `bytes` bytes from global `src` (16-byte aligned, a multiple of
// 16 bytes).  Nothing reaches the CTA: a later copy reads the data from L2.
__device__ __forceinline__ void bulk_prefetch_l2(const void *src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}
// Arrive on `bar` once all previously issued tcgen05.mma of this thread completed.
__device__ __forceinline__ void umma_commit(uint64_t *bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_u32(bar))
        : "memory");
}

// 32 lanes x 32 bit, 16 consecutive columns: thread t gets lane (base + t).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32"
        " {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}
// 32 lanes x 32 bit, 32 consecutive columns: thread t writes lane (base + t).
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_ld_wait() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor, K-major, 128-byte swizzle: rows of 128 bytes,
// 8-row groups 1024 bytes apart (SBO), LBO unused, version 1 (sm_100).
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t smem_addr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu);        // start address
    d |= static_cast<uint64_t>(1u) << 16;                            // LBO (ignored)
    d |= static_cast<uint64_t>((1024u >> 4) & 0x3FFFu) << 32;        // SBO
    d |= static_cast<uint64_t>(1u) << 46;                            // version
    d |= static_cast<uint64_t>(2u) << 61;                            // SWIZZLE_128B
    return d;
}

}  // namespace sherry
