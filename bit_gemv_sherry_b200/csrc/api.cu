// api.cu -- shared host utilities of libsherry: status strings, the last CUDA
// error text, the device error word, and the packed-size query.
#include <cuda.h>

#include <cstdio>
#include <cstring>

#include "common.cuh"

namespace sherry {

namespace {
thread_local char g_last_error[256] = "";
}

void set_last_error(const char *what, cudaError_t err) {
    std::snprintf(g_last_error, sizeof(g_last_error), "%s: %s (%s)", what, cudaGetErrorName(err),
                  cudaGetErrorString(err));
}

void set_last_error_text(const char *text) {
    std::snprintf(g_last_error, sizeof(g_last_error), "%s", text);
}

sherry_status launch_status(const char *what) {
    const cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) {
        set_last_error(what, err);
        return SHERRY_ERR_CUDA;
    }
    return SHERRY_OK;
}

namespace {
void *driver_entry(const char *name) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
        return nullptr;
    return p;
}
}  // namespace

unsigned long long context_id() {
    using GetCurrentFn = CUresult (*)(CUcontext *);
    using GetIdFn = CUresult (*)(CUcontext, unsigned long long *);
    static const GetCurrentFn get_current =
        reinterpret_cast<GetCurrentFn>(driver_entry("cuCtxGetCurrent"));
    static const GetIdFn get_id = reinterpret_cast<GetIdFn>(driver_entry("cuCtxGetId"));
    if (!get_current || !get_id) return 0;
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr || get_id(ctx, &id) != CUDA_SUCCESS)
        return 0;
    return id;
}

int sm_count() {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    int &c = cached[dev & 63];
    if (c == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1)
            n = 148;
        c = n;
    }
    return c;
}

}  // namespace sherry

extern "C" size_t sherry_packed_bytes(int64_t N, int64_t K) {
    if (N < 1 || K < SHERRY_TILE_K || K % SHERRY_TILE_K) return 0;
    const size_t rows = (size_t)((N + SHERRY_ROW_GROUP - 1) / SHERRY_ROW_GROUP) * SHERRY_ROW_GROUP;
    return rows * (size_t)(K / SHERRY_TILE_K) * SHERRY_WORDS_PER_TILE * 4;
}

extern "C" const char *sherry_status_string(sherry_status s) {
    switch (s) {
        case SHERRY_OK: return "ok";
        case SHERRY_ERR_NULL: return "a required pointer is NULL";
        case SHERRY_ERR_SHAPE: return "invalid shape (N, M, B >= 1; K a multiple of 128, <= 131072)";
        case SHERRY_ERR_ALIGN: return "a pointer is not aligned as required";
        case SHERRY_ERR_UNSUPPORTED: return "size not supported by the kernels";
        case SHERRY_ERR_CUDA: return "CUDA error (see sherry_last_error)";
        case SHERRY_ERR_TIMEOUT: return "a bounded device-side wait timed out";
        case SHERRY_ERR_WORKSPACE: return "workspace missing or too small";
    }
    return "unknown status";
}

extern "C" const char *sherry_last_error(void) { return sherry::g_last_error; }

extern "C" int sherry_version(void) { return 100; }
