// Host-side bookkeeping shared by the C ABI entry points: status names, the per-thread error
// detail, and the cached SM count used to size persistent grids.
#include <cuda_runtime.h>
#include <stdarg.h>
#include <stdio.h>

#include "tk_device.cuh"

namespace tk {
namespace {
thread_local char g_detail[512] = "";
}

void set_error_detail(const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_detail, sizeof(g_detail), fmt, ap);
    va_end(ap);
}

tk_status fail_arg(const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_detail, sizeof(g_detail), fmt, ap);
    va_end(ap);
    return TK_ERR_INVALID_ARG;
}

tk_status check_launch(cudaError_t err, const char* what) {
    if (err == cudaSuccess) return TK_OK;
    set_error_detail("%s: %s (%s)", what, cudaGetErrorName(err), cudaGetErrorString(err));
    return TK_ERR_CUDA;
}

int num_sms() {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
    if (cached[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) n = 1;
        cached[dev] = n;
    }
    return cached[dev];
}

}  // namespace tk

extern "C" const char* tk_status_str(int status) {
    switch (status) {
        case TK_OK: return "TK_OK";
        case TK_ERR_INVALID_ARG: return "TK_ERR_INVALID_ARG";
        case TK_ERR_CUDA: return "TK_ERR_CUDA";
        default: return "TK_STATUS_UNKNOWN";
    }
}

extern "C" const char* tk_last_error_detail(void) { return tk::g_detail; }

extern "C" int tk_abi_version(void) { return (1 << 16) | 0; }
