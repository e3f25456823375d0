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

int current_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) dev = 0;
    return dev;
}

std::mutex& setup_mutex() {
    static std::mutex m;
    return m;
}

int num_sms() {
    static std::atomic<int> cached[kMaxDevices];
    const int dev = current_device();
    int n = cached[dev].load(std::memory_order_acquire);
    if (n == 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) n = 1;
        cached[dev].store(n, std::memory_order_release);
    }
    return n;
}

namespace {

// Waits on an mbarrier that nothing ever arrives on, with the library's bounded wait: the wait
// must give up after limit_ns, flag TK_DEVERR_TIMEOUT and let the kernel return normally.
__global__ void bounded_wait_selftest_kernel(uint64_t limit_ns, int32_t* err_flag) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    __syncthreads();
    if (!mbar_wait_bounded(&bar, 0, limit_ns)) {
        if (threadIdx.x == 0) flag_error(err_flag, TK_DEVERR_TIMEOUT);
    }
}

}  // namespace
}  // namespace tk

extern "C" tk_status tk_selftest_bounded_wait(int64_t limit_ns, int32_t* err_flag, void* stream) {
    using namespace tk;
    if (limit_ns < 1 || limit_ns > INT64_C(2000000000))
        return fail_arg("tk_selftest_bounded_wait: limit_ns=%lld outside [1, 2e9]", (long long)limit_ns);
    if (err_flag == nullptr) return fail_arg("tk_selftest_bounded_wait: err_flag must not be NULL");
    const cudaError_t err = launch_pdl(bounded_wait_selftest_kernel, dim3(1), dim3(32), 0,
                                       static_cast<cudaStream_t>(stream),
                                       static_cast<uint64_t>(limit_ns), err_flag);
    return check_launch(err, "bounded_wait_selftest_kernel");
}

extern "C" const char* tk_status_str(int status) {
    switch (status) {
        case TK_OK: return "TK_OK";
        case TK_ERR_INVALID_ARG: return "TK_ERR_INVALID_ARG";
        case TK_ERR_CUDA: return "TK_ERR_CUDA";
        default: return "TK_STATUS_UNKNOWN";
    }
}

extern "C" const char* tk_last_error_detail(void) { return tk::g_detail; }

extern "C" int tk_abi_version(void) { return (1 << 16) | 3; }
