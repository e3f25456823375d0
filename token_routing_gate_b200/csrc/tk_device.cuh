// Device-side helpers shared by the kernels of libtk_route.so: inline PTX for mbarriers, 1-D
// bulk (TMA) copies, programmatic dependent launch and FP8 conversion, plus the host-side
// launch helper and error bookkeeping. sm_100a only.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "tk_route.h"

namespace tk {

constexpr unsigned kFullMask = 0xffffffffu;

// ------------------------------------------------------------------ host-side error detail
void set_error_detail(const char* fmt, ...);
tk_status fail_arg(const char* fmt, ...);
tk_status check_launch(cudaError_t err, const char* what);

// Launch with programmatic dependent launch allowed. No kernel triggers its dependents early
// (griddepcontrol.launch_dependents): measured on B200, letting the next kernel's CTAs become
// resident while this one still runs slowed the whole step by 15%; with the implicit trigger
// at grid completion the launch latency is still hidden. Every kernel calls pdl_wait() before
// it reads global memory that an earlier stream operation may have written.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

int num_sms();  // SM count of the current device (cached per device)

// Launch shapes (occupancy, shared-memory opt-in) are worked out once per device on the first
// call and cached: current_device() indexes the caches, setup_mutex() serialises their filling.
constexpr int kMaxDevices = 64;
int current_device();
std::mutex& setup_mutex();

// Zeroes the padding rows of an expert-sorted buffer (rows r < offsets[E] with token_of[r] ==
// -1): row_bytes per row, and scale_cols fp32 scales per row when out_scale is given.
cudaError_t launch_pad_zero(const int32_t* offsets, const int32_t* token_of, int E, int64_t rmax,
                            uint8_t* out, int64_t row_bytes, float* out_scale, int scale_cols,
                            int32_t* err_flag, cudaStream_t s);

// ------------------------------------------------------------------ device-side helpers
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void flag_error(int32_t* err_flag, int bits) {
    if (err_flag != nullptr) atomicOr(err_flag, bits);
}

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
                 : "memory");
}

// Makes an initialised mbarrier and earlier shared-memory writes visible to the async proxy.
__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

// Waits for the mbarrier phase with the given parity, for at most `limit_ns` nanoseconds.
// Returns false on timeout (the caller flags TK_DEVERR_TIMEOUT and skips the dependent work).
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  uint64_t limit_ns = 1000000000ull) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_timer_ns() - t0 > limit_ns) return false;
    }
    return true;
}

// 1-D bulk copy global -> shared (TMA engine), completion counted on `bar` in bytes.
// One destination CTA (no cluster broadcast). dst/src 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_load(void* smem_dst, const void* gmem_src, uint32_t bytes,
                                          uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(smem_addr(smem_dst)), "l"(gmem_src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

// L2 policy that marks lines for early eviction: for data that is written (or read) once and
// then not touched again by this kernel or the next, so it goes to DRAM ahead of lines that
// are still live.
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// Explicit evict-normal policy. On B200 a bulk load that carries it ran faster than one with no
// policy operand in every context measured (reduce after dispatch, and reduce back to back).
__device__ __forceinline__ uint64_t l2_policy_evict_normal() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// Evict-last policy: lines kept ahead of evict-normal and evict-first ones.
__device__ __forceinline__ uint64_t l2_policy_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// Policy by number, for the kernels' tuning switches: 0 none, 1 evict-normal, 2 evict-first,
// 3 evict-last.
__device__ __forceinline__ uint64_t l2_policy(int which) {
    return which == 2 ? l2_policy_evict_first()
                      : (which == 3 ? l2_policy_evict_last() : l2_policy_evict_normal());
}

// bulk_load with an L2 cache-policy hint.
__device__ __forceinline__ void bulk_load_hint(void* smem_dst, const void* gmem_src, uint32_t bytes,
                                               uint64_t* bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1], %2, [%3], %4;"
        ::"r"(smem_addr(smem_dst)), "l"(gmem_src), "r"(bytes), "r"(smem_addr(bar)), "l"(policy)
        : "memory");
}

// bulk_store with an L2 cache-policy hint.
__device__ __forceinline__ void bulk_store_hint(void* gmem_dst, const void* smem_src, uint32_t bytes,
                                                uint64_t policy) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group.L2::cache_hint [%0], [%1], %2, %3;"
                 ::"l"(gmem_dst), "r"(smem_addr(smem_src)), "r"(bytes), "l"(policy)
                 : "memory");
}

// 1-D bulk copy shared -> global (TMA engine) in the current bulk async-group.
__device__ __forceinline__ void bulk_store(void* gmem_dst, const void* smem_src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gmem_dst),
                 "r"(smem_addr(smem_src)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void bulk_commit() {
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// Waits until every committed bulk store has finished reading its shared-memory source.
__device__ __forceinline__ void bulk_wait_read_all() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

// Two fp32 values -> two E4M3 codes (round to nearest even, saturating at +-448); `lo` lands
// in the low byte.
__device__ __forceinline__ uint16_t cvt_e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

__device__ __forceinline__ void st_v4(void* p, uint4 v) {
    asm volatile("st.global.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w)
                 : "memory");
}

// 16-byte store with an L2 cache-policy hint.
__device__ __forceinline__ void st_v4_hint(void* p, uint4 v, uint64_t policy) {
    asm volatile("st.global.L2::cache_hint.v4.u32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(p), "r"(v.x),
                 "r"(v.y), "r"(v.z), "r"(v.w), "l"(policy)
                 : "memory");
}

}  // namespace tk
