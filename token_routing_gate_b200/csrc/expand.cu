// Fused expand / dispatch: every token row goes to its k slots of the expert-sorted buffer
// (147227.xyz "刚刚！DeepSeek开源高性能GPU算子库TileKernels", section "moe/": fused expand),
// optionally quantised on the way to per-token, per-128-channel FP8 E4M3 (the quant/ module's
// per-token granularity in section "quant/"; FP8 dispatch in 機器之心 "性能表現").
//
// The pages describe TileLang kernels for SM90 and give no kernel design; this one is built
// for B200's bulk-copy (TMA) engine. The path is pure bandwidth (one read of x, k writes), so
// no tensor core is involved. One CTA per token:
//   bf16 : one elected thread bulk-loads the token row into shared memory (mbarrier with
//          transaction count) and issues k bulk stores of it to the k slots; the threads do no
//          data movement at all. Rows longer than 32 KB are moved in 32 KB pieces.
//   E4M3 : the row is bulk-loaded, each warp quantises 128-channel blocks (amax by warp
//          reduction, scale = amax/448, code = cvt.rn.satfinite.e4m3x2(x/scale) with IEEE
//          division), writes codes to shared memory, and the elected thread bulk-stores the
//          code row to the k slots; scales go out as plain stores.
// The k copies are stored with an L2 evict-first policy: nothing reads them again before they
// reach DRAM, and without the hint they stay dirty in L2 and are written back while the next
// kernel runs.
// Padding rows (only when segments are aligned to more than one row) are zeroed by a separate
// small kernel that scans token_of for -1 below offsets[E] and bulk-stores zeros over them.
#include <cuda_runtime.h>
#include <stdint.h>

#include "quant_e4m3.cuh"
#include "tk_device.cuh"

namespace tk {
namespace {

#ifndef TK_EXPAND_STORE_POLICY   // L2 policy of the k stores: 0 none, 1 evict-normal, 2 evict-first, 3 evict-last
#define TK_EXPAND_STORE_POLICY 2
#endif

constexpr uint32_t kCopyChunkBytes = 32768;  // bf16 bytes staged per bulk load

#ifndef TK_EXPAND_WIDE_ROW_CTAS_PER_SM  // resident CTAs per SM for rows of 8 KB or more (0: all that fit)
#define TK_EXPAND_WIDE_ROW_CTAS_PER_SM 8
#endif
#ifndef TK_EXPAND_LOAD_POLICY   // L2 policy of the token-row loads: 0 none, 1 evict-normal, 2 evict-first
#define TK_EXPAND_LOAD_POLICY 0
#endif

__device__ __forceinline__ void load_copy(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    if (TK_EXPAND_LOAD_POLICY != 0) bulk_load_hint(dst, src, bytes, bar, l2_policy(TK_EXPAND_LOAD_POLICY));
    else bulk_load(dst, src, bytes, bar);
}

__device__ __forceinline__ void store_copy(void* dst, const void* src, uint32_t bytes, uint64_t policy) {
    if (TK_EXPAND_STORE_POLICY != 0) bulk_store_hint(dst, src, bytes, policy);
    else bulk_store(dst, src, bytes);
}
constexpr int kFp8Threads = 256;
constexpr int kFp8ChunkChannels = 8192;      // channels quantised per stage

__global__ void __launch_bounds__(32)
expand_bf16_kernel(const uint8_t* __restrict__ x, const int32_t* __restrict__ slot_of, int k,
                   uint32_t row_bytes, int64_t rmax, uint8_t* __restrict__ out,
                   int32_t* err_flag) {
    extern __shared__ __align__(128) uint8_t stage[];
    __shared__ __align__(8) uint64_t bar;
    const int lane = threadIdx.x;
    const int64_t t = blockIdx.x;
    if (lane == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    __syncwarp();
    pdl_wait();
    int64_t my_slot = -1;
    if (lane < k) {
        const int64_t s = slot_of[t * k + lane];
        if (s >= 0 && s < rmax) my_slot = s;
        else if (s != -1) flag_error(err_flag, TK_DEVERR_SLOT_RANGE);
    }
    const uint8_t* src = x + t * row_bytes;
    const uint32_t nchunks = (row_bytes + kCopyChunkBytes - 1) / kCopyChunkBytes;
    const uint64_t policy = l2_policy(TK_EXPAND_STORE_POLICY);
    for (uint32_t c = 0; c < nchunks; ++c) {
        const uint32_t off = c * kCopyChunkBytes;
        const uint32_t bytes = min(kCopyChunkBytes, row_bytes - off);
        int ok = 1;
        if (lane == 0) {
            if (c > 0) {
                bulk_wait_read_all();      // previous piece fully read by its stores
                fence_proxy_async_smem();
            }
            mbar_arrive_expect_tx(&bar, bytes);
            load_copy(stage, src + off, bytes, &bar);
            ok = mbar_wait_bounded(&bar, c & 1u) ? 1 : 0;
            if (!ok) {
                flag_error(err_flag, TK_DEVERR_TIMEOUT);
                mbar_wait_bounded(&bar, c & 1u);  // give the copy in flight a second chance
            }
        }
        ok = __shfl_sync(kFullMask, ok, 0);
        if (!ok) break;
        for (int j = 0; j < k; ++j) {
            const int64_t s = __shfl_sync(kFullMask, my_slot, j);
            if (lane == 0 && s >= 0) store_copy(out + s * row_bytes + off, stage, bytes, policy);
        }
        if (lane == 0) bulk_commit();
    }
    if (lane == 0) bulk_wait_read_all();
}

__global__ void __launch_bounds__(kFp8Threads)
expand_fp8_kernel(const uint16_t* __restrict__ x, const int32_t* __restrict__ slot_of, int k,
                  int H, int64_t rmax, uint8_t* __restrict__ out_q, float* __restrict__ out_scale,
                  int32_t* err_flag) {
    extern __shared__ __align__(128) uint8_t sm[];
    const int chunk = min(H, kFp8ChunkChannels);
    uint16_t* xin = reinterpret_cast<uint16_t*>(sm);                       // [chunk] bf16
    uint8_t* qo = sm + static_cast<size_t>(chunk) * 2;                      // [chunk] E4M3
    float* sc = reinterpret_cast<float*>(sm + static_cast<size_t>(chunk) * 3);  // [chunk/128]
    __shared__ __align__(8) uint64_t bar;
    __shared__ int64_t slots[TK_MAX_TOPK];
    __shared__ int load_ok;
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int64_t t = blockIdx.x;
    if (tid == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    __syncthreads();
    pdl_wait();
    if (tid < k) {
        const int64_t s = slot_of[t * k + tid];
        int64_t v = -1;
        if (s >= 0 && s < rmax) v = s;
        else if (s != -1) flag_error(err_flag, TK_DEVERR_SLOT_RANGE);
        slots[tid] = v;
    }
    const int nb_row = H / 128;
    const int nchunks = (H + chunk - 1) / chunk;
    const uint64_t policy = l2_policy(TK_EXPAND_STORE_POLICY);
    for (int c = 0; c < nchunks; ++c) {
        const int ch0 = c * chunk;
        const int chn = min(chunk, H - ch0);
        if (tid == 0) {
            if (c > 0) bulk_wait_read_all();
            fence_proxy_async_smem();
            mbar_arrive_expect_tx(&bar, static_cast<uint32_t>(chn) * 2u);
            load_copy(xin, x + t * H + ch0, static_cast<uint32_t>(chn) * 2u, &bar);
            int ok = mbar_wait_bounded(&bar, static_cast<uint32_t>(c) & 1u) ? 1 : 0;
            if (!ok) {
                flag_error(err_flag, TK_DEVERR_TIMEOUT);
                mbar_wait_bounded(&bar, static_cast<uint32_t>(c) & 1u);
            }
            load_ok = ok;
        }
        __syncthreads();
        if (!load_ok) break;
        const int nb = chn / 128;
        for (int b = warp; b < nb; b += kFp8Threads / 32) {
            const float scale = quantize_block_e4m3(xin + b * 128, qo + b * 128, lane);
            if (lane == 0) sc[b] = scale;
        }
        fence_proxy_async_smem();
        __syncthreads();
        if (tid == 0) {
            for (int j = 0; j < k; ++j) {
                const int64_t s = slots[j];
                if (s >= 0) store_copy(out_q + s * H + ch0, qo, static_cast<uint32_t>(chn), policy);
            }
            bulk_commit();
        }
        const int b0 = ch0 / 128;
        for (int i = tid; i < k * nb; i += kFp8Threads) {
            const int j = i / nb;
            const int b = i - j * nb;
            const int64_t s = slots[j];
            if (s >= 0) out_scale[s * nb_row + b0 + b] = sc[b];
        }
        __syncthreads();
    }
    if (tid == 0) bulk_wait_read_all();
}

}  // namespace
}  // namespace tk

namespace tk {
namespace {

// Shared memory reserved per bf16 expand CTA: its row stage, raised for rows of 8 KB or more so
// that TK_EXPAND_WIDE_ROW_CTAS_PER_SM CTAs are resident per SM instead of all that fit (15 with
// 14 KB rows). On three B200s, 8 CTAs took expand from 168-171.6 to 165.8-168.6 us and the
// serial routing step 2.5-3.6 us lower at T=8192, H=7168; 4 KB rows lost 5 % with fewer CTAs.
uint32_t expand_smem_reserve(uint32_t stage) {
    if (TK_EXPAND_WIDE_ROW_CTAS_PER_SM <= 0 || stage < 8192) return stage;
    static std::atomic<int> smem_per_sm[kMaxDevices];
    const int dev = current_device();
    int per_sm = smem_per_sm[dev].load(std::memory_order_acquire);
    if (per_sm == 0) {
        if (cudaDeviceGetAttribute(&per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) != cudaSuccess ||
            per_sm < 1)
            per_sm = -1;
        smem_per_sm[dev].store(per_sm, std::memory_order_release);
    }
    if (per_sm < 0) return stage;
    // the runtime keeps 1 KB per resident CTA, and the kernel has a little static shared memory
    int64_t reserve = per_sm / TK_EXPAND_WIDE_ROW_CTAS_PER_SM - 2048;
    if (reserve > 47 * 1024) reserve = 47 * 1024;  // dynamic + static stay within the default 48 KB
    return reserve > static_cast<int64_t>(stage) ? static_cast<uint32_t>(reserve) : stage;
}

}  // namespace
}  // namespace tk

extern "C" tk_status tk_expand(const void* x, const int32_t* slot_of, const int32_t* offsets,
                               const int32_t* token_of, int T, int E, int k, int H, int align,
                               int out_dtype, void* out, float* out_scale, int32_t* err_flag,
                               void* stream) {
    using namespace tk;
    if (T < 0) return fail_arg("tk_expand: T=%d must be >= 0", T);
    if (E < 1 || E > TK_MAX_EXPERTS) return fail_arg("tk_expand: E=%d outside [1, %d]", E, TK_MAX_EXPERTS);
    if (k < 1 || k > TK_MAX_TOPK) return fail_arg("tk_expand: k=%d outside [1, %d]", k, TK_MAX_TOPK);
    if (align < 1 || align > 4096) return fail_arg("tk_expand: align=%d outside [1, 4096]", align);
    if (out_dtype != TK_OUT_BF16 && out_dtype != TK_OUT_FP8_E4M3)
        return fail_arg("tk_expand: unknown out_dtype %d", out_dtype);
    if (H < 8 || H % 8 != 0) return fail_arg("tk_expand: H=%d must be a positive multiple of 8", H);
    if (out_dtype == TK_OUT_FP8_E4M3 && H % 128 != 0)
        return fail_arg("tk_expand: H=%d must be a multiple of 128 for E4M3 output", H);
    if (static_cast<int64_t>(H) * 2 > INT32_MAX) return fail_arg("tk_expand: H too large");
    const int64_t rmax = tk_max_rows(T, E, k, align);
    if (rmax > INT32_MAX) return fail_arg("tk_expand: T*k + E*(align-1) exceeds int32");
    if (T == 0) return TK_OK;
    if (x == nullptr || slot_of == nullptr || offsets == nullptr || out == nullptr)
        return fail_arg("tk_expand: x, slot_of, offsets and out must not be NULL");
    if (align > 1 && token_of == nullptr) return fail_arg("tk_expand: token_of is needed when align > 1");
    if (out_dtype == TK_OUT_FP8_E4M3 && out_scale == nullptr)
        return fail_arg("tk_expand: out_scale must not be NULL for E4M3 output");
    if (reinterpret_cast<uintptr_t>(x) % 16 != 0 || reinterpret_cast<uintptr_t>(out) % 16 != 0)
        return fail_arg("tk_expand: x and out must be 16-byte aligned");
    if (out_scale != nullptr && reinterpret_cast<uintptr_t>(out_scale) % 4 != 0)
        return fail_arg("tk_expand: out_scale must be 4-byte aligned");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t err;
    if (out_dtype == TK_OUT_BF16) {
        const uint32_t row_bytes = static_cast<uint32_t>(H) * 2u;
        const uint32_t stage = row_bytes < kCopyChunkBytes ? row_bytes : kCopyChunkBytes;
        err = launch_pdl(expand_bf16_kernel, dim3(T), dim3(32), expand_smem_reserve(stage), s,
                         static_cast<const uint8_t*>(x), slot_of, k, row_bytes, rmax,
                         static_cast<uint8_t*>(out), err_flag);
        if (err != cudaSuccess) return check_launch(err, "expand_bf16_kernel");
    } else {
        const int chunk = H < kFp8ChunkChannels ? H : kFp8ChunkChannels;
        const size_t smem = static_cast<size_t>(chunk) * 3 + static_cast<size_t>(chunk / 128) * 4;
        err = launch_pdl(expand_fp8_kernel, dim3(T), dim3(kFp8Threads), smem, s,
                         static_cast<const uint16_t*>(x), slot_of, k, H, rmax,
                         static_cast<uint8_t*>(out), out_scale, err_flag);
        if (err != cudaSuccess) return check_launch(err, "expand_fp8_kernel");
    }
    if (align > 1) {
        const bool fp8 = out_dtype == TK_OUT_FP8_E4M3;
        err = launch_pad_zero(offsets, token_of, E, rmax, static_cast<uint8_t*>(out),
                              fp8 ? H : static_cast<int64_t>(H) * 2,
                              fp8 ? out_scale : static_cast<float*>(nullptr), fp8 ? H / 128 : 0,
                              err_flag, s);
        if (err != cudaSuccess) return check_launch(err, "expand_pad_kernel");
    }
    return TK_OK;
}
