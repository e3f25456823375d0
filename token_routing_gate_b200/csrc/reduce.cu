// Fused reduce / combine: out[t] = bf16( sum_j w[t,j] * y[slot_of[t,j]] ), fp32 accumulation
// in slot order j = 0..k-1, one fmaf per term (147227.xyz "刚刚！DeepSeek开源高性能GPU算子库
// TileKernels", section "moe/": fused reduce; BF16 combine in 機器之心 "性能表現").
//
// Pure bandwidth: k scattered 2H-byte rows read, one 2H-byte row written per token. Work unit =
// one warp x (token, 64 consecutive 8-channel vectors); each lane owns two vectors 32 apart,
// so every load instruction of the warp covers 512 contiguous bytes of one row. A lane issues
// all its loads for up to 8 rows (16 x 16 bytes in flight) before the first FMA, which keeps
// enough bytes in flight per SM to cover HBM latency. The grid is persistent (a few CTAs per
// SM, sized by the occupancy calculator) and strides over units.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "tk_device.cuh"

namespace tk {
namespace {

constexpr int kRedThreads = 256;
constexpr int kRedWarps = kRedThreads / 32;
constexpr int kU = 2;    // 8-channel vectors per lane per unit
constexpr int kKC = 8;   // rows whose loads are issued together

__device__ __forceinline__ float lo_bf16(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float hi_bf16(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const uint32_t l = static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(lo)));
    const uint32_t h = static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(hi)));
    return l | (h << 16);
}

__global__ void __launch_bounds__(kRedThreads)
reduce_kernel(const uint8_t* __restrict__ y, int64_t y_rows, const int32_t* __restrict__ slot_of,
              const float* __restrict__ w, int T, int k, int H, uint8_t* __restrict__ out,
              int32_t* err_flag) {
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const int V = H / 8;                                 // 16-byte vectors per row
    const int units_per_token = (V + 32 * kU - 1) / (32 * kU);
    const int64_t total_units = static_cast<int64_t>(T) * units_per_token;
    const int64_t row_bytes = static_cast<int64_t>(H) * 2;
    for (int64_t unit = static_cast<int64_t>(blockIdx.x) * kRedWarps + (threadIdx.x >> 5);
         unit < total_units; unit += static_cast<int64_t>(gridDim.x) * kRedWarps) {
        const int64_t t = unit / units_per_token;
        const int vbase = static_cast<int>(unit - t * units_per_token) * (32 * kU);
        int64_t my_slot = -1;
        float my_w = 1.0f;
        if (lane < k) {
            const int64_t s = slot_of[t * k + lane];
            if (s >= 0 && s < y_rows) my_slot = s;
            else if (s != -1) flag_error(err_flag, TK_DEVERR_SLOT_RANGE);
            if (w != nullptr) my_w = w[t * k + lane];
        }
        float acc[kU][8];
#pragma unroll
        for (int u = 0; u < kU; ++u)
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[u][e] = 0.0f;
        bool vec_ok[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) vec_ok[u] = vbase + u * 32 + lane < V;

        for (int j0 = 0; j0 < k; j0 += kKC) {
            uint4 v[kKC][kU];
            int64_t sl[kKC];
#pragma unroll
            for (int jj = 0; jj < kKC; ++jj) {
                sl[jj] = __shfl_sync(kFullMask, my_slot, (j0 + jj) & 31);
                const bool live = (j0 + jj < k) && sl[jj] >= 0;
#pragma unroll
                for (int u = 0; u < kU; ++u) {
                    v[jj][u] = make_uint4(0u, 0u, 0u, 0u);
                    if (live && vec_ok[u])
                        v[jj][u] = ld_stream_v4(y + sl[jj] * row_bytes +
                                                static_cast<int64_t>(vbase + u * 32 + lane) * 16);
                }
            }
#pragma unroll
            for (int jj = 0; jj < kKC; ++jj) {
                const float wj = __shfl_sync(kFullMask, my_w, (j0 + jj) & 31);
                if (j0 + jj < k && sl[jj] >= 0) {
#pragma unroll
                    for (int u = 0; u < kU; ++u) {
                        const uint4 q = v[jj][u];
                        acc[u][0] = __fmaf_rn(wj, lo_bf16(q.x), acc[u][0]);
                        acc[u][1] = __fmaf_rn(wj, hi_bf16(q.x), acc[u][1]);
                        acc[u][2] = __fmaf_rn(wj, lo_bf16(q.y), acc[u][2]);
                        acc[u][3] = __fmaf_rn(wj, hi_bf16(q.y), acc[u][3]);
                        acc[u][4] = __fmaf_rn(wj, lo_bf16(q.z), acc[u][4]);
                        acc[u][5] = __fmaf_rn(wj, hi_bf16(q.z), acc[u][5]);
                        acc[u][6] = __fmaf_rn(wj, lo_bf16(q.w), acc[u][6]);
                        acc[u][7] = __fmaf_rn(wj, hi_bf16(q.w), acc[u][7]);
                    }
                }
            }
        }
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            if (!vec_ok[u]) continue;
            uint4 o;
            o.x = pack_bf16x2(acc[u][0], acc[u][1]);
            o.y = pack_bf16x2(acc[u][2], acc[u][3]);
            o.z = pack_bf16x2(acc[u][4], acc[u][5]);
            o.w = pack_bf16x2(acc[u][6], acc[u][7]);
            st_v4(out + t * row_bytes + static_cast<int64_t>(vbase + u * 32 + lane) * 16, o);
        }
    }
}

int reduce_grid(int64_t total_units) {
    static int blocks_per_sm = 0;
    if (blocks_per_sm == 0) {
        int b = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, reduce_kernel, kRedThreads, 0) != cudaSuccess || b < 1) b = 1;
        blocks_per_sm = b;
    }
    const int64_t want = (total_units + kRedWarps - 1) / kRedWarps;
    const int64_t cap = static_cast<int64_t>(num_sms()) * blocks_per_sm;
    return static_cast<int>(want < cap ? want : cap);
}

}  // namespace
}  // namespace tk

extern "C" tk_status tk_reduce(const void* y, int64_t y_rows, const int32_t* slot_of, const float* w,
                               int T, int k, int H, void* out, int32_t* err_flag, void* stream) {
    using namespace tk;
    if (T < 0) return fail_arg("tk_reduce: T=%d must be >= 0", T);
    if (k < 1 || k > TK_MAX_TOPK) return fail_arg("tk_reduce: k=%d outside [1, %d]", k, TK_MAX_TOPK);
    if (H < 8 || H % 8 != 0) return fail_arg("tk_reduce: H=%d must be a positive multiple of 8", H);
    if (y_rows < 0) return fail_arg("tk_reduce: y_rows=%lld must be >= 0", (long long)y_rows);
    if (T == 0) return TK_OK;
    if (slot_of == nullptr || out == nullptr || (y == nullptr && y_rows > 0))
        return fail_arg("tk_reduce: y, slot_of and out must not be NULL");
    if (reinterpret_cast<uintptr_t>(y) % 16 != 0 || reinterpret_cast<uintptr_t>(out) % 16 != 0)
        return fail_arg("tk_reduce: y and out must be 16-byte aligned");
    const int V = H / 8;
    const int64_t units = static_cast<int64_t>(T) * ((V + 32 * kU - 1) / (32 * kU));
    const int grid = reduce_grid(units);
    cudaError_t err = launch_pdl(reduce_kernel, dim3(grid), dim3(kRedThreads), 0,
                                 static_cast<cudaStream_t>(stream), static_cast<const uint8_t*>(y),
                                 y_rows, slot_of, w, T, k, H, static_cast<uint8_t*>(out), err_flag);
    return check_launch(err, "reduce_kernel");
}
