// Backward of the fused expand / reduce (the training use of these ops; TileKernels is
// described as training and inference kernels, m.yhxrc.cn "剛剛，DeepSeek 悶聲開源", section
// "簡介"). The forward reduce out[t] = sum_j w[t,j] * y[slot_of[t,j]] is linear in y and w:
//   d_y[slot_of[t,j]] = bf16(w[t,j] * g[t])        d_w[t,j] = <g[t], y[slot_of[t,j]]>
// and the backward of expand (a copy of row t to k slots) is the unweighted reduce of the
// gradient rows, which tk_expand_backward runs with the reduce kernel.
//
// reduce_backward_kernel: warp-specialised like the forward reduce. A unit is (token t, 1024-
// channel chunk c); a CTA takes whole tokens (t = blockIdx.x, += gridDim.x) and their chunks in
// order. Warp 0 bulk-loads the chunk of g and the k chunks of y into a stage of a shared ring;
// consumer warps write 16 bytes of d_y per row and add the chunk's partial dot products (exact
// bf16 x bf16 products summed in double) into per-warp accumulators, which each warp writes out
// at the token's last chunk. dw_combine_kernel then adds the four per-warp sums of every pair in
// a fixed order, so d_w is deterministic.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <initializer_list>

#include "tk_device.cuh"

namespace tk {
namespace {

constexpr int kConsumerWarps = 4;
constexpr int kBwdThreads = 32 * (1 + kConsumerWarps);
constexpr int kChunkCh = 8 * 32 * kConsumerWarps;  // channels per unit, one vector per thread
constexpr int kChunkBytes = kChunkCh * 2;
#ifndef TK_BACKWARD_STAGE_KB
#define TK_BACKWARD_STAGE_KB 40
#endif
#ifndef TK_BACKWARD_STORE_EVICT_FIRST   // d_y rows are written once and not read here
#define TK_BACKWARD_STORE_EVICT_FIRST 1
#endif
constexpr int kStageBudget = TK_BACKWARD_STAGE_KB * 1024;
constexpr int kRegRows = 8;  // up to this k, per-thread register accumulators for d_w

#ifndef TK_BACKWARD_CTAS_PER_SM  // resident CTAs per SM at most (0: as many as fit)
#define TK_BACKWARD_CTAS_PER_SM 3
#endif
#ifndef TK_BACKWARD_LOAD_POLICY   // L2 policy of the row loads: 0 none, 1 evict-normal, 2 evict-first
#define TK_BACKWARD_LOAD_POLICY 1
#endif

__device__ __forceinline__ void store_dy(void* p, uint4 v) {
    if (TK_BACKWARD_STORE_EVICT_FIRST) st_v4_hint(p, v, l2_policy_evict_first());
    else st_v4(p, v);
}

__device__ __forceinline__ void load_row(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    if (TK_BACKWARD_LOAD_POLICY != 0) bulk_load_hint(dst, src, bytes, bar, l2_policy(TK_BACKWARD_LOAD_POLICY));
    else bulk_load(dst, src, bytes, bar);
}

struct StageMeta {
    float w[TK_MAX_TOPK];
    int32_t slot[TK_MAX_TOPK];  // -1: skip this row
};

__device__ __forceinline__ float lo_bf16(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float hi_bf16(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const uint32_t l = static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(lo)));
    const uint32_t h = static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(hi)));
    return l | (h << 16);
}

int stages_for(int k) {
    int s = kStageBudget / ((k + 1) * kChunkBytes);
    return s < 1 ? 1 : (s > 8 ? 8 : s);
}

size_t smem_bytes(int k, int S) {
    return static_cast<size_t>(S) * (k + 1) * kChunkBytes + static_cast<size_t>(S) * sizeof(StageMeta) +
           static_cast<size_t>(2 * S) * sizeof(uint64_t) +
           static_cast<size_t>(kConsumerWarps) * TK_MAX_TOPK * sizeof(double);
}

__global__ void __launch_bounds__(kBwdThreads)
reduce_backward_kernel(const uint8_t* __restrict__ g, const uint8_t* __restrict__ y, int64_t y_rows,
                       const int32_t* __restrict__ slot_of, const float* __restrict__ w, int T,
                       int k, int H, int S, uint8_t* __restrict__ d_y,
                       double* __restrict__ dw_part, int32_t* err_flag) {
    extern __shared__ __align__(128) uint8_t sm[];
    const int stage_bytes = (k + 1) * kChunkBytes;
    uint8_t* data = sm;
    StageMeta* meta = reinterpret_cast<StageMeta*>(sm + static_cast<size_t>(S) * stage_bytes);
    uint64_t* full = reinterpret_cast<uint64_t*>(meta + S);
    uint64_t* empty = full + S;
    double* dacc = reinterpret_cast<double*>(empty + S);  // [kConsumerWarps][TK_MAX_TOPK]
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
        fence_barrier_init();
    }
    for (int i = threadIdx.x; i < kConsumerWarps * TK_MAX_TOPK; i += blockDim.x) dacc[i] = 0.0;
    __syncthreads();
    pdl_wait();

    const int chunks = (H + kChunkCh - 1) / kChunkCh;
    const int64_t row_bytes = static_cast<int64_t>(H) * 2;

    if (warp == 0) {
        // ---------------- producer
        int it = 0;
        for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
            int64_t sl = -1;
            float wl = 1.0f;
            if (lane < k) {
                const int64_t v = slot_of[t * k + lane];
                if (v >= 0 && v < y_rows) sl = v;
                else if (v != -1) flag_error(err_flag, TK_DEVERR_SLOT_RANGE);
                if (w != nullptr) wl = w[t * k + lane];
            }
            const unsigned vmask = __ballot_sync(kFullMask, sl >= 0);
            for (int c = 0; c < chunks; ++c, ++it) {
                const int s = it % S;
                const uint32_t ph = static_cast<uint32_t>(it / S) & 1u;
                const int ch0 = c * kChunkCh;
                const uint32_t bytes = static_cast<uint32_t>(min(kChunkCh, H - ch0)) * 2u;
                int ok = 1;
                if (lane == 0) ok = mbar_wait_bounded(&empty[s], ph ^ 1u) ? 1 : 0;
                ok = __shfl_sync(kFullMask, ok, 0);
                if (!ok) {
                    if (lane == 0) flag_error(err_flag, TK_DEVERR_TIMEOUT);
                    return;
                }
                if (lane < k) {
                    meta[s].w[lane] = wl;
                    meta[s].slot[lane] = static_cast<int32_t>(sl);
                }
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(1 + __popc(vmask)) * bytes);
                    load_row(data + static_cast<size_t>(s) * stage_bytes, g + t * row_bytes + ch0 * 2,
                             bytes, &full[s]);
                }
                __syncwarp();
                if (sl >= 0)
                    load_row(data + static_cast<size_t>(s) * stage_bytes + static_cast<size_t>(1 + lane) * kChunkBytes,
                             y + sl * row_bytes + static_cast<int64_t>(ch0) * 2, bytes, &full[s]);
            }
        }
    } else {
        // ---------------- consumers
        const int ct = threadIdx.x - 32;
        const int cw = warp - 1;
        // k <= 8: each thread keeps its partial dot product of every row in registers for the
        // whole token and the warp reduces once per token; larger k reduces every chunk into
        // per-warp shared accumulators.
        const bool reg_acc = k <= kRegRows;
        double accd[kRegRows];
#pragma unroll
        for (int j = 0; j < kRegRows; ++j) accd[j] = 0.0;
        int it = 0;
        for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
            for (int c = 0; c < chunks; ++c, ++it) {
                const int s = it % S;
                const uint32_t ph = static_cast<uint32_t>(it / S) & 1u;
                if (!mbar_wait_bounded(&full[s], ph)) {
                    flag_error(err_flag, TK_DEVERR_TIMEOUT);
                    return;
                }
                const int ch0 = c * kChunkCh;
                const int chn = min(kChunkCh, H - ch0);
                const bool live = ct * 8 < chn;
                const uint8_t* base = data + static_cast<size_t>(s) * stage_bytes + ct * 16;
                uint8_t* dy_base = d_y + static_cast<int64_t>(ch0 + ct * 8) * 2;
                float gv[8];
                if (live) {
                    const uint4 q = *reinterpret_cast<const uint4*>(base);
                    gv[0] = lo_bf16(q.x); gv[1] = hi_bf16(q.x); gv[2] = lo_bf16(q.y); gv[3] = hi_bf16(q.y);
                    gv[4] = lo_bf16(q.z); gv[5] = hi_bf16(q.z); gv[6] = lo_bf16(q.w); gv[7] = hi_bf16(q.w);
                }
                if (reg_acc) {
                    double gd[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) gd[e] = live ? static_cast<double>(gv[e]) : 0.0;
#pragma unroll
                    for (int j = 0; j < kRegRows; ++j) {
                        if (j >= k) break;
                        const int32_t sl = meta[s].slot[j];
                        if (sl < 0 || !live) continue;
                        const float wj = meta[s].w[j];
                        const uint4 q = *reinterpret_cast<const uint4*>(base + (1 + j) * kChunkBytes);
                        accd[j] = fma(gd[0], static_cast<double>(lo_bf16(q.x)), accd[j]);
                        accd[j] = fma(gd[1], static_cast<double>(hi_bf16(q.x)), accd[j]);
                        accd[j] = fma(gd[2], static_cast<double>(lo_bf16(q.y)), accd[j]);
                        accd[j] = fma(gd[3], static_cast<double>(hi_bf16(q.y)), accd[j]);
                        accd[j] = fma(gd[4], static_cast<double>(lo_bf16(q.z)), accd[j]);
                        accd[j] = fma(gd[5], static_cast<double>(hi_bf16(q.z)), accd[j]);
                        accd[j] = fma(gd[6], static_cast<double>(lo_bf16(q.w)), accd[j]);
                        accd[j] = fma(gd[7], static_cast<double>(hi_bf16(q.w)), accd[j]);
                        uint4 o;
                        o.x = pack_bf16x2(__fmul_rn(wj, gv[0]), __fmul_rn(wj, gv[1]));
                        o.y = pack_bf16x2(__fmul_rn(wj, gv[2]), __fmul_rn(wj, gv[3]));
                        o.z = pack_bf16x2(__fmul_rn(wj, gv[4]), __fmul_rn(wj, gv[5]));
                        o.w = pack_bf16x2(__fmul_rn(wj, gv[6]), __fmul_rn(wj, gv[7]));
                        store_dy(dy_base + static_cast<int64_t>(sl) * row_bytes, o);
                    }
                } else {
                    for (int j = 0; j < k; ++j) {
                        const int32_t sl = meta[s].slot[j];
                        if (sl < 0) continue;  // the same for the whole warp
                        double part = 0.0;
                        if (live) {
                            const float wj = meta[s].w[j];
                            const uint4 q = *reinterpret_cast<const uint4*>(base + (1 + j) * kChunkBytes);
                            const float yv[8] = {lo_bf16(q.x), hi_bf16(q.x), lo_bf16(q.y), hi_bf16(q.y),
                                                 lo_bf16(q.z), hi_bf16(q.z), lo_bf16(q.w), hi_bf16(q.w)};
#pragma unroll
                            for (int e = 0; e < 8; ++e)
                                part = fma(static_cast<double>(gv[e]), static_cast<double>(yv[e]), part);
                            uint4 o;
                            o.x = pack_bf16x2(__fmul_rn(wj, gv[0]), __fmul_rn(wj, gv[1]));
                            o.y = pack_bf16x2(__fmul_rn(wj, gv[2]), __fmul_rn(wj, gv[3]));
                            o.z = pack_bf16x2(__fmul_rn(wj, gv[4]), __fmul_rn(wj, gv[5]));
                            o.w = pack_bf16x2(__fmul_rn(wj, gv[6]), __fmul_rn(wj, gv[7]));
                            store_dy(dy_base + static_cast<int64_t>(sl) * row_bytes, o);
                        }
#pragma unroll
                        for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(kFullMask, part, off);
                        if (lane == 0) dacc[cw * TK_MAX_TOPK + j] += part;
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[s]);
                if (c == chunks - 1) {  // token done: this warp's sums go out, accumulators reset
                    if (reg_acc) {
#pragma unroll
                        for (int j = 0; j < kRegRows; ++j) {
                            if (j >= k) break;
                            double v = accd[j];
#pragma unroll
                            for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(kFullMask, v, off);
                            if (lane == 0) dw_part[(t * k + j) * kConsumerWarps + cw] = v;
                            accd[j] = 0.0;
                        }
                    } else {
                        if (lane < k) {
                            dw_part[(t * k + lane) * kConsumerWarps + cw] = dacc[cw * TK_MAX_TOPK + lane];
                            dacc[cw * TK_MAX_TOPK + lane] = 0.0;
                        }
                        __syncwarp();
                    }
                }
            }
        }
    }
}

__global__ void dw_combine_kernel(const double* __restrict__ dw_part, int64_t pairs,
                                  float* __restrict__ d_w) {
    pdl_wait();
    for (int64_t p = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; p < pairs;
         p += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        double v = 0.0;
#pragma unroll
        for (int i = 0; i < kConsumerWarps; ++i) v += dw_part[p * kConsumerWarps + i];
        d_w[p] = static_cast<float>(v);
    }
}

struct Shape {
    int S = 0, grid_cap = 0;
};

// Launch shape for k on the current device, worked out once.
cudaError_t launch_shape(int k, Shape& out) {
    static Shape shapes[kMaxDevices][TK_MAX_TOPK + 1];
    static std::atomic<bool> ready[kMaxDevices][TK_MAX_TOPK + 1];
    static int configured[kMaxDevices];
    const int dev = current_device();
    if (ready[dev][k].load(std::memory_order_acquire)) {
        out = shapes[dev][k];
        return cudaSuccess;
    }
    std::lock_guard<std::mutex> lock(setup_mutex());
    if (!ready[dev][k].load(std::memory_order_relaxed)) {
        const int S = stages_for(k);
        const size_t smem = smem_bytes(k, S);
        cudaError_t err = cudaSuccess;
        if (static_cast<int>(smem) > configured[dev]) {
            err = cudaFuncSetAttribute(reduce_backward_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
            if (err != cudaSuccess) return err;
            configured[dev] = static_cast<int>(smem);
        }
        int per_sm = 0;
        err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, reduce_backward_kernel, kBwdThreads, smem);
        if (err != cudaSuccess) return err;
        // Launched after a kernel that leaves L2 full of dirty lines (its own previous call, or
        // any write-heavy step), 3 CTAs per SM measured 1-2 % faster than the 5 that fit.
        if (TK_BACKWARD_CTAS_PER_SM > 0 && per_sm > TK_BACKWARD_CTAS_PER_SM) per_sm = TK_BACKWARD_CTAS_PER_SM;
        shapes[dev][k].S = S;
        shapes[dev][k].grid_cap = num_sms() * (per_sm < 1 ? 1 : per_sm);
        ready[dev][k].store(true, std::memory_order_release);
    }
    out = shapes[dev][k];
    return cudaSuccess;
}

}  // namespace
}  // namespace tk

extern "C" size_t tk_reduce_backward_workspace_bytes(int T, int k) {
    if (T < 0 || k < 1) return 0;
    const size_t pairs = static_cast<size_t>(T > 0 ? T : 1) * static_cast<size_t>(k);
    return pairs * tk::kConsumerWarps * sizeof(double);
}

extern "C" tk_status tk_reduce_backward(const void* grad_out, const void* y, int64_t y_rows,
                                        const int32_t* slot_of, const int32_t* offsets,
                                        const int32_t* token_of, const float* w, int T, int E,
                                        int k, int H, void* d_y, float* d_w, void* workspace,
                                        size_t workspace_bytes, int32_t* err_flag, void* stream) {
    using namespace tk;
    if (T < 0) return fail_arg("tk_reduce_backward: T=%d must be >= 0", T);
    if (E < 1 || E > TK_MAX_EXPERTS) return fail_arg("tk_reduce_backward: E=%d outside [1, %d]", E, TK_MAX_EXPERTS);
    if (k < 1 || k > TK_MAX_TOPK) return fail_arg("tk_reduce_backward: k=%d outside [1, %d]", k, TK_MAX_TOPK);
    if (H < 8 || H % 8 != 0) return fail_arg("tk_reduce_backward: H=%d must be a positive multiple of 8", H);
    if (y_rows < 0 || y_rows > INT32_MAX) return fail_arg("tk_reduce_backward: y_rows=%lld out of range", (long long)y_rows);
    if (T == 0) return TK_OK;
    if (grad_out == nullptr || y == nullptr || slot_of == nullptr || d_y == nullptr || d_w == nullptr ||
        workspace == nullptr)
        return fail_arg("tk_reduce_backward: grad_out, y, slot_of, d_y, d_w and workspace must not be NULL");
    if ((offsets == nullptr) != (token_of == nullptr))
        return fail_arg("tk_reduce_backward: offsets and token_of go together (both or neither)");
    for (const void* p : {grad_out, y, static_cast<const void*>(d_y)})
        if (reinterpret_cast<uintptr_t>(p) % 16 != 0)
            return fail_arg("tk_reduce_backward: grad_out, y and d_y must be 16-byte aligned");
    if (reinterpret_cast<uintptr_t>(workspace) % 16 != 0)
        return fail_arg("tk_reduce_backward: workspace must be 16-byte aligned");
    const size_t need = tk_reduce_backward_workspace_bytes(T, k);
    if (workspace_bytes < need)
        return fail_arg("tk_reduce_backward: workspace holds %zu bytes, needs %zu", workspace_bytes, need);
    Shape sh;
    const cudaError_t e = launch_shape(k, sh);
    if (e != cudaSuccess) return check_launch(e, "reduce_backward_kernel setup");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    double* dw_part = static_cast<double*>(workspace);
    const int grid = T < sh.grid_cap ? T : sh.grid_cap;
    cudaError_t err = launch_pdl(reduce_backward_kernel, dim3(grid), dim3(kBwdThreads), smem_bytes(k, sh.S), s,
                                 static_cast<const uint8_t*>(grad_out), static_cast<const uint8_t*>(y),
                                 y_rows, slot_of, w, T, k, H, sh.S, static_cast<uint8_t*>(d_y), dw_part,
                                 err_flag);
    if (err != cudaSuccess) return check_launch(err, "reduce_backward_kernel");
    const int64_t pairs = static_cast<int64_t>(T) * k;
    int64_t cgrid = (pairs + 255) / 256;
    if (cgrid > num_sms() * 8) cgrid = num_sms() * 8;
    err = launch_pdl(dw_combine_kernel, dim3(static_cast<unsigned>(cgrid)), dim3(256), 0, s,
                     static_cast<const double*>(dw_part), pairs, d_w);
    if (err != cudaSuccess) return check_launch(err, "dw_combine_kernel");
    if (offsets != nullptr) {
        err = launch_pad_zero(offsets, token_of, E, y_rows, static_cast<uint8_t*>(d_y),
                              static_cast<int64_t>(H) * 2, nullptr, 0, err_flag, s);
        if (err != cudaSuccess) return check_launch(err, "expand_pad_kernel");
    }
    return TK_OK;
}

extern "C" tk_status tk_expand_backward(const void* d_xe, int64_t xe_rows, const int32_t* slot_of,
                                        int T, int k, int H, void* d_x, int32_t* err_flag,
                                        void* stream) {
    // d_x[t] = sum_j d_xe[slot_of[t,j]]: the unweighted reduce, same kernel and arithmetic
    return tk_reduce(d_xe, xe_rows, slot_of, nullptr, T, k, H, d_x, err_flag, stream);
}
