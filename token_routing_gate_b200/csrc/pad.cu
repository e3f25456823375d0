// Zero-fill of padding rows, shared by tk_expand and tk_reduce_backward: rows r below
// offsets[E] whose token_of[r] is -1 (the rows that round an expert's segment up to the
// alignment) are overwritten with zeros.
#include <cuda_runtime.h>
#include <stdint.h>

#include "tk_device.cuh"

namespace tk {
namespace {

constexpr int kPadThreads = 256;
constexpr uint32_t kZeroChunkBytes = 32768;  // zeroed shared buffer, reused for longer rows

// Zeroes padding rows: rows r < offsets[E] with token_of[r] == -1. Padding comes in runs of up
// to align-1 rows at the end of each expert's segment, so rows are dealt out round-robin over
// CTAs (row r goes to CTA r % gridDim.x) to spread every run over many SMs. A thread that finds
// a padding row enqueues bulk stores of a zeroed shared buffer over it (plus plain stores for
// E4M3 scales), so the zeroing runs on the copy engines while the thread moves on.
__global__ void __launch_bounds__(kPadThreads)
expand_pad_kernel(const int32_t* __restrict__ offsets, const int32_t* __restrict__ token_of,
                  int E, int64_t rmax, uint8_t* __restrict__ out, int64_t row_bytes,
                  float* __restrict__ out_scale, int scale_cols, int32_t* err_flag) {
    extern __shared__ __align__(128) uint8_t zeros[];  // min(row_bytes, kZeroChunkBytes)
    const uint32_t zbytes = static_cast<uint32_t>(row_bytes < kZeroChunkBytes ? row_bytes : kZeroChunkBytes);
    for (uint32_t o = threadIdx.x * 16u; o < zbytes; o += kPadThreads * 16u)
        *reinterpret_cast<uint4*>(zeros + o) = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async_smem();
    __syncthreads();
    pdl_wait();
    int64_t R = offsets[E];
    if (R < 0 || R > rmax) {
        if (blockIdx.x == 0 && threadIdx.x == 0) flag_error(err_flag, TK_DEVERR_ROWS_RANGE);
        R = R < 0 ? 0 : rmax;
    }
    bool issued = false;
    for (int64_t r = blockIdx.x + static_cast<int64_t>(threadIdx.x) * gridDim.x; r < R;
         r += static_cast<int64_t>(kPadThreads) * gridDim.x) {
        if (token_of[r] != -1) continue;
        uint8_t* row = out + r * row_bytes;
        for (int64_t o = 0; o < row_bytes; o += zbytes) {
            const int64_t left = row_bytes - o;
            bulk_store(row + o, zeros, static_cast<uint32_t>(left < zbytes ? left : zbytes));
        }
        issued = true;
        if (out_scale != nullptr)
            for (int c = 0; c < scale_cols; ++c) out_scale[r * scale_cols + c] = 0.0f;
    }
    if (issued) {
        bulk_commit();
        bulk_wait_read_all();  // the shared zero buffer must outlive the stores that read it
    }
}

}  // namespace

cudaError_t launch_pad_zero(const int32_t* offsets, const int32_t* token_of, int E, int64_t rmax,
                            uint8_t* out, int64_t row_bytes, float* out_scale, int scale_cols,
                            int32_t* err_flag, cudaStream_t s) {
    int64_t grid = (rmax + kPadThreads - 1) / kPadThreads;
    const int64_t cap = static_cast<int64_t>(num_sms()) * 4;
    if (grid > cap) grid = cap;
    if (grid < 1) grid = 1;
    const size_t zsmem = static_cast<size_t>(row_bytes < kZeroChunkBytes ? row_bytes : kZeroChunkBytes);
    return launch_pdl(expand_pad_kernel, dim3(static_cast<unsigned>(grid)), dim3(kPadThreads), zsmem, s,
                      offsets, token_of, E, rmax, out, row_bytes, out_scale, scale_cols, err_flag);
}

}  // namespace tk
