// Per-token, per-128-channel E4M3 quantisation of one block by one warp (the quant/ module's
// per-token granularity, 147227.xyz "刚刚！DeepSeek开源高性能GPU算子库TileKernels", section
// "quant/"; FP8 dispatch in 機器之心 "性能表現"): amax over the 128 channels, scale = amax/448
// (IEEE division), code = cvt.rn.satfinite.e4m3x2(x / scale) with IEEE division; an all-zero
// block gets scale 0 and codes 0. Shared by the expand and the expert-parallel dispatch kernels.
#pragma once

#include <stdint.h>

#include "tk_device.cuh"

namespace tk {

__device__ __forceinline__ float bf16_bits_to_float(uint32_t h) { return __uint_as_float(h << 16); }

// xin: the block's 128 bf16 values in shared memory; lane l handles channels 4l .. 4l+3 and
// writes their 4 codes to qo (shared memory). Returns the block's scale on every lane.
__device__ __forceinline__ float quantize_block_e4m3(const uint16_t* xin, uint8_t* qo, int lane) {
    const int cc = lane * 4;
    const uint2 raw = *reinterpret_cast<const uint2*>(xin + cc);
    const float f0 = bf16_bits_to_float(raw.x & 0xffffu);
    const float f1 = bf16_bits_to_float(raw.x >> 16);
    const float f2 = bf16_bits_to_float(raw.y & 0xffffu);
    const float f3 = bf16_bits_to_float(raw.y >> 16);
    const float a = fmaxf(fmaxf(fabsf(f0), fabsf(f1)), fmaxf(fabsf(f2), fabsf(f3)));
    // non-negative floats order like their bit patterns
    const float amax = __uint_as_float(__reduce_max_sync(kFullMask, __float_as_uint(a)));
    uint32_t q = 0u;
    float scale = 0.0f;
    if (amax != 0.0f) {
        scale = __fdiv_rn(amax, 448.0f);
        const uint32_t lo = cvt_e4m3x2(__fdiv_rn(f0, scale), __fdiv_rn(f1, scale));
        const uint32_t hi = cvt_e4m3x2(__fdiv_rn(f2, scale), __fdiv_rn(f3, scale));
        q = lo | (hi << 16);
    }
    *reinterpret_cast<uint32_t*>(qo + cc) = q;
    return scale;
}

}  // namespace tk
