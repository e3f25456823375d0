// Per-token gate arithmetic shared by the gate kernel and the fused gate + route-map kernel
// (one warp per token; lane l holds experts l, l+32, l+64, ...). See gate_topk.cu for the
// method and its sources.
#pragma once

#include <math.h>
#include <stdint.h>

#include "tk_device.cuh"

namespace tk {
namespace gate {

// e^x in fp32 for the selection key (the fixed exponential described at the top of
// gate_topk.cu). x is clamped to [-110, 100] first:
// e^-110 rounds to zero and e^100 overflows, so the clamp changes no result.
__device__ __forceinline__ float key_expf(float x) {
    if (x != x) return x;
    x = fminf(fmaxf(x, -110.0f), 100.0f);
    const float n = rintf(__fmul_rn(x, 0x1.715476p+0f));   // x * log2(e), nearest even integer
    float r = __fmaf_rn(-n, 0x1.62e4p-1f, x);               // ln2 high part: n*hi is exact
    r = __fmaf_rn(-n, 0x1.7f7d1cp-20f, r);                  // ln2 low part
    float p = 0x1.a01a02p-13f;                               // 1/7!
    p = __fmaf_rn(p, r, 0x1.6c16c2p-10f);                    // 1/6!
    p = __fmaf_rn(p, r, 0x1.111112p-7f);                     // 1/5!
    p = __fmaf_rn(p, r, 0x1.555556p-5f);                     // 1/4!
    p = __fmaf_rn(p, r, 0x1.555556p-3f);                     // 1/3!
    p = __fmaf_rn(p, r, 0.5f);                               // 1/2!
    p = __fmaf_rn(p, r, 1.0f);
    p = __fmaf_rn(p, r, 1.0f);
    const int ni = static_cast<int>(n);
    const int n1 = ni / 2;
    const int n2 = ni - n1;
    // scale by 2^n in two exact-or-single-rounding steps (|n1|, |n2| <= 80)
    const float s1 = __int_as_float((n1 + 127) << 23);
    const float s2 = __int_as_float((n2 + 127) << 23);
    return __fmul_rn(__fmul_rn(p, s1), s2);
}

__device__ __forceinline__ float key_sigmoidf(float l) {
    return __fdiv_rn(1.0f, __fadd_rn(1.0f, key_expf(-l)));
}

// Order-preserving map of an fp32 key to uint32 (larger key -> larger integer). -0 is folded
// onto +0 and NaN onto -inf first, so float equality and integer equality agree.
__device__ __forceinline__ uint32_t ordered_key(float key) {
    if (key != key) key = -INFINITY;
    key = __fadd_rn(key, 0.0f);  // -0 + 0 = +0
    const uint32_t u = __float_as_uint(key);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Packs an ordered key and an expert index into one 64-bit value whose unsigned order is
// (key descending, index ascending): the high word is the key's image, the low word ~e.
__device__ __forceinline__ uint64_t pack_key(uint32_t ord, int e) {
    return (static_cast<uint64_t>(ord) << 32) | static_cast<uint32_t>(~e);
}

// Sorts a lane's EPL packed values in descending order (bitonic network, fully unrolled).
template <int EPL>
__device__ __forceinline__ void sort_desc(uint64_t (&v)[EPL]) {
#pragma unroll
    for (int size = 2; size <= EPL; size <<= 1) {
#pragma unroll
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
#pragma unroll
            for (int i = 0; i < EPL; ++i) {
                const int l = i ^ stride;
                if (l > i) {
                    const bool desc = (i & size) == 0;
                    const uint64_t a = v[i], b = v[l];
                    const bool swap = desc ? (a < b) : (a > b);
                    v[i] = swap ? b : a;
                    v[l] = swap ? a : b;
                }
            }
        }
    }
}

// Keys of the lane's experts, packed with their indices (0 for an absent expert e >= E). Every
// real key maps above 0 (-inf maps to 0x007FFFFF), so 0 also marks an expert already chosen and
// real experts always win over absent ones.
template <int EPL>
__device__ __forceinline__ void build_keys(const float (&lg)[EPL], const float (&b)[EPL],
                                           bool has_bias, int E, int lane, uint64_t (&v)[EPL]) {
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        const int e = i * 32 + lane;
        v[i] = 0;
        if (e < E) {
            const float l = lg[i];
            const float key = has_bias ? __fadd_rn(key_sigmoidf(l), b[i]) : l;
            v[i] = pack_key(ordered_key(key), e);
        }
    }
}

// k rounds of (warp max of the key image, then the lowest index among the lanes holding it);
// lane j returns the j-th winner (lanes >= k return 0).
template <int EPL>
__device__ __forceinline__ int select_topk(uint64_t (&v)[EPL], int k, int lane) {
    if (EPL > 1) sort_desc<EPL>(v);
    int my_e = 0;
    for (int j = 0; j < k; ++j) {
        const uint32_t hi = static_cast<uint32_t>(v[0] >> 32);
        const uint32_t m = __reduce_max_sync(kFullMask, hi);
        const uint32_t lo = static_cast<uint32_t>(v[0]);
        const uint32_t win = __reduce_max_sync(kFullMask, hi == m ? lo : 0u);  // ~e: lower e wins
        if (lane == j) my_e = static_cast<int>(~win);
        if (hi == m && lo == win) {  // the one lane holding the winner drops it
#pragma unroll
            for (int i = 0; i + 1 < EPL; ++i) v[i] = v[i + 1];
            v[EPL - 1] = 0;
        }
    }
    return my_e;
}

// Weights of the chosen experts (double, rounded once to fp32); lanes j < k write idx_out[j]
// and w_out[j] (this token's k entries).
template <int EPL>
__device__ __forceinline__ void write_choice(const float* __restrict__ row, int my_e, int E, int k,
                                             int score_fn, int renormalize, int lane,
                                             int32_t* __restrict__ idx_out,
                                             float* __restrict__ w_out) {
    const float my_l = lane < k ? row[my_e] : 0.0f;
    const float top_l = __shfl_sync(kFullMask, my_l, 0);
    double s = 0.0;
    bool zero_all = false;
    if (score_fn == TK_SCORE_SIGMOID) {
        if (lane < k) s = 1.0 / (1.0 + exp(-static_cast<double>(my_l)));
    } else {
        // no bias with softmax, so the first winner holds the largest logit
        if (top_l == -INFINITY || top_l != top_l) {
            zero_all = true;
        } else if (lane < k) {
            s = exp(static_cast<double>(my_l) - static_cast<double>(top_l));
        }
    }
    double denom;
    if (renormalize) {
        double acc = s;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(kFullMask, acc, off);
        denom = acc;
    } else if (score_fn == TK_SCORE_SOFTMAX) {
        // full softmax denominator over all E experts
        double z = 0.0;
        if (!zero_all) {
#pragma unroll
            for (int i = 0; i < EPL; ++i) {
                const int e = i * 32 + lane;
                if (e < E) z += exp(static_cast<double>(row[e]) - static_cast<double>(top_l));
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(kFullMask, z, off);
        denom = z;
    } else {
        denom = 1.0;
    }
    if (lane < k) {
        idx_out[lane] = my_e;
        w_out[lane] = (zero_all || denom == 0.0) ? 0.0f : static_cast<float>(s / denom);
    }
}

}  // namespace gate
}  // namespace tk
