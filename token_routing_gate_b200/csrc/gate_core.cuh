// Per-token gate arithmetic of the gate kernel (one warp per token; lane l holds experts l,
// l+32, l+64, ...). See gate_topk.cu for the method and its sources.
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

// Inverse of ordered_key for the image of a real key (any value >= the image of -inf).
__device__ __forceinline__ float key_of_image(uint32_t u) {
    return __uint_as_float((u & 0x80000000u) ? (u & 0x7fffffffu) : ~u);
}

// Hardware approximations for the candidate filter only (no result is taken from them).
// PTX ISA: rcp.approx.f32 is within 1 ulp; ex2.approx.f32 within a few ulp (relative error
// about 2^-22); .ftz flushes subnormal results to zero.
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float rcp_approx(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Approximate logistic value 1 / (1 + 2^(-l log2 e)). Rounding l log2 e to fp32 moves the
// exponent by at most |l| log2 e 2^-24, a relative error of at most 6e-6 in 2^x for
// |l| <= 100; with the approximations' own errors the value is within 2^-17 of the true
// logistic value there (its slope in log e^-l is s(1-s) <= 1/4), as is the exact key's fp32
// sigmoid (within 2^-22). Beyond |l| = 100 both are 0 or 1 to within 2^-126.
__device__ __forceinline__ float approx_sigmoidf(float l) {
    return rcp_approx(1.0f + ex2_approx(l * -0x1.715476p+0f));
}

// Order-preserving image of an approximate key: NaN ranks as -inf (fmaxf keeps the other
// operand), so a NaN logit sorts at the bottom exactly as its exact key does.
__device__ __forceinline__ uint32_t approx_image(float a) {
    a = fmaxf(a, -INFINITY);
    const uint32_t u = __float_as_uint(a);
    return u ^ ((static_cast<uint32_t>(static_cast<int32_t>(u) >> 31)) | 0x80000000u);
}

// Images of the lane's approximate keys (0 for an absent expert e >= E). Without a bias the
// key is the logit itself (-0 folded onto +0 like the exact key), so the image is exact.
template <int EPL>
__device__ __forceinline__ void approx_images(const float (&lg)[EPL], const float (&b)[EPL],
                                              bool has_bias, int E, int lane, uint32_t (&u)[EPL]) {
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        const int e = i * 32 + lane;
        const float a = has_bias ? __fadd_rn(approx_sigmoidf(lg[i]), b[i]) : __fadd_rn(lg[i], 0.0f);
        u[i] = e < E ? approx_image(a) : 0u;
    }
}

// A value with at least k of the 32 lanes' values >= it, cheaply: with G = the smallest power
// of two >= k, the minimum over G groups of 32/G adjacent lanes of each group's maximum (each
// group contributes one value >= it). 0 when some group holds no expert.
__device__ __forceinline__ uint32_t group_threshold(uint32_t v, int k) {
    const int width = 32 >> (32 - __clz(k - 1));  // lanes per group: 32 / G (k in [1, 32])
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const uint32_t o = __shfl_xor_sync(kFullMask, v, off);
        v = off < width ? max(v, o) : min(v, o);
    }
    return v;
}

// The k-th largest of the 32 lanes' values, counted with multiplicity: at least k lanes hold a
// value >= the result. 0 when fewer than k lanes hold a nonzero value. Warp-uniform.
__device__ __forceinline__ uint32_t kth_lane_max(uint32_t v, int k) {
    int have = 0;
    for (int r = 0; r < k; ++r) {
        const uint32_t m = __reduce_max_sync(kFullMask, v);
        if (m == 0) return 0;
        have += __popc(__ballot_sync(kFullMask, v == m));
        if (have >= k) return m;
        if (v == m) v = 0;
    }
    return 0;
}

__device__ __forceinline__ uint32_t lanemask_lt() {
    uint32_t m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// One warp's shared scratch: the candidates (expert, logit bits) in (slot of the lane's list,
// lane) order, and the chosen experts with their logits by (token of the batch, rank): token q's
// rank-j choice at entry q*k + j.
struct Candidates {
    uint2 el[32];
    int by_rank[32];
    float l_by_rank[32];
};

// Ballots of the lane's experts whose image is >= cut; returns their number (warp-uniform).
template <int EPL>
__device__ __forceinline__ int count_candidates(const uint32_t (&u)[EPL], uint32_t cut,
                                                uint32_t (&bal)[EPL]) {
    int C = 0;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        bal[i] = __ballot_sync(kFullMask, u[i] >= cut);
        C += __popc(bal[i]);
    }
    return C;
}

// Writes the balloted candidates (at most 32) to the warp's list, candidate c at entry c.
template <int EPL>
__device__ __forceinline__ void gather_candidates(const uint32_t (&bal)[EPL], const float (&lg)[EPL],
                                                  int lane, Candidates& c) {
    const uint32_t lt = lanemask_lt();
    int base = 0;
    __syncwarp();  // the previous token's reads of the list are done
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        if ((bal[i] >> lane) & 1u)
            c.el[base + __popc(bal[i] & lt)] = make_uint2(static_cast<uint32_t>(i * 32 + lane),
                                                          __float_as_uint(lg[i]));
        base += __popc(bal[i]);
    }
    __syncwarp();
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

// Outputs of a batch of n consecutive tokens (n*k <= 32) whose choices sit in c.by_rank /
// c.l_by_rank: lane q*k + j takes token q's rank-j choice and computes its unbiased score in
// double -- the logistic value 1 / (1 + e^-l), or for softmax (renormalised only) e^(l - l0)
// with l0 the token's rank-0 logit, its largest (the full softmax denominator cancels in the
// renormalisation; an infinite or NaN l0 gives zero weights) -- adds the k scores of its token
// in rank order when renormalising (the order of the defining sum), and writes entry q*k + j of
// the batch's outputs (consecutive in idx_out and w_out), rounded once to fp32. One pass serves
// up to 32/k tokens, so the double arithmetic runs on up to every lane instead of k of them per
// token.
__device__ __forceinline__ void write_batch(const Candidates& c, int n, int k, int score_fn,
                                            int renormalize, int lane,
                                            int32_t* __restrict__ idx_out, float* __restrict__ w_out) {
    __syncwarp();  // the batch's choices are in c
    const bool mine = lane < n * k;
    const int first = lane - lane % k;  // this token's rank-0 lane (mod 32 past the batch)
    double s = 0.0;
    int e = 0;
    if (mine) {
        e = c.by_rank[lane];
        const float l = c.l_by_rank[lane];
        if (score_fn == TK_SCORE_SIGMOID) {
            s = 1.0 / (1.0 + exp(-static_cast<double>(l)));
        } else {
            const float l0 = c.l_by_rank[first];
            if (l0 != -INFINITY && l0 == l0) s = exp(static_cast<double>(l) - static_cast<double>(l0));
        }
    }
    double denom = 1.0;
    if (renormalize) {
        denom = 0.0;
        for (int j = 0; j < k; ++j) denom += __shfl_sync(kFullMask, s, first + j);
    }
    if (mine) {
        idx_out[lane] = e;
        w_out[lane] = !renormalize ? static_cast<float>(s)
                                   : (denom == 0.0 ? 0.0f : static_cast<float>(s / denom));
    }
    __syncwarp();  // c may be refilled
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
