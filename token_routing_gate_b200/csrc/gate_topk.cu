// Gate: expert scoring, top-k selection and renormalisation, one warp per token.
//
// Selection follows the one-warp-per-token TopK kernel sketched in "DeepSeek 的 GPU 内核帝国"
// (zhichai.net), section "MoE TopK 门控": the token's expert scores live in the warp's
// registers, and each of k rounds takes the warp-wide maximum, resolves equal maxima to the
// lowest expert index, records the winner and removes it. Here each lane holds experts
// lane, lane+32, lane+64, ... (so every load of a logits row is one coalesced 128-byte line)
// and a round is two warp reductions (redux.sync): the maximum of an order-preserving integer
// image of the key, then the minimum expert index among the lanes holding that maximum.
//
// Key: the logit when no bias is given; with a bias (sigmoid scoring) the fp32 value
// sigmoid(l) + b, where sigmoid uses a fixed fp32 exponential (Cody-Waite reduction by ln 2,
// degree-7 Taylor polynomial, every step one IEEE fp32 operation), so the same key bits -- and
// the same selected experts -- come out on any IEEE fp32 machine that follows the same steps.
// Weights: the chosen experts' unbiased scores in double (library exp), renormalised over the
// k chosen ones when asked, rounded once to fp32.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "tk_device.cuh"

namespace tk {
namespace {

constexpr int kGateWarps = 8;  // tokens per CTA

// e^x in fp32 for the selection key (see file comment). x is clamped to [-110, 100] first:
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

// One warp per token. The grid is one wave of resident warps and the T tokens are split evenly
// over the nwarps warps (warp w takes tokens [w*T/nwarps, (w+1)*T/nwarps), so warps differ by
// at most one token and every SM gets the same work); the next token's logits are loaded while
// the current one is processed. EPL = experts held per lane (E <= 32 * EPL).
template <int EPL>
__global__ void __launch_bounds__(kGateWarps * 32)
gate_topk_kernel(const float* __restrict__ logits, const float* __restrict__ bias, int T, int E,
                 int k, int score_fn, int renormalize, int nwarps,
                 int32_t* __restrict__ topk_idx, float* __restrict__ topk_w) {
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int64_t wid = static_cast<int64_t>(blockIdx.x) * kGateWarps + (threadIdx.x >> 5);
    if (wid >= nwarps) return;
    const int64_t t_begin = wid * T / nwarps;
    const int64_t t_end = (wid + 1) * T / nwarps;
    if (t_begin >= t_end) return;

    float b[EPL];  // this lane's selection biases, shared by all tokens
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        const int e = i * 32 + lane;
        b[i] = (bias != nullptr && e < E) ? bias[e] : 0.0f;
    }
    float lg[EPL];  // logits of the token being routed, then of the next one (prefetch)
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        const int e = i * 32 + lane;
        lg[i] = e < E ? logits[t_begin * E + e] : 0.0f;
    }

    for (int64_t t = t_begin; t < t_end; ++t) {
        const float* row = logits + t * E;

        // Every real key maps above 0 (-inf maps to 0x007FFFFF), so 0 marks an absent expert
        // (e >= E) or one already chosen, and real experts always win over absent ones.
        uint64_t v[EPL];
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
            const int e = i * 32 + lane;
            v[i] = 0;
            if (e < E) {
                const float l = lg[i];
                const float key = bias != nullptr ? __fadd_rn(key_sigmoidf(l), b[i]) : l;
                v[i] = pack_key(ordered_key(key), e);
            }
        }
        if (t + 1 < t_end) {  // the registers are free again: start the next token's loads
#pragma unroll
            for (int i = 0; i < EPL; ++i) {
                const int e = i * 32 + lane;
                lg[i] = e < E ? row[E + e] : 0.0f;
            }
        }
        if (EPL > 1) sort_desc<EPL>(v);

        int my_e = 0;  // lane j keeps the j-th winner
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
        const float my_l = lane < k ? row[my_e] : 0.0f;

        // ---- weights (double), lanes 0..k-1 hold the chosen experts in order
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
            const int64_t o = t * k + lane;
            topk_idx[o] = my_e;
            topk_w[o] = (zero_all || denom == 0.0) ? 0.0f : static_cast<float>(s / denom);
        }
    }
}

template <int EPL>
cudaError_t launch_gate(const float* logits, const float* bias, int T, int E, int k, int score_fn,
                        int renormalize, int32_t* idx, float* w, cudaStream_t s) {
    // one wave: as many warps as fit on the GPU at once, each taking a run of consecutive tokens
    static std::atomic<int> resident[kMaxDevices];
    const int dev = current_device();
    int resident_warps = resident[dev].load(std::memory_order_acquire);
    if (resident_warps == 0) {
        int per_sm = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, gate_topk_kernel<EPL>,
                                                          kGateWarps * 32, 0) != cudaSuccess || per_sm < 1)
            per_sm = 1;
        resident_warps = per_sm * kGateWarps * num_sms();
        resident[dev].store(resident_warps, std::memory_order_release);
    }
    const int warps = min(T, resident_warps);
    const dim3 grid((warps + kGateWarps - 1) / kGateWarps);
    return launch_pdl(gate_topk_kernel<EPL>, grid, dim3(kGateWarps * 32), 0, s, logits, bias, T, E,
                      k, score_fn, renormalize, warps, idx, w);
}

}  // namespace
}  // namespace tk

extern "C" tk_status tk_gate_topk(const float* logits, const float* bias, int T, int E, int k,
                                  int score_fn, int renormalize, int32_t* topk_idx, float* topk_w,
                                  void* stream) {
    using namespace tk;
    if (T < 0) return fail_arg("tk_gate_topk: T=%d must be >= 0", T);
    if (E < 1 || E > TK_MAX_EXPERTS) return fail_arg("tk_gate_topk: E=%d outside [1, %d]", E, TK_MAX_EXPERTS);
    if (k < 1 || k > E || k > TK_MAX_TOPK)
        return fail_arg("tk_gate_topk: k=%d outside [1, min(E=%d, %d)]", k, E, TK_MAX_TOPK);
    if (score_fn != TK_SCORE_SOFTMAX && score_fn != TK_SCORE_SIGMOID)
        return fail_arg("tk_gate_topk: unknown score_fn %d", score_fn);
    if (score_fn == TK_SCORE_SOFTMAX && bias != nullptr)
        return fail_arg("tk_gate_topk: a selection bias is only defined for sigmoid scoring");
    if (T == 0) return TK_OK;
    if (logits == nullptr || topk_idx == nullptr || topk_w == nullptr)
        return fail_arg("tk_gate_topk: logits, topk_idx and topk_w must not be NULL");
    if (static_cast<int64_t>(T) * E > INT64_C(1) << 40)
        return fail_arg("tk_gate_topk: T*E too large");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int epl = (E + 31) / 32;
    cudaError_t err;
    if (epl <= 1) err = launch_gate<1>(logits, bias, T, E, k, score_fn, renormalize, topk_idx, topk_w, s);
    else if (epl <= 2) err = launch_gate<2>(logits, bias, T, E, k, score_fn, renormalize, topk_idx, topk_w, s);
    else if (epl <= 4) err = launch_gate<4>(logits, bias, T, E, k, score_fn, renormalize, topk_idx, topk_w, s);
    else if (epl <= 8) err = launch_gate<8>(logits, bias, T, E, k, score_fn, renormalize, topk_idx, topk_w, s);
    else if (epl <= 16) err = launch_gate<16>(logits, bias, T, E, k, score_fn, renormalize, topk_idx, topk_w, s);
    else err = launch_gate<32>(logits, bias, T, E, k, score_fn, renormalize, topk_idx, topk_w, s);
    return check_launch(err, "gate_topk_kernel");
}
