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

#include "gate_core.cuh"
#include "tk_device.cuh"

namespace tk {
namespace {

constexpr int kGateWarps = 8;  // tokens per CTA

// Selection in two passes, with the same result as ranking all E exact keys:
//  1. Approximate keys A_e (the logit itself without a bias; approx_sigmoidf(l) + b with one)
//     satisfy |A_e - K_e| <= eps for the exact keys K_e, where eps = 2^-12 + 2^-20 * max|b|
//     is more than 30 times the bound in approx_sigmoidf's comment (the two additions of b
//     round by at most an ulp of 1 + max|b| between them). Without a bias eps = 0.
//  2. A threshold theta that at least k approximate keys reach (first the cheap
//     group_threshold, then the k-th largest lane maximum when the cheap one leaves more than
//     32 candidates). The k-th largest exact key is then >= theta - eps, and every expert whose
//     exact key reaches it has A >= theta - 2 eps. Those experts (the candidates) get their
//     exact keys, one per lane in ascending expert order, and k rounds of warp reductions select
//     among them exactly as among all E: one reduction per round over (key offset, lane) packed
//     into a word while the candidates' key images span less than 2^26, else two (the key, then
//     the lowest index holding it). Each winner records its expert and logit by rank; with
//     logistic scores the weights of up to 32/k consecutive tokens are then computed together.
// More than 32 candidates (many equal or nearly equal keys), a non-finite or huge bias, or
// fewer than k lanes holding an expert send the token down the full path: every exact key, a
// per-lane sort and k rounds over the sorted lists.
//
// Weights are computed in fp64 and rounded once to fp32, so they are the correctly rounded
// fp32 values of the defining quotient except in rare halfway cases: fp32 weights within 1e-6
// relative but a few ulps off those values would move reduce outputs that nearly cancel by more
// than one bf16 ulp.
__device__ __forceinline__ float filter_margin(const float* b, int epl, bool has_bias, bool* ok) {
    if (!has_bias) {
        *ok = true;
        return 0.0f;
    }
    float m = 0.0f;
    bool finite = true;
    for (int i = 0; i < epl; ++i) {
        finite = finite && isfinite(b[i]);
        m = fmaxf(m, fabsf(b[i]));
    }
    finite = __all_sync(kFullMask, finite);
    // |b| of finite values are non-negative floats: their bit patterns order like the values
    m = __uint_as_float(__reduce_max_sync(kFullMask, __float_as_uint(finite ? m : 0.0f)));
    *ok = finite && m < 0x1p+20f;
    return __fmaf_ru(m, 0x1p-20f, 0x1p-12f);
}

// Candidate cut for a threshold image: theta itself without a bias, else the image of
// theta - 2 eps rounded down.
__device__ __forceinline__ uint32_t cut_of(uint32_t theta, bool has_bias, float eps) {
    return has_bias ? gate::ordered_key(__fsub_rd(gate::key_of_image(theta), 2.0f * eps)) : theta;
}

template <int EPL>
__device__ __forceinline__ void prefetch_row(const float* row, int E, int lane, float (&lg)[EPL]) {
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        const int e = i * 32 + lane;
        lg[i] = e < E ? row[e] : 0.0f;
    }
}

// One warp per token. The grid is one wave of resident warps and the T tokens are split evenly
// over the nwarps warps (warp w takes tokens [w*T/nwarps, (w+1)*T/nwarps), so warps differ by
// at most one token and every SM gets the same work); the next token's logits are loaded while
// the current one is processed. EPL = experts held per lane (E <= 32 * EPL); kFull: E is exactly
// 32 * EPL, so no lane's expert is absent and E is a constant. With logistic scores a warp keeps
// the choices of up to 32/k consecutive tokens and computes their weights in one pass.
template <int EPL, bool kFull>
__global__ void __launch_bounds__(kGateWarps * 32, EPL <= 8 ? 4 : 1)
gate_topk_kernel(const float* __restrict__ logits, const float* __restrict__ bias, int T, int E_in,
                 int k, int score_fn, int renormalize, int nwarps,
                 int32_t* __restrict__ topk_idx, float* __restrict__ topk_w) {
    __shared__ gate::Candidates cands[kGateWarps];
    pdl_wait();
    const int E = kFull ? 32 * EPL : E_in;
    const int lane = threadIdx.x & 31;
    const int64_t wid = static_cast<int64_t>(blockIdx.x) * kGateWarps + (threadIdx.x >> 5);
    if (wid >= nwarps) return;
    const int64_t t_begin = wid * T / nwarps;
    const int64_t t_end = (wid + 1) * T / nwarps;
    if (t_begin >= t_end) return;
    gate::Candidates& cand = cands[threadIdx.x >> 5];
    const bool has_bias = bias != nullptr;
    const bool sigmoid = score_fn == TK_SCORE_SIGMOID;
    // weights from the chosen experts alone (logistic scores, or renormalised softmax) are
    // computed for up to 32/k consecutive tokens at once when the warp routes several; a warp
    // with one token (and plain softmax, which needs the whole row) writes each token directly
    const bool batched = (sigmoid || renormalize) && t_end - t_begin > 1;
    const int batch = batched ? 32 / k : 1;  // tokens per weight pass

    float b[EPL];  // this lane's selection biases, shared by all tokens
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        const int e = i * 32 + lane;
        b[i] = (has_bias && e < E) ? bias[e] : 0.0f;
    }
    bool can_filter;
    const float eps = filter_margin(b, EPL, has_bias, &can_filter);
    float lg[EPL];  // logits of the token being routed, then of the next one (prefetch)
    prefetch_row<EPL>(logits + t_begin * E, E, lane, lg);

    int64_t t_batch = t_begin;  // first token of the open weight batch
    for (int64_t t = t_begin; t < t_end; ++t) {
        const float* row = logits + t * E;
        const int slot = static_cast<int>(t - t_batch);
        int C = 33;  // > 32: full path
        if (can_filter) {
            uint32_t u[EPL], bal[EPL];
            gate::approx_images<EPL>(lg, b, has_bias, E, lane, u);
            uint32_t lane_max = u[0];
#pragma unroll
            for (int i = 1; i < EPL; ++i) lane_max = max(lane_max, u[i]);
            uint32_t theta = gate::group_threshold(lane_max, k);
            if (theta != 0) C = gate::count_candidates<EPL>(u, cut_of(theta, has_bias, eps), bal);
            if (C > 32) {
                theta = gate::kth_lane_max(lane_max, k);
                if (theta != 0) C = gate::count_candidates<EPL>(u, cut_of(theta, has_bias, eps), bal);
            }
            if (C <= 32) gate::gather_candidates<EPL>(bal, lg, lane, cand);
        }
        if (C > 32) {  // full path (the current logits are still in lg)
            uint64_t v[EPL];
            gate::build_keys<EPL>(lg, b, has_bias, E, lane, v);
            if (t + 1 < t_end) prefetch_row<EPL>(row + E, E, lane, lg);
            const int my_e = gate::select_topk<EPL>(v, k, lane);
            if (!batched) {
                gate::write_choice<EPL>(row, my_e, E, k, score_fn, renormalize, lane,
                                        topk_idx + t * k, topk_w + t * k);
                continue;
            }
            if (lane < k) {
                cand.by_rank[slot * k + lane] = my_e;
                cand.l_by_rank[slot * k + lane] = row[my_e];
            }
        } else {
            // the candidates are captured: start the next token's loads
            if (t + 1 < t_end) prefetch_row<EPL>(row + E, E, lane, lg);
            // exact keys of the candidates, one per lane
            int e = 0;
            float l = 0.0f;
            uint32_t hi = 0, lo = 0;
            if (lane < C) {
                const uint2 el = cand.el[lane];
                e = static_cast<int>(el.x);
                l = __uint_as_float(el.y);
                const float key = has_bias ? __fadd_rn(gate::key_sigmoidf(l), __ldg(bias + e)) : l;
                hi = gate::ordered_key(key);
                lo = ~static_cast<uint32_t>(e);
            }
            // k rounds: the largest key, ties to the lower expert index; the winner keeps its rank
            int rank = k;
            const uint32_t top = __reduce_max_sync(kFullMask, hi);
            const uint32_t bottom = __reduce_min_sync(kFullMask, lane < C ? hi : 0xFFFFFFFFu);
            if (top - bottom < (1u << 26)) {
                // one reduction per round: the key's offset above the lowest candidate key and the
                // lane (candidates sit in ascending expert order, so a lower lane is a lower
                // index) packed into one word that orders like (key, -index); 0 marks "taken"
                uint32_t p = lane < C ? ((hi - bottom + 1u) << 5) | static_cast<uint32_t>(31 - lane) : 0u;
                for (int j = 0; j < k; ++j) {
                    if (p == __reduce_max_sync(kFullMask, p)) {
                        rank = j;
                        p = 0;
                    }
                }
            } else {
                for (int j = 0; j < k; ++j) {
                    const uint32_t m = __reduce_max_sync(kFullMask, hi);
                    const uint32_t win = __reduce_max_sync(kFullMask, hi == m ? lo : 0u);
                    if (hi == m && lo == win) {
                        rank = j;
                        hi = 0;
                    }
                }
            }
            const bool chosen = rank < k;
            if (!batched) {  // softmax weights need the whole row: lane j takes the j-th expert
                if (chosen) cand.by_rank[rank] = e;
                __syncwarp();
                const int my_e = lane < k ? cand.by_rank[lane] : 0;
                gate::write_choice<EPL>(row, my_e, E, k, score_fn, renormalize, lane,
                                        topk_idx + t * k, topk_w + t * k);
                continue;
            }
            if (chosen) {
                cand.by_rank[slot * k + rank] = e;
                cand.l_by_rank[slot * k + rank] = l;
            }
        }
        if (slot + 1 == batch || t + 1 == t_end) {
            gate::write_batch(cand, slot + 1, k, score_fn, renormalize, lane, topk_idx + t_batch * k,
                              topk_w + t_batch * k);
            t_batch = t + 1;
        }
    }
}

template <int EPL, bool kFull>
cudaError_t launch_gate(const float* logits, const float* bias, int T, int E, int k, int score_fn,
                        int renormalize, int32_t* idx, float* w, cudaStream_t s) {
    // one wave: as many warps as fit on the GPU at once, each taking a run of consecutive tokens
    static std::atomic<int> resident[kMaxDevices];
    const int dev = current_device();
    int resident_warps = resident[dev].load(std::memory_order_acquire);
    if (resident_warps == 0) {
        int per_sm = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, gate_topk_kernel<EPL, kFull>,
                                                          kGateWarps * 32, 0) != cudaSuccess || per_sm < 1)
            per_sm = 1;
        resident_warps = per_sm * kGateWarps * num_sms();
        resident[dev].store(resident_warps, std::memory_order_release);
    }
    const int warps = min(T, resident_warps);
    const dim3 grid((warps + kGateWarps - 1) / kGateWarps);
    return launch_pdl(gate_topk_kernel<EPL, kFull>, grid, dim3(kGateWarps * 32), 0, s, logits, bias, T, E,
                      k, score_fn, renormalize, warps, idx, w);
}

template <int EPL>
cudaError_t launch_gate_epl(const float* logits, const float* bias, int T, int E, int k, int score_fn,
                            int renormalize, int32_t* idx, float* w, cudaStream_t s) {
    if (E == 32 * EPL)
        return launch_gate<EPL, true>(logits, bias, T, E, k, score_fn, renormalize, idx, w, s);
    return launch_gate<EPL, false>(logits, bias, T, E, k, score_fn, renormalize, idx, w, s);
}

// Largest |approx_sigmoidf(l) - key_sigmoidf(l)| over the finite fp32 l with |l| <= 2^7: the
// positive-and-negative bit patterns below 0x43000001 (2^7), grid-stride.
__global__ void __launch_bounds__(256) gate_margin_kernel(uint32_t* max_err_bits) {
    constexpr uint32_t kLimit = 0x43000001u;  // bit patterns of [0, 2^7]
    uint32_t worst = 0;
    const uint64_t n = 2ull * kLimit;
    for (uint64_t i = static_cast<uint64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<uint64_t>(gridDim.x) * blockDim.x) {
        const uint32_t mag = static_cast<uint32_t>(i >> 1);
        const float l = __uint_as_float(mag | (static_cast<uint32_t>(i & 1) << 31));
        const float d = fabsf(gate::approx_sigmoidf(l) - gate::key_sigmoidf(l));
        worst = max(worst, __float_as_uint(d));  // non-negative floats order like their bits
    }
    worst = __reduce_max_sync(kFullMask, worst);
    if ((threadIdx.x & 31) == 0) atomicMax(max_err_bits, worst);
}

}  // namespace
}  // namespace tk

extern "C" tk_status tk_selftest_gate_margin(float* max_err, void* stream) {
    using namespace tk;
    if (max_err == nullptr) return fail_arg("tk_selftest_gate_margin: max_err must not be NULL");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t err = cudaMemsetAsync(max_err, 0, sizeof(float), s);
    if (err != cudaSuccess) return check_launch(err, "tk_selftest_gate_margin: cudaMemsetAsync");
    gate_margin_kernel<<<num_sms() * 8, 256, 0, s>>>(reinterpret_cast<uint32_t*>(max_err));
    return check_launch(cudaGetLastError(), "gate_margin_kernel");
}

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
    if (epl <= 1) err = launch_gate_epl<1>(logits, bias, T, E, k, score_fn, renormalize, topk_idx, topk_w, s);
    else if (epl <= 2) err = launch_gate_epl<2>(logits, bias, T, E, k, score_fn, renormalize, topk_idx, topk_w, s);
    else if (epl <= 4) err = launch_gate_epl<4>(logits, bias, T, E, k, score_fn, renormalize, topk_idx, topk_w, s);
    else if (epl <= 8) err = launch_gate_epl<8>(logits, bias, T, E, k, score_fn, renormalize, topk_idx, topk_w, s);
    else if (epl <= 16) err = launch_gate_epl<16>(logits, bias, T, E, k, score_fn, renormalize, topk_idx, topk_w, s);
    else err = launch_gate_epl<32>(logits, bias, T, E, k, score_fn, renormalize, topk_idx, topk_w, s);
    return check_launch(err, "gate_topk_kernel");
}
