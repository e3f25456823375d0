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
        uint64_t v[EPL];
        gate::build_keys<EPL>(lg, b, bias != nullptr, E, lane, v);
        if (t + 1 < t_end) {  // the registers are free again: start the next token's loads
#pragma unroll
            for (int i = 0; i < EPL; ++i) {
                const int e = i * 32 + lane;
                lg[i] = e < E ? row[E + e] : 0.0f;
            }
        }
        const int my_e = gate::select_topk<EPL>(v, k, lane);
        gate::write_choice<EPL>(row, my_e, E, k, score_fn, renormalize, lane, topk_idx + t * k,
                                topk_w + t * k);
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
