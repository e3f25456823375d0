// Load-balance statistics and the tensor-parallel expert mask, the two small routing ops that
// the TileKernels moe/ module lists next to gating and expand/reduce (147227.xyz "刚刚！DeepSeek
// 开源高性能GPU算子库TileKernels", section "moe/": tensor-parallel mask, load-balance loss
// computation). The pages give no formulas; the readings are stated at the C declarations.
//
// Balance statistics, deterministic and in double:
//   balance_partial_kernel: one CTA per tile of 64 tokens, one warp per 4 tokens (per 8 when
//     E > 256, to bound registers). Each lane holds experts lane, lane+32, ... of a token,
//     normalises their unbiased scores over the row (warp reductions) and adds them into
//     per-lane double accumulators, loading the next token's logits meanwhile; the CTA then
//     sums its warps in order and writes one row of a [tiles x E] partial-sum matrix. Up to
//     256 experts, the scores' exponentials and reciprocals take a short double-precision path
//     (below) for arguments of magnitude <= 708 and the library's exp and division beyond.
//   balance_final_kernel: one CTA sums each column (up to 8 threads per column, each over a
//     contiguous range of tiles with 16 loads in flight, the range sums then added in order),
//     forms P, f and the loss with a fixed-order tree. The grouping depends on T and E only, so
//     results do not depend on the GPU.
// Over several data-parallel ranks the same statistics of the whole batch come from
// tk_balance_score_sums (each rank's column sums, in tile order) + an all-reduce of the sums,
// the counts and T + tk_balance_finalize (the final kernel over one "tile" of summed values).
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "tk_device.cuh"

namespace tk {
namespace {

constexpr int kStatTileTokens = 64;
constexpr int kFinalThreads = 1024;
constexpr int kMaxColumnSplit = 8;

// Warps of a partial CTA: 16 (4 tokens each) while a lane's experts fit in few registers, else 8
// (8 tokens each). More warps hide the latency of the double exponential's dependent chain; the
// tile of 64 tokens, and so the partial matrix, is the same either way.
template <int EPL>
__host__ __device__ constexpr int stat_warps() { return EPL <= 8 ? 16 : 8; }

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(kFullMask, v, off);
    return v;
}

__device__ __forceinline__ float warp_max_f(float v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(kFullMask, v, off));
    return v;
}

// Double-precision e^x for |x| <= kFastExpLimit by Tang's table-driven method (P. T. P. Tang,
// "Table-driven implementation of the exponential function in IEEE floating-point arithmetic",
// ACM TOMS 15(2), 1989): x = (32 m + j) ln2/32 + r with |r| <= ln2/64, so
// e^x = 2^m * 2^(j/32) * e^r; e^r - 1 is its Taylor polynomial of degree 6 (the omitted terms
// are below 2^-60 relative), 2^(j/32) comes from a 32-entry table, and 2^m is added to the
// exponent field (the result stays a normal number in this range). n = 32 m + j is x * 32/ln2
// rounded to the nearest integer by adding and subtracting 1.5 * 2^52; ln2/32 is split into a
// 37-bit head, whose product with |n| < 2^16 is exact, and a tail.
constexpr double kFastExpLimit = 708.0;

__device__ __forceinline__ double exp_table_driven(double x, const double* __restrict__ two_j32) {
    constexpr double kShift = 0x1.8p52;                 // 1.5 * 2^52
    constexpr double k32OverLn2 = 0x1.71547652b82fep+5;  // 32 / ln2
    constexpr double kLn2Over32Hi = 0x1.62e42fefa0000p-6;
    constexpr double kLn2Over32Lo = 0x1.cf79abc9e3b3ap-45;
    const double shifted = fma(x, k32OverLn2, kShift);
    const int n = __double2loint(shifted);              // the rounded x * 32/ln2, two's complement
    const double nd = shifted - kShift;
    double r = fma(-nd, kLn2Over32Hi, x);
    r = fma(-nd, kLn2Over32Lo, r);
    double p = 1.0 / 720.0;
    p = fma(p, r, 1.0 / 120.0);
    p = fma(p, r, 1.0 / 24.0);
    p = fma(p, r, 1.0 / 6.0);
    p = fma(p, r, 0.5);
    p = fma(p, r, 1.0);
    p *= r;                                              // e^r - 1
    const double t = two_j32[n & 31];
    const double y = fma(t, p, t);                       // 2^(j/32) e^r, in [0.98, 2.03)
    const int exponent_add = static_cast<int>(static_cast<uint32_t>(n >> 5) << 20);  // 2^m
    return __hiloint2double(__double2hiint(y) + exponent_add, __double2loint(y));
}

// 1/d for d >= 1 of moderate size: the hardware approximation refined by two Newton-Raphson
// steps y <- y + y (1 - d y), each of which squares the relative error.
__device__ __forceinline__ double reciprocal_newton(double d) {
    double y;
    asm("rcp.approx.ftz.f64 %0, %1;" : "=d"(y) : "d"(d));
    y = fma(y, fma(-d, y, 1.0), y);
    return fma(y, fma(-d, y, 1.0), y);
}

// The unbiased logistic score 1/(1 + e^-l) and the softmax numerator e^x (x = l - max <= 0).
// The short path takes its argument clamped to the fast range, so it is safe (and branch-free,
// letting a lane's experts interleave) for any input; in_short_range says whether its result
// stands, else the library form below replaces it.
__device__ __forceinline__ bool logistic_in_short_range(float l) {
    return fabsf(l) <= static_cast<float>(kFastExpLimit);  // false for NaN
}
__device__ __forceinline__ double logistic_short(float l, const double* __restrict__ two_j32) {
    const double x = fmin(fmax(-static_cast<double>(l), -kFastExpLimit), kFastExpLimit);
    return reciprocal_newton(1.0 + exp_table_driven(x, two_j32));
}
__device__ __forceinline__ double logistic_library(float l) {
    return 1.0 / (1.0 + exp(-static_cast<double>(l)));
}
__device__ __forceinline__ double logistic_score(float l, const double* __restrict__ two_j32) {
    return logistic_in_short_range(l) ? logistic_short(l, two_j32) : logistic_library(l);
}
__device__ __forceinline__ bool numerator_in_short_range(double x) { return x >= -kFastExpLimit; }
__device__ __forceinline__ double numerator_short(double x, const double* __restrict__ two_j32) {
    return exp_table_driven(fmin(fmax(x, -kFastExpLimit), 0.0), two_j32);
}

// Fills the 2^(j/32) table of a CTA (the library's exp2, within an ulp); the caller syncs.
__device__ __forceinline__ void fill_two_j32(double* two_j32) {
    if (threadIdx.x < 32) two_j32[threadIdx.x] = exp2(static_cast<double>(threadIdx.x) / 32.0);
}

// One token's logits, lane-strided (experts lane, lane+32, ...); -inf past E or past T.
template <int EPL>
__device__ __forceinline__ void load_logits(const float* __restrict__ logits, int64_t t, int T, int E,
                                            int lane, float (&l)[EPL]) {
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        const int e = i * 32 + lane;
        l[i] = (t < T && e < E) ? logits[t * E + e] : -INFINITY;
    }
}

// Rows [c0, c1) of column e of a [tiles x E] matrix of doubles, summed in row order. The loads of
// 16 rows go out together before their additions, so the range costs (c1-c0)/16 memory round
// trips instead of one per few rows; the additions are those of a plain loop over c.
__device__ __forceinline__ double column_range_sum(const double* __restrict__ partial, int c0, int c1,
                                                   int E, int e) {
    constexpr int kBatch = 16;
    double sum = 0.0;
    int c = c0;
    for (; c + kBatch <= c1; c += kBatch) {
        double v[kBatch];
#pragma unroll
        for (int j = 0; j < kBatch; ++j) v[j] = partial[static_cast<int64_t>(c + j) * E + e];
#pragma unroll
        for (int j = 0; j < kBatch; ++j) sum += v[j];
    }
    for (; c < c1; ++c) sum += partial[static_cast<int64_t>(c) * E + e];
    return sum;
}

// Column sums of a [tiles x E] partial matrix by one CTA of kFinalThreads threads, into
// out[e] for e < E (shared memory or global). With E small enough, S = min(kFinalThreads / E,
// kMaxColumnSplit) threads share a column: thread (s, e) sums rows [s*chunk, (s+1)*chunk), and
// the S range sums are added in order s = 0, 1, ... Every kernel that sums a partial matrix
// calls this with the same block size, so equal inputs give equal bits; the grouping depends on
// tiles and E only. Ends with __syncthreads().
__device__ __forceinline__ void column_sums(const double* __restrict__ partial, int tiles, int E,
                                            double* __restrict__ split /* [kMaxColumnSplit*E] smem, E <= kFinalThreads */,
                                            double* __restrict__ out) {
    int S = kFinalThreads / E;
    if (S > kMaxColumnSplit) S = kMaxColumnSplit;
    if (S < 1) S = 1;
    const int chunk = (tiles + S - 1) / S;
    for (int i = threadIdx.x; i < S * E; i += blockDim.x) {
        const int e = i % E;
        const int sp = i / E;
        int c0 = sp * chunk, c1 = c0 + chunk;
        if (c0 > tiles) c0 = tiles;
        if (c1 > tiles) c1 = tiles;
        split[sp * E + e] = column_range_sum(partial, c0, c1, E, e);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        double v = 0.0;
        for (int sp = 0; sp < S; ++sp) v += split[sp * E + e];
        out[e] = v;
    }
    __syncthreads();
}

// The short path for up to 8 experts per lane: its branch-free form interleaves a lane's experts,
// which at 16 or 32 experts per lane would spill; those forms call the library per expert.
template <int EPL>
constexpr bool kShortPath = EPL <= 8;

template <int EPL>
__global__ void __launch_bounds__(stat_warps<EPL>() * 32, EPL == 16 ? 2 : 1)
balance_partial_kernel(const float* __restrict__ logits, int T, int E, int score_fn,
                       double* __restrict__ partial) {
    constexpr int kStatWarps = stat_warps<EPL>();
    constexpr int kStatTokensPerWarp = kStatTileTokens / kStatWarps;
    extern __shared__ double wsum[];  // [kStatWarps][E]
    __shared__ double two_j32[32];
    fill_two_j32(two_j32);
    __syncthreads();
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    double acc[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) acc[i] = 0.0;
    const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kStatTileTokens + warp * kStatTokensPerWarp;
    // the next token's logits are loaded while this token's scores are computed
    float l[EPL], nxt[EPL];
    load_logits<EPL>(logits, t0, T, E, lane, l);
    for (int q = 0; q < kStatTokensPerWarp; ++q) {
        const int64_t t = t0 + q;
        if (t >= T) break;
        // (past this warp's last token nothing is loaded: T stands for "no token")
        load_logits<EPL>(logits, q + 1 < kStatTokensPerWarp ? t + 1 : static_cast<int64_t>(T), T, E,
                         lane, nxt);
        double s[EPL];
        double z = 0.0;
        if (score_fn == TK_SCORE_SOFTMAX) {
            float m = -INFINITY;
#pragma unroll
            for (int i = 0; i < EPL; ++i) m = fmaxf(m, l[i]);
            m = warp_max_f(m);
            if constexpr (kShortPath<EPL>) {
                bool slow = false;
#pragma unroll
                for (int i = 0; i < EPL; ++i) {
                    const double x = static_cast<double>(l[i]) - static_cast<double>(m);
                    s[i] = numerator_short(x, two_j32);
                    slow = slow || (i * 32 + lane < E && !numerator_in_short_range(x));
                }
                if (__any_sync(kFullMask, slow)) {
#pragma unroll
                    for (int i = 0; i < EPL; ++i) {
                        const double x = static_cast<double>(l[i]) - static_cast<double>(m);
                        if (!numerator_in_short_range(x)) s[i] = exp(x);
                    }
                }
            } else {
#pragma unroll
                for (int i = 0; i < EPL; ++i)
                    s[i] = i * 32 + lane < E ? exp(static_cast<double>(l[i]) - static_cast<double>(m)) : 0.0;
            }
        } else {
            if constexpr (kShortPath<EPL>) {
                bool slow = false;
#pragma unroll
                for (int i = 0; i < EPL; ++i) {
                    s[i] = logistic_short(l[i], two_j32);
                    slow = slow || (i * 32 + lane < E && !logistic_in_short_range(l[i]));
                }
                if (__any_sync(kFullMask, slow)) {
#pragma unroll
                    for (int i = 0; i < EPL; ++i)
                        if (!logistic_in_short_range(l[i])) s[i] = logistic_library(l[i]);
                }
            } else {
#pragma unroll
                for (int i = 0; i < EPL; ++i) s[i] = i * 32 + lane < E ? logistic_library(l[i]) : 0.0;
            }
        }
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
            if (kShortPath<EPL> && i * 32 + lane >= E) s[i] = 0.0;
            z += s[i];
        }
        const double rz = 1.0 / warp_sum_d(z);
#pragma unroll
        for (int i = 0; i < EPL; ++i) acc[i] += s[i] * rz;
#pragma unroll
        for (int i = 0; i < EPL; ++i) l[i] = nxt[i];
    }
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        const int e = i * 32 + lane;
        if (e < E) wsum[warp * E + e] = acc[i];
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        double v = 0.0;
#pragma unroll
        for (int w = 0; w < kStatWarps; ++w) v += wsum[w * E + e];
        partial[static_cast<int64_t>(blockIdx.x) * E + e] = v;
    }
}

static_assert(TK_MAX_EXPERTS <= kFinalThreads, "column_sums' split buffer holds kFinalThreads doubles");

__global__ void __launch_bounds__(kFinalThreads)
balance_final_kernel(const double* __restrict__ partial, int tiles, const int32_t* __restrict__ counts,
                     int64_t T, int E, int k, float* __restrict__ P, float* __restrict__ f,
                     float* __restrict__ loss) {
    __shared__ double split[kFinalThreads];
    __shared__ double sums[TK_MAX_EXPERTS];
    __shared__ double prod[kFinalThreads];
    pdl_wait();
    column_sums(partial, tiles, E, split, sums);
    // each thread owns experts e = threadIdx.x + i * blockDim.x and keeps their f*P sum
    double mine = 0.0;
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        const double Pe = T > 0 ? sums[e] / static_cast<double>(T) : 0.0;
        const double fe = T > 0 ? static_cast<double>(E) * counts[e] / (static_cast<double>(k) * static_cast<double>(T)) : 0.0;
        P[e] = static_cast<float>(Pe);
        f[e] = static_cast<float>(fe);
        mine += fe * Pe;
    }
    prod[threadIdx.x] = mine;
    __syncthreads();
    for (int half = blockDim.x / 2; half > 0; half >>= 1) {  // fixed-order pairwise tree
        if (threadIdx.x < half) prod[threadIdx.x] += prod[threadIdx.x + half];
        __syncthreads();
    }
    if (threadIdx.x == 0) *loss = static_cast<float>(prod[0]);
}

// Column sums of the partial matrix (the same additions as the final kernel).
__global__ void __launch_bounds__(kFinalThreads)
balance_colsum_kernel(const double* __restrict__ partial, int tiles, int E, double* __restrict__ sums) {
    __shared__ double split[kFinalThreads];
    pdl_wait();
    column_sums(partial, tiles, E, split, sums);
}

template <int EPL>
cudaError_t launch_partial(const float* logits, int T, int E, int score_fn, double* partial,
                           int tiles, cudaStream_t s) {
    constexpr int kStatWarps = stat_warps<EPL>();
    const size_t smem = static_cast<size_t>(kStatWarps) * E * sizeof(double);
    static std::atomic<bool> configured[kMaxDevices];
    const int dev = current_device();
    if (smem > 48 * 1024 && !configured[dev].load(std::memory_order_acquire)) {
        std::lock_guard<std::mutex> lock(setup_mutex());
        const cudaError_t e = cudaFuncSetAttribute(balance_partial_kernel<EPL>,
                                                   cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   kStatWarps * TK_MAX_EXPERTS * static_cast<int>(sizeof(double)));
        if (e != cudaSuccess) return e;
        configured[dev].store(true, std::memory_order_release);
    }
    return launch_pdl(balance_partial_kernel<EPL>, dim3(tiles), dim3(kStatWarps * 32), smem, s,
                      logits, T, E, score_fn, partial);
}

// Largest relative differences, over every finite fp32 l with |l| <= kFastExpLimit, between the
// short path and the library: [0] e^-l (which covers e^x for the softmax numerators, x = -l),
// [1] the logistic score 1/(1 + e^-l). Positive doubles order like their bit patterns.
__global__ void __launch_bounds__(256) balance_exp_check_kernel(unsigned long long* max_rel_bits) {
    __shared__ double two_j32[32];
    fill_two_j32(two_j32);
    __syncthreads();
    const uint32_t limit = __float_as_uint(static_cast<float>(kFastExpLimit)) + 1u;  // bit patterns of [0, 708]
    const uint64_t n = 2ull * limit;
    double worst_exp = 0.0, worst_sig = 0.0;
    for (uint64_t i = static_cast<uint64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<uint64_t>(gridDim.x) * blockDim.x) {
        const uint32_t mag = static_cast<uint32_t>(i >> 1);
        const float l = __uint_as_float(mag | (static_cast<uint32_t>(i & 1) << 31));
        const double ref_e = exp(-static_cast<double>(l));
        const double ref_s = 1.0 / (1.0 + ref_e);
        const double e = exp_table_driven(-static_cast<double>(l), two_j32);
        const double sg = logistic_score(l, two_j32);
        worst_exp = fmax(worst_exp, fabs(e - ref_e) / ref_e);
        worst_sig = fmax(worst_sig, fabs(sg - ref_s) / ref_s);
    }
    unsigned long long be = __double_as_longlong(worst_exp), bs = __double_as_longlong(worst_sig);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        be = max(be, __shfl_xor_sync(kFullMask, be, off));
        bs = max(bs, __shfl_xor_sync(kFullMask, bs, off));
    }
    if ((threadIdx.x & 31) == 0) {
        atomicMax(max_rel_bits, be);
        atomicMax(max_rel_bits + 1, bs);
    }
}

__global__ void tp_mask_kernel(const int32_t* __restrict__ in, int64_t n, int lo, int el,
                               int32_t* __restrict__ out) {
    pdl_wait();
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int e = in[i];
        out[i] = (e >= lo && e < lo + el) ? e - lo : -1;
    }
}

int stat_tiles(int T) { return (T + kStatTileTokens - 1) / kStatTileTokens; }

cudaError_t launch_partials(const float* logits, int T, int E, int score_fn, double* partial,
                            int tiles, cudaStream_t s) {
    const int epl = (E + 31) / 32;
    if (epl <= 1) return launch_partial<1>(logits, T, E, score_fn, partial, tiles, s);
    if (epl <= 2) return launch_partial<2>(logits, T, E, score_fn, partial, tiles, s);
    if (epl <= 4) return launch_partial<4>(logits, T, E, score_fn, partial, tiles, s);
    if (epl <= 8) return launch_partial<8>(logits, T, E, score_fn, partial, tiles, s);
    if (epl <= 16) return launch_partial<16>(logits, T, E, score_fn, partial, tiles, s);
    return launch_partial<32>(logits, T, E, score_fn, partial, tiles, s);
}

}  // namespace
}  // namespace tk

extern "C" size_t tk_balance_stats_workspace_bytes(int T, int E) {
    if (T < 0 || E < 1) return 0;
    const int tiles = tk::stat_tiles(T) > 0 ? tk::stat_tiles(T) : 1;
    return static_cast<size_t>(tiles) * static_cast<size_t>(E) * sizeof(double);
}

extern "C" tk_status tk_balance_stats(const float* logits, const int32_t* counts, int T, int E,
                                      int k, int score_fn, float* P, float* f, float* loss,
                                      void* workspace, size_t workspace_bytes, void* stream) {
    using namespace tk;
    if (T < 0) return fail_arg("tk_balance_stats: T=%d must be >= 0", T);
    if (E < 1 || E > TK_MAX_EXPERTS) return fail_arg("tk_balance_stats: E=%d outside [1, %d]", E, TK_MAX_EXPERTS);
    if (k < 1 || k > E || k > TK_MAX_TOPK)
        return fail_arg("tk_balance_stats: k=%d outside [1, min(E=%d, %d)]", k, E, TK_MAX_TOPK);
    if (score_fn != TK_SCORE_SOFTMAX && score_fn != TK_SCORE_SIGMOID)
        return fail_arg("tk_balance_stats: unknown score_fn %d", score_fn);
    if (counts == nullptr || P == nullptr || f == nullptr || loss == nullptr || workspace == nullptr)
        return fail_arg("tk_balance_stats: counts, P, f, loss and workspace must not be NULL");
    if (T > 0 && logits == nullptr) return fail_arg("tk_balance_stats: logits must not be NULL");
    const size_t need = tk_balance_stats_workspace_bytes(T, E);
    if (workspace_bytes < need)
        return fail_arg("tk_balance_stats: workspace holds %zu bytes, needs %zu", workspace_bytes, need);
    if (reinterpret_cast<uintptr_t>(workspace) % 16 != 0)
        return fail_arg("tk_balance_stats: workspace must be 16-byte aligned");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    double* partial = static_cast<double*>(workspace);
    const int tiles = stat_tiles(T);
    cudaError_t err = cudaSuccess;
    if (tiles > 0) {
        err = launch_partials(logits, T, E, score_fn, partial, tiles, s);
        if (err != cudaSuccess) return check_launch(err, "balance_partial_kernel");
    }
    err = launch_pdl(balance_final_kernel, dim3(1), dim3(kFinalThreads), 0, s,
                     static_cast<const double*>(partial), tiles, counts, static_cast<int64_t>(T), E,
                     k, P, f, loss);
    return check_launch(err, "balance_final_kernel");
}

extern "C" tk_status tk_balance_score_sums(const float* logits, int T, int E, int score_fn,
                                           double* sums, void* workspace, size_t workspace_bytes,
                                           void* stream) {
    using namespace tk;
    if (T < 0) return fail_arg("tk_balance_score_sums: T=%d must be >= 0", T);
    if (E < 1 || E > TK_MAX_EXPERTS) return fail_arg("tk_balance_score_sums: E=%d outside [1, %d]", E, TK_MAX_EXPERTS);
    if (score_fn != TK_SCORE_SOFTMAX && score_fn != TK_SCORE_SIGMOID)
        return fail_arg("tk_balance_score_sums: unknown score_fn %d", score_fn);
    if (sums == nullptr || workspace == nullptr)
        return fail_arg("tk_balance_score_sums: sums and workspace must not be NULL");
    if (T > 0 && logits == nullptr) return fail_arg("tk_balance_score_sums: logits must not be NULL");
    const size_t need = tk_balance_stats_workspace_bytes(T, E);
    if (workspace_bytes < need)
        return fail_arg("tk_balance_score_sums: workspace holds %zu bytes, needs %zu", workspace_bytes, need);
    if (reinterpret_cast<uintptr_t>(workspace) % 16 != 0)
        return fail_arg("tk_balance_score_sums: workspace must be 16-byte aligned");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    double* partial = static_cast<double*>(workspace);
    const int tiles = stat_tiles(T);
    if (tiles > 0) {
        const cudaError_t e = launch_partials(logits, T, E, score_fn, partial, tiles, s);
        if (e != cudaSuccess) return check_launch(e, "balance_partial_kernel");
    }
    const cudaError_t e = launch_pdl(balance_colsum_kernel, dim3(1), dim3(kFinalThreads), 0, s,
                                     static_cast<const double*>(partial), tiles, E, sums);
    return check_launch(e, "balance_colsum_kernel");
}

extern "C" tk_status tk_balance_finalize(const double* sums, const int32_t* counts, int64_t T,
                                         int E, int k, float* P, float* f, float* loss,
                                         void* stream) {
    using namespace tk;
    if (T < 0) return fail_arg("tk_balance_finalize: T=%lld must be >= 0", (long long)T);
    if (E < 1 || E > TK_MAX_EXPERTS) return fail_arg("tk_balance_finalize: E=%d outside [1, %d]", E, TK_MAX_EXPERTS);
    if (k < 1 || k > E || k > TK_MAX_TOPK)
        return fail_arg("tk_balance_finalize: k=%d outside [1, min(E=%d, %d)]", k, E, TK_MAX_TOPK);
    if (sums == nullptr || counts == nullptr || P == nullptr || f == nullptr || loss == nullptr)
        return fail_arg("tk_balance_finalize: sums, counts, P, f and loss must not be NULL");
    const cudaError_t e = launch_pdl(balance_final_kernel, dim3(1), dim3(kFinalThreads), 0,
                                     static_cast<cudaStream_t>(stream), sums, 1, counts, T, E, k, P,
                                     f, loss);
    return check_launch(e, "balance_final_kernel");
}

extern "C" tk_status tk_selftest_balance_exp(double* max_rel_err, void* stream) {
    using namespace tk;
    if (max_rel_err == nullptr) return fail_arg("tk_selftest_balance_exp: max_rel_err must not be NULL");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t err = cudaMemsetAsync(max_rel_err, 0, 2 * sizeof(double), s);
    if (err != cudaSuccess) return check_launch(err, "tk_selftest_balance_exp: cudaMemsetAsync");
    balance_exp_check_kernel<<<num_sms() * 8, 256, 0, s>>>(
        reinterpret_cast<unsigned long long*>(max_rel_err));
    return check_launch(cudaGetLastError(), "balance_exp_check_kernel");
}

extern "C" tk_status tk_tp_mask(const int32_t* topk_idx, int T, int k, int E, int tp_size,
                                int tp_rank, int32_t* out_idx, void* stream) {
    using namespace tk;
    if (T < 0) return fail_arg("tk_tp_mask: T=%d must be >= 0", T);
    if (k < 1 || k > TK_MAX_TOPK) return fail_arg("tk_tp_mask: k=%d outside [1, %d]", k, TK_MAX_TOPK);
    if (E < 1 || E > TK_MAX_EXPERTS) return fail_arg("tk_tp_mask: E=%d outside [1, %d]", E, TK_MAX_EXPERTS);
    if (tp_size < 1 || E % tp_size != 0)
        return fail_arg("tk_tp_mask: tp_size=%d must divide E=%d", tp_size, E);
    if (tp_rank < 0 || tp_rank >= tp_size)
        return fail_arg("tk_tp_mask: tp_rank=%d outside [0, %d)", tp_rank, tp_size);
    if (T == 0) return TK_OK;
    if (topk_idx == nullptr || out_idx == nullptr) return fail_arg("tk_tp_mask: NULL pointer");
    const int el = E / tp_size;
    const int64_t n = static_cast<int64_t>(T) * k;
    int64_t grid = (n + 255) / 256;
    const int64_t cap = static_cast<int64_t>(num_sms()) * 8;
    if (grid > cap) grid = cap;
    const cudaError_t err = launch_pdl(tp_mask_kernel, dim3(static_cast<unsigned>(grid)), dim3(256), 0,
                                       static_cast<cudaStream_t>(stream), topk_idx, n, tp_rank * el,
                                       el, out_idx);
    return check_launch(err, "tp_mask_kernel");
}
