/*
 * tk_oracle.cpp -- TEST INFRASTRUCTURE ONLY (see tk_oracle.h).
 *
 * Plain single-threaded C++17. Build with -O2 -ffp-contract=off and without -ffast-math, so
 * every fp32 operation written here is exactly one IEEE round-to-nearest operation and fmaf
 * appears only where it is written. Nothing here is blocked, fused or reordered: each step is
 * the definition it cites, written out as a loop.
 */
#include "tk_oracle.h"

/* TKO_PLANT (default 0) compiles one deliberate mistake into the oracle; only the mutation test
 * (tests/test_oracle_mutations.py) builds such variants, to show that the pins catch each. */
#ifndef TKO_PLANT
#define TKO_PLANT 0
#endif

#include <algorithm>
#include <cmath>
#include <cstring>
#include <limits>
#include <vector>

namespace {

float bits_to_float(uint32_t u) { float f; std::memcpy(&f, &u, 4); return f; }
uint32_t float_to_bits(float f) { uint32_t u; std::memcpy(&u, &f, 4); return u; }

float bf16_to_float(uint16_t h) { return bits_to_float(static_cast<uint32_t>(h) << 16); }

/* 2^n as an fp32 value for n in [-126, 127] (built from the exponent field). */
float pow2f(int n) { return bits_to_float(static_cast<uint32_t>(n + 127) << 23); }

}  // namespace

extern "C" {

/* ------------------------------------------------------------------------------------------
 * fp32 exponential for the selection key.
 *
 * The pages give no formula for the sigmoid score, and two different fp32 exponentials can
 * disagree in the last bit, which can change which expert wins a near-tie. So the key's
 * exponential is pinned to one published method, stated here and written out independently in
 * the CUDA library: Cody & Waite's argument reduction (Cody and Waite, "Software Manual for the
 * Elementary Functions", 1980, exp chapter) followed by the Taylor series of e^r.
 *   n = rint(x * log2(e))                 (fp32 multiply, round to nearest even integer)
 *   r = fmaf(-n, LN2_HI, x); r = fmaf(-n, LN2_LO, r)
 *       LN2_HI = 0x1.62e4p-1 has 9 trailing zero bits, so n*LN2_HI is exact for |n| < 512;
 *       LN2_LO = ln 2 - LN2_HI rounded to fp32.
 *   p = 1 + r + r^2/2! + ... + r^7/7!      (Horner with fmaf; coefficients 1/i! rounded to fp32)
 *   e^x = p * 2^n1 * 2^n2 with n1 = n/2 (truncated), n2 = n - n1: the first product is exact,
 *       the second rounds once (so overflow gives +inf and deep underflow a correctly rounded
 *       subnormal or zero).
 * x is first clamped to [-110, 100]; e^-110 rounds to 0 and e^100 overflows, so the clamp does
 * not change any result. |r| <= ln2/2 + tiny, so the truncation error r^8/8! * e^|r| < 8e-9,
 * well under half an fp32 ulp; the tests bound the total error by 2 ulp against double exp.
 * ---------------------------------------------------------------------------------------- */
float tko_spec_expf(float x) {
    if (x != x) return x;
    if (x < -110.0f) x = -110.0f;
    if (x > 100.0f) x = 100.0f;
    const float kLog2e = 0x1.715476p+0f;
    const float kLn2Hi = 0x1.62e4p-1f;
    const float kLn2Lo = 0x1.7f7d1cp-20f;
    const float n = std::rint(x * kLog2e);
    float r = std::fmaf(-n, kLn2Hi, x);
    r = std::fmaf(-n, kLn2Lo, r);
    float p = 0x1.a01a02p-13f;            /* 1/7! */
#if TKO_PLANT == 1
    p = std::fmaf(p, r, 0.0f);            /* planted: 1/6! dropped */
#else
    p = std::fmaf(p, r, 0x1.6c16c2p-10f); /* 1/6! */
#endif
    p = std::fmaf(p, r, 0x1.111112p-7f);  /* 1/5! */
    p = std::fmaf(p, r, 0x1.555556p-5f);  /* 1/4! */
    p = std::fmaf(p, r, 0x1.555556p-3f);  /* 1/3! */
    p = std::fmaf(p, r, 0.5f);            /* 1/2! */
    p = std::fmaf(p, r, 1.0f);            /* 1/1! */
    p = std::fmaf(p, r, 1.0f);            /* 1/0! */
    const int ni = static_cast<int>(n);
    const int n1 = ni / 2;
    const int n2 = ni - n1;
    return (p * pow2f(n1)) * pow2f(n2);
}

void tko_spec_expf_array(const float* x, float* y, int64_t n) {
    for (int64_t i = 0; i < n; ++i) y[i] = tko_spec_expf(x[i]);
}

/* Logistic score s = 1 / (1 + e^-l), three fp32 operations after the exponential. */
float tko_spec_sigmoidf(float l) {
    const float e = tko_spec_expf(-l);
    const float d = 1.0f + e;
    return 1.0f / d;
}

void tko_spec_sigmoidf_array(const float* x, float* y, int64_t n) {
    for (int64_t i = 0; i < n; ++i) y[i] = tko_spec_sigmoidf(x[i]);
}

/* ------------------------------------------------------------------------------------------
 * fp32 -> E4M3 (OCP FP8: 1 sign, 4 exponent bits with bias 7, 3 mantissa bits; no infinity;
 * largest finite magnitude 1.75 * 2^8 = 448; subnormals m * 2^-9). Round to nearest, ties to
 * even; magnitudes above 448 saturate to 448; the sign is kept, so a negative value that
 * rounds to zero gives the code 0x80. NaN gives 0x7F with its sign.
 * The rounding works on the exact grid: a / quantum is exact in fp32 because the quantum is a
 * power of two, and rint() rounds it to the nearest even integer.
 * ---------------------------------------------------------------------------------------- */
uint8_t tko_e4m3_encode(float v) {
    const uint32_t bits = float_to_bits(v);
    const uint8_t sign = static_cast<uint8_t>((bits >> 31) << 7);
    const float a = std::fabs(v);
    if (a != a) return static_cast<uint8_t>(sign | 0x7F);
    if (a >= 448.0f) return static_cast<uint8_t>(sign | 0x7E);
    if (a < 0x1p-6f) {                             /* subnormal range, quantum 2^-9 */
        const float m = std::rint(a * 512.0f);    /* 0..8 */
        return static_cast<uint8_t>(sign | static_cast<uint8_t>(m)); /* m == 8 is code 0x08 = 2^-6 */
    }
    int e = static_cast<int>((float_to_bits(a) >> 23) & 0xFF) - 127; /* floor(log2 a), -6..8 */
    const float quantum = pow2f(e - 3);
#if TKO_PLANT == 6
    int m = static_cast<int>(std::round(a / quantum)); /* planted: ties away from zero */
#else
    int m = static_cast<int>(std::rint(a / quantum)); /* 8..16 */
#endif
    if (m == 16) { m = 8; e += 1; }
    return static_cast<uint8_t>(sign | ((e + 7) << 3) | (m - 8));
}

void tko_e4m3_encode_array(const float* x, uint8_t* y, int64_t n) {
    for (int64_t i = 0; i < n; ++i) y[i] = tko_e4m3_encode(x[i]);
}

/* fp32 -> bf16 keeping the upper 16 bits after round to nearest even of the lower 16. */
uint16_t tko_bf16_rne(float f) {
    uint32_t u = float_to_bits(f);
    if ((u & 0x7FFFFFFFu) > 0x7F800000u) return static_cast<uint16_t>((u >> 16) | 0x40u);
#if TKO_PLANT == 9
    const uint32_t lsb = 0u; u += 0u * lsb;  /* planted: truncation */
#else
    const uint32_t lsb = (u >> 16) & 1u;
    u += 0x7FFFu + lsb;
#endif
    return static_cast<uint16_t>(u >> 16);
}

void tko_bf16_rne_array(const float* x, uint16_t* y, int64_t n) {
    for (int64_t i = 0; i < n; ++i) y[i] = tko_bf16_rne(x[i]);
}

/* ------------------------------------------------------------------------------------------
 * Gate: scoring, top-k selection, renormalisation.
 * The TileKernels feature lists (機器之心 "Tile Kernels" section; 147227.xyz "moe/" section)
 * name top-k expert selection with scoring and weight normalisation; the zhichai.net essay's
 * "MoE TopK 门控" sketch selects by k rounds of max/argmax, lower index on ties, writing the
 * winners in round order. A stable sort by key, descending, gives exactly that order.
 *  - key: with no bias the key is the logit itself (softmax and sigmoid are strictly
 *    increasing, so this ranks the exact scores); with a bias (sigmoid only) the key is the
 *    fp32 value sigmoid(l) + b, using tko_spec_sigmoidf. NaN keys rank as -inf.
 *  - weights: the unbiased score of each chosen expert in double -- softmax probability
 *    exp(l_e - max)/sum over all E, or 1/(1+exp(-l_e)) -- divided by the sum over the k chosen
 *    when renormalize != 0, then rounded to fp32. A zero sum gives zero weights.
 * ---------------------------------------------------------------------------------------- */
int tko_gate_topk(const float* logits, const float* bias, int T, int E, int k, int score_fn,
                  int renormalize, int32_t* topk_idx, float* topk_w) {
    if (T < 0 || E < 1 || k < 1 || k > E) return -1;
    if (score_fn != TKO_SCORE_SOFTMAX && score_fn != TKO_SCORE_SIGMOID) return -1;
    if (score_fn == TKO_SCORE_SOFTMAX && bias != nullptr) return -2;
    if (T > 0 && (logits == nullptr || topk_idx == nullptr || topk_w == nullptr)) return -1;
    const float ninf = -std::numeric_limits<float>::infinity();
    std::vector<float> key(E);
    std::vector<int> order(E);
    for (int t = 0; t < T; ++t) {
        const float* l = logits + static_cast<int64_t>(t) * E;
        for (int e = 0; e < E; ++e) {
            float kv = l[e];
            if (bias != nullptr) kv = tko_spec_sigmoidf(l[e]) + bias[e];
            if (kv != kv) kv = ninf;
            key[e] = kv;
            order[e] = e;
        }
#if TKO_PLANT == 2
        std::stable_sort(order.begin(), order.end(),  /* planted: ties to the higher index */
                         [&](int a, int b) { return key[a] > key[b] || (key[a] == key[b] && a > b); });
#else
        std::stable_sort(order.begin(), order.end(),
                         [&](int a, int b) { return key[a] > key[b]; });
#endif
        std::vector<double> s(k);
        if (score_fn == TKO_SCORE_SIGMOID) {
            for (int j = 0; j < k; ++j) {
                const double lj = static_cast<double>(l[order[j]]);
                s[j] = 1.0 / (1.0 + std::exp(-lj));
#if TKO_PLANT == 3
                if (bias != nullptr) s[j] += bias[order[j]];  /* planted: biased weights */
#endif
            }
        } else {
            double m = -std::numeric_limits<double>::infinity();
            for (int e = 0; e < E; ++e) m = std::max(m, static_cast<double>(l[e]));
            if (m == -std::numeric_limits<double>::infinity()) {
                for (int j = 0; j < k; ++j) s[j] = 0.0;
            } else {
                double z = 0.0;
                for (int e = 0; e < E; ++e) z += std::exp(static_cast<double>(l[e]) - m);
                for (int j = 0; j < k; ++j) s[j] = std::exp(static_cast<double>(l[order[j]]) - m) / z;
            }
        }
        double denom = 1.0;
        if (renormalize) {
#if TKO_PLANT != 17
            denom = 0.0;
            for (int j = 0; j < k; ++j) denom += s[j];
#endif  /* (plant 17: the renormalisation is skipped) */
        }
        for (int j = 0; j < k; ++j) {
            topk_idx[static_cast<int64_t>(t) * k + j] = order[j];
            topk_w[static_cast<int64_t>(t) * k + j] =
                denom == 0.0 ? 0.0f : static_cast<float>(s[j] / denom);
        }
    }
    return 0;
}

int64_t tko_max_rows(int T, int E, int k, int align) {
    return static_cast<int64_t>(T) * k + static_cast<int64_t>(E) * (align - 1);
}

/* ------------------------------------------------------------------------------------------
 * Token-to-expert map (機器之心 "Tile Kernels" feature list: token-to-expert mapping).
 * Pair p = t*k + j. One pass counts, a scan places each expert's segment (rounded up to a
 * multiple of align, padding rows keep token -1), a second pass in p order hands out slots, so
 * each segment lists its tokens in increasing order (a stable expert-major permutation).
 * Expert -1 marks a masked pair (see tko_tp_mask): skipped without being an error.
 * ---------------------------------------------------------------------------------------- */
int tko_route_map(const int32_t* topk_idx, int T, int E, int k, int align, int32_t* counts,
                  int32_t* offsets, int32_t* slot_of, int32_t* token_of) {
    if (T < 0 || E < 1 || k < 1 || align < 1) return -1;
    const int64_t pairs = static_cast<int64_t>(T) * k;
    const int64_t rmax = tko_max_rows(T, E, k, align);
    int bad = 0;
    for (int e = 0; e < E; ++e) counts[e] = 0;
    for (int64_t p = 0; p < pairs; ++p) {
        const int e = topk_idx[p];
        if (e < 0 || e >= E) {
            if (e != -1) bad = 1;  /* -1 = masked pair, not an error */
            continue;
        }
        counts[e] += 1;
    }
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) {
#if TKO_PLANT == 4
        const int32_t padded = (counts[e] / align + 1) * align;  /* planted: off-by-one rounding */
#else
        const int32_t padded = (counts[e] + align - 1) / align * align;
#endif
        offsets[e + 1] = offsets[e] + padded;
    }
#if TKO_PLANT == 18
    for (int64_t r = 0; r < rmax; ++r) token_of[r] = 0;   /* planted: padding rows name token 0 */
#else
    for (int64_t r = 0; r < rmax; ++r) token_of[r] = -1;
#endif
    std::vector<int32_t> fill(E, 0);
    for (int64_t p = 0; p < pairs; ++p) {
        const int e = topk_idx[p];
        if (e < 0 || e >= E) { slot_of[p] = -1; continue; }
#if TKO_PLANT == 5
        const int32_t slot = offsets[e] + counts[e] - 1 - fill[e];  /* planted: unstable order */
#else
        const int32_t slot = offsets[e] + fill[e];
#endif
        fill[e] += 1;
        slot_of[p] = slot;
        token_of[slot] = static_cast<int32_t>(p / k);
    }
    return bad;
}

/* ------------------------------------------------------------------------------------------
 * Per-token, per-128-channel E4M3 quantisation (the quant/ module's per-token granularity on
 * 147227.xyz "2、quant/"; FP8 dispatch in 機器之心 "性能表現"). The pages give no formula;
 * this is the amax scaling that maps the block's largest magnitude onto E4M3's largest
 * finite value: scale = amax / 448, q = e4m3(x / scale), both IEEE fp32 divisions.
 * ---------------------------------------------------------------------------------------- */
int tko_quantize_row_e4m3(const uint16_t* xrow, int H, uint8_t* q, float* scales) {
    if (H <= 0 || H % 128 != 0) return -1;
    for (int b = 0; b < H / 128; ++b) {
        float amax = 0.0f;
        for (int c = 0; c < 128; ++c) amax = std::max(amax, std::fabs(bf16_to_float(xrow[b * 128 + c])));
#if TKO_PLANT == 20
        if (amax == 0.0f) amax = 1e-30f;  /* planted: an epsilon guard instead of scale 0 */
#else
        if (amax == 0.0f) {
            scales[b] = 0.0f;
            for (int c = 0; c < 128; ++c) q[b * 128 + c] = 0x00;
            continue;
        }
#endif
#if TKO_PLANT == 7
        const float scale = amax / 447.0f;  /* planted: wrong E4M3 maximum */
#else
        const float scale = amax / 448.0f;
#endif
        scales[b] = scale;
        for (int c = 0; c < 128; ++c) q[b * 128 + c] = tko_e4m3_encode(bf16_to_float(xrow[b * 128 + c]) / scale);
    }
    return 0;
}

/* ------------------------------------------------------------------------------------------
 * Expand (fused expand/dispatch, 147227.xyz "moe/" and 機器之心 "Tile Kernels"): every token
 * row is written to each of its k slots; padding rows are zero. FP8 output quantises each
 * token row once and gives all k copies the same codes and scales.
 * ---------------------------------------------------------------------------------------- */
int tko_expand(const uint16_t* x, const int32_t* slot_of, const int32_t* offsets, int T, int E,
               int k, int H, int out_dtype, void* out, float* out_scale) {
    if (T < 0 || E < 1 || k < 1 || H <= 0) return -1;
    if (out_dtype == TKO_OUT_FP8_E4M3 && (H % 128 != 0 || out_scale == nullptr)) return -1;
    if (out_dtype != TKO_OUT_BF16 && out_dtype != TKO_OUT_FP8_E4M3) return -1;
    const int64_t rows = offsets[E];
    const int nb = H / 128;
    int bad = 0;
    if (out_dtype == TKO_OUT_BF16) {
        uint16_t* o = static_cast<uint16_t*>(out);
        std::memset(o, 0, static_cast<size_t>(rows) * H * sizeof(uint16_t));
        for (int t = 0; t < T; ++t)
            for (int j = 0; j < k; ++j) {
                const int64_t slot = slot_of[static_cast<int64_t>(t) * k + j];
                if (slot < 0 || slot >= rows) { bad = 1; continue; }
                std::memcpy(o + slot * H, x + static_cast<int64_t>(t) * H, H * sizeof(uint16_t));
            }
    } else {
        uint8_t* o = static_cast<uint8_t*>(out);
        std::memset(o, 0, static_cast<size_t>(rows) * H);
        for (int64_t r = 0; r < rows * nb; ++r) out_scale[r] = 0.0f;
        std::vector<uint8_t> q(H);
        std::vector<float> sc(nb);
        for (int t = 0; t < T; ++t) {
            tko_quantize_row_e4m3(x + static_cast<int64_t>(t) * H, H, q.data(), sc.data());
            for (int j = 0; j < k; ++j) {
                const int64_t slot = slot_of[static_cast<int64_t>(t) * k + j];
                if (slot < 0 || slot >= rows) { bad = 1; continue; }
                std::memcpy(o + slot * H, q.data(), H);
                std::memcpy(out_scale + slot * nb, sc.data(), nb * sizeof(float));
            }
        }
    }
    return bad;
}

/* ------------------------------------------------------------------------------------------
 * Reduce (fused reduce/combine, same sources; BF16 combine in 機器之心 "性能表現"): each
 * token's output is the weighted sum of its k expert rows, accumulated in fp32 in slot order
 * j = 0..k-1 with one fmaf per term, rounded once to bf16.
 * ---------------------------------------------------------------------------------------- */
int tko_reduce_token(const uint16_t* y, int64_t y_rows, const int32_t* slot_row,
                     const float* w_row, int k, int H, uint16_t* out_row) {
    int bad = 0;
    for (int c = 0; c < H; ++c) {
        float acc = 0.0f;
        for (int jj = 0; jj < k; ++jj) {
#if TKO_PLANT == 8
            const int j = k - 1 - jj;  /* planted: reverse slot order */
#else
            const int j = jj;
#endif
            const int64_t slot = slot_row[j];
            if (slot < 0 || slot >= y_rows) { bad = 1; continue; }
            const float wj = w_row != nullptr ? w_row[j] : 1.0f;
            acc = std::fmaf(wj, bf16_to_float(y[slot * H + c]), acc);
        }
        out_row[c] = tko_bf16_rne(acc);
    }
    return bad;
}

int tko_reduce(const uint16_t* y, int64_t y_rows, const int32_t* slot_of, const float* w, int T,
               int k, int H, uint16_t* out) {
    if (T < 0 || k < 1 || H <= 0 || y_rows < 0) return -1;
    int bad = 0;
    for (int t = 0; t < T; ++t) {
        const int64_t p = static_cast<int64_t>(t) * k;
        bad |= tko_reduce_token(y, y_rows, slot_of + p, w != nullptr ? w + p : nullptr, k, H,
                                out + static_cast<int64_t>(t) * H);
    }
    return bad;
}

/* ------------------------------------------------------------------------------------------
 * Load-balance statistics (147227.xyz "moe/": load-balance loss computation; the pages give no
 * formula). The reading: the usual auxiliary balance loss of routed MoE layers -- the fraction
 * of routed pairs per expert times the mean normalised routing score of that expert, summed
 * and scaled so that perfectly balanced routing gives 1. Scores are the unbiased ones (the
 * selection bias only steers selection).
 * ---------------------------------------------------------------------------------------- */
int tko_balance_stats(const float* logits, const int32_t* counts, int T, int E, int k,
                      int score_fn, double* P, double* f, double* loss) {
    if (T < 0 || E < 1 || k < 1 || k > E) return -1;
    if (score_fn != TKO_SCORE_SOFTMAX && score_fn != TKO_SCORE_SIGMOID) return -1;
    std::vector<double> p(E);
    for (int i = 0; i < E; ++i) P[i] = 0.0;
    for (int t = 0; t < T; ++t) {
        const float* l = logits + static_cast<int64_t>(t) * E;
        double z = 0.0;
        if (score_fn == TKO_SCORE_SOFTMAX) {
            double m = -std::numeric_limits<double>::infinity();
            for (int i = 0; i < E; ++i) m = std::max(m, static_cast<double>(l[i]));
            for (int i = 0; i < E; ++i) { p[i] = std::exp(static_cast<double>(l[i]) - m); z += p[i]; }
        } else {
            for (int i = 0; i < E; ++i) { p[i] = 1.0 / (1.0 + std::exp(-static_cast<double>(l[i]))); z += p[i]; }
        }
        for (int i = 0; i < E; ++i) P[i] += p[i] / z;
    }
    double acc = 0.0;
    for (int i = 0; i < E; ++i) {
        P[i] = T > 0 ? P[i] / T : 0.0;
#if TKO_PLANT == 10
        f[i] = T > 0 ? static_cast<double>(counts[i]) / (static_cast<double>(k) * T) : 0.0;  /* planted */
#else
        f[i] = T > 0 ? static_cast<double>(E) * counts[i] / (static_cast<double>(k) * T) : 0.0;
#endif
        acc += f[i] * P[i];
    }
    *loss = acc;
    return 0;
}

/* ------------------------------------------------------------------------------------------
 * Tensor-parallel mask (147227.xyz "moe/": tensor-parallel mask; no definition on the pages).
 * The reading: experts are owned in E/tp_size contiguous groups; a rank keeps its own pairs,
 * renumbered locally, and masks the rest with -1.
 * ---------------------------------------------------------------------------------------- */
int tko_tp_mask(const int32_t* topk_idx, int T, int k, int E, int tp_size, int tp_rank,
                int32_t* out_idx) {
    if (T < 0 || k < 1 || E < 1 || tp_size < 1 || E % tp_size != 0 || tp_rank < 0 ||
        tp_rank >= tp_size)
        return -1;
    const int el = E / tp_size;
    const int lo = tp_rank * el;
    for (int64_t p = 0; p < static_cast<int64_t>(T) * k; ++p) {
        const int e = topk_idx[p];
#if TKO_PLANT == 12
        out_idx[p] = (e >= lo && e < lo + el) ? e : -1;  /* planted: not renumbered */
#elif TKO_PLANT == 19
        out_idx[p] = (e >= lo && e <= lo + el) ? e - lo : -1;  /* planted: inclusive upper bound */
#else
        out_idx[p] = (e >= lo && e < lo + el) ? e - lo : -1;
#endif
    }
    return 0;
}

/* ------------------------------------------------------------------------------------------
 * Backward of the fused reduce (the training use of the fused expand/reduce; TileKernels is
 * described as training and inference kernels, m.yhxrc.cn "簡介"). out = sum_j w_j y_j is
 * linear in y and in w, so d_y_j = w_j * g and d_w_j = <g, y_j>. d_y is rounded like every bf16
 * output here (fp32 product, then bf16); d_w is the dot product in double, rounded once.
 * The backward of expand (a copy to k rows) is the unweighted reduce of the row gradients,
 * which tko_reduce with w = NULL already states.
 * ---------------------------------------------------------------------------------------- */
int tko_reduce_backward(const uint16_t* grad_out, const uint16_t* y, int64_t y_rows,
                        const int32_t* slot_of, const int32_t* offsets, const float* w, int T,
                        int E, int k, int H, uint16_t* d_y, float* d_w) {
    if (T < 0 || E < 1 || k < 1 || H <= 0 || y_rows < 0) return -1;
    const int64_t rows = offsets[E];
    std::memset(d_y, 0, static_cast<size_t>(rows) * H * sizeof(uint16_t));
    int bad = 0;
    for (int t = 0; t < T; ++t) {
        const uint16_t* g = grad_out + static_cast<int64_t>(t) * H;
        for (int j = 0; j < k; ++j) {
            const int64_t p = static_cast<int64_t>(t) * k + j;
            const int64_t slot = slot_of[p];
            if (slot < 0 || slot >= y_rows || slot >= rows) {
                if (slot != -1) bad = 1;
                d_w[p] = 0.0f;
                continue;
            }
            const float wj = w != nullptr ? w[p] : 1.0f;
            double dot = 0.0;
            for (int c = 0; c < H; ++c) {
                const float gc = bf16_to_float(g[c]);
                dot += static_cast<double>(gc) * static_cast<double>(bf16_to_float(y[slot * H + c]));
#if TKO_PLANT == 21
                d_y[slot * H + c] = tko_bf16_rne(bf16_to_float(tko_bf16_rne(wj)) * gc);  /* planted: w rounded to bf16 first */
#else
                d_y[slot * H + c] = tko_bf16_rne(wj * gc);
#endif
            }
#if TKO_PLANT == 11
            d_w[p] = static_cast<float>(dot * wj);  /* planted: weighted dot product */
#else
            d_w[p] = static_cast<float>(dot);
#endif
        }
    }
    return bad;
}

/* ------------------------------------------------------------------------------------------
 * Expert-parallel dispatch and combine over G ranks. Sources: 147227.xyz "刚刚！DeepSeek开源高
 * 性能GPU算子库TileKernels" (its DeepEP paragraph: an expert-parallel all-to-all library over
 * NVLink with native FP8 dispatch) and 機器之心 "剛剛，DeepSeek開始頻繁更新：Tile Kernels、
 * DeepEP V2", section "性能表現" (the DeepSeek-V3 setting with FP8 dispatch and BF16 combine).
 * Neither page gives a layout or a formula; the readings, each the plainest one:
 *  - experts are owned in G contiguous groups of E/G (expert e lives on rank e / (E/G));
 *  - a token goes once to every rank that owns at least one of its experts (not once per
 *    expert); masked pairs (expert -1) go nowhere;
 *  - a destination's receive buffer holds the rows of source 0, then source 1, ..., each
 *    source's rows in token order;
 *  - each received row carries the token's k choices renumbered to the destination's local
 *    experts (-1 for experts of other ranks) and the matching weights (0 for those);
 *  - the destination combines its own experts' rows of a received token like the single-GPU
 *    reduce (fp32 fmaf in slot order) and rounds the partial sum to bf16 (BF16 combine);
 *  - the source adds the bf16 partial rows of the token's destinations in ascending rank
 *    order in fp32 and rounds once to bf16.
 * ---------------------------------------------------------------------------------------- */
static int ep_owner(int e, int E, int G) {
#if TKO_PLANT == 14
    return e % G;  /* planted: experts dealt round-robin over the ranks */
#else
    return e / (E / G);
#endif
}

int tko_ep_layout(const int32_t* topk_idx, int T, int E, int k, int G, int32_t* send_counts,
                  int32_t* dest_pos) {
    if (T < 0 || E < 1 || k < 1 || G < 1 || E % G != 0) return -1;
    for (int d = 0; d < G; ++d) send_counts[d] = 0;
    std::vector<char> goes(G);
    for (int t = 0; t < T; ++t) {
        std::fill(goes.begin(), goes.end(), 0);
        for (int j = 0; j < k; ++j) {
            const int e = topk_idx[static_cast<int64_t>(t) * k + j];
            if (e == -1) continue;
            if (e < 0 || e >= E) return -2;
            goes[ep_owner(e, E, G)] = 1;
        }
        for (int d = 0; d < G; ++d)
            dest_pos[static_cast<int64_t>(t) * G + d] = goes[d] ? send_counts[d]++ : -1;
    }
    return 0;
}

int tko_ep_recv_bases(const int32_t* count_matrix, int G, int64_t* base, int64_t* recv_rows) {
    if (G < 1) return -1;
    for (int d = 0; d < G; ++d) {
        int64_t acc = 0;
        for (int s = 0; s < G; ++s) {
#if TKO_PLANT == 16
            acc += count_matrix[static_cast<int64_t>(s) * G + d];  /* planted: inclusive prefix */
            base[static_cast<int64_t>(s) * G + d] = acc;
#else
            base[static_cast<int64_t>(s) * G + d] = acc;
            acc += count_matrix[static_cast<int64_t>(s) * G + d];
#endif
        }
        recv_rows[d] = acc;
    }
    return 0;
}

int tko_ep_dispatch(const uint16_t* x, const int32_t* topk_idx, const float* topk_w,
                    const int32_t* dest_pos, int T, int E, int k, int H, int G, int d,
                    int64_t base_row, int out_dtype, void* recv_x, float* recv_scale,
                    int32_t* recv_idx, float* recv_w) {
    if (T < 0 || E < 1 || k < 1 || H <= 0 || G < 1 || E % G != 0 || d < 0 || d >= G) return -1;
    if (out_dtype != TKO_OUT_BF16 && out_dtype != TKO_OUT_FP8_E4M3) return -1;
    if (out_dtype == TKO_OUT_FP8_E4M3 && H % 128 != 0) return -1;
    const int el = E / G;
    for (int t = 0; t < T; ++t) {
        const int pos = dest_pos[static_cast<int64_t>(t) * G + d];
        if (pos < 0) continue;
        const int64_t row = base_row + pos;
        const uint16_t* xr = x + static_cast<int64_t>(t) * H;
        if (out_dtype == TKO_OUT_BF16) {
            std::memcpy(static_cast<uint16_t*>(recv_x) + row * H, xr, sizeof(uint16_t) * H);
        } else {
            tko_quantize_row_e4m3(xr, H, static_cast<uint8_t*>(recv_x) + row * H,
                                  recv_scale + row * (H / 128));
        }
        for (int j = 0; j < k; ++j) {
            const int64_t p = static_cast<int64_t>(t) * k + j;
            const int e = topk_idx[p];
            const bool mine = e >= 0 && e < E && ep_owner(e, E, G) == d;
#if TKO_PLANT == 15
            recv_idx[row * k + j] = mine ? e : -1;  /* planted: global expert id sent */
#else
            recv_idx[row * k + j] = mine ? e - d * el : -1;
#endif
            recv_w[row * k + j] = mine ? topk_w[p] : 0.0f;
        }
    }
    return 0;
}

int tko_ep_combine(const uint16_t* const* partial, const int64_t* base_row,
                   const int32_t* dest_pos, int T, int G, int H, uint16_t* out) {
    if (T < 0 || G < 1 || H <= 0) return -1;
    for (int t = 0; t < T; ++t) {
        for (int c = 0; c < H; ++c) {
            float acc = 0.0f;
            for (int dd = 0; dd < G; ++dd) {
#if TKO_PLANT == 13
                const int d = G - 1 - dd;  /* planted: descending rank order */
#else
                const int d = dd;
#endif
                const int pos = dest_pos[static_cast<int64_t>(t) * G + d];
                if (pos < 0) continue;
                acc = acc + bf16_to_float(partial[d][(base_row[d] + pos) * H + c]);
            }
            out[static_cast<int64_t>(t) * H + c] = tko_bf16_rne(acc);
        }
    }
    return 0;
}

}  // extern "C"
