/*
 * tk_oracle.h -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, single-threaded CPU statement of the MoE gating-and-routing path
 * (gate/score/select/renormalise -> token-to-expert map -> expand -> reduce). It exists to
 * check the CUDA library against. Only the test suite, the package's smoke check and the
 * benchmark's CPU-baseline leg may load it. It shares no code, header, table or helper with
 * the CUDA library, and the CUDA library never calls it.
 *
 * Sources (web pages about DeepSeek's TileKernels; none prints code for these steps):
 *  - "刚刚！DeepSeek开源高性能GPU算子库TileKernels" (147227.xyz), section "1、moe/（14个算子）":
 *    the moe/ module covers top-k gating, expert scoring, token-to-expert mapping, fused
 *    expand/reduce, a tensor-parallel mask and a load-balance loss.
 *  - "剛剛，DeepSeek開始頻繁更新：Tile Kernels、DeepEP V2" (機器之心), section "Tile Kernels",
 *    feature list: gating = top-k expert selection and scoring; MoE routing = token-to-expert
 *    mapping, fused expansion/reduction and weight normalisation; section "性能表現": the
 *    DeepSeek-V3 setting (8K tokens, hidden 7168, top-8, FP8 dispatch, BF16 combine).
 *  - "DeepSeek 的 GPU 内核帝国" (zhichai.net), section "MoE TopK 门控": a one-warp-per-token
 *    top-k kernel that takes num_topk rounds of (max, argmax with a 'min' index reducer),
 *    writing indices in selection order.
 *
 * Conventions: all arrays are contiguous row-major host arrays owned by the caller.
 * bf16 values travel as uint16_t bit patterns, e4m3 values as uint8_t codes.
 * Every function returns 0 on success and a negative number on invalid arguments.
 */
#ifndef TK_ORACLE_H
#define TK_ORACLE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { TKO_SCORE_SOFTMAX = 0, TKO_SCORE_SIGMOID = 1 };
enum { TKO_OUT_BF16 = 0, TKO_OUT_FP8_E4M3 = 1 };

/* ---- scalar building blocks (exported so the tests can pin them) ---- */

/* The fp32 exponential used for selection keys: Cody-Waite reduction by ln 2 and the degree-7
 * Taylor polynomial of e^r, every step one IEEE fp32 round-to-nearest operation. */
float tko_spec_expf(float x);
void tko_spec_expf_array(const float* x, float* y, int64_t n);
/* fp32 logistic function built on tko_spec_expf: 1 / (1 + exp(-l)). */
float tko_spec_sigmoidf(float l);
void tko_spec_sigmoidf_array(const float* x, float* y, int64_t n);
/* fp32 -> OCP FP8 E4M3 code, round to nearest even, saturating to +-448 (satfinite). */
uint8_t tko_e4m3_encode(float v);
void tko_e4m3_encode_array(const float* x, uint8_t* y, int64_t n);
/* fp32 -> bf16 bits, round to nearest even. */
uint16_t tko_bf16_rne(float f);
void tko_bf16_rne_array(const float* x, uint16_t* y, int64_t n);

/* ---- the four steps ---- */

/* Gate: per token, rank experts by key (logit when bias == NULL; fp32 sigmoid(logit)+bias
 * when a bias is given, sigmoid only), descending, equal keys -> lower expert index first;
 * keep the first k in that order. Weights are the unbiased scores of the chosen experts
 * (softmax probability or sigmoid), renormalised over the k when renormalize != 0, computed
 * in double and rounded once to fp32. Returns -1 on bad arguments, -2 for softmax + bias. */
int tko_gate_topk(const float* logits, const float* bias, int T, int E, int k, int score_fn,
                  int renormalize, int32_t* topk_idx, float* topk_w);

/* The number of rows of the expert-sorted buffer in the worst case: T*k + E*(align-1). */
int64_t tko_max_rows(int T, int E, int k, int align);

/* Token-to-expert map. counts[E]; offsets[E+1] = exclusive scan of counts rounded up to a
 * multiple of align; slot_of[T*k] = offsets[e] + (number of earlier pairs on expert e);
 * token_of[R_max] = token of each real row, -1 for padding rows and rows past offsets[E].
 * A pair whose expert is -1 is masked: not counted, slot -1. Any other expert outside [0,E)
 * is treated the same way and reported (returns 1). */
int tko_route_map(const int32_t* topk_idx, int T, int E, int k, int align, int32_t* counts,
                  int32_t* offsets, int32_t* slot_of, int32_t* token_of);

/* Per-token, per-128-channel E4M3 quantisation of one bf16 row of H channels (H % 128 == 0):
 * scale = amax/448 (fp32 IEEE division), q = e4m3(x/scale); a block with amax == 0 gets
 * scale 0 and all codes 0x00. */
int tko_quantize_row_e4m3(const uint16_t* xrow, int H, uint8_t* q, float* scales);

/* Expand: rows [0, offsets[E]) of out are first zeroed, then out[slot_of[t*k+j]] = row t of x
 * (bf16), or its E4M3 codes with out_scale[slot] = its scales (fp8). Rows at and beyond
 * offsets[E] are not touched. out must hold tko_max_rows() rows. */
int tko_expand(const uint16_t* x, const int32_t* slot_of, const int32_t* offsets, int T, int E,
               int k, int H, int out_dtype, void* out, float* out_scale);

/* Reduce for one token: acc = 0; for j = 0..k-1 in order acc = fmaf(w_j, y[slot_j], acc)
 * (w_j = 1 when w == NULL); out = bf16(acc). slot_row holds the token's k slots, w_row its k
 * weights (or NULL). A slot outside [0, y_rows) contributes nothing (returns 1). */
int tko_reduce_token(const uint16_t* y, int64_t y_rows, const int32_t* slot_row,
                     const float* w_row, int k, int H, uint16_t* out_row);
/* Reduce for all T tokens. */
int tko_reduce(const uint16_t* y, int64_t y_rows, const int32_t* slot_of, const float* w, int T,
               int k, int H, uint16_t* out);

/* ---- next rows: load-balance statistics, tensor-parallel mask, backward ---- */

/* Load-balance statistics (147227.xyz "moe/" lists a load-balance loss among the routing ops;
 * no formula on the pages). Per token the unbiased scores are normalised over all E experts:
 * p[t,i] = softmax(l_t)_i, or sigmoid(l_ti) / sum_j sigmoid(l_tj) for sigmoid scoring. Then
 *   P[i] = (1/T) sum_t p[t,i],  f[i] = E * counts[i] / (k*T),  loss = sum_i f[i] * P[i]
 * (loss = 1 for perfectly balanced routing). All in double; T = 0 gives zeros. */
int tko_balance_stats(const float* logits, const int32_t* counts, int T, int E, int k,
                      int score_fn, double* P, double* f, double* loss);

/* Tensor-parallel expert mask: experts are split into tp_size contiguous groups of E/tp_size;
 * rank tp_rank keeps pairs on its own group, renumbered to local indices 0..E/tp_size-1, and
 * marks every other pair -1 (a masked pair, which the route map skips). */
int tko_tp_mask(const int32_t* topk_idx, int T, int k, int E, int tp_size, int tp_rank,
                int32_t* out_idx);

/* Backward of the weighted reduce out[t] = sum_j w[t,j] * y[slot_of[t,j]]:
 *   d_y[slot_of[t,j], c] = bf16( fp32(w[t,j] * g[t,c]) )      (w = NULL: weight 1)
 *   d_w[t,j] = fp32( sum_c double(g[t,c]) * double(y[slot_of[t,j], c]) )  (summed in c order)
 * Rows of d_y in [0, offsets[E]) that no pair references (padding) are zero; rows at and
 * beyond offsets[E] are not written. A pair with an out-of-range slot gets d_w = 0. */
int tko_reduce_backward(const uint16_t* grad_out, const uint16_t* y, int64_t y_rows,
                        const int32_t* slot_of, const int32_t* offsets, const float* w, int T,
                        int E, int k, int H, uint16_t* d_y, float* d_w);

/* ---- expert-parallel dispatch / combine over G ranks (experts in G contiguous groups) ---- */

/* For one source rank: dest_pos[t*G+d] = position of token t among this rank's tokens that go
 * to rank d (token order), or -1 when no expert of t lives on d; send_counts[d] = how many go.
 * Returns -2 for an expert outside [0,E) other than the masked -1. */
int tko_ep_layout(const int32_t* topk_idx, int T, int E, int k, int G, int32_t* send_counts,
                  int32_t* dest_pos);
/* From the G x G matrix count_matrix[s*G+d] (rows source s sends to rank d):
 * base[s*G+d] = first row of source s in rank d's receive buffer (sources in rank order),
 * recv_rows[d] = rows rank d receives. */
int tko_ep_recv_bases(const int32_t* count_matrix, int G, int64_t* base, int64_t* recv_rows);
/* Writes source rank's tokens bound for rank d into d's receive buffer at rows
 * base_row + dest_pos[t*G+d]: the row (bf16, or E4M3 codes + per-128-channel scales), the k
 * choices renumbered to d's local experts (-1 elsewhere) and their weights (0 elsewhere). */
int tko_ep_dispatch(const uint16_t* x, const int32_t* topk_idx, const float* topk_w,
                    const int32_t* dest_pos, int T, int E, int k, int H, int G, int d,
                    int64_t base_row, int out_dtype, void* recv_x, float* recv_scale,
                    int32_t* recv_idx, float* recv_w);
/* out[t] = bf16( sum over d ascending with dest_pos[t*G+d] >= 0 of
 *                fp32(partial[d][base_row[d] + dest_pos[t*G+d]]) ), fp32 adds. */
int tko_ep_combine(const uint16_t* const* partial, const int64_t* base_row,
                   const int32_t* dest_pos, int T, int G, int H, uint16_t* out);

#ifdef __cplusplus
}
#endif
#endif /* TK_ORACLE_H */
