/*
 * tk_route.h -- C ABI of libtk_route.so: the MoE gating-and-routing hot path on one B200.
 *
 * The path is the one the TileKernels moe/ module is described as covering ("刚刚！DeepSeek开源
 * 高性能GPU算子库TileKernels", 147227.xyz, section "1、moe/（14个算子）"; feature list in
 * "剛剛，DeepSeek開始頻繁更新：Tile Kernels、DeepEP V2", 機器之心, section "Tile Kernels"):
 *   1. tk_gate_topk  -- expert scoring, top-k selection, weight renormalisation
 *   2. tk_route_map  -- token-to-expert map: per-expert counts, segment offsets, slots
 *   3. tk_expand     -- fused expand (dispatch): every token row copied to its k slots of an
 *                       expert-sorted buffer, optionally quantised to FP8 E4M3 on the way
 *   4. tk_reduce     -- fused reduce (combine): weighted sum of each token's k expert rows
 * The pages give no signatures; arguments follow the problem statement above.
 *
 * Conventions for every call:
 *  - Pointers named as device pointers must be CUDA device memory (or managed memory) that
 *    the caller allocated and owns; the library never allocates or frees memory.
 *  - Tensors are dense and row-major. bf16 data is passed as void* (2 bytes per element),
 *    E4M3 data as void* (1 byte per element).
 *  - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream). Every call
 *    only enqueues work on it and returns without synchronising the host.
 *  - Arguments are checked on the host before anything is enqueued; a bad argument returns
 *    TK_ERR_INVALID_ARG and enqueues nothing. tk_last_error_detail() says what was wrong.
 *  - Data errors that only the device can see (an expert index outside [0,E), a slot outside
 *    a buffer) never fault: the kernel skips the offending element and ORs a TK_DEVERR_* bit
 *    into *err_flag when err_flag (a device int32, nullable) is given. The caller zeroes
 *    *err_flag beforehand and reads it after synchronising the stream.
 *  - Kernels launch with programmatic dependent launch enabled (the launch latency of a kernel
 *    overlaps the end of the previous one); no kernel reads an input before the previous
 *    kernel on the stream has completed.
 */
#ifndef TK_ROUTE_H
#define TK_ROUTE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define TK_API __attribute__((visibility("default")))
#else
#define TK_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum tk_status {
    TK_OK = 0,
    TK_ERR_INVALID_ARG = 1, /* rejected on the host; nothing was enqueued */
    TK_ERR_CUDA = 2         /* a CUDA runtime call or launch failed (detail has its name) */
} tk_status;

typedef enum tk_score_fn { TK_SCORE_SOFTMAX = 0, TK_SCORE_SIGMOID = 1 } tk_score_fn;
typedef enum tk_out_dtype { TK_OUT_BF16 = 0, TK_OUT_FP8_E4M3 = 1 } tk_out_dtype;

/* Bits ORed into *err_flag by the kernels. */
#define TK_DEVERR_EXPERT_RANGE 1 /* tk_route_map: a topk_idx entry outside [0,E), other than -1 (skipped, slot -1) */
#define TK_DEVERR_DUP_EXPERT 2   /* tk_route_map: a token lists one expert twice (slots then overlap) */
#define TK_DEVERR_SLOT_RANGE 4   /* tk_expand / tk_reduce: a slot outside the buffer (skipped) */
#define TK_DEVERR_ROWS_RANGE 8   /* tk_expand: offsets[E] above the worst-case row count (clamped) */
#define TK_DEVERR_TIMEOUT 16     /* a bounded wait inside a kernel gave up (work skipped) */

/* Limits of the warp-per-token gate. */
#define TK_MAX_EXPERTS 1024
#define TK_MAX_TOPK 32
#define TK_MAX_EP_RANKS 32   /* expert-parallel ranks (tk_ep_*) */

/*
 * Gate: expert scoring, top-k selection and weight normalisation (機器之心 "Tile Kernels"
 * feature list: gating = top-k expert selection and scoring; routing includes weight
 * normalisation). Selection follows the one-warp-per-token kernel sketched in the zhichai.net
 * essay "DeepSeek 的 GPU 内核帝国", section "MoE TopK 门控": k rounds of max/argmax, ties to
 * the lower expert index, winners written in round order.
 *
 *   logits  device, fp32 [T, E]
 *   bias    device, fp32 [E] or NULL. Selection bias, sigmoid only: the key is then the fp32
 *           value sigmoid(logit) + bias (sigmoid evaluated with the library's fixed fp32
 *           exponential, Cody-Waite reduction + degree-7 Taylor polynomial); without a bias
 *           the key is the logit (both score functions are increasing). NaN keys rank as -inf.
 *   T >= 0, 1 <= E <= 1024, 1 <= k <= min(E, 32)
 *   score_fn     TK_SCORE_SOFTMAX or TK_SCORE_SIGMOID (softmax with a bias is rejected)
 *   renormalize  nonzero: weights are divided by their sum over the k chosen experts
 *   topk_idx     device, int32 [T, k]: chosen experts, best first
 *   topk_w       device, fp32 [T, k]: the unbiased scores of the chosen experts (softmax
 *                probability or sigmoid), computed in double and rounded once to fp32;
 *                a zero sum gives zero weights
 */
TK_API tk_status tk_gate_topk(const float* logits, const float* bias, int T, int E, int k, int score_fn,
                       int renormalize, int32_t* topk_idx, float* topk_w, void* stream);

/* Worst-case number of rows of the expert-sorted buffer: T*k + E*(align-1). */
TK_API int64_t tk_max_rows(int T, int E, int k, int align);

/* Bytes of device workspace tk_route_map needs for T tokens and E experts. */
TK_API size_t tk_route_map_workspace_bytes(int T, int E, int k);

/*
 * Token-to-expert map (機器之心 "Tile Kernels" feature list: token-to-expert mapping).
 * Pair p = t*k + j.
 *   topk_idx  device, int32 [T, k], 1 <= k <= 32: a token's experts other than -1 are
 *             distinct (so k may exceed E when pairs are masked, as after tk_tp_mask or on an
 *             expert-parallel destination)
 *   align     >= 1 (<= 4096): each expert's segment is padded to a multiple of align rows
 *   counts    device, int32 [E]: pairs routed to each expert
 *   offsets   device, int32 [E+1]: offsets[0] = 0, offsets[e+1] = offsets[e] +
 *             ceil(counts[e]/align)*align; offsets[E] = R, the rows in use
 *   slot_of   device, int32 [T*k]: row of pair p = offsets[e] + (number of pairs p' < p on
 *             expert e), so each segment lists its tokens in increasing order (-1 for a pair
 *             whose expert is out of range). Expert -1 marks a masked pair (tk_tp_mask): it is
 *             skipped like an out-of-range one but sets no error bit.
 *   token_of  device, int32 [tk_max_rows()]: token of each row, -1 for padding rows and for
 *             rows at and beyond R
 *   workspace device, at least tk_route_map_workspace_bytes(T, E, k) bytes, 16-byte
 *             aligned, no initial contents needed; not shared by calls that may overlap
 * T*k + E*(align-1) must fit in int32.
 */
TK_API tk_status tk_route_map(const int32_t* topk_idx, int T, int E, int k, int align, int32_t* counts,
                       int32_t* offsets, int32_t* slot_of, int32_t* token_of, void* workspace,
                       size_t workspace_bytes, int32_t* err_flag, void* stream);

/*
 * Route map of one window of experts: the tensor-parallel mask (tk_tp_mask) fused into the route
 * map (147227.xyz "moe/": tensor-parallel mask, next to the token-to-expert mapping). A pair
 * whose expert lies in [expert_lo, expert_lo + E) is routed to local expert e - expert_lo; every
 * other pair is masked (slot -1). The outputs are those of tk_tp_mask(tp_size = E_total / E,
 * tp_rank = expert_lo / E) followed by tk_route_map with E experts, without the masked index
 * array or the extra launch; unlike that pair of calls, an index outside [0, E_total) other than
 * -1 sets TK_DEVERR_EXPERT_RANGE.
 *   E_total   all experts the indices refer to; 0 <= expert_lo and expert_lo + E <= E_total
 *   E         the window's experts (1 <= E <= 1024): counts [E], offsets [E+1], token_of
 *             [tk_max_rows(T, E, k, align)] and the workspace (tk_route_map_workspace_bytes(T,
 *             E, k)) are sized by it
 * Every other argument as in tk_route_map.
 */
TK_API tk_status tk_route_map_window(const int32_t* topk_idx, int T, int E_total, int k,
                                     int expert_lo, int E, int align, int32_t* counts,
                                     int32_t* offsets, int32_t* slot_of, int32_t* token_of,
                                     void* workspace, size_t workspace_bytes, int32_t* err_flag,
                                     void* stream);

/*
 * Allocation-free form of tk_route_map (the pages have no counterpart: this exists only for
 * callers that cannot allocate device memory, such as a serving engine or plugin host that
 * owns all device memory and hands a component only its inputs and outputs, or a
 * latency-critical loop that must not call cudaMalloc, which can synchronise the device).
 * Same arguments, results and errors as tk_route_map, without workspace: the scratch it needs
 * is a 2 MiB array built into the library (every GPU that loads the library holds it until
 * the process exits). It serves T and E with E * 4*ceil(ceil(T/128)/4) <= 524288 (e.g.
 * T <= 262144 at E = 256, T <= 65536 at E = 1024); larger sizes return TK_ERR_INVALID_ARG and
 * enqueue nothing. The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current and caches it for the life of the process;
 * make that first call before any stream capture. A device reset (cudaDeviceReset) after the
 * first call on that device is not supported: the cached address would be stale. All calls on a device share the array and nothing in it needs to start
 * at zero; calls that can overlap on the GPU (other streams, other host threads) race on it
 * and must be serialised by the caller. The call allocates nothing.
 */
TK_API tk_status tk_route_map_static(const int32_t* topk_idx, int T, int E, int k, int align,
                                     int32_t* counts, int32_t* offsets, int32_t* slot_of,
                                     int32_t* token_of, int32_t* err_flag, void* stream);

/*
 * Fused expand / dispatch (147227.xyz "moe/": fused expand; 機器之心 "性能表現": FP8 dispatch
 * in the DeepSeek-V3 setting). Row t of x goes to rows slot_of[t*k+j], j < k, of out; padding
 * rows (token_of == -1 below offsets[E]) are written as zeros; rows at and beyond offsets[E]
 * are not written.
 *   x          device, bf16 [T, H], 16-byte aligned
 *   slot_of    device, int32 [T*k] from tk_route_map
 *   offsets    device, int32 [E+1] from tk_route_map
 *   token_of   device, int32 [tk_max_rows()] from tk_route_map (may be NULL when align == 1)
 *   H          channels per row: H % 8 == 0 for bf16 output, H % 128 == 0 for E4M3 output
 *   out_dtype  TK_OUT_BF16: out is bf16 [tk_max_rows(), H];
 *              TK_OUT_FP8_E4M3: out is E4M3 [tk_max_rows(), H] and out_scale fp32
 *              [tk_max_rows(), H/128]: per token and 128-channel block, scale = amax/448 and
 *              code = E4M3(x/scale), round to nearest even, saturating at +-448 (IEEE fp32
 *              division); a block with amax 0 gets scale 0 and codes 0. Padding rows get codes
 *              0 and scale 0.
 *   out        device, 16-byte aligned
 */
TK_API tk_status tk_expand(const void* x, const int32_t* slot_of, const int32_t* offsets,
                    const int32_t* token_of, int T, int E, int k, int H, int align, int out_dtype,
                    void* out, float* out_scale, int32_t* err_flag, void* stream);

/*
 * Fused reduce / combine (147227.xyz "moe/": fused reduce; 機器之心 "性能表現": BF16
 * combine). For each token t and channel c:
 *   acc = 0; for j = 0..k-1 in order: acc = fmaf(w[t*k+j], float(y[slot_of[t*k+j], c]), acc)
 *   out[t, c] = bf16(acc), round to nearest even.
 *   y        device, bf16 [y_rows, H], 16-byte aligned (expert outputs in expert-sorted rows)
 *   slot_of  device, int32 [T*k]; a slot outside [0, y_rows) contributes nothing
 *   w        device, fp32 [T*k] or NULL (weight 1 for every term)
 *   H % 8 == 0
 *   out      device, bf16 [T, H], 16-byte aligned
 */
TK_API tk_status tk_reduce(const void* y, int64_t y_rows, const int32_t* slot_of, const float* w, int T,
                    int k, int H, void* out, int32_t* err_flag, void* stream);

/*
 * tk_reduce for slot maps in which most pairs are masked (-1): the rows an expert-parallel
 * destination receives (each lists k choices, about k/G of them local) or a route map after
 * tk_tp_mask. Same arguments, arithmetic and results, bit for bit. It steps through its work
 * units with O(1) updates instead of a 64-bit division per unit, which is what limits units with
 * few valid rows (measured on B200: the reduce of an expert-parallel destination 22 % faster);
 * with every pair valid tk_reduce is the faster of the two (by about 2 %).
 */
TK_API tk_status tk_reduce_masked(const void* y, int64_t y_rows, const int32_t* slot_of,
                                  const float* w, int T, int k, int H, void* out,
                                  int32_t* err_flag, void* stream);

/*
 * Load-balance statistics (147227.xyz "moe/": load-balance loss computation; no formula on the
 * pages -- this is the usual auxiliary balance loss of routed MoE layers). With p[t,i] the
 * unbiased scores of token t normalised over all E experts (softmax, or sigmoid divided by its
 * row sum):
 *   P[i] = (1/T) sum_t p[t,i],   f[i] = E * counts[i] / (k*T),   loss = sum_i f[i] * P[i]
 * so perfectly balanced routing gives loss = 1. Computed in double (deterministic: fixed
 * 64-token tiles and fixed-order sums), written as fp32.
 *   logits    device, fp32 [T, E] (the gate's logits; the selection bias is not used)
 *   counts    device, int32 [E] (tk_route_map's counts)
 *   P, f      device, fp32 [E];  loss  device, fp32 [1]
 *   workspace device, tk_balance_stats_workspace_bytes(T, E) bytes, 16-byte aligned
 */
TK_API size_t tk_balance_stats_workspace_bytes(int T, int E);
TK_API tk_status tk_balance_stats(const float* logits, const int32_t* counts, int T, int E, int k,
                                  int score_fn, float* P, float* f, float* loss, void* workspace,
                                  size_t workspace_bytes, void* stream);

/*
 * The same statistics over a batch split across data-parallel ranks, in two calls around an
 * all-reduce (the only exchange the routing path has):
 *   tk_balance_score_sums: sums[e] = sum over this rank's T tokens of p[t,e] (double, the
 *     per-64-token-tile partials added in tile order, as in tk_balance_stats);
 *   tk_balance_finalize: from sums and counts summed over all ranks and the total token count
 *     T_total: P = sums/T_total, f = E*counts/(k*T_total), loss = sum_e f*P (fixed-order tree).
 * On one rank, tk_balance_score_sums then tk_balance_finalize(sums, counts, T) equals
 * tk_balance_stats bit for bit.
 *   sums      device, double [E];  workspace as for tk_balance_stats
 */
TK_API tk_status tk_balance_score_sums(const float* logits, int T, int E, int score_fn,
                                       double* sums, void* workspace, size_t workspace_bytes,
                                       void* stream);
TK_API tk_status tk_balance_finalize(const double* sums, const int32_t* counts, int64_t T_total,
                                     int E, int k, float* P, float* f, float* loss, void* stream);

/*
 * Tensor-parallel expert mask (147227.xyz "moe/": tensor-parallel mask; no definition on the
 * pages). Experts are owned in tp_size contiguous groups of E/tp_size; for rank tp_rank,
 * out_idx = topk_idx - tp_rank*E/tp_size where the expert is in the rank's group, else -1 (a
 * masked pair, which tk_route_map skips). Route the result with E/tp_size experts.
 * out_idx may equal topk_idx (in place). tp_size must divide E.
 */
TK_API tk_status tk_tp_mask(const int32_t* topk_idx, int T, int k, int E, int tp_size,
                            int tp_rank, int32_t* out_idx, void* stream);

/*
 * Backward of tk_reduce (its inputs y and w), for training: with g = d(loss)/d(out) [T, H],
 *   d_y[slot_of[t,j], c] = bf16(fp32(w[t,j] * g[t,c]))       (w = NULL: weight 1)
 *   d_w[t,j]             = fp32(sum_c g[t,c] * y[slot_of[t,j], c])   (double accumulation)
 *   grad_out  device, bf16 [T, H];  y  device, bf16 [y_rows, H];  d_y  device, bf16 [y_rows, H]
 *   offsets, token_of  from tk_route_map, or both NULL: with them, padding rows of d_y below
 *             offsets[E] are zeroed, so d_y is complete up to offsets[E]; rows no pair
 *             references are otherwise not written
 *   d_w       device, fp32 [T, k] (0 for a pair whose slot is -1 or out of range)
 *   workspace device, tk_reduce_backward_workspace_bytes(T, k) bytes, 16-byte aligned
 * d_w is deterministic; it matches the exact dot product rounded to fp32 within 1 ulp.
 */
TK_API size_t tk_reduce_backward_workspace_bytes(int T, int k);
TK_API tk_status tk_reduce_backward(const void* grad_out, const void* y, int64_t y_rows,
                                    const int32_t* slot_of, const int32_t* offsets,
                                    const int32_t* token_of, const float* w, int T, int E, int k,
                                    int H, void* d_y, float* d_w, void* workspace,
                                    size_t workspace_bytes, int32_t* err_flag, void* stream);

/*
 * Backward of tk_expand (bf16): d_x[t] = sum_j d_xe[slot_of[t,j]], the unweighted reduce of the
 * gradient rows -- same kernel and arithmetic as tk_reduce with w = NULL.
 */
TK_API tk_status tk_expand_backward(const void* d_xe, int64_t xe_rows, const int32_t* slot_of,
                                    int T, int k, int H, void* d_x, int32_t* err_flag,
                                    void* stream);

/*
 * Expert-parallel dispatch and combine over G ranks (147227.xyz "刚刚！DeepSeek开源高性能GPU算子库
 * TileKernels", its DeepEP paragraph: an expert-parallel all-to-all over NVLink with native FP8
 * dispatch; 機器之心 "剛剛，DeepSeek開始頻繁更新：Tile Kernels、DeepEP V2", section "性能表現":
 * FP8 dispatch, BF16 combine). Neither page gives a layout; the one used here:
 *   - expert e lives on rank e / (E/G) (G contiguous groups; G must divide E);
 *   - a token goes once to each rank that owns at least one of its experts;
 *   - rank d's receive buffers hold the rows of source rank 0, then 1, ..., each source's rows
 *     in token order (a source's first row there is its base_row, the sum of the rows lower
 *     ranks send to d -- the caller exchanges the G x G send counts to get it);
 *   - each received row carries the token's k choices renumbered to d's local experts
 *     (0 .. E/G-1; -1 for other ranks' experts) and the weights (0 for other ranks' experts),
 *     so rank d routes them with tk_route_map (E/G experts), expands, runs its experts, and
 *     combines its own experts' rows per received token with tk_reduce into a bf16 partial;
 *   - the source sums the partial rows of a token over its destination ranks in ascending
 *     rank order, in fp32, rounded once to bf16 (tk_ep_combine).
 * The kernels only read and write through the pointers given; on several GPUs those are peer
 * addresses of the other ranks' buffers (the caller maps them, e.g. with symmetric memory) and
 * the caller orders the phases across ranks (a collective between dispatch and the
 * destinations' work, and between that and combine). No kernel waits on another rank.
 */

/* Bytes of device workspace tk_ep_layout needs. */
TK_API size_t tk_ep_layout_workspace_bytes(int T, int G);

/*
 * Send layout of one source rank: the route map over destination ranks.
 *   topk_idx      device, int32 [T, k] (expert -1 = masked pair: goes nowhere)
 *   send_counts   device, int32 [G]: tokens this rank sends to each rank
 *   send_offsets  device, int32 [G+1]: exclusive scan of send_counts
 *   dest_slot     device, int32 [T, G]: send_offsets[d] + (position of token t among the tokens
 *                 sent to d, in token order), or -1 when t does not go to d
 *   send_token    device, int32 [T*G]: the token of each send row (rows past send_offsets[G]
 *                 hold -1) -- a packed send buffer for a library all-to-all is
 *                 tk_expand(x, dest_slot, send_offsets, send_token, T, G, G, ...)
 *   workspace     device, tk_ep_layout_workspace_bytes(T, G) bytes, 16-byte aligned
 *   err_flag      device int32 or NULL: TK_DEVERR_EXPERT_RANGE for an expert outside [0,E)
 * 1 <= G <= TK_MAX_EP_RANKS, G divides E.
 */
TK_API tk_status tk_ep_layout(const int32_t* topk_idx, int T, int E, int k, int G,
                              int32_t* send_counts, int32_t* send_offsets, int32_t* dest_slot,
                              int32_t* send_token, void* workspace, size_t workspace_bytes,
                              int32_t* err_flag, void* stream);

/* One destination rank's receive buffers as seen from a source (device pointers, possibly a
 * peer GPU's memory; all 16-byte aligned). */
typedef struct tk_ep_peer {
    void* x;          /* [rows, H]: bf16 rows, or E4M3 codes (one byte per channel) */
    float* scale;     /* [rows, H/128] per-128-channel scales (E4M3 only; else NULL) */
    int32_t* idx;     /* [rows, k] local expert ids, -1 for other ranks' experts */
    float* w;         /* [rows, k] weights, 0 for other ranks' experts */
    int64_t base_row; /* first row of this source's block in these buffers */
    int64_t rows;     /* capacity of these buffers in rows (writes past it are skipped and
                         flagged TK_DEVERR_ROWS_RANGE) */
} tk_ep_peer;

/*
 * Dispatch of one source rank: every token row goes to each of its destination ranks, at row
 * base_row + (dest_slot[t*G+d] - send_offsets[d]) of rank d's buffers, as bf16 or quantised on
 * the way to E4M3 with per-128-channel scales (the same arithmetic as tk_expand's E4M3 path),
 * with its k local expert ids and weights. One bulk load of each row, one bulk store per
 * destination.
 *   x             device, bf16 [T, H], 16-byte aligned;  topk_idx, topk_w  device [T, k]
 *   dest_slot, send_offsets   from tk_ep_layout
 *   peers         HOST array of G descriptors (copied into the launch; may be freed on return)
 * H % 8 == 0 (H % 128 == 0 for E4M3).
 */
TK_API tk_status tk_ep_dispatch(const void* x, const int32_t* topk_idx, const float* topk_w,
                                const int32_t* dest_slot, const int32_t* send_offsets, int T,
                                int E, int k, int H, int G, int out_dtype, const tk_ep_peer* peers,
                                int32_t* err_flag, void* stream);

/*
 * Combine of one source rank: out[t] = bf16( sum over ranks d ascending with
 * dest_slot[t*G+d] >= 0 of fp32(partial[d][base_row[d] + dest_slot[t*G+d] - send_offsets[d]]) ),
 * fp32 adds (a token that went nowhere gets zeros). partial[d] is rank d's bf16 [rows[d], H]
 * buffer of per-received-row partial sums (tk_reduce over its local experts).
 *   partial, base_row, rows   HOST arrays of G entries (partial[d]: device pointer, possibly a
 *                 peer's memory, 16-byte aligned)
 *   out           device, bf16 [T, H], 16-byte aligned
 * A row index outside [0, rows[d]) is skipped and flagged TK_DEVERR_SLOT_RANGE.
 */
TK_API tk_status tk_ep_combine(const void* const* partial, const int64_t* base_row,
                               const int64_t* rows, const int32_t* dest_slot,
                               const int32_t* send_offsets, int T, int G, int H, void* out,
                               int32_t* err_flag, void* stream);

/*
 * Self-test of the library's bounded waits (no counterpart on the pages: it exists so that the
 * failure path can be exercised without faulting a GPU). One warp waits on an mbarrier that
 * nothing ever completes, using the same bounded wait as every kernel here; after limit_ns
 * nanoseconds (1 .. 2e9) the wait gives up, TK_DEVERR_TIMEOUT is ORed into *err_flag (device
 * int32) and the kernel returns, leaving the context usable.
 */
TK_API tk_status tk_selftest_bounded_wait(int64_t limit_ns, int32_t* err_flag, void* stream);

/*
 * Self-test of the gate's candidate filter (no counterpart on the pages: it checks on the GPU
 * the error bound the filter's margin rests on). For every finite fp32 logit l with
 * |l| <= 2^7 (about 2.2e9 values), the absolute difference between the filter's approximate
 * logistic value (ex2.approx / rcp.approx) and the exact fp32 sigmoid of the selection key;
 * the largest one is written to *max_err (device float; set to 0 first by this call). The
 * filter assumes it is below 2^-17 and keeps a margin of 2^-12.
 */
TK_API tk_status tk_selftest_gate_margin(float* max_err, void* stream);

/*
 * Self-test of the load-balance statistics' double-precision scores (no counterpart on the
 * pages: it checks on the GPU the accuracy of the short path that tk_balance_stats and
 * tk_balance_score_sums use for arguments of magnitude <= 708 -- a table-driven exponential
 * and a Newton-refined reciprocal -- against the library's exp and division). For every finite
 * fp32 l with |l| <= 708 (about 2.3e9 values), writes to max_rel_err[0] the largest relative
 * difference of e^-l and to max_rel_err[1] that of the logistic score 1/(1 + e^-l) (device
 * doubles, set to 0 first by this call). Both are expected within a few ulps (2^-50).
 */
TK_API tk_status tk_selftest_balance_exp(double* max_rel_err, void* stream);

/* Name of a status code (static string). */
TK_API const char* tk_status_str(int status);

/* Text describing the last non-OK status returned on the calling host thread (static
 * thread-local buffer, valid until the next call on that thread). */
TK_API const char* tk_last_error_detail(void);

/* ABI version of this header: (major << 16) | minor. The minor number grows when entry points
 * are added (1.2: tk_selftest_gate_margin and tk_selftest_balance_exp; 1.3:
 * tk_route_map_window); the major number would change only if an existing signature or meaning
 * did. */
TK_API int tk_abi_version(void);

#ifdef __cplusplus
}
#endif
#endif /* TK_ROUTE_H */
