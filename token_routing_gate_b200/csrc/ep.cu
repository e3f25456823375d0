// Expert-parallel dispatch over G ranks: the send layout and the fused (quantise +) send.
// Sources: 147227.xyz "刚刚！DeepSeek开源高性能GPU算子库TileKernels", its DeepEP paragraph
// (an expert-parallel all-to-all over NVLink with native FP8 dispatch), and 機器之心 "剛剛，
// DeepSeek開始頻繁更新：Tile Kernels、DeepEP V2", section "性能表現" (FP8 dispatch, BF16
// combine in the DeepSeek-V3 setting). The pages give no layout; the one used (experts in G
// contiguous groups, a token sent once per destination rank, receive rows source-major in token
// order, local expert ids) is stated with the entry points in tk_route.h.
//
// Layout = the token-to-expert map over ranks: a small kernel turns each token's k experts into
// the set of ranks that own them (rank d or -1, one entry per rank), and tk_route_map routes
// those "pairs" with G experts, giving per-rank counts, offsets and each token's stable position
// in every destination's list.
//
// Dispatch: one CTA per token. An elected lane bulk-loads the token row into shared memory
// (mbarrier with transaction count, bounded wait), then issues one bulk store of it per
// destination rank straight into that rank's receive buffer (a peer GPU's memory on several
// GPUs), so the transfer needs no staging copy; with E4M3 output the warps quantise the row in
// shared memory first and the codes are what is stored (the row crosses the link once per
// destination, at one byte per channel). The lanes write the k local expert ids and weights of
// the row for each destination. No kernel waits on another rank: the caller orders the phases.
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>

#include "quant_e4m3.cuh"
#include "tk_device.cuh"

namespace tk {
namespace {

constexpr uint32_t kEpChunkBytes = 32768;   // bf16 bytes staged per bulk load
constexpr int kEpFp8Threads = 256;
constexpr int kEpFp8ChunkChannels = 8192;   // channels quantised per stage
// Both dispatch kernels stay within the 48 KB of shared memory a CTA gets without an opt-in
// attribute: the dynamic stage below plus under 1 KB of static barriers and row counts.
constexpr size_t kEpFp8SmemMax = static_cast<size_t>(kEpFp8ChunkChannels) * 3 + (kEpFp8ChunkChannels / 128) * 4;
static_assert(kEpChunkBytes + 1024 <= 48 * 1024, "bf16 dispatch stage exceeds the default shared memory");
static_assert(kEpFp8SmemMax + 1024 <= 48 * 1024, "E4M3 dispatch stage exceeds the default shared memory");
constexpr int kMaskThreads = 256;

struct EpPeers {
    uint8_t* x[TK_MAX_EP_RANKS];
    float* scale[TK_MAX_EP_RANKS];
    int32_t* idx[TK_MAX_EP_RANKS];
    float* w[TK_MAX_EP_RANKS];
    int64_t base[TK_MAX_EP_RANKS];
    int64_t rows[TK_MAX_EP_RANKS];
};

size_t align_up(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

// rank_idx[t*G + d] = d if some expert of token t lives on rank d, else -1.
__global__ void __launch_bounds__(kMaskThreads)
ep_mask_kernel(const int32_t* __restrict__ topk_idx, int T, int E, int k, int G,
               int32_t* __restrict__ rank_idx, int32_t* err_flag) {
    pdl_wait();
    const int el = E / G;
    for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < T;
         t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        uint32_t mask = 0u;
        for (int j = 0; j < k; ++j) {
            const int e = topk_idx[t * k + j];
            if (e == -1) continue;
            if (e < 0 || e >= E) {
                flag_error(err_flag, TK_DEVERR_EXPERT_RANGE);
                continue;
            }
            mask |= 1u << (e / el);
        }
        for (int d = 0; d < G; ++d) rank_idx[t * G + d] = (mask >> d) & 1u ? d : -1;
    }
}

// Row of token t in destination `lane`'s buffers, or -1 (lanes >= G: -1).
__device__ __forceinline__ int64_t dest_row(const int32_t* dest_slot, const int32_t* send_offsets,
                                            const EpPeers& peers, int64_t t, int G, int lane,
                                            int32_t* err_flag) {
    if (lane >= G) return -1;
    const int raw = dest_slot[t * G + lane];
    if (raw == -1) return -1;
    const int64_t pos = static_cast<int64_t>(raw) - send_offsets[lane];
    const int64_t row = peers.base[lane] + pos;
    if (raw < 0 || pos < 0 || row >= peers.rows[lane]) {
        flag_error(err_flag, TK_DEVERR_ROWS_RANGE);
        return -1;
    }
    return row;
}

// Lanes j < k write the row's k local expert ids and weights into every destination's buffers.
__device__ __forceinline__ void write_choices(const EpPeers& peers, int64_t my_row, int G, int k,
                                              int el, int e, float wt, int lane) {
    const int owner = e >= 0 ? e / el : -1;
    for (int d = 0; d < G; ++d) {
        const int64_t row = __shfl_sync(kFullMask, my_row, d);
        if (row >= 0 && lane < k) {
            const bool mine = owner == d;
            peers.idx[d][row * k + lane] = mine ? e - d * el : -1;
            peers.w[d][row * k + lane] = mine ? wt : 0.0f;
        }
    }
}

__global__ void __launch_bounds__(32)
ep_dispatch_bf16_kernel(const uint8_t* __restrict__ x, const int32_t* __restrict__ topk_idx,
                        const float* __restrict__ topk_w, const int32_t* __restrict__ dest_slot,
                        const int32_t* __restrict__ send_offsets, int E, int k, int G,
                        uint32_t row_bytes, const __grid_constant__ EpPeers peers,
                        int32_t* err_flag) {
    extern __shared__ __align__(128) uint8_t stage[];
    __shared__ __align__(8) uint64_t bar;
    const int lane = threadIdx.x;
    const int64_t t = blockIdx.x;
    if (lane == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    __syncwarp();
    pdl_wait();
    const uint8_t* src = x + t * row_bytes;
    // the first piece of the row does not depend on where it goes: start its load before the
    // destinations are worked out
    if (lane == 0) {
        const uint32_t bytes0 = min(kEpChunkBytes, row_bytes);
        mbar_arrive_expect_tx(&bar, bytes0);
        bulk_load(stage, src, bytes0, &bar);
    }
    const int64_t my_row = dest_row(dest_slot, send_offsets, peers, t, G, lane, err_flag);
    int e = -1;
    float wt = 0.0f;
    if (lane < k) {
        e = topk_idx[t * k + lane];
        wt = topk_w[t * k + lane];
        if (e < -1 || e >= E) e = -1;   // tk_ep_layout flags these
    }
    write_choices(peers, my_row, G, k, E / G, e, wt, lane);

    const uint32_t nchunks = (row_bytes + kEpChunkBytes - 1) / kEpChunkBytes;
    for (uint32_t c = 0; c < nchunks; ++c) {
        const uint32_t off = c * kEpChunkBytes;
        const uint32_t bytes = min(kEpChunkBytes, row_bytes - off);
        int ok = 1;
        if (lane == 0) {
            if (c > 0) {
                bulk_wait_read_all();      // previous piece fully read by its stores
                fence_proxy_async_smem();
                mbar_arrive_expect_tx(&bar, bytes);
                bulk_load(stage, src + off, bytes, &bar);
            }
            ok = mbar_wait_bounded(&bar, c & 1u) ? 1 : 0;
            if (!ok) {
                flag_error(err_flag, TK_DEVERR_TIMEOUT);
                mbar_wait_bounded(&bar, c & 1u);  // give the copy in flight a second chance
            }
        }
        ok = __shfl_sync(kFullMask, ok, 0);
        if (!ok) break;
        for (int d = 0; d < G; ++d) {
            const int64_t row = __shfl_sync(kFullMask, my_row, d);
            if (lane == 0 && row >= 0) bulk_store(peers.x[d] + row * row_bytes + off, stage, bytes);
        }
        if (lane == 0) bulk_commit();
    }
    if (lane == 0) bulk_wait_read_all();
}

__global__ void __launch_bounds__(kEpFp8Threads)
ep_dispatch_fp8_kernel(const uint16_t* __restrict__ x, const int32_t* __restrict__ topk_idx,
                       const float* __restrict__ topk_w, const int32_t* __restrict__ dest_slot,
                       const int32_t* __restrict__ send_offsets, int E, int k, int G, int H,
                       const __grid_constant__ EpPeers peers, int32_t* err_flag) {
    extern __shared__ __align__(128) uint8_t sm[];
    const int chunk = min(H, kEpFp8ChunkChannels);
    uint16_t* xin = reinterpret_cast<uint16_t*>(sm);                          // [chunk] bf16
    uint8_t* qo = sm + static_cast<size_t>(chunk) * 2;                         // [chunk] E4M3
    float* sc = reinterpret_cast<float*>(sm + static_cast<size_t>(chunk) * 3);  // [chunk/128]
    __shared__ __align__(8) uint64_t bar;
    __shared__ int64_t rows[TK_MAX_EP_RANKS];
    __shared__ int load_ok;
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int64_t t = blockIdx.x;
    if (tid == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    __syncthreads();
    pdl_wait();
    // the first piece of the row does not depend on where it goes: start its load before the
    // destinations are worked out
    if (tid == 0) {
        const uint32_t bytes0 = static_cast<uint32_t>(min(chunk, H)) * 2u;
        mbar_arrive_expect_tx(&bar, bytes0);
        bulk_load(xin, x + t * H, bytes0, &bar);
    }
    if (warp == 0) {
        const int64_t my_row = dest_row(dest_slot, send_offsets, peers, t, G, lane, err_flag);
        if (lane < G) rows[lane] = my_row;
        int e = -1;
        float wt = 0.0f;
        if (lane < k) {
            e = topk_idx[t * k + lane];
            wt = topk_w[t * k + lane];
            if (e < -1 || e >= E) e = -1;
        }
        write_choices(peers, my_row, G, k, E / G, e, wt, lane);
    }
    __syncthreads();

    const int nb_row = H / 128;
    const int nchunks = (H + chunk - 1) / chunk;
    for (int c = 0; c < nchunks; ++c) {
        const int ch0 = c * chunk;
        const int chn = min(chunk, H - ch0);
        if (tid == 0) {
            if (c > 0) {
                bulk_wait_read_all();
                fence_proxy_async_smem();
                mbar_arrive_expect_tx(&bar, static_cast<uint32_t>(chn) * 2u);
                bulk_load(xin, x + t * H + ch0, static_cast<uint32_t>(chn) * 2u, &bar);
            }
            int ok = mbar_wait_bounded(&bar, static_cast<uint32_t>(c) & 1u) ? 1 : 0;
            if (!ok) {
                flag_error(err_flag, TK_DEVERR_TIMEOUT);
                mbar_wait_bounded(&bar, static_cast<uint32_t>(c) & 1u);
            }
            load_ok = ok;
        }
        __syncthreads();
        if (!load_ok) break;
        const int nb = chn / 128;
        for (int b = warp; b < nb; b += kEpFp8Threads / 32) {
            const float scale = quantize_block_e4m3(xin + b * 128, qo + b * 128, lane);
            if (lane == 0) sc[b] = scale;
        }
        fence_proxy_async_smem();
        __syncthreads();
        if (tid == 0) {
            for (int d = 0; d < G; ++d) {
                const int64_t row = rows[d];
                if (row >= 0) bulk_store(peers.x[d] + row * H + ch0, qo, static_cast<uint32_t>(chn));
            }
            bulk_commit();
        }
        const int b0 = ch0 / 128;
        for (int i = tid; i < G * nb; i += kEpFp8Threads) {
            const int d = i / nb;
            const int b = i - d * nb;
            const int64_t row = rows[d];
            if (row >= 0) peers.scale[d][row * nb_row + b0 + b] = sc[b];
        }
        __syncthreads();
    }
    if (tid == 0) bulk_wait_read_all();
}

}  // namespace
}  // namespace tk

extern "C" size_t tk_ep_layout_workspace_bytes(int T, int G) {
    if (T < 0 || G < 1 || G > TK_MAX_EP_RANKS) return 0;
    return tk::align_up(static_cast<size_t>(T) * G * sizeof(int32_t)) +
           tk_route_map_workspace_bytes(T, G, G);
}

extern "C" tk_status tk_ep_layout(const int32_t* topk_idx, int T, int E, int k, int G,
                                  int32_t* send_counts, int32_t* send_offsets, int32_t* dest_slot,
                                  int32_t* send_token, void* workspace, size_t workspace_bytes,
                                  int32_t* err_flag, void* stream) {
    using namespace tk;
    if (T < 0) return fail_arg("tk_ep_layout: T=%d must be >= 0", T);
    if (G < 1 || G > TK_MAX_EP_RANKS) return fail_arg("tk_ep_layout: G=%d outside [1, %d]", G, TK_MAX_EP_RANKS);
    if (E < 1 || E > TK_MAX_EXPERTS || E % G != 0)
        return fail_arg("tk_ep_layout: E=%d must be in [1, %d] and a multiple of G=%d", E, TK_MAX_EXPERTS, G);
    if (k < 1 || k > TK_MAX_TOPK) return fail_arg("tk_ep_layout: k=%d outside [1, %d]", k, TK_MAX_TOPK);
    if (send_counts == nullptr || send_offsets == nullptr || (T > 0 && (topk_idx == nullptr ||
        dest_slot == nullptr || send_token == nullptr)))
        return fail_arg("tk_ep_layout: output and input pointers must not be NULL");
    const size_t need = tk_ep_layout_workspace_bytes(T, G);
    if (workspace_bytes < need || (need > 0 && workspace == nullptr))
        return fail_arg("tk_ep_layout: workspace of %zu bytes, %zu needed", workspace_bytes, need);
    if (reinterpret_cast<uintptr_t>(workspace) % 16 != 0) return fail_arg("tk_ep_layout: workspace must be 16-byte aligned");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t* rank_idx = static_cast<int32_t*>(workspace);
    const size_t head = align_up(static_cast<size_t>(T) * G * sizeof(int32_t));
    if (T > 0) {
        const int grid = static_cast<int>(std::min<int64_t>((T + kMaskThreads - 1) / kMaskThreads, 4 * num_sms()));
        const cudaError_t e = launch_pdl(ep_mask_kernel, dim3(grid), dim3(kMaskThreads), 0, s, topk_idx,
                                         T, E, k, G, rank_idx, err_flag);
        if (e != cudaSuccess) return check_launch(e, "ep_mask_kernel");
    }
    return tk_route_map(rank_idx, T, G, G, 1, send_counts, send_offsets, dest_slot, send_token,
                        static_cast<uint8_t*>(workspace) + head, workspace_bytes - head, err_flag, stream);
}

extern "C" tk_status tk_ep_dispatch(const void* x, const int32_t* topk_idx, const float* topk_w,
                                    const int32_t* dest_slot, const int32_t* send_offsets, int T,
                                    int E, int k, int H, int G, int out_dtype,
                                    const tk_ep_peer* peers, int32_t* err_flag, void* stream) {
    using namespace tk;
    if (T < 0) return fail_arg("tk_ep_dispatch: T=%d must be >= 0", T);
    if (G < 1 || G > TK_MAX_EP_RANKS) return fail_arg("tk_ep_dispatch: G=%d outside [1, %d]", G, TK_MAX_EP_RANKS);
    if (E < 1 || E > TK_MAX_EXPERTS || E % G != 0)
        return fail_arg("tk_ep_dispatch: E=%d must be in [1, %d] and a multiple of G=%d", E, TK_MAX_EXPERTS, G);
    if (k < 1 || k > TK_MAX_TOPK) return fail_arg("tk_ep_dispatch: k=%d outside [1, %d]", k, TK_MAX_TOPK);
    if (out_dtype != TK_OUT_BF16 && out_dtype != TK_OUT_FP8_E4M3)
        return fail_arg("tk_ep_dispatch: unknown out_dtype %d", out_dtype);
    if (H < 8 || H % 8 != 0) return fail_arg("tk_ep_dispatch: H=%d must be a positive multiple of 8", H);
    if (out_dtype == TK_OUT_FP8_E4M3 && H % 128 != 0)
        return fail_arg("tk_ep_dispatch: H=%d must be a multiple of 128 for E4M3 output", H);
    if (static_cast<int64_t>(H) * 2 > INT32_MAX) return fail_arg("tk_ep_dispatch: H too large");
    if (peers == nullptr) return fail_arg("tk_ep_dispatch: peers must not be NULL");
    if (T == 0) return TK_OK;
    if (x == nullptr || topk_idx == nullptr || topk_w == nullptr || dest_slot == nullptr ||
        send_offsets == nullptr)
        return fail_arg("tk_ep_dispatch: x, topk_idx, topk_w, dest_slot and send_offsets must not be NULL");
    if (reinterpret_cast<uintptr_t>(x) % 16 != 0) return fail_arg("tk_ep_dispatch: x must be 16-byte aligned");
    EpPeers p{};
    for (int d = 0; d < G; ++d) {
        const tk_ep_peer& q = peers[d];
        if (q.rows < 0 || q.base_row < 0) return fail_arg("tk_ep_dispatch: rank %d has negative rows or base_row", d);
        if (q.rows > 0) {
            if (q.x == nullptr || q.idx == nullptr || q.w == nullptr ||
                (out_dtype == TK_OUT_FP8_E4M3 && q.scale == nullptr))
                return fail_arg("tk_ep_dispatch: rank %d's receive buffers must not be NULL", d);
            if (reinterpret_cast<uintptr_t>(q.x) % 16 != 0)
                return fail_arg("tk_ep_dispatch: rank %d's receive rows must be 16-byte aligned", d);
        }
        p.x[d] = static_cast<uint8_t*>(q.x);
        p.scale[d] = q.scale;
        p.idx[d] = q.idx;
        p.w[d] = q.w;
        p.base[d] = q.base_row;
        p.rows[d] = q.rows;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t err;
    if (out_dtype == TK_OUT_BF16) {
        const uint32_t row_bytes = static_cast<uint32_t>(H) * 2u;
        const uint32_t smem = min(row_bytes, kEpChunkBytes);
        err = launch_pdl(ep_dispatch_bf16_kernel, dim3(T), dim3(32), smem, s,
                         static_cast<const uint8_t*>(x), topk_idx, topk_w, dest_slot, send_offsets, E,
                         k, G, row_bytes, p, err_flag);
        return check_launch(err, "ep_dispatch_bf16_kernel");
    }
    const int chunk = H < kEpFp8ChunkChannels ? H : kEpFp8ChunkChannels;
    const size_t smem = static_cast<size_t>(chunk) * 3 + static_cast<size_t>(chunk / 128) * 4;
    err = launch_pdl(ep_dispatch_fp8_kernel, dim3(T), dim3(kEpFp8Threads), smem, s,
                     static_cast<const uint16_t*>(x), topk_idx, topk_w, dest_slot, send_offsets, E, k,
                     G, H, p, err_flag);
    return check_launch(err, "ep_dispatch_fp8_kernel");
}
