// Token-to-expert map: per-expert histogram -> scan for segment offsets -> stable expert-major
// slots (機器之心 "剛剛，DeepSeek開始頻繁更新", section "Tile Kernels": token-to-expert
// mapping is one of the MoE routing ops).
//
// The pairs p = t*k + j are cut into tiles of kTileTokens tokens. Three short kernels (the last
// two run as one kernel, route_scan_scatter_kernel, while the batch has at most 128 tiles):
//   count   : one CTA per tile counts its pairs per expert in shared memory (integer atomics,
//             so the counts do not depend on their order) and writes a row of the
//             [tiles x E] count matrix; the grid also fills token_of with -1.
//   scan    : one CTA turns each column of the matrix into exclusive per-tile prefixes, sums
//             the column into counts[e], rounds it up to the alignment and scans over experts
//             for offsets[].
//   scatter : one CTA per tile marks, per expert, which of its tokens chose that expert in a
//             shared-memory bitmap; a pair's rank inside the tile is the population count of
//             the bits below its token. slot = offsets[e] + tile prefix[e] + rank -- the same
//             number a sequential pass in p order hands out, with no dependence on thread
//             timing.
#include <cuda_runtime.h>
#include <stdint.h>

#include "tk_device.cuh"

namespace tk {
namespace {

constexpr int kTileTokens = 256;               // tokens per tile
constexpr int kTileWords = kTileTokens / 32;   // bitmap words per expert
constexpr int kRouteThreads = 512;
constexpr int kPairsPerThread = kTileTokens * TK_MAX_TOPK / kRouteThreads;  // 16
constexpr int kScanThreads = 1024;
constexpr int kScanBatch = 32;                 // column loads in flight per thread
constexpr int kFusedMaxTiles = 128;            // up to here every scatter CTA scans for itself

inline int num_tiles(int T) { return (T + kTileTokens - 1) / kTileTokens; }

// The scan kernel gives each expert its own thread: E rounded up to whole warps.
inline int scan_threads(int E) {
    const int t = (E + 31) / 32 * 32;
    return t < kScanThreads ? t : kScanThreads;
}

__global__ void __launch_bounds__(kRouteThreads)
route_count_kernel(const int32_t* __restrict__ topk_idx, int T, int E, int k,
                   int32_t* __restrict__ tile_counts, int32_t* __restrict__ token_of,
                   int64_t rmax, int32_t* err_flag) {
    extern __shared__ int32_t cnt[];  // [E]
    pdl_wait();
    const int tile = blockIdx.x;
    const int64_t p0 = static_cast<int64_t>(tile) * kTileTokens * k;
    const int64_t p1 = min(static_cast<int64_t>(T), static_cast<int64_t>(tile + 1) * kTileTokens) * k;
    // all index loads of this thread first, so their latencies overlap
    const int iters = static_cast<int>((p1 - p0 + kRouteThreads - 1) / kRouteThreads);
    int e_reg[kPairsPerThread];
#pragma unroll
    for (int i = 0; i < kPairsPerThread; ++i) {
        const int64_t p = p0 + threadIdx.x + static_cast<int64_t>(i) * kRouteThreads;
        e_reg[i] = (i < iters && p < p1) ? topk_idx[p] : -1;
    }
    for (int e = threadIdx.x; e < E; e += kRouteThreads) cnt[e] = 0;
    // every row starts as "no token"; the scatter kernel fills the real rows afterwards
    for (int64_t r = static_cast<int64_t>(blockIdx.x) * kRouteThreads + threadIdx.x; r < rmax;
         r += static_cast<int64_t>(gridDim.x) * kRouteThreads)
        token_of[r] = -1;
    __syncthreads();
#pragma unroll
    for (int i = 0; i < kPairsPerThread; ++i) {
        if (i >= iters) break;
        const int64_t p = p0 + threadIdx.x + static_cast<int64_t>(i) * kRouteThreads;
        if (p >= p1) continue;
        const int e = e_reg[i];
        if (e < 0 || e >= E) {  // -1 is a masked pair (tk_tp_mask), anything else an error
            if (e != -1) flag_error(err_flag, TK_DEVERR_EXPERT_RANGE);
            continue;
        }
        atomicAdd(&cnt[e], 1);  // integer counts: the order of the additions does not matter
    }
    __syncthreads();
    if (p0 < p1 || tile == 0) {
        for (int e = threadIdx.x; e < E; e += kRouteThreads)
            tile_counts[static_cast<int64_t>(tile) * E + e] = cnt[e];
    }
}

// ---- rank phase shared by every scatter variant: bitmap of the tile's tokens per expert, then
// slot = base[e] + (number of the tile's earlier tokens on expert e)
__device__ __forceinline__ void tile_mark(uint32_t* bitmap, const int (&e_reg)[kPairsPerThread],
                                          int iters, int64_t p0, int64_t p1, int k, int t0, int E,
                                          int32_t* err_flag) {
#pragma unroll
    for (int i = 0; i < kPairsPerThread; ++i) {
        if (i >= iters) break;
        const int64_t p = p0 + threadIdx.x + static_cast<int64_t>(i) * kRouteThreads;
        const int e = e_reg[i];
        if (p >= p1 || e < 0 || e >= E) continue;  // out-of-range experts: flagged elsewhere
        const int tl = static_cast<int>(p / k) - t0;
        const uint32_t bit = 1u << (tl & 31);
        const uint32_t old = atomicOr(&bitmap[e * kTileWords + (tl >> 5)], bit);
        if (old & bit) flag_error(err_flag, TK_DEVERR_DUP_EXPERT);
    }
}

__device__ __forceinline__ void tile_scatter(const uint32_t* bitmap, const int32_t* base,
                                             const int (&e_reg)[kPairsPerThread], int iters,
                                             int64_t p0, int64_t p1, int k, int t0, int E,
                                             int32_t* slot_of, int32_t* token_of) {
#pragma unroll
    for (int i = 0; i < kPairsPerThread; ++i) {
        if (i >= iters) break;
        const int64_t p = p0 + threadIdx.x + static_cast<int64_t>(i) * kRouteThreads;
        if (p >= p1) continue;
        const int e = e_reg[i];
        if (e < 0 || e >= E) {
            slot_of[p] = -1;
            continue;
        }
        const int t = static_cast<int>(p / k);
        const int tl = t - t0;
        const uint32_t* bm = bitmap + e * kTileWords;
        int rank = __popc(bm[tl >> 5] & ((1u << (tl & 31)) - 1u));
        for (int w = 0; w < (tl >> 5); ++w) rank += __popc(bm[w]);
        const int32_t slot = base[e] + rank;
        slot_of[p] = slot;
        token_of[slot] = t;
    }
}

__device__ __forceinline__ int load_tile(const int32_t* topk_idx, int64_t p0, int64_t p1,
                                         int (&e_reg)[kPairsPerThread]) {
    const int iters = static_cast<int>((p1 - p0 + kRouteThreads - 1) / kRouteThreads);
#pragma unroll
    for (int i = 0; i < kPairsPerThread; ++i) {
        const int64_t p = p0 + threadIdx.x + static_cast<int64_t>(i) * kRouteThreads;
        e_reg[i] = (i < iters && p < p1) ? topk_idx[p] : -1;
    }
    return iters;
}

// Exclusive scan of ceil(total[e]/align)*align over experts, for a whole CTA of kRouteThreads
// threads: writes excl[e] (the segment offset of expert e) and returns the grand total R.
__device__ __forceinline__ int32_t cta_padded_scan(const int32_t* total, int E, int align,
                                                   int32_t* excl, int32_t* warp_tot) {
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    int32_t carry = 0;
    for (int e0 = 0; e0 < E; e0 += kRouteThreads) {
        const int e = e0 + threadIdx.x;
        const int32_t padded = e < E ? (total[e] + align - 1) / align * align : 0;
        int32_t incl = padded;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int32_t u = __shfl_up_sync(kFullMask, incl, off);
            if (lane >= off) incl += u;
        }
        if (lane == 31) warp_tot[warp] = incl;
        __syncthreads();
        if (warp == 0) {
            constexpr int nw = kRouteThreads / 32;
            int32_t u = lane < nw ? warp_tot[lane] : 0;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int32_t q = __shfl_up_sync(kFullMask, u, off);
                if (lane >= off) u += q;
            }
            if (lane < nw) warp_tot[lane] = u;
        }
        __syncthreads();
        if (e < E) excl[e] = carry + (warp > 0 ? warp_tot[warp - 1] : 0) + incl - padded;
        carry += warp_tot[kRouteThreads / 32 - 1];
        __syncthreads();
    }
    return carry;
}

// Single CTA. Column e of tile_counts becomes exclusive per-tile prefixes (in place).
__global__ void __launch_bounds__(kScanThreads)
route_scan_kernel(int32_t* __restrict__ tile_counts, int tiles, int E, int align,
                  int32_t* __restrict__ counts, int32_t* __restrict__ offsets) {
    __shared__ int32_t warp_tot[kScanThreads / 32];
    __shared__ int32_t carry;
    pdl_wait();
    if (threadIdx.x == 0) carry = 0;
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    // experts in chunks of blockDim.x; each thread owns one expert of the chunk
    for (int e0 = 0; e0 < E; e0 += blockDim.x) {
        const int e = e0 + threadIdx.x;
        int32_t padded = 0;
        if (e < E) {
            int32_t run = 0;
            for (int c0 = 0; c0 < tiles; c0 += kScanBatch) {
                int32_t v[kScanBatch];
#pragma unroll
                for (int i = 0; i < kScanBatch; ++i)
                    v[i] = c0 + i < tiles ? tile_counts[static_cast<int64_t>(c0 + i) * E + e] : 0;
#pragma unroll
                for (int i = 0; i < kScanBatch; ++i) {
                    if (c0 + i < tiles) tile_counts[static_cast<int64_t>(c0 + i) * E + e] = run;
                    run += v[i];
                }
            }
            counts[e] = run;
            padded = (run + align - 1) / align * align;
        }
        // block-wide exclusive scan of padded over this chunk of experts
        int32_t incl = padded;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int32_t v = __shfl_up_sync(kFullMask, incl, off);
            if (lane >= off) incl += v;
        }
        if (lane == 31) warp_tot[warp] = incl;
        __syncthreads();
        if (warp == 0) {
            const int nw = blockDim.x / 32;
            int32_t v = lane < nw ? warp_tot[lane] : 0;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int32_t u = __shfl_up_sync(kFullMask, v, off);
                if (lane >= off) v += u;
            }
            if (lane < nw) warp_tot[lane] = v;  // inclusive over warps
        }
        __syncthreads();
        const int32_t warp_excl = warp > 0 ? warp_tot[warp - 1] : 0;
        const int32_t excl = carry + warp_excl + incl - padded;
        if (e < E) offsets[e] = excl;
        const int32_t chunk_total = warp_tot[blockDim.x / 32 - 1];
        __syncthreads();
        if (threadIdx.x == 0) carry += chunk_total;
        __syncthreads();
    }
    if (threadIdx.x == 0) offsets[E] = carry;
}

__global__ void __launch_bounds__(kRouteThreads)
route_scatter_kernel(const int32_t* __restrict__ topk_idx, int T, int E, int k,
                     const int32_t* __restrict__ tile_prefix, const int32_t* __restrict__ offsets,
                     int32_t* __restrict__ slot_of, int32_t* __restrict__ token_of,
                     int32_t* err_flag) {
    extern __shared__ uint32_t smem[];
    uint32_t* bitmap = smem;                                          // [E][kTileWords]
    int32_t* base = reinterpret_cast<int32_t*>(smem + E * kTileWords);  // [E]
    pdl_wait();
    const int tile = blockIdx.x;
    const int t0 = tile * kTileTokens;
    const int64_t p0 = static_cast<int64_t>(t0) * k;
    const int64_t p1 = static_cast<int64_t>(min(T, t0 + kTileTokens)) * k;
    int e_reg[kPairsPerThread];
    const int iters = load_tile(topk_idx, p0, p1, e_reg);
    for (int i = threadIdx.x; i < E * kTileWords; i += kRouteThreads) bitmap[i] = 0u;
    for (int e = threadIdx.x; e < E; e += kRouteThreads)
        base[e] = offsets[e] + tile_prefix[static_cast<int64_t>(tile) * E + e];
    __syncthreads();
    tile_mark(bitmap, e_reg, iters, p0, p1, k, t0, E, err_flag);
    __syncthreads();
    tile_scatter(bitmap, base, e_reg, iters, p0, p1, k, t0, E, slot_of, token_of);
}

// Scan and scatter in one kernel, for batches of at most kFusedMaxTiles tiles: every CTA reads
// the whole (small) count matrix itself -- its own tile's prefix per expert, and every column's
// total for the offsets -- instead of waiting for a separate scan kernel. CTA 0 also writes
// counts[] and offsets[]. The slot arithmetic is the same as route_scan + route_scatter.
__global__ void __launch_bounds__(kRouteThreads, 1)
route_scan_scatter_kernel(const int32_t* __restrict__ topk_idx, int T, int E, int k, int align,
                          const int32_t* __restrict__ tile_counts, int tiles,
                          int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                          int32_t* __restrict__ slot_of, int32_t* __restrict__ token_of,
                          int32_t* err_flag) {
    extern __shared__ uint32_t smem[];
    uint32_t* bitmap = smem;                                              // [E][kTileWords]
    int32_t* before = reinterpret_cast<int32_t*>(bitmap + E * kTileWords);  // [E]
    int32_t* total = before + E;                                          // [E]
    int32_t* base = total + E;                                            // [E]
    __shared__ int32_t warp_tot[kRouteThreads / 32];
    pdl_wait();
    const int tile = blockIdx.x;
    const int t0 = tile * kTileTokens;
    const int64_t p0 = static_cast<int64_t>(t0) * k;
    const int64_t p1 = static_cast<int64_t>(min(T, t0 + kTileTokens)) * k;
    int e_reg[kPairsPerThread];
    const int iters = load_tile(topk_idx, p0, p1, e_reg);
    for (int i = threadIdx.x; i < E * kTileWords; i += kRouteThreads) bitmap[i] = 0u;
    // per expert: the count over the tiles before this one, and the column total
    for (int e = threadIdx.x; e < E; e += kRouteThreads) {
        int32_t b = 0, tot = 0;
        for (int c0 = 0; c0 < tiles; c0 += kScanBatch) {
            int32_t v[kScanBatch];
#pragma unroll
            for (int i = 0; i < kScanBatch; ++i)
                v[i] = c0 + i < tiles ? tile_counts[static_cast<int64_t>(c0 + i) * E + e] : 0;
#pragma unroll
            for (int i = 0; i < kScanBatch; ++i) {
                if (c0 + i < tile) b += v[i];
                tot += v[i];
            }
        }
        before[e] = b;
        total[e] = tot;
    }
    __syncthreads();
    const int32_t R = cta_padded_scan(total, E, align, base, warp_tot);
    for (int e = threadIdx.x; e < E; e += kRouteThreads) {
        if (tile == 0) {
            counts[e] = total[e];
            offsets[e] = base[e];
        }
        base[e] += before[e];
    }
    if (tile == 0 && threadIdx.x == 0) offsets[E] = R;
    __syncthreads();
    tile_mark(bitmap, e_reg, iters, p0, p1, k, t0, E, err_flag);
    __syncthreads();
    tile_scatter(bitmap, base, e_reg, iters, p0, p1, k, t0, E, slot_of, token_of);
}

}  // namespace

size_t route_map_workspace_bytes_impl(int T, int E) {
    const int tiles = num_tiles(T) > 0 ? num_tiles(T) : 1;
    return static_cast<size_t>(tiles) * static_cast<size_t>(E) * sizeof(int32_t);
}

}  // namespace tk

extern "C" int64_t tk_max_rows(int T, int E, int k, int align) {
    return static_cast<int64_t>(T) * k + static_cast<int64_t>(E) * (align - 1);
}

extern "C" size_t tk_route_map_workspace_bytes(int T, int E, int k) {
    (void)k;
    if (T < 0 || E < 1) return 0;
    return tk::route_map_workspace_bytes_impl(T, E);
}

extern "C" tk_status tk_route_map(const int32_t* topk_idx, int T, int E, int k, int align,
                                  int32_t* counts, int32_t* offsets, int32_t* slot_of,
                                  int32_t* token_of, void* workspace, size_t workspace_bytes,
                                  int32_t* err_flag, void* stream) {
    using namespace tk;
    if (T < 0) return fail_arg("tk_route_map: T=%d must be >= 0", T);
    if (E < 1 || E > TK_MAX_EXPERTS) return fail_arg("tk_route_map: E=%d outside [1, %d]", E, TK_MAX_EXPERTS);
    if (k < 1 || k > TK_MAX_TOPK) return fail_arg("tk_route_map: k=%d outside [1, %d]", k, TK_MAX_TOPK);
    if (align < 1 || align > 4096) return fail_arg("tk_route_map: align=%d outside [1, 4096]", align);
    const int64_t rmax = tk_max_rows(T, E, k, align);
    if (rmax > INT32_MAX) return fail_arg("tk_route_map: T*k + E*(align-1) = %lld exceeds int32", (long long)rmax);
    if (counts == nullptr || offsets == nullptr || workspace == nullptr)
        return fail_arg("tk_route_map: counts, offsets and workspace must not be NULL");
    if (T > 0 && (topk_idx == nullptr || slot_of == nullptr))
        return fail_arg("tk_route_map: topk_idx and slot_of must not be NULL");
    if (rmax > 0 && token_of == nullptr) return fail_arg("tk_route_map: token_of must not be NULL");
    const size_t need = route_map_workspace_bytes_impl(T, E);
    if (workspace_bytes < need)
        return fail_arg("tk_route_map: workspace holds %zu bytes, needs %zu", workspace_bytes, need);
    if (reinterpret_cast<uintptr_t>(workspace) % 16 != 0)
        return fail_arg("tk_route_map: workspace must be 16-byte aligned");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t* tile_counts = static_cast<int32_t*>(workspace);
    const int tiles = num_tiles(T);
    const int count_grid = tiles > 0 ? tiles : 1;
    cudaError_t err = launch_pdl(route_count_kernel, dim3(count_grid), dim3(kRouteThreads),
                                 static_cast<size_t>(E) * sizeof(int32_t), s, topk_idx, T, E, k,
                                 tile_counts, token_of, rmax, err_flag);
    if (err != cudaSuccess) return check_launch(err, "route_count_kernel");
    if (tiles > 0 && tiles <= kFusedMaxTiles) {
        const size_t smem = static_cast<size_t>(E) * (kTileWords + 3) * sizeof(uint32_t);
        err = launch_pdl(route_scan_scatter_kernel, dim3(tiles), dim3(kRouteThreads), smem, s,
                         topk_idx, T, E, k, align, static_cast<const int32_t*>(tile_counts), tiles,
                         counts, offsets, slot_of, token_of, err_flag);
        return check_launch(err, "route_scan_scatter_kernel");
    }
    err = launch_pdl(route_scan_kernel, dim3(1), dim3(scan_threads(E)), 0, s, tile_counts, tiles, E,
                     align, counts, offsets);
    if (err != cudaSuccess) return check_launch(err, "route_scan_kernel");
    if (tiles > 0) {
        const size_t smem = static_cast<size_t>(E) * (kTileWords + 1) * sizeof(uint32_t);
        err = launch_pdl(route_scatter_kernel, dim3(tiles), dim3(kRouteThreads), smem, s, topk_idx,
                         T, E, k, static_cast<const int32_t*>(tile_counts),
                         static_cast<const int32_t*>(offsets), slot_of, token_of, err_flag);
        if (err != cudaSuccess) return check_launch(err, "route_scatter_kernel");
    }
    return TK_OK;
}

// ------------------------------------------------------------------------------------------
// Allocation-free variant of tk_route_map.
//
// Some callers cannot hand the library a workspace: a serving engine or plugin host that owns
// every byte of device memory and passes a component only its input and output buffers, or a
// latency-critical loop where a cudaMalloc (which can synchronise the device) is not allowed.
// For them the tile-count matrix lives in a fixed array compiled into this library. Every GPU
// that loads the library reserves it (1 MiB) until the process exits.
//
// The array's name is only a host-side stand-in in host code; its device address is looked up
// with cudaGetSymbolAddress once per device (with that device current) on the first call on
// that device, and cached. The kernels write every entry they later read, so nothing in the
// array has to start at zero. All calls on one device share the array: calls that can overlap
// on the GPU (other streams, other host threads) race on it and must be serialised by the
// caller.
// ------------------------------------------------------------------------------------------
#include <mutex>

namespace {
constexpr size_t kStaticScratchInts = 256 * 1024;  // 1 MiB of int32 tile counts
static __device__ __align__(256) int32_t tk_route_static_scratch[kStaticScratchInts];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
int32_t* g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of tk_route_static_scratch on the current device (looked up once per device).
tk_status static_scratch(int32_t** out) {
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return tk::check_launch(err, "tk_route_map_static: cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices)
        return tk::fail_arg("tk_route_map_static: device index %d is beyond %d", dev, kMaxDevices);
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (g_scratch_ptr[dev] == nullptr) {
        void* p = nullptr;
        err = cudaGetSymbolAddress(&p, tk_route_static_scratch);
        if (err != cudaSuccess)
            return tk::check_launch(err, "tk_route_map_static: cudaGetSymbolAddress");
        g_scratch_ptr[dev] = static_cast<int32_t*>(p);
    }
    *out = g_scratch_ptr[dev];
    return TK_OK;
}
}  // namespace

extern "C" tk_status tk_route_map_static(const int32_t* topk_idx, int T, int E, int k, int align,
                                         int32_t* counts, int32_t* offsets, int32_t* slot_of,
                                         int32_t* token_of, int32_t* err_flag, void* stream) {
    using namespace tk;
    if (T < 0) return fail_arg("tk_route_map_static: T=%d must be >= 0", T);
    if (E < 1 || E > TK_MAX_EXPERTS)
        return fail_arg("tk_route_map_static: E=%d outside [1, %d]", E, TK_MAX_EXPERTS);
    if (k < 1 || k > TK_MAX_TOPK) return fail_arg("tk_route_map_static: k=%d outside [1, %d]", k, TK_MAX_TOPK);
    if (align < 1 || align > 4096)
        return fail_arg("tk_route_map_static: align=%d outside [1, 4096]", align);
    const int64_t rmax = tk_max_rows(T, E, k, align);
    if (rmax > INT32_MAX)
        return fail_arg("tk_route_map_static: T*k + E*(align-1) = %lld exceeds int32", (long long)rmax);
    const size_t need = route_map_workspace_bytes_impl(T, E) / sizeof(int32_t);
    if (need > kStaticScratchInts)
        return fail_arg("tk_route_map_static: T=%d, E=%d need %zu scratch entries but the built-in "
                        "buffer holds %zu (at most %zu tiles of 256 tokens times E); use "
                        "tk_route_map with a caller workspace", T, E, need, kStaticScratchInts,
                        kStaticScratchInts / static_cast<size_t>(E));
    if (counts == nullptr || offsets == nullptr)
        return fail_arg("tk_route_map_static: counts and offsets must not be NULL");
    if (T > 0 && (topk_idx == nullptr || slot_of == nullptr))
        return fail_arg("tk_route_map_static: topk_idx and slot_of must not be NULL");
    if (rmax > 0 && token_of == nullptr) return fail_arg("tk_route_map_static: token_of must not be NULL");
    int32_t* tile_counts = nullptr;
    const tk_status st = static_scratch(&tile_counts);
    if (st != TK_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int tiles = num_tiles(T);
    const int count_grid = tiles > 0 ? tiles : 1;
    cudaError_t err = launch_pdl(route_count_kernel, dim3(count_grid), dim3(kRouteThreads),
                                 static_cast<size_t>(E) * sizeof(int32_t), s, topk_idx, T, E, k,
                                 tile_counts, token_of, rmax, err_flag);
    if (err != cudaSuccess) return check_launch(err, "route_count_kernel");
    err = launch_pdl(route_scan_kernel, dim3(1), dim3(kScanThreads), 0, s, tile_counts, tiles, E,
                     align, counts, offsets);
    if (err != cudaSuccess) return check_launch(err, "route_scan_kernel");
    if (tiles > 0) {
        const size_t smem = static_cast<size_t>(E) * (kTileWords + 1) * sizeof(uint32_t);
        err = launch_pdl(route_scatter_kernel, dim3(tiles), dim3(kRouteThreads), smem, s, topk_idx,
                         T, E, k, static_cast<const int32_t*>(tile_counts),
                         static_cast<const int32_t*>(offsets), slot_of, token_of, err_flag);
        if (err != cudaSuccess) return check_launch(err, "route_scatter_kernel");
    }
    return TK_OK;
}
