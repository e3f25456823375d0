// Token-to-expert map: per-expert histogram -> scan for segment offsets -> stable expert-major
// slots (機器之心 "剛剛，DeepSeek開始頻繁更新", section "Tile Kernels": token-to-expert
// mapping is one of the MoE routing ops).
//
// The pairs p = t*k + j are cut into tiles of kTileTokens tokens. Three short kernels (the last
// two run as one kernel, route_scan_scatter_kernel, while the count matrix is small):
//   count   : one CTA per tile counts its pairs per expert in shared memory (integer atomics,
//             so the counts do not depend on their order) and writes a column of the
//             [E x tiles] count matrix (expert-major, each expert's row padded to a multiple of
//             4 tiles so that it reads as 16-byte vectors); the grid also fills token_of with -1.
//   scan    : turns each expert's row into exclusive per-tile prefixes, sums it into
//             counts[e], rounds it up to the alignment and scans over experts for offsets[]
//             (for large matrices the rows are scanned on many CTAs and the scatter kernel
//             forms the offsets).
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

constexpr int kTileTokens = 128;               // tokens per tile
constexpr int kTileWords = kTileTokens / 32;   // bitmap words per expert
constexpr int kRouteThreads = 512;
constexpr int kPairsPerThread = kTileTokens * TK_MAX_TOPK / kRouteThreads;  // 8
constexpr int kScanThreads = 1024;
constexpr int kRowBatch = 8;                   // 16-byte loads in flight per expert row
// The fused scan + scatter kernel has every CTA read the whole count matrix; beyond this many
// entries the many-CTA row scan reads it once instead (at E = 256 and k = 8 after an L2 flush:
// 16,384 tokens fused 13-15 us, separate 19.5; 32,768 tokens fused 25.6, separate 21.5).
constexpr int64_t kFusedMaxEntries = 32 * 1024;

inline int num_tiles(int T) { return (T + kTileTokens - 1) / kTileTokens; }
// Row length of the count matrix: the tiles rounded up to whole 16-byte vectors.
inline int row_stride(int tiles) { return (tiles + 3) / 4 * 4; }

// The scan kernel gives each expert its own thread: E rounded up to whole warps.
inline int scan_threads(int E) {
    const int t = (E + 31) / 32 * 32;
    return t < kScanThreads ? t : kScanThreads;
}

// Exact n / k for 0 <= n < 2^16 and 1 <= k <= 32 by a multiply-high with m = ceil(2^32 / k):
// n * m / 2^32 = n / k + n * r / (k * 2^32) with r = m*k - 2^32 < k, and the second term is
// below 2^-16 / k, too small to carry n / k past the next integer.
struct DivK {
    uint64_t m;
    __device__ __forceinline__ explicit DivK(int k)
        : m((UINT64_C(0x100000000) + static_cast<uint64_t>(k) - 1) / static_cast<uint64_t>(k)) {}
    __device__ __forceinline__ int operator()(int n) const {
        return static_cast<int>((static_cast<uint64_t>(n) * m) >> 32);
    }
};

// Pairs p0 + threadIdx.x + i * kRouteThreads, i < the result, lie inside a tile of n pairs.
__device__ __forceinline__ int pairs_of_thread(int n) {
    return n > static_cast<int>(threadIdx.x) ? (n - 1 - static_cast<int>(threadIdx.x)) / kRouteThreads + 1 : 0;
}

// The local expert of a pair's index: raw - lo inside the window [lo, lo + E), else -1
// (masked). The whole map is the window lo = 0, E = all experts.
__device__ __forceinline__ int window_expert(int raw, int lo, int E) {
    const int64_t e = static_cast<int64_t>(raw) - lo;
    return (e >= 0 && e < E) ? static_cast<int>(e) : -1;
}

// kWindow: the experts [lo, lo + E) of e_total (tk_route_map_window); otherwise all E of them,
// with the same code as before windows existed.
template <bool kWindow>
__global__ void __launch_bounds__(kRouteThreads)
route_count_kernel(const int32_t* __restrict__ topk_idx, int T, int E, int k, int lo, int e_total,
                   int32_t* __restrict__ tile_counts, int stride, int32_t* __restrict__ token_of,
                   int64_t rmax, int32_t* err_flag) {
    extern __shared__ int32_t cnt[];  // [E]
    pdl_wait();
    const int tile = blockIdx.x;
    const int64_t p0 = static_cast<int64_t>(tile) * kTileTokens * k;
    const int n = static_cast<int>(min(static_cast<int64_t>(T), static_cast<int64_t>(tile + 1) * kTileTokens) * k - p0);
    // all index loads of this thread first, so their latencies overlap
    int e_reg[kPairsPerThread];
    const int mine = pairs_of_thread(n);
#pragma unroll
    for (int i = 0; i < kPairsPerThread; ++i) {
        if (i >= mine) break;
        e_reg[i] = topk_idx[p0 + threadIdx.x + i * kRouteThreads];
    }
    for (int e = threadIdx.x; e < E; e += kRouteThreads) cnt[e] = 0;
    // every row starts as "no token"; the scatter kernel fills the real rows afterwards
    for (int64_t r = static_cast<int64_t>(blockIdx.x) * kRouteThreads + threadIdx.x; r < rmax;
         r += static_cast<int64_t>(gridDim.x) * kRouteThreads)
        token_of[r] = -1;
    __syncthreads();
#pragma unroll
    for (int i = 0; i < kPairsPerThread; ++i) {
        if (i >= mine) break;
        int e = e_reg[i];
        if constexpr (kWindow) {
            // -1 is a masked pair (tk_tp_mask), an index outside [0, e_total) an error
            if (e != -1 && (e < 0 || e >= e_total)) flag_error(err_flag, TK_DEVERR_EXPERT_RANGE);
            e = window_expert(e, lo, E);
            if (e < 0) continue;
        } else if (e < 0 || e >= E) {  // -1 is a masked pair (tk_tp_mask), anything else an error
            if (e != -1) flag_error(err_flag, TK_DEVERR_EXPERT_RANGE);
            continue;
        }
        atomicAdd(&cnt[e], 1);  // integer counts: the order of the additions does not matter
    }
    __syncthreads();
    if (n > 0) {
        for (int e = threadIdx.x; e < E; e += kRouteThreads)
            tile_counts[static_cast<int64_t>(e) * stride + tile] = cnt[e];
    }
    // the last tile also zeroes each row's padding, so rows can be summed in whole vectors
    if (tile == gridDim.x - 1) {
        const int pad = stride - (tile + 1);
        for (int i = threadIdx.x; i < E * pad; i += kRouteThreads)
            tile_counts[static_cast<int64_t>(i / pad) * stride + tile + 1 + i % pad] = 0;
    }
}

// ---- rank phase shared by every scatter variant: bitmap of the tile's tokens per expert, then
// slot = base[e] + (number of the tile's earlier tokens on expert e)
__device__ __forceinline__ void tile_mark(uint32_t* bitmap, const int (&e_reg)[kPairsPerThread],
                                          int n, const DivK& divk, int E, int32_t* err_flag) {
    const int mine = pairs_of_thread(n);
#pragma unroll
    for (int i = 0; i < kPairsPerThread; ++i) {
        if (i >= mine) break;
        const int pl = threadIdx.x + i * kRouteThreads;
        const int e = e_reg[i];
        if (e < 0 || e >= E) continue;  // out-of-range experts: flagged elsewhere
        const int tl = divk(pl);
        const uint32_t bit = 1u << (tl & 31);
        const uint32_t old = atomicOr(&bitmap[e * kTileWords + (tl >> 5)], bit);
        if (old & bit) flag_error(err_flag, TK_DEVERR_DUP_EXPERT);
    }
}

__device__ __forceinline__ void tile_scatter(const uint32_t* bitmap, const int32_t* base,
                                             const int (&e_reg)[kPairsPerThread], int n,
                                             const DivK& divk, int64_t p0, int t0, int E,
                                             int32_t* slot_of, int32_t* token_of) {
    const int mine = pairs_of_thread(n);
#pragma unroll
    for (int i = 0; i < kPairsPerThread; ++i) {
        if (i >= mine) break;
        const int pl = threadIdx.x + i * kRouteThreads;
        const int e = e_reg[i];
        if (e < 0 || e >= E) {
            slot_of[p0 + pl] = -1;
            continue;
        }
        const int tl = divk(pl);
        const uint32_t* bm = bitmap + e * kTileWords;
        int rank = __popc(bm[tl >> 5] & ((1u << (tl & 31)) - 1u));
#pragma unroll
        for (int w = 0; w + 1 < kTileWords; ++w)
            if (w < (tl >> 5)) rank += __popc(bm[w]);
        const int32_t slot = base[e] + rank;
        slot_of[p0 + pl] = slot;
        token_of[slot] = t0 + tl;
    }
}

__device__ __forceinline__ void load_tile(const int32_t* topk_idx, int64_t p0, int n,
                                          int (&e_reg)[kPairsPerThread]) {
    const int mine = pairs_of_thread(n);
#pragma unroll
    for (int i = 0; i < kPairsPerThread; ++i) {
        if (i >= mine) break;
        e_reg[i] = topk_idx[p0 + threadIdx.x + i * kRouteThreads];
    }
}

// The loaded indices as local experts (window_expert), in place. Called once the loads have
// had the bitmap clearing and a barrier to arrive, so the mapping does not wait on them.
__device__ __forceinline__ void to_window(int (&e_reg)[kPairsPerThread], int n, int lo, int E) {
    const int mine = pairs_of_thread(n);
#pragma unroll
    for (int i = 0; i < kPairsPerThread; ++i) {
        if (i >= mine) break;
        e_reg[i] = window_expert(e_reg[i], lo, E);
    }
}

// Sums of expert rows of the count matrix over the tiles before `tile` and over all tiles,
// into before[e] and total[e]. P = 1, 2, 4 or 8 neighbouring threads share a row, each summing
// every P-th 16-byte vector (kRowBatch loads in flight), then they add their sums. Padding
// entries past the last tile are zero (written by the count kernel), so whole vectors are
// summed; only the vector that holds `tile` is masked.
__device__ __forceinline__ void row_sums(const int32_t* tile_counts, int stride, int E, int tile,
                                         int32_t* before, int32_t* total) {
    int P = 1;
    while (P < 8 && P * 2 * E <= kRouteThreads) P *= 2;
    const int part = threadIdx.x % P;
    const int n4 = stride / 4;
    const int rounds = (E * P + kRouteThreads - 1) / kRouteThreads;
    for (int r = 0; r < rounds; ++r) {
        const int e = (r * kRouteThreads + threadIdx.x) / P;
        int32_t b = 0, tot = 0;
        if (e < E) {
            const int4* r4 = reinterpret_cast<const int4*>(tile_counts + static_cast<int64_t>(e) * stride);
            for (int c0 = part; c0 < n4; c0 += P * kRowBatch) {
                int4 v[kRowBatch];
#pragma unroll
                for (int i = 0; i < kRowBatch; ++i) {
                    const int c4 = c0 + i * P;
                    v[i] = c4 < n4 ? r4[c4] : make_int4(0, 0, 0, 0);
                }
#pragma unroll
                for (int i = 0; i < kRowBatch; ++i) {
                    const int c = (c0 + i * P) * 4;
                    const int32_t s4 = v[i].x + v[i].y + v[i].z + v[i].w;
                    tot += s4;
                    if (c + 4 <= tile) {
                        b += s4;
                    } else if (c < tile) {
                        b += v[i].x + (c + 1 < tile ? v[i].y : 0) + (c + 2 < tile ? v[i].z : 0);
                    }
                }
            }
        }
        for (int off = 1; off < P; off <<= 1) {
            b += __shfl_xor_sync(kFullMask, b, off);
            tot += __shfl_xor_sync(kFullMask, tot, off);
        }
        if (e < E && part == 0) {
            before[e] = b;
            total[e] = tot;
        }
    }
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

// Single CTA. Each expert's row of tile_counts becomes exclusive per-tile prefixes (in place).
__global__ void __launch_bounds__(kScanThreads)
route_scan_kernel(int32_t* __restrict__ tile_counts, int tiles, int stride, int E, int align,
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
            int4* r4 = reinterpret_cast<int4*>(tile_counts + static_cast<int64_t>(e) * stride);
            const int n4 = (tiles + 3) / 4;
            int32_t run = 0;
            for (int c0 = 0; c0 < n4; c0 += kRowBatch) {
                int4 v[kRowBatch];
#pragma unroll
                for (int i = 0; i < kRowBatch; ++i) v[i] = c0 + i < n4 ? r4[c0 + i] : make_int4(0, 0, 0, 0);
#pragma unroll
                for (int i = 0; i < kRowBatch; ++i) {
                    if (c0 + i >= n4) break;
                    const int c = (c0 + i) * 4;
                    int4 o;
                    o.x = run; run += c + 0 < tiles ? v[i].x : 0;
                    o.y = run; run += c + 1 < tiles ? v[i].y : 0;
                    o.z = run; run += c + 2 < tiles ? v[i].z : 0;
                    o.w = run; run += c + 3 < tiles ? v[i].w : 0;
                    r4[c0 + i] = o;
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

// Many CTAs, for count matrices too large for the fused kernel: G = threads per expert row (a
// power of two <= 32, so a row's threads sit in one warp), kRouteThreads / G rows per CTA. A
// thread owns `seg` consecutive 16-byte vectors of its row: it sums them, the row's G threads
// exclusive-scan their sums with shuffles, and the thread rewrites its vectors as exclusive
// per-tile prefixes (in place; the padding past the last tile is zero, written by the count
// kernel, so whole vectors are summed). counts[e] gets the row total. The expert offsets are
// formed by the scatter kernel from counts.
struct RowScanShape {
    int G, seg, grid;
};
inline RowScanShape row_scan_shape(int stride, int E) {
    const int n4 = stride / 4;
    int G = 1;
    while (G < 32 && G * kRowBatch < n4) G *= 2;
    const int rows_per_cta = kRouteThreads / G;
    return {G, (n4 + G - 1) / G, (E + rows_per_cta - 1) / rows_per_cta};
}

__global__ void __launch_bounds__(kRouteThreads)
route_row_scan_kernel(int32_t* __restrict__ tile_counts, int stride, int E, int G, int seg,
                      int32_t* __restrict__ counts) {
    pdl_wait();
    const int rows_per_cta = kRouteThreads / G;
    const int e = blockIdx.x * rows_per_cta + static_cast<int>(threadIdx.x) / G;
    const int part = static_cast<int>(threadIdx.x) % G;
    const int n4 = stride / 4;
    const int v0 = part * seg;
    const int v1 = min(n4, v0 + seg);
    int4* r4 = reinterpret_cast<int4*>(tile_counts + static_cast<int64_t>(e < E ? e : 0) * stride);
    int32_t mine = 0;
    if (e < E) {
        for (int c0 = v0; c0 < v1; c0 += kRowBatch) {
            int4 v[kRowBatch];
#pragma unroll
            for (int i = 0; i < kRowBatch; ++i) v[i] = c0 + i < v1 ? r4[c0 + i] : make_int4(0, 0, 0, 0);
#pragma unroll
            for (int i = 0; i < kRowBatch; ++i) mine += v[i].x + v[i].y + v[i].z + v[i].w;
        }
    }
    // exclusive scan of the parts' sums over the row's G lanes (aligned groups within a warp)
    int32_t incl = mine;
    for (int off = 1; off < G; off <<= 1) {
        const int32_t u = __shfl_up_sync(kFullMask, incl, off, G);
        if (part >= off) incl += u;
    }
    const int32_t total = __shfl_sync(kFullMask, incl, G - 1, G);
    if (e >= E) return;
    int32_t run = incl - mine;
    for (int c0 = v0; c0 < v1; c0 += kRowBatch) {
        int4 v[kRowBatch];
#pragma unroll
        for (int i = 0; i < kRowBatch; ++i) v[i] = c0 + i < v1 ? r4[c0 + i] : make_int4(0, 0, 0, 0);
#pragma unroll
        for (int i = 0; i < kRowBatch; ++i) {
            if (c0 + i >= v1) break;
            int4 o;
            o.x = run; run += v[i].x;
            o.y = run; run += v[i].y;
            o.z = run; run += v[i].z;
            o.w = run; run += v[i].w;
            r4[c0 + i] = o;
        }
    }
    if (part == 0) counts[e] = total;
}

// One CTA per tile: forms the expert offsets from counts itself (CTA 0 also writes them out),
// then ranks and scatters the tile's pairs like the fused kernel.
template <bool kWindow>
__global__ void __launch_bounds__(kRouteThreads)
route_scatter_kernel(const int32_t* __restrict__ topk_idx, int T, int E, int k, int lo, int align,
                     const int32_t* __restrict__ tile_prefix, int stride,
                     const int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                     int32_t* __restrict__ slot_of, int32_t* __restrict__ token_of,
                     int32_t* err_flag) {
    extern __shared__ uint32_t smem[];
    uint32_t* bitmap = smem;                                          // [E][kTileWords]
    int32_t* base = reinterpret_cast<int32_t*>(smem + E * kTileWords);  // [E]
    int32_t* total = base + E;                                        // [E]
    __shared__ int32_t warp_tot[kRouteThreads / 32];
    pdl_wait();
    const int tile = blockIdx.x;
    const int t0 = tile * kTileTokens;
    const int64_t p0 = static_cast<int64_t>(t0) * k;
    const int n = (min(T, t0 + kTileTokens) - t0) * k;
    const DivK divk(k);
    int e_reg[kPairsPerThread];
    load_tile(topk_idx, p0, n, e_reg);
    for (int i = threadIdx.x; i < E * kTileWords; i += kRouteThreads) bitmap[i] = 0u;
    __syncthreads();
    if constexpr (kWindow) to_window(e_reg, n, lo, E);
    tile_mark(bitmap, e_reg, n, divk, E, err_flag);
    for (int e = threadIdx.x; e < E; e += kRouteThreads) total[e] = counts[e];
    __syncthreads();
    const int32_t R = cta_padded_scan(total, E, align, base, warp_tot);
    for (int e = threadIdx.x; e < E; e += kRouteThreads) {
        if (tile == 0) offsets[e] = base[e];
        base[e] += tile_prefix[static_cast<int64_t>(e) * stride + tile];
    }
    if (tile == 0 && threadIdx.x == 0) offsets[E] = R;
    __syncthreads();
    tile_scatter(bitmap, base, e_reg, n, divk, p0, t0, E, slot_of, token_of);
}

// The scan and scatter of a count matrix too large for the fused kernel (and of every matrix
// in the allocation-free entry point). With no tile the single-CTA scan writes the (zero)
// counts and offsets.
template <bool kWindow>
cudaError_t launch_scan_then_scatter(const int32_t* topk_idx, int T, int E, int k, int lo, int align,
                                     int32_t* tile_counts, int tiles, int stride, int32_t* counts,
                                     int32_t* offsets, int32_t* slot_of, int32_t* token_of,
                                     int32_t* err_flag, cudaStream_t s, const char** what) {
    if (tiles == 0) {
        *what = "route_scan_kernel";
        return launch_pdl(route_scan_kernel, dim3(1), dim3(scan_threads(E)), 0, s, tile_counts, tiles,
                          stride, E, align, counts, offsets);
    }
    const RowScanShape rs = row_scan_shape(stride, E);
    *what = "route_row_scan_kernel";
    cudaError_t err = launch_pdl(route_row_scan_kernel, dim3(rs.grid), dim3(kRouteThreads), 0, s,
                                 tile_counts, stride, E, rs.G, rs.seg, counts);
    if (err != cudaSuccess) return err;
    *what = "route_scatter_kernel";
    const size_t smem = static_cast<size_t>(E) * (kTileWords + 2) * sizeof(uint32_t);
    return launch_pdl(route_scatter_kernel<kWindow>, dim3(tiles), dim3(kRouteThreads), smem, s, topk_idx,
                      T, E, k, lo, align, static_cast<const int32_t*>(tile_counts), stride,
                      static_cast<const int32_t*>(counts), offsets, slot_of, token_of, err_flag);
}

// Scan and scatter in one kernel, for count matrices of at most kFusedMaxEntries entries: every
// CTA reads the whole (small) count matrix itself -- its own tile's prefix per expert, and every
// row's total for the offsets -- instead of waiting for a separate scan kernel. CTA 0 also
// writes counts[] and offsets[]. The slot arithmetic is the same as route_scan + route_scatter.
template <bool kWindow>
__global__ void __launch_bounds__(kRouteThreads, 1)
route_scan_scatter_kernel(const int32_t* __restrict__ topk_idx, int T, int E, int k, int lo, int align,
                          const int32_t* __restrict__ tile_counts, int stride,
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
    const int n = (min(T, t0 + kTileTokens) - t0) * k;
    const DivK divk(k);
    int e_reg[kPairsPerThread];
    load_tile(topk_idx, p0, n, e_reg);
    for (int i = threadIdx.x; i < E * kTileWords; i += kRouteThreads) bitmap[i] = 0u;
    __syncthreads();
    // the tile's bitmap does not depend on the scan: marked before the row sums' loads (issuing
    // those first, alongside the index loads, measured no faster)
    if constexpr (kWindow) to_window(e_reg, n, lo, E);
    tile_mark(bitmap, e_reg, n, divk, E, err_flag);
    // per expert: the count over the tiles before this one, and the row total
    row_sums(tile_counts, stride, E, tile, before, total);
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
    tile_scatter(bitmap, base, e_reg, n, divk, p0, t0, E, slot_of, token_of);
}

}  // namespace

size_t route_map_workspace_bytes_impl(int T, int E) {
    const int tiles = num_tiles(T) > 0 ? num_tiles(T) : 1;
    return static_cast<size_t>(row_stride(tiles)) * static_cast<size_t>(E) * sizeof(int32_t);
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

namespace tk {
namespace {

// The route map of the experts [lo, lo + E) of e_total (the whole map: lo = 0, E = e_total).
template <bool kWindow>
tk_status route_map_launch(const char* fn, const int32_t* topk_idx, int T, int e_total, int k, int lo,
                         int E, int align, int32_t* counts, int32_t* offsets, int32_t* slot_of,
                         int32_t* token_of, void* workspace, size_t workspace_bytes,
                         int32_t* err_flag, void* stream) {
    if (T < 0) return fail_arg("%s: T=%d must be >= 0", fn, T);
    if (E < 1 || E > TK_MAX_EXPERTS) return fail_arg("%s: E=%d outside [1, %d]", fn, E, TK_MAX_EXPERTS);
    if (lo < 0 || e_total < E || lo > e_total - E)
        return fail_arg("%s: the window [%d, %d + %d) is not inside [0, %d)", fn, lo, lo, E, e_total);
    if (k < 1 || k > TK_MAX_TOPK) return fail_arg("%s: k=%d outside [1, %d]", fn, k, TK_MAX_TOPK);
    if (align < 1 || align > 4096) return fail_arg("%s: align=%d outside [1, 4096]", fn, align);
    const int64_t rmax = tk_max_rows(T, E, k, align);
    if (rmax > INT32_MAX) return fail_arg("%s: T*k + E*(align-1) = %lld exceeds int32", fn, (long long)rmax);
    if (counts == nullptr || offsets == nullptr || workspace == nullptr)
        return fail_arg("%s: counts, offsets and workspace must not be NULL", fn);
    if (T > 0 && (topk_idx == nullptr || slot_of == nullptr))
        return fail_arg("%s: topk_idx and slot_of must not be NULL", fn);
    if (rmax > 0 && token_of == nullptr) return fail_arg("%s: token_of must not be NULL", fn);
    const size_t need = route_map_workspace_bytes_impl(T, E);
    if (workspace_bytes < need)
        return fail_arg("%s: workspace holds %zu bytes, needs %zu", fn, workspace_bytes, need);
    if (reinterpret_cast<uintptr_t>(workspace) % 16 != 0)
        return fail_arg("%s: workspace must be 16-byte aligned", fn);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t* tile_counts = static_cast<int32_t*>(workspace);
    const int tiles = num_tiles(T);
    const int stride = row_stride(tiles);
    const int count_grid = tiles > 0 ? tiles : 1;
    cudaError_t err = launch_pdl(route_count_kernel<kWindow>, dim3(count_grid), dim3(kRouteThreads),
                                 static_cast<size_t>(E) * sizeof(int32_t), s, topk_idx, T, E, k, lo,
                                 e_total, tile_counts, stride, token_of, rmax, err_flag);
    if (err != cudaSuccess) return check_launch(err, "route_count_kernel");
    if (tiles > 0 && static_cast<int64_t>(stride) * E <= kFusedMaxEntries) {
        const size_t smem = static_cast<size_t>(E) * (kTileWords + 3) * sizeof(uint32_t);
        err = launch_pdl(route_scan_scatter_kernel<kWindow>, dim3(tiles), dim3(kRouteThreads), smem, s,
                         topk_idx, T, E, k, lo, align, static_cast<const int32_t*>(tile_counts),
                         stride, counts, offsets, slot_of, token_of, err_flag);
        return check_launch(err, "route_scan_scatter_kernel");
    }
    const char* what = "";
    err = launch_scan_then_scatter<kWindow>(topk_idx, T, E, k, lo, align, tile_counts, tiles, stride,
                                            counts, offsets, slot_of, token_of, err_flag, s, &what);
    return check_launch(err, what);
}

tk_status route_map_impl(const char* fn, const int32_t* topk_idx, int T, int e_total, int k, int lo,
                         int E, int align, int32_t* counts, int32_t* offsets, int32_t* slot_of,
                         int32_t* token_of, void* workspace, size_t workspace_bytes,
                         int32_t* err_flag, void* stream) {
    if (lo == 0 && E == e_total)
        return route_map_launch<false>(fn, topk_idx, T, e_total, k, lo, E, align, counts, offsets,
                                       slot_of, token_of, workspace, workspace_bytes, err_flag, stream);
    return route_map_launch<true>(fn, topk_idx, T, e_total, k, lo, E, align, counts, offsets, slot_of,
                                  token_of, workspace, workspace_bytes, err_flag, stream);
}

}  // namespace
}  // namespace tk

extern "C" tk_status tk_route_map(const int32_t* topk_idx, int T, int E, int k, int align,
                                  int32_t* counts, int32_t* offsets, int32_t* slot_of,
                                  int32_t* token_of, void* workspace, size_t workspace_bytes,
                                  int32_t* err_flag, void* stream) {
    return tk::route_map_impl("tk_route_map", topk_idx, T, E, k, 0, E, align, counts, offsets,
                              slot_of, token_of, workspace, workspace_bytes, err_flag, stream);
}

extern "C" tk_status tk_route_map_window(const int32_t* topk_idx, int T, int E_total, int k,
                                         int expert_lo, int E, int align, int32_t* counts,
                                         int32_t* offsets, int32_t* slot_of, int32_t* token_of,
                                         void* workspace, size_t workspace_bytes, int32_t* err_flag,
                                         void* stream) {
    return tk::route_map_impl("tk_route_map_window", topk_idx, T, E_total, k, expert_lo, E, align,
                              counts, offsets, slot_of, token_of, workspace, workspace_bytes,
                              err_flag, stream);
}

// ------------------------------------------------------------------------------------------
// Allocation-free variant of tk_route_map.
//
// Some callers cannot hand the library a workspace: a serving engine or plugin host that owns
// every byte of device memory and passes a component only its input and output buffers, or a
// latency-critical loop where a cudaMalloc (which can synchronise the device) is not allowed.
// For them the tile-count matrix lives in a fixed array compiled into this library. Every GPU
// that loads the library reserves it (2 MiB) until the process exits.
//
// The array's name is only a host-side stand-in in host code; its device address is looked up
// with cudaGetSymbolAddress once per device (with that device current) on the first call on
// that device, and cached for the life of the process (a device reset after that first call is
// not supported: the cached address would be stale). The kernels write every entry they later read, so nothing in the
// array has to start at zero. All calls on one device share the array: calls that can overlap
// on the GPU (other streams, other host threads) race on it and must be serialised by the
// caller.
// ------------------------------------------------------------------------------------------
#include <mutex>

namespace {
constexpr size_t kStaticScratchInts = 512 * 1024;  // 2 MiB of int32 tile counts
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
                        "buffer holds %zu (E times the tiles of %d tokens rounded up to a multiple "
                        "of 4, at most %zu tiles here); use tk_route_map with a caller workspace",
                        T, E, need, kStaticScratchInts, kTileTokens,
                        kStaticScratchInts / static_cast<size_t>(E) / 4 * 4);
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
    const int stride = row_stride(tiles);
    const int count_grid = tiles > 0 ? tiles : 1;
    cudaError_t err = launch_pdl(route_count_kernel<false>, dim3(count_grid), dim3(kRouteThreads),
                                 static_cast<size_t>(E) * sizeof(int32_t), s, topk_idx, T, E, k, 0,
                                 E, tile_counts, stride, token_of, rmax, err_flag);
    if (err != cudaSuccess) return check_launch(err, "route_count_kernel");
    const char* what = "";
    err = launch_scan_then_scatter<false>(topk_idx, T, E, k, 0, align, tile_counts, tiles, stride,
                                          counts, offsets, slot_of, token_of, err_flag, s, &what);
    return check_launch(err, what);
}
