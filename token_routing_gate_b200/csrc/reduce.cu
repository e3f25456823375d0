// Fused reduce / combine: out[t] = bf16( sum_j w[t,j] * y[slot_of[t,j]] ), fp32 accumulation
// in slot order j = 0..k-1, one fmaf per term (147227.xyz "刚刚！DeepSeek开源高性能GPU算子库
// TileKernels", section "moe/": fused reduce; BF16 combine in 機器之心 "性能表現").
//
// Pure bandwidth: per token, k scattered 2H-byte rows read and one 2H-byte row written. The
// loads go through the bulk-copy (TMA) engine so that the bytes in flight do not depend on
// registers: a unit of work is (token t, 1024-channel chunk c). Each CTA is warp-specialised:
//   warp 0      producer: lanes j < k read slot j and weight j of the unit, and the unit's valid
//               rows (masked pairs and absent rows skipped) get consecutive 2 KB places in a
//               shared-memory byte ring, in slot order; their weights go to the unit's entry
//               (one of 16), and one 1-D bulk load per valid row chunk completes on the entry's
//               "full" mbarrier (transaction count = bytes issued).
//   warps 1..4  consumers: wait "full", each thread combines one 8-channel vector of the unit
//               across its valid row chunks (16-byte shared loads, fmaf in slot order), writes
//               16 bytes of bf16 output, then the warp arrives on the entry's "empty" mbarrier.
// The ring holds 32 KB, so a unit whose k = 8 rows are all valid takes 16 KB (two in flight, as a
// fixed two-stage ring would), while a unit with few valid rows -- a masked route map, an
// expert-parallel destination's rows -- takes only what it loads and up to 16 units are in
// flight. Six CTAs fit on an SM; the dense reduce keeps five (160 KB of loads in flight per
// SM): after a write-heavy kernel (expand in the routing step) five took 171 us at T=8192 where
// six took 183, while after a read-heavy one six were 4 us faster. A measured sweep on B200
// (ring size, chunk width, consumer warps) put this shape at the HBM copy roofline; deeper
// rings with fewer CTAs per SM were up to 30% slower. The grid is persistent (SM count x CTAs
// per SM) and CTAs stride over units.
// The row loads carry an explicit L2 evict-normal policy. Measured on B200 at T=8192, H=7168,
// k=8: with it the reduce after dispatch and the reduce run back to back were both faster than
// with no policy operand (forward step 366.8 -> 364.9 us; back-to-back reduce 155.5 -> 152.9 us).
// Evict-first won the forward step (361.7 us) but cost 16 us back to back, so it is not used.
// Every wait is bounded (1 s); a timeout flags TK_DEVERR_TIMEOUT and ends the CTA's loop.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <type_traits>
#include <stdint.h>

#include "tk_device.cuh"

namespace tk {
namespace {

#ifndef TK_REDUCE_CONSUMER_WARPS
#define TK_REDUCE_CONSUMER_WARPS 4
#endif
#ifndef TK_REDUCE_VECS_PER_THREAD
#define TK_REDUCE_VECS_PER_THREAD 1
#endif
#ifndef TK_REDUCE_LOAD_POLICY   // L2 policy of the row loads: 0 none, 1 evict-normal, 2 evict-first
#define TK_REDUCE_LOAD_POLICY 1
#endif
#ifndef TK_REDUCE_STAGE_KB
#define TK_REDUCE_STAGE_KB 32
#endif

#ifndef TK_REDUCE_DENSE_CTAS_PER_SM  // resident CTAs per SM of the dense reduce (0: as many as fit)
#define TK_REDUCE_DENSE_CTAS_PER_SM 5
#endif
#ifndef TK_REDUCE_MASKED_VECS_PER_THREAD
#define TK_REDUCE_MASKED_VECS_PER_THREAD 2
#endif

constexpr int kConsumerWarps = TK_REDUCE_CONSUMER_WARPS;
// 8-channel vectors per consumer thread and unit: the dense reduce (every pair valid) and the
// masked form (tk_reduce_masked: most pairs -1, so a unit's few valid rows are small and wider
// units carry the per-unit work over more bytes)
constexpr int kVecsDense = TK_REDUCE_VECS_PER_THREAD;
constexpr int kVecsMasked = TK_REDUCE_MASKED_VECS_PER_THREAD;
constexpr int kRedThreads = 32 * (1 + kConsumerWarps);
constexpr int kStageBudget = TK_REDUCE_STAGE_KB * 1024;    // shared bytes of row data per CTA

// Channels of one unit and bf16 bytes of one of its row chunks, for kV vectors per thread.
template <int kV>
struct UnitShape {
    static constexpr int ch = 8 * 32 * kConsumerWarps * kV;
    static constexpr int bytes = ch * 2;
};
constexpr int kRingEntries = 16;                           // units in flight at most

// One unit's entry in the ring: its valid rows sit back to back at `off`, in slot order, and
// w[i] is the weight of the i-th of them.
struct EntryMeta {
    float w[TK_MAX_TOPK];
    int32_t n;
    uint32_t off;
};

__device__ __forceinline__ float lo_bf16(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float hi_bf16(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const uint32_t l = static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(lo)));
    const uint32_t h = static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(hi)));
    return l | (h << 16);
}

// Bytes of the row ring: the budget, and at least one unit with all k rows valid.
int ring_bytes_for(int k, int chunk_bytes) {
    return k * chunk_bytes > kStageBudget ? k * chunk_bytes : kStageBudget;
}

size_t smem_bytes(int ring) {
    return static_cast<size_t>(ring) + kRingEntries * sizeof(EntryMeta) +
           2 * kRingEntries * sizeof(uint64_t);
}

// Where the j-th row of token t comes from. fetch() reads the pair's index (one unit ahead of
// use); lane_ctx() caches what lane j needs to resolve it; resolve() gives the row's address,
// or nullptr for a row that does not exist (flagging an index that is not a valid one).
//
// SlotRows (the reduce): row j of token t is y[slot_of[t*k + j]]; slot -1 is a masked pair.
struct SlotRows {
    const uint8_t* y;
    int64_t y_rows;
    const int32_t* slot_of;
    struct Lane {};
    __device__ __forceinline__ Lane lane_ctx(int) const { return {}; }
    __device__ __forceinline__ int64_t fetch(int64_t t, int j, int k) const { return slot_of[t * k + j]; }
    __device__ __forceinline__ const uint8_t* resolve(const Lane&, int64_t raw, int64_t row_bytes,
                                                      int32_t* err) const {
        if (raw >= 0 && raw < y_rows) return y + raw * row_bytes;
        if (raw != -1) flag_error(err, TK_DEVERR_SLOT_RANGE);
        return nullptr;
    }
};

// RankRows (the expert-parallel combine): "row j" of token t is the partial row rank j holds
// for it, at base[j] + (dest_slot[t*G + j] - send_offsets[j]) in rank j's partial buffer
// (dest_slot -1: the token did not go to rank j).
struct RankRows {
    const uint8_t* part[TK_MAX_EP_RANKS];
    int64_t base[TK_MAX_EP_RANKS];
    int64_t rows[TK_MAX_EP_RANKS];
    const int32_t* dest_slot;
    const int32_t* send_offsets;
    int G;
    struct Lane {
        const uint8_t* part;
        int64_t base, rows;
        int32_t off;
    };
    __device__ __forceinline__ Lane lane_ctx(int j) const {
        Lane L{nullptr, 0, 0, 0};
        if (j < G) {
            L.part = part[j];
            L.base = base[j];
            L.rows = rows[j];
            L.off = send_offsets[j];
        }
        return L;
    }
    __device__ __forceinline__ int64_t fetch(int64_t t, int j, int) const { return dest_slot[t * G + j]; }
    __device__ __forceinline__ const uint8_t* resolve(const Lane& L, int64_t raw, int64_t row_bytes,
                                                      int32_t* err) const {
        if (raw == -1) return nullptr;
        const int64_t row = L.base + (raw - L.off);
        if (raw < 0 || raw < L.off || row >= L.rows) {
            flag_error(err, TK_DEVERR_SLOT_RANGE);
            return nullptr;
        }
        return L.part + row * row_bytes;
    }
};

// kStep: step each unit's (token, chunk) and ring offset by O(1) updates instead of 64-bit
// division and modulo (the tk_reduce_masked form; see the entry points).
template <class Rows, bool kStep, int kVecs>
__global__ void __launch_bounds__(kRedThreads)
reduce_kernel(const __grid_constant__ Rows rows, const float* __restrict__ w, int T, int k, int H,
              int ring, uint8_t* __restrict__ out, int32_t* err_flag) {
    constexpr int kChunkCh = UnitShape<kVecs>::ch;
    constexpr int kChunkBytes = UnitShape<kVecs>::bytes;
    extern __shared__ __align__(128) uint8_t sm[];
    uint8_t* data = sm;                                                    // [ring] row bytes
    EntryMeta* meta = reinterpret_cast<EntryMeta*>(sm + ring);             // [kRingEntries]
    uint64_t* full = reinterpret_cast<uint64_t*>(meta + kRingEntries);
    uint64_t* empty = full + kRingEntries;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int e = 0; e < kRingEntries; ++e) {
            mbar_init(&full[e], 1);
            mbar_init(&empty[e], kConsumerWarps);
        }
        fence_barrier_init();
    }
    __syncthreads();
    pdl_wait();

    const int chunks = (H + kChunkCh - 1) / kChunkCh;
    const int64_t units = static_cast<int64_t>(T) * chunks;
    const int64_t row_bytes = static_cast<int64_t>(H) * 2;
    // kStep: a CTA's units are blockIdx.x, blockIdx.x + G, ... (G = gridDim.x); unit u is token
    // u / chunks, chunk u % chunks, both stepped by (G / chunks, G % chunks).
    const int64_t step_t = static_cast<int64_t>(gridDim.x) / chunks;
    const int step_c = static_cast<int>(static_cast<int64_t>(gridDim.x) - step_t * chunks);
    const int64_t t_first = static_cast<int64_t>(blockIdx.x) / chunks;
    const int c_first = static_cast<int>(static_cast<int64_t>(blockIdx.x) - t_first * chunks);

    if (warp == 0) {
        // ---------------- producer. Unit `it` takes entry it % kRingEntries and the next
        // (valid rows) * 2 KB of the ring (wrapping to its start when the rest of the ring is
        // too short). Before reusing space or an entry it waits, oldest first, for the
        // consumers to release earlier units; lane e remembers where entry e's bytes end.
        // The slots and weights of the next unit are fetched while the current one waits.
        const typename Rows::Lane lctx = rows.lane_ctx(lane);
        int64_t u = blockIdx.x;
        int64_t nxt_sl = -1;
        float nxt_w = 1.0f;
        if (lane < k && u < units) {
            const int64_t t = u / chunks;
            nxt_sl = rows.fetch(t, lane, k);
            if (w != nullptr) nxt_w = w[t * k + lane];
        }
        uint64_t head = 0, tail = 0;   // ring bytes handed out / released so far
        uint64_t my_end = 0;           // lane e: end of entry e's bytes
        int rel = 0;                   // units known to be released
        int64_t st_tn = t_first + step_t;   // kStep: token of the next unit, this unit's chunk,
        int st_cn = c_first + step_c;       // the next unit's chunk, the ring offset
        if (st_cn >= chunks) {
            st_cn -= chunks;
            ++st_tn;
        }
        int st_c = c_first;
        uint32_t ring_off = 0;
        for (int it = 0; u < units; u += gridDim.x, ++it) {
            int ch0;
            if constexpr (kStep) {
                ch0 = st_c * kChunkCh;
            } else {
                const int64_t t = u / chunks;
                ch0 = static_cast<int>(u - t * chunks) * kChunkCh;
            }
            const uint32_t bytes = static_cast<uint32_t>(min(kChunkCh, H - ch0)) * 2u;
            const int64_t raw = nxt_sl;
            const float wl = nxt_w;
            const int64_t un = u + gridDim.x;
            if (lane < k && un < units) {
                int64_t tn;
                if constexpr (kStep) tn = st_tn;
                else tn = un / chunks;
                nxt_sl = rows.fetch(tn, lane, k);
                if (w != nullptr) nxt_w = w[tn * k + lane];
            }
            if constexpr (kStep) {
                st_c = st_cn;
                st_tn += step_t;
                st_cn += step_c;
                if (st_cn >= chunks) {
                    st_cn -= chunks;
                    ++st_tn;
                }
            }
            const uint8_t* rowp = lane < k ? rows.resolve(lctx, raw, row_bytes, err_flag) : nullptr;
            const unsigned vmask = __ballot_sync(kFullMask, rowp != nullptr);
            const int nvalid = __popc(vmask);
            const int pos = __popc(vmask & ((1u << lane) - 1u));   // this row's place among them
            uint64_t h = head;
            uint32_t off;
            if constexpr (kStep) off = ring_off;
            else off = static_cast<uint32_t>(h % static_cast<uint64_t>(ring));
            const uint32_t need = static_cast<uint32_t>(nvalid) * kChunkBytes;
            if (off + need > static_cast<uint32_t>(ring)) {   // no room before the end: wrap
                h += static_cast<uint32_t>(ring) - off;
                off = 0;
            }
            const uint64_t h_end = h + need;
            int ok = 1;
            // Space: the bytes from the oldest unreleased unit to this unit's end must fit in the
            // ring. Once every earlier unit is released nothing is live, and the unit fits even
            // when the gap skipped by wrapping makes that span longer than the ring (a unit of
            // more than half the ring after a smaller one would otherwise wait forever).
            while (it - rel >= kRingEntries || (rel < it && h_end - tail > static_cast<uint64_t>(ring))) {
                const int e = rel % kRingEntries;
                if (lane == 0) ok = mbar_wait_bounded(&empty[e], static_cast<uint32_t>(rel / kRingEntries) & 1u) ? 1 : 0;
                ok = __shfl_sync(kFullMask, ok, 0);
                if (!ok) break;
                tail = __shfl_sync(kFullMask, my_end, e);
                ++rel;
            }
            if (!ok) {
                if (lane == 0) flag_error(err_flag, TK_DEVERR_TIMEOUT);
                break;
            }
            head = h_end;
            if constexpr (kStep) ring_off = off + need;
            const int e = it % kRingEntries;
            if (lane == e) my_end = h_end;
            if (rowp != nullptr) meta[e].w[pos] = wl;
            if (lane == 0) {
                meta[e].n = nvalid;
                meta[e].off = off;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive_expect_tx(&full[e], static_cast<uint32_t>(nvalid) * bytes);
            __syncwarp();
            if (rowp != nullptr) {
                uint8_t* dst = data + off + static_cast<uint32_t>(pos) * kChunkBytes;
                const uint8_t* src = rowp + static_cast<int64_t>(ch0) * 2;
                if (TK_REDUCE_LOAD_POLICY != 0) bulk_load_hint(dst, src, bytes, &full[e], l2_policy(TK_REDUCE_LOAD_POLICY));
                else bulk_load(dst, src, bytes, &full[e]);
            }
        }
    } else {
        // ---------------- consumers
        const int ct = threadIdx.x - 32;  // 0 .. 32*kConsumerWarps-1
        int it = 0;
        int64_t st_t = t_first;   // kStep: this unit's token and chunk
        int st_c = c_first;
        for (int64_t u = blockIdx.x; u < units; u += gridDim.x, ++it) {
            const int e = it % kRingEntries;
            if (!mbar_wait_bounded(&full[e], static_cast<uint32_t>(it / kRingEntries) & 1u)) {
                flag_error(err_flag, TK_DEVERR_TIMEOUT);
                break;
            }
            int64_t t;
            int ch0;
            if constexpr (kStep) {
                t = st_t;
                ch0 = st_c * kChunkCh;
                st_t += step_t;
                st_c += step_c;
                if (st_c >= chunks) {
                    st_c -= chunks;
                    ++st_t;
                }
            } else {
                t = u / chunks;
                ch0 = static_cast<int>(u - t * chunks) * kChunkCh;
            }
            const int chn = min(kChunkCh, H - ch0);
            const int n = meta[e].n;
            const uint8_t* rows_at = data + meta[e].off;
#pragma unroll
            for (int q = 0; q < kVecs; ++q) {
                const int vec = ct + q * 32 * kConsumerWarps;   // 8-channel vector within the unit
                if (vec * 8 >= chn) break;
                float acc[8];
#pragma unroll
                for (int c = 0; c < 8; ++c) acc[c] = 0.0f;
                const uint8_t* base = rows_at + vec * 16;
                for (int i = 0; i < n; ++i) {   // the valid rows in slot order
                    const float wj = meta[e].w[i];
                    const uint4 q4 = *reinterpret_cast<const uint4*>(base + i * kChunkBytes);
                    acc[0] = __fmaf_rn(wj, lo_bf16(q4.x), acc[0]);
                    acc[1] = __fmaf_rn(wj, hi_bf16(q4.x), acc[1]);
                    acc[2] = __fmaf_rn(wj, lo_bf16(q4.y), acc[2]);
                    acc[3] = __fmaf_rn(wj, hi_bf16(q4.y), acc[3]);
                    acc[4] = __fmaf_rn(wj, lo_bf16(q4.z), acc[4]);
                    acc[5] = __fmaf_rn(wj, hi_bf16(q4.z), acc[5]);
                    acc[6] = __fmaf_rn(wj, lo_bf16(q4.w), acc[6]);
                    acc[7] = __fmaf_rn(wj, hi_bf16(q4.w), acc[7]);
                }
                uint4 o;
                o.x = pack_bf16x2(acc[0], acc[1]);
                o.y = pack_bf16x2(acc[2], acc[3]);
                o.z = pack_bf16x2(acc[4], acc[5]);
                o.w = pack_bf16x2(acc[6], acc[7]);
                st_v4(out + t * row_bytes + static_cast<int64_t>(ch0 + vec * 8) * 2, o);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[e]);
        }
    }
}

struct LaunchShape {
    int grid_cap = 0;   // SMs x resident CTAs for the current ring size
    int ring = 0;       // ring bytes
};

// Launch shape for k on the current device, worked out once per row source (the kernel's
// shared-memory limit is raised to the largest size any k needs).
template <class Rows, bool kStep, int kVecs>
cudaError_t launch_shape(int k, LaunchShape& out) {
    static LaunchShape shapes[kMaxDevices][TK_MAX_TOPK + 1];
    static std::atomic<bool> ready[kMaxDevices][TK_MAX_TOPK + 1];
    static int configured_smem[kMaxDevices];
    const int dev = current_device();
    if (ready[dev][k].load(std::memory_order_acquire)) {
        out = shapes[dev][k];
        return cudaSuccess;
    }
    std::lock_guard<std::mutex> lock(setup_mutex());
    if (!ready[dev][k].load(std::memory_order_relaxed)) {
        const int ring = ring_bytes_for(k, UnitShape<kVecs>::bytes);
        const size_t smem = smem_bytes(ring);
        cudaError_t err = cudaSuccess;
        if (static_cast<int>(smem) > configured_smem[dev]) {
            err = cudaFuncSetAttribute(reduce_kernel<Rows, kStep, kVecs>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
            if (err != cudaSuccess) return err;
            configured_smem[dev] = static_cast<int>(smem);
        }
        int per_sm = 0;
        err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, reduce_kernel<Rows, kStep, kVecs>, kRedThreads, smem);
        if (err != cudaSuccess) return err;
        if constexpr (std::is_same<Rows, SlotRows>::value && !kStep) {
            if (TK_REDUCE_DENSE_CTAS_PER_SM > 0 && per_sm > TK_REDUCE_DENSE_CTAS_PER_SM)
                per_sm = TK_REDUCE_DENSE_CTAS_PER_SM;
        }
        shapes[dev][k].grid_cap = num_sms() * (per_sm < 1 ? 1 : per_sm);
        shapes[dev][k].ring = ring;
        ready[dev][k].store(true, std::memory_order_release);
    }
    out = shapes[dev][k];
    return cudaSuccess;
}

template <class Rows, bool kStep = false, int kVecs = kVecsDense>
cudaError_t launch_reduce(const Rows& rows, const float* w, int T, int k, int H, void* out,
                          int32_t* err_flag, void* stream, const char** what) {
    *what = "reduce_kernel setup";
    LaunchShape shape;
    const cudaError_t e = launch_shape<Rows, kStep, kVecs>(k, shape);
    if (e != cudaSuccess) return e;
    *what = "reduce_kernel";
    constexpr int kChunkCh = UnitShape<kVecs>::ch;
    const int64_t chunks = (H + kChunkCh - 1) / kChunkCh;
    const int64_t units = static_cast<int64_t>(T) * chunks;
    const int grid = static_cast<int>(units < shape.grid_cap ? units : shape.grid_cap);
    return launch_pdl(reduce_kernel<Rows, kStep, kVecs>, dim3(grid), dim3(kRedThreads), smem_bytes(shape.ring),
                      static_cast<cudaStream_t>(stream), rows, w, T, k, H, shape.ring,
                      static_cast<uint8_t*>(out), err_flag);
}

}  // namespace
}  // namespace tk

namespace tk {
namespace {

template <bool kStep>
tk_status reduce_entry(const char* name, const void* y, int64_t y_rows, const int32_t* slot_of,
                       const float* w, int T, int k, int H, void* out, int32_t* err_flag,
                       void* stream) {
    if (T < 0) return fail_arg("%s: T=%d must be >= 0", name, T);
    if (k < 1 || k > TK_MAX_TOPK) return fail_arg("%s: k=%d outside [1, %d]", name, k, TK_MAX_TOPK);
    if (H < 8 || H % 8 != 0) return fail_arg("%s: H=%d must be a positive multiple of 8", name, H);
    if (y_rows < 0) return fail_arg("%s: y_rows=%lld must be >= 0", name, (long long)y_rows);
    if (T == 0) return TK_OK;
    if (slot_of == nullptr || out == nullptr || (y == nullptr && y_rows > 0))
        return fail_arg("%s: y, slot_of and out must not be NULL", name);
    if (reinterpret_cast<uintptr_t>(y) % 16 != 0 || reinterpret_cast<uintptr_t>(out) % 16 != 0)
        return fail_arg("%s: y and out must be 16-byte aligned", name);
    const SlotRows rows{static_cast<const uint8_t*>(y), y_rows, slot_of};
    const char* what = "";
    const cudaError_t err = launch_reduce<SlotRows, kStep, kStep ? kVecsMasked : kVecsDense>(
        rows, w, T, k, H, out, err_flag, stream, &what);
    return check_launch(err, what);
}

}  // namespace
}  // namespace tk

extern "C" tk_status tk_reduce(const void* y, int64_t y_rows, const int32_t* slot_of, const float* w,
                               int T, int k, int H, void* out, int32_t* err_flag, void* stream) {
    return tk::reduce_entry<false>("tk_reduce", y, y_rows, slot_of, w, T, k, H, out, err_flag, stream);
}

extern "C" tk_status tk_reduce_masked(const void* y, int64_t y_rows, const int32_t* slot_of,
                                      const float* w, int T, int k, int H, void* out,
                                      int32_t* err_flag, void* stream) {
    return tk::reduce_entry<true>("tk_reduce_masked", y, y_rows, slot_of, w, T, k, H, out, err_flag,
                                  stream);
}

extern "C" tk_status tk_ep_combine(const void* const* partial, const int64_t* base_row,
                                   const int64_t* rows, const int32_t* dest_slot,
                                   const int32_t* send_offsets, int T, int G, int H, void* out,
                                   int32_t* err_flag, void* stream) {
    using namespace tk;
    if (T < 0) return fail_arg("tk_ep_combine: T=%d must be >= 0", T);
    if (G < 1 || G > TK_MAX_EP_RANKS) return fail_arg("tk_ep_combine: G=%d outside [1, %d]", G, TK_MAX_EP_RANKS);
    if (H < 8 || H % 8 != 0) return fail_arg("tk_ep_combine: H=%d must be a positive multiple of 8", H);
    if (T == 0) return TK_OK;
    if (partial == nullptr || base_row == nullptr || rows == nullptr || dest_slot == nullptr ||
        send_offsets == nullptr || out == nullptr)
        return fail_arg("tk_ep_combine: no pointer argument may be NULL");
    if (reinterpret_cast<uintptr_t>(out) % 16 != 0) return fail_arg("tk_ep_combine: out must be 16-byte aligned");
    RankRows rr{};
    for (int d = 0; d < G; ++d) {
        if (rows[d] < 0 || base_row[d] < 0) return fail_arg("tk_ep_combine: rank %d has negative rows or base", d);
        if (rows[d] > 0 && (partial[d] == nullptr || reinterpret_cast<uintptr_t>(partial[d]) % 16 != 0))
            return fail_arg("tk_ep_combine: partial[%d] must be a 16-byte aligned buffer", d);
        rr.part[d] = static_cast<const uint8_t*>(partial[d]);
        rr.base[d] = base_row[d];
        rr.rows[d] = rows[d];
    }
    rr.dest_slot = dest_slot;
    rr.send_offsets = send_offsets;
    rr.G = G;
    const char* what = "";
    const cudaError_t err = launch_reduce(rr, nullptr, T, G, H, out, err_flag, stream, &what);
    return check_launch(err, what);
}
