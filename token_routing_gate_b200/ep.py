"""Host side of expert-parallel dispatch and combine over G ranks.

Sources: 147227.xyz "刚刚！DeepSeek开源高性能GPU算子库TileKernels" (its DeepEP paragraph: an
expert-parallel all-to-all over NVLink with native FP8 dispatch) and 機器之心 "剛剛，DeepSeek開始
頻繁更新：Tile Kernels、DeepEP V2", section "性能表現" (FP8 dispatch, BF16 combine). The layout and
the arithmetic are stated with the tk_ep_* entry points in include/tk_route.h.

One step, for every rank s at once:
  1. tk_ep_layout: where each of s's tokens goes (per destination rank: count, position).
  2. The G x G send counts are exchanged (an all-gather of G ints per rank); rank d's receive
     buffer holds source 0's rows first, then source 1's, ..., so source s writes at
     base[s][d] = sum of what lower ranks send to d (recv_bases).
  3. tk_ep_dispatch: s writes its rows (bf16 or E4M3) and local choices into every destination's
     buffers -- peer memory on several GPUs.
  4. After a cross-rank barrier, each destination routes its received rows over its own E/G
     experts (tk_route_map), runs them, and combines its experts' outputs per received row into a
     bf16 partial (tk_reduce).
  5. After a second barrier, tk_ep_combine: s sums the partials of each token over its
     destinations in rank order.
No kernel waits on another rank; the barriers are collectives between the launches.

Two drivers: VirtualRanks runs G ranks in one process on one device, one after another (the
single-GPU check of the path); EpGroup runs one rank per process with the receive buffers in
torch symmetric memory, whose peer addresses the kernels write and read directly.
"""
import torch
import torch.distributed as tdist

from . import tk


def recv_bases(count_matrix):
    """count_matrix [G, G] (row s: rows rank s sends to each rank) -> (base [G, G], recv_rows [G]),
    base[s][d] = sum_{s' < s} count_matrix[s'][d], recv_rows[d] = column sums. int64, on the CPU."""
    cm = torch.as_tensor(count_matrix).to(device="cpu", dtype=torch.int64)
    if cm.dim() != 2 or cm.shape[0] != cm.shape[1]:
        raise ValueError("count matrix must be G x G")
    if (cm < 0).any():
        raise ValueError("negative send count")
    return torch.cumsum(cm, dim=0) - cm, cm.sum(dim=0)


def exchange_counts(send_counts, group=None):
    """Every rank's send counts, stacked: [G, G] with row s from rank s (all-gather of G ints)."""
    G = tdist.get_world_size(group)
    parts = [torch.empty_like(send_counts) for _ in range(G)]
    tdist.all_gather(parts, send_counts.contiguous(), group=group)
    return torch.stack(parts)


def capacity_rows(max_tokens, G):
    """Rows a receive buffer needs in the worst case: every token of every rank."""
    return int(max_tokens) * int(G)


class RankBuffers:
    """One rank's receive buffers (rows, E4M3 scales, local choices and weights) and its partial
    rows, all with `rows` rows. `alloc(shape, dtype)` supplies the memory."""

    def __init__(self, rows, H, k, out_dtype, device, alloc=None):
        if alloc is None:
            def alloc(shape, dtype):
                return torch.empty(shape, dtype=dtype, device=device)
        self.rows, self.H, self.k, self.out_dtype = rows, H, k, out_dtype
        self.x = alloc((rows, H), torch.uint8 if out_dtype == "fp8" else torch.bfloat16)
        self.scale = alloc((rows, H // 128), torch.float32) if out_dtype == "fp8" else None
        self.idx = alloc((rows, k), torch.int32)
        self.w = alloc((rows, k), torch.float32)
        self.partial = alloc((rows, H), torch.bfloat16)
        self._checked = False

    def peer(self, base_row):
        """Descriptor of these buffers for a source writing from base_row on. The buffers are
        checked on the first call only (a step builds G descriptors per source, and
        re-checking every tensor each time cost more host time than a dispatch kernel takes)."""
        checked, self._checked = self._checked, True
        return tk.ep_peer(self.x, self.idx, self.w, base_row, self.rows, scale=self.scale,
                          checked=checked)


def local_combine(bufs, n, E_local, align, expert_fn, d, stream=None):
    """Destination side: route rank d's n received rows over its E_local experts, get the
    experts' outputs from expert_fn(d, bufs, n, route_map) (bf16 [rows, H] indexed by local
    slots), and write the per-row partial sums into bufs.partial[:n]."""
    if n == 0:
        return None
    rm = tk.route_map(bufs.idx[:n], E_local, align, stream=stream)
    y = expert_fn(d, bufs, n, rm)
    tk.reduce(y, rm.slot_of, bufs.w[:n], out=bufs.partial[:n], stream=stream, masked=True)
    return rm


class VirtualRanks:
    """G expert-parallel ranks in one process on one device. Each rank's kernels only read and
    write memory, never wait on another rank, so running the ranks' launches one after another
    on one stream gives exactly what G GPUs would compute (the cross-rank barriers become stream
    order)."""

    def __init__(self, G, E, k, H, max_tokens, out_dtype="bf16", align=1, device="cuda"):
        if E % G:
            raise ValueError("G must divide E")
        self.G, self.E, self.k, self.H, self.align = G, E, k, H, align
        self.out_dtype = out_dtype
        self.capacity = capacity_rows(max_tokens, G)
        self.bufs = [RankBuffers(self.capacity, H, k, out_dtype, device) for _ in range(G)]
        self._layouts = {}   # (rank, T) -> preallocated layout outputs

    def _layout_out(self, s, T, device):
        key = (s, T)
        if key not in self._layouts:
            G = self.G
            self._layouts[key] = tk.EpLayout(
                torch.empty(G, dtype=torch.int32, device=device),
                torch.empty(G + 1, dtype=torch.int32, device=device),
                torch.empty(T, G, dtype=torch.int32, device=device),
                torch.empty(T * G, dtype=torch.int32, device=device),
                tk._workspace(int(tk.lib.tk_ep_layout_workspace_bytes(T, G)), device), G)
        return self._layouts[key]

    def step(self, xs, idxs, ws, expert_fn, outs=None, err_flag=None, stream=None, mark=None):
        """One step of all G ranks. mark(name), if given, is called at the phase boundaries
        ("layout", "dispatch", "experts", "combine": the end of each phase)."""
        G = self.G
        mark = mark or (lambda name: None)
        layouts = [tk.ep_layout(idxs[s], self.E, G, out=self._layout_out(s, idxs[s].shape[0], idxs[s].device),
                                err_flag=err_flag, stream=stream) for s in range(G)]
        cm = torch.stack([lay.send_counts for lay in layouts]).cpu()      # the count exchange
        base, recv_rows = recv_bases(cm)
        if int(recv_rows.max()) > self.capacity:
            raise RuntimeError("receive buffer too small")
        mark("layout")
        for s in range(G):
            peers = [self.bufs[d].peer(int(base[s, d])) for d in range(G)]
            tk.ep_dispatch(xs[s], idxs[s], ws[s], layouts[s], self.E, peers, self.out_dtype,
                           err_flag=err_flag, stream=stream)
        mark("dispatch")
        rms = [local_combine(self.bufs[d], int(recv_rows[d]), self.E // G, self.align, expert_fn, d,
                             stream=stream) for d in range(G)]
        mark("experts")
        if outs is None:
            outs = [None] * G
        for s in range(G):
            outs[s] = tk.ep_combine([b.partial for b in self.bufs], base[s].tolist(),
                                    recv_rows.tolist(), layouts[s], self.H, out=outs[s],
                                    err_flag=err_flag, stream=stream)
        mark("combine")
        return {"layouts": layouts, "count_matrix": cm, "base": base, "recv_rows": recv_rows,
                "route_maps": rms, "out": outs}


class EpGroup:
    """One expert-parallel rank per process (one GPU each). The receive buffers live in torch
    symmetric memory, so every rank holds the peer addresses of every other rank's buffers;
    dispatch writes and combine reads them directly. Barriers are collectives of the group."""

    def __init__(self, E, k, H, max_tokens, out_dtype="bf16", align=1, group=None, device=None):
        import torch.distributed._symmetric_memory as symm

        self.G = tdist.get_world_size(group)
        self.rank = tdist.get_rank(group)
        if E % self.G:
            raise ValueError("G must divide E")
        self.E, self.k, self.H, self.align, self.out_dtype = E, k, H, align, out_dtype
        self.group = group
        self.capacity = capacity_rows(max_tokens, self.G)
        device = device or torch.device("cuda", torch.cuda.current_device())
        self._fields, total = [], 0

        def alloc(shape, dtype):   # carve every field out of one symmetric allocation
            nonlocal total
            n = 1
            for v in shape:
                n *= v
            nbytes = n * torch.tensor([], dtype=dtype).element_size()
            self._fields.append((total, shape, dtype))
            total = (total + nbytes + 255) // 256 * 256
            return None

        RankBuffers(self.capacity, H, k, out_dtype, device, alloc=alloc)   # sizes only
        self._raw = symm.empty(max(total, 256), dtype=torch.uint8, device=device)
        self._hdl = symm.rendezvous(self._raw, group if group is not None else tdist.group.WORLD.group_name)
        ptrs = list(self._hdl.buffer_ptrs)
        fields = iter(self._fields)

        def local(shape, dtype):
            off, shp, dt = next(fields)
            n = 1
            for v in shp:
                n *= v
            return self._raw[off:off + n * torch.tensor([], dtype=dt).element_size()].view(dt).view(shp)

        self.bufs = RankBuffers(self.capacity, H, k, out_dtype, device, alloc=local)
        offs = [f[0] for f in self._fields]
        names = ["x", "scale", "idx", "w", "partial"] if out_dtype == "fp8" else ["x", "idx", "w", "partial"]
        self.peer_addr = [{n: ptrs[r] + o for n, o in zip(names, offs)} for r in range(self.G)]

    def _barrier(self):
        tdist.barrier(group=self.group)

    def step(self, x, idx, w, expert_fn, out=None, err_flag=None, stream=None):
        G, r = self.G, self.rank
        lay = tk.ep_layout(idx, self.E, G, err_flag=err_flag, stream=stream)
        base, recv_rows = recv_bases(exchange_counts(lay.send_counts, self.group))
        if int(recv_rows.max()) > self.capacity:
            raise RuntimeError("receive buffer too small")
        peers = [tk.EpPeer(a["x"], a.get("scale"), a["idx"], a["w"], int(base[r, d]), self.capacity)
                 for d, a in enumerate(self.peer_addr)]
        tk.ep_dispatch(x, idx, w, lay, self.E, peers, self.out_dtype, err_flag=err_flag, stream=stream)
        self._barrier()
        local_combine(self.bufs, int(recv_rows[r]), self.E // G, self.align, expert_fn, r, stream=stream)
        self._barrier()
        out = tk.ep_combine([a["partial"] for a in self.peer_addr], base[r].tolist(),
                            recv_rows.tolist(), lay, self.H, out=out, err_flag=err_flag, stream=stream)
        self._barrier()   # no rank reuses its buffers while a peer still reads them
        return out
