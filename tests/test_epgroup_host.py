"""EpGroup.step's host logic on three gloo ranks (CPU processes), with torch's symmetric memory
replaced by a fake that hands out made-up peer addresses and the four kernels replaced by
recorders. The counts really go through the all-gather; the test checks what each rank's
dispatch and combine are given:
- the exchanged count matrix is every rank's layout counts (the oracle's), row by row;
- rank r writes into rank d's buffers at d's receive address, starting at base[r][d], bounded by
  the capacity;
- rank r routes and combines exactly the rows it received;
- rank r's combine reads every rank's partial buffer, in rank order, at base[r][d].
"""
import os
import socket

import numpy as np
import torch
import torch.multiprocessing as mp

E, K, H = 24, 3, 256
TOKENS = [13, 0, 21]          # uneven, one rank with no tokens


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _choices(rank):
    T = TOKENS[rank]
    if T == 0:
        return np.zeros((0, K), np.int32)
    rng = np.random.default_rng(300 + rank)
    idx = np.stack([rng.choice(E, K, replace=False) for _ in range(T)]).astype(np.int32)
    idx[rng.random(idx.shape) < 0.15] = -1
    return idx


def _worker(rank, world, port, result_dir):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed._symmetric_memory as symm

    import oracle
    from token_routing_gate_b200 import dist, ep, tk

    fake_base = [(r + 1) << 40 for r in range(world)]   # never dereferenced: the kernels are fakes

    class FakeHandle:
        buffer_ptrs = fake_base

    symm.empty = lambda n, dtype, device: torch.empty(n, dtype=dtype)
    symm.rendezvous = lambda t, group: FakeHandle()
    rec = {}

    def fake_layout(idx, E_, G, err_flag=None, stream=None, out=None):
        counts, _ = oracle.ep_layout(idx.numpy(), E_, G)
        z = torch.zeros(1, dtype=torch.int32)
        return tk.EpLayout(torch.as_tensor(counts, dtype=torch.int32), z, z, z, z, G)

    def fake_dispatch(x, idx, w, lay, E_, peers, out_dtype, err_flag=None, stream=None):
        rec["peers"] = [(p.x, p.idx, p.w, p.base_row, p.rows) for p in peers]

    def fake_local(bufs, n, E_local, align, expert_fn, d, stream=None):
        rec["local"] = (n, E_local, d)

    def fake_combine(partials, base_rows, rows, lay, H_, out=None, err_flag=None, stream=None):
        rec["combine"] = (list(partials), list(base_rows), list(rows))
        return out

    tk.ep_layout, tk.ep_dispatch, tk.ep_combine = fake_layout, fake_dispatch, fake_combine
    ep.local_combine = fake_local

    assert dist.init("gloo", timeout_s=60)
    try:
        g = ep.EpGroup(E, K, H, max(TOKENS), "bf16", device="cpu")
        x = torch.zeros(TOKENS[rank], H, dtype=torch.bfloat16)
        idx = torch.from_numpy(_choices(rank))
        w = torch.zeros(TOKENS[rank], K)
        g.step(x, idx, w, expert_fn=None)

        cm = np.stack([oracle.ep_layout(_choices(r), E, world)[0] for r in range(world)])
        base, recv = ep.recv_bases(torch.as_tensor(cm))
        offs = {n: g.peer_addr[0][n] - fake_base[0] for n in ("x", "idx", "w", "partial")}
        assert rec["peers"] == [(fake_base[d] + offs["x"], fake_base[d] + offs["idx"],
                                 fake_base[d] + offs["w"], int(base[rank, d]), g.capacity)
                                for d in range(world)]
        assert rec["local"] == (int(recv[rank]), E // world, rank)
        partials, base_rows, rows = rec["combine"]
        assert partials == [fake_base[d] + offs["partial"] for d in range(world)]
        assert base_rows == base[rank].tolist() and rows == recv.tolist()
        open(os.path.join(result_dir, f"ok{rank}"), "w").close()
    finally:
        dist.finish()


def test_epgroup_step_bookkeeping_on_three_ranks(tmp_path):
    from token_routing_gate_b200 import build

    build.build()
    world = 3
    mp.spawn(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    assert all((tmp_path / f"ok{r}").exists() for r in range(world))
