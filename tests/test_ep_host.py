"""Host logic of the expert-parallel path, on CPU: the receive bases from the G x G send counts
(against the oracle), and the count exchange between ranks over gloo -- every rank must end up
with the same count matrix and bases, since each source writes into its peers' buffers at the
base it computes itself."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp


def test_recv_bases_match_the_oracle(oracle_lib):
    from token_routing_gate_b200 import ep

    rng = np.random.default_rng(41)
    for G in (1, 2, 3, 8, 32):
        cm = rng.integers(0, 1000, (G, G)).astype(np.int32)
        base, recv = ep.recv_bases(torch.from_numpy(cm))
        o_base, o_recv = oracle_lib.ep_recv_bases(cm)
        np.testing.assert_array_equal(base.numpy(), o_base)
        np.testing.assert_array_equal(recv.numpy(), o_recv)
    with pytest.raises(ValueError):
        ep.recv_bases(torch.zeros(2, 3, dtype=torch.int32))
    with pytest.raises(ValueError):
        ep.recv_bases(torch.tensor([[1, -1], [0, 0]]))
    assert ep.capacity_rows(8192, 8) == 65536


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, result_dir):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as tdist

    import oracle
    from token_routing_gate_b200 import dist, ep

    assert dist.init("gloo", timeout_s=60)
    E, k, T = 24, 4, 50 + 7 * rank          # ranks hold different numbers of tokens
    rng = np.random.default_rng(100 + rank)
    idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    counts, dest = oracle.ep_layout(idx, E, world)
    cm = ep.exchange_counts(torch.from_numpy(counts))
    base, recv = ep.recv_bases(cm)
    np.testing.assert_array_equal(cm[rank].numpy(), counts)
    gathered = [None] * world
    tdist.all_gather_object(gathered, (counts, base.numpy(), recv.numpy(), idx))
    if rank == 0:
        for g in gathered:                  # one matrix, the same bases on every rank
            np.testing.assert_array_equal(g[1], gathered[0][1])
            np.testing.assert_array_equal(g[2], gathered[0][2])
        o_base, o_recv = oracle.ep_recv_bases(np.stack([g[0] for g in gathered]))
        np.testing.assert_array_equal(base.numpy(), o_base)
        np.testing.assert_array_equal(recv.numpy(), o_recv)
        # the blocks the sources write into each destination tile it exactly, without overlap
        for d in range(world):
            spans = sorted((int(o_base[s, d]), int(o_base[s, d]) + int(gathered[s][0][d]))
                           for s in range(world))
            assert spans[0][0] == 0 and spans[-1][1] == o_recv[d]
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
        open(os.path.join(result_dir, "ok"), "w").close()
    dist.finish()


def test_count_exchange_three_gloo_ranks(tmp_path, oracle_lib):
    world = 3
    mp.spawn(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    assert (tmp_path / "ok").exists()


def _balance_worker(rank, world, port, result_dir):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as tdist

    from token_routing_gate_b200 import dist

    assert dist.init("gloo", timeout_s=60)
    E = 16
    g = torch.Generator().manual_seed(rank)
    sums = torch.randint(0, 1 << 20, (E,), generator=g).to(torch.float64) / 64.0   # exact in double
    counts = torch.randint(0, 1000, (E,), generator=g, dtype=torch.int32)
    T = 100 + rank
    s2, c2, T2 = dist.allreduce_balance_inputs(sums.clone(), counts, T)
    gathered = [None] * world
    tdist.all_gather_object(gathered, (sums, counts, T, s2, c2, T2))
    if rank == 0:
        want_s = sum(x[0] for x in gathered)
        want_c = sum(x[1] for x in gathered)
        for x in gathered:   # every rank holds the same totals
            assert torch.equal(x[3], want_s) and torch.equal(x[4], want_c.to(torch.int32))
            assert x[5] == sum(y[2] for y in gathered)
        open(os.path.join(result_dir, "ok"), "w").close()
    dist.finish()


def test_balance_inputs_allreduce_three_gloo_ranks(tmp_path):
    world = 3
    mp.spawn(_balance_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    assert (tmp_path / "ok").exists()


def test_balance_inputs_single_rank_unchanged():
    from token_routing_gate_b200 import dist

    sums = torch.arange(4, dtype=torch.float64)
    counts = torch.arange(4, dtype=torch.int32)
    s, c, T = dist.allreduce_balance_inputs(sums, counts, 7)
    assert s is sums and c is counts and T == 7


def test_epgroup_carves_one_symmetric_allocation(monkeypatch):
    # EpGroup's host logic with torch's symmetric memory replaced by a CPU fake: every field of
    # the receive buffers is a view of the one allocation at the offset that the peer addresses
    # use, fields are 256-byte aligned and do not overlap, and each rank's addresses are its base
    # plus the same offsets
    import torch.distributed as tdist
    import torch.distributed._symmetric_memory as symm

    from token_routing_gate_b200 import ep

    class FakeHandle:
        def __init__(self, t):
            self.buffer_ptrs = [t.data_ptr() + (1 << 40) * r for r in range(1)]

    monkeypatch.setattr(symm, "empty", lambda n, dtype, device: torch.empty(n, dtype=dtype))
    monkeypatch.setattr(symm, "rendezvous", lambda t, group: FakeHandle(t))
    tdist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0,
                             world_size=1)
    try:
        for out_dtype, names in (("bf16", ["x", "idx", "w", "partial"]),
                                 ("fp8", ["x", "scale", "idx", "w", "partial"])):
            g = ep.EpGroup(E=32, k=4, H=256, max_tokens=10, out_dtype=out_dtype, device="cpu")
            assert g.G == 1 and g.capacity == 10
            base = g._raw.data_ptr()
            spans = []
            for name in names:
                t = getattr(g.bufs, name)
                off = t.data_ptr() - base
                assert off % 256 == 0 and g.peer_addr[0][name] == base + off
                spans.append((off, off + t.numel() * t.element_size()))
            spans.sort()
            assert all(a[1] <= b[0] for a, b in zip(spans, spans[1:]))
            assert spans[-1][1] <= g._raw.numel()
            assert set(g.peer_addr[0]) == set(names)
    finally:
        tdist.destroy_process_group()
