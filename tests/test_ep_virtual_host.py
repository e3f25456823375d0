"""Host-side bookkeeping of VirtualRanks.step (G expert-parallel ranks on one device), checked
without a GPU: the library calls are replaced by recorders, so the test sees which buffers and
which row bases each dispatch and combine is given.

What must hold (the layout stated with the tk_ep_* entry points):
- source s writes into destination d's buffers starting at base[s][d] = the rows lower sources
  send to d (recv_bases of the exchanged count matrix), with the buffers' full capacity as bound;
- destination d combines exactly the rows it received;
- source s's combine reads the destinations' partial rows in rank order at base[s][d];
- the phases run in order, and a receive buffer too small for a step is refused before any
  dispatch.
"""
import numpy as np
import pytest
import torch


@pytest.fixture
def vr_env(monkeypatch):
    from token_routing_gate_b200 import build

    build.build()
    from token_routing_gate_b200 import ep, tk

    rec = {"dispatch": [], "combine": [], "local": [], "marks": []}

    def fake_layout(idx, E, G, out=None, err_flag=None, stream=None):
        el = E // G
        owners = [{int(e) // el for e in row if e >= 0} for row in idx.tolist()]
        counts = [sum(d in o for o in owners) for d in range(G)]
        out.send_counts.copy_(torch.tensor(counts, dtype=torch.int32))
        return out

    def fake_peer(x, idx, w, base_row, rows, scale=None, checked=False):
        return {"x": x, "base_row": int(base_row), "rows": int(rows)}

    def fake_dispatch(x, idx, w, layout, E, peers, out_dtype="bf16", err_flag=None, stream=None):
        rec["dispatch"].append((x, peers))

    def fake_local_combine(bufs, n, E_local, align, expert_fn, d, stream=None):
        rec["local"].append((d, n, bufs))
        return None

    def fake_combine(partials, base_rows, rows, layout, H, out=None, err_flag=None, stream=None):
        rec["combine"].append((list(partials), list(base_rows), list(rows)))
        return out

    monkeypatch.setattr(tk, "ep_layout", fake_layout)
    monkeypatch.setattr(tk, "ep_peer", fake_peer)
    monkeypatch.setattr(tk, "ep_dispatch", fake_dispatch)
    monkeypatch.setattr(tk, "ep_combine", fake_combine)
    monkeypatch.setattr(ep, "local_combine", fake_local_combine)
    return ep, rec


def _choices(rng, T, E, k):
    if T == 0:
        return torch.zeros(0, k, dtype=torch.int32)
    idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    idx[rng.random(idx.shape) < 0.2] = -1
    return torch.from_numpy(idx)


def test_bases_buffers_and_order(vr_env):
    ep, rec = vr_env
    G, E, k, H = 3, 12, 3, 8
    Ts = [7, 0, 11]
    rng = np.random.default_rng(5)
    vr = ep.VirtualRanks(G, E, k, H, max(Ts), "bf16", 1, device="cpu")
    xs = [torch.zeros(T, H, dtype=torch.bfloat16) for T in Ts]
    idxs = [_choices(rng, T, E, k) for T in Ts]
    ws = [torch.zeros(T, k) for T in Ts]
    res = vr.step(xs, idxs, ws, expert_fn=None, mark=rec["marks"].append)

    cm = res["count_matrix"]
    base, recv = ep.recv_bases(cm)
    assert rec["marks"] == ["layout", "dispatch", "experts", "combine"]
    # dispatch: one per source, in rank order, destination d's buffers at base[s][d]
    assert len(rec["dispatch"]) == G and all(x is xs[s] for s, (x, _) in enumerate(rec["dispatch"]))
    for s, (_, peers) in enumerate(rec["dispatch"]):
        assert len(peers) == G
        for d, p in enumerate(peers):
            assert p["x"] is vr.bufs[d].x
            assert p["base_row"] == int(base[s, d]) and p["rows"] == vr.capacity
    # each destination combines exactly what it received
    assert [(d, n) for d, n, _ in rec["local"]] == [(d, int(recv[d])) for d in range(G) if recv[d] > 0]
    for d, _, bufs in rec["local"]:
        assert bufs is vr.bufs[d]
    # source s reads the partials of destinations 0..G-1 at base[s][d]
    assert len(rec["combine"]) == G
    for s, (partials, base_rows, rows) in enumerate(rec["combine"]):
        assert all(p is vr.bufs[d].partial for d, p in enumerate(partials))
        assert base_rows == base[s].tolist() and rows == recv.tolist()
    # the count matrix is the sources' layouts stacked row by row
    for s in range(G):
        assert cm[s].tolist() == res["layouts"][s].send_counts.tolist()


def test_receive_overflow_is_refused_before_dispatch(vr_env):
    ep, rec = vr_env
    G, E, k, H = 2, 4, 1, 8
    vr = ep.VirtualRanks(G, E, k, H, 3, "bf16", 1, device="cpu")   # capacity 6 rows per rank
    idxs = [torch.zeros(4, k, dtype=torch.int32) for _ in range(G)]  # 4 tokens each, all to rank 0
    xs = [torch.zeros(4, H, dtype=torch.bfloat16) for _ in range(G)]
    ws = [torch.zeros(4, k) for _ in range(G)]
    with pytest.raises(RuntimeError, match="receive buffer"):
        vr.step(xs, idxs, ws, expert_fn=None)
    assert rec["dispatch"] == []
