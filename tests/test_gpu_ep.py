"""Expert-parallel dispatch / combine on one GPU: G ranks run as VirtualRanks (each rank's kernels
only read and write memory and never wait on another rank, so their launches can run one after
another on one device), compared with the oracle's statement of the same step. Layout, receive
buffers (rows, E4M3 codes and scales, local choices, weights) and the combine are bit-exact; the
destinations' partial sums are the single-GPU reduce (within 1 bf16 ulp, 0 expected)."""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import bf16_bits, bf16_ulp_diff
from token_routing_gate_b200 import ep, tk

pytestmark = pytest.mark.gpu


def _choices(rng, T, E, k, masked=0.0):
    if T == 0:
        return np.zeros((0, k), dtype=np.int32)
    idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    if masked:
        idx[rng.random(idx.shape) < masked] = -1
    return idx


def _bits(rng, shape):
    return bf16_bits(torch.from_numpy(rng.standard_normal(shape).astype(np.float32)).to(torch.bfloat16))


def _max_ulp(a_bits, b_bits):
    d = bf16_ulp_diff(a_bits, b_bits)
    return int(d.max()) if d.size else 0


def _to_bf16(bits, dev="cuda"):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(dev).view(torch.bfloat16)


class _Experts:
    """Seeded expert outputs per destination rank, the same on the GPU and for the oracle."""

    def __init__(self, seed, H, E_local, k, align):
        self.seed, self.H, self.el, self.k, self.align = seed, H, E_local, k, align
        self.host = {}

    def for_oracle(self, d, rows):
        rng = np.random.default_rng(self.seed + d)
        self.host[d] = _bits(rng, (rows, self.H))
        return self.host[d]

    def for_gpu(self, d, bufs, n, rm):
        return _to_bf16(self.host[d])


def _run(G, E, k, H, Ts, out_dtype="bf16", align=1, masked=0.1, seed=7):
    rng = np.random.default_rng(seed)
    xs = [_bits(rng, (T, H)) for T in Ts]
    idxs = [_choices(rng, T, E, k, masked) for T in Ts]
    ws = [rng.random((T, k)).astype(np.float32) for T in Ts]
    experts = _Experts(seed * 1000, H, E // G, k, align)
    ref = oracle.ep_forward(xs, idxs, ws, experts.for_oracle, E, G, align,
                            oracle.OUT_FP8_E4M3 if out_dtype == "fp8" else oracle.OUT_BF16)
    vr = ep.VirtualRanks(G, E, k, H, max(Ts), out_dtype, align)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    res = vr.step([_to_bf16(x) for x in xs], [torch.from_numpy(i).cuda() for i in idxs],
                  [torch.from_numpy(w).cuda() for w in ws], experts.for_gpu, err_flag=err)
    torch.cuda.synchronize()
    return ref, vr, res, err


def _check(ref, vr, res, err, G, out_dtype):
    assert err.item() == 0
    np.testing.assert_array_equal(res["count_matrix"].numpy(), ref["count_matrix"])
    np.testing.assert_array_equal(res["base"].numpy(), ref["base"])
    for s, lay in enumerate(res["layouts"]):
        counts, dest = ref["layout"][s]
        np.testing.assert_array_equal(lay.send_counts.cpu().numpy(), counts)
        off = lay.send_offsets.cpu().numpy()
        assert off[0] == 0 and np.array_equal(np.diff(off), counts)
        ds = lay.dest_slot.cpu().numpy()
        np.testing.assert_array_equal(np.where(ds >= 0, ds - off[:-1][None, :], -1), dest)
    for d in range(G):
        n = int(ref["recv_rows"][d])
        b = vr.bufs[d]
        rx, rs, ri, rw = ref["recv"][d]
        if out_dtype == "fp8":
            np.testing.assert_array_equal(b.x[:n].cpu().numpy(), rx)
            np.testing.assert_array_equal(b.scale[:n].cpu().numpy(), rs)
        else:
            np.testing.assert_array_equal(bf16_bits(b.x[:n]), rx)
        np.testing.assert_array_equal(b.idx[:n].cpu().numpy(), ri)
        np.testing.assert_array_equal(b.w[:n].cpu().numpy(), rw)
        if n:
            D = ref["dest"][d]
            rm = res["route_maps"][d]
            np.testing.assert_array_equal(rm.slot_of.cpu().numpy(), D["slot_of"])
            assert _max_ulp(bf16_bits(b.partial[:n]), ref["partials"][d]) <= 1
    # combine: bit-exact against the oracle's combine of the GPU's own partials, and within
    # 1 ulp of the oracle end to end
    parts = [bf16_bits(vr.bufs[d].partial[:max(int(ref["recv_rows"][d]), 1)]) for d in range(G)]
    for s in range(G):
        got = bf16_bits(res["out"][s])
        np.testing.assert_array_equal(got, oracle.ep_combine(parts, ref["base"][s], ref["layout"][s][1]))
        assert _max_ulp(got, ref["out"][s]) <= 1


@pytest.mark.parametrize("G,E,k", [(1, 16, 4), (2, 16, 4), (4, 32, 6), (8, 64, 8), (32, 64, 4)])
def test_ep_layout_matches_oracle(G, E, k):
    rng = np.random.default_rng(G * 31 + k)
    T = 1000
    idx = _choices(rng, T, E, k, masked=0.15)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    lay = tk.ep_layout(torch.from_numpy(idx).cuda(), E, G, err_flag=err)
    counts, dest = oracle.ep_layout(idx, E, G)
    torch.cuda.synchronize()
    assert err.item() == 0
    np.testing.assert_array_equal(lay.send_counts.cpu().numpy(), counts)
    off = lay.send_offsets.cpu().numpy()
    ds = lay.dest_slot.cpu().numpy()
    np.testing.assert_array_equal(np.where(ds >= 0, ds - off[:-1][None, :], -1), dest)
    tok = lay.send_token.cpu().numpy()
    for d in range(G):   # the send list of each destination names its tokens in order
        np.testing.assert_array_equal(tok[off[d]:off[d + 1]], np.nonzero(dest[:, d] >= 0)[0])
    assert np.all(tok[off[G]:] == -1)


@pytest.mark.parametrize("out_dtype", ["bf16", "fp8"])
@pytest.mark.parametrize("G,E,k,H,Ts,align", [
    (2, 16, 4, 256, [300, 257], 1),
    (4, 32, 6, 1024, [123, 400, 1, 77], 1),
    (8, 64, 8, 384, [64] * 8, 4),
    (3, 24, 24, 128, [50, 0, 31], 1),
], ids=["G2", "G4_ragged", "G8_align4", "G3_k_all"])
def test_ep_forward_matches_oracle(out_dtype, G, E, k, H, Ts, align):
    ref, vr, res, err = _run(G, E, k, H, Ts, out_dtype, align)
    _check(ref, vr, res, err, G, out_dtype)


def test_ep_deepseek_v3_shape():
    # 8 ranks x 96 tokens, 256 experts (32 per rank), top-8, hidden 7168, FP8 dispatch
    G, E, k, H = 8, 256, 8, 7168
    ref, vr, res, err = _run(G, E, k, H, [96] * G, "fp8", masked=0.0, seed=11)
    _check(ref, vr, res, err, G, "fp8")


def test_ep_one_rank_is_the_single_gpu_path():
    rng = np.random.default_rng(5)
    T, E, k, H = 700, 32, 4, 512
    x = _to_bf16(_bits(rng, (T, H)))
    idx = torch.from_numpy(_choices(rng, T, E, k)).cuda()
    w = torch.from_numpy(rng.random((T, k)).astype(np.float32)).cuda()
    y = _to_bf16(_bits(rng, (T * k, H)))
    vr = ep.VirtualRanks(1, E, k, H, T)
    res = vr.step([x], [idx], [w], lambda d, bufs, n, rm: y)
    rm = tk.route_map(idx, E)
    single = tk.reduce(y, rm.slot_of, w)
    torch.cuda.synchronize()
    assert torch.equal(vr.bufs[0].x[:T].view(torch.int16), x.view(torch.int16))
    assert torch.equal(res["out"][0].view(torch.int16), single.view(torch.int16))


def test_ep_overflow_is_flagged_not_written():
    rng = np.random.default_rng(9)
    G, E, k, H, T = 2, 8, 2, 64, 100
    idx = torch.from_numpy(_choices(rng, T, E, k)).cuda()
    x = _to_bf16(_bits(rng, (T, H)))
    w = torch.ones(T, k, device="cuda")
    lay = tk.ep_layout(idx, E, G)
    cap = 10
    bufs = [ep.RankBuffers(cap + 4, H, k, "bf16", "cuda") for _ in range(G)]
    for b in bufs:
        b.x.fill_(3.0)
    peers = [tk.ep_peer(b.x, b.idx, b.w, 0, cap) for b in bufs]
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    tk.ep_dispatch(x, idx, w, lay, E, peers, err_flag=err)
    torch.cuda.synchronize()
    assert err.item() & tk.DEVERR_ROWS_RANGE
    for b in bufs:   # rows past the capacity stay untouched
        assert torch.all(b.x[cap:] == 3.0)
    err.zero_()
    out = tk.ep_combine([b.partial for b in bufs], [0] * G, [cap] * G, lay, H, err_flag=err)
    torch.cuda.synchronize()
    assert err.item() & tk.DEVERR_SLOT_RANGE


def test_ep_writes_stay_inside_the_receive_blocks():
    # every destination's buffers are pre-filled; after the step, rows at and past recv_rows
    # (and the whole buffer of a rank that receives nothing) are unchanged
    G, E, k, H = 4, 16, 2, 256
    rng = np.random.default_rng(13)
    Ts = [40, 0, 25, 60]
    xs = [_to_bf16(_bits(rng, (T, H))) for T in Ts]
    idxs = []
    for T in Ts:   # nothing goes to rank 3's experts (12..15)
        idxs.append(torch.from_numpy(_choices(rng, T, 12, k)).cuda())
    ws = [torch.rand(T, k, device="cuda") for T in Ts]
    vr = ep.VirtualRanks(G, E, k, H, max(Ts))
    for b in vr.bufs:
        b.x.fill_(-5.0)
        b.idx.fill_(-7)
        b.w.fill_(-9.0)
        b.partial.fill_(-11.0)
    res = vr.step(xs, idxs, ws, lambda d, bufs, n, rm: torch.ones(tk.max_rows(n, E // G, k, 1), H,
                                                                     dtype=torch.bfloat16, device="cuda"))
    torch.cuda.synchronize()
    recv = res["recv_rows"].tolist()
    assert recv[3] == 0
    for d, b in enumerate(vr.bufs):
        n = recv[d]
        assert torch.all(b.x[n:] == -5.0) and torch.all(b.idx[n:] == -7)
        assert torch.all(b.w[n:] == -9.0) and torch.all(b.partial[n:] == -11.0)
        assert not torch.any(b.idx[:n] == -7)
