"""Parity of the next routing ops with the oracle: load-balance statistics, the tensor-parallel
expert mask (and routing of its masked output), and the backward of reduce and expand."""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import bf16_bits, bf16_ulp_diff, bits_to_f32
from token_routing_gate_b200 import tk
from token_routing_gate_b200 import workloads as W

pytestmark = pytest.mark.gpu

ULP32 = 2.0 ** -23  # both sides accumulate in double; the fp32 outputs differ by rounding only


# E=300 and E=1024 take the partial kernel's 8-warp forms (shared memory above 48 KB at 1024)
# and the final sums' uneven (3 threads per column) and unsplit (1 per column) forms
LARGE_E = [W.V3.with_(T=515, E=300, k=6, name="T515_E300_k6_sigmoid_bias"),
           W.MID.with_(T=333, E=1024, k=8, name="T333_E1024_k8_softmax")]


@pytest.mark.parametrize("wl", [W.V3, W.MID, W.TINY.with_(T=77, E=37, k=5),
                                W.SKEW.with_(T=1000), *LARGE_E], ids=lambda w: w.name)
def test_balance_stats(wl):
    logits, bias = W.gate_inputs(wl, "cuda")
    idx, _ = tk.gate_topk(logits, wl.k, wl.score, bias)
    rm = tk.route_map(idx, wl.E, 1)
    P, f, loss = tk.balance_stats(logits, rm.counts, wl.k, wl.score)
    P2, f2, loss2 = tk.balance_stats(logits, rm.counts, wl.k, wl.score)
    torch.cuda.synchronize()
    assert torch.equal(P, P2) and torch.equal(loss, loss2)          # deterministic
    fn = oracle.SOFTMAX if wl.score == "softmax" else oracle.SIGMOID
    Pr, fr, lr = oracle.balance_stats(logits.cpu().numpy(), rm.counts.cpu().numpy(), wl.k, fn)
    np.testing.assert_allclose(P.cpu().numpy(), Pr, rtol=ULP32, atol=0)
    np.testing.assert_allclose(f.cpu().numpy(), fr, rtol=ULP32, atol=0)
    assert abs(loss.item() - lr) <= ULP32 * abs(lr)


def test_balance_stats_empty_batch():
    counts = torch.zeros(16, dtype=torch.int32, device="cuda")
    P, f, loss = tk.balance_stats(torch.empty(0, 16, device="cuda"), counts, 2, "softmax")
    torch.cuda.synchronize()
    assert (P == 0).all() and (f == 0).all() and loss.item() == 0.0


def _balance_vs_oracle(logits, k, score):
    logits_d = torch.from_numpy(logits).cuda()
    idx, _ = tk.gate_topk(logits_d, k, score)
    rm = tk.route_map(idx, logits.shape[1], 1)
    P, f, loss = tk.balance_stats(logits_d, rm.counts, k, score)
    torch.cuda.synchronize()
    fn = oracle.SOFTMAX if score == "softmax" else oracle.SIGMOID
    Pr, fr, lr = oracle.balance_stats(logits, rm.counts.cpu().numpy(), k, fn)
    np.testing.assert_allclose(P.cpu().numpy(), Pr, rtol=ULP32, atol=0, equal_nan=True)
    np.testing.assert_allclose(f.cpu().numpy(), fr, rtol=ULP32, atol=0)
    np.testing.assert_allclose(loss.cpu().numpy(), np.float32(lr), rtol=ULP32, atol=0, equal_nan=True)
    return Pr


@pytest.mark.parametrize("score", ["sigmoid", "softmax"])
def test_balance_stats_extreme_logits(score):
    """Scores computed on both sides of the statistics' short double-precision path (magnitudes
    up to 708) and on the library path beyond: rows scaled to 300, 707.9, 708, 708.1, 750, 1e4
    and 1e30, the boundary values themselves, and infinite logits (-inf only for softmax, where
    +inf makes the row's maximum infinite)."""
    rng = np.random.default_rng(31 + (score == "softmax"))
    T, E, k = 900, 96, 6
    scale = rng.choice([1.0, 300.0, 707.9, 708.0, 708.1, 750.0, 1e4, 1e30], size=(T, 1))
    logits = (rng.standard_normal((T, E)) * scale).astype(np.float32)
    pick = rng.random((T, E))
    logits[pick < 0.02] = np.float32(708.0)
    logits[(pick >= 0.02) & (pick < 0.04)] = np.float32(-708.0)
    logits[(pick >= 0.04) & (pick < 0.05)] = np.nextafter(np.float32(708.0), np.float32(np.inf))
    logits[(pick >= 0.05) & (pick < 0.06)] = -np.inf
    if score == "sigmoid":
        logits[(pick >= 0.06) & (pick < 0.07)] = np.inf
    Pr = _balance_vs_oracle(logits, k, score)
    assert np.isfinite(Pr).all()


def test_balance_stats_non_finite_rows():
    """A NaN logit makes its token's normalised scores NaN (so every P), and a sigmoid row whose
    scores all underflow to 0 divides 0 by 0: both sides give NaN in the same places."""
    rng = np.random.default_rng(33)
    logits = rng.standard_normal((300, 64)).astype(np.float32)
    logits[17, 5] = np.nan
    _balance_vs_oracle(logits, 4, "sigmoid")
    _balance_vs_oracle(logits, 4, "softmax")
    logits = rng.standard_normal((300, 64)).astype(np.float32)
    logits[40, :] = -800.0
    assert np.isnan(_balance_vs_oracle(logits, 4, "sigmoid")).all()


def test_balance_short_path_accuracy():
    """Exhaustively over every fp32 logit with |l| <= 708: the statistics' table-driven e^-l and
    Newton-refined logistic score stay within 2^-50 relative of the library's exp and division."""
    err = tk.selftest_balance_exp()
    torch.cuda.synchronize()
    e_exp, e_sig = (float(v) for v in err.cpu())
    print(f"largest relative difference: exp {e_exp:.3e}, logistic {e_sig:.3e}")
    assert e_exp < 2.0 ** -50 and e_sig < 2.0 ** -50


@pytest.mark.parametrize("wl", [W.MID, W.V3.with_(T=3000), *LARGE_E], ids=lambda w: w.name)
def test_balance_sums_then_finalize_is_the_one_call(wl):
    logits, bias = W.gate_inputs(wl, "cuda")
    idx, _ = tk.gate_topk(logits, wl.k, wl.score, bias)
    rm = tk.route_map(idx, wl.E, 1)
    one = tk.balance_stats(logits, rm.counts, wl.k, wl.score)
    sums = tk.balance_score_sums(logits, wl.score)
    two = tk.balance_finalize(sums, rm.counts, wl.T, wl.k)
    torch.cuda.synchronize()
    for a, b in zip(one, two):
        assert torch.equal(a, b)


@pytest.mark.parametrize("shards", [2, 3, 8])
def test_global_balance_stats_over_rank_shards(shards):
    # a batch split unevenly over ranks: per-rank sums and counts, added in rank order (what the
    # all-reduce computes), then finalize == the statistics of the whole batch
    wl = W.V3.with_(T=5000)
    logits, bias = W.gate_inputs(wl, "cuda")
    idx, _ = tk.gate_topk(logits, wl.k, wl.score, bias)
    cuts = np.linspace(0, wl.T, shards + 1).astype(int)
    cuts[1] = 7                                   # a tiny first shard
    sums = torch.zeros(wl.E, dtype=torch.float64, device="cuda")
    counts = torch.zeros(wl.E, dtype=torch.int32, device="cuda")
    for a, b in zip(cuts[:-1], cuts[1:]):
        sums += tk.balance_score_sums(logits[a:b].contiguous(), wl.score)
        counts += tk.route_map(idx[a:b].contiguous(), wl.E, 1).counts
    P, f, loss = tk.balance_finalize(sums, counts, wl.T, wl.k)
    full = tk.route_map(idx, wl.E, 1).counts
    torch.cuda.synchronize()
    assert torch.equal(counts, full)
    Pr, fr, lr = oracle.balance_stats(logits.cpu().numpy(), full.cpu().numpy(), wl.k, oracle.SIGMOID)
    np.testing.assert_allclose(P.cpu().numpy(), Pr, rtol=ULP32, atol=0)
    np.testing.assert_allclose(f.cpu().numpy(), fr, rtol=ULP32, atol=0)
    assert abs(loss.item() - lr) <= ULP32 * abs(lr)


@pytest.mark.parametrize("k", [8, 12, 16, 24, 32])
def test_reduce_mixed_valid_counts(k):
    """Tokens keep a random number of their k choices (the rest masked -1), so consecutive units
    of the reduce's row ring need very different amounts of it -- a unit of more than half the
    ring right after a small one included. Both forms match the oracle, no wait gives up."""
    rng = np.random.default_rng(k)
    T, E, H = 1500, 64, 2304
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    keep = rng.integers(0, k + 1, T)
    keep[rng.random(T) < 0.3] = k                     # many fully valid tokens among them
    for t in range(T):
        idx[t, rng.permutation(k)[keep[t]:]] = -1
    w = rng.random((T, k)).astype(np.float32)
    counts, offsets, slot_of, token_of, rc = oracle.route_map(idx, E, 1)
    rows = max(int(offsets[-1]), 1)
    y = torch.randn(rows, H, generator=torch.Generator().manual_seed(k)).to(torch.bfloat16)
    ref = oracle.reduce(bf16_bits(y), slot_of, w)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    yd, sd, wd = y.cuda(), torch.from_numpy(slot_of).cuda(), torch.from_numpy(w).cuda()
    a = tk.reduce(yd, sd, wd, err_flag=err)
    b = tk.reduce(yd, sd, wd, err_flag=err, masked=True)
    torch.cuda.synchronize()
    assert err.item() == 0
    np.testing.assert_array_equal(bf16_bits(a), ref)
    np.testing.assert_array_equal(bf16_bits(b), ref)


@pytest.mark.parametrize("case", ["dense", "tp8", "ep_like", "ragged"])
def test_reduce_masked_equals_reduce(case):
    wl = {"dense": W.V3.with_(T=3000, H=1024), "tp8": W.V3.with_(T=4000, H=512),
          "ep_like": W.V3.with_(T=2500, H=7168), "ragged": W.MID.with_(T=777, H=200)}[case]
    logits, bias = W.gate_inputs(wl, "cuda")
    idx, w = tk.gate_topk(logits, wl.k, wl.score, bias)
    E = wl.E
    if case == "tp8":                       # 7/8 of the pairs masked
        idx = tk.tp_mask(idx, wl.E, 8, 3)
        E = wl.E // 8
    if case == "ep_like":                   # keep one expert group of eight, as a destination would
        idx = torch.where((idx // 32) == 5, idx - 160, torch.full_like(idx, -1))
        E = 32
    rm = tk.route_map(idx, E, 1)
    y = W.expert_outputs(wl.with_(E=E), "cuda", rows=max(tk.max_rows(wl.T, E, wl.k, 1), 1))
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    a = tk.reduce(y, rm.slot_of, w, err_flag=err)
    b = tk.reduce(y, rm.slot_of, w, err_flag=err, masked=True)
    c = tk.reduce(y, rm.slot_of, None, err_flag=err, masked=True)
    d = tk.reduce(y, rm.slot_of, None, err_flag=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert torch.equal(c.view(torch.int16), d.view(torch.int16))
    if case == "ragged":                    # and the oracle, element by element
        ref = oracle.reduce(bf16_bits(y), rm.slot_of.cpu().numpy(), w.cpu().numpy())
        assert bf16_ulp_diff(bf16_bits(b), ref).max() <= 1


@pytest.mark.parametrize("tp", [1, 2, 8])
def test_tp_mask_then_route(tp):
    wl = W.V3.with_(T=3000)
    logits, bias = W.gate_inputs(wl, "cuda")
    idx, _ = tk.gate_topk(logits, wl.k, wl.score, bias)
    idx_h = idx.cpu().numpy()
    owned = torch.zeros_like(idx)
    for r in range(tp):
        m = tk.tp_mask(idx, wl.E, tp, r)
        ref = oracle.tp_mask(idx_h, wl.E, tp, r)
        np.testing.assert_array_equal(m.cpu().numpy(), ref)
        owned += (m >= 0).int()
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        rm = tk.route_map(m, wl.E // tp, 128, err_flag=err)
        torch.cuda.synchronize()
        assert err.item() == 0                                      # masked pairs are not errors
        counts, offsets, slot_of, token_of, rc = oracle.route_map(ref, wl.E // tp, 128)
        assert rc == 0
        np.testing.assert_array_equal(rm.counts.cpu().numpy(), counts)
        np.testing.assert_array_equal(rm.offsets.cpu().numpy(), offsets)
        np.testing.assert_array_equal(rm.slot_of.cpu().numpy(), slot_of)
        np.testing.assert_array_equal(rm.token_of.cpu().numpy(), token_of)
    assert (owned == 1).all()
    inplace = idx.clone()
    tk.tp_mask(inplace, wl.E, tp, tp - 1, out=inplace)
    np.testing.assert_array_equal(inplace.cpu().numpy(), oracle.tp_mask(idx_h, wl.E, tp, tp - 1))


@pytest.mark.parametrize("T,E,k,tp,align", [
    (3000, 256, 8, 8, 128),    # V3 experts over 8 tensor-parallel ranks
    (8192, 256, 8, 2, 1),      # the V3 batch, two ranks
    (40000, 64, 6, 4, 4),      # several tiles per CTA, fused count matrix
    (20000, 1024, 4, 2, 16),   # 512 local experts: count matrix past the fused limit
    (77, 37, 5, 1, 3),         # the whole map as one window
])
def test_route_map_window_equals_mask_then_route(T, E, k, tp, align):
    """tk_route_map_window on each rank's expert window gives exactly tk_tp_mask followed by
    tk_route_map with the local experts (and the oracle's tp_mask + route_map)."""
    rng = np.random.default_rng(T + E + tp)
    idx_h = np.argsort(rng.random((T, E)), axis=1)[:, :k].astype(np.int32)
    if T > 10:
        idx_h[5, 1] = -1                      # a pair masked before the call
    idx = torch.from_numpy(idx_h).cuda()
    el = E // tp
    for r in range(tp):
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        got = tk.route_map_window(idx, E, r * el, el, align, err_flag=err)
        ref = tk.route_map(tk.tp_mask(idx, E, tp, r), el, align)
        torch.cuda.synchronize()
        assert err.item() == 0
        for a, b in ((got.counts, ref.counts), (got.offsets, ref.offsets), (got.slot_of, ref.slot_of),
                     (got.token_of, ref.token_of)):
            assert torch.equal(a, b)
        counts, offsets, slot_of, token_of, rc = oracle.route_map(oracle.tp_mask(idx_h, E, tp, r), el, align)
        assert rc == 0
        np.testing.assert_array_equal(got.slot_of.cpu().numpy(), slot_of)
        np.testing.assert_array_equal(got.offsets.cpu().numpy(), offsets)
        np.testing.assert_array_equal(got.token_of.cpu().numpy(), token_of)


def test_route_map_window_flags_indices_outside_all_experts():
    """An index outside [0, E_total) other than -1 sets the expert-range bit and is masked; one
    outside the window but inside [0, E_total) is only masked."""
    T, E, k = 600, 64, 4
    rng = np.random.default_rng(9)
    idx_h = np.argsort(rng.random((T, E)), axis=1)[:, :k].astype(np.int32)
    idx_h[3, 0], idx_h[4, 2] = E, -5
    idx = torch.from_numpy(idx_h).cuda()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    got = tk.route_map_window(idx, E, 16, 16, 1, err_flag=err)
    torch.cuda.synchronize()
    assert err.item() & 1                     # TK_DEVERR_EXPERT_RANGE
    slots = got.slot_of.cpu().numpy()
    assert slots[3, 0] == -1 and slots[4, 2] == -1
    clean = idx_h.copy()
    clean[3, 0], clean[4, 2] = -1, -1
    counts, offsets, slot_of, token_of, _ = oracle.route_map(oracle.tp_mask(clean, E, 4, 1), 16, 1)
    np.testing.assert_array_equal(slots, slot_of)
    np.testing.assert_array_equal(got.counts.cpu().numpy(), counts)


@pytest.mark.parametrize("T,E,k,H,align,weighted", [
    (300, 16, 4, 264, 8, True),      # ragged chunk, padding rows
    (2048, 256, 8, 7168, 1, True),   # DeepSeek-V3 row shape
    (129, 8, 1, 2048, 4, False),     # k = 1, unit weights
    (40, 64, 32, 1024, 1, True),     # largest k: one stage per CTA
])
def test_reduce_backward(T, E, k, H, align, weighted):
    wl = W.V3.with_(T=T, E=E, k=k, H=H, align=align, bias=False, seed=T + H)
    logits, _ = W.gate_inputs(wl, "cuda")
    idx, w = tk.gate_topk(logits, k, "sigmoid")
    rm = tk.route_map(idx, E, align)
    rows = wl.max_rows
    y = W.expert_outputs(wl, "cuda", rows=rows)
    g = W.activations(wl.with_(seed=wl.seed + 5), "cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    d_y = torch.full_like(y, 7.0)                                      # garbage where not written
    d_y, d_w = tk.reduce_backward(g, y, rm.slot_of, w if weighted else None, E, rm=rm, d_y=d_y,
                                  err_flag=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    offsets = rm.offsets.cpu().numpy()
    R = int(offsets[-1])
    dy_ref, dw_ref, rc = oracle.reduce_backward(bf16_bits(g), bf16_bits(y), rm.slot_of.cpu().numpy(),
                                                offsets, w.cpu().numpy() if weighted else None, E)
    assert rc == 0
    np.testing.assert_array_equal(bf16_bits(d_y)[:R], dy_ref[:R])
    np.testing.assert_allclose(d_w.cpu().numpy(), dw_ref, rtol=ULP32, atol=0)
    d_w2 = tk.reduce_backward(g, y, rm.slot_of, w if weighted else None, E, rm=rm)[1]
    torch.cuda.synchronize()
    assert torch.equal(d_w, d_w2)                                      # deterministic


def test_reduce_backward_full_size_properties():
    wl = W.V3
    logits, bias = W.gate_inputs(wl, "cuda")
    idx, w = tk.gate_topk(logits, wl.k, wl.score, bias)
    rm = tk.route_map(idx, wl.E, 1)
    y = W.expert_outputs(wl, "cuda")
    g = W.activations(wl.with_(seed=77), "cuda")
    d_y, d_w = tk.reduce_backward(g, y, rm.slot_of, w, wl.E, rm=rm)
    torch.cuda.synchronize()
    sl = rm.slot_of.long()
    # d_y[slot] = bf16(w * g) for every pair (fp32 product, round to nearest even)
    want = (w[:, :, None] * g.float()[:, None, :]).to(torch.bfloat16)
    assert torch.equal(d_y[sl].view(torch.int16), want.view(torch.int16))
    # d_w = <g, y[slot]>: exact products summed in double, then fp32
    exact = torch.einsum("tc,tjc->tj", g.double(), y[sl].double())
    assert torch.all((d_w.double() - exact).abs() <= ULP32 * exact.abs() + 1e-30)


def test_expand_backward_is_the_unweighted_reduce():
    wl = W.V3.with_(T=1024, align=128, skew=True)
    logits, _ = W.gate_inputs(wl, "cuda")
    idx, _ = tk.gate_topk(logits, wl.k, "sigmoid")
    rm = tk.route_map(idx, wl.E, wl.align)
    d_xe = W.expert_outputs(wl, "cuda")
    d_x = tk.expand_backward(d_xe, rm.slot_of)
    ref_gpu = tk.reduce(d_xe, rm.slot_of, None)
    torch.cuda.synchronize()
    assert torch.equal(d_x.view(torch.int16), ref_gpu.view(torch.int16))
    ref = oracle.reduce(bf16_bits(d_xe), rm.slot_of.cpu().numpy(), None)
    np.testing.assert_array_equal(bf16_bits(d_x), ref)
