"""Selection keys at planted one-ulp near-ties ("DeepSeek 的 GPU 内核帝国", section "MoE TopK
门控": the 'min' index reducer decides equal keys; the key's fp32 exponential is fixed so that
both sides produce the same bits).

The CPU tests check the construction itself: the pairs are planted (at least 10^4 of them one
fp32 ulp apart), a plain numpy restatement of the selection on the oracle's keys reproduces the
oracle's indices, and an exponential one ulp off changes thousands of selections, so the GPU
test below would catch a kernel whose key exponential differed from the oracle's in the last
bit. They also report the margin the seeded DeepSeek-V3-shaped workloads leave at the k-th key.
The GPU test runs the gate through the C ABI on the planted logits and compares every index
bit for bit with the oracle."""
import numpy as np
import pytest

import near_ties as N
import oracle
from token_routing_gate_b200 import workloads as W

T_PLANT, E, K = 8192, 256, 8


def _bias(wl):
    return W.gate_inputs(wl.with_(T=1), "cpu")[1].numpy()


def _emulated_selection(e_minus_l, bias, k):
    """Indices of the k largest keys fl(fl(1 / fl(1 + e)) + b), ties to the lower index, from
    given exponentials e = exp(-l) (numpy float32 arithmetic, stable sort)."""
    one = np.float32(1)
    keys = (one / (one + e_minus_l) + bias[None, :]).astype(np.float32)
    return np.argsort(-keys, axis=1, kind="stable")[:, :k].astype(np.int32)


@pytest.mark.parametrize("wl", [W.V3, W.V3_FP8], ids=lambda w: w.name)
def test_pairs_are_planted(wl):
    bias = _bias(wl)
    logits, pairs, offset = N.planted_logits(T_PLANT, E, bias, seed=wl.seed)
    keys = N.keys_of(logits, np.broadcast_to(bias, logits.shape))
    rows = np.arange(T_PLANT)
    assert (offset != 99).all()
    for i in range(len(N.PAIR_RANKS)):
        ka, kb = keys[rows, pairs[:, i, 0]], keys[rows, pairs[:, i, 1]]
        np.testing.assert_array_equal(N.ulp_gap(ka, kb), np.abs(offset[:, i]))
        np.testing.assert_array_equal(np.sign(kb.astype(np.float64) - ka), np.sign(offset[:, i]))
    assert (np.abs(offset) == 1).sum() >= 10_000
    assert (offset == 0).sum() >= 2_000
    # every planted pair lies on the ladder the oracle selects from: ranks 2/3, 5/6 both
    # selected, and at 8/9 exactly one of the two is
    idx, _ = oracle.gate_topk(logits, bias, K, oracle.SIGMOID)
    chosen = np.zeros((T_PLANT, E), dtype=bool)
    chosen[rows[:, None], idx] = True
    for i, (pa, pb) in enumerate(N.PAIR_RANKS):
        both = chosen[rows, pairs[:, i, 0]].astype(int) + chosen[rows, pairs[:, i, 1]]
        assert (both == (1 if pb == K else 2)).all()


def test_numpy_restatement_matches_oracle_and_one_ulp_flips_selections():
    bias = _bias(W.V3)
    logits, _, _ = N.planted_logits(T_PLANT, E, bias, seed=W.V3.seed)
    idx, _ = oracle.gate_topk(logits, bias, K, oracle.SIGMOID)
    e = oracle.spec_expf(-logits).reshape(logits.shape)
    np.testing.assert_array_equal(_emulated_selection(e, bias, K), idx)
    up = np.nextafter(e, np.float32(np.inf))
    down = np.nextafter(e, np.float32(-np.inf))
    rng = np.random.default_rng(0)
    half = np.where(rng.random(e.shape) < 0.5, up, e)
    for name, pert in (("+1 ulp", up), ("-1 ulp", down), ("+1 ulp on half", half)):
        changed = (_emulated_selection(pert, bias, K) != idx).any(axis=1).sum()
        assert changed >= 1000, (name, changed)


@pytest.mark.parametrize("wl", [W.V3, W.V3_FP8], ids=lambda w: w.name)
def test_report_boundary_margin_of_seeded_workloads(wl):
    """How close the seeded inputs come to a tie at the k-th key (diagnostic; the seeded
    V3-shaped batches leave at least 11 ulps at every token)."""
    logits, bias = W.gate_inputs(wl, "cpu")
    gaps = N.boundary_gaps(logits.numpy(), bias.numpy(), wl.k)
    close = int((gaps <= 4).sum())
    print(f"{wl.name}: tokens with a k/(k+1) key gap <= 4 ulp: {close}; smallest gap "
          f"{int(gaps.min())} ulp")
    assert close == 0


@pytest.mark.gpu
@pytest.mark.parametrize("wl", [W.V3, W.V3_FP8], ids=lambda w: w.name)
def test_gpu_selection_at_planted_near_ties(wl):
    import torch

    from gpu_helpers import assert_weights_close
    from token_routing_gate_b200 import tk

    bias = _bias(wl)
    logits, _, offset = N.planted_logits(T_PLANT, E, bias, seed=wl.seed)
    assert (np.abs(offset) <= 2).sum() >= 20_000
    o_idx, o_w = oracle.gate_topk(logits, bias, K, oracle.SIGMOID)
    idx, w = tk.gate_topk(torch.from_numpy(logits).cuda(), K, "sigmoid",
                          torch.from_numpy(bias).cuda(), True)
    torch.cuda.synchronize()
    got = idx.cpu().numpy()
    bad = (got != o_idx).any(axis=1)
    assert not bad.any(), f"{bad.sum()} tokens select differently; first {np.flatnonzero(bad)[:5]}"
    assert_weights_close(w.cpu().numpy(), o_w)
    # the same inputs drawn on the device side (the large parity tests' inputs): margin report
    lg_dev, b_dev = W.gate_inputs(wl, "cuda")
    gaps = N.boundary_gaps(lg_dev.cpu().numpy(), b_dev.cpu().numpy(), wl.k)
    print(f"{wl.name} (device draw): k/(k+1) gaps <= 4 ulp: {int((gaps <= 4).sum())}, "
          f"smallest {int(gaps.min())}")
