"""Edge cases of the CUDA path against the oracle, compared in full: empty and ragged batches,
k = 1 and k = E, expert counts that are not multiples of the warp width, ties, masked (-inf)
experts, all tokens on one expert, empty experts, several alignments, rows that need more than
one bulk-copy stage, zero and signed-zero FP8 blocks, and both renormalisation modes."""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import assert_weights_close, bf16_bits, bf16_ulp_diff
from token_routing_gate_b200 import tk
from token_routing_gate_b200.workloads import Workload

pytestmark = pytest.mark.gpu


def _case(T, E, k, H, score="sigmoid", bias=False, align=1, out_dtype="bf16", seed=7):
    return Workload(f"edge_T{T}_E{E}_k{k}_H{H}", T, E, k, H, score, bias, False, align, out_dtype, seed)


def _full_check(wl, logits, bias, x, y, renormalize=True, check_order_only=False):
    """Run the four calls and compare everything with the oracle; returns the GPU outputs."""
    dev = "cuda"
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    lg_d = torch.as_tensor(logits, device=dev)
    b_d = torch.as_tensor(bias, device=dev) if bias is not None else None
    x_d = torch.as_tensor(x).view(torch.bfloat16).to(dev) if x.dtype == np.uint16 else x.to(dev)
    y_d = torch.as_tensor(y).view(torch.bfloat16).to(dev) if y.dtype == np.uint16 else y.to(dev)
    idx, w = tk.gate_topk(lg_d, wl.k, wl.score, b_d, renormalize)
    rm = tk.route_map(idx, wl.E, wl.align, err_flag=err)
    if wl.out_dtype == "fp8":
        xq, xs = tk.expand(x_d, rm, wl.E, wl.k, "fp8", err_flag=err)
    else:
        xe = tk.expand(x_d, rm, wl.E, wl.k, "bf16", err_flag=err)
    out = tk.reduce(y_d, rm.slot_of, w, err_flag=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    fn = oracle.SOFTMAX if wl.score == "softmax" else oracle.SIGMOID
    o_idx, o_w = oracle.gate_topk(np.asarray(logits, np.float32), bias, wl.k, fn, renormalize)
    np.testing.assert_array_equal(idx.cpu().numpy(), o_idx)
    assert_weights_close(w.cpu().numpy(), o_w)
    counts, offsets, slot_of, token_of, _ = oracle.route_map(o_idx, wl.E, wl.align)
    np.testing.assert_array_equal(rm.counts.cpu().numpy(), counts)
    np.testing.assert_array_equal(rm.offsets.cpu().numpy(), offsets)
    np.testing.assert_array_equal(rm.slot_of.cpu().numpy(), slot_of)
    np.testing.assert_array_equal(rm.token_of.cpu().numpy()[:len(token_of)], token_of)
    R = int(offsets[-1])
    xb = bf16_bits(x_d)
    if wl.out_dtype == "fp8":
        q_ref, s_ref = oracle.expand(xb, slot_of, offsets, wl.E, wl.align, oracle.OUT_FP8_E4M3)
        np.testing.assert_array_equal(xq.cpu().numpy()[:R], q_ref[:R])
        np.testing.assert_array_equal(xs.cpu().numpy()[:R], s_ref[:R])
    else:
        xe_ref, _ = oracle.expand(xb, slot_of, offsets, wl.E, wl.align)
        np.testing.assert_array_equal(bf16_bits(xe)[:R], xe_ref[:R])
    out_ref = oracle.reduce(bf16_bits(y_d), slot_of, o_w)
    assert bf16_ulp_diff(bf16_bits(out), out_ref).max(initial=0) <= 1  # (an empty batch has no rows)
    np.testing.assert_array_equal(bf16_bits(out), oracle.reduce(bf16_bits(y_d), slot_of, w.cpu().numpy()))
    return dict(idx=idx, w=w, rm=rm, out=out)


def _rand_inputs(wl, rng, rows=None):
    logits = rng.standard_normal((wl.T, wl.E)).astype(np.float32)
    bias = rng.uniform(-0.1, 0.1, wl.E).astype(np.float32) if wl.bias else None
    x = torch.randn(wl.T, wl.H, generator=torch.Generator().manual_seed(wl.seed)).to(torch.bfloat16)
    rows = wl.max_rows if rows is None else rows
    y = torch.randn(max(rows, 1), wl.H, generator=torch.Generator().manual_seed(wl.seed + 1)).to(torch.bfloat16)
    return logits, bias, x, y


@pytest.mark.parametrize("T,E,k,H,score,bias,align,out", [
    (1, 8, 1, 8, "softmax", False, 1, "bf16"),          # single token, k = 1, minimal H
    (3, 16, 16, 64, "softmax", False, 1, "bf16"),       # k = E
    (5, 32, 32, 128, "sigmoid", True, 1, "fp8"),        # k = E = warp width
    (20000, 24, 3, 64, "sigmoid", True, 1, "bf16"),     # several tokens per gate warp
    (40000, 16, 2, 8, "softmax", False, 4, "bf16"),     # 313 tiles, small count matrix: fused
    (20000, 512, 4, 8, "sigmoid", True, 4, "bf16"),     # count matrix > 32K: many-CTA row scan
    (33000, 256, 8, 8, "sigmoid", True, 1, "bf16"),     # 258 tiles: row scan, 16 threads per row, 3 idle
    (257, 37, 5, 264, "sigmoid", True, 1, "bf16"),      # ragged T, E % 32 != 0, H % 128 != 0
    (300, 1000, 12, 256, "softmax", False, 7, "bf16"),  # E close to the limit, odd alignment
    (64, 1024, 32, 128, "sigmoid", True, 128, "fp8"),   # largest E and k
    (513, 64, 6, 2048, "softmax", False, 128, "fp8"),   # many padding rows
    (40, 48, 4, 20480, "sigmoid", False, 16, "bf16"),   # 40 KB rows: two bulk-copy stages, padded
    (40, 48, 4, 9216, "sigmoid", True, 16, "fp8"),      # 9216 channels: two quantisation stages
])
def test_shapes(T, E, k, H, score, bias, align, out):
    wl = _case(T, E, k, H, score, bias, align, out, seed=T + E)
    _full_check(wl, *_rand_inputs(wl, np.random.default_rng(T * E)))


def test_empty_batch():
    wl = _case(0, 16, 2, 256, align=4)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    idx, w = tk.gate_topk(torch.empty(0, 16, device="cuda"), 2, "sigmoid")
    rm = tk.route_map(idx, 16, 4, err_flag=err)
    xe = tk.expand(torch.empty(0, 256, dtype=torch.bfloat16, device="cuda"), rm, 16, 2)
    out = tk.reduce(xe, rm.slot_of, w)
    torch.cuda.synchronize()
    assert err.item() == 0 and out.shape == (0, 256)
    assert rm.counts.cpu().tolist() == [0] * 16 and rm.offsets.cpu().tolist() == [0] * 17
    assert (rm.token_of.cpu() == -1).all() and rm.token_of.numel() == wl.max_rows


@pytest.mark.parametrize("score", ["softmax", "sigmoid"])
def test_all_equal_logits_break_ties_low(score):
    wl = _case(70, 40, 8, 64, score)
    logits, bias, x, y = _rand_inputs(wl, np.random.default_rng(1))
    logits[:] = 0.25
    r = _full_check(wl, logits, None, x, y)
    assert (r["idx"].cpu().numpy() == np.arange(8)[None, :]).all()
    assert (r["w"].cpu().numpy() == 0.125).all()


def test_few_levels_many_ties_with_bias():
    wl = _case(400, 64, 6, 128, "sigmoid", True)
    rng = np.random.default_rng(2)
    logits = (rng.integers(-2, 3, (wl.T, wl.E)) * 0.5).astype(np.float32)
    bias = (rng.integers(-1, 2, wl.E) * 0.125).astype(np.float32)
    _, _, x, y = _rand_inputs(wl, rng)
    _full_check(wl, logits, bias, x, y)


def test_masked_experts_softmax():
    wl = _case(100, 32, 4, 64, "softmax")
    logits, _, x, y = _rand_inputs(wl, np.random.default_rng(3))
    logits[:, 1::2] = -np.inf                      # half the experts masked
    logits[:5, :] = -np.inf                        # tokens with nothing unmasked
    logits[5:9, 4:] = -np.inf                      # tokens with exactly 2 finite experts < k
    r = _full_check(wl, logits, None, x, y)
    w = r["w"].cpu().numpy()
    assert (w[:5] == 0).all()


def test_every_token_on_one_expert_and_empty_experts():
    wl = _case(600, 64, 4, 128, "sigmoid", True, align=128)
    logits, bias, x, y = _rand_inputs(wl, np.random.default_rng(4))
    bias[:] = -0.1
    bias[13] = 5.0                                 # every token picks expert 13 first
    logits[:, 40:] = -30.0                         # experts 40.. stay empty
    r = _full_check(wl, logits, bias, x, y)
    assert (r["idx"][:, 0] == 13).all()
    assert r["rm"].counts[13].item() == 600


@pytest.mark.parametrize("renormalize", [False, True])
@pytest.mark.parametrize("score", ["softmax", "sigmoid"])
def test_renormalize_modes(score, renormalize):
    wl = _case(333, 96, 6, 64, score)
    _full_check(wl, *_rand_inputs(wl, np.random.default_rng(5)), renormalize=renormalize)


def test_fp8_zero_and_signed_zero_blocks():
    wl = _case(16, 8, 2, 512, "sigmoid", True, out_dtype="fp8")
    logits, bias, x, y = _rand_inputs(wl, np.random.default_rng(6))
    x = x.clone()
    x[0, :] = 0.0                                  # all blocks amax 0
    x[1, :128] = -0.0                              # a block of -0 only: amax 0 -> codes 0x00
    x[2, :128] = 0.0
    x[2, 5] = -0.0                                 # -0 inside a live block -> 0x80
    x[2, 6] = 3.0
    x[3, 128:256] = 1e-30                          # tiny values: scale underflows toward 0
    x[3, 130] = -2e-30
    x[4, 256:384] = 300.0                          # equal magnitudes: all land on 448
    _full_check(wl, logits, bias, x, y)


def test_expand_then_unweighted_reduce_k1_identity():
    wl = _case(2000, 16, 1, 7168, "sigmoid", True)
    logits, bias, x, _ = _rand_inputs(wl, np.random.default_rng(8), rows=0)
    xd = x.cuda()
    idx, w = tk.gate_topk(torch.as_tensor(logits, device="cuda"), 1, "sigmoid", torch.as_tensor(bias, device="cuda"))
    rm = tk.route_map(idx, 16, 1)
    xe = tk.expand(xd, rm, 16, 1)
    out = tk.reduce(xe, rm.slot_of, None)
    torch.cuda.synchronize()
    xb = bf16_bits(xd)
    xb[xb == 0x8000] = 0                           # fmaf(1, -0, +0) = +0
    np.testing.assert_array_equal(bf16_bits(out), xb)


def test_non_default_stream():
    wl = _case(512, 64, 4, 256, "sigmoid", True)
    logits, bias, x, y = _rand_inputs(wl, np.random.default_rng(9))
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        idx, w = tk.gate_topk(torch.as_tensor(logits, device="cuda"), 4, "sigmoid",
                              torch.as_tensor(bias, device="cuda"))
        rm = tk.route_map(idx, 64, 1)
        out = tk.reduce(y.cuda(), rm.slot_of, w)
    s.synchronize()
    o_idx, o_w = oracle.gate_topk(logits, bias, 4, oracle.SIGMOID)
    np.testing.assert_array_equal(idx.cpu().numpy(), o_idx)
    _, _, slot_of, _, _ = oracle.route_map(o_idx, 64, 1)
    ref = oracle.reduce(bf16_bits(y), slot_of, o_w)
    assert bf16_ulp_diff(bf16_bits(out), ref).max() <= 1
