"""Parity of the CUDA path (through the C ABI) with the CPU oracle on the five seeded
workloads: indices, counts, offsets, slots and E4M3 bytes/scales bit-exact, weights within 1e-6
relative, reduce within 1 bf16 ulp. Every workload is compared element by element over whole
tensors: gate, route map, every row of the expert-sorted buffer (E4M3 codes and scales for the
FP8-dispatch case, zero padding rows for the skewed case) and every element of the reduce."""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import (DeviceRun, assert_weights_close, assert_weights_round_alike, bf16_bits,
                         bf16_ulp_diff, score_fn)
from token_routing_gate_b200 import workloads as W

pytestmark = pytest.mark.gpu

SMALL = [W.TINY, W.MID]
LARGE = [W.V3, W.SKEW, W.V3_FP8]


def _inputs(wl, device):
    logits, bias = W.gate_inputs(wl, device)
    x = W.activations(wl, device)
    y = W.expert_outputs(wl, device)
    return logits, bias, x, y


def _check_gate_and_route(wl, run, logits, bias):
    lg = logits.cpu().numpy()
    b = bias.cpu().numpy() if bias is not None else None
    o_idx, o_w = oracle.gate_topk(lg, b, wl.k, score_fn(wl))
    np.testing.assert_array_equal(run.idx.cpu().numpy(), o_idx)
    assert_weights_close(run.w.cpu().numpy(), o_w)
    assert_weights_round_alike(run.w.cpu().numpy(), o_w)
    counts, offsets, slot_of, token_of, rc = oracle.route_map(o_idx, wl.E, wl.align)
    assert rc == 0
    np.testing.assert_array_equal(run.rm.counts.cpu().numpy(), counts)
    np.testing.assert_array_equal(run.rm.offsets.cpu().numpy(), offsets)
    np.testing.assert_array_equal(run.rm.slot_of.cpu().numpy(), slot_of)
    np.testing.assert_array_equal(run.rm.token_of.cpu().numpy(), token_of)
    return o_idx, o_w, slot_of, offsets


@pytest.mark.parametrize("wl", SMALL, ids=lambda w: w.name)
def test_small_workload_full_parity(wl):
    torch.manual_seed(0)
    logits, bias, x, y = _inputs(wl, "cpu")
    dev = [t.cuda() if t is not None else None for t in (logits, bias, x, y)]
    run = DeviceRun(wl, *dev)
    assert run.err.item() == 0
    o_idx, o_w, slot_of, offsets = _check_gate_and_route(wl, run, logits, bias)
    R = int(offsets[-1])
    xe_ref, _ = oracle.expand(bf16_bits(x), slot_of, offsets, wl.E, wl.align)
    np.testing.assert_array_equal(bf16_bits(run.xe)[:R], xe_ref[:R])
    out_ref = oracle.reduce(bf16_bits(y), slot_of, o_w)
    d = bf16_ulp_diff(bf16_bits(run.out), out_ref)
    assert d.max() <= 1, d.max()
    # the GPU's own weights reproduce the oracle's reduce bit for bit
    out_same_w = oracle.reduce(bf16_bits(y), slot_of, run.w.cpu().numpy())
    np.testing.assert_array_equal(bf16_bits(run.out), out_same_w)


SLAB = 8192   # rows per comparison slab (the oracle's rows go to the device one slab at a time)


def _assert_rows_equal(got, ref, rows, what):
    """got: device tensor, ref: the oracle's host array; rows [0, rows) equal byte for byte."""
    as_int = {np.dtype(np.uint16): (np.int16, torch.int16), np.dtype(np.float32): (np.int32, torch.int32),
              np.dtype(np.uint8): (np.uint8, torch.uint8)}
    np_t, torch_t = as_int[ref.dtype]
    for r0 in range(0, rows, SLAB):
        r1 = min(rows, r0 + SLAB)
        want = torch.from_numpy(np.ascontiguousarray(ref[r0:r1]).view(np_t)).to(got.device)
        have = got[r0:r1].contiguous().view(torch_t)
        if not torch.equal(have, want):
            bad = (have != want).reshape(r1 - r0, -1).any(dim=1).nonzero()[:5].flatten() + r0
            raise AssertionError(f"{what}: rows {bad.tolist()} differ from the oracle")


def _assert_reduce_within_ulp(out, out_ref, ulps=1):
    """Every element of out (device bf16 [T,H]) within `ulps` bf16 ulps of the oracle's bits."""
    T = out.shape[0]
    worst = 0
    for r0 in range(0, T, SLAB):
        r1 = min(T, r0 + SLAB)
        d = bf16_ulp_diff(bf16_bits(out[r0:r1]), out_ref[r0:r1])
        worst = max(worst, int(d.max()))
    assert worst <= ulps, worst
    return worst


@pytest.mark.parametrize("wl", LARGE, ids=lambda w: w.name)
def test_large_workload_parity(wl):
    """Whole tensors at the DeepSeek-V3 sizes: every row of the expert-sorted buffer (bf16 rows,
    or E4M3 codes and scales, padding included) and every element of the reduce output against
    the oracle's own expand and reduce of the same inputs."""
    logits, bias, x, y = _inputs(wl, "cuda")
    run = DeviceRun(wl, logits, bias, x, y)
    assert run.err.item() == 0
    o_idx, o_w, slot_of, offsets = _check_gate_and_route(wl, run, logits, bias)
    R = int(offsets[-1])
    x_bits = bf16_bits(x)
    if wl.out_dtype == "bf16":
        xe_ref, _ = oracle.expand(x_bits, slot_of, offsets, wl.E, wl.align)
        _assert_rows_equal(run.xe, xe_ref, R, "expand (bf16)")
        del xe_ref
    else:
        q_ref, s_ref = oracle.expand(x_bits, slot_of, offsets, wl.E, wl.align, oracle.OUT_FP8_E4M3)
        _assert_rows_equal(run.xq, q_ref, R, "expand (E4M3 codes)")
        _assert_rows_equal(run.xs, s_ref, R, "expand (E4M3 scales)")
        del q_ref, s_ref
    del x_bits
    y_bits = bf16_bits(y)
    out_ref = oracle.reduce(y_bits, slot_of, o_w)
    _assert_reduce_within_ulp(run.out, out_ref)
    # with the GPU's own weights the oracle's reduce is reproduced bit for bit
    out_same_w = oracle.reduce(y_bits, slot_of, run.w.cpu().numpy())
    _assert_reduce_within_ulp(run.out, out_same_w, ulps=0)


def test_pipeline_is_deterministic():
    wl = W.V3_FP8.with_(T=2048)
    logits, bias, x, y = _inputs(wl, "cuda")
    a = DeviceRun(wl, logits, bias, x, y)
    b = DeviceRun(wl, logits, bias, x, y)
    for name in ("idx", "w", "xq", "xs", "out"):
        assert torch.equal(getattr(a, name).view(torch.uint8), getattr(b, name).view(torch.uint8)), name
    for name in ("counts", "offsets", "slot_of", "token_of"):
        assert torch.equal(getattr(a.rm, name), getattr(b.rm, name)), name


# ---------------------------------------------------------------- randomised sweep
# TK_FULL_TEST=1 widens it (more seeds and shapes); TK_SEED moves the base seed.
import os

_FULL = os.environ.get("TK_FULL_TEST", "0") == "1"
_BASE = int(os.environ.get("TK_SEED", "4242"))


@pytest.mark.parametrize("case", range(24 if _FULL else 6))
def test_random_shapes_against_oracle(case):
    rng = np.random.default_rng(_BASE + case)
    E = int(rng.choice([8, 16, 33, 64, 128, 256, 300, 1024]))
    k = int(rng.integers(1, min(E, 32) + 1))
    T = int(rng.integers(1, 3000))
    out_dtype = str(rng.choice(["bf16", "fp8"]))
    score = str(rng.choice(["softmax", "sigmoid"]))
    bias = bool(rng.integers(0, 2)) and score == "sigmoid"
    align = int(rng.choice([1, 1, 4, 128] if E <= 64 else [1, 4]))
    rmax = T * k + E * (align - 1)
    hs = [128, 256, 1024, 2176] if out_dtype == "fp8" else [8, 72, 264, 1024, 3000]
    hs = [h for h in hs if rmax * h <= 40_000_000] or hs[:1]   # keep the CPU-side inputs small
    H = int(rng.choice(hs))
    wl = W.Workload(f"rand{case}", T, E, k, H, score, bias, bool(rng.integers(0, 2)), align,
                    out_dtype, _BASE + 1000 + case)
    logits, b, x, y = _inputs(wl, "cpu")
    dev = [t.cuda() if t is not None else None for t in (logits, b, x, y)]
    run = DeviceRun(wl, *dev)
    assert run.err.item() == 0
    o_idx, o_w, slot_of, offsets = _check_gate_and_route(wl, run, logits, b)
    R = int(offsets[-1])
    if out_dtype == "fp8":
        q_ref, s_ref = oracle.expand(bf16_bits(x), slot_of, offsets, wl.E, wl.align, oracle.OUT_FP8_E4M3)
        np.testing.assert_array_equal(run.xq.cpu().numpy()[:R], q_ref[:R])
        np.testing.assert_array_equal(run.xs.cpu().numpy()[:R], s_ref[:R])
    else:
        xe_ref, _ = oracle.expand(bf16_bits(x), slot_of, offsets, wl.E, wl.align)
        np.testing.assert_array_equal(bf16_bits(run.xe)[:R], xe_ref[:R])
    out_ref = oracle.reduce(bf16_bits(y), slot_of, o_w)
    assert bf16_ulp_diff(bf16_bits(run.out), out_ref).max() <= 1
