"""Pins for the CPU oracle: each check ties it to something other than itself -- a library
routine (numpy, scipy, torch casts), brute force, a closed form, an invariant, or a case worked
out by hand (tests/golden/hand_cases.json). A dropped term, a wrong sign, a swapped index or an
off-by-one in any oracle step fails at least one of these."""
import itertools
import json
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
with open(os.path.join(HERE, "golden", "hand_cases.json")) as f:
    HAND = json.load(f)


def _sigmoid(x):
    return 1.0 / (1.0 + math.exp(-x))


def _eval(expr):
    return eval(expr, {"__builtins__": {}}, {"math": math, "sigmoid": _sigmoid})


def _ulp32(x):
    """Spacing of fp32 numbers at |x| (the fp32 ulp), as float64."""
    x = np.abs(np.asarray(x, dtype=np.float64)).astype(np.float32)
    return (np.nextafter(x, np.float32(np.inf)) - x).astype(np.float64)


# ---------------------------------------------------------------- fp32 exponential for keys
def test_spec_exp_accuracy_dense(oracle_lib):
    xs = np.concatenate([np.linspace(-20, 20, 400_001, dtype=np.float32),
                         np.random.default_rng(0).uniform(-87, 88, 200_000).astype(np.float32)])
    got = oracle_lib.spec_expf(xs).astype(np.float64)
    exact = np.exp(xs.astype(np.float64))
    err_ulp = np.abs(got - exact) / _ulp32(exact)
    # faithfully rounded: never a full ulp off, and mostly correctly rounded
    assert err_ulp.max() < 1.0, err_ulp.max()
    assert np.mean(err_ulp <= 0.5) > 0.9


def test_spec_exp_subnormal_and_limits(oracle_lib):
    xs = np.array([0.0, -0.0, 100.0, 89.0, -110.0, -104.0, np.inf, -np.inf], dtype=np.float32)
    got = oracle_lib.spec_expf(xs)
    assert got[0] == 1.0 and got[1] == 1.0
    assert np.isinf(got[2]) and np.isinf(got[3]) and np.isinf(got[6])
    assert got[4] == 0.0 and got[5] == 0.0 and got[7] == 0.0
    assert np.isnan(oracle_lib.spec_expf(np.array([np.nan], dtype=np.float32))[0])
    # deep underflow: within one subnormal step of the exact value
    xs = np.linspace(-103.5, -87.5, 2001, dtype=np.float32)
    got = oracle_lib.spec_expf(xs).astype(np.float64)
    exact = np.exp(xs.astype(np.float64))
    tiny = 2.0 ** -149
    assert np.all(np.abs(got - exact) <= np.maximum(2 * _ulp32(exact), tiny))
    # powers of two: e^(n ln 2) = 2^n within 2 ulp
    n = np.arange(-120, 127, dtype=np.float64)
    got = oracle_lib.spec_expf((n * math.log(2)).astype(np.float32)).astype(np.float64)
    exact = np.exp((n * math.log(2)).astype(np.float32).astype(np.float64))
    assert np.all(np.abs(got - exact) <= 2 * _ulp32(exact))


def test_spec_sigmoid(oracle_lib):
    xs = np.linspace(-30, 30, 600_001, dtype=np.float32)
    got = oracle_lib.spec_sigmoidf(xs).astype(np.float64)
    exact = scipy.special.expit(xs.astype(np.float64))
    assert np.all(np.abs(got - exact) <= 3 * _ulp32(exact))
    assert oracle_lib.spec_sigmoidf(np.array([0.0], np.float32))[0] == 0.5
    assert np.all(np.diff(got) >= 0)  # non-decreasing
    ends = oracle_lib.spec_sigmoidf(np.array([-np.inf, np.inf, 200, -200], np.float32))
    assert list(ends) == [0.0, 1.0, 1.0, 0.0]


# ---------------------------------------------------------------- bf16 rounding
def test_bf16_rne_matches_torch(oracle_lib):
    rng = np.random.default_rng(1)
    bits = rng.integers(0, 2**32, 1_000_000, dtype=np.uint64).astype(np.uint32)
    bits = bits[((bits >> 23) & 0xFF) != 0xFF]                       # finite only
    halfway = (rng.integers(0, 2**16, 50_000, dtype=np.uint32) << 16)
    halfway = np.concatenate([halfway | 0x8000, halfway | 0x7FFF, halfway | 0x8001])
    halfway = halfway[((halfway >> 23) & 0xFF) < 0xFE]
    x = np.concatenate([bits, halfway]).view(np.float32)
    x = np.concatenate([x, rng.standard_normal(100_000).astype(np.float32)])
    got = oracle_lib.bf16_rne(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(got, ref)


# ---------------------------------------------------------------- E4M3 encoder
def _e4m3_table():
    codes = torch.arange(0, 0x7F, dtype=torch.uint8)                 # 0x00..0x7E, finite >= 0
    vals = codes.view(torch.float8_e4m3fn).to(torch.float32).numpy().astype(np.float64)
    return codes.numpy(), vals


def test_e4m3_table_shape():
    codes, vals = _e4m3_table()
    assert vals[0] == 0.0 and vals[-1] == 448.0 and vals[1] == 2.0 ** -9
    assert np.all(np.diff(vals) > 0)


def _nearest_even(a, vals):
    """Brute-force round-to-nearest-even of |values| onto the E4M3 grid (codes 0x00-0x7E),
    saturating above 448."""
    i = np.clip(np.searchsorted(vals, a), 1, len(vals) - 1)
    lo, hi = vals[i - 1], vals[i]
    dlo, dhi = a - lo, hi - a
    pick_hi = (dhi < dlo) | ((dhi == dlo) & ((i % 2) == 0))
    code = np.where(pick_hi, i, i - 1)
    code = np.where(a >= 448.0, 0x7E, code)
    return code.astype(np.uint8)


def test_e4m3_encoder_brute_force(oracle_lib):
    _, vals = _e4m3_table()
    # every fp32 exponent from 2^-14 to 2^8, all top-11 mantissa patterns, and low bits that
    # straddle each rounding boundary
    top = np.arange(2 ** 11, dtype=np.uint32) << 12
    low = np.array([0, 1, 0x7FF, 0x800, 0x801, 0xFFF], dtype=np.uint32)
    exps = np.arange(127 - 14, 127 + 9, dtype=np.uint32) << 23
    bits = (exps[:, None, None] | top[None, :, None] | low[None, None, :]).reshape(-1)
    x = bits.view(np.float32)
    x = np.concatenate([x, np.random.default_rng(2).uniform(0, 470, 500_000).astype(np.float32),
                        np.array([0.0, 2.0 ** -10, 3 * 2.0 ** -10, 448.0, 464.0, 1e30, np.inf],
                                 dtype=np.float32)])
    want = _nearest_even(x.astype(np.float64), vals)
    got = oracle_lib.e4m3_encode(x)
    np.testing.assert_array_equal(got, want)
    got_neg = oracle_lib.e4m3_encode(-x)
    np.testing.assert_array_equal(got_neg, want | 0x80)


def test_e4m3_encoder_matches_torch_cast(oracle_lib):
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.standard_normal(500_000) * 100,
                        rng.uniform(-448, 448, 200_000),
                        rng.standard_normal(100_000) * 1e-3]).astype(np.float32)
    x = x[np.abs(x) <= 448]
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = oracle_lib.e4m3_encode(x)
    # torch keeps -0 for tiny negatives too; compare all codes
    np.testing.assert_array_equal(got, ref)


def test_e4m3_special_values(oracle_lib):
    x = np.array([-0.0, -1e-4, 449.0, 1e9, -1e9, np.inf, -np.inf], dtype=np.float32)
    assert list(oracle_lib.e4m3_encode(x)) == [0x80, 0x80, 0x7E, 0x7E, 0xFE, 0x7E, 0xFE]


# ---------------------------------------------------------------- gate
def _keys(oracle_lib, logits, bias):
    if bias is None:
        return logits.astype(np.float32)
    s = oracle_lib.spec_sigmoidf(logits).reshape(logits.shape)
    return (s + bias[None, :].astype(np.float32)).astype(np.float32)


@pytest.mark.parametrize("score,with_bias", [("softmax", False), ("sigmoid", False),
                                             ("sigmoid", True)])
@pytest.mark.parametrize("E,k", [(6, 1), (6, 3), (8, 4), (9, 9), (12, 5)])
def test_gate_brute_force(oracle_lib, score, with_bias, E, k):
    rng = np.random.default_rng(E * 100 + k)
    T = 40
    # a few logit levels only, so ties are common
    logits = (rng.integers(-3, 4, (T, E)) * 0.5).astype(np.float32)
    bias = (rng.integers(-2, 3, E) * 0.05).astype(np.float32) if with_bias else None
    fn = oracle_lib.SOFTMAX if score == "softmax" else oracle_lib.SIGMOID
    idx, w = oracle_lib.gate_topk(logits, bias, k, fn)
    keys = _keys(oracle_lib, logits, bias).astype(np.float64)
    for t in range(T):
        chosen = list(idx[t])
        assert len(set(chosen)) == k and all(0 <= e < E for e in chosen)
        best = max(sum(keys[t, list(c)]) for c in itertools.combinations(range(E), k))
        assert sum(keys[t, chosen]) == best
        # order: descending key, equal keys by ascending expert (python's sort as the library)
        assert chosen == sorted(range(E), key=lambda e: (-keys[t, e], e))[:k]
        assert abs(float(np.sum(w[t], dtype=np.float64)) - 1.0) <= 1e-6


def test_gate_all_equal(oracle_lib):
    logits = np.zeros((5, 16), dtype=np.float32)
    for fn in (oracle_lib.SOFTMAX, oracle_lib.SIGMOID):
        idx, w = oracle_lib.gate_topk(logits, None, 4, fn)
        assert (idx == np.arange(4)[None, :]).all()
        assert (w == 0.25).all()


def test_gate_softmax_weights_library(oracle_lib):
    rng = np.random.default_rng(7)
    logits = rng.standard_normal((64, 32)).astype(np.float32)
    p = scipy.special.softmax(logits.astype(np.float64), axis=1)
    # k = E: renormalised over all experts is the full softmax
    idx, w = oracle_lib.gate_topk(logits, None, 32, oracle_lib.SOFTMAX)
    np.testing.assert_allclose(w, np.take_along_axis(p, idx, 1), rtol=1e-6)
    # not renormalised: the chosen experts' softmax probabilities
    idx, w = oracle_lib.gate_topk(logits, None, 6, oracle_lib.SOFTMAX, renormalize=False)
    np.testing.assert_allclose(w, np.take_along_axis(p, idx, 1), rtol=1e-6)
    # renormalised: ratios are exp of logit differences, sum is one
    idx, w = oracle_lib.gate_topk(logits, None, 6, oracle_lib.SOFTMAX)
    l_sel = np.take_along_axis(logits, idx, 1).astype(np.float64)
    np.testing.assert_allclose(w[:, 1:] / w[:, :1], np.exp(l_sel[:, 1:] - l_sel[:, :1]), rtol=2e-6)
    np.testing.assert_allclose(w.sum(1, dtype=np.float64), 1.0, atol=1e-6)
    assert np.all(np.diff(w, axis=1) <= 0)


def test_gate_sigmoid_weights_library(oracle_lib):
    rng = np.random.default_rng(8)
    logits = rng.standard_normal((64, 40)).astype(np.float32)
    bias = rng.uniform(-0.1, 0.1, 40).astype(np.float32)
    idx, w = oracle_lib.gate_topk(logits, bias, 8, oracle_lib.SIGMOID, renormalize=False)
    s = scipy.special.expit(np.take_along_axis(logits, idx, 1).astype(np.float64))
    np.testing.assert_allclose(w, s, rtol=1e-6)
    idx2, w2 = oracle_lib.gate_topk(logits, bias, 8, oracle_lib.SIGMOID)
    assert (idx2 == idx).all()
    np.testing.assert_allclose(w2, s / s.sum(1, keepdims=True), rtol=1e-6)


def test_gate_softmax_bias_rejected(oracle_lib):
    with pytest.raises(ValueError):
        oracle_lib.gate_topk(np.zeros((2, 4), np.float32), np.zeros(4, np.float32), 2,
                             oracle_lib.SOFTMAX)


@pytest.mark.parametrize("case", HAND["gate"], ids=lambda c: c["name"])
def test_gate_hand_cases(oracle_lib, case):
    logits = np.array(case["logits"], dtype=np.float32)
    bias = np.array(case["bias"], dtype=np.float32) if case["bias"] is not None else None
    fn = oracle_lib.SOFTMAX if case["score"] == "softmax" else oracle_lib.SIGMOID
    idx, w = oracle_lib.gate_topk(logits, bias, case["k"], fn)
    assert idx.tolist() == case["idx"]
    want = np.array([[_eval(e) for e in row] for row in case["w"]])
    np.testing.assert_allclose(w, want, rtol=1e-6)


# ---------------------------------------------------------------- route map
@pytest.mark.parametrize("case", HAND["route_map"], ids=lambda c: c["name"])
def test_route_map_hand_cases(oracle_lib, case):
    counts, offsets, slot_of, token_of, rc = oracle_lib.route_map(np.array(case["topk_idx"]),
                                                                  case["E"], case["align"])
    assert rc == 0
    assert counts.tolist() == case["counts"]
    assert offsets.tolist() == case["offsets"]
    assert slot_of.tolist() == case["slot_of"]
    assert token_of.tolist() == case["token_of"]


@pytest.mark.parametrize("T,E,k,align", [(0, 4, 2, 1), (1, 8, 8, 1), (37, 16, 3, 1),
                                         (300, 64, 6, 128), (513, 10, 4, 7)])
def test_route_map_against_stable_argsort(oracle_lib, T, E, k, align):
    rng = np.random.default_rng(T + E)
    # k distinct experts per token, skewed towards low experts so some stay empty
    pri = rng.standard_normal((T, E)) - np.arange(E)[None, :] * 0.3
    idx = np.argsort(-pri, axis=1, kind="stable")[:, :k].astype(np.int32)
    counts, offsets, slot_of, token_of, rc = oracle_lib.route_map(idx, E, align)
    assert rc == 0
    flat = idx.reshape(-1)
    np.testing.assert_array_equal(counts, np.bincount(flat, minlength=E))
    assert counts.sum() == T * k
    padded = -(-counts // align) * align
    np.testing.assert_array_equal(offsets, np.concatenate([[0], np.cumsum(padded)]))
    order = np.argsort(flat, kind="stable")                    # pairs grouped by expert, stable
    sorted_e = flat[order]
    first = np.searchsorted(sorted_e, np.arange(E))
    want_slot = np.empty(T * k, dtype=np.int64)
    want_slot[order] = offsets[sorted_e] + (np.arange(T * k) - first[sorted_e])
    np.testing.assert_array_equal(slot_of.reshape(-1), want_slot)
    rows = np.full(T * k + E * (align - 1), -1)
    rows[want_slot] = np.arange(T * k) // k
    np.testing.assert_array_equal(token_of, rows)
    for e in range(E):  # stability: tokens increase within each segment
        seg = token_of[offsets[e]:offsets[e] + counts[e]]
        assert np.all(np.diff(seg) > 0)


def test_route_map_bad_index(oracle_lib):
    idx = np.array([[0, 5], [1, -1]], dtype=np.int32)
    counts, offsets, slot_of, token_of, rc = oracle_lib.route_map(idx, 4, 1)
    assert rc == 1
    assert counts.tolist() == [1, 1, 0, 0]
    assert slot_of.tolist() == [[0, -1], [1, -1]]


# ---------------------------------------------------------------- expand / reduce
def _bf16_bits(a):
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _bits_to_f32(b):
    return (b.astype(np.uint32) << 16).view(np.float32)


@pytest.mark.parametrize("align", [1, 128])
def test_expand_then_unweighted_reduce_k1_is_identity(oracle_lib, align):
    rng = np.random.default_rng(11)
    T, E, H = 200, 12, 64
    x = _bf16_bits(rng.standard_normal((T, H)))
    x[0, :4] = [0x8000, 0x0000, 0x7F7F, 0x0001]  # -0, +0, big, subnormal
    idx = rng.integers(0, E, (T, 1)).astype(np.int32)
    counts, offsets, slot_of, token_of, _ = oracle_lib.route_map(idx, E, align)
    xe, _ = oracle_lib.expand(x, slot_of, offsets, E, align)
    out = oracle_lib.reduce(xe, slot_of, None)
    # fmaf(1, v, +0) turns -0 into +0; every other value comes back bit for bit
    x_want = x.copy()
    x_want[x_want == 0x8000] = 0
    np.testing.assert_array_equal(out, x_want)
    pad = token_of[:offsets[-1]] == -1
    assert np.all(xe[:offsets[-1]][pad] == 0)


def test_reduce_equal_rows_closed_form(oracle_lib):
    rng = np.random.default_rng(12)
    T, k, H = 50, 8, 128
    v = _bf16_bits(rng.standard_normal((T, H)))
    y = np.repeat(v, k, axis=0)                       # row t*k+j = v[t]
    slot_of = np.arange(T * k, dtype=np.int32).reshape(T, k)
    w = rng.uniform(0.1, 1, (T, k)).astype(np.float32)
    w = (w / w.sum(1, keepdims=True)).astype(np.float32)
    out = _bits_to_f32(oracle_lib.reduce(y, slot_of, w)).astype(np.float64)
    vv = _bits_to_f32(v).astype(np.float64)
    ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(vv), 1e-30))) - 7)
    assert np.all(np.abs(out - vv) <= ulp)


def test_reduce_exact_sum_within_bound(oracle_lib):
    rng = np.random.default_rng(13)
    T, k, H, R = 64, 8, 256, 700
    y = _bf16_bits(rng.standard_normal((R, H)))
    slot_of = np.stack([rng.choice(R, k, replace=False) for _ in range(T)]).astype(np.int32)
    w = rng.uniform(0, 1, (T, k)).astype(np.float32)
    out = _bits_to_f32(oracle_lib.reduce(y, slot_of, w)).astype(np.float64)
    terms = w[:, :, None].astype(np.float64) * _bits_to_f32(y)[slot_of].astype(np.float64)
    exact = terms.sum(1)
    # fp32 accumulation error <= k * 2^-24 * sum|terms|, then one bf16 rounding (2^-8 relative)
    bound = k * 2.0 ** -24 * np.abs(terms).sum(1) + np.abs(exact) * 2.0 ** -8
    assert np.all(np.abs(out - exact) <= bound)
    # one term per slot: moving a weight to the wrong slot breaks this
    out_swapped = _bits_to_f32(oracle_lib.reduce(y, slot_of[:, ::-1].copy(), w)).astype(np.float64)
    assert np.any(np.abs(out_swapped - exact) > bound)


@pytest.mark.parametrize("case", HAND["reduce"], ids=lambda c: c["name"])
def test_reduce_hand_cases(oracle_lib, case):
    y = _bf16_bits(np.array(case["y"], dtype=np.float32))
    out = oracle_lib.reduce_token(y, np.array(case["slot_row"]), np.array(case["w_row"]))
    np.testing.assert_array_equal(_bits_to_f32(out), np.array(case["out"], dtype=np.float32))


def test_reduce_skips_out_of_range_slot(oracle_lib):
    y = _bf16_bits(np.ones((4, 8), np.float32))
    out = oracle_lib.reduce_token(y, np.array([1, 9, -1]), np.array([0.5, 0.25, 0.25]))
    assert np.all(_bits_to_f32(out) == 0.5)


@pytest.mark.parametrize("case", HAND["fp8"], ids=lambda c: c["name"])
def test_fp8_hand_cases(oracle_lib, case):
    H = case["H"]
    x = np.zeros(H, dtype=np.float32)
    x[:len(case["x_first"])] = case["x_first"]
    q, s = oracle_lib.quantize_row_e4m3(_bf16_bits(x))
    assert q[:4].tolist() == case["codes_first"]
    assert np.all(q[4:] == case["rest_code"])
    assert s[0] == np.float32(2.0) / np.float32(448.0)
    assert s[1] == 0.0


def test_fp8_quantisation_properties(oracle_lib):
    _, vals = _e4m3_table()
    rng = np.random.default_rng(14)
    H = 7168
    for scale_in in (1.0, 1e-3, 300.0, 1e-30):
        xf = (rng.standard_normal(H) * scale_in).astype(np.float32)
        xb = _bf16_bits(xf)
        xf = _bits_to_f32(xb).astype(np.float64)
        q, s = oracle_lib.quantize_row_e4m3(xb)
        assert s.shape == (H // 128,)
        mag = vals[q & 0x7F] * np.where(q & 0x80, -1.0, 1.0)
        deq = mag * np.repeat(s.astype(np.float64), 128)
        blocks = xf.reshape(-1, 128)
        amax = np.abs(blocks).max(1)
        np.testing.assert_array_equal(s, (amax.astype(np.float32) / np.float32(448.0)))
        # the block maximum lands on +-448 exactly
        arg = np.abs(blocks).argmax(1)
        assert np.all((q.reshape(-1, 128)[np.arange(H // 128), arg] & 0x7F) == 0x7E)
        # E4M3 keeps 3 mantissa bits: relative error <= 2^-4 for normals, 2^-10*scale absolute
        # in the subnormal range
        tol = np.maximum(np.abs(xf) * 2.0 ** -4, np.repeat(s.astype(np.float64), 128) * 2.0 ** -10)
        assert np.all(np.abs(deq - xf) <= tol * (1 + 1e-6))


def test_fp8_expand_same_codes_in_every_slot(oracle_lib):
    rng = np.random.default_rng(15)
    T, E, k, H, align = 40, 8, 3, 256, 4
    x = _bf16_bits(rng.standard_normal((T, H)))
    pri = rng.standard_normal((T, E))
    idx = np.argsort(-pri, axis=1)[:, :k].astype(np.int32)
    counts, offsets, slot_of, token_of, _ = oracle_lib.route_map(idx, E, align)
    q, s = oracle_lib.expand(x, slot_of, offsets, E, align, oracle_lib.OUT_FP8_E4M3)
    for t in range(T):
        qt, st = oracle_lib.quantize_row_e4m3(x[t])
        for j in range(k):
            np.testing.assert_array_equal(q[slot_of[t, j]], qt)
            np.testing.assert_array_equal(s[slot_of[t, j]], st)
    pad = np.where(token_of[:offsets[-1]] == -1)[0]
    assert np.all(q[pad] == 0) and np.all(s[pad] == 0)


# ---------------------------------------------------------------- load-balance statistics
def test_balance_stats_uniform_scores_closed_form(oracle_lib):
    # equal logits: every normalised score is 1/E, so P = 1/E and loss = sum f / E = 1
    T, E, k = 37, 12, 3
    rng = np.random.default_rng(20)
    counts = np.bincount(rng.integers(0, E, T * k), minlength=E).astype(np.int32)
    for fn in (oracle_lib.SOFTMAX, oracle_lib.SIGMOID):
        P, f, loss = oracle_lib.balance_stats(np.full((T, E), 0.3, np.float32), counts, k, fn)
        np.testing.assert_allclose(P, 1.0 / E, rtol=1e-14)
        np.testing.assert_allclose(f, E * counts / (k * T), rtol=1e-14)
        assert abs(loss - 1.0) < 1e-12


def test_balance_stats_against_library(oracle_lib):
    rng = np.random.default_rng(21)
    T, E, k = 200, 40, 6
    logits = rng.standard_normal((T, E)).astype(np.float32)
    idx, _ = oracle_lib.gate_topk(logits, None, k, oracle_lib.SOFTMAX)
    counts, *_ = oracle_lib.route_map(idx, E, 1)
    P, f, loss = oracle_lib.balance_stats(logits, counts, k, oracle_lib.SOFTMAX)
    p = scipy.special.softmax(logits.astype(np.float64), axis=1)
    np.testing.assert_allclose(P, p.mean(0), rtol=1e-12)
    np.testing.assert_allclose(f, np.bincount(idx.ravel(), minlength=E) * E / (k * T), rtol=1e-14)
    assert abs(loss - float(np.dot(f, P))) < 1e-12
    s = scipy.special.expit(logits.astype(np.float64))
    P2, _, _ = oracle_lib.balance_stats(logits, counts, k, oracle_lib.SIGMOID)
    np.testing.assert_allclose(P2, (s / s.sum(1, keepdims=True)).mean(0), rtol=1e-12)
    assert abs(P2.sum() - 1.0) < 1e-12


def test_balance_stats_all_on_one_expert(oracle_lib):
    # every token routes only to expert 0 with (almost) all of its score: loss -> E
    T, E = 50, 8
    logits = np.full((T, E), -60.0, np.float32)
    logits[:, 0] = 60.0
    counts = np.zeros(E, np.int32)
    counts[0] = T
    P, f, loss = oracle_lib.balance_stats(logits, counts, 1, oracle_lib.SOFTMAX)
    assert f[0] == E and abs(P[0] - 1.0) < 1e-12 and abs(loss - E) < 1e-9


# ---------------------------------------------------------------- tensor-parallel mask
def test_tp_mask_partitions_every_pair(oracle_lib):
    rng = np.random.default_rng(22)
    T, E, k, tp = 90, 24, 4, 3
    idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    owners = np.zeros_like(idx)
    rebuilt = np.full_like(idx, -100)
    for r in range(tp):
        m = oracle_lib.tp_mask(idx, E, tp, r)
        kept = m >= 0
        assert np.all(m[kept] < E // tp)
        owners += kept
        rebuilt[kept] = m[kept] + r * (E // tp)
    assert np.all(owners == 1)            # each pair kept by exactly one rank
    np.testing.assert_array_equal(rebuilt, idx)
    with pytest.raises(ValueError):
        oracle_lib.tp_mask(idx, E, 5, 0)  # E not divisible


def test_masked_pairs_are_skipped_by_the_route_map(oracle_lib):
    idx = np.array([[0, -1], [-1, 2], [1, 0]], dtype=np.int32)
    counts, offsets, slot_of, token_of, rc = oracle_lib.route_map(idx, 3, 1)
    assert rc == 0                        # -1 is a masked pair, not an error
    assert counts.tolist() == [2, 1, 1] and offsets.tolist() == [0, 2, 3, 4]
    assert slot_of.tolist() == [[0, -1], [-1, 3], [2, 1]]


# ---------------------------------------------------------------- reduce backward
def _route(oracle_lib, T, E, k, align, seed):
    rng = np.random.default_rng(seed)
    idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    counts, offsets, slot_of, token_of, _ = oracle_lib.route_map(idx, E, align)
    return idx, offsets, slot_of, token_of


def test_reduce_backward_adjoint_identity(oracle_lib):
    # <g, reduce(y; w)> = sum_tj w_tj * d_w_tj exactly in real arithmetic (reduce is linear in y)
    T, E, k, H = 60, 10, 3, 64
    rng = np.random.default_rng(23)
    _, offsets, slot_of, token_of = _route(oracle_lib, T, E, k, 1, 23)
    R = int(offsets[-1])
    y = _bf16_bits(rng.standard_normal((R, H)))
    g = _bf16_bits(rng.standard_normal((T, H)))
    w = rng.uniform(0, 1, (T, k)).astype(np.float32)
    d_y, d_w, rc = oracle_lib.reduce_backward(g, y, slot_of, offsets, w, E)
    assert rc == 0
    yf = _bits_to_f32(y).astype(np.float64)
    gf = _bits_to_f32(g).astype(np.float64)
    exact_dw = np.einsum("tc,tjc->tj", gf, yf[slot_of])
    np.testing.assert_allclose(d_w, exact_dw.astype(np.float32), rtol=0, atol=0)
    lhs = float(np.sum(gf * np.einsum("tj,tjc->tc", w.astype(np.float64), yf[slot_of])))
    rhs = float(np.sum(w.astype(np.float64) * exact_dw))
    assert abs(lhs - rhs) <= 1e-9 * max(1.0, abs(lhs))
    # d_y rows: w * g rounded to bf16, one row per pair
    for t in range(T):
        for j in range(k):
            want = oracle_lib.bf16_rne((w[t, j] * _bits_to_f32(g[t])).astype(np.float32))
            np.testing.assert_array_equal(d_y[slot_of[t, j]], want)


def test_reduce_backward_unit_weights_and_padding(oracle_lib):
    T, E, k, H, align = 33, 6, 2, 16, 8
    rng = np.random.default_rng(24)
    _, offsets, slot_of, token_of = _route(oracle_lib, T, E, k, align, 24)
    R = int(offsets[-1])
    y = _bf16_bits(rng.standard_normal((tko_rows := T * k + E * (align - 1), H)))
    g = _bf16_bits(rng.standard_normal((T, H)))
    d_y, d_w, rc = oracle_lib.reduce_backward(g, y, slot_of, offsets, None, E)
    for t in range(T):
        for j in range(k):
            np.testing.assert_array_equal(d_y[slot_of[t, j]], g[t])    # weight 1: a copy
    pad = np.where(token_of[:R] == -1)[0]
    assert len(pad) > 0 and np.all(d_y[pad] == 0)
    # the backward of expand is the unweighted reduce: <expand(x), G> = <x, reduce(G)> exactly
    x = _bf16_bits(rng.standard_normal((T, H)))
    xe, _ = oracle_lib.expand(x, slot_of, offsets, E, align)
    G = _bf16_bits(rng.standard_normal((tko_rows, H)))
    back = oracle_lib.reduce(G, slot_of, None)
    Gf = _bits_to_f32(G).astype(np.float64)
    lhs = float(np.sum(_bits_to_f32(xe).astype(np.float64) * Gf))
    rhs_exact = float(np.sum(_bits_to_f32(x).astype(np.float64) * Gf[slot_of].sum(1)))
    assert abs(lhs - rhs_exact) <= 1e-9 * max(1.0, abs(lhs))
    # and the fp32/bf16 reduce of G is that sum rounded (within the reduce's own bound)
    exact = Gf[slot_of].sum(1)
    assert np.all(np.abs(_bits_to_f32(back) - exact) <= k * 2.0 ** -24 * np.abs(Gf[slot_of]).sum(1) + np.abs(exact) * 2.0 ** -8)


# ---------------------------------------------------------------- expert-parallel dispatch / combine
def _ep_choices(rng, T, E, k, masked=0.0):
    idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    if masked:
        idx[rng.random(idx.shape) < masked] = -1
    return idx


def _bf16_bits(a):
    return torch.from_numpy(np.asarray(a, dtype=np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_ep_layout_invariants(oracle_lib):
    # dest_pos >= 0 exactly for the ranks owning one of the token's experts (E/G contiguous
    # experts per rank), numbered 0, 1, 2, ... in token order; counts are the totals.
    rng = np.random.default_rng(31)
    for G, E, k, T in [(1, 8, 3, 20), (2, 8, 3, 50), (4, 16, 5, 64), (8, 64, 8, 40), (3, 12, 12, 9)]:
        idx = _ep_choices(rng, T, E, k, masked=0.2)
        counts, dest = oracle_lib.ep_layout(idx, E, G)
        group = E // G
        for d in range(G):
            goes = np.array([any(e >= 0 and e // group == d for e in row) for row in idx])
            assert np.array_equal(dest[:, d] >= 0, goes)
            assert dest[goes, d].tolist() == list(range(int(goes.sum())))
            assert counts[d] == goes.sum()


def test_ep_layout_masked_and_bad_index(oracle_lib):
    idx = np.array([[-1, -1], [3, -1]], dtype=np.int32)
    counts, dest = oracle_lib.ep_layout(idx, 4, 2)
    assert dest.tolist() == [[-1, -1], [-1, 0]] and counts.tolist() == [0, 1]
    with pytest.raises(ValueError):
        oracle_lib.ep_layout(np.array([[4, 0]], dtype=np.int32), 4, 2)
    with pytest.raises(ValueError):
        oracle_lib.ep_layout(idx, 6, 4)   # E not a multiple of G


def test_ep_recv_bases_hand_case(oracle_lib):
    # rank d receives source 0's rows first, then source 1's, ...: base[s][d] = sum_{s'<s} c[s'][d]
    base, recv = oracle_lib.ep_recv_bases(np.array([[1, 2, 0], [3, 4, 5], [0, 6, 7]]))
    assert base.tolist() == [[0, 0, 0], [1, 2, 0], [4, 6, 5]]
    assert recv.tolist() == [4, 12, 12]


@pytest.mark.parametrize("out_dtype", [0, 1], ids=["bf16", "fp8"])
def test_ep_dispatch_rows_and_local_ids(oracle_lib, out_dtype):
    rng = np.random.default_rng(33)
    G, E, k, T, H = 4, 16, 3, 30, 256
    group = E // G
    xs = [_bf16_bits(rng.standard_normal((T, H))) for _ in range(G)]
    idxs = [_ep_choices(rng, T, E, k, masked=0.1) for _ in range(G)]
    ws = [rng.random((T, k)).astype(np.float32) for _ in range(G)]
    r = oracle_lib.ep_forward(xs, idxs, ws, lambda d, n: np.zeros((n, H), np.uint16), E, G,
                              out_dtype=out_dtype)
    for d in range(G):
        rx, rs, ri, rw = r["recv"][d]
        row = 0
        for s in range(G):
            dest = r["layout"][s][1]
            for t in range(T):
                if dest[t, d] < 0:
                    continue
                if out_dtype == 0:
                    np.testing.assert_array_equal(rx[row], xs[s][t])
                else:
                    q, sc = oracle_lib.quantize_row_e4m3(xs[s][t])
                    np.testing.assert_array_equal(rx[row], q)
                    np.testing.assert_array_equal(rs[row], sc)
                for j in range(k):
                    e = idxs[s][t, j]
                    mine = e >= 0 and e // group == d
                    assert ri[row, j] == (e - d * group if mine else -1)
                    assert rw[row, j] == (ws[s][t, j] if mine else 0.0)
                row += 1
        assert row == r["recv_rows"][d]


def test_ep_combine_rank_order(oracle_lib):
    # fp32 adds in ascending rank order: 2^27 + (-2^27) + 1 = 1; the reverse order gives 0
    H = 8
    parts = [_bf16_bits(np.full((1, H), v)) for v in (2.0 ** 27, -(2.0 ** 27), 1.0)]
    out = oracle_lib.ep_combine(parts, np.zeros(3, np.int64), np.zeros((1, 3), np.int32))
    assert np.all(out == _bf16_bits(np.ones((1, H))))
    # a token no rank received combines to zero
    out = oracle_lib.ep_combine(parts, np.zeros(3, np.int64), np.full((1, 3), -1, np.int32))
    assert np.all(out == 0)


def test_ep_one_rank_is_the_single_rank_path(oracle_lib):
    rng = np.random.default_rng(35)
    E, k, T, H = 12, 4, 40, 64
    x = _bf16_bits(rng.standard_normal((T, H)))
    idx = _ep_choices(rng, T, E, k)
    w = rng.random((T, k)).astype(np.float32)
    ys = {}

    def make_y(d, n):
        ys[d] = _bf16_bits(rng.standard_normal((n, H)))
        return ys[d]

    r = oracle_lib.ep_forward([x], [idx], [w], make_y, E, 1)
    np.testing.assert_array_equal(r["recv"][0][0], x)
    counts, offsets, slot_of, token_of, _ = oracle_lib.route_map(idx, E, 1)
    np.testing.assert_array_equal(r["out"][0], oracle_lib.reduce(ys[0], slot_of, w))


def test_ep_tokens_on_one_rank_match_that_ranks_reduce(oracle_lib):
    rng = np.random.default_rng(36)
    G, E, k, T, H = 4, 32, 4, 25, 40
    group = E // G
    idxs = []
    for _ in range(G):
        home = rng.integers(0, G, T)
        idxs.append(np.stack([home[t] * group + rng.choice(group, k, replace=False)
                              for t in range(T)]).astype(np.int32))
    xs = [_bf16_bits(rng.standard_normal((T, H))) for _ in range(G)]
    ws = [rng.random((T, k)).astype(np.float32) for _ in range(G)]
    r = oracle_lib.ep_forward(xs, idxs, ws, lambda d, n: _bf16_bits(rng.standard_normal((n, H))),
                              E, G)
    for s in range(G):
        dest = r["layout"][s][1]
        for t in range(T):
            (d,) = np.nonzero(dest[t] >= 0)[0]
            row = r["base"][s, d] + dest[t, d]
            D = r["dest"][d]
            want = oracle_lib.reduce_token(D["y"], D["slot_of"][row], ws[s][t])
            np.testing.assert_array_equal(r["out"][s][t], want)


def test_ep_closed_form_equal_rows(oracle_lib):
    # every expert output row is v and every weight 1/4: rank d's partial is (n_d/4) v exactly,
    # and the partials of a token add up to v exactly, whatever the split over ranks
    rng = np.random.default_rng(37)
    G, E, k, T, H = 4, 16, 4, 30, 16
    v = _bf16_bits(rng.integers(-64, 64, H) / 8.0)
    xs = [_bf16_bits(rng.standard_normal((T, H))) for _ in range(G)]
    idxs = [_ep_choices(rng, T, E, k) for _ in range(G)]
    ws = [np.full((T, k), 0.25, np.float32) for _ in range(G)]
    r = oracle_lib.ep_forward(xs, idxs, ws, lambda d, n: np.tile(v, (n, 1)), E, G)
    for s in range(G):
        assert np.all(r["out"][s] == v[None, :])


@pytest.mark.parametrize("case", HAND["ep"], ids=lambda c: c["name"])
def test_ep_hand_case(oracle_lib, case):
    E, G, H = case["E"], case["G"], case["H"]
    idxs = [np.array(s["idx"], dtype=np.int32) for s in case["sources"]]
    ws = [np.array(s["w"], dtype=np.float32) for s in case["sources"]]
    xs = [_bf16_bits(np.full((len(s["idx"]), H), 1.0)) for s in case["sources"]]
    ys = [np.asarray(r, dtype=np.float64) for r in case["y_rows"]]

    def make_y(d, rows):
        y = np.zeros((rows, H))
        y[:len(ys[d])] = ys[d][:, None]
        return _bf16_bits(y)

    r = oracle_lib.ep_forward(xs, idxs, ws, make_y, E, G)
    assert r["count_matrix"].tolist() == case["send_counts"]
    assert [lay[1].tolist() for lay in r["layout"]] == case["dest_pos"]
    assert r["base"].tolist() == case["base"] and r["recv_rows"].tolist() == case["recv_rows"]
    for d in range(G):
        assert r["recv"][d][2].tolist() == case["recv_idx"][d]
        assert r["recv"][d][3].tolist() == case["recv_w"][d]
        assert r["dest"][d]["offsets"].tolist() == case["dest_offsets"][d]
    for s, want in enumerate(case["out"]):
        np.testing.assert_array_equal(r["out"][s], _bf16_bits(np.repeat(np.array(want)[:, None], H, 1)))
