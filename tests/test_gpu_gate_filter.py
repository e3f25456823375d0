"""The gate's candidate filter against the oracle ("DeepSeek 的 GPU 内核帝国", section "MoE TopK
门控": select the k largest keys, equal keys to the lower index).

The kernel ranks cheap approximate keys first and computes exact keys only for the experts
that can still be among the k largest (all within a proven margin of the k-th); a token with
more than 32 such experts, or a non-finite or huge bias, takes the full path over every exact
key. These cases put many experts inside the margin -- clusters of near-equal keys straddling
the k-th, below and above 32 candidates -- and push the margin with large biases, non-finite
values and extreme logits. Indices must equal the oracle's bit for bit, weights within 1e-6
relative where the oracle's weights are finite."""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import assert_weights_close
from token_routing_gate_b200 import tk

pytestmark = pytest.mark.gpu


def _check(logits, bias, k, score="sigmoid", renormalize=True):
    logits = np.ascontiguousarray(logits, np.float32)
    b = None if bias is None else np.ascontiguousarray(bias, np.float32)
    idx, w = tk.gate_topk(torch.from_numpy(logits).cuda(), k, score,
                          None if b is None else torch.from_numpy(b).cuda(), renormalize)
    torch.cuda.synchronize()
    fn = oracle.SOFTMAX if score == "softmax" else oracle.SIGMOID
    o_idx, o_w = oracle.gate_topk(logits, b, k, fn, renormalize)
    got = idx.cpu().numpy()
    bad = (got != o_idx).any(axis=1)
    assert not bad.any(), f"{bad.sum()} tokens differ, first {np.flatnonzero(bad)[:5]}"
    # weights of the tokens whose oracle weights are finite (non-finite logits leave them open)
    fin = np.isfinite(o_w).all(axis=1)
    assert_weights_close(w.cpu().numpy()[fin], o_w[fin])
    return got


def _clusters(T, E, rng, spread, with_bias):
    """Per token: a cluster of c ~ U{2..48} experts whose logits lie within `spread` of a common
    centre (so their keys are within the filter's margin of one another), placed so that the
    k-th key falls inside it; the other experts sit clearly above (a few) or below."""
    logits = rng.normal(-3.0, 0.5, (T, E)).astype(np.float32)
    for t in range(T):
        c = int(rng.integers(2, 49))
        above = int(rng.integers(0, 6))
        members = rng.choice(E, c + above, replace=False)
        centre = rng.uniform(-1.0, 1.5)
        logits[t, members[:c]] = centre + rng.uniform(-spread, spread, c)
        logits[t, members[c:]] = centre + rng.uniform(2.0, 4.0, above)
        if rng.random() < 0.3:                    # exact ties inside the cluster
            tie = members[:c][: max(2, c // 3)]
            logits[t, tie] = logits[t, tie[0]]
    bias = rng.uniform(-1e-4, 1e-4, E).astype(np.float32) if with_bias else None
    return logits, bias


@pytest.mark.parametrize("with_bias", [True, False])
@pytest.mark.parametrize("E,k", [(256, 8), (64, 6), (300, 12), (1024, 32)])
def test_clusters_inside_the_margin(E, k, with_bias):
    rng = np.random.default_rng(E * 100 + k + with_bias)
    logits, bias = _clusters(1500, E, rng, 3e-4, with_bias)
    _check(logits, bias, k)


def test_clusters_with_one_ulp_spacing():
    """Cluster members one or a few fp32 ulps apart in the logit (no bias: the key is the
    logit, margin 0)."""
    rng = np.random.default_rng(11)
    T, E, k = 2000, 256, 8
    logits = rng.normal(-3.0, 0.5, (T, E)).astype(np.float32)
    for t in range(T):
        c = int(rng.integers(2, 40))
        members = rng.choice(E, c, replace=False)
        v = np.float32(rng.uniform(0.5, 2.0))
        for m in members:
            logits[t, m] = v
            v = np.nextafter(v, np.float32(np.inf)) if rng.random() < 0.7 else v
    _check(logits, None, k)


@pytest.mark.parametrize("scale", [1.0, 30.0, 1000.0, 5e5, 3e6])
def test_bias_magnitudes(scale):
    """The margin grows with max|b|; at 2^20 and beyond the kernel takes the full path."""
    rng = np.random.default_rng(int(scale) % 1000 + 3)
    T, E, k = 1024, 256, 8
    logits = rng.standard_normal((T, E)).astype(np.float32)
    bias = rng.uniform(-scale, scale, E).astype(np.float32)
    # a group of experts whose biases are equal makes their order depend on the sigmoid alone
    bias[:40] = bias[0]
    _check(logits, bias, k)


@pytest.mark.parametrize("bad", [np.inf, -np.inf, np.nan])
def test_non_finite_bias(bad):
    rng = np.random.default_rng(5)
    T, E, k = 300, 96, 6
    logits = rng.standard_normal((T, E)).astype(np.float32)
    bias = rng.uniform(-0.1, 0.1, E).astype(np.float32)
    bias[[3, 50]] = bad
    _check(logits, bias, k)


@pytest.mark.parametrize("with_bias", [True, False])
def test_extreme_and_non_finite_logits(with_bias):
    rng = np.random.default_rng(6 + with_bias)
    T, E, k = 2000, 256, 8
    logits = rng.standard_normal((T, E)).astype(np.float32) * rng.choice(
        [1.0, 30.0, 90.0, 120.0, 1e4, 1e30], size=(T, 1)).astype(np.float32)
    special = rng.random((T, E))
    logits[special < 0.01] = np.inf
    logits[(special >= 0.01) & (special < 0.02)] = -np.inf
    logits[(special >= 0.02) & (special < 0.03)] = np.nan
    logits[:20] = np.nan                              # tokens with nothing but NaN
    logits[20:40] = -np.inf
    logits[40:60, :] = np.inf
    bias = rng.uniform(-0.1, 0.1, E).astype(np.float32) if with_bias else None
    _check(logits, bias, k)


@pytest.mark.parametrize("E", [1, 2, 31, 33, 63, 65, 129, 255])
def test_expert_counts_off_the_lane_grid(E):
    rng = np.random.default_rng(E)
    for k in sorted({1, min(E, 2), min(E, 8), E if E <= 32 else 32}):
        logits = rng.standard_normal((257, E)).astype(np.float32)
        bias = rng.uniform(-0.1, 0.1, E).astype(np.float32)
        _check(logits, bias, k)
        _check(logits, None, k, "softmax")


def test_approximate_sigmoid_within_the_filter_bound():
    """Exhaustively over every finite fp32 logit with |l| <= 128: the filter's approximate
    logistic value (ex2.approx / rcp.approx) stays within 2^-17 of the selection key's exact
    fp32 sigmoid -- the bound its 2^-12 margin is built on. Beyond 128 both are 0 or 1."""
    err = tk.selftest_gate_margin()
    torch.cuda.synchronize()
    worst = float(err.item())
    print(f"largest |approximate - exact| logistic value: {worst:.3e} ({np.log2(worst):.2f} in log2)")
    assert worst < 2.0 ** -17


@pytest.mark.parametrize("score", ["softmax", "sigmoid"])
def test_candidate_keys_spanning_many_binades(score):
    """Candidate keys that lie many binades apart (their integer images further apart than the
    one-reduction rounds can pack), so the selection takes the two-reduction rounds; half the
    tokens stay in one binade as a control."""
    rng = np.random.default_rng(21 + (score == "sigmoid"))
    T, E, k = 3000, 256, 8
    logits = (rng.standard_normal((T, E)) - 6.0).astype(np.float32)
    bias = None
    if score == "softmax":
        for t in range(0, T, 2):  # top 12 logits 4^j: 1 ... 4^11, spread over 22 binades
            logits[t, rng.choice(E, 12, replace=False)] = 4.0 ** np.arange(12)
    else:
        bias = np.zeros(E, np.float32)
        top = rng.choice(E, 12, replace=False)
        bias[top] = 10.0 ** np.linspace(-2.0, 5.0, 12)  # keys from about 0.01 to 1e5
        logits[1::2, top] = 4.0                          # the control tokens: sigmoid ~ 1 everywhere
    _check(logits, bias, k, score)


@pytest.mark.parametrize("score", ["sigmoid", "softmax"])
@pytest.mark.parametrize("renormalize", [True, False])
@pytest.mark.parametrize("k", [8, 6, 5, 3])
def test_weight_batches_with_full_path_tokens(k, renormalize, score):
    """Enough tokens that each warp routes several and computes their weights together (32/k
    tokens per pass; logistic scores, or softmax when renormalised), with every third token sent
    down the full path (40 equal top keys) in the middle of a batch. Plain softmax writes each
    token's weights from the whole row."""
    rng = np.random.default_rng(40 + k + renormalize + 10 * (score == "softmax"))
    T, E = 20000, 256
    logits = rng.standard_normal((T, E)).astype(np.float32)
    tied = rng.choice(E, 40, replace=False)
    bias = None
    if score == "sigmoid":
        bias = rng.uniform(-0.1, 0.1, E).astype(np.float32)
        bias[tied] = 0.05
    logits[::3, :] -= 4.0
    logits[::3][:, tied] = 3.0
    _check(logits, bias, k, score, renormalize)
