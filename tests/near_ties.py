"""Adversarial gate inputs: selection keys planted one fp32 ulp apart.

With sigmoid scoring and a selection bias the key of expert e is the fp32 value
sigmoid(l_e) + b_e ("DeepSeek 的 GPU 内核帝国", section "MoE TopK 门控": k rounds of max with
a 'min' index reducer; the key's exponential is fixed so that both sides of a comparison get
the same bits). A near-tie between two keys is decided by their last bit, so an exponential
that is off by one ulp on either side flips the selection there. This module builds logits
whose keys, computed with the oracle's pinned sigmoid and IEEE fp32 addition, form a descending
ladder per token with three planted pairs at ranks (2,3), (5,6) and (8,9) (1-based): the
second key of each pair is the first key's fp32 neighbour above or below it, or equal to it.
The (8,9) pair sits on the k = 8 boundary, so it decides which experts are selected; the other
two decide the order of the selected ones.

Only the construction lives here; every expected value in the tests comes from the oracle's
gate on these logits.
"""
import numpy as np

import oracle

PAIR_RANKS = ((1, 2), (4, 5), (7, 8))   # 0-based ladder positions of the planted pairs
LADDER = 9


def keys_of(logits, bias):
    """Selection keys fl(sigmoid(l) + b) in fp32 (numpy's float32 add rounds to nearest even)."""
    s = oracle.spec_sigmoidf(logits).reshape(np.shape(logits))
    return (s.astype(np.float32) + np.asarray(bias, np.float32)).astype(np.float32)


def _logit(p):
    p = np.clip(p, 1e-6, 1 - 1e-6)
    return np.log(p / (1.0 - p))


def _solve_logit(target_key, b):
    """For each row, an fp32 logit whose key fl(sigmoid(l) + b) equals target_key exactly, or
    NaN when none is found. Scans a grid of candidates around the real solution whose step is
    a quarter of a key ulp divided by the sigmoid's slope, so consecutive candidates change the
    key by less than an ulp and the grid cannot step over the target."""
    target_key = np.asarray(target_key, np.float32)
    s_star = np.clip(target_key.astype(np.float64) - b.astype(np.float64), 1e-6, 1 - 1e-6)
    l_star = _logit(s_star)
    slope = np.maximum(s_star * (1.0 - s_star), 1e-9)
    kulp = np.spacing(np.abs(target_key)).astype(np.float64)
    step = kulp / (4.0 * slope)
    W = 96
    offs = np.arange(W, dtype=np.float64) - W // 2
    cand = (l_star[:, None] + offs[None, :] * step[:, None]).astype(np.float32)
    keys = keys_of(cand, np.broadcast_to(b[:, None], cand.shape))
    hit = keys == target_key[:, None]
    found = hit.any(axis=1)
    first = np.argmax(hit, axis=1)
    out = np.where(found, cand[np.arange(len(cand)), first], np.float32(np.nan))
    return out.astype(np.float32)


def _step_ulps(k, n):
    """k moved n fp32 ulps (n may be negative)."""
    k = np.asarray(k, np.float32).copy()
    for _ in range(abs(int(n))):
        k = np.nextafter(k, np.float32(np.inf if n > 0 else -np.inf))
    return k


# offsets (in key ulps) tried in turn for each requested relation: where the sigmoid's value
# lies in a coarser binade than the key (s >= 1/2 > key), only every second key is reachable,
# so the nearest reachable neighbour is two ulps away
_TRIES = {-1: (-1, -2), 0: (0, 1, -1), 1: (1, 2)}


def planted_logits(T, E, bias, seed):
    """(logits fp32 [T,E], pairs int [T,3,2] of planted expert pairs, offset int [T,3]: the
    second key of the pair minus the first, in fp32 ulps -- one of -2, -1, 0, 1, 2 -- or 99
    where no logit reaching a neighbouring key was found; that pair is left unplanted).

    Ladder: a top key u ~ U(0.40, 0.88) per token and descending steps of U(0.005, 0.025);
    the ladder's experts are a random choice of 9; all other experts get logits U(-10, -4)
    (keys below 0.12, under the ladder's lowest key, which stays above 0.2)."""
    assert E >= LADDER + 1
    rng = np.random.default_rng(seed)
    bias = np.asarray(bias, np.float32)
    logits = rng.uniform(-10.0, -4.0, size=(T, E)).astype(np.float32)
    perm = np.argsort(rng.random((T, E)), axis=1)[:, :LADDER]
    u = rng.uniform(0.40, 0.88, size=T)
    steps = rng.uniform(0.005, 0.025, size=(T, LADDER))
    steps[:, 0] = 0.0
    targets = u[:, None] - np.cumsum(steps, axis=1)
    rows = np.arange(T)
    for pos in range(LADDER):
        e = perm[:, pos]
        logits[rows, e] = _logit(targets[:, pos] - bias[e]).astype(np.float32)
    want = rng.choice([-1, 0, 1], size=(T, len(PAIR_RANKS)), p=[0.4, 0.2, 0.4])
    pairs = np.zeros((T, len(PAIR_RANKS), 2), dtype=np.int64)
    offset = np.full((T, len(PAIR_RANKS)), 99, dtype=np.int64)
    for i, (pa, pb) in enumerate(PAIR_RANKS):
        ea, eb = perm[:, pa], perm[:, pb]
        pairs[:, i, 0], pairs[:, i, 1] = ea, eb
        ka = keys_of(logits[rows, ea], bias[ea])
        for rel, tries in _TRIES.items():
            sel = np.flatnonzero(want[:, i] == rel)
            for n in tries:
                if sel.size == 0:
                    break
                lb = _solve_logit(_step_ulps(ka[sel], n), bias[eb[sel]])
                hit = ~np.isnan(lb)
                logits[rows[sel[hit]], eb[sel[hit]]] = lb[hit]
                offset[sel[hit], i] = n
                sel = sel[~hit]
    return logits, pairs, offset


def ulp_gap(a, b):
    """Distance in fp32 ulps between finite fp32 arrays a and b (order-preserving integer map)."""
    def ordered(x):
        i = np.asarray(x, np.float32).view(np.int32).astype(np.int64)
        return np.where(i < 0, -(i & 0x7FFFFFFF), i)
    return np.abs(ordered(a) - ordered(b))


def boundary_gaps(logits, bias, k):
    """Per token, the gap in ulps between the k-th and (k+1)-th largest selection key (the
    margin that decides the selected set)."""
    keys = keys_of(logits, np.broadcast_to(np.asarray(bias, np.float32), logits.shape))
    keys = np.where(np.isnan(keys), np.float32(-np.inf), keys)
    top = -np.sort(-keys, axis=1)[:, k - 1:k + 1]
    return ulp_gap(top[:, 0], top[:, 1])
