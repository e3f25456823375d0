"""Seeded random configurations of the whole path against the oracle, compared in full (the same
checks as the edge cases): expert counts on and off the warp grid up to 1024, k up to 32 and
up to E, batches from empty to several tokens per gate warp, every alignment the route map
takes, both scores with and without a selection bias, both renormalisation modes, and bf16 or
E4M3 expansion. The configurations are drawn once from a fixed seed, so a failure names a
reproducible case."""
import numpy as np
import pytest

from test_gpu_edges import _case, _full_check, _rand_inputs

pytestmark = pytest.mark.gpu


def _configs(n=48, seed=2026):
    rng = np.random.default_rng(seed)
    out = []
    while len(out) < n:
        E = int(rng.choice([1, 2, 7, 16, 31, 32, 33, 64, 96, 100, 128, 200, 256, 300, 512, 777, 1024]))
        k = int(rng.integers(1, min(E, 32) + 1))
        T = int(rng.choice([0, 1, int(rng.integers(2, 600)), int(rng.integers(600, 5000)),
                            int(rng.integers(9000, 14000))], p=[0.05, 0.1, 0.35, 0.3, 0.2]))
        fp8 = bool(rng.random() < 0.3)
        H = int(rng.choice([128, 256, 1024, 2048])) if fp8 else int(8 * rng.integers(1, 257))
        if T * k * H > 40_000_000:  # keep each case to about a second of oracle time
            continue
        score = str(rng.choice(["softmax", "sigmoid"]))
        bias = score == "sigmoid" and bool(rng.random() < 0.7)
        align = int(rng.choice([1, 1, 2, 4, 7, 16, 128]))
        renorm = bool(rng.random() < 0.8)
        out.append((T, E, k, H, score, bias, align, "fp8" if fp8 else "bf16", renorm))
    return out


@pytest.mark.parametrize("T,E,k,H,score,bias,align,out,renorm", _configs(),
                         ids=lambda v: str(v))
def test_random_configuration(T, E, k, H, score, bias, align, out, renorm):
    wl = _case(T, E, k, H, score, bias, align, out, seed=T + 7 * E + k)
    _full_check(wl, *_rand_inputs(wl, np.random.default_rng(T * 31 + E * 7 + k)), renormalize=renorm)
