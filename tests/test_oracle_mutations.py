"""Mutation test of the oracle's pins: each planted mistake (a dropped series term, the wrong
tie-break, biased weights, an off-by-one padding, unstable slots, the wrong E4M3 rounding or
scale, the wrong reduction order, truncating bf16 rounding, a missing factor in the balance
loss, a weighted gradient, an un-renumbered TP mask, the expert-parallel combine in the wrong
rank order, experts dealt round-robin over ranks, global expert ids sent, inclusive receive
bases, skipped renormalisation, padding rows naming token 0, an inclusive TP-group bound, an
epsilon guard in place of the zero scale of an all-zero FP8 block, a gradient weight rounded to
bf16 first) is compiled into a copy of the oracle,
and the pins that cover that step must fail against it. The unplanted build must pass them."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PINS = os.path.join(ROOT, "tests", "test_oracle_pins.py")

# planted mistake -> pytest -k expression selecting the pins that cover the mutated step
MUTATIONS = {
    1: "spec_exp or spec_sigmoid",
    2: "gate_brute_force or gate_hand_cases",
    3: "sigmoid_weights_library or gate_hand_cases",
    4: "route_map",
    5: "route_map",
    6: "e4m3",
    7: "fp8",
    8: "reduce_exact_sum or reduce_hand or reduce_equal_rows",
    9: "bf16_rne",
    10: "balance_stats",
    11: "reduce_backward",
    12: "tp_mask",
    13: "ep_combine_rank_order",
    14: "ep_layout or ep_dispatch",
    15: "ep_dispatch",
    16: "ep_recv_bases or ep_hand_case",
    17: "gate_softmax_weights_library or sigmoid_weights_library or gate_all_equal",
    18: "route_map",
    19: "tp_mask",
    20: "fp8",
    21: "reduce_backward",
}


def _run_pins(lib_path, expr):
    env = dict(os.environ, TKO_LIB=lib_path)
    r = subprocess.run([sys.executable, "-m", "pytest", PINS, "-q", "-x", "-p", "no:cacheprovider",
                        "-k", expr], cwd=ROOT, env=env, capture_output=True, text=True)
    return r.returncode, r.stdout[-800:]


@pytest.fixture(scope="module")
def variants(tmp_path_factory):
    from concurrent.futures import ThreadPoolExecutor

    from oracle.build import build_variant

    d = tmp_path_factory.mktemp("oracle_variants")
    plants = [0] + sorted(MUTATIONS)
    with ThreadPoolExecutor(8) as ex:
        paths = list(ex.map(lambda n: build_variant(n, str(d / f"libtko_plant{n}.so")), plants))
    return dict(zip(plants, paths))


def test_unplanted_build_passes_every_selected_pin(variants):
    expr = " or ".join(f"({e})" for e in MUTATIONS.values())
    rc, out = _run_pins(variants[0], expr)
    assert rc == 0, out


@pytest.mark.parametrize("plant", sorted(MUTATIONS))
def test_planted_mistake_is_caught(variants, plant):
    rc, out = _run_pins(variants[plant], MUTATIONS[plant])
    assert rc == 1, f"planted mistake {plant} slipped past the pins:\n{out}"
