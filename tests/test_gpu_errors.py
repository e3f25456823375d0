"""Device-detected data errors: invalid indices and slots are skipped (no memory access outside
any buffer) and reported through the error flag; the rest of the output still matches the
oracle, which skips the same elements. Host-side argument errors raise before any launch."""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import bf16_bits, bf16_ulp_diff
from token_routing_gate_b200 import tk

pytestmark = pytest.mark.gpu


def test_out_of_range_experts_are_skipped_and_flagged():
    T, E, k = 300, 16, 3
    rng = np.random.default_rng(0)
    idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    idx[5, 1] = -3
    idx[77, 0] = E + 5
    idx[299, 2] = 1 << 30
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    rm = tk.route_map(torch.as_tensor(idx, device="cuda"), E, 1, err_flag=err)
    torch.cuda.synchronize()
    assert err.item() & tk.DEVERR_EXPERT_RANGE
    counts, offsets, slot_of, token_of, rc = oracle.route_map(idx, E, 1)
    assert rc == 1
    np.testing.assert_array_equal(rm.counts.cpu().numpy(), counts)
    np.testing.assert_array_equal(rm.offsets.cpu().numpy(), offsets)
    np.testing.assert_array_equal(rm.slot_of.cpu().numpy(), slot_of)
    np.testing.assert_array_equal(rm.token_of.cpu().numpy(), token_of)
    # expand and reduce skip the pairs whose slot is -1 without flagging them again
    err.zero_()
    x = torch.randn(T, 64, device="cuda").to(torch.bfloat16)
    xe = tk.expand(x, rm, E, k, err_flag=err)
    w = torch.rand(T, k, device="cuda")
    out = tk.reduce(xe, rm.slot_of, w, err_flag=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    R = int(offsets[-1])
    xe_ref, _ = oracle.expand(bf16_bits(x), slot_of, offsets, E, 1)
    np.testing.assert_array_equal(bf16_bits(xe)[:R], xe_ref[:R])
    ref = oracle.reduce(bf16_bits(xe), slot_of, w.cpu().numpy())
    np.testing.assert_array_equal(bf16_bits(out), ref)


def test_duplicate_expert_is_flagged_and_stays_in_bounds():
    T, E, k = 50, 8, 2
    idx = np.tile(np.array([[0, 1]], np.int32), (T, 1))
    idx[10] = [3, 3]
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    rm = tk.route_map(torch.as_tensor(idx, device="cuda"), E, 1, err_flag=err)
    torch.cuda.synchronize()
    assert err.item() & tk.DEVERR_DUP_EXPERT
    slots = rm.slot_of.cpu().numpy()
    assert slots.min() >= 0 and slots.max() < T * k


def test_reduce_skips_slots_outside_y():
    T, k, H, rows = 64, 4, 256, 100
    rng = np.random.default_rng(1)
    slot_of = rng.integers(0, rows, (T, k)).astype(np.int32)
    slot_of[3, 2] = rows            # one past the end
    slot_of[9, 0] = 1 << 29
    slot_of[20, 3] = -7
    y = torch.randn(rows, H, device="cuda").to(torch.bfloat16)
    w = torch.rand(T, k, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = tk.reduce(y, torch.as_tensor(slot_of, device="cuda"), w, err_flag=err)
    torch.cuda.synchronize()
    assert err.item() & tk.DEVERR_SLOT_RANGE
    ref = oracle.reduce(bf16_bits(y), slot_of, w.cpu().numpy())
    assert bf16_ulp_diff(bf16_bits(out), ref).max() == 0


def test_expand_skips_slots_outside_buffer():
    T, E, k, H = 32, 4, 2, 64
    idx = np.tile(np.array([[0, 1]], np.int32), (T, 1))
    rm = tk.route_map(torch.as_tensor(idx, device="cuda"), E, 1)
    torch.cuda.synchronize()
    bad = rm.slot_of.clone()
    bad[4, 1] = T * k + 10          # beyond the worst-case row count
    rm.slot_of = bad
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    x = torch.randn(T, H, device="cuda").to(torch.bfloat16)
    xe = torch.zeros(T * k, H, dtype=torch.bfloat16, device="cuda")
    tk.expand(x, rm, E, k, out=xe, err_flag=err)
    torch.cuda.synchronize()
    assert err.item() & tk.DEVERR_SLOT_RANGE
    s = bad.cpu().numpy()
    for t in range(T):
        for j in range(k):
            if s[t, j] < T * k:
                assert torch.equal(xe[s[t, j]], x[t])


def test_host_errors_raise_before_launch():
    x = torch.zeros(4, 12, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(tk.TkError, match="H=12"):
        tk.reduce(x, torch.zeros(4, 2, dtype=torch.int32, device="cuda"))
    with pytest.raises(tk.TkError, match="bias"):
        tk.gate_topk(torch.zeros(4, 8, device="cuda"), 2, "softmax", torch.zeros(8, device="cuda"))


def test_bounded_wait_gives_up_and_the_context_stays_usable():
    import time
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    t0 = time.perf_counter()
    tk.selftest_bounded_wait(20_000_000, err)          # 20 ms on a barrier nothing completes
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    assert err.item() == tk.DEVERR_TIMEOUT
    assert 0.015 < dt < 5.0
    # the context still works: a full routing step right after
    x = torch.randn(64, 256, device="cuda").to(torch.bfloat16)
    idx, w = tk.gate_topk(torch.randn(64, 16, device="cuda"), 2, "sigmoid")
    rm = tk.route_map(idx, 16)
    out = tk.reduce(tk.expand(x, rm, 16, 2), rm.slot_of, None)
    torch.cuda.synchronize()
    assert torch.equal(out.float(), (2 * x.float()).to(torch.bfloat16).float())
