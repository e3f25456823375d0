"""tk_route_map_static: the allocation-free form of the route map, for callers that cannot
allocate device memory (an engine or plugin host that owns all device memory and hands over only
inputs and outputs, or a latency-critical loop that must not call cudaMalloc). It must give the
same results as tk_route_map with a caller workspace. Called twice in a row with different
problems, so the second call runs on whatever the first one left in the shared built-in buffer.
This file is collected last on purpose."""
import ctypes

import pytest
import torch

from token_routing_gate_b200 import tk
from token_routing_gate_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _static_route_map(idx, E, align):
    T, k = idx.shape
    dev = idx.device
    rows = max(tk.max_rows(T, E, k, align), 1)
    # outputs start as garbage so that nothing passes by accident
    counts = torch.full((E,), -7, dtype=torch.int32, device=dev)
    offsets = torch.full((E + 1,), -7, dtype=torch.int32, device=dev)
    slot_of = torch.full((T, k), -7, dtype=torch.int32, device=dev)
    token_of = torch.full((rows,), -7, dtype=torch.int32, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = tk.lib.tk_route_map_static(tk._ptr(idx), T, E, k, align, tk._ptr(counts), tk._ptr(offsets),
                                    tk._ptr(slot_of), tk._ptr(token_of), tk._ptr(err), stream)
    assert rc == 0, tk.lib.tk_last_error_detail().decode()
    return counts, offsets, slot_of, token_of, err


CASES = [
    W.V3,                                                   # T=8192, E=256, k=8, sigmoid + bias
    W.MID.with_(T=300, align=128, seed=77),                 # ragged T, padded segments
]


def test_static_route_map_matches_workspace_version_twice_in_a_row():
    for wl in CASES:  # two calls of the static entry point, one after the other
        logits, bias = W.gate_inputs(wl, "cuda")
        idx, _ = tk.gate_topk(logits, wl.k, wl.score, bias)
        ref = tk.route_map(idx, wl.E, wl.align)
        counts, offsets, slot_of, token_of, err = _static_route_map(idx, wl.E, wl.align)
        torch.cuda.synchronize()
        assert err.item() == 0
        assert torch.equal(counts, ref.counts)
        assert torch.equal(offsets, ref.offsets)
        assert torch.equal(slot_of, ref.slot_of)
        assert torch.equal(token_of, ref.token_of)


def test_static_route_map_rejects_sizes_beyond_its_buffer():
    fake = ctypes.c_void_p(0x10000)  # never touched: the call stops at the size check
    T, E, k = 300_000, 256, 8         # ceil(300000/256) * 256 > 262144 entries
    rc = tk.lib.tk_route_map_static(fake, T, E, k, 1, fake, fake, fake, fake, None, None)
    assert rc == 1
    assert "built-in buffer" in tk.lib.tk_last_error_detail().decode()
