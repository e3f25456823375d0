"""tk_route_map_static: the allocation-free form of the route map, for callers that cannot
allocate device memory (an engine or plugin host that owns all device memory and hands over only
inputs and outputs, or a latency-critical loop that must not call cudaMalloc). It must give the
same results as tk_route_map with a caller workspace, and as the oracle's route map. Called
several times in a row with different problems (among them an empty batch and the largest size
the built-in buffer takes), so each call runs on whatever the previous one left in the shared
buffer.
This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
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
    W.V3.with_(T=0, align=4),                               # empty batch: only the -1 fill
    # the largest size the built-in buffer takes: 512 tiles of 128 tokens * 1024 = 524288 entries, and
    # E = 1024 puts all 1024 threads of the scan kernel to work
    W.MID.with_(T=65536, E=1024, k=1, score="sigmoid", seed=78),
]


def _routed(wl):
    if wl.T == 0:
        return torch.empty((0, wl.k), dtype=torch.int32, device="cuda")
    logits, bias = W.gate_inputs(wl, "cuda")
    idx, _ = tk.gate_topk(logits, wl.k, wl.score, bias)
    return idx


def test_static_route_map_matches_workspace_version_and_oracle():
    for wl in CASES:  # calls of the static entry point one after the other, sizes changing
        idx = _routed(wl)
        ref = tk.route_map(idx, wl.E, wl.align)
        counts, offsets, slot_of, token_of, err = _static_route_map(idx, wl.E, wl.align)
        torch.cuda.synchronize()
        assert err.item() == 0, wl
        assert torch.equal(counts, ref.counts), wl
        assert torch.equal(offsets, ref.offsets), wl
        assert torch.equal(slot_of, ref.slot_of), wl
        assert torch.equal(token_of[:ref.token_of.numel()], ref.token_of), wl
        o_counts, o_offsets, o_slot, o_token, rc = oracle.route_map(idx.cpu().numpy(), wl.E, wl.align)
        assert rc == 0
        np.testing.assert_array_equal(counts.cpu().numpy(), o_counts)
        np.testing.assert_array_equal(offsets.cpu().numpy(), o_offsets)
        np.testing.assert_array_equal(slot_of.cpu().numpy(), o_slot)
        np.testing.assert_array_equal(token_of.cpu().numpy()[:o_token.size], o_token)


@pytest.mark.parametrize("T,E,k", [(300_000, 256, 8),   # 2344 tiles of 128 tokens * 256 > 524288
                                   (65_537, 1024, 1)])  # one tile past the largest accepted size
def test_static_route_map_rejects_sizes_beyond_its_buffer(T, E, k):
    fake = ctypes.c_void_p(0x10000)  # never touched: the call stops at the size check
    rc = tk.lib.tk_route_map_static(fake, T, E, k, 1, fake, fake, fake, fake, None, None)
    assert rc == 1
    assert "built-in buffer" in tk.lib.tk_last_error_detail().decode()
