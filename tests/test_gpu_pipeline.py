"""RoutingPipeline (two batches in flight): every batch's outputs equal those of the same batch
run alone through the four calls, with batches that differ, more batches than routing slots,
and both output formats."""
import pytest
import torch

from token_routing_gate_b200 import tk
from token_routing_gate_b200 import workloads as W
from token_routing_gate_b200.pipeline import RoutingPipeline

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("wl", [W.V3.with_(T=2048, H=1024), W.V3_FP8.with_(T=1500, H=2048),
                                W.SKEW.with_(T=1000, H=512)], ids=lambda w: w.name)
def test_pipelined_batches_equal_single_runs(wl):
    n = 5
    batches = []
    for i in range(n):
        b = wl.with_(seed=wl.seed + 31 * i)
        logits, bias = W.gate_inputs(b, "cuda")
        batches.append((logits, bias, W.activations(b, "cuda"), W.expert_outputs(b, "cuda")))
    R = tk.max_rows(wl.T, wl.E, wl.k, wl.align)
    fp8 = wl.out_dtype == "fp8"
    xe = torch.empty(R, wl.H, dtype=torch.uint8 if fp8 else torch.bfloat16, device="cuda")
    xs = torch.empty(R, wl.H // 128, dtype=torch.float32, device="cuda") if fp8 else None
    outs = [torch.empty(wl.T, wl.H, dtype=torch.bfloat16, device="cuda") for _ in range(n)]
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    pipe = RoutingPipeline(wl.T, wl.E, wl.k, wl.score, wl.align)
    h = pipe.route(batches[0][0], batches[0][1], err_flag=err)
    for i in range(n):
        nxt = pipe.route(batches[i + 1][0], batches[i + 1][1], err_flag=err) if i + 1 < n else None
        pipe.dispatch_combine(h, batches[i][2], batches[i][3], outs[i], xe, wl.out_dtype, xs, err_flag=err)
        h = nxt
    torch.cuda.synchronize()
    assert err.item() == 0
    for i, (logits, bias, x, y) in enumerate(batches):
        idx, w = tk.gate_topk(logits, wl.k, wl.score, bias)
        rm = tk.route_map(idx, wl.E, wl.align)
        alone = tk.reduce(y, rm.slot_of, w)
        torch.cuda.synchronize()
        assert torch.equal(outs[i].view(torch.int16), alone.view(torch.int16)), f"batch {i}"
