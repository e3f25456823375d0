"""The four calls captured into a CUDA graph and replayed: outputs equal an eager run bit for
bit, and a replay after new inputs are copied into the captured buffers equals an eager run on
those inputs. First-call setup (launch shapes, shared-memory opt-in) is done eagerly before the
capture, and every output is preallocated, so nothing allocates while capturing."""
import pytest
import torch

from token_routing_gate_b200 import tk
from token_routing_gate_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("wl", [W.V3.with_(T=2048, H=1024), W.V3_FP8.with_(T=1024, H=2048),
                                W.SKEW.with_(T=1500, H=512)], ids=lambda w: w.name)
def test_step_replays_from_a_cuda_graph(wl):
    logits, bias = W.gate_inputs(wl, "cuda")
    x = W.activations(wl, "cuda")
    y = W.expert_outputs(wl, "cuda")
    R = tk.max_rows(wl.T, wl.E, wl.k, wl.align)
    fp8 = wl.out_dtype == "fp8"
    idx = torch.empty(wl.T, wl.k, dtype=torch.int32, device="cuda")
    w = torch.empty(wl.T, wl.k, device="cuda")
    rm = tk.route_map(idx.zero_(), wl.E, wl.align)
    xe = torch.empty(R, wl.H, dtype=torch.uint8 if fp8 else torch.bfloat16, device="cuda")
    xs = torch.empty(R, wl.H // 128, device="cuda") if fp8 else None
    out = torch.empty(wl.T, wl.H, dtype=torch.bfloat16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")

    def step():
        tk.gate_topk(logits, wl.k, wl.score, bias, True, idx, w)
        tk.route_map(idx, wl.E, wl.align, out=rm, err_flag=err)
        tk.expand(x, rm, wl.E, wl.k, wl.out_dtype, out=xe, out_scale=xs, err_flag=err)
        tk.reduce(y, rm.slot_of, w, out=out, err_flag=err)

    def snapshot():
        vals = [idx, w.view(torch.int32), rm.slot_of, rm.offsets, out.view(torch.int16)]
        return [v.clone() for v in vals]

    step()                                     # eager: first-call setup, reference results
    torch.cuda.synchronize()
    eager = snapshot()

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        for t in (idx, w, rm.slot_of, out):
            t.zero_()
        with torch.cuda.graph(g, stream=s):
            step()
    g.replay()
    torch.cuda.synchronize()
    assert err.item() == 0
    for a, b in zip(eager, snapshot()):
        assert torch.equal(a, b)

    # new inputs in the captured buffers: the replay follows them
    nxt = wl.with_(seed=wl.seed + 1)
    l2, _ = W.gate_inputs(nxt, "cuda")
    logits.copy_(l2)
    x.copy_(W.activations(nxt, "cuda"))
    torch.cuda.synchronize()
    g.replay()
    torch.cuda.synchronize()
    replayed = snapshot()
    step()
    torch.cuda.synchronize()
    for a, b in zip(replayed, snapshot()):
        assert torch.equal(a, b)
    assert not torch.equal(eager[0], replayed[0])   # the routing did change
