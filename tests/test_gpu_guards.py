"""Every output buffer sits between two canary regions; after each call the canaries must be
unchanged, i.e. no kernel writes outside the rows and elements its arguments describe."""
import pytest
import torch

from token_routing_gate_b200 import tk
from token_routing_gate_b200 import workloads as W

pytestmark = pytest.mark.gpu

GUARD = 4096  # bytes on each side (a multiple of 16, so the buffer stays 16-byte aligned)
CANARY = 0xA5


class Guarded:
    """A tensor view with canary bytes before and after it."""

    def __init__(self, shape, dtype):
        n = 1
        for s in shape:
            n *= s
        nbytes = n * torch.tensor([], dtype=dtype).element_size()
        self.raw = torch.full((GUARD + nbytes + GUARD,), CANARY, dtype=torch.uint8, device="cuda")
        self.t = self.raw[GUARD:GUARD + nbytes].view(dtype).view(*shape) if n else \
            torch.empty(shape, dtype=dtype, device="cuda")

    def intact(self):
        return bool((self.raw[:GUARD] == CANARY).all() and (self.raw[-GUARD:] == CANARY).all())


@pytest.mark.parametrize("wl", [W.V3.with_(T=3000), W.SKEW.with_(T=2000), W.V3_FP8.with_(T=777),
                                W.MID.with_(T=555, align=7)], ids=lambda w: w.name)
def test_no_writes_outside_outputs(wl):
    logits, bias = W.gate_inputs(wl, "cuda")
    x = W.activations(wl, "cuda")
    y = W.expert_outputs(wl, "cuda")
    T, E, k, H = wl.T, wl.E, wl.k, wl.H
    rows = wl.max_rows
    g = {
        "idx": Guarded((T, k), torch.int32), "w": Guarded((T, k), torch.float32),
        "counts": Guarded((E,), torch.int32), "offsets": Guarded((E + 1,), torch.int32),
        "slot_of": Guarded((T, k), torch.int32), "token_of": Guarded((rows,), torch.int32),
        "ws": Guarded((tk.route_map_workspace_bytes(T, E, k) // 4 + 4,), torch.int32),
        "out": Guarded((T, H), torch.bfloat16), "err": Guarded((1,), torch.int32),
    }
    if wl.out_dtype == "fp8":
        g["xe"] = Guarded((rows, H), torch.uint8)
        g["xs"] = Guarded((rows, H // 128), torch.float32)
    else:
        g["xe"] = Guarded((rows, H), torch.bfloat16)
    g["err"].t.zero_()
    tk.gate_topk(logits, k, wl.score, bias, True, g["idx"].t, g["w"].t)
    rm = tk.RouteMap(g["counts"].t, g["offsets"].t, g["slot_of"].t, g["token_of"].t,
                     g["ws"].t.view(torch.uint8), wl.align)
    tk.route_map(g["idx"].t, E, wl.align, out=rm, err_flag=g["err"].t)
    tk.expand(x, rm, E, k, wl.out_dtype, out=g["xe"].t, out_scale=g["xs"].t if "xs" in g else None,
              err_flag=g["err"].t)
    tk.reduce(y, rm.slot_of, g["w"].t, out=g["out"].t, err_flag=g["err"].t)
    # next-row ops into guarded outputs too
    g["dy"] = Guarded((rows, H), torch.bfloat16)
    g["dw"] = Guarded((T, k), torch.float32)
    g["bws"] = Guarded((tk.lib.tk_reduce_backward_workspace_bytes(T, k) // 4,), torch.int32)
    g["dx"] = Guarded((T, H), torch.bfloat16)
    g["P"], g["f"], g["loss"] = Guarded((E,), torch.float32), Guarded((E,), torch.float32), Guarded((1,), torch.float32)
    g["sws"] = Guarded((tk.lib.tk_balance_stats_workspace_bytes(T, E) // 4,), torch.int32)
    g["mask"] = Guarded((T, k), torch.int32)
    grad = W.activations(wl.with_(seed=wl.seed + 9), "cuda")
    tk.reduce_backward(grad, y, rm.slot_of, g["w"].t, E, rm=rm, d_y=g["dy"].t, d_w=g["dw"].t,
                       workspace=g["bws"].t.view(torch.uint8), err_flag=g["err"].t)
    tk.expand_backward(y, rm.slot_of, out=g["dx"].t, err_flag=g["err"].t)
    tk.balance_stats(logits, rm.counts, k, wl.score, workspace=g["sws"].t.view(torch.uint8),
                     out=(g["P"].t, g["f"].t, g["loss"].t))
    tk.tp_mask(g["idx"].t, E, 2 if E % 2 == 0 else 1, 0, out=g["mask"].t)
    torch.cuda.synchronize()
    assert g["err"].t.item() == 0
    broken = [name for name, buf in g.items() if not buf.intact()]
    assert not broken, f"canaries overwritten around: {broken}"
