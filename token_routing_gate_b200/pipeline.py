"""Two batches in flight: the routing of the next batch overlaps the expand/reduce of this one.

Gate and route map are latency-bound (tens of microseconds, little HBM traffic); expand and
reduce are HBM-bound. For a stream of independent batches (micro-batches of a serving engine,
say) the routing of batch i+1 can run on its own CUDA stream while batch i's expand and reduce
use the memory system; every batch still goes through all four calls and gets exactly the
results it would get alone.

    pipe = RoutingPipeline(T, E, k, score, align)
    h = pipe.route(logits[0], bias)                  # gate + route map of batch 0
    for i in range(n):
        nxt = pipe.route(logits[i + 1], bias) if i + 1 < n else None   # overlaps the next line
        pipe.dispatch_combine(h, x[i], y[i], out[i], xe)               # expand + reduce of batch i
        h = nxt

`route` writes one of `depth` sets of routing outputs (top-k indices and weights, route map)
and records an event; `dispatch_combine` makes the caller's stream wait for that event, then
runs expand and reduce. A set is reused only after the reduce that read it has finished. The
routing stream does not wait for the caller's stream: pass `ready` (a CUDA event) when the
batch's logits are produced on another stream.

Tensors the caller passes in are used on the routing stream (and, for `dispatch_combine`, on
`stream` when it is not the current one); both calls mark them with `record_stream`, so the
caching allocator does not hand their memory to anyone else before that work has run, even
if the caller drops its last reference right after the call.
"""
import torch

from . import tk


def _keep_for(stream, *tensors):
    """Keep the tensors' memory from being reused until the work queued on `stream` is done."""
    for t in tensors:
        if t is not None:
            t.record_stream(stream)


class RouteHandle:
    """Routing outputs of one batch and the event that marks them complete."""

    def __init__(self, idx, w, rm, event, slot):
        self.idx, self.w, self.rm, self.event, self.slot = idx, w, rm, event, slot


class RoutingPipeline:
    def __init__(self, T, E, k, score="sigmoid", align=1, renormalize=True, depth=2, device=None):
        device = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
        self.T, self.E, self.k, self.score, self.align = T, E, k, score, align
        self.renormalize = renormalize
        self.stream = torch.cuda.Stream(device=device)
        self.sets = []
        for _ in range(depth):
            idx = torch.zeros(T, k, dtype=torch.int32, device=device)
            w = torch.empty(T, k, dtype=torch.float32, device=device)
            rm = tk.route_map(idx, E, align)      # allocates the route-map buffers once
            # allocated on the current stream, used on ours
            _keep_for(self.stream, idx, w, rm.counts, rm.offsets, rm.slot_of, rm.token_of,
                      rm.workspace)
            self.sets.append((idx, w, rm))
        self.done = [None] * depth                # event: the last reduce that read the set
        self.n = 0
        torch.cuda.current_stream(device).synchronize()

    def route(self, logits, bias=None, ready=None, err_flag=None):
        """Gate + route map of one batch on the routing stream; returns its handle."""
        slot = self.n % len(self.sets)
        self.n += 1
        idx, w, rm = self.sets[slot]
        s = self.stream
        if self.done[slot] is not None:
            s.wait_event(self.done[slot])
        if ready is not None:
            s.wait_event(ready)
        _keep_for(s, logits, bias, err_flag)
        tk.gate_topk(logits, self.k, self.score, bias, self.renormalize, idx, w, s)
        tk.route_map(idx, self.E, self.align, out=rm, err_flag=err_flag, stream=s)
        ev = torch.cuda.Event()
        ev.record(s)
        return RouteHandle(idx, w, rm, ev, slot)

    def dispatch_combine(self, h, x, y, out, xe, out_dtype="bf16", xs=None, err_flag=None,
                         stream=None):
        """Expand x by the batch's route map into xe (E4M3 codes + xs scales for "fp8"), then
        reduce y by its slots and weights into out, on `stream` (default: the current one)."""
        s = stream if stream is not None else torch.cuda.current_stream()
        s.wait_event(h.event)
        if s != torch.cuda.current_stream():
            _keep_for(s, x, y, out, xe, xs, err_flag)
        tk.expand(x, h.rm, self.E, self.k, out_dtype, out=xe, out_scale=xs, err_flag=err_flag, stream=s)
        tk.reduce(y, h.rm.slot_of, h.w, out=out, err_flag=err_flag, stream=s)
        ev = torch.cuda.Event()
        ev.record(s)
        self.done[h.slot] = ev
        return out
