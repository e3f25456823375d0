"""Host-side ordering of RoutingPipeline (two batches in flight), checked without a GPU: CUDA
streams and events are replaced by recording stand-ins and the library calls by recorders, so the
test sees exactly which stream each call is issued on and which events each stream waits for.

What must hold for the results to be those of running every batch alone:
- routing outputs alternate between `depth` sets;
- the routing stream waits for the event of the last reduce that read a set before it
  overwrites that set;
- expand and reduce run on the caller's stream after it waited for that batch's routing event;
- a `ready` event given with the logits is waited for before the gate runs.
"""
import pytest
import torch


class FakeEvent:
    n = 0

    def __init__(self, *a, **kw):
        FakeEvent.n += 1
        self.id = FakeEvent.n
        self.stream = None

    def record(self, stream):
        self.stream = stream
        stream.log.append(("record", self.id))

    def __repr__(self):
        return f"E{self.id}"


class FakeStream:
    def __init__(self, name="routing", device=None):
        self.name = name
        self.log = []

    def wait_event(self, ev):
        self.log.append(("wait", ev.id))

    def synchronize(self):
        pass


@pytest.fixture
def pipeline(monkeypatch):
    from token_routing_gate_b200 import build

    build.build()
    from token_routing_gate_b200 import pipeline as P
    from token_routing_gate_b200 import tk

    calls = []
    caller = FakeStream("caller")

    def fake_route_map(idx, E, align=1, out=None, err_flag=None, stream=None):
        if out is None:   # construction: allocate the set's route map
            return tk.RouteMap(torch.zeros(E, dtype=torch.int32), torch.zeros(E + 1, dtype=torch.int32),
                               torch.zeros(idx.shape, dtype=torch.int32), torch.zeros(1, dtype=torch.int32),
                               torch.zeros(16, dtype=torch.uint8), align)
        calls.append(("route_map", stream.name, id(idx)))
        stream.log.append(("route_map", id(idx)))
        return out

    def fake_gate(logits, k, score, bias, renorm, idx, w, stream):
        calls.append(("gate", stream.name, id(idx)))
        stream.log.append(("gate", id(idx)))

    def fake_expand(x, rm, E, k, out_dtype, out=None, out_scale=None, err_flag=None, stream=None):
        calls.append(("expand", stream.name, id(rm)))
        stream.log.append(("expand", id(rm)))

    def fake_reduce(y, slot_of, w, out=None, err_flag=None, stream=None):
        calls.append(("reduce", stream.name, id(slot_of)))
        stream.log.append(("reduce", id(slot_of)))

    monkeypatch.setattr(P.tk, "route_map", fake_route_map)
    monkeypatch.setattr(P.tk, "gate_topk", fake_gate)
    monkeypatch.setattr(P.tk, "expand", fake_expand)
    monkeypatch.setattr(P.tk, "reduce", fake_reduce)
    monkeypatch.setattr(P.torch.cuda, "Stream", FakeStream)
    monkeypatch.setattr(P.torch.cuda, "Event", FakeEvent)
    monkeypatch.setattr(P.torch.cuda, "current_stream", lambda *a: caller)
    monkeypatch.setattr(P.torch.cuda, "current_device", lambda: 0)
    kept = []
    monkeypatch.setattr(P, "_keep_for", lambda stream, *ts: kept.append(
        (stream.name, [t for t in ts if t is not None])))
    pipe = P.RoutingPipeline(T=8, E=4, k=2, device="cpu")
    pipe.kept = kept
    return pipe, caller, calls


def test_sets_alternate_and_reuse_waits_for_the_reduce(pipeline):
    pipe, caller, calls = pipeline
    routing = pipe.stream
    h0 = pipe.route("logits0")
    h1 = pipe.route("logits1")
    assert (h0.slot, h1.slot) == (0, 1) and h0.idx is not h1.idx
    # the first use of each set waits for nothing
    assert [e for e in routing.log if e[0] == "wait"] == []
    pipe.dispatch_combine(h0, "x0", "y0", "out0", "xe")
    done0 = pipe.done[0]
    h2 = pipe.route("logits2")                  # reuses set 0
    assert h2.slot == 0 and h2.idx is h0.idx
    i_wait = routing.log.index(("wait", done0.id))
    i_gate = max(i for i, e in enumerate(routing.log) if e == ("gate", id(h2.idx)))
    assert i_wait < i_gate                       # set 0 is overwritten only after its reduce
    assert done0.stream is caller                # that event marks the reduce on the caller's stream


def test_expand_and_reduce_wait_for_their_routing(pipeline):
    pipe, caller, calls = pipeline
    h = pipe.route("logits")
    assert h.event.stream is pipe.stream
    pipe.dispatch_combine(h, "x", "y", "out", "xe")
    log = caller.log
    i_wait = log.index(("wait", h.event.id))
    assert log[i_wait + 1] == ("expand", id(h.rm)) and log[i_wait + 2] == ("reduce", id(h.rm.slot_of))
    assert log[i_wait + 3] == ("record", pipe.done[h.slot].id)
    # gate and route map ran on the routing stream, expand and reduce on the caller's
    assert [c[:2] for c in calls] == [("gate", "routing"), ("route_map", "routing"),
                                      ("expand", "caller"), ("reduce", "caller")]


def test_ready_event_is_waited_for_before_the_gate(pipeline):
    pipe, caller, calls = pipeline
    ready = FakeEvent()
    h = pipe.route("logits", ready=ready)
    log = pipe.stream.log
    assert log.index(("wait", ready.id)) < log.index(("gate", id(h.idx)))
    assert log[-1] == ("record", h.event.id)


def test_caller_tensors_are_kept_alive_for_the_streams_that_use_them(pipeline):
    pipe, caller, calls = pipeline
    # construction: every tensor of both sets is marked for the routing stream
    assert [k[0] for k in pipe.kept] == ["routing", "routing"]
    assert all(len(k[1]) == 7 for k in pipe.kept)
    pipe.kept.clear()
    h = pipe.route("logits", bias="bias", err_flag="flag")
    assert pipe.kept == [("routing", ["logits", "bias", "flag"])]
    pipe.kept.clear()
    pipe.dispatch_combine(h, "x", "y", "out", "xe")          # the current stream: nothing to do
    assert pipe.kept == []
    other = FakeStream("other")
    pipe.dispatch_combine(h, "x", "y", "out", "xe", xs="xs", stream=other)
    assert pipe.kept == [("other", ["x", "y", "out", "xe", "xs"])]
