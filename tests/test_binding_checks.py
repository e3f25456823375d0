"""The Python binding checks every tensor before it reaches the library: a tensor that is not on a
CUDA device, not contiguous, of the wrong dtype or too small for what the call touches raises
ValueError/TypeError before any library call. These tests need no GPU: CPU tensors exercise the
device check, and a stand-in that reports a CUDA device exercises the dtype and size checks."""
import pytest
import torch


@pytest.fixture(scope="module")
def tk():
    from token_routing_gate_b200 import build

    build.build()
    from token_routing_gate_b200 import tk as mod

    return mod


class OnCuda:
    """A CPU tensor that reports a CUDA device and the address 0 (NULL): should a check not fire,
    the library refuses the NULL on the host, so nothing is ever read through it."""

    def __init__(self, t):
        self._t = t
        self.device = torch.device("cuda", 0)
        self.dtype = t.dtype
        self.shape = t.shape

    def dim(self):
        return self._t.dim()

    def numel(self):
        return self._t.numel()

    def is_contiguous(self):
        return self._t.is_contiguous()

    def data_ptr(self):
        return 0


def cuda_like(*shape, dtype=torch.float32):
    return OnCuda(torch.zeros(*shape, dtype=dtype))


def test_cpu_tensors_are_refused(tk):
    logits = torch.zeros(4, 16)
    with pytest.raises(ValueError, match="CUDA device"):
        tk.gate_topk(logits, 2, "softmax")
    with pytest.raises(ValueError, match="CUDA device"):
        tk.route_map(torch.zeros(4, 2, dtype=torch.int32), 16)
    with pytest.raises(ValueError, match="CUDA device"):
        tk.reduce(torch.zeros(8, 64, dtype=torch.bfloat16), torch.zeros(4, 2, dtype=torch.int32),
                  out=torch.zeros(4, 64, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="CUDA device"):
        tk.tp_mask(torch.zeros(4, 2, dtype=torch.int32), 16, 2, 0)


def test_ptr_checks(tk):
    t = cuda_like(4, 8)
    with pytest.raises(TypeError, match="float32"):
        tk._ptr(cuda_like(4, 8, dtype=torch.float64), tk.F32, 32, "logits")
    with pytest.raises(ValueError, match="needs 33"):
        tk._ptr(t, tk.F32, 33, "logits")
    with pytest.raises(ValueError, match="contiguous"):
        tk._ptr(OnCuda(torch.zeros(8, 4).t()), tk.F32, 0, "logits")
    with pytest.raises(TypeError, match="uint8 or torch.float8_e4m3fn"):
        tk._ptr(cuda_like(4, dtype=torch.bfloat16), tk.E4M3, 0, "out")
    assert tk._ptr(None, tk.F32, 10, "bias") is None


def test_wrong_dtypes_are_refused_before_the_call(tk):
    idx64 = cuda_like(4, 2, dtype=torch.int64)
    with pytest.raises(TypeError, match="slot_of"):
        tk.reduce(cuda_like(8, 64, dtype=torch.bfloat16), idx64,
                  out=cuda_like(4, 64, dtype=torch.bfloat16))
    with pytest.raises(TypeError, match="y must be torch.bfloat16"):
        tk.reduce(cuda_like(8, 64), cuda_like(4, 2, dtype=torch.int32),
                  out=cuda_like(4, 64, dtype=torch.bfloat16))
    with pytest.raises(TypeError, match="topk_idx"):
        tk.gate_topk(cuda_like(4, 16), 2, "softmax", topk_idx=idx64, topk_w=cuda_like(4, 2))


def test_small_outputs_are_refused_before_the_call(tk):
    # an output one element short would be written past its end
    with pytest.raises(ValueError, match="out holds 255 elements; the call needs 256"):
        tk.reduce(cuda_like(8, 64, dtype=torch.bfloat16), cuda_like(4, 2, dtype=torch.int32),
                  out=OnCuda(torch.zeros(255, dtype=torch.bfloat16)))
    with pytest.raises(ValueError, match="topk_w"):
        tk.gate_topk(cuda_like(4, 16), 3, "softmax", topk_idx=cuda_like(4, 3, dtype=torch.int32),
                     topk_w=cuda_like(4, 2))
    T, E, k, align = 10, 8, 2, 4
    R = tk.max_rows(T, E, k, align)
    rm = tk.RouteMap(cuda_like(E, dtype=torch.int32), cuda_like(E + 1, dtype=torch.int32),
                     cuda_like(T, k, dtype=torch.int32), cuda_like(R - 1, dtype=torch.int32),
                     cuda_like(tk.route_map_workspace_bytes(T, E, k), dtype=torch.uint8), align)
    with pytest.raises(ValueError, match="token_of"):
        tk.route_map(cuda_like(T, k, dtype=torch.int32), E, align, out=rm)
    rm.token_of = cuda_like(R, dtype=torch.int32)
    rm.workspace = cuda_like(tk.route_map_workspace_bytes(T, E, k) // 4, dtype=torch.int32)
    with pytest.raises(TypeError, match="workspace"):
        tk.route_map(cuda_like(T, k, dtype=torch.int32), E, align, out=rm)
    with pytest.raises(ValueError, match="out holds"):
        tk.expand(cuda_like(T, 64, dtype=torch.bfloat16), rm, E, k,
                  out=cuda_like(R - 1, 64, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="out_scale"):
        tk.expand(cuda_like(T, 256, dtype=torch.bfloat16), rm, E, k, "fp8",
                  out=cuda_like(R, 256, dtype=torch.uint8), out_scale=cuda_like(R, 1))


def test_ep_buffers_are_checked(tk):
    with pytest.raises(ValueError, match="rows"):
        tk.ep_peer(cuda_like(9, 64, dtype=torch.bfloat16), cuda_like(10, 2, dtype=torch.int32),
                   cuda_like(10, 2), 0, 10)
    with pytest.raises(TypeError, match="idx"):
        tk.ep_peer(cuda_like(10, 64, dtype=torch.bfloat16), cuda_like(10, 2, dtype=torch.int64),
                   cuda_like(10, 2), 0, 10)
    # a descriptor of buffers already checked takes their addresses as they are
    x, idx, w = (torch.zeros(10, 64, dtype=torch.bfloat16), torch.zeros(10, 2, dtype=torch.int32),
                 torch.zeros(10, 2))
    again = tk.ep_peer(x, idx, w, 7, 10, checked=True)
    assert (again.x, again.idx, again.w, again.scale, again.base_row) == (
        x.data_ptr(), idx.data_ptr(), w.data_ptr(), None, 7)
    peer = tk.ep_peer(123456, 234560, 345600, 5, 10)   # raw addresses pass unchecked
    assert peer.x == 123456 and peer.idx == 234560 and peer.rows == 10 and peer.base_row == 5
