"""Thin Python binding of libtk_route.so (C ABI in include/tk_route.h).

Argument marshalling only: torch tensors supply device memory and the current CUDA stream,
every step runs in the library's kernels. The names follow the C entry points without the
``tk_`` prefix. Missing outputs are allocated with torch (caching allocator) before the call;
pass preallocated tensors to keep allocation out of a timed loop. There is no fallback: if the
library is not built, importing this module raises.

Every tensor handed to the library is checked first: on a CUDA device, contiguous, of the dtype
the C declaration names, and holding at least the elements the call reads or writes (a smaller
output would otherwise be written past its end). A failed check raises ValueError or TypeError
before anything runs; the library's own argument checks then raise TkError.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtk_route.so")

SCORE = {"softmax": 0, "sigmoid": 1}
OUT_DTYPE = {"bf16": 0, "fp8": 1}

DEVERR_EXPERT_RANGE = 1
DEVERR_DUP_EXPERT = 2
DEVERR_SLOT_RANGE = 4
DEVERR_ROWS_RANGE = 8
DEVERR_TIMEOUT = 16

# every C entry point declared in include/tk_route.h
ABI_SYMBOLS = ("tk_gate_topk", "tk_max_rows", "tk_route_map_workspace_bytes", "tk_route_map",
               "tk_route_map_window",
               "tk_route_map_static", "tk_expand", "tk_reduce", "tk_reduce_masked", "tk_balance_stats_workspace_bytes",
               "tk_balance_stats", "tk_balance_score_sums", "tk_balance_finalize", "tk_tp_mask", "tk_reduce_backward_workspace_bytes",
               "tk_reduce_backward", "tk_expand_backward", "tk_ep_layout_workspace_bytes",
               "tk_ep_layout", "tk_ep_dispatch", "tk_ep_combine", "tk_selftest_bounded_wait",
               "tk_selftest_gate_margin", "tk_selftest_balance_exp",
               "tk_status_str", "tk_last_error_detail", "tk_abi_version")


class EpPeer(ctypes.Structure):
    """tk_ep_peer: one destination rank's receive buffers (device addresses)."""
    _fields_ = [("x", ctypes.c_void_p), ("scale", ctypes.c_void_p), ("idx", ctypes.c_void_p),
                ("w", ctypes.c_void_p), ("base_row", ctypes.c_int64), ("rows", ctypes.c_int64)]


class TkError(RuntimeError):
    def __init__(self, fn, status, detail):
        super().__init__(f"{fn} failed: {status} -- {detail}")
        self.status = status
        self.detail = detail


def _load():
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"{LIB_PATH} is not built; run `python -m token_routing_gate_b200.build` "
            "(the CUDA library is required, there is no CPU path)")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
    L.tk_gate_topk.argtypes = [vp, vp, i32, i32, i32, i32, i32, vp, vp, vp]
    L.tk_gate_topk.restype = i32
    L.tk_max_rows.argtypes = [i32, i32, i32, i32]
    L.tk_max_rows.restype = i64
    L.tk_route_map_workspace_bytes.argtypes = [i32, i32, i32]
    L.tk_route_map_workspace_bytes.restype = sz
    L.tk_route_map.argtypes = [vp, i32, i32, i32, i32, vp, vp, vp, vp, vp, sz, vp, vp]
    L.tk_route_map.restype = i32
    L.tk_route_map_window.argtypes = [vp, i32, i32, i32, i32, i32, i32, vp, vp, vp, vp, vp, sz, vp, vp]
    L.tk_route_map_window.restype = i32
    L.tk_route_map_static.argtypes = [vp, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp]
    L.tk_route_map_static.restype = i32
    L.tk_expand.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, vp, vp, vp, vp]
    L.tk_expand.restype = i32
    L.tk_reduce.argtypes = [vp, i64, vp, vp, i32, i32, i32, vp, vp, vp]
    L.tk_reduce.restype = i32
    L.tk_reduce_masked.argtypes = L.tk_reduce.argtypes
    L.tk_reduce_masked.restype = i32
    L.tk_balance_stats_workspace_bytes.argtypes = [i32, i32]
    L.tk_balance_stats_workspace_bytes.restype = sz
    L.tk_balance_stats.argtypes = [vp, vp, i32, i32, i32, i32, vp, vp, vp, vp, sz, vp]
    L.tk_balance_stats.restype = i32
    L.tk_balance_score_sums.argtypes = [vp, i32, i32, i32, vp, vp, sz, vp]
    L.tk_balance_score_sums.restype = i32
    L.tk_balance_finalize.argtypes = [vp, vp, i64, i32, i32, vp, vp, vp, vp]
    L.tk_balance_finalize.restype = i32
    L.tk_tp_mask.argtypes = [vp, i32, i32, i32, i32, i32, vp, vp]
    L.tk_tp_mask.restype = i32
    L.tk_reduce_backward_workspace_bytes.argtypes = [i32, i32]
    L.tk_reduce_backward_workspace_bytes.restype = sz
    L.tk_reduce_backward.argtypes = [vp, vp, i64, vp, vp, vp, vp, i32, i32, i32, i32, vp, vp, vp, sz,
                                     vp, vp]
    L.tk_reduce_backward.restype = i32
    L.tk_expand_backward.argtypes = [vp, i64, vp, i32, i32, i32, vp, vp, vp]
    L.tk_expand_backward.restype = i32
    L.tk_ep_layout_workspace_bytes.argtypes = [i32, i32]
    L.tk_ep_layout_workspace_bytes.restype = sz
    L.tk_ep_layout.argtypes = [vp, i32, i32, i32, i32, vp, vp, vp, vp, vp, sz, vp, vp]
    L.tk_ep_layout.restype = i32
    L.tk_ep_dispatch.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32,
                                 ctypes.POINTER(EpPeer), vp, vp]
    L.tk_ep_dispatch.restype = i32
    L.tk_ep_combine.argtypes = [ctypes.POINTER(ctypes.c_void_p), ctypes.POINTER(ctypes.c_int64),
                                ctypes.POINTER(ctypes.c_int64), vp, vp, i32, i32, i32, vp, vp, vp]
    L.tk_ep_combine.restype = i32
    L.tk_selftest_bounded_wait.argtypes = [i64, vp, vp]
    L.tk_selftest_bounded_wait.restype = i32
    L.tk_selftest_gate_margin.argtypes = [vp, vp]
    L.tk_selftest_gate_margin.restype = i32
    L.tk_selftest_balance_exp.argtypes = [vp, vp]
    L.tk_selftest_balance_exp.restype = i32
    L.tk_status_str.argtypes = [i32]
    L.tk_status_str.restype = ctypes.c_char_p
    L.tk_last_error_detail.argtypes = []
    L.tk_last_error_detail.restype = ctypes.c_char_p
    L.tk_abi_version.argtypes = []
    L.tk_abi_version.restype = i32
    return L


lib = _load()


def _check(fn, status):
    if status != 0:
        raise TkError(fn, lib.tk_status_str(status).decode(), lib.tk_last_error_detail().decode())


F32, F64, I32, BF16, U8 = torch.float32, torch.float64, torch.int32, torch.bfloat16, torch.uint8
E4M3 = (torch.uint8, torch.float8_e4m3fn)     # E4M3 codes: raw bytes or torch's fp8 type


def _ptr(t, dtype=None, numel=0, name="tensor"):
    """Device address of a tensor for the library (None stays NULL). The tensor must be on a CUDA
    device and contiguous; `dtype` (one dtype or a tuple) and `numel` (the fewest elements the
    call touches) are checked when given."""
    if t is None:
        return None
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be on a CUDA device, not {t.device}")
    if dtype is not None:
        ok = dtype if isinstance(dtype, tuple) else (dtype,)
        if t.dtype not in ok:
            raise TypeError(f"{name} must be {' or '.join(str(d) for d in ok)}, not {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.numel() < numel:
        raise ValueError(f"{name} holds {t.numel()} elements; the call needs {numel}")
    return ctypes.c_void_p(t.data_ptr())


def _shape2(t, name):
    if t.dim() != 2:
        raise ValueError(f"{name} must be 2-D, got shape {tuple(t.shape)}")
    return t.shape


def _flag(err_flag):
    return _ptr(err_flag, I32, 1, "err_flag")


def _ws(workspace, nbytes):
    """Workspaces are byte tensors: their numel() is passed as the byte count."""
    return _ptr(workspace, U8, nbytes, "workspace")


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def max_rows(T, E, k, align=1):
    return int(lib.tk_max_rows(T, E, k, align))


def route_map_workspace_bytes(T, E, k):
    return int(lib.tk_route_map_workspace_bytes(T, E, k))


def gate_topk(logits, k, score="sigmoid", bias=None, renormalize=True, topk_idx=None, topk_w=None,
              stream=None):
    """logits fp32 [T,E] -> (topk_idx int32 [T,k], topk_w fp32 [T,k])."""
    T, E = _shape2(logits, "logits")
    if topk_idx is None:
        topk_idx = torch.empty(T, k, dtype=torch.int32, device=logits.device)
    if topk_w is None:
        topk_w = torch.empty(T, k, dtype=torch.float32, device=logits.device)
    _check("tk_gate_topk", lib.tk_gate_topk(_ptr(logits, F32, T * E, "logits"), _ptr(bias, F32, E, "bias"),
                                            T, E, k, SCORE[score], int(bool(renormalize)),
                                            _ptr(topk_idx, I32, T * k, "topk_idx"),
                                            _ptr(topk_w, F32, T * k, "topk_w"), _stream(stream)))
    return topk_idx, topk_w


class RouteMap:
    """Outputs of route_map: counts [E], offsets [E+1], slot_of [T,k], token_of [max_rows]."""

    def __init__(self, counts, offsets, slot_of, token_of, workspace, align):
        self.counts, self.offsets, self.slot_of, self.token_of = counts, offsets, slot_of, token_of
        self.workspace = workspace
        self.align = align


def route_map(topk_idx, E, align=1, out=None, err_flag=None, stream=None):
    T, k = _shape2(topk_idx, "topk_idx")
    dev = topk_idx.device
    if out is None:
        ws = max(route_map_workspace_bytes(T, E, k), 16)
        out = RouteMap(torch.empty(E, dtype=torch.int32, device=dev),
                       torch.empty(E + 1, dtype=torch.int32, device=dev),
                       torch.empty(T, k, dtype=torch.int32, device=dev),
                       torch.empty(max(max_rows(T, E, k, align), 1), dtype=torch.int32, device=dev),
                       torch.empty((ws + 15) // 16, 16, dtype=torch.uint8, device=dev), align)
    _check("tk_route_map", lib.tk_route_map(
        _ptr(topk_idx, I32, T * k, "topk_idx"), T, E, k, align, _ptr(out.counts, I32, E, "counts"),
        _ptr(out.offsets, I32, E + 1, "offsets"), _ptr(out.slot_of, I32, T * k, "slot_of"),
        _ptr(out.token_of, I32, max_rows(T, E, k, align), "token_of"),
        _ws(out.workspace, route_map_workspace_bytes(T, E, k)), out.workspace.numel(), _flag(err_flag),
        _stream(stream)))
    return out


def route_map_window(topk_idx, E_total, expert_lo, E, align=1, out=None, err_flag=None, stream=None):
    """Route map of the experts [expert_lo, expert_lo + E) of E_total (others masked): the same
    outputs as tp_mask followed by route_map with E experts, in one call."""
    T, k = _shape2(topk_idx, "topk_idx")
    dev = topk_idx.device
    if out is None:
        ws = max(route_map_workspace_bytes(T, E, k), 16)
        out = RouteMap(torch.empty(E, dtype=torch.int32, device=dev),
                       torch.empty(E + 1, dtype=torch.int32, device=dev),
                       torch.empty(T, k, dtype=torch.int32, device=dev),
                       torch.empty(max(max_rows(T, E, k, align), 1), dtype=torch.int32, device=dev),
                       torch.empty((ws + 15) // 16, 16, dtype=torch.uint8, device=dev), align)
    _check("tk_route_map_window", lib.tk_route_map_window(
        _ptr(topk_idx, I32, T * k, "topk_idx"), T, E_total, k, expert_lo, E, align,
        _ptr(out.counts, I32, E, "counts"), _ptr(out.offsets, I32, E + 1, "offsets"),
        _ptr(out.slot_of, I32, T * k, "slot_of"),
        _ptr(out.token_of, I32, max_rows(T, E, k, align), "token_of"),
        _ws(out.workspace, route_map_workspace_bytes(T, E, k)), out.workspace.numel(), _flag(err_flag),
        _stream(stream)))
    return out


def expand(x, rm, E, k, out_dtype="bf16", out=None, out_scale=None, err_flag=None, stream=None):
    """x bf16 [T,H] -> out [max_rows, H] (bf16, or E4M3 as uint8 with fp32 scales [max_rows, H/128])."""
    T, H = _shape2(x, "x")
    R_max = max_rows(T, E, k, rm.align)
    R = max(R_max, 1)
    if out is None:
        out = torch.empty(R, H, dtype=torch.bfloat16 if out_dtype == "bf16" else torch.uint8,
                          device=x.device)
    if out_dtype == "fp8" and out_scale is None:
        out_scale = torch.empty(R, H // 128, dtype=torch.float32, device=x.device)
    _check("tk_expand", lib.tk_expand(
        _ptr(x, BF16, T * H, "x"), _ptr(rm.slot_of, I32, T * k, "slot_of"),
        _ptr(rm.offsets, I32, E + 1, "offsets"), _ptr(rm.token_of, I32, R_max, "token_of"), T, E, k, H,
        rm.align, OUT_DTYPE[out_dtype], _ptr(out, E4M3 if out_dtype == "fp8" else BF16, R_max * H, "out"),
        _ptr(out_scale, F32, R_max * (H // 128), "out_scale"), _flag(err_flag), _stream(stream)))
    return (out, out_scale) if out_dtype == "fp8" else out


def reduce(y, slot_of, w=None, out=None, err_flag=None, stream=None, masked=False):
    """y bf16 [rows,H], slot_of int32 [T,k], w fp32 [T,k] or None -> out bf16 [T,H].
    masked=True calls tk_reduce_masked (same results; faster when most pairs are -1)."""
    T, k = _shape2(slot_of, "slot_of")
    rows, H = _shape2(y, "y")
    if out is None:
        out = torch.empty(T, H, dtype=torch.bfloat16, device=y.device)
    fn, name = (lib.tk_reduce_masked, "tk_reduce_masked") if masked else (lib.tk_reduce, "tk_reduce")
    _check(name, fn(_ptr(y, BF16, rows * H, "y"), rows, _ptr(slot_of, I32, T * k, "slot_of"),
                    _ptr(w, F32, T * k, "w"), T, k, H, _ptr(out, BF16, T * H, "out"), _flag(err_flag),
                    _stream(stream)))
    return out


def _workspace(nbytes, device):
    return torch.empty((max(nbytes, 16) + 15) // 16, 16, dtype=torch.uint8, device=device)


def balance_stats(logits, counts, k, score="sigmoid", workspace=None, out=None, stream=None):
    """Load-balance statistics -> (P fp32 [E], f fp32 [E], loss fp32 [1])."""
    T, E = _shape2(logits, "logits")
    dev = counts.device
    ws_bytes = int(lib.tk_balance_stats_workspace_bytes(T, E))
    if workspace is None:
        workspace = _workspace(ws_bytes, dev)
    if out is None:
        out = (torch.empty(E, dtype=torch.float32, device=dev),
               torch.empty(E, dtype=torch.float32, device=dev),
               torch.empty(1, dtype=torch.float32, device=dev))
    P, f, loss = out
    _check("tk_balance_stats", lib.tk_balance_stats(
        _ptr(logits, F32, T * E, "logits"), _ptr(counts, I32, E, "counts"), T, E, k, SCORE[score],
        _ptr(P, F32, E, "P"), _ptr(f, F32, E, "f"), _ptr(loss, F32, 1, "loss"),
        _ws(workspace, ws_bytes), workspace.numel(), _stream(stream)))
    return P, f, loss


def balance_score_sums(logits, score="sigmoid", workspace=None, out=None, stream=None):
    """Per-expert sums (double [E]) of the normalised unbiased scores over this batch's tokens."""
    T, E = _shape2(logits, "logits")
    dev = logits.device
    ws_bytes = int(lib.tk_balance_stats_workspace_bytes(T, E))
    if workspace is None:
        workspace = _workspace(ws_bytes, dev)
    if out is None:
        out = torch.empty(E, dtype=torch.float64, device=dev)
    _check("tk_balance_score_sums", lib.tk_balance_score_sums(
        _ptr(logits, F32, T * E, "logits"), T, E, SCORE[score], _ptr(out, F64, E, "sums"),
        _ws(workspace, ws_bytes), workspace.numel(), _stream(stream)))
    return out


def balance_finalize(sums, counts, T_total, k, out=None, stream=None):
    """(P, f, loss) fp32 from score sums and counts summed over ranks and the total token count."""
    E = sums.shape[0]
    dev = sums.device
    if out is None:
        out = (torch.empty(E, device=dev), torch.empty(E, device=dev), torch.empty(1, device=dev))
    P, f, loss = out
    _check("tk_balance_finalize", lib.tk_balance_finalize(
        _ptr(sums, F64, E, "sums"), _ptr(counts, I32, E, "counts"), int(T_total), E, k,
        _ptr(P, F32, E, "P"), _ptr(f, F32, E, "f"), _ptr(loss, F32, 1, "loss"), _stream(stream)))
    return P, f, loss


def tp_mask(topk_idx, E, tp_size, tp_rank, out=None, stream=None):
    """Keep this rank's experts (renumbered locally), mark the rest -1."""
    T, k = _shape2(topk_idx, "topk_idx")
    if out is None:
        out = torch.empty_like(topk_idx)
    _check("tk_tp_mask", lib.tk_tp_mask(_ptr(topk_idx, I32, T * k, "topk_idx"), T, k, E, tp_size, tp_rank,
                                        _ptr(out, I32, T * k, "out"), _stream(stream)))
    return out


def reduce_backward(grad_out, y, slot_of, w, E, rm=None, d_y=None, d_w=None, workspace=None,
                    err_flag=None, stream=None):
    """Backward of reduce -> (d_y bf16 [rows, H], d_w fp32 [T, k]). With a RouteMap `rm`,
    padding rows of d_y are zeroed."""
    T, k = _shape2(slot_of, "slot_of")
    H = _shape2(grad_out, "grad_out")[1]
    rows = _shape2(y, "y")[0]
    dev = grad_out.device
    if d_y is None:
        d_y = torch.empty_like(y)
    if d_w is None:
        d_w = torch.empty(T, k, dtype=torch.float32, device=dev)
    ws_bytes = int(lib.tk_reduce_backward_workspace_bytes(T, k))
    if workspace is None:
        workspace = _workspace(ws_bytes, dev)
    _check("tk_reduce_backward", lib.tk_reduce_backward(
        _ptr(grad_out, BF16, T * H, "grad_out"), _ptr(y, BF16, rows * H, "y"), rows,
        _ptr(slot_of, I32, T * k, "slot_of"),
        _ptr(rm.offsets, I32, E + 1, "offsets") if rm is not None else None,
        _ptr(rm.token_of, I32, max_rows(T, E, k, rm.align), "token_of") if rm is not None else None,
        _ptr(w, F32, T * k, "w"), T, E, k, H, _ptr(d_y, BF16, rows * H, "d_y"),
        _ptr(d_w, F32, T * k, "d_w"), _ws(workspace, ws_bytes), workspace.numel(),
        _flag(err_flag), _stream(stream)))
    return d_y, d_w


def expand_backward(d_xe, slot_of, out=None, err_flag=None, stream=None):
    """Backward of a bf16 expand: d_x[t] = sum_j d_xe[slot_of[t, j]]."""
    T, k = _shape2(slot_of, "slot_of")
    rows, H = _shape2(d_xe, "d_xe")
    if out is None:
        out = torch.empty(T, H, dtype=torch.bfloat16, device=d_xe.device)
    _check("tk_expand_backward", lib.tk_expand_backward(
        _ptr(d_xe, BF16, rows * H, "d_xe"), rows, _ptr(slot_of, I32, T * k, "slot_of"), T, k, H,
        _ptr(out, BF16, T * H, "out"), _flag(err_flag), _stream(stream)))
    return out


def selftest_bounded_wait(limit_ns, err_flag, stream=None):
    """Run the bounded-wait self-test kernel (it always times out and flags DEVERR_TIMEOUT)."""
    _check("tk_selftest_bounded_wait", lib.tk_selftest_bounded_wait(int(limit_ns), _flag(err_flag),
                                                                    _stream(stream)))


def selftest_gate_margin(max_err=None, stream=None):
    """Largest |approximate - exact| logistic value over the finite fp32 logits |l| <= 2^7 (the
    bound the gate's candidate filter rests on), as a device float tensor [1]."""
    if max_err is None:
        max_err = torch.empty(1, dtype=torch.float32, device="cuda")
    _check("tk_selftest_gate_margin", lib.tk_selftest_gate_margin(_ptr(max_err, F32, 1, "max_err"),
                                                                  _stream(stream)))
    return max_err


def selftest_balance_exp(max_rel_err=None, stream=None):
    """Largest relative differences between the balance statistics' short double-precision path
    and the library over every finite fp32 l with |l| <= 708: [e^-l, 1/(1 + e^-l)], as a device
    double tensor [2]."""
    if max_rel_err is None:
        max_rel_err = torch.empty(2, dtype=torch.float64, device="cuda")
    _check("tk_selftest_balance_exp", lib.tk_selftest_balance_exp(
        _ptr(max_rel_err, F64, 2, "max_rel_err"), _stream(stream)))
    return max_rel_err


# ---------------------------------------------------------------- expert-parallel dispatch / combine
def _addr(t, dtype=None, rows=0, name="buffer"):
    """Device address of a tensor, or a raw integer address (e.g. a peer's buffer, which only its
    owner can check). A tensor is checked as by _ptr and must have at least `rows` rows."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if t.dim() < 1 or t.shape[0] < rows:
        raise ValueError(f"{name} has shape {tuple(t.shape)}; the call needs {rows} rows")
    return _ptr(t, dtype, 0, name).value


class EpLayout:
    """Send layout of one source rank (tk_ep_layout): the route map over destination ranks."""

    def __init__(self, send_counts, send_offsets, dest_slot, send_token, workspace, G):
        self.send_counts, self.send_offsets = send_counts, send_offsets
        self.dest_slot, self.send_token, self.workspace, self.G = dest_slot, send_token, workspace, G


def ep_layout(topk_idx, E, G, out=None, err_flag=None, stream=None):
    T, k = _shape2(topk_idx, "topk_idx")
    dev = topk_idx.device
    if out is None:
        out = EpLayout(torch.empty(G, dtype=torch.int32, device=dev),
                       torch.empty(G + 1, dtype=torch.int32, device=dev),
                       torch.empty(T, G, dtype=torch.int32, device=dev),
                       torch.empty(T * G, dtype=torch.int32, device=dev),
                       _workspace(int(lib.tk_ep_layout_workspace_bytes(T, G)), dev), G)
    _check("tk_ep_layout", lib.tk_ep_layout(
        _ptr(topk_idx, I32, T * k, "topk_idx"), T, E, k, G, _ptr(out.send_counts, I32, G, "send_counts"),
        _ptr(out.send_offsets, I32, G + 1, "send_offsets"), _ptr(out.dest_slot, I32, T * G, "dest_slot"),
        _ptr(out.send_token, I32, T * G, "send_token"),
        _ws(out.workspace, int(lib.tk_ep_layout_workspace_bytes(T, G))), out.workspace.numel(),
        _flag(err_flag), _stream(stream)))
    return out


def _raw(t):
    return None if t is None else (t if isinstance(t, int) else t.data_ptr())


def ep_peer(x, idx, w, base_row, rows, scale=None, checked=False):
    """Descriptor of one destination's receive buffers: tensors or raw device addresses.
    checked=True: the same tensors passed an earlier call's checks, only their addresses are read."""
    rows = int(rows)
    if checked:
        return EpPeer(_raw(x), _raw(scale), _raw(idx), _raw(w), int(base_row), rows)
    return EpPeer(_addr(x, (BF16,) + E4M3, rows, "x"), _addr(scale, F32, rows, "scale"),
                  _addr(idx, I32, rows, "idx"), _addr(w, F32, rows, "w"), int(base_row), rows)


def ep_dispatch(x, topk_idx, topk_w, layout, E, peers, out_dtype="bf16", err_flag=None,
                stream=None):
    """Writes this rank's tokens into the G destinations' receive buffers (peers: G EpPeer)."""
    T, H = _shape2(x, "x")
    k = _shape2(topk_idx, "topk_idx")[1]
    G = layout.G
    if len(peers) != G:
        raise ValueError(f"{len(peers)} peer descriptors for G={G}")
    arr = (EpPeer * G)(*peers)
    _check("tk_ep_dispatch", lib.tk_ep_dispatch(
        _ptr(x, BF16, T * H, "x"), _ptr(topk_idx, I32, T * k, "topk_idx"), _ptr(topk_w, F32, T * k, "topk_w"),
        _ptr(layout.dest_slot, I32, T * G, "dest_slot"), _ptr(layout.send_offsets, I32, G + 1, "send_offsets"),
        T, E, k, H, G, OUT_DTYPE[out_dtype], arr, _flag(err_flag), _stream(stream)))


def ep_combine(partials, base_rows, rows, layout, H, out=None, err_flag=None, stream=None):
    """out[t] = bf16(sum over destinations d ascending of partials[d][base_rows[d] + position]).
    partials: G tensors or raw device addresses of bf16 [rows[d], H] buffers."""
    G = layout.G
    T = layout.dest_slot.shape[0]
    if out is None:
        out = torch.empty(T, H, dtype=torch.bfloat16, device=layout.dest_slot.device)
    if len(partials) != G or len(base_rows) != G or len(rows) != G:
        raise ValueError(f"partials, base_rows and rows need G={G} entries each")
    ptrs = (ctypes.c_void_p * G)(*[_addr(p, BF16, int(r), f"partials[{d}]")
                                   for d, (p, r) in enumerate(zip(partials, rows))])
    base = (ctypes.c_int64 * G)(*[int(b) for b in base_rows])
    nrows = (ctypes.c_int64 * G)(*[int(r) for r in rows])
    _check("tk_ep_combine", lib.tk_ep_combine(
        ptrs, base, nrows, _ptr(layout.dest_slot, I32, T * G, "dest_slot"),
        _ptr(layout.send_offsets, I32, G + 1, "send_offsets"), T, G, H, _ptr(out, BF16, T * H, "out"),
        _flag(err_flag), _stream(stream)))
    return out
