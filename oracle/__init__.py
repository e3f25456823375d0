"""Python access to the CPU oracle -- TEST INFRASTRUCTURE ONLY.

Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg may
import this package. The CUDA library does not use it, and it does not use the CUDA library.
Arguments are numpy arrays (C-contiguous); bf16 tensors travel as uint16 bit patterns and
E4M3 codes as uint8. Each wrapper allocates its outputs and returns them, unless the caller
passes them in `out` (arrays of the exact shape and dtype, reused as they are: a timing loop can
then keep allocation out of what it measures).
"""
import ctypes
import os

import numpy as np

from .build import LIB, build_oracle

SOFTMAX = 0
SIGMOID = 1
OUT_BF16 = 0
OUT_FP8_E4M3 = 1

_lib = None


def lib():
    global _lib
    if _lib is None:
        # TKO_LIB points at a planted-mistake build (the mutation test only)
        path = os.environ.get("TKO_LIB") or (LIB if os.path.exists(LIB) else build_oracle())
        _lib = ctypes.CDLL(path)
        _declare(_lib)
    return _lib


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None else None


def _declare(L):
    vp, i32, i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
    L.tko_spec_expf.argtypes = [ctypes.c_float]
    L.tko_spec_expf.restype = ctypes.c_float
    L.tko_spec_sigmoidf.argtypes = [ctypes.c_float]
    L.tko_spec_sigmoidf.restype = ctypes.c_float
    L.tko_e4m3_encode.argtypes = [ctypes.c_float]
    L.tko_e4m3_encode.restype = ctypes.c_uint8
    L.tko_bf16_rne.argtypes = [ctypes.c_float]
    L.tko_bf16_rne.restype = ctypes.c_uint16
    for name in ("tko_spec_expf_array", "tko_spec_sigmoidf_array", "tko_e4m3_encode_array",
                 "tko_bf16_rne_array"):
        getattr(L, name).argtypes = [vp, vp, i64]
        getattr(L, name).restype = None
    L.tko_gate_topk.argtypes = [vp, vp, i32, i32, i32, i32, i32, vp, vp]
    L.tko_gate_topk.restype = i32
    L.tko_max_rows.argtypes = [i32, i32, i32, i32]
    L.tko_max_rows.restype = i64
    L.tko_route_map.argtypes = [vp, i32, i32, i32, i32, vp, vp, vp, vp]
    L.tko_route_map.restype = i32
    L.tko_quantize_row_e4m3.argtypes = [vp, i32, vp, vp]
    L.tko_quantize_row_e4m3.restype = i32
    L.tko_expand.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, vp, vp]
    L.tko_expand.restype = i32
    L.tko_reduce_token.argtypes = [vp, i64, vp, vp, i32, i32, vp]
    L.tko_reduce_token.restype = i32
    L.tko_reduce.argtypes = [vp, i64, vp, vp, i32, i32, i32, vp]
    L.tko_reduce.restype = i32
    L.tko_balance_stats.argtypes = [vp, vp, i32, i32, i32, i32, vp, vp, vp]
    L.tko_balance_stats.restype = i32
    L.tko_tp_mask.argtypes = [vp, i32, i32, i32, i32, i32, vp]
    L.tko_tp_mask.restype = i32
    L.tko_reduce_backward.argtypes = [vp, vp, i64, vp, vp, vp, i32, i32, i32, i32, vp, vp]
    L.tko_reduce_backward.restype = i32
    L.tko_ep_layout.argtypes = [vp, i32, i32, i32, i32, vp, vp]
    L.tko_ep_layout.restype = i32
    L.tko_ep_recv_bases.argtypes = [vp, i32, vp, vp]
    L.tko_ep_recv_bases.restype = i32
    L.tko_ep_dispatch.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i64, i32, vp, vp,
                                  vp, vp]
    L.tko_ep_dispatch.restype = i32
    L.tko_ep_combine.argtypes = [vp, vp, vp, i32, i32, i32, vp]
    L.tko_ep_combine.restype = i32


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _vector(fn, x, out_dtype):
    x = _c(x, np.float32).reshape(-1)
    y = np.empty(x.shape, dtype=out_dtype)
    fn(_p(x), _p(y), x.size)
    return y


def spec_expf(x):
    return _vector(lib().tko_spec_expf_array, x, np.float32)


def spec_sigmoidf(x):
    return _vector(lib().tko_spec_sigmoidf_array, x, np.float32)


def e4m3_encode(x):
    return _vector(lib().tko_e4m3_encode_array, x, np.uint8)


def bf16_rne(x):
    return _vector(lib().tko_bf16_rne_array, x, np.uint16)


def max_rows(T, E, k, align):
    return int(lib().tko_max_rows(T, E, k, align))


def _outputs(out, *specs):
    """The caller's output arrays (checked against (shape, dtype) specs), or new ones."""
    if out is None:
        return [np.empty(shape, dtype=dt) for shape, dt in specs]
    out = list(out)
    for a, (shape, dt) in zip(out, specs):
        if a.shape != tuple(shape) or a.dtype != np.dtype(dt) or not a.flags.c_contiguous:
            raise ValueError(f"output array {a.shape} {a.dtype} does not match {tuple(shape)} {dt}")
    return out


def gate_topk(logits, bias, k, score_fn, renormalize=True, out=None):
    logits = _c(logits, np.float32)
    T, E = logits.shape
    b = _c(bias, np.float32) if bias is not None else None
    idx, w = _outputs(out, ((T, k), np.int32), ((T, k), np.float32))
    rc = lib().tko_gate_topk(_p(logits), _p(b), T, E, k, score_fn, int(bool(renormalize)),
                             _p(idx), _p(w))
    if rc < 0:
        raise ValueError(f"tko_gate_topk rejected its arguments (rc={rc})")
    return idx, w


def route_map(topk_idx, E, align=1, out=None):
    topk_idx = _c(topk_idx, np.int32)
    T, k = topk_idx.shape
    counts, offsets, slot_of, token_of = _outputs(
        out, ((E,), np.int32), ((E + 1,), np.int32), ((T, k), np.int32),
        ((max_rows(T, E, k, align),), np.int32))
    rc = lib().tko_route_map(_p(topk_idx), T, E, k, align, _p(counts), _p(offsets), _p(slot_of),
                             _p(token_of))
    if rc < 0:
        raise ValueError(f"tko_route_map rejected its arguments (rc={rc})")
    return counts, offsets, slot_of, token_of, rc


def quantize_row_e4m3(xrow_bits):
    xrow_bits = _c(xrow_bits, np.uint16).reshape(-1)
    H = xrow_bits.size
    q = np.empty(H, dtype=np.uint8)
    s = np.empty(H // 128, dtype=np.float32)
    if lib().tko_quantize_row_e4m3(_p(xrow_bits), H, _p(q), _p(s)) < 0:
        raise ValueError("tko_quantize_row_e4m3 needs H % 128 == 0")
    return q, s


def expand(x_bits, slot_of, offsets, E, align=1, out_dtype=OUT_BF16, out=None):
    """Returns (out, out_scale); out has max_rows(T, E, k, align) rows, rows past offsets[E]
    are left as zero here (the oracle never writes them; caller-given arrays keep what they
    held there)."""
    x_bits = _c(x_bits, np.uint16)
    slot_of = _c(slot_of, np.int32)
    offsets = _c(offsets, np.int32)
    T, H = x_bits.shape
    k = slot_of.shape[1]
    rmax = max_rows(T, E, k, align)
    if out is not None:
        if out_dtype == OUT_BF16:
            (out,) = _outputs(out[:1], ((rmax, H), np.uint16))
            scale = None
        else:
            out, scale = _outputs(out, ((rmax, H), np.uint8), ((rmax, H // 128), np.float32))
    elif out_dtype == OUT_BF16:
        out = np.zeros((rmax, H), dtype=np.uint16)
        scale = None
    else:
        out = np.zeros((rmax, H), dtype=np.uint8)
        scale = np.zeros((rmax, H // 128), dtype=np.float32)
    rc = lib().tko_expand(_p(x_bits), _p(slot_of), _p(offsets), T, E, k, H, out_dtype, _p(out),
                          _p(scale))
    if rc < 0:
        raise ValueError(f"tko_expand rejected its arguments (rc={rc})")
    return out, scale


def reduce_token(y_bits, slot_row, w_row):
    y_bits = _c(y_bits, np.uint16)
    slot_row = _c(slot_row, np.int32).reshape(-1)
    w_row = _c(w_row, np.float32).reshape(-1) if w_row is not None else None
    H = y_bits.shape[1]
    out = np.empty(H, dtype=np.uint16)
    lib().tko_reduce_token(_p(y_bits), y_bits.shape[0], _p(slot_row), _p(w_row), slot_row.size, H,
                           _p(out))
    return out


def reduce(y_bits, slot_of, w, out=None):
    y_bits = _c(y_bits, np.uint16)
    slot_of = _c(slot_of, np.int32)
    w = _c(w, np.float32) if w is not None else None
    T, k = slot_of.shape
    H = y_bits.shape[1]
    (out,) = _outputs(None if out is None else (out,), ((T, H), np.uint16))
    rc = lib().tko_reduce(_p(y_bits), y_bits.shape[0], _p(slot_of), _p(w), T, k, H, _p(out))
    if rc < 0:
        raise ValueError(f"tko_reduce rejected its arguments (rc={rc})")
    return out


def balance_stats(logits, counts, k, score_fn):
    """(P [E], f [E], loss) in float64."""
    logits = _c(logits, np.float32)
    T, E = logits.shape
    counts = _c(counts, np.int32)
    P = np.empty(E, dtype=np.float64)
    f = np.empty(E, dtype=np.float64)
    loss = np.empty(1, dtype=np.float64)
    if lib().tko_balance_stats(_p(logits), _p(counts), T, E, k, score_fn, _p(P), _p(f), _p(loss)) < 0:
        raise ValueError("tko_balance_stats rejected its arguments")
    return P, f, float(loss[0])


def tp_mask(topk_idx, E, tp_size, tp_rank):
    topk_idx = _c(topk_idx, np.int32)
    T, k = topk_idx.shape
    out = np.empty_like(topk_idx)
    if lib().tko_tp_mask(_p(topk_idx), T, k, E, tp_size, tp_rank, _p(out)) < 0:
        raise ValueError("tko_tp_mask rejected its arguments")
    return out


def reduce_backward(grad_bits, y_bits, slot_of, offsets, w, E):
    """(d_y bits [y_rows, H] -- rows at and past offsets[E] left 0 --, d_w [T, k] fp32, rc)."""
    grad_bits = _c(grad_bits, np.uint16)
    y_bits = _c(y_bits, np.uint16)
    slot_of = _c(slot_of, np.int32)
    offsets = _c(offsets, np.int32)
    w = _c(w, np.float32) if w is not None else None
    T, H = grad_bits.shape
    k = slot_of.shape[1]
    d_y = np.zeros_like(y_bits)
    d_w = np.empty((T, k), dtype=np.float32)
    rc = lib().tko_reduce_backward(_p(grad_bits), _p(y_bits), y_bits.shape[0], _p(slot_of),
                                   _p(offsets), _p(w), T, E, k, H, _p(d_y), _p(d_w))
    if rc < 0:
        raise ValueError("tko_reduce_backward rejected its arguments")
    return d_y, d_w, rc


# ---------------------------------------------------------------- expert-parallel dispatch / combine
def ep_layout(topk_idx, E, G):
    """(send_counts [G], dest_pos [T, G]) of one source rank."""
    topk_idx = _c(topk_idx, np.int32)
    T, k = topk_idx.shape
    counts = np.empty(G, dtype=np.int32)
    dest_pos = np.empty((T, G), dtype=np.int32)
    rc = lib().tko_ep_layout(_p(topk_idx), T, E, k, G, _p(counts), _p(dest_pos))
    if rc < 0:
        raise ValueError(f"tko_ep_layout rejected its arguments (rc={rc})")
    return counts, dest_pos


def ep_recv_bases(count_matrix):
    """count_matrix [G, G] (source, destination) -> (base [G, G] int64, recv_rows [G] int64)."""
    cm = _c(count_matrix, np.int32)
    G = cm.shape[0]
    base = np.empty((G, G), dtype=np.int64)
    recv = np.empty(G, dtype=np.int64)
    if lib().tko_ep_recv_bases(_p(cm), G, _p(base), _p(recv)) < 0:
        raise ValueError("tko_ep_recv_bases rejected its arguments")
    return base, recv


def ep_dispatch(x_bits, topk_idx, topk_w, dest_pos, E, G, d, base_row, recv, out_dtype=OUT_BF16):
    """Writes one source's rows bound for rank d into recv = (recv_x, recv_scale, recv_idx,
    recv_w), the destination's receive buffers (numpy arrays, modified in place)."""
    x_bits = _c(x_bits, np.uint16)
    topk_idx = _c(topk_idx, np.int32)
    topk_w = _c(topk_w, np.float32)
    dest_pos = _c(dest_pos, np.int32)
    T, H = x_bits.shape
    k = topk_idx.shape[1]
    rx, rs, ri, rw = recv
    rc = lib().tko_ep_dispatch(_p(x_bits), _p(topk_idx), _p(topk_w), _p(dest_pos), T, E, k, H, G,
                               d, int(base_row), out_dtype, _p(rx), _p(rs), _p(ri), _p(rw))
    if rc < 0:
        raise ValueError(f"tko_ep_dispatch rejected its arguments (rc={rc})")


def ep_combine(partials, base_rows, dest_pos):
    """partials[d]: bf16 bits [rows_d, H] of every rank d; base_rows [G]: this source's first row
    in each rank's buffer; dest_pos [T, G] of this source. Returns out bits [T, H]."""
    dest_pos = _c(dest_pos, np.int32)
    T, G = dest_pos.shape
    parts = [_c(a, np.uint16) for a in partials]
    H = parts[0].shape[1]
    ptrs = (ctypes.c_void_p * G)(*[a.ctypes.data for a in parts])
    base = _c(base_rows, np.int64)
    out = np.empty((T, H), dtype=np.uint16)
    if lib().tko_ep_combine(ptrs, _p(base), _p(dest_pos), T, G, H, _p(out)) < 0:
        raise ValueError("tko_ep_combine rejected its arguments")
    return out


def ep_forward(xs, idxs, ws, make_y, E, G, align=1, out_dtype=OUT_BF16):
    """The whole expert-parallel forward over G ranks, stated step by step with the functions
    above (and the single-rank route map and reduce on each destination). xs[s], idxs[s],
    ws[s]: source rank s's token rows (bf16 bits), choices and weights. make_y(d, rows) returns
    rank d's expert outputs (bf16 bits [rows, H]) indexed by its local slots. Returns a dict of
    every intermediate and the per-source outputs."""
    k = idxs[0].shape[1]
    H = xs[0].shape[1]
    el = E // G
    lay = [ep_layout(idxs[s], E, G) for s in range(G)]
    cm = np.stack([c for c, _ in lay])
    base, recv_rows = ep_recv_bases(cm)
    recv = []
    for d in range(G):
        n = int(recv_rows[d])
        if out_dtype == OUT_BF16:
            rx, rs = np.zeros((n, H), dtype=np.uint16), np.zeros((n, 1), dtype=np.float32)
        else:
            rx, rs = np.zeros((n, H), dtype=np.uint8), np.zeros((n, H // 128), dtype=np.float32)
        buf = (rx, rs, np.full((n, k), -7, dtype=np.int32), np.zeros((n, k), dtype=np.float32))
        for s in range(G):
            ep_dispatch(xs[s], idxs[s], ws[s], lay[s][1], E, G, d, base[s, d], buf, out_dtype)
        recv.append(buf)
    dest, partials = [], []
    for d in range(G):
        n = int(recv_rows[d])
        counts, offsets, slot_of, token_of, rc = route_map(recv[d][2], el, align)
        y = make_y(d, max(max_rows(n, el, k, align), 1))
        part = reduce(y, slot_of, recv[d][3]) if n > 0 else np.zeros((0, H), dtype=np.uint16)
        dest.append({"counts": counts, "offsets": offsets, "slot_of": slot_of, "token_of": token_of,
                     "y": y})
        partials.append(part if n > 0 else np.zeros((1, H), dtype=np.uint16))
    outs = [ep_combine(partials, base[s], lay[s][1]) for s in range(G)]
    return {"layout": lay, "count_matrix": cm, "base": base, "recv_rows": recv_rows, "recv": recv,
            "dest": dest, "partials": partials, "out": outs}
