"""Shared pieces of the GPU tests: run the CUDA path through the C ABI, run the oracle on the
same inputs, compare."""
import numpy as np
import torch

import oracle
from token_routing_gate_b200 import tk


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor (any device) -> numpy uint16 bit patterns."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32)


def bf16_ulp_diff(a_bits: np.ndarray, b_bits: np.ndarray) -> np.ndarray:
    """Distance in bf16 ulps between two arrays of bf16 bit patterns (finite values)."""
    def ordered(u):
        u = u.astype(np.int32)
        return np.where(u & 0x8000, 0x8000 - (u & 0x7FFF), 0x8000 + u)   # +-0 map to 0x8000
    return np.abs(ordered(a_bits) - ordered(b_bits))


def score_fn(wl):
    return oracle.SOFTMAX if wl.score == "softmax" else oracle.SIGMOID


class DeviceRun:
    """The four C-ABI calls on device tensors, with an error flag."""

    def __init__(self, wl, logits, bias, x, y, renormalize=True, stream=None):
        self.wl = wl
        self.err = torch.zeros(1, dtype=torch.int32, device=logits.device)
        self.idx, self.w = tk.gate_topk(logits, wl.k, wl.score, bias, renormalize, stream=stream)
        self.rm = tk.route_map(self.idx, wl.E, wl.align, err_flag=self.err, stream=stream)
        if wl.out_dtype == "fp8":
            self.xq, self.xs = tk.expand(x, self.rm, wl.E, wl.k, "fp8", err_flag=self.err,
                                         stream=stream)
        else:
            self.xe = tk.expand(x, self.rm, wl.E, wl.k, "bf16", err_flag=self.err, stream=stream)
        self.out = tk.reduce(y, self.rm.slot_of, self.w, err_flag=self.err, stream=stream)
        torch.cuda.synchronize()


def assert_weights_close(w_gpu, w_ref, rtol=1e-6):
    w_gpu = np.asarray(w_gpu, np.float64)
    w_ref = np.asarray(w_ref, np.float64)
    err = np.abs(w_gpu - w_ref)
    bad = err > rtol * np.abs(w_ref)
    assert not bad.any(), f"{bad.sum()} weights off by more than {rtol} relative; worst {err.max()}"


def assert_weights_round_alike(w_gpu, w_ref, max_share=1e-5):
    """Both sides compute the weights in fp64 and round once to fp32, so they round alike: at
    most a share `max_share` of them (and at least one allowed) may differ, by one fp32 ulp."""
    a = np.ascontiguousarray(w_gpu, np.float32).view(np.int32).astype(np.int64)
    b = np.ascontiguousarray(w_ref, np.float32).view(np.int32).astype(np.int64)
    diff = np.abs(a - b)
    n_diff = int((diff != 0).sum())
    assert n_diff <= max(1, int(max_share * diff.size)), f"{n_diff} of {diff.size} weights differ"
    assert diff.max(initial=0) <= 1, f"a weight differs by {diff.max()} fp32 ulps"
