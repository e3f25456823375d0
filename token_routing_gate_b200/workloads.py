"""Seeded synthetic workloads for the gate -> route map -> expand -> reduce path.

This module only draws inputs; it holds none of the method's arithmetic, so the CUDA library's
tests and the CPU oracle can both take their inputs from it. Shapes follow the DeepSeek-V3
setting that the 機器之心 page ("剛剛，DeepSeek開始頻繁更新", section "性能表現") uses for its
expert-parallel benchmark (8K tokens, hidden 7168, top-8 of 256 experts, FP8 dispatch, BF16
combine), plus a tiny case, a mid-size softmax case and a skewed-load case.

Token data (logits, x, y) is drawn from generators seeded with `seed` (1000 + case number);
per-expert parameters (the selection bias, the skew ranking) from `param_seed`, so data-parallel
shards that change `seed` still share one set of parameters. Draws run on the CPU or on a CUDA
device; the two give different (but each reproducible) streams.
"""
from dataclasses import dataclass, replace

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    T: int              # tokens
    E: int              # experts
    k: int              # experts per token
    H: int              # hidden size (channels per row)
    score: str          # "softmax" or "sigmoid"
    bias: bool          # per-expert selection bias U(-0.1, 0.1), sigmoid only
    skew: bool          # add -2.2*ln(rank) over a random expert ranking to the logits
    align: int          # per-expert segment padding (rows)
    out_dtype: str      # expand output: "bf16" or "fp8"
    seed: int           # token data (logits, x, y); differs per data-parallel shard
    param_seed: int = -1  # per-expert parameters (bias, skew ranking); -1 = same as seed

    @property
    def pairs(self) -> int:
        return self.T * self.k

    @property
    def max_rows(self) -> int:
        return self.T * self.k + self.E * (self.align - 1)

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


TINY = Workload("tiny_T128_E16_k2_H256_softmax", 128, 16, 2, 256, "softmax", False, False, 1,
                "bf16", 1001)
MID = Workload("T4096_E64_k6_H2048_softmax", 4096, 64, 6, 2048, "softmax", False, False, 1,
               "bf16", 1002)
V3 = Workload("T8192_E256_k8_H7168_sigmoid_bias", 8192, 256, 8, 7168, "sigmoid", True, False, 1,
              "bf16", 1003)
SKEW = Workload("T16384_E256_k8_H7168_skewed_align128", 16384, 256, 8, 7168, "sigmoid", False,
                True, 128, "bf16", 1004)
V3_FP8 = Workload("T8192_E256_k8_H7168_sigmoid_bias_fp8_dispatch", 8192, 256, 8, 7168, "sigmoid",
                  True, False, 1, "fp8", 1005)

ALL = (TINY, MID, V3, SKEW, V3_FP8)
BY_NAME = {w.name: w for w in ALL}


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def gate_inputs(wl: Workload, device="cpu"):
    """(logits fp32 [T,E], bias fp32 [E] or None). Logits are N(0,1); the skewed case adds
    2*ln(1/rank^1.1) = -2.2*ln(rank) for a random ranking 1..E of the experts."""
    g = _gen(wl.seed, device)
    logits = torch.randn(wl.T, wl.E, generator=g, device=device, dtype=torch.float32)
    gp = _gen(wl.seed if wl.param_seed < 0 else wl.param_seed, "cpu")
    bias = None
    if wl.bias:
        bias = (torch.rand(wl.E, generator=gp, dtype=torch.float32) * 0.2 - 0.1).to(device)
    if wl.skew:
        rank = torch.randperm(wl.E, generator=gp).to(torch.float32) + 1.0
        logits = logits + (-2.2 * torch.log(rank)).to(device)[None, :]
    return logits.contiguous(), bias


def activations(wl: Workload, device="cpu"):
    """Token activations x, bf16 N(0,1) [T,H]."""
    g = _gen(wl.seed + 100_000, device)
    return torch.randn(wl.T, wl.H, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)


def expert_outputs(wl: Workload, device="cpu", rows=None):
    """Expert outputs y, bf16 N(0,1) [rows, H] (default: the worst-case row count)."""
    g = _gen(wl.seed + 200_000, device)
    rows = wl.max_rows if rows is None else rows
    return torch.randn(rows, wl.H, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)
