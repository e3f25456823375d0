"""Process-per-GPU plumbing for data-parallel runs of the routing path.

The path shards by tokens with no exchange: every rank routes its own batch through its own
expert-sorted buffer, so the only cross-rank traffic is the timing reduction (a barrier and a
max over ranks). torch.distributed supplies it ("nccl" on GPUs, "gloo" on CPU).
"""
import datetime
import os

import torch
import torch.distributed as tdist


def rank_env():
    """(rank, world_size, local_rank) from the torchrun environment, defaulting to one process."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str, timeout_s: float = 120.0) -> bool:
    """Initialise the default process group when more than one rank runs; returns whether it did."""
    _, world, _ = rank_env()
    if world <= 1 or tdist.is_initialized():
        return tdist.is_initialized()
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    tdist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))
    return True


def shard_seed(base_seed: int, rank: int) -> int:
    """Seed of rank `rank`'s synthetic batch (rank 0 keeps the single-GPU seed)."""
    return base_seed + 7919 * rank


def barrier(device=None) -> None:
    if tdist.is_initialized():
        if device is not None and device.type == "cuda":
            tdist.barrier(device_ids=[device.index])
        else:
            tdist.barrier()


def max_over_ranks(value: float, device=None) -> float:
    if not tdist.is_initialized():
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device or "cpu")
    tdist.all_reduce(t, op=tdist.ReduceOp.MAX)
    return float(t.item())


def aggregate_rate(units_per_rank: float, world: int, max_seconds: float) -> float:
    """Whole-job throughput: the units all ranks processed over the slowest rank's time."""
    return units_per_rank * world / max_seconds if max_seconds > 0 else float("nan")


def finish() -> None:
    if tdist.is_initialized():
        tdist.destroy_process_group()
