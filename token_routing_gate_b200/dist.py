"""Process-per-GPU plumbing for data-parallel runs of the routing path.

The path shards by tokens with no exchange: every rank routes its own batch through its own
expert-sorted buffer, so the cross-rank traffic is the timing reduction (a barrier and a max
over ranks) and, when the load-balance loss of the whole batch is wanted, one all-reduce of
2E+1 numbers. torch.distributed supplies them ("nccl" on GPUs, "gloo" on CPU).
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


def allreduce_balance_inputs(sums, counts, T, group=None):
    """The global batch's load-balance inputs from every rank's own: sums (double [E], the
    per-expert score sums of tk_balance_score_sums), counts (int32 [E]) and T, each summed over
    the ranks of `group` in one all-reduce of 2E+1 doubles (integers below 2^53 are exact).
    Returns (sums, counts, T_total); with one rank, the inputs unchanged."""
    if not tdist.is_initialized() or tdist.get_world_size(group) == 1:
        return sums, counts, int(T)
    E = sums.shape[0]
    buf = torch.cat([sums.to(torch.float64), counts.to(torch.float64),
                     torch.tensor([float(T)], dtype=torch.float64, device=sums.device)])
    tdist.all_reduce(buf, group=group)
    return buf[:E].contiguous(), buf[E:2 * E].round().to(torch.int32), int(buf[2 * E].item())


def global_balance_stats(logits, counts, k, score, group=None, stream=None):
    """Load-balance statistics (P, f, loss) of the batch spread over the ranks of `group`: each
    rank's score sums, one all-reduce, then the finalize kernel (tk_balance_score_sums,
    allreduce_balance_inputs, tk_balance_finalize)."""
    from . import tk

    sums = tk.balance_score_sums(logits, score, stream=stream)
    sums, counts_all, T_all = allreduce_balance_inputs(sums, counts, logits.shape[0], group)
    return tk.balance_finalize(sums, counts_all, T_all, k, stream=stream)


def finish() -> None:
    if tdist.is_initialized():
        tdist.destroy_process_group()
