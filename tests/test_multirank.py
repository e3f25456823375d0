"""The N > 1 host path on CPU: two gloo ranks, each routing its own token shard (no data-path
exchange). Checks the rank environment, per-rank seeds, the max-over-ranks timing reduction,
the whole-job rate, and that sharding by tokens is exact: the gate result of each shard equals
the matching rows of the gate over the concatenated batch (the oracle stands in for the
device path on CPU)."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, result_dir):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as tdist

    import oracle
    from token_routing_gate_b200 import dist
    from token_routing_gate_b200 import workloads as W

    assert dist.rank_env() == (rank, world, rank)
    assert dist.init("gloo", timeout_s=60)
    wl = W.V3.with_(T=96, H=128)
    seed = dist.shard_seed(wl.seed, rank)
    logits, bias = W.gate_inputs(wl.with_(seed=seed, param_seed=wl.seed), "cpu")
    idx, w = oracle.gate_topk(logits.numpy(), bias.numpy(), wl.k, oracle.SIGMOID)
    counts, offsets, slot_of, token_of, rc = oracle.route_map(idx, wl.E, wl.align)
    assert rc == 0 and counts.sum() == wl.T * wl.k
    # timing reduction: the slowest rank decides
    t = 1.0 + rank
    mx = dist.max_over_ranks(t)
    assert mx == float(world)
    assert dist.aggregate_rate(wl.T, world, mx) == wl.T * world / world
    gathered = [None] * world
    tdist.all_gather_object(gathered, (seed, logits.numpy(), bias.numpy(), idx, w))
    dist.barrier()
    if rank == 0:
        seeds = [g[0] for g in gathered]
        assert len(set(seeds)) == world and seeds[0] == wl.seed
        # the bias is per expert, shared by every rank's workload definition
        for g in gathered:
            np.testing.assert_array_equal(g[2], gathered[0][2])
        full_logits = np.concatenate([g[1] for g in gathered])
        full_idx, full_w = oracle.gate_topk(full_logits, gathered[0][2], wl.k, oracle.SIGMOID)
        np.testing.assert_array_equal(full_idx, np.concatenate([g[3] for g in gathered]))
        np.testing.assert_array_equal(full_w, np.concatenate([g[4] for g in gathered]))
        open(os.path.join(result_dir, "ok"), "w").close()
    dist.finish()


def test_two_gloo_ranks(tmp_path, oracle_lib):
    world = 2
    mp.spawn(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    assert (tmp_path / "ok").exists()
