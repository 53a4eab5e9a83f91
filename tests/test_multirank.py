"""The multi-rank logic of bench.py on CPU with the gloo backend (world size
2): ranks draw their own seeded problems, the step time is the max over
ranks, and the whole-job value counts every rank's work (weak scaling)."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        from block_sparse_attention_psa_b200.inputs import make_qkv

        # each rank times a different amount; every rank must see the max
        local_ms = 10.0 + 5.0 * rank
        total = bench.max_over_ranks(local_ms, world)
        q, _, _ = make_qkv(1, 1, 128, 64, "clustered", seed=rank)
        digest = float(q.float().sum())
        gathered = [None] * world
        dist.all_gather_object(gathered, digest)
        out[rank] = (total, gathered)
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_ranks_max_timing_and_distinct_problems():
    world = 2
    port = _free_port()
    # the manager's server process is started by spawn too: nothing here forks
    with mp.get_context("spawn").Manager() as manager:
        out = manager.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = {rank: out[rank] for rank in range(world)}
    for rank in range(world):
        total, digests = res[rank]
        assert total == 15.0
        assert digests[0] != digests[1]          # independent seeded problems


def test_weak_scaling_value():
    import bench

    one = bench.weak_scaling_value(6.6e12, 1, 2.0)
    eight = bench.weak_scaling_value(6.6e12, 8, 2.0)
    assert abs(eight - 8 * one) < 1e-9
