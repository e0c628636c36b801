"""Host-side multi-rank logic of bench.py, run as two gloo ranks on the CPU: every rank
times its own replica of the workload, the job time is the slowest rank's, and the
whole-job throughput counts the elements of every replica."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, results):
    import torch.distributed as dist

    import bench

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = 10.0 + 5.0 * rank  # rank 1 is the slowest
        results[rank] = bench.max_over_ranks(local_ms)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    world = 2
    port = _free_port()
    with mp.Manager() as mgr:
        results = mgr.dict()
        mp.spawn(_rank_main, args=(world, port, results), nprocs=world, join=True)
        assert dict(results) == {0: 15.0, 1: 15.0}


def test_weak_scaling_value_counts_every_replica():
    import bench

    assert bench.weak_scaling_value(1_000_000, 1, 1.0) == pytest.approx(1.0)
    assert bench.weak_scaling_value(1_000_000, 4, 2.0) == pytest.approx(2.0)
    assert bench.max_over_ranks(3.5) == 3.5
