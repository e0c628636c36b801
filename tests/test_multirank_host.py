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


def test_shard_range_covers_the_batch_in_order():
    import bench

    for B in range(1, 40):
        for world in range(1, 9):
            if B < world:
                continue
            ranges = [bench.shard_range(B, world, r) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == B
            assert all(ranges[r][1] == ranges[r + 1][0] for r in range(world - 1))
            sizes = [b1 - b0 for b0, b1 in ranges]
            assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 1


def _shard_main(rank, world, port, results):
    """Each rank runs the CPU oracle's fused core on its batch shard of one workload and the
    ranks all-gather their shards of y: the result must be the oracle's output for the whole
    batch, on every rank (the sharded path's one collective, over gloo)."""
    import numpy as np
    import torch
    import torch.distributed as dist

    import bench
    from oracle import oracle as orc
    from selective_scan_02_b200.inputs import Workload, make_inputs

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl = Workload("shard", 5, 8, 6, 5, 4, 0, "f32", "f32", 21)  # 5 images over 2 ranks: 3 + 2
        inp = make_inputs(wl)
        b0, b1 = bench.shard_range(wl.B, world, rank)
        sl = slice(b0, b1)
        y_local = orc.forward_core(inp["x"][sl], inp["A_logs"], inp["Ds"], inp["dt_bias"], dts=inp["dts"][sl],
                                   Bs=inp["Bs"][sl], Cs=inp["Cs"][sl])
        y_all = bench.gather_shards(torch.from_numpy(y_local), wl.B, world).numpy()
        ref = orc.forward_core(inp["x"], inp["A_logs"], inp["Ds"], inp["dt_bias"], dts=inp["dts"], Bs=inp["Bs"],
                               Cs=inp["Cs"])
        results[rank] = (y_all.shape == ref.shape, bool(np.array_equal(y_all, ref)), (b0, b1))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_gather_their_batch_shards():
    world = 2
    port = _free_port()
    with mp.Manager() as mgr:
        results = mgr.dict()
        mp.spawn(_shard_main, args=(world, port, results), nprocs=world, join=True)
        assert dict(results) == {0: (True, True, (0, 3)), 1: (True, True, (3, 5))}
