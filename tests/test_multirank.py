"""The N > 1 path of bench.py on CPU: two gloo ranks.  Each rank processes its
own copy of the workload (weak scaling, no data-path collective); the step
time is the slowest rank's, and only rank 0 runs the oracle reference arm."""
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


def _rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        # ranks time different durations: everyone reports the slowest
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, world)
        thr = bench.aggregate_throughput(1000, world, 4, ms)

        class Args:
            steps, warmup = 1, 3
        ref = bench.run_reference(Args(), rank, world) if rank != 0 else "skipped"
        out[rank] = (ms, thr, ref)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_and_only_rank0_reports():
    world = 2
    port = _free_port()
    # spawn, not fork: this process may already run threads (OpenMP, torch)
    with mp.get_context("spawn").Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for rank in range(world):
        ms, thr, ref = res[rank]
        assert ms == pytest.approx(15.0)                # the slowest rank
        assert thr == pytest.approx(1000 * 2 * 4 / 0.015)  # units of all ranks / max time
    assert res[1][2] is None                            # rank 1 prints nothing


def test_single_rank_is_unchanged():
    import bench
    assert bench.max_over_ranks(7.5, 1) == 7.5
    assert bench.aggregate_throughput(10, 1, 2, 1000.0) == pytest.approx(20.0)
