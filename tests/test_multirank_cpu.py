"""The multi-rank path of bench.py on CPU: two gloo ranks (world size 2) spawned as processes.

With N GPUs every rank runs its own copy of the workload (weak scaling, no data-path collective);
what crosses ranks is the timing: a barrier, the slowest rank's elapsed time (max over ranks), the
whole-job throughput computed from it, and the reference arm that only rank 0 runs.
"""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world, init_method=f"tcp://127.0.0.1:{port}")
    try:
        # each rank measured a different time; every rank must report the slowest one
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, world)
        bench.barrier(world, cuda=False)
        rate = bench.whole_job_rate(65536, world, ms)
        # the reference arm: rank 0 alone prints; the other ranks return at once without work
        ref = None
        if rank != 0:
            class A:
                steps, warmup = 1, 0
            ref = bench.run_reference(A())
        out[rank] = (ms, rate, ref)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_max_time_and_whole_job_rate():
    world = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    assert sorted(res) == [0, 1]
    for rank in (0, 1):
        ms, rate, ref = res[rank]
        assert ms == 15.0  # the slower rank's time, on both ranks
        assert rate == pytest.approx(2 * 65536 / 0.015)  # both ranks' tokens over the slowest time
    assert res[1][2] is None


def test_single_rank_helpers_need_no_process_group():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.whole_job_rate(100, 1, 2.0) == pytest.approx(50_000.0)
