"""The multi-rank host logic of bench.py on CPU: two gloo ranks.

bench.py --gpus N runs N independent replicas (no data-path collective); what
crosses ranks is the barrier around the timed region and the max over ranks of
the step time, from which the whole-job rate is computed. The reference arm
runs on rank 0 only. These are checked here with world_size 2 on the gloo
backend.
"""
import datetime
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, result_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        bench.barrier(world)
        # each rank timed its own replica; the slowest one decides
        ms_local = [2.0, 5.0][rank]
        assert bench.max_over_ranks(ms_local, world) == 5.0
        ms, rate = bench.whole_job_rate(1_000_000, ms_local, world)
        assert ms == 5.0 and abs(rate - world * 1_000_000 / 5e-3) < 1e-6
        # the reference arm: rank 0 alone does the work and prints
        if rank != 0:
            assert bench.run_reference(None, world, rank) is None
        bench.barrier(world)
        with open(os.path.join(result_dir, f"ok{rank}"), "w") as f:
            f.write("ok")
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    assert sorted(os.listdir(tmp_path)) == ["ok0", "ok1"]


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert not dist.is_initialized()
    bench.barrier(1)
    assert bench.max_over_ranks(3.25, 1) == 3.25
    ms, rate = bench.whole_job_rate(500, 2.0, 1)
    assert ms == 2.0 and rate == pytest.approx(250_000.0)
