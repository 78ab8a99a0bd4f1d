"""The benchmark's multi-rank path on CPU: world size 2 over gloo.

Replicas run independently; the only collectives are the timing barrier and a
max over ranks of the elapsed time, from which the whole-job throughput counts
every rank's tokens.  The reference arm does its work on rank 0 only.
"""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, out):
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()
        m = bench.max_over_ranks(times[rank], dist, "cpu")
        out[rank] = (m, bench.whole_job_throughput(world, 4096, 10, m))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_time_and_count_all_tokens():
    world, times = 2, [12.5, 20.0]
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank_main, args=(world, _free_port(), times, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0] == res[1]
    m, v = res[0]
    assert m == max(times)
    assert v == pytest.approx(world * 4096 * 10 / (max(times) / 1e3))


def test_reference_arm_does_no_work_off_rank_zero(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")

    class Args:
        gpus, steps, warmup = 2, 3, 3
    from workloads import CONFIGS
    assert bench.run_reference(Args, CONFIGS["tiny_fp32"]) == 0


def test_single_process_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.0) == 3.0
    assert bench.whole_job_throughput(1, 64, 5, 1.0) == pytest.approx(64 * 5 / 1e-3)
