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


def test_reference_arm_prints_one_contract_line_on_rank_zero(monkeypatch, capsys):
    """The reference arm (the oracle on the host cores) runs without a GPU: one JSON
    line with the contract's keys, its own cpu_baseline and a zero-copy e2e."""
    import json
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.delenv("RANK", raising=False)

    class Args:
        gpus, steps, warmup = 1, 1, 3
    from workloads import CONFIGS
    assert bench.run_reference(Args, CONFIGS["tiny_fp32"]) == 0
    lines = [ln for ln in capsys.readouterr().out.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["steps"] == 1 and d["warmup"] == 3
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert d["config"]["workload"].startswith("tiny_fp32")
