"""Multi-rank logic of bench.py on the CPU: world size 2 over gloo.

Each rank runs its own replica with no collective on the data path; the only
exchange is the max over ranks of the timings, after which rank 0 reports the
whole-job rate.  These tests run that exchange with real gloo ranks.
"""
import os
import socket
import sys
from types import SimpleNamespace

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


# per-rank timings (ms): rank 1 is slower on some entries, rank 0 on others
RANK_TIMES = {0: [10.0, 4.0, 1.5, 30.0, 2.0], 1: [12.5, 3.0, 1.75, 29.0, 2.5]}


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()
        got = bench.max_over_ranks(RANK_TIMES[rank], world, torch.device("cpu"))
        dist.barrier()
        out[rank] = got
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    expect = [max(a, b) for a, b in zip(RANK_TIMES[0], RANK_TIMES[1])]
    assert res[0] == expect
    assert res[1] == expect          # every rank sees the same reduced values


def test_max_over_ranks_single_rank_is_identity():
    assert bench.max_over_ranks([3.0, 1.0], 1, torch.device("cpu")) == [3.0, 1.0]


def test_whole_job_rate_counts_all_ranks():
    # 2 replicas of 1e12 FLOPs each, slowest 1000 ms -> 2 TFLOP/s for the job
    assert bench.whole_job_rate(2, 1e12, 1000.0) == pytest.approx(2.0)
    assert bench.whole_job_rate(1, 137438953472.0 * 2 / 2, 100.0) == pytest.approx(1.37438953472)
    # weak scaling: doubling the ranks at a fixed per-rank time doubles the rate
    assert bench.whole_job_rate(8, 5e11, 7.0) == pytest.approx(4 * bench.whole_job_rate(2, 5e11, 7.0))


def test_reference_arm_other_ranks_exit_without_work(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    args = SimpleNamespace(workload="tiny", steps=3, warmup=3, gpus=2)
    assert bench.run_reference(args) == 0
    assert capsys.readouterr().out == ""


def test_reference_step_budget():
    # the default bench length must keep the oracle arm within a few minutes
    per = bench.reference_step_seconds(2000, 5)
    assert per * (2000 + 5) <= bench.REFERENCE_RUN_SECONDS + 1e-9
    assert bench.reference_step_seconds(3, 3) == 2.0
