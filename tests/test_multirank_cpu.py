"""The multi-rank host logic of bench.py, run as two gloo ranks on the CPU.

One process per GPU, no collective on the data path: every rank runs its own
workload on its own seeded inputs, and the only exchange is the max of one
timing scalar over ranks.  These tests run that plumbing with world size 2
over gloo on 127.0.0.1.
"""

import os
import socket
import sys
import time

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    import bench
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        w, r, lr = bench.dist_env()
        # each rank times its own steps; the job time is the slowest rank's
        local_ms = 10.0 + 5.0 * rank
        job_ms = bench.max_over_ranks(local_ms, torch.device("cpu"), w)
        # each rank draws its own inputs (seed offset = rank)
        c, (q, k, v), mask, score, kv_len, doc = bench.make_inputs("fp32_causal_small", "cpu", seed_offset=r)
        torch.save({"rank": (w, r, lr), "job_ms": job_ms, "q": q, "k": k},
                   os.path.join(out_dir, f"rank{rank}.pt"))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.fixture(scope="module")
def two_ranks(tmp_path_factory):
    out = tmp_path_factory.mktemp("ranks")
    ctx = mp.start_processes(_worker, args=(2, _free_port(), str(out)), nprocs=2, join=False, start_method="spawn")
    # join() returns once a process exits (True when all have); a failing rank raises
    deadline = time.monotonic() + 240
    while not ctx.join(timeout=5):
        assert time.monotonic() < deadline, "ranks did not finish"
    return [torch.load(os.path.join(out, f"rank{r}.pt")) for r in range(2)]


def test_env_and_max_over_ranks(two_ranks):
    for r, d in enumerate(two_ranks):
        assert d["rank"] == (2, r, r)
        assert d["job_ms"] == 15.0  # max of 10 and 15, on every rank


def test_each_rank_draws_its_own_inputs(two_ranks):
    a, b = two_ranks
    assert a["q"].shape == b["q"].shape
    assert not torch.equal(a["q"], b["q"]) and not torch.equal(a["k"], b["k"])
    # and rank 0's draw is the single-GPU workload itself
    sys.path.insert(0, ROOT)
    import bench
    _, (q0, _, _), *_ = bench.make_inputs("fp32_causal_small", "cpu", seed_offset=0)
    assert torch.equal(a["q"], q0)


def test_whole_job_rate_is_weak_scaling():
    sys.path.insert(0, ROOT)
    import bench
    # 2 ranks each doing 1e12 FLOP per step in 1 ms (slowest rank): 2000 TFLOP/s
    assert bench.whole_job_rate(1e12, 2, 1.0, 1e12) == pytest.approx(2000.0)
    assert bench.whole_job_rate(1e12, 1, 1.0, 1e12) == pytest.approx(1000.0)
    assert bench.max_over_ranks(3.5, torch.device("cpu"), 1) == 3.5


def test_reference_arm_runs_on_rank0_only(monkeypatch, capsys):
    """Under torchrun the oracle arm is timed on rank 0; other ranks exit at once."""
    sys.path.insert(0, ROOT)
    import argparse

    import bench
    monkeypatch.setenv("RANK", "1")
    args = argparse.Namespace(workload="fp32_causal_small", gpus=2, steps=1, warmup=3)
    assert bench.run_reference(args) == 0
    assert capsys.readouterr().out == ""
