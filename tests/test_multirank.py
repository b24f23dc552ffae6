"""The multi-rank plumbing of bench.py on the CPU: two gloo ranks on 127.0.0.1.

bench.py runs independent replicas, one rank per GPU with a fixed per-GPU batch;
no data-path collective exists.  What the ranks share is the timing: every rank
contributes its own device time, all take the same MAX all-reduce, and the
whole-job throughput counts every rank's samples over the slowest rank's time.
"""
from __future__ import annotations

import argparse
import datetime
import os
import socket

import pytest


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import torch.distributed as dist
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms = bench.slowest_rank_ms(10.0 + 5.0 * rank, dist, device="cpu")
        q.put((rank, ms, bench.job_throughput(world, 4, 20, ms)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_time():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        res = sorted(q.get(timeout=120) for _ in procs)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert [p.exitcode for p in procs] == [0, 0]
    assert [r for r, _, _ in res] == [0, 1]
    for _, ms, value in res:
        assert ms == 15.0                        # the slower rank's time, on both ranks
        assert value == pytest.approx(2 * 4 * 20 / 0.015)


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.slowest_rank_ms(12.5, None) == 12.5
    assert bench.job_throughput(1, 1, 200, 2500.0) == pytest.approx(80.0)


def test_reference_arm_other_ranks_exit_without_work(monkeypatch, capsys):
    import bench
    from vla_flow_matching_b200 import synth
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    args = argparse.Namespace(steps=1, warmup=3, gpus=2, time_grid="pi0", x_prediction=False,
                              causal_actions=False, precision="bf16")
    assert bench.run_reference(args, synth.WORKLOADS["tiny"]) == 0
    assert capsys.readouterr().out == ""


def test_bench_refuses_a_gpu_count_without_that_many_ranks():
    """`bench.py --gpus N` must run as N ranks; run alone it exits non-zero
    instead of timing one GPU under an N-GPU label."""
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ)
    env.pop("WORLD_SIZE", None)
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "4", "--steps", "1",
                        "--warmup", "3"], capture_output=True, text=True, env=env, timeout=120)
    assert r.returncode != 0 and "--nproc-per-node 4" in r.stderr
    assert r.stdout.strip() == ""
