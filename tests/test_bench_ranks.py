"""The multi-rank logic of bench.py on CPU: two gloo ranks on 127.0.0.1.

The decode path has no data-path collective (every rank decodes its own
replica layer), so what the ranks share is the timing protocol: the same
collective steps in the same order, the step time taken as the maximum over
ranks, and one JSON line from rank 0.  These tests run that protocol with
the gloo backend in spawned processes, no GPU involved.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, outq):
    import datetime
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    try:
        # per-rank step times: rank r's slowest-step time is 10 + r ms
        torch.distributed.barrier()
        ms = bench.max_over_ranks(10.0 + rank, torch.device("cpu"))
        torch.distributed.barrier()
        us_step, job = bench.job_value(ms, steps=5, world=world)
        outq.put((rank, ms, us_step, job, bench.rank_seed(2, rank)))
    finally:
        torch.distributed.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_step_time():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    for rank, ms, us_step, job, seed in got:
        assert ms == 11.0                       # max over ranks, on every rank
        assert us_step == pytest.approx(11.0 * 1e3 / 5)
        assert job == pytest.approx(us_step / world)
    seeds = [g[4] for g in got]
    assert seeds[0] is None and seeds[1] is not None    # distinct replica workloads


def test_single_process_needs_no_process_group():
    assert bench.max_over_ranks(3.5, torch.device("cpu")) == 3.5
    assert bench.job_value(2.0, steps=4, world=1) == (500.0, 500.0)
    assert len({bench.rank_seed(2, r) for r in range(8)}) == 8


def test_reference_arm_runs_on_rank_zero_only():
    """Under torchrun the oracle arm is timed by rank 0 alone; other ranks
    exit at once, printing nothing."""
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--config", "1", "--cpu-budget", "0.2", "--steps", "2", "--warmup", "3"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""
    env = dict(os.environ, WORLD_SIZE="2", RANK="0", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--config", "1", "--cpu-budget", "0.2", "--steps", "2", "--warmup", "3"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    res = json.loads(lines[0])
    assert res["impl"] == "reference" and res["n_gpus"] == 2
    assert res["cpu_baseline"]["kind"] == "oracle" and res["value"] > 0
    assert res["e2e"]["h2d_bytes_per_step"] == 0
