"""Host logic of the multi-rank bench on CPU (gloo, world size 2).

bench.py runs one replica per GPU under torchrun: no data-path collective,
the job's time is the slowest rank's and the throughput counts every rank's
units.  These tests run that logic with two gloo ranks on the CPU, and check
that the reference arm leaves all ranks but rank 0 without work.
"""
import datetime
import importlib.util
import multiprocessing as mp
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _load_bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, elapsed_ms, out):
    import torch
    import torch.distributed as dist

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        bench = _load_bench()
        env = {"WORLD_SIZE": str(world), "RANK": str(rank), "LOCAL_RANK": str(rank)}
        got_ranks = bench.ranks_from_env(env)
        mx = bench.max_over_ranks(elapsed_ms[rank], torch.device("cpu"))
        ms_step, value = bench.job_throughput(mx, 5, 8192, world)
        dist.barrier()
        out.put((rank, got_ranks, mx, ms_step, value))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_gloo_world2():
    world = 2
    elapsed = [10.0, 17.5]  # rank 1 is the slowest
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, elapsed, out)) for r in range(world)]
    for p in procs:
        p.start()
    results = sorted(out.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ranks, mx, ms_step, value in results:
        assert ranks == (world, rank, rank)
        assert mx == 17.5                      # every rank sees the slowest rank's time
        assert ms_step == pytest.approx(3.5)   # 5 timed steps
        assert value == pytest.approx(8192 * world / 3.5e-3)


def test_single_process_needs_no_process_group():
    import torch

    bench = _load_bench()
    assert bench.ranks_from_env({}) == (1, 0, 0)
    assert bench.max_over_ranks(4.25, torch.device("cpu")) == 4.25
    assert bench.job_throughput(10.0, 5, 100, 1) == pytest.approx((2.0, 50000.0))


def test_reference_arm_only_rank0_works():
    """Under torchrun the reference arm runs on rank 0 alone: another rank
    exits 0 at once and prints nothing."""
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""
