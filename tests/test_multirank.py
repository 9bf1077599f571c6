"""Host logic of the multi-GPU benchmark path, run as world-size-2 gloo ranks on CPU.

The layer shards by sequence with no exchange: N ranks run N independent replicas,
and the job's time for a step is the slowest rank's.  These tests check that
aggregation (max over ranks, whole-job tokens/s), that the reference arm does its
work on rank 0 only, and the launch-size validation, without a GPU."""

import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import torch.distributed as dist
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = [3.0, 5.0][rank]  # rank 1 is the slower one
        ms_job = bench.max_over_ranks(ms, world, "cpu")
        tps = bench.job_tokens_per_s(world, 16, ms_job)
        dist.barrier()
        q.put((rank, ms_job, tps))
    finally:
        dist.destroy_process_group()


def test_two_rank_aggregation_takes_the_slowest_rank():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, ms_job, tps in res:
        assert ms_job == 5.0
        assert tps == pytest.approx(2 * 16 / 5e-3)


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(7.5, 1, "cpu") == 7.5
    assert bench.job_tokens_per_s(1, 16, 2.0) == pytest.approx(8000.0)


def _run_bench(env_extra, *args, timeout=300):
    env = dict(os.environ, **env_extra)
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], env=env, cwd=ROOT,
                          capture_output=True, text=True, timeout=timeout)


def test_reference_arm_runs_on_rank_zero_only():
    r = _run_bench({"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"}, "--impl", "reference", "--gpus", "2",
                   "--steps", "1", "--warmup", "0")
    assert r.returncode == 0
    assert r.stdout.strip() == ""


def test_gpu_count_must_match_world_size():
    r = _run_bench({"RANK": "0", "WORLD_SIZE": "1", "LOCAL_RANK": "0"}, "--gpus", "2", "--steps", "1",
                   "--warmup", "3")
    assert r.returncode != 0
    assert "WORLD_SIZE" in (r.stderr + r.stdout)
