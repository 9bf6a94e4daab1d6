"""Host logic of the multi-process benchmark, on CPU ranks over gloo.

bench.py runs one process per GPU; with N > 1 every rank runs its own
replica of the workload and the job's time is the slowest rank's. These
tests run that logic with world_size 2 on the CPU (no GPU, no NCCL)."""

import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, out):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = bench.max_over_ranks(times[rank], world, torch.device("cpu"))
        out.put((rank, ms, bench.job_value(1000.0, world, ms)))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_value_gloo():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    times = [2.5, 4.0]
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, times, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # every rank sees the slowest rank's time; the job value counts both ranks' work
    assert [g[1] for g in got] == [4.0, 4.0]
    assert all(g[2] == pytest.approx(2 * 1000.0 / 4e-3) for g in got)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.0, 1, None) == 3.0
    assert bench.job_value(10.0, 1, 1.0) == pytest.approx(1e4)


def _run_bench(env_extra, args):
    env = dict(os.environ, IQ8R_REF_BUDGET_S="2", **env_extra)
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + args, env=env, cwd=ROOT,
                          capture_output=True, text=True, timeout=300)


def test_reference_arm_rank0_prints_other_ranks_exit_quietly():
    args = ["--impl", "reference", "--gpus", "2", "--steps", "2", "--warmup", "3", "--config", "pr1"]
    r1 = _run_bench({"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"}, args)
    assert r1.returncode == 0 and r1.stdout.strip() == ""
    r0 = _run_bench({"RANK": "0", "WORLD_SIZE": "2", "LOCAL_RANK": "0"}, args)
    assert r0.returncode == 0, r0.stderr
    line = json.loads(r0.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "GB/s"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["unit"] == line["unit"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["value"] > 0
