"""Host logic of the multi-process benchmark on CPU: two gloo ranks take the
slowest rank's time and report whole-job throughput; the reference arm runs
on rank 0 only (the other ranks exit at once, with no output)."""
from __future__ import annotations

import os
import subprocess
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    sys.path.insert(0, ROOT)
    import bench
    import torch
    ms = [3.0, 5.0][rank]
    got = bench.max_over_ranks(ms, world, torch.device("cpu"))
    value = bench.whole_job_value(world, 10, 1e9, got / 1e3, 1e9)
    q.put((rank, got, value))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 1000
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [5.0, 5.0]
    # 2 ranks x 10 steps x 1 GB in 5 ms
    assert all(r[2] == pytest.approx(2 * 10 * 1.0 / 0.005) for r in res)


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "0"], cwd=ROOT, env=env,
                         capture_output=True, text=True, timeout=300)
    assert out.returncode == 0 and out.stdout.strip() == ""


def test_cpu_baseline_reports_all_threads_and_one():
    """The benchmark's oracle baseline on a small workload: a value on all
    threads and one on a single thread, both positive, threads restored."""
    sys.path.insert(0, ROOT)
    import bench
    import oracle
    import synth.workloads as W
    cb, per_pass = bench.cpu_baseline(W.PR1, W.PR1.Ms, 0.5)
    assert cb["value"] > 0 and cb["single_thread"]["value"] > 0 and per_pass > 0
    assert cb["kind"] == "oracle" and cb["cores"] == oracle.Oracle().threads()
    assert cb["quantize_s"] > 0


def test_cpu_baseline_prefill_unit():
    """A TFLOP/s workload reports its CPU baseline in TFLOP/s (tiny sample)."""
    import dataclasses

    import bench
    import synth.workloads as W
    small = dataclasses.replace(W.PREFILL, N=64, K=512, Ms=(1024,))
    cb, _ = bench.cpu_baseline(small, small.Ms, 0.2)
    assert cb["unit"] == "TFLOP/s" and cb["value"] > 0
    assert cb["single_thread"]["unit"] == "TFLOP/s"
