"""Host logic of the bench: the multi-rank aggregation over gloo (world size 2, CPU), the
whole-job throughput, and the reference arm (the oracle timed on the CPU)."""
import json
import os
import subprocess
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # each rank times its own replica; the job's time is the slowest rank's
        ms = bench.max_over_ranks(1.5 + rank, world)
        out[rank] = (ms, bench.job_tflops(1e12, world, ms))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    port = 29500 + os.getpid() % 1000
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p_ in procs:
        p_.start()
    for p_ in procs:
        p_.join(timeout=120)
        assert p_.exitcode == 0
    assert out[0] == out[1]
    ms, tf = out[0]
    assert ms == 2.5
    assert tf == pytest.approx(2 * 1e12 / 2.5e-3 / 1e12)


def test_single_rank_helpers():
    assert bench.max_over_ranks(3.0, 1) == 3.0
    assert bench.causal_flops(1, 32, 16384, 128, 128) == pytest.approx(2.199023255552e12)
    assert bench.job_tflops(1e12, 1, 1.0) == pytest.approx(1000.0)


def test_reference_arm_prints_one_line():
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
           "--workload", "small_s256", "--steps", "1", "--warmup", "3"]
    res = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert res.returncode == 0, res.stderr
    lines = [l for l in res.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "TFLOP/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0
