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


class _FakeNVML:
    """Stands in for pynvml: a cumulative energy counter (millijoules) that grows by a fixed
    amount per reading."""

    def __init__(self, step_mj):
        self.mj = 1_000_000
        self.step = step_mj

    def nvmlDeviceGetTotalEnergyConsumption(self, handle):
        self.mj += self.step
        return self.mj


def test_energy_summary_and_window_with_fake_nvml():
    e = bench.energy_summary(1e12, 10, 5000, 7000, 0.5)    # 2 J for 10 TFLOP
    assert e["tflop_per_j"] == 5.0 and e["avg_w"] == 4.0 and e["joules"] == 2.0
    assert bench.energy_summary(1e12, 10, 7000, 7000, 0.5)["tflop_per_j"] is None
    calls = []
    nv = _FakeNVML(step_mj=250)
    r = bench.measure_energy(nv, None, lambda: calls.append(1), 2e11, lambda: None, seconds=0.05)
    # one counter step between the two readings: 0.25 J for r["calls"] launches
    assert r["joules"] == 0.25 and r["calls"] >= 3
    assert abs(r["tflop_per_j"] - 2e11 * r["calls"] / 0.25 / 1e12) < 1e-3
    assert len(calls) > r["calls"]   # the warm-up ran first


def test_decode_reference_arm_prints_one_line():
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
           "--workload", "decode_gqa_b64_s4k", "--steps", "1", "--warmup", "3",
           "--cpu-seconds", "0.5"]
    res = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert res.returncode == 0, res.stderr
    lines = [l for l in res.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "GB/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["d2h_bytes_per_step"] == 0


def test_reference_arm_under_two_ranks_prints_once():
    """Launched like the multi-GPU bench (torchrun, 2 ranks): rank 0 alone runs the oracle
    and prints one line for the whole job; rank 1 exits 0 without work."""
    port = 29700 + os.getpid() % 200
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "small_s256",
           "--gpus", "2", "--steps", "1", "--warmup", "3"]
    res = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [l for l in res.stdout.splitlines() if l.strip().startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0


def _shard_main(rank, world, port, out):
    """Each rank computes its slice of one problem with the fp64 oracle; rank 0 gathers the
    slices over gloo and checks them against the whole problem."""
    import numpy as np
    import torch

    import synth
    from bf16_causal_prefill_attn_b200 import shard
    from oracle import attention

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, S, Hq, Hkv = 1, 96, 12, 3
        q, k, v = synth.make_qkv(B, S, Hq, Hkv, 16, 16, seed=4)
        kv_lo, kv_hi, q_lo, q_hi = shard.head_partition(Hq, Hkv, world, rank)
        qs, ks, vs = shard.slice_heads(q, k, v, Hq, Hkv, world, rank)
        o, _ = attention.causal_attention(qs.float().numpy(), ks.float().numpy(),
                                          vs.float().numpy())
        ranges = [None] * world
        dist.all_gather_object(ranges, (q_lo, q_hi, kv_lo, kv_hi))
        parts = [None] * world
        dist.all_gather_object(parts, o)
        if rank == 0:
            heads = [h for lo, hi, _, _ in ranges for h in range(lo, hi)]
            full, _ = attention.causal_attention(q.float().numpy(), k.float().numpy(),
                                                 v.float().numpy())
            got = np.concatenate([p_ for p_ in parts if p_.shape[2]], axis=2)
            out["heads"] = heads
            out["max_err"] = float(np.abs(got - full).max())
    finally:
        dist.destroy_process_group()


def test_head_split_gloo_world2_covers_every_head_once():
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    port = 30500 + os.getpid() % 1000
    procs = [ctx.Process(target=_shard_main, args=(r, 2, port, out)) for r in range(2)]
    for p_ in procs:
        p_.start()
    for p_ in procs:
        p_.join(timeout=180)
        assert p_.exitcode == 0
    assert out["heads"] == list(range(12))         # every query head once, in order
    assert out["max_err"] == 0.0                   # slices reassemble the whole problem


def test_head_partition_edge_cases():
    from bf16_causal_prefill_attn_b200 import shard
    for Hq, Hkv in ((32, 8), (32, 32), (16, 16), (12, 3)):
        for world in (1, 2, 3, 4, 8, 9):
            got = [shard.head_partition(Hq, Hkv, world, r) for r in range(world)]
            kv = [h for lo, hi, _, _ in got for h in range(lo, hi)]
            qh = [h for _, _, lo, hi in got for h in range(lo, hi)]
            assert kv == list(range(Hkv)) and qh == list(range(Hq))
            sizes = [hi - lo for lo, hi, _, _ in got]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard.head_partition(6, 4, 2, 0)
    with pytest.raises(ValueError):
        shard.head_partition(8, 4, 2, 2)
