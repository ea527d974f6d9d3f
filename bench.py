"""Benchmark: causal prefill attention TFLOP/s on B200 through the C-ABI library.

One step = one pass of the whole hot path over one batch of synthetic input:
  FP8   per-tensor e4m3 quantisation of Q, K and V, then the lean-P attention kernel;
  BF16  the attention kernel.
The headline `value` is the FP8 step on the workload (default: GQA Hq=32/Hkv=8,
S=16384, d=128, outlier-channel inputs); the BF16 step is timed on the same workload
and reported under "bf16".  Throughput counts causal FLOPs 2*B*Hq*S^2/2*(d_qk+d_v).

Timing: W warm-up steps, then K steps, each bracketed by CUDA events on the launching
stream, with a 256 MiB L2 flush written between steps outside the events; a barrier and
a device synchronisation bracket the whole timed region; multi-GPU runs take the max over
ranks.  `e2e` repeats the FP8 step through the same calls with pinned host buffers: the
host->device copies of Q, K, V and the device->host copy of O are inside its timing.  Its
value pipelines K steps over three streams (the copy in of step i+1 and the copy out of
step i-1 overlap the compute of step i; time = whole region / K); `e2e.serial` times each
step's copies and compute back to back.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                       [--impl reference] [--no-cpu-baseline]
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "causal prefill attn TFLOP/s (FP8 e4m3, BF16) at 16K/32K; % of B200 tensor peak"
UNIT = "TFLOP/s"
NOMINAL_FP8_TFLOPS = 4500.0
NOMINAL_BF16_TFLOPS = 2250.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# prefill work unit and schedule (attn_select_prefill_kernel): auto (the library default:
# dynamic take-over of units, head pairs for FP8, tile pairs for BF16); a unit (tile pairs
# "single", head pairs "heads") with one CTA per unit, a static persistent grid ("-static")
# or dynamic take-over ("-dynamic")
KERNEL_IDS = {"auto": lambda pkg: pkg.ATTN_KERNEL_AUTO,
              "single": lambda pkg: pkg.ATTN_KERNEL_SINGLE,
              "heads": lambda pkg: pkg.ATTN_KERNEL_HEADS,
              "single-static": lambda pkg: pkg.ATTN_KERNEL_SINGLE | pkg.ATTN_KERNEL_PERSISTENT,
              "heads-static": lambda pkg: pkg.ATTN_KERNEL_HEADS | pkg.ATTN_KERNEL_PERSISTENT,
              "single-dynamic": lambda pkg: pkg.ATTN_KERNEL_SINGLE | pkg.ATTN_KERNEL_DYNAMIC,
              "heads-dynamic": lambda pkg: pkg.ATTN_KERNEL_HEADS | pkg.ATTN_KERNEL_DYNAMIC}

def bf16_pipeline(Hq, Hkv):
    """The BF16 prefill pipeline the library picks when no pipeline flag is selected (the
    bench selects none): S-ahead with grouped-query heads, P over S otherwise."""
    return "S-ahead" if Hq > Hkv else "P over S"


WORKLOADS = {
    # name: (B, S, Hq, Hkv, d_qk, d_v, distribution, description)
    "small_s256": (1, 256, 1, 1, 128, 128, "gaussian",
                   "causal prefill B=1 H=1 S=256 d=128, Gaussian inputs (oracle-sized case)"),
    "gqa16k_outlier": (1, 16384, 32, 8, 128, 128, "outlier",
                       "GQA causal prefill B=1 Hq=32 Hkv=8 S=16384 d=128, outlier-channel inputs"),
    "mha32k_gaussian": (1, 32768, 32, 32, 128, 128, "gaussian",
                        "causal prefill B=1 H=32 S=32768 d=128, Gaussian inputs"),
    "mla16k_outlier": (1, 16384, 16, 16, 192, 128, "outlier",
                       "MLA-shaped causal prefill B=1 H=16 S=16384 d_qk=192 d_v=128, outlier inputs"),
    "mla32k_outlier": (1, 32768, 16, 16, 192, 128, "outlier",
                       "MLA-shaped causal prefill B=1 H=16 S=32768 d_qk=192 d_v=128, outlier inputs"),
}
# decode over a paged KV cache: name -> (B, L, Hq, Hkv, page_size, description)
DECODE_WORKLOADS = {
    "decode_gqa_b64_s4k": (64, 4096, 32, 8, 64,
                           "paged decode B=64 sequences x 4096 cached tokens, Hq=32 Hkv=8 d=128, "
                           "pages of 64 tokens in shuffled order"),
    "decode_gqa_b16_s32k": (16, 32768, 32, 8, 64,
                            "paged decode B=16 sequences x 32768 cached tokens, Hq=32 Hkv=8 "
                            "d=128, pages of 64 tokens in shuffled order"),
}
DECODE_METRIC = "paged decode attention KV-cache read GB/s (FP8 e4m3, BF16); % of B200 HBM"

for _s in (1024, 2048, 4096, 8192, 16384, 32768):
    WORKLOADS[f"sweep_s{_s // 1024}k"] = (
        32768 // _s, _s, 32, 8, 128, 128, "gaussian",
        f"sweep B*S=32768 S={_s} Hq=32 Hkv=8 d=128, Gaussian inputs")


def causal_flops(B, Hq, S, d_qk, d_v):
    return 2.0 * B * Hq * S * S / 2.0 * (d_qk + d_v)


def max_over_ranks(x, world, device=None):
    """The maximum of a per-rank float over all ranks (the job's time is its slowest rank)."""
    if world == 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tflops(flops_per_rank, world, ms):
    """Whole-job throughput: every rank processes its own problem (weak scaling)."""
    return flops_per_rank * world / (ms * 1e-3) / 1e12


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def gpu_selector(dev_index):
    """The GPU as nvidia-smi / NVML name it: its UUID (they ignore CUDA_VISIBLE_DEVICES, so
    a CUDA ordinal can name another GPU), else the ordinal."""
    try:
        import torch
        u = str(torch.cuda.get_device_properties(dev_index).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return str(dev_index)


# ----------------------------------------------------------------------------- energy
def energy_summary(flops_per_call, calls, mj_start, mj_end, seconds):
    """TFLOP/J and mean power from two readings of the NVML cumulative energy counter
    (millijoules) around `calls` back-to-back launches of `flops_per_call` each."""
    joules = (mj_end - mj_start) / 1000.0
    if joules <= 0 or seconds <= 0:
        return {"tflop_per_j": None, "joules": joules, "avg_w": None, "calls": calls,
                "seconds": round(seconds, 3)}
    return {"tflop_per_j": round(flops_per_call * calls / joules / 1e12, 4),
            "joules": round(joules, 3), "avg_w": round(joules / seconds, 1), "calls": calls,
            "seconds": round(seconds, 3),
            "sustained_tflops": round(flops_per_call * calls / seconds / 1e12, 2)}


def measure_energy(nvml, handle, fn, flops_per_call, sync, seconds=3.0):
    """Run fn back to back for about `seconds` (after a warm-up of the same length, so that
    clocks and power have settled) and read the energy counter around the measured window."""
    t0 = time.perf_counter()
    n = 0
    while time.perf_counter() - t0 < seconds or n < 3:  # warm-up; also sizes the window
        fn()
        n += 1
        if n % 8 == 0:
            sync()
    sync()
    calls = max(3, int(n * seconds / max(time.perf_counter() - t0, 1e-6)))
    e0 = nvml.nvmlDeviceGetTotalEnergyConsumption(handle)
    t1 = time.perf_counter()
    for _ in range(calls):
        fn()
    sync()
    t2 = time.perf_counter()
    e1 = nvml.nvmlDeviceGetTotalEnergyConsumption(handle)
    return energy_summary(flops_per_call, calls, e0, e1, t2 - t1)


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 50 ms while active."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = []
        try:
            for line in open(self.path):
                parts = [x.strip() for x in line.split(",")]
                if len(parts) == 7:
                    rows.append(parts)
        except OSError:
            pass
        finally:
            try:
                os.unlink(self.path)
            except OSError:
                pass
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        sm = [float(r[0]) for r in rows if r[0].replace(".", "").isdigit()]
        mx = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[3 + i] == "Active"})
        # samples under load: SM clock above idle
        loaded = [x for x in sm if x > 600] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


# ----------------------------------------------------------------------------- decode leg
def gpu_bench_decode(args, rank, world, local_rank):
    """Decode over a paged KV cache: K timed calls (split + combine kernels) per precision,
    CUDA events around each call; the caches (> L2) are read once per call."""
    import torch
    import torch.distributed as dist

    import bf16_causal_prefill_attn_b200 as pkg

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    B, L, Hq, Hkv, page, desc = DECODE_WORKLOADS[args.workload]
    P = B * L // page
    gen = torch.Generator(device=dev)
    gen.manual_seed(1000 + rank)
    kc = torch.randn((P, page, Hkv, 128), generator=gen, device=dev).to(torch.bfloat16)
    vc = torch.randn((P, page, Hkv, 128), generator=gen, device=dev).to(torch.bfloat16)
    q = torch.randn((B, Hq, 128), generator=gen, device=dev).to(torch.bfloat16)
    table = torch.randperm(P, generator=gen, device=dev).to(torch.int32).reshape(B, L // page)
    lens = torch.full((B,), L, dtype=torch.int32, device=dev)
    (q8, dq), (k8, dk), (v8, dv) = [pkg.attn_quantize_e4m3(t.reshape(-1, t.shape[-2], 128))
                                    for t in (q, kc, vc)]
    k8, v8, q8 = k8.reshape(kc.shape), v8.reshape(vc.shape), q8.reshape(q.shape)
    o = torch.empty((B, Hq, 128), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, Hq), dtype=torch.float32, device=dev)
    ws_bytes = pkg.attn_decode_workspace_size(B, Hq, Hkv, L)
    ws = torch.empty((ws_bytes + 15) // 16 * 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def call_fp8():
        pkg.attn_decode_paged(q8, k8, v8, table, lens, L, descale_q=dq, descale_k=dk,
                              descale_v=dv, out=o, lse=lse, workspace=ws)

    def call_bf16():
        pkg.attn_decode_paged(q, kc, vc, table, lens, L, out=o, lse=lse, workspace=ws)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    def timed(fn, K, W):
        for _ in range(W):
            fn()
        barrier()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(K)]
        for a, b_ in evs:
            a.record(stream)
            fn()
            b_.record(stream)
        barrier()
        st = pkg.attn_device_status()
        if st != pkg.ATTN_OK:
            raise RuntimeError(f"device status {pkg.status_string(st)}")
        return statistics.mean(a.elapsed_time(b_) for a, b_ in evs)

    peaks, peak_src = load_peaks()
    with ClockSampler(gpu_selector(local_rank)) as clk:
        fp8_ms = max_over_ranks(timed(call_fp8, args.steps, args.warmup), world, dev)
        bf16_ms = max_over_ranks(timed(call_bf16, args.steps, args.warmup), world, dev)
    clocks = clk.summary()

    # e2e: the query uploaded from pinned host memory and the output read back every call
    q_h = q8.cpu().pin_memory()
    o_h = torch.empty(o.shape, dtype=o.dtype).pin_memory()

    def call_e2e():
        q8.copy_(q_h, non_blocking=True)
        call_fp8()
        o_h.copy_(o, non_blocking=True)

    e2e_ms = max_over_ranks(timed(call_e2e, args.steps, args.warmup), world, dev)

    def kv_bytes(e):
        return 2.0 * B * L * Hkv * 128 * e
    io_bytes = B * Hq * 128 * 2 + B * Hq * 4       # o (bf16) and lse written
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    flops = 2.0 * B * Hq * L * 256
    traffic = load_traffic(args.workload, "traffic_decode.json", DECODE_SOURCES)
    fp8_gbs = (kv_bytes(1) + B * Hq * 128 + io_bytes) / (fp8_ms * 1e-3) / 1e9
    bf16_gbs = (kv_bytes(2) + B * Hq * 256 + io_bytes) / (bf16_ms * 1e-3) / 1e9
    return {
        "metric": DECODE_METRIC,
        "value": round(fp8_gbs * world, 1),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(fp8_ms, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "e4m3",
        "data": "synthetic",
        "config": decode_config(args, world),
        "roofline": {"bound": "hbm", "achieved": round(fp8_gbs, 1), "peak": hbm,
                     "unit": "GB/s", "frac": round(fp8_gbs / hbm, 4),
                     "peak_source": f"{peak_src} copy bandwidth",
                     "kernel": "decode_split_kernel<fp8> + decode_combine_kernel",
                     "tflops": round(flops / (fp8_ms * 1e-3) / 1e12, 2),
                     "traffic": traffic.get("fp8"),
                     "traffic_of": "decode_split_kernel (the combine kernel reads its partials "
                                   "from L2)"},
        "bf16": {"value": round(bf16_gbs * world, 1), "unit": "GB/s",
                 "ms_per_step": round(bf16_ms, 4),
                 "roofline": {"bound": "hbm", "achieved": round(bf16_gbs, 1), "peak": hbm,
                              "unit": "GB/s", "frac": round(bf16_gbs / hbm, 4),
                              "tflops": round(flops / (bf16_ms * 1e-3) / 1e12, 2),
                              "traffic": traffic.get("bf16")}},
        "e2e": {"value": round((kv_bytes(1) + B * Hq * 128 + io_bytes) / (e2e_ms * 1e-3) / 1e9
                               * world, 1),
                "unit": "GB/s", "h2d_bytes_per_step": B * Hq * 128, "d2h_bytes_per_step":
                B * Hq * 128 * 2, "ms_per_step": round(e2e_ms, 4)},
        "gpu_launches": args.steps * 2,
        "clocks": clocks,
    }


# ----------------------------------------------------------------------------- GPU leg
def gpu_bench(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import bf16_causal_prefill_attn_b200 as pkg
    import synth

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    pkg.attn_select_prefill_kernel(KERNEL_IDS[args.kernel](pkg))
    B, S, Hq, Hkv, dqk, dv, distn, desc = WORKLOADS[args.workload]
    if args.split == "heads":
        # one problem shared by all ranks: rank r takes a contiguous range of kv heads and
        # their query heads; no data-path collective
        from bf16_causal_prefill_attn_b200 import shard
        q_h, k_h, v_h = synth.make_qkv(B, S, Hq, Hkv, dqk, dv, seed=0, dist=distn)
        q_h, k_h, v_h = shard.slice_heads(q_h, k_h, v_h, Hq, Hkv, world, rank)
        job_flops = causal_flops(B, Hq, S, dqk, dv)
        Hq, Hkv = q_h.shape[2], k_h.shape[2]
        flops = causal_flops(B, Hq, S, dqk, dv)
    else:
        q_h, k_h, v_h = synth.make_qkv(B, S, Hq, Hkv, dqk, dv, seed=rank, dist=distn)
        flops = causal_flops(B, Hq, S, dqk, dv)
        job_flops = flops * world
    q_h, k_h, v_h = q_h.pin_memory(), k_h.pin_memory(), v_h.pin_memory()
    q, k, v = q_h.to(dev), k_h.to(dev), v_h.to(dev)
    stream = torch.cuda.current_stream(dev)
    # outputs and scratch allocated once (the library never allocates)
    q8 = torch.empty(q.shape, dtype=torch.uint8, device=dev)
    k8 = torch.empty(k.shape, dtype=torch.uint8, device=dev)
    v8 = torch.empty(v.shape, dtype=torch.uint8, device=dev)
    ds = [torch.empty(1, dtype=torch.float32, device=dev) for _ in range(3)]
    ws = [torch.empty(4, dtype=torch.int32, device=dev) for _ in range(3)]
    o = torch.empty((B, S, Hq, dv), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, Hq, S), dtype=torch.float32, device=dev)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.int32, device=dev)
    o_h = torch.empty(o.shape, dtype=torch.bfloat16).pin_memory()

    def fp8_step(ev_a=None, ev_b=None):
        pkg.attn_quantize_qkv_e4m3(q, k, v, hadamard=args.hadamard, out=(q8, k8, v8),
                                   descales=ds, workspace=ws[0])
        if ev_a is not None:
            ev_a.record(stream)
        pkg.attn_fwd(q8, k8, v8, descale_q=ds[0], descale_k=ds[1], descale_v=ds[2], out=o, lse=lse,
                     unrotate=args.hadamard, exact_p=args.exact_p)
        if ev_b is not None:
            ev_b.record(stream)

    def bf16_step(ev_a=None, ev_b=None):
        if ev_a is not None:
            ev_a.record(stream)
        pkg.attn_fwd(q, k, v, out=o, lse=lse)
        if ev_b is not None:
            ev_b.record(stream)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    def timed(step, K, W):
        for _ in range(W):
            flush.zero_()
            step()
        barrier()
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K)]
        for i in range(K):
            flush.zero_()
            s0, k0, k1, s1 = evs[i]
            s0.record(stream)
            step(k0, k1)
            s1.record(stream)
        barrier()
        step_ms = [e[0].elapsed_time(e[3]) for e in evs]
        kern_ms = [e[1].elapsed_time(e[2]) for e in evs]
        st = pkg.attn_device_status()
        if st != pkg.ATTN_OK:
            raise RuntimeError(f"device status {pkg.status_string(st)}")
        return step_ms, kern_ms

    peaks, peak_src = load_peaks()
    with ClockSampler(gpu_selector(local_rank)) as clk:
        fp8_step_ms, fp8_kern_ms = timed(fp8_step, args.steps, args.warmup)
        bf16_step_ms, bf16_kern_ms = timed(bf16_step, args.steps, args.warmup)
    clocks = clk.summary()

    # end to end: pinned host buffers, H2D of the inputs and D2H of O inside the timing
    def e2e_step(ev_a=None, ev_b=None):
        q.copy_(q_h, non_blocking=True)
        k.copy_(k_h, non_blocking=True)
        v.copy_(v_h, non_blocking=True)
        fp8_step(ev_a, ev_b)
        o_h.copy_(o, non_blocking=True)

    e2e_ms, _ = timed(e2e_step, max(3, args.steps // 4), max(1, args.warmup // 2))

    # end to end, pipelined: the same calls on three streams, so that the host->device copy
    # of step i+1 and the device->host copy of step i-1 (opposite PCIe directions) overlap
    # the compute of step i.  Two device buffer sets; every step still copies its own inputs
    # in and its own result out.  Time = the whole K-step region / K.
    def e2e_pipelined(K, W):
        s_in, s_cmp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
        bufs = []
        for _ in range(2):
            bufs.append({"q": torch.empty_like(q), "k": torch.empty_like(k), "v": torch.empty_like(v),
                         "q8": torch.empty_like(q8), "k8": torch.empty_like(k8),
                         "v8": torch.empty_like(v8), "ds": [torch.empty_like(x) for x in ds],
                         "ws": [torch.empty_like(x) for x in ws], "o": torch.empty_like(o),
                         "lse": torch.empty_like(lse),
                         "o_h": torch.empty(o.shape, dtype=torch.bfloat16).pin_memory(),
                         "in": torch.cuda.Event(), "cmp": torch.cuda.Event(),
                         "out": torch.cuda.Event(), "used": False})

        def run(n):
            for i in range(n):
                bf = bufs[i % 2]
                with torch.cuda.stream(s_in):
                    if bf["used"]:
                        s_in.wait_event(bf["cmp"])       # the inputs of step i-2 were consumed
                    bf["q"].copy_(q_h, non_blocking=True)
                    bf["k"].copy_(k_h, non_blocking=True)
                    bf["v"].copy_(v_h, non_blocking=True)
                    bf["in"].record(s_in)
                with torch.cuda.stream(s_cmp):
                    s_cmp.wait_event(bf["in"])
                    if bf["used"]:
                        s_cmp.wait_event(bf["out"])      # O of step i-2 has left the device
                    pkg.attn_quantize_qkv_e4m3(bf["q"], bf["k"], bf["v"], hadamard=args.hadamard,
                                               out=(bf["q8"], bf["k8"], bf["v8"]),
                                               descales=bf["ds"], workspace=bf["ws"][0],
                                               stream=s_cmp)
                    pkg.attn_fwd(bf["q8"], bf["k8"], bf["v8"], descale_q=bf["ds"][0],
                                 descale_k=bf["ds"][1], descale_v=bf["ds"][2], out=bf["o"],
                                 lse=bf["lse"], unrotate=args.hadamard, exact_p=args.exact_p,
                                 stream=s_cmp)
                    bf["cmp"].record(s_cmp)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(bf["cmp"])
                    bf["o_h"].copy_(bf["o"], non_blocking=True)
                    bf["out"].record(s_out)
                bf["used"] = True

        run(W)
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s_in)
        s_cmp.wait_event(e0)
        s_out.wait_event(e0)
        run(K)
        s_out.wait_stream(s_in)
        s_out.wait_stream(s_cmp)
        e1.record(s_out)
        barrier()
        st = pkg.attn_device_status()
        if st != pkg.ATTN_OK:
            raise RuntimeError(f"device status {pkg.status_string(st)}")
        return e0.elapsed_time(e1) / K

    e2e_pipe_ms = e2e_pipelined(max(4, args.steps // 2), 2)

    # energy of the attention kernels at sustained clocks (NVML cumulative counter)
    energy = None
    if not args.no_energy:
        try:
            import pynvml
            pynvml.nvmlInit()
            sel = gpu_selector(local_rank)
            handle = (pynvml.nvmlDeviceGetHandleByUUID(sel) if sel.startswith("GPU-")
                      else pynvml.nvmlDeviceGetHandleByIndex(int(sel)))
            sync = lambda: torch.cuda.synchronize(dev)
            with ClockSampler(gpu_selector(local_rank)) as eclk:
                e_fp8 = measure_energy(pynvml, handle, lambda: pkg.attn_fwd(
                    q8, k8, v8, descale_q=ds[0], descale_k=ds[1], descale_v=ds[2], out=o, lse=lse,
                    unrotate=args.hadamard, exact_p=args.exact_p), flops, sync)
                e_bf16 = measure_energy(pynvml, handle, lambda: pkg.attn_fwd(q, k, v, out=o, lse=lse),
                                        flops, sync)
            energy = {"fp8": e_fp8, "bf16": e_bf16, "clocks": eclk.summary(),
                      "source": "nvmlDeviceGetTotalEnergyConsumption around back-to-back "
                                "attention launches (whole-board energy, this GPU)"}
        except Exception as exc:  # NVML missing or not permitted: report why, keep the run
            energy = {"unavailable": f"{type(exc).__name__}: {exc}"}
    h2d = sum(t.numel() * t.element_size() for t in (q_h, k_h, v_h))
    d2h = o_h.numel() * o_h.element_size()

    fp8_ms = max_over_ranks(statistics.mean(fp8_step_ms), world, dev)
    fp8_kern = max_over_ranks(statistics.mean(fp8_kern_ms), world, dev)
    bf16_ms = max_over_ranks(statistics.mean(bf16_step_ms), world, dev)
    bf16_kern = max_over_ranks(statistics.mean(bf16_kern_ms), world, dev)
    e2e_mean = max_over_ranks(statistics.mean(e2e_ms), world, dev)
    e2e_pipe = max_over_ranks(e2e_pipe_ms, world, dev)
    bf16_peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    fp8_peak = 2.0 * bf16_peak  # measured bf16 peak x the nominal fp8/bf16 ratio (2)
    fp8_kern_tf = flops / (fp8_kern * 1e-3) / 1e12
    bf16_kern_tf = flops / (bf16_kern * 1e-3) / 1e12
    # counters were taken for the lean-P kernel only
    traffic = {} if args.exact_p else load_traffic(args.workload)
    result = {
        "metric": METRIC,
        "value": round(job_tflops(job_flops, 1, fp8_ms), 2),
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(fp8_ms, 4),
        "higher_is_better": True,
        "scaling": "strong" if args.split == "heads" else "weak",
        "vs_baseline": None,
        "dtype": "e4m3",
        "data": "synthetic",
        "config": prefill_config(args, world, Hq, Hkv),
        "roofline": {"bound": "tensor", "achieved": round(fp8_kern_tf, 2),
                     "peak": round(fp8_peak, 1), "unit": "TFLOP/s",
                     "frac": round(fp8_kern_tf / fp8_peak, 4),
                     "peak_source": f"{peak_src} bf16 cuBLAS burst x2 (fp8/bf16 nominal ratio)",
                     "frac_of_nominal_4500": round(fp8_kern_tf / NOMINAL_FP8_TFLOPS, 4),
                     "kernel": "attn_fwd_kernel<fp8, exact P>" if args.exact_p else "attn_fwd_kernel<fp8>", "kernel_ms": round(fp8_kern, 4),
                     "kernel_ms_median": round(statistics.median(fp8_kern_ms), 4),
                     "kernel_ms_min": round(min(fp8_kern_ms), 4),
                     "traffic": traffic.get("fp8")},
        "bf16": {"value": round(job_tflops(job_flops, 1, bf16_ms), 2), "unit": UNIT,
                 "ms_per_step": round(bf16_ms, 4), "dtype": "bf16",
                 "roofline": {"bound": "tensor", "achieved": round(bf16_kern_tf, 2),
                              "peak": round(bf16_peak, 1), "unit": "TFLOP/s",
                              "frac": round(bf16_kern_tf / bf16_peak, 4),
                              "peak_source": f"{peak_src} bf16 cuBLAS burst",
                              "frac_of_nominal_2250": round(bf16_kern_tf / NOMINAL_BF16_TFLOPS, 4),
                              "kernel": f"attn_fwd_kernel<bf16>, {bf16_pipeline(Hq, Hkv)} pipeline",
                              "kernel_ms": round(bf16_kern, 4),
                              "kernel_ms_median": round(statistics.median(bf16_kern_ms), 4),
                              "kernel_ms_min": round(min(bf16_kern_ms), 4),
                              "traffic": traffic.get("bf16")}},
        "e2e": {"value": round(job_tflops(job_flops, 1, e2e_pipe), 2), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": round(e2e_pipe, 4),
                "mode": "K steps pipelined over three streams (inputs in, compute, result out); "
                        "time of the whole region / K",
                "serial": {"value": round(job_tflops(job_flops, 1, e2e_mean), 2),
                           "ms_per_step": round(e2e_mean, 4),
                           "mode": "each step: copies in, quantise + attention, copy out"}},
        # per FP8 step: 2 quantiser kernels + 1 attention kernel; per BF16 step: 1
        "gpu_launches": args.steps * 3 + args.steps,
        "clocks": clocks,
    }
    if energy is not None:
        result["energy"] = energy
    if world == 1 and not args.no_extras and args.workload == "gqa16k_outlier":
        with ClockSampler(gpu_selector(local_rank)) as xclk:
            extras = headline_extras(args, dev, peaks, peak_src)
        extras["clocks"] = xclk.summary()
        result["extra"] = extras
    return result


# ----------------------------------------------------------------------------- headline shapes
EXTRA_PREFILL = ("mha32k_gaussian", "mla32k_outlier", "sweep_s1k", "sweep_s4k")
EXTRA_DECODE = "decode_gqa_b64_s4k"


def headline_extras(args, dev, peaks, peak_src):
    """Kernel throughput on the pages' own headline shapes, next to the main workload:
    MHA 32 heads at S = 32768 on Gaussian inputs (FP8 and BF16), the MLA shape at
    S = 32768 (FP8) and two points of the sequence-length sweep (B * S = 32768 at S = 1024
    and 4096, FP8 and BF16), each timed over a few launches with an L2 flush between them,
    and one paged-decode workload (GB/s against the copy bandwidth)."""
    import copy

    import torch

    import bf16_causal_prefill_attn_b200 as pkg
    import synth

    bf16_peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    out = {}

    def time_kernel(fn, K=8, W=3):
        for _ in range(W):
            flush.zero_()
            fn()
        torch.cuda.synchronize(dev)
        ms = []
        for _ in range(K):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            b.synchronize()
            ms.append(a.elapsed_time(b))
        st = pkg.attn_device_status()
        if st != pkg.ATTN_OK:
            raise RuntimeError(f"device status {pkg.status_string(st)}")
        return statistics.median(ms)

    for name in EXTRA_PREFILL:
        B, S, Hq, Hkv, dqk, dv, distn, desc = WORKLOADS[name]
        flops = causal_flops(B, Hq, S, dqk, dv)
        q, k, v = [t.to(dev) for t in synth.make_qkv(B, S, Hq, Hkv, dqk, dv, seed=0, dist=distn)]
        (q8, dq), (k8, dk), (v8, dvs) = pkg.attn_quantize_qkv_e4m3(q, k, v)
        o = torch.empty((B, S, Hq, dv), dtype=torch.bfloat16, device=dev)
        lse = torch.empty((B, Hq, S), dtype=torch.float32, device=dev)
        ms8 = time_kernel(lambda: pkg.attn_fwd(q8, k8, v8, descale_q=dq, descale_k=dk,
                                               descale_v=dvs, out=o, lse=lse))
        tf8 = flops / (ms8 * 1e-3) / 1e12
        entry = {"workload": desc, "fp8": {
            "kernel_ms": round(ms8, 4), "tflops": round(tf8, 1),
            "roofline": {"bound": "tensor", "achieved": round(tf8, 1),
                         "peak": round(2 * bf16_peak, 1), "unit": "TFLOP/s",
                         "frac": round(tf8 / (2 * bf16_peak), 4),
                         "frac_of_nominal_4500": round(tf8 / NOMINAL_FP8_TFLOPS, 4),
                         "peak_source": f"{peak_src} bf16 cuBLAS burst x2"}}}
        if dqk == 128:
            msb = time_kernel(lambda: pkg.attn_fwd(q, k, v, out=o, lse=lse))
            tfb = flops / (msb * 1e-3) / 1e12
            entry["bf16"] = {"kernel_ms": round(msb, 4), "tflops": round(tfb, 1),
                             "roofline": {"bound": "tensor", "achieved": round(tfb, 1),
                                          "peak": round(bf16_peak, 1), "unit": "TFLOP/s",
                                          "frac": round(tfb / bf16_peak, 4),
                                          "frac_of_nominal_2250": round(tfb / NOMINAL_BF16_TFLOPS, 4),
                                          "peak_source": f"{peak_src} bf16 cuBLAS burst",
                                          "kernel": f"attn_fwd_kernel<bf16>, {bf16_pipeline(Hq, Hkv)} pipeline"}}
        out[name] = entry
        del q, k, v, q8, k8, v8, o, lse
        torch.cuda.empty_cache()
    da = copy.copy(args)
    da.workload, da.steps, da.warmup = EXTRA_DECODE, 10, 3
    d = gpu_bench_decode(da, 0, 1, dev.index)
    out[EXTRA_DECODE] = {"workload": d["config"]["workload"], "fp8": d["roofline"],
                         "bf16": d["bf16"]["roofline"]}
    return out


PREFILL_SOURCES = ("attn_fwd.cuh", "ptx.cuh")
DECODE_SOURCES = ("decode.cuh", "ptx.cuh")


def kernel_source_hash(names=PREFILL_SOURCES):
    """Hash of a kernel's sources, to tie ncu counters to the code measured."""
    import hashlib
    h = hashlib.sha256()
    for name in names:
        with open(os.path.join(ROOT, "bf16_causal_prefill_attn_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def load_traffic(workload, fname="traffic.json", names=PREFILL_SOURCES):
    """DRAM bytes (read + write) per launch from the committed ncu summary, if it covers
    this workload and the current kernel source; otherwise null."""
    p = os.path.join(ROOT, "profiles", fname)
    try:
        with open(p) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return {}
    if d.get("kernel_source_hash") != kernel_source_hash(names):
        return {}
    return d.get("workloads", {}).get(workload, {})


# ----------------------------------------------------------------------------- CPU leg
_CPU_CACHE = {}


def cpu_model():
    """The host CPU's model name (first 'model name' entry of /proc/cpuinfo)."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        return os.cpu_count() or 1


def cpu_reference(workload, budget_s, rank=0):
    """The oracle (fp64 attention on the dequantised FP8 inputs), as it stands, on this
    host's cores, on a stratified sample of the workload: passes over every (batch, head)
    slice, each pass taking every 64th query row from an offset (0, 32, 16, 48, 8, ... --
    the first pass also the last row), until the time budget is spent (at least one pass
    of one slice).  The value is the sample's causal FLOPs (sum over the sampled rows of
    2 (i + 1) (d_qk + d_v)) over its time, i.e. the full problem's time extrapolated by the
    exact causal row-cost ratio.  The e4m3 codes of the whole tensors are made once and each
    slice is dequantised before its timing starts."""
    import numpy as np

    import synth
    from oracle import attention, quantize

    B, S, Hq, Hkv, dqk, dv, distn, desc = WORKLOADS[workload]
    key = (workload, rank)
    if key not in _CPU_CACHE:
        q, k, v = synth.make_qkv(B, S, Hq, Hkv, dqk, dv, seed=rank, dist=distn)
        _CPU_CACHE[key] = [quantize.quantize_e4m3(t.float().numpy()) for t in (q, k, v)]
    (qc, dq), (kc, dk), (vc, dvs) = _CPU_CACHE[key]
    G = Hq // Hkv
    order = np.random.default_rng(0).permutation(B * Hq)
    # row offsets in bit-reversed order, so every prefix of passes is spread over the rows
    offsets = [int(f"{i:06b}"[::-1], 2) for i in range(64)]
    done_flops, dt, slices, rows_done, passes = 0.0, 0.0, 0, 0, 0
    for off in offsets:
        rows = np.arange(off, S, 64)
        if off == 0:
            rows = np.unique(np.append(rows, S - 1))
        if rows.size == 0:
            continue
        row_flops = float(sum(2.0 * (int(i) + 1) * (dqk + dv) for i in rows))
        for idx in order:
            b, h = divmod(int(idx), Hq)
            g = h // G
            qd = quantize.dequantize(qc[b:b + 1, :, h:h + 1], dq)
            kd = quantize.dequantize(kc[b:b + 1, :, g:g + 1], dk)
            vd = quantize.dequantize(vc[b:b + 1, :, g:g + 1], dvs)
            t0 = time.perf_counter()
            attention.causal_attention_rows(qd, kd, vd, rows, [0], batch=0)
            dt += time.perf_counter() - t0
            done_flops += row_flops
            rows_done += rows.size
            slices += 1
            if dt >= budget_s:
                break
        passes += 1
        if dt >= budget_s:
            break
    return {"value": done_flops / dt / 1e12, "unit": UNIT, "cores": oracle_threads(),
            "cpu_model": cpu_model(), "kind": "oracle",
            "sample": f"{rows_done} causal query rows of {desc}: {passes} stratified pass(es) "
                      f"of every 64th row from an offset over the {B * Hq} (batch, head) "
                      f"slices ({slices} slice visits); fp64, all visible keys; {dt:.1f} s; "
                      "time extrapolated to the whole problem by the causal row-cost ratio; "
                      "input generation, quantisation and dequantisation not timed",
            "seconds": dt}


def cpu_reference_decode(workload, budget_s):
    """The decode oracle (fp64, paged gather + softmax per head), as it stands, on a bounded
    sample: sequences of the workload's length and heads, each with its own query, over one
    synthetic cache (made before the timing); value in GB/s of the FP8 KV bytes it stands
    for, like the GPU line."""
    import numpy as np

    from oracle import decode

    B, L, Hq, Hkv, page, desc = DECODE_WORKLOADS[workload]
    rng = np.random.default_rng(0)
    P = L // page
    kc = rng.standard_normal((P, page, Hkv, 128))
    vc = rng.standard_normal((P, page, Hkv, 128))
    table = rng.permutation(P).astype(np.int32)[None]
    lens = np.array([L], dtype=np.int32)
    n = 0
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < budget_s or n == 0:
        q = rng.standard_normal((1, Hq, 128))
        decode.decode_attention(q, kc, vc, table, lens, page)
        n += 1
    dt = time.perf_counter() - t0
    return {"value": n * 2.0 * L * Hkv * 128 / dt / 1e9, "unit": "GB/s",
            "cores": oracle_threads(), "cpu_model": cpu_model(), "kind": "oracle",
            "sample": f"{n} sequences of {L} cached tokens (all {Hq} query heads each) of "
                      f"{desc}; {dt:.1f} s; cache generation not timed",
            "seconds": dt}


def decode_config(args, world):
    """The `config` object of a decode line (the same for the GPU arm and the reference arm)."""
    B, L, Hq, Hkv, page, desc = DECODE_WORKLOADS[args.workload]
    kv = lambda e: 2.0 * B * L * Hkv * 128 * e
    return {"workload": desc, "name": args.workload, "B": B, "L": L, "Hq": Hq, "Hkv": Hkv,
            "d": 128, "page_size": page,
            "step": "one decode call (split-KV kernel + combine kernel)",
            "l2": f"no flush: the caches ({kv(1) / 1e9:.2f} GB FP8, "
                  f"{kv(2) / 1e9:.2f} GB BF16) exceed the 126 MB L2",
            "parallelism": f"replicas x{world} (independent problems per GPU)"}


def prefill_config(args, world, rank_hq, rank_hkv):
    """The `config` object of a prefill line (the same for the GPU arm and the reference
    arm); rank_hq / rank_hkv: the heads one rank computes."""
    B, S, Hq, Hkv, dqk, dv, distn, desc = WORKLOADS[args.workload]
    return {"workload": desc, "name": args.workload, "B": B, "S": S, "Hq": Hq, "Hkv": Hkv,
            "d_qk": dqk, "d_v": dv, "hadamard": bool(args.hadamard),
            "kernel": args.kernel,
            "step": "e4m3 quantisation of Q, K, V + "
                    + ("exact-P attention (ablation)" if args.exact_p else "lean-P attention"),
            "l2": "256 MiB L2 flush written between steps, outside the timed step",
            "parallelism": (f"heads split x{world} (one problem; each GPU {rank_hkv} kv heads "
                            f"and their {rank_hq} query heads; no data-path collective)"
                            if args.split == "heads" else
                            f"replicas x{world} (independent problems per GPU)")}


def reference_main(args, rank, world):
    if rank != 0:
        return 0
    budget = max(1.0, 20.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        cpu_reference(args.workload, budget / 4)
    vals, secs = [], 0.0
    last = None
    for _ in range(args.steps):
        last = cpu_reference(args.workload, budget)
        vals.append(last["value"])
        secs += last["seconds"]
    B, S, Hq, Hkv, dqk, dv, distn, desc = WORKLOADS[args.workload]
    rank_hq, rank_hkv = Hq, Hkv
    if args.split == "heads":
        from bf16_causal_prefill_attn_b200 import shard
        kv_lo, kv_hi, q_lo, q_hi = shard.head_partition(Hq, Hkv, world, 0)
        rank_hq, rank_hkv = q_hi - q_lo, kv_hi - kv_lo
    value = statistics.mean(vals)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": secs * 1e3 / max(1, args.steps), "higher_is_better": True,
            "scaling": "strong" if args.split == "heads" else "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic",
            "config": prefill_config(args, world, rank_hq, rank_hkv),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": last["cores"],
                             "cpu_model": last["cpu_model"], "kind": "oracle",
                             "sample": last["sample"]},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="gqa16k_outlier",
                    choices=sorted(WORKLOADS) + sorted(DECODE_WORKLOADS))
    ap.add_argument("--hadamard", action="store_true")
    ap.add_argument("--no-energy", action="store_true",
                    help="skip the NVML energy windows (about 12 s of extra GPU time)")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the headline shapes (MHA 32K, MLA 32K, paged decode) timed after "
                         "the default workload")
    ap.add_argument("--exact-p", action="store_true",
                    help="FP8 probabilities by exponential + e4m3 rounding (the ablation of lean P)")
    ap.add_argument("--kernel", default="auto", choices=list(KERNEL_IDS),
                    help="work unit and schedule of the prefill kernel (default: the "
                         "library's automatic choice)")
    ap.add_argument("--split", default="replicas", choices=["replicas", "heads"],
                    help="multi-GPU: an independent problem per GPU (weak scaling), or one "
                         "problem divided by kv heads (strong scaling)")
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3
    if args.split == "heads" and args.workload in WORKLOADS:
        world_ = int(os.environ.get("WORLD_SIZE", "1"))
        if world_ > WORKLOADS[args.workload][3]:
            ap.error("--split heads needs at most Hkv GPUs")
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if args.workload in DECODE_WORKLOADS:
            if rank == 0:
                c = cpu_reference_decode(args.workload, min(args.cpu_seconds, 20.0))
                c.pop("seconds", None)
                B, L, Hq, Hkv, page, desc = DECODE_WORKLOADS[args.workload]
                print(json.dumps({"impl": "reference", "metric": DECODE_METRIC,
                                  "value": c["value"], "unit": "GB/s", "n_gpus": world,
                                  "steps": args.steps, "warmup": args.warmup,
                                  "higher_is_better": True, "scaling": "weak",
                                  "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                                  "config": decode_config(args, world),
                                  "cpu_baseline": c,
                                  "e2e": {"value": c["value"], "unit": "GB/s",
                                          "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}),
                      flush=True)
            return 0
        return reference_main(args, rank, world)
    # the oracle baseline is measured before any CUDA call (no fork after CUDA init)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        if args.workload in WORKLOADS:
            cpu = cpu_reference(args.workload, args.cpu_seconds)
        else:
            cpu = cpu_reference_decode(args.workload, min(args.cpu_seconds, 10.0))
        cpu.pop("seconds", None)
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        if args.workload in DECODE_WORKLOADS:
            res = gpu_bench_decode(args, rank, world, local_rank)
        else:
            res = gpu_bench(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    if rank == 0:
        res["cpu_baseline"] = cpu
        print(json.dumps(res), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
