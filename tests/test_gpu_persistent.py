"""The multi-unit schedules against one CTA per unit: the static persistent grid (one CTA
per SM running a list of units) and the dynamic one (CTAs taking over the units of CTAs not
yet started, by cluster launch control).  A unit is computed by the same code whichever
CTA runs it, so outputs, lse and the lean-P dumps must be bitwise identical.  Small static
grids (down to a single CTA running every unit) carry the per-slot phase counts, the K/V
ring positions, the unit queue and the Q hand-over through many units; problems with more
units than SMs make the dynamic schedule take units over."""
import numpy as np
import pytest
import torch

import bf16_causal_prefill_attn_b200 as pkg
import synth

pytestmark = pytest.mark.gpu

CAPS = [1, 2, 7, 0]   # 0: one CTA per SM


def _run(fn, kernel, cap):
    pkg.attn_select_prefill_kernel(kernel)
    pkg.attn_selftest_max_ctas(cap)
    try:
        out = fn()
        torch.cuda.synchronize()
        assert pkg.attn_device_status() == pkg.ATTN_OK
        return out
    finally:
        pkg.attn_select_prefill_kernel(pkg.ATTN_KERNEL_AUTO)
        pkg.attn_selftest_max_ctas(0)


def _same(a, b):
    """Bitwise equality (the dumps hold a NaN fill where nothing is written)."""
    for x, y in zip(a, b):
        if x is None:
            assert y is None
        else:
            assert x.dtype == y.dtype and x.shape == y.shape
            assert torch.equal(x.contiguous().view(torch.uint8), y.contiguous().view(torch.uint8))


@pytest.mark.parametrize("unit", ["single", "heads"])
@pytest.mark.parametrize("B,S,Hq,Hkv,dqk,causal,fp8", [
    (2, 640, 4, 2, 128, True, True),      # odd tile count: units with one slot
    (2, 640, 4, 2, 128, True, False),
    (1, 512, 4, 4, 192, True, True),      # MLA head dimension
    (3, 384, 6, 2, 128, False, False),    # full attention, G = 3
    (4, 1024, 8, 2, 128, True, True),     # 128 units: several per CTA at every cap
    (8, 1024, 8, 2, 128, True, False),    # 256 units: more than SMs (dynamic take-over)
    (8, 1024, 8, 2, 128, True, True),
])
def test_persistent_equals_one_cta_per_unit(unit, B, S, Hq, Hkv, dqk, causal, fp8):
    q, k, v = [t.cuda() for t in synth.make_qkv(B, S, Hq, Hkv, dqk, 128, seed=S + Hq, dist="outlier")]
    args = {}
    if fp8:
        (q, dq), (k, dk), (v, dv) = pkg.attn_quantize_qkv_e4m3(q, k, v)
        args = dict(descale_q=dq, descale_k=dk, descale_v=dv)
    fn = lambda: pkg.attn_fwd(q, k, v, causal=causal, **args)
    u = pkg.ATTN_KERNEL_HEADS if unit == "heads" else pkg.ATTN_KERNEL_SINGLE
    ref = _run(fn, u, 0)
    for cap in CAPS:
        _same(_run(fn, u | pkg.ATTN_KERNEL_PERSISTENT, cap), ref)
    for _ in range(3):   # which CTA takes which unit varies from run to run
        _same(_run(fn, u | pkg.ATTN_KERNEL_DYNAMIC, 0), ref)


@pytest.mark.parametrize("fp8", [False, True])
def test_persistent_varlen_equals_one_cta_per_unit(fp8):
    """Packed sequences with empty, one-token and ragged members: the units that a short
    sequence lacks are skipped by every role of the CTA alike."""
    lengths = [129, 1, 300, 0, 128, 64, 513, 127, 0, 700] * 6
    lead, tail, Hq, Hkv = 16, 40, 4, 2
    T = lead + sum(lengths) + tail
    q, k, v = [t[0].cuda() for t in synth.make_qkv(1, T, Hq, Hkv, 128, 128, seed=5, dist="gaussian")]
    cu = torch.from_numpy(np.concatenate([[lead], lead + np.cumsum(lengths)]).astype(np.int32)).cuda()
    args = {}
    if fp8:
        (q, dq), (k, dk), (v, dv) = pkg.attn_quantize_qkv_e4m3(q, k, v)
        args = dict(descale_q=dq, descale_k=dk, descale_v=dv)

    def fn():
        o = torch.full((T, Hq, 128), 7.0, dtype=torch.bfloat16, device="cuda")
        lse = torch.full((Hq, T), 7.0, dtype=torch.float32, device="cuda")
        pkg.attn_fwd_varlen(q, k, v, cu, max(lengths), causal=True, out=o, lse=lse, **args)
        return o, lse

    ref = _run(fn, pkg.ATTN_KERNEL_SINGLE, 0)
    for cap in CAPS:
        _same(_run(fn, pkg.ATTN_KERNEL_SINGLE | pkg.ATTN_KERNEL_PERSISTENT, cap), ref)
        _same(_run(fn, pkg.ATTN_KERNEL_HEADS | pkg.ATTN_KERNEL_PERSISTENT, cap), ref)
    for u in (pkg.ATTN_KERNEL_SINGLE, pkg.ATTN_KERNEL_HEADS):
        _same(_run(fn, u | pkg.ATTN_KERNEL_DYNAMIC, 0), ref)


def test_persistent_dump_equals_one_cta_per_unit():
    """Raw scores, lean-P codes and shifts of every row from the test-only dump."""
    q, k, v = [t.cuda() for t in synth.make_qkv(2, 384, 2, 1, 128, 128, seed=3, dist="outlier")]
    (q8, dq), (k8, dk), (v8, dv) = pkg.attn_quantize_qkv_e4m3(q, k, v)
    fn = lambda: pkg.attn_fwd_fp8_dump(q8, k8, v8, dq, dk, dv, causal=True)
    ref = _run(fn, pkg.ATTN_KERNEL_SINGLE, 0)
    for cap in (1, 3):
        _same(_run(fn, pkg.ATTN_KERNEL_SINGLE | pkg.ATTN_KERNEL_PERSISTENT, cap), ref)
    _same(_run(fn, pkg.ATTN_KERNEL_SINGLE | pkg.ATTN_KERNEL_DYNAMIC, 0), ref)



@pytest.mark.parametrize("B,S,Hq,Hkv,dqk,causal", [
    (2, 640, 4, 2, 128, True),      # grouped heads (S-ahead by default), odd tile count
    (2, 512, 4, 4, 128, True),      # a kv head per query head (P over S by default)
    (1, 512, 4, 4, 192, True),      # MLA head dimension
    (3, 384, 6, 2, 128, False),     # full attention, G = 3
    (8, 1024, 8, 2, 128, True),     # more units than SMs
])
def test_bf16_pipelines_equal(B, S, Hq, Hkv, dqk, causal):
    """The two BF16 pipelines (S ahead of PV on its own warp, P in TMEM columns of its own;
    P written over S, PV then S from one warp) issue the same MMAs in the same order per
    slot on the same P: outputs and lse are bitwise identical, on every unit and schedule."""
    q, k, v = [t.cuda() for t in synth.make_qkv(B, S, Hq, Hkv, dqk, 128, seed=S + 7 * Hq, dist="outlier")]
    fn = lambda: pkg.attn_fwd(q, k, v, causal=causal)
    ref = _run(fn, pkg.ATTN_KERNEL_SINGLE | pkg.ATTN_KERNEL_BF16_P_OVER_S, 0)
    for u in (pkg.ATTN_KERNEL_SINGLE, pkg.ATTN_KERNEL_HEADS):
        for pipe in (pkg.ATTN_KERNEL_BF16_S_AHEAD, pkg.ATTN_KERNEL_BF16_P_OVER_S):
            _same(_run(fn, u | pipe, 0), ref)
            _same(_run(fn, u | pipe | pkg.ATTN_KERNEL_DYNAMIC, 0), ref)
            for cap in (1, 3):
                _same(_run(fn, u | pipe | pkg.ATTN_KERNEL_PERSISTENT, cap), ref)
    _same(_run(fn, pkg.ATTN_KERNEL_AUTO, 0), ref)


@pytest.mark.parametrize("Hq,Hkv", [(4, 2), (4, 4)])
def test_bf16_pipelines_equal_varlen(Hq, Hkv):
    """The same for packed sequences with empty, one-token and ragged members."""
    lengths = [129, 1, 300, 0, 128, 64, 513, 127, 0, 700] * 3
    lead, tail = 16, 40
    T = lead + sum(lengths) + tail
    q, k, v = [t[0].cuda() for t in synth.make_qkv(1, T, Hq, Hkv, 128, 128, seed=9, dist="gaussian")]
    cu = torch.from_numpy(np.concatenate([[lead], lead + np.cumsum(lengths)]).astype(np.int32)).cuda()

    def fn():
        o = torch.full((T, Hq, 128), 7.0, dtype=torch.bfloat16, device="cuda")
        lse = torch.full((Hq, T), 7.0, dtype=torch.float32, device="cuda")
        pkg.attn_fwd_varlen(q, k, v, cu, max(lengths), causal=True, out=o, lse=lse)
        return o, lse

    ref = _run(fn, pkg.ATTN_KERNEL_SINGLE | pkg.ATTN_KERNEL_BF16_P_OVER_S, 0)
    for pipe in (pkg.ATTN_KERNEL_BF16_S_AHEAD, pkg.ATTN_KERNEL_BF16_P_OVER_S):
        for u in (pkg.ATTN_KERNEL_SINGLE, pkg.ATTN_KERNEL_HEADS):
            _same(_run(fn, u | pipe | pkg.ATTN_KERNEL_DYNAMIC, 0), ref)
            _same(_run(fn, u | pipe | pkg.ATTN_KERNEL_PERSISTENT, 2), ref)
