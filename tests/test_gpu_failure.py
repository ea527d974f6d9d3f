"""Failure detection on the GPU without a fault: bounded waits that run out report
ATTN_ERR_TIMEOUT through the device error word, and the context stays usable."""
import numpy as np
import pytest
import torch

import bf16_causal_prefill_attn_b200 as pkg
import synth
from oracle import attention

pytestmark = pytest.mark.gpu


def _small_case():
    q, k, v = synth.make_qkv(1, 256, 2, 1, 128, 128, seed=77)
    ref, _ = attention.causal_attention(q.float().numpy(), k.float().numpy(), v.float().numpy())
    return (q.cuda(), k.cuda(), v.cuda()), ref


def test_wait_on_a_flag_nothing_sets_times_out():
    assert pkg.attn_device_status() == pkg.ATTN_OK
    pkg.attn_selftest_wait_timeout(2_000_000)  # 2 ms
    assert pkg.attn_device_status() == pkg.ATTN_ERR_TIMEOUT
    # reported once, then cleared
    assert pkg.attn_device_status() == pkg.ATTN_OK
    # the context still works
    (q, k, v), ref = _small_case()
    o, _ = pkg.attn_fwd(q, k, v)
    assert pkg.attn_device_status() == pkg.ATTN_OK
    assert np.abs(o.float().cpu().numpy() - ref).max() <= 1e-2


@pytest.mark.usefixtures("prefill_kernel")
@pytest.mark.parametrize("fp8", [False, True])
def test_attention_unwinds_when_its_waits_run_out(fp8):
    """The load warp stops before key tile 1, so the MMA warp's wait for that tile can never
    be satisfied: it must give up after the 1 ms limit, the kernel must report
    ATTN_ERR_TIMEOUT and unwind, and the next launch must be correct."""
    (q, k, v), ref = _small_case()
    args = {}
    if fp8:
        (q8, dq), (k8, dk), (v8, dv) = [pkg.attn_quantize_e4m3(t) for t in (q, k, v)]
        q, k, v = q8, k8, v8
        args = dict(descale_q=dq, descale_k=dk, descale_v=dv)
    o = torch.full((1, 256, 2, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    pkg.attn_set_wait_timeout_ns(1_000_000)
    pkg.attn_selftest_stall_tile(1)
    try:
        pkg.attn_fwd(q, k, v, out=o, **args)
        st = pkg.attn_device_status()
    finally:
        pkg.attn_selftest_stall_tile(-1)
        pkg.attn_set_wait_timeout_ns(0)
    assert st == pkg.ATTN_ERR_TIMEOUT
    # rows of query tile 1 need key tile 1: their epilogue never ran
    assert torch.isnan(o[0, 128:].float()).all()
    assert pkg.attn_device_status() == pkg.ATTN_OK
    o, _ = pkg.attn_fwd(q, k, v, **args)
    assert pkg.attn_device_status() == pkg.ATTN_OK
    if not fp8:
        assert np.abs(o.float().cpu().numpy() - ref).max() <= 1e-2


def test_selftest_rejects_bad_limits():
    with pytest.raises(pkg.AttnError):
        pkg.attn_selftest_wait_timeout(0)
