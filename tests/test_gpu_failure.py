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


def test_attention_unwinds_when_its_waits_run_out():
    (q, k, v), ref = _small_case()
    pkg.attn_set_wait_timeout_ns(1)  # every wait that is not already satisfied gives up
    try:
        pkg.attn_fwd(q, k, v)
        st = pkg.attn_device_status()
    finally:
        pkg.attn_set_wait_timeout_ns(0)
    assert st in (pkg.ATTN_ERR_TIMEOUT, pkg.ATTN_OK)
    assert pkg.attn_device_status() == pkg.ATTN_OK
    o, _ = pkg.attn_fwd(q, k, v)
    assert pkg.attn_device_status() == pkg.ATTN_OK
    assert np.abs(o.float().cpu().numpy() - ref).max() <= 1e-2


def test_selftest_rejects_bad_limits():
    with pytest.raises(pkg.AttnError):
        pkg.attn_selftest_wait_timeout(0)
