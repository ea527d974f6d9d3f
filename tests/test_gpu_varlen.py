"""Sequences of any length on the GPU: packed variable-length batches (attn_fwd_varlen) and
a fixed S that is not a multiple of 128 (attn_fwd), BF16 and FP8, against the oracle per
sequence; tokens outside every sequence untouched; invalid cu_seqlens reported by the
device status without a fault."""
import numpy as np
import pytest
import torch

import bf16_causal_prefill_attn_b200 as pkg
import synth
from oracle import attention, leanp, quantize

pytestmark = pytest.mark.gpu


def rel_rms(got, ref):
    return float(np.sqrt(((got - ref) ** 2).sum() / (ref ** 2).sum()))


def _packed(lengths, lead, tail, Hq, Hkv, dqk, seed, dist):
    """One synthetic [T, H, d] tensor per operand holding every sequence back to back."""
    T = lead + sum(lengths) + tail
    q, k, v = synth.make_qkv(1, T, Hq, Hkv, dqk, 128, seed=seed, dist=dist)
    cu = np.concatenate([[lead], lead + np.cumsum(lengths)]).astype(np.int32)
    return q[0], k[0], v[0], cu, T


CASES = [
    ([129, 1, 300, 0, 128, 64, 513, 127], 16, 40, 4, 2, 128, True, "gaussian"),
    ([200, 77, 256], 0, 0, 2, 1, 128, False, "outlier"),
    ([190, 1, 129], 8, 8, 2, 2, 192, True, "outlier"),
]


@pytest.mark.parametrize("lengths,lead,tail,Hq,Hkv,dqk,causal,dist", CASES)
def test_varlen_bf16(lengths, lead, tail, Hq, Hkv, dqk, causal, dist):
    q, k, v, cu, T = _packed(lengths, lead, tail, Hq, Hkv, dqk, 11, dist)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    cu_d = torch.from_numpy(cu).cuda()
    o = torch.full((T, Hq, 128), 7.0, dtype=torch.bfloat16, device="cuda")   # sentinel
    lse = torch.full((Hq, T), 7.0, dtype=torch.float32, device="cuda")
    pkg.attn_fwd_varlen(qd, kd, vd, cu_d, max(lengths), causal=causal, out=o, lse=lse)
    torch.cuda.synchronize()
    assert pkg.attn_device_status() == pkg.ATTN_OK
    o_h, lse_h = o.float().cpu().numpy(), lse.cpu().numpy()
    f64 = lambda t: t.float().numpy().astype(np.float64)
    G = Hq // Hkv
    for b, n in enumerate(lengths):
        t0 = int(cu[b])
        if n == 0:
            continue
        sl = slice(t0, t0 + n)
        ref, lref = attention.causal_attention(f64(q[None, sl]), f64(k[None, sl]),
                                               f64(v[None, sl]), causal=causal)
        mag, _ = attention.causal_attention(f64(q[None, sl]), f64(k[None, sl]),
                                            np.abs(f64(v[None, sl])), causal=causal)
        err = np.abs(o_h[sl] - ref[0])
        assert (err / (1e-2 * np.maximum(1.0, mag[0]))).max() <= 1.0, (b, float(err.max()))
        assert rel_rms(o_h[sl], ref[0]) <= 5e-3
        assert np.abs(lse_h[:, sl] - lref[0]).max() <= 2e-3
        if causal:
            assert torch.equal(o[t0].cpu(), v[t0, [h // G for h in range(Hq)]])
    # tokens outside every sequence keep the sentinel
    outside = np.r_[0:lead, T - tail:T]
    assert np.all(o_h[outside] == 7.0) and np.all(lse_h[:, outside] == 7.0)


@pytest.mark.parametrize("lengths,lead,tail,Hq,Hkv,dqk,causal,dist", CASES)
def test_varlen_fp8(lengths, lead, tail, Hq, Hkv, dqk, causal, dist):
    q, k, v, cu, T = _packed(lengths, lead, tail, Hq, Hkv, dqk, 12, dist)
    dev = [pkg.attn_quantize_e4m3(t.cuda()) for t in (q, k, v)]
    host = [quantize.quantize_e4m3(t.float().numpy()) for t in (q, k, v)]
    for (c, d), (hc, hd) in zip(dev, host):
        assert np.array_equal(c.cpu().numpy(), hc) and d.item() == float(hd)
    (q8, dq), (k8, dk), (v8, dv) = dev
    cu_d = torch.from_numpy(cu).cuda()
    o = torch.full((T, Hq, 128), 7.0, dtype=torch.bfloat16, device="cuda")
    pkg.attn_fwd_varlen(q8, k8, v8, cu_d, max(lengths), causal=causal, descale_q=dq,
                        descale_k=dk, descale_v=dv, out=o, return_lse=False)
    torch.cuda.synchronize()
    assert pkg.attn_device_status() == pkg.ATTN_OK
    o_h = o.float().cpu().numpy()
    got_all, emu_all, ref_all = [], [], []
    for b, n in enumerate(lengths):
        t0 = int(cu[b])
        if n == 0:
            continue
        sl = slice(t0, t0 + n)
        codes = [hc[None, sl] for hc, _ in host]
        deq = [quantize.dequantize(c, s) for c, (_, s) in zip(codes, host)]
        ref, _ = attention.causal_attention(*deq, causal=causal)
        emu, _ = leanp.attention_rows(codes[0], codes[1], codes[2], host[0][1], host[1][1],
                                      host[2][1], np.arange(n), list(range(Hq)), causal=causal)
        got_all.append(o_h[sl])
        emu_all.append(emu.transpose(1, 0, 2))
        ref_all.append(ref[0])
    got, emu, ref = (np.concatenate(x) for x in (got_all, emu_all, ref_all))
    assert rel_rms(got, emu) <= 5e-3
    assert rel_rms(got, ref) <= (3e-2 if causal else rel_rms(emu, ref) + 2e-3)
    outside = np.r_[0:lead, T - tail:T]
    assert np.all(o_h[outside] == 7.0)


@pytest.mark.parametrize("B,S,Hq,Hkv,dtype", [(2, 200, 2, 1, "bf16"), (1, 1000, 2, 2, "fp8"),
                                              (3, 77, 4, 2, "fp8")])
def test_fixed_length_not_multiple_of_128(B, S, Hq, Hkv, dtype):
    q, k, v = synth.make_qkv(B, S, Hq, Hkv, 128, 128, seed=S, dist="gaussian")
    if dtype == "bf16":
        o, lse = pkg.attn_fwd(q.cuda(), k.cuda(), v.cuda())
        ref, lref = attention.causal_attention(*(t.float().numpy().astype(np.float64) for t in (q, k, v)))
        torch.cuda.synchronize()
        assert rel_rms(o.float().cpu().numpy(), ref) <= 5e-3
        assert np.abs(lse.cpu().numpy() - lref).max() <= 2e-3
    else:
        dev = [pkg.attn_quantize_e4m3(t.cuda()) for t in (q, k, v)]
        host = [quantize.quantize_e4m3(t.float().numpy()) for t in (q, k, v)]
        (q8, dq), (k8, dk), (v8, dv) = dev
        o, lse = pkg.attn_fwd(q8, k8, v8, descale_q=dq, descale_k=dk, descale_v=dv)
        torch.cuda.synchronize()
        deq = [quantize.dequantize(c, s) for c, s in host]
        ref, _ = attention.causal_attention(*deq)
        emu = np.zeros_like(ref)
        for b in range(B):
            eo, _ = leanp.attention_rows(host[0][0], host[1][0], host[2][0], host[0][1],
                                         host[1][1], host[2][1], np.arange(S), list(range(Hq)),
                                         batch=b)
            emu[b] = eo.transpose(1, 0, 2)
        got = o.float().cpu().numpy()
        assert rel_rms(got, emu) <= 5e-3 and rel_rms(got, ref) <= 3e-2
    assert pkg.attn_device_status() == pkg.ATTN_OK


def test_invalid_seqlens_reported_not_faulted():
    q, k, v, cu, T = _packed([100, 50], 0, 0, 2, 1, 128, 3, "gaussian")
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    bad = torch.tensor([0, 120, 100], dtype=torch.int32, device="cuda")   # decreasing
    pkg.attn_fwd_varlen(qd, kd, vd, bad, 120)
    assert pkg.attn_device_status() == pkg.ATTN_ERR_INVALID_ARG
    # the context is intact: a valid call afterwards succeeds
    pkg.attn_fwd_varlen(qd, kd, vd, torch.from_numpy(cu).cuda(), 100)
    assert pkg.attn_device_status() == pkg.ATTN_OK
