"""GPU exact-P ablation (ATTN_FLAG_EXACT_P) against the oracle: shifts bit-exact and codes
equal to the correctly rounded e4m3 of 2^x except where 2^x lies within the hardware
exponential's error of a rounding midpoint, on the kernel's own scores; outputs within
the FP8 tolerance of fp64 and close to the exact-P emulator."""
import numpy as np
import pytest
import torch

import bf16_causal_prefill_attn_b200 as pkg
import synth
from oracle import attention, e4m3, leanp, quantize

pytestmark = pytest.mark.gpu

FP8_REL_RMS = 3e-2


def rel_rms(got, ref):
    return float(np.sqrt(((got - ref) ** 2).sum() / (ref ** 2).sum()))


def _inputs(B, S, Hq, Hkv, dqk, seed, dist):
    q, k, v = synth.make_qkv(B, S, Hq, Hkv, dqk, 128, seed=seed, dist=dist)
    dev = [pkg.attn_quantize_e4m3(t.cuda()) for t in (q, k, v)]
    host = [quantize.quantize_e4m3(t.float().numpy()) for t in (q, k, v)]
    for (c, d), (hc, hd) in zip(dev, host):
        assert np.array_equal(c.cpu().numpy(), hc) and d.item() == float(hd)
    return dev, host


@pytest.mark.parametrize("B,S,Hq,Hkv,dqk,causal,dist", [
    (1, 384, 2, 1, 128, True, "gaussian"),
    (1, 256, 2, 2, 192, True, "outlier"),
    (2, 256, 2, 1, 128, False, "outlier"),
])
def test_exact_p_codes_against_oracle(B, S, Hq, Hkv, dqk, causal, dist):
    dev, host = _inputs(B, S, Hq, Hkv, dqk, 300 + S, dist)
    (q8, dq), (k8, dk), (v8, dv) = dev
    o, lse, ds, dc, dks = pkg.attn_fwd_fp8_dump(q8, k8, v8, dq, dk, dv, causal=causal, exact_p=True)
    torch.cuda.synchronize()
    assert pkg.attn_device_status() == pkg.ATTN_OK
    o_n, lse_n = pkg.attn_fwd(q8, k8, v8, causal=causal, descale_q=dq, descale_k=dk,
                              descale_v=dv, exact_p=True)
    assert torch.equal(o, o_n) and torch.equal(lse, lse_n)   # the dump changes nothing
    ds, dc, dks = ds.cpu().numpy(), dc.cpu().numpy(), dks.cpu().numpy()
    a = leanp.slope(dqk, host[0][1], host[1][1])
    n_codes = n_diff = 0
    for b in range(B):
        for h in range(Hq):
            for i in range(S):
                nt = (i // 128 + 1) if causal else S // 128
                srow = ds[b, h, i, : nt * 128]
                codes, ks, mref = leanp.encode_row_exact(srow, a)
                assert np.array_equal(dks[b, h, i, : nt * 2], ks), (b, h, i)
                got = dc[b, h, i, : nt * 128]
                diff = np.nonzero(got != codes)[0]
                n_codes += int(np.isfinite(srow).sum())
                n_diff += diff.size
                for j in diff:
                    # a different code is only allowed one step away, where 2^x lies within
                    # 2^-20 (relative) of the midpoint between the two candidates
                    assert abs(int(got[j]) - int(codes[j])) == 1, (b, h, i, j)
                    x = leanp.exact_arg(srow[j:j + 1], a, mref[j // 128], int(ks[j // 64]))[0]
                    mid = 0.5 * (e4m3.e4m3_decode(got[j]) + e4m3.e4m3_decode(codes[j]))
                    assert abs(np.exp2(np.float64(x)) / mid - 1) <= 2.0 ** -20, (b, h, i, j)
    assert n_diff <= 1e-3 * n_codes, (n_diff, n_codes)


@pytest.mark.parametrize("B,S,Hq,Hkv,dqk,causal,dist", [
    (1, 256, 4, 2, 128, True, "gaussian"),
    (2, 512, 2, 1, 128, True, "outlier"),
    (1, 384, 2, 2, 192, True, "outlier"),
])
def test_exact_p_matches_fp64(B, S, Hq, Hkv, dqk, causal, dist):
    dev, host = _inputs(B, S, Hq, Hkv, dqk, 17 + S, dist)
    (q8, dq), (k8, dk), (v8, dv) = dev
    o, lse = pkg.attn_fwd(q8, k8, v8, causal=causal, descale_q=dq, descale_k=dk, descale_v=dv,
                          exact_p=True)
    o_lean, _ = pkg.attn_fwd(q8, k8, v8, causal=causal, descale_q=dq, descale_k=dk, descale_v=dv)
    torch.cuda.synchronize()
    assert pkg.attn_device_status() == pkg.ATTN_OK
    deq = [quantize.dequantize(c, s) for c, s in host]
    ref, lref = attention.causal_attention(*deq, causal=causal)
    got = o.float().cpu().numpy()
    emu = np.zeros_like(ref)
    for b in range(B):
        eo, _ = leanp.attention_rows_exact(host[0][0], host[1][0], host[2][0], host[0][1],
                                           host[1][1], host[2][1], np.arange(S),
                                           list(range(Hq)), batch=b, causal=causal)
        emu[b] = eo.transpose(1, 0, 2)
    assert rel_rms(got, emu) <= 5e-3
    assert rel_rms(got, ref) <= FP8_REL_RMS
    # the normaliser is the sum of the same rounded values: lse within the e4m3 rounding
    assert np.abs(lse.cpu().numpy() - lref).max() <= np.log(17 / 16) + 1e-3
    # the ablation changes the probabilities, not the rest of the path
    assert not torch.equal(o, o_lean)
