"""GPU causal prefill attention against the oracle on seeded inputs: BF16 and FP8 outputs
within the stated tolerances, lean-P codes and shifts bit-exact against the emulator
replayed on the kernel's own scores, determinism."""
import numpy as np
import pytest
import torch

import bf16_causal_prefill_attn_b200 as pkg
import synth
from oracle import attention, hadamard, leanp, quantize

pytestmark = [pytest.mark.gpu, pytest.mark.usefixtures("prefill_kernel")]

BF16_MAX_ABS = 1e-2
BF16_REL_RMS = 5e-3
FP8_REL_RMS = 3e-2


def rel_rms(got, ref):
    return float(np.sqrt(((got - ref) ** 2).sum() / (ref ** 2).sum()))


def assert_bf16_close(got, ref, mag):
    """max-abs 1e-2 and rel-RMS 5e-3 against fp64.  P and O are rounded to bf16, so the
    error of o_id is up to about 2^-9 (sum_j p_ij |v_jd| + |o_id|): an absolute 1e-2 only
    holds where those magnitudes are O(1).  Elementwise the bound is therefore
    1e-2 * max(1, mag_id) with mag = attention applied to |V| (>= |o|); for unit-scale
    inputs mag <= max|v| ~ 1 and this is the plain max-abs 1e-2."""
    err = np.abs(got - ref)
    bound = BF16_MAX_ABS * np.maximum(1.0, mag)
    worst = float((err / bound).max())
    rr = rel_rms(got, ref)
    assert worst <= 1.0 and rr <= BF16_REL_RMS, (float(err.max()), worst, rr)


def quantize_dev(ts, rotate=False):
    return [pkg.attn_quantize_e4m3(t.cuda(), hadamard=rotate) for t in ts]


@pytest.mark.parametrize("B,S,Hq,Hkv,dqk,causal,dist", [
    (1, 256, 1, 1, 128, True, "gaussian"),      # the small reference case
    (2, 512, 4, 2, 128, True, "gaussian"),      # batch + grouped-query heads
    (1, 1024, 2, 1, 128, True, "outlier"),      # several tiles, outlier channels
    (1, 384, 2, 2, 192, True, "gaussian"),      # MLA shape in BF16
    (1, 256, 2, 1, 128, False, "gaussian"),     # full (non-causal) attention
    (1, 128, 3, 3, 128, True, "outlier"),       # a single tile
    (2, 384, 6, 2, 128, True, "gaussian"),      # odd group size (G = 3), odd tile count
    (1, 640, 4, 4, 192, True, "outlier"),       # MLA heads, five tiles
])
def test_bf16_matches_fp64(B, S, Hq, Hkv, dqk, causal, dist):
    q, k, v = synth.make_qkv(B, S, Hq, Hkv, dqk, 128, seed=S + Hq, dist=dist)
    o, lse = pkg.attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal)
    torch.cuda.synchronize()
    assert pkg.attn_device_status() == pkg.ATTN_OK
    ref, lref = attention.causal_attention(q.float().numpy(), k.float().numpy(),
                                           v.float().numpy(), causal=causal)
    mag, _ = attention.causal_attention(q.float().numpy(), k.float().numpy(),
                                        np.abs(v.float().numpy()), causal=causal)
    got = o.float().cpu().numpy()
    assert_bf16_close(got, ref, mag)
    if dist == "gaussian":
        assert np.abs(got - ref).max() <= BF16_MAX_ABS
    assert np.abs(lse.cpu().numpy() - lref).max() <= 2e-3
    if causal:
        # row 0 sees key 0 only: o = v0 exactly (after bf16 rounding of v0, which v already is)
        G = Hq // Hkv
        assert torch.equal(o[:, 0].cpu(), v[:, 0, [h // G for h in range(Hq)]])


def _fp8_inputs(B, S, Hq, Hkv, dqk, seed, dist, rotate=False):
    q, k, v = synth.make_qkv(B, S, Hq, Hkv, dqk, 128, seed=seed, dist=dist)
    dev = quantize_dev((q, k, v), rotate)
    host = [quantize.quantize_e4m3(t.float().numpy(), rotate=rotate) for t in (q, k, v)]
    for (c, d), (hc, hd) in zip(dev, host):
        assert np.array_equal(c.cpu().numpy(), hc) and d.item() == float(hd)
    return (q, k, v), dev, host


@pytest.mark.parametrize("B,S,Hq,Hkv,dqk,causal,dist", [
    (1, 256, 4, 2, 128, True, "gaussian"),
    (2, 512, 2, 1, 128, True, "outlier"),
    (1, 384, 2, 2, 192, True, "outlier"),       # MLA shape
    (1, 256, 2, 2, 128, False, "gaussian"),
    (1, 1024, 1, 1, 128, True, "gaussian"),
    (2, 384, 6, 2, 128, True, "outlier"),       # G = 3, odd tile count
    (1, 640, 2, 2, 192, True, "gaussian"),      # MLA shape, five tiles
])
def test_fp8_matches_fp64_on_quantised_inputs(B, S, Hq, Hkv, dqk, causal, dist, key_tile):
    _, dev, host = _fp8_inputs(B, S, Hq, Hkv, dqk, 7 + S, dist)
    (q8, dq), (k8, dk), (v8, dv) = dev
    o, lse = pkg.attn_fwd(q8, k8, v8, causal=causal, descale_q=dq, descale_k=dk, descale_v=dv)
    torch.cuda.synchronize()
    assert pkg.attn_device_status() == pkg.ATTN_OK
    deq = [quantize.dequantize(c, s) for c, s in host]
    ref, lref = attention.causal_attention(*deq, causal=causal)
    got = o.float().cpu().numpy()
    # the method itself (emulator on the oracle's scores) and the kernel against it
    emu = np.zeros_like(ref)
    for b in range(B):
        eo, _ = leanp.attention_rows(host[0][0], host[1][0], host[2][0], host[0][1], host[1][1],
                                     host[2][1], np.arange(S), list(range(Hq)), batch=b,
                                     causal=causal, tile=key_tile)
        emu[b] = eo.transpose(1, 0, 2)
    assert rel_rms(got, emu) <= 5e-3
    # the FP8 bar holds on the causal contract; full attention over short rows is the
    # most diffuse case, where lean-P's own error reaches the bar (kernel == method there)
    bar = FP8_REL_RMS if causal else rel_rms(emu, ref) + 2e-3
    assert rel_rms(got, ref) <= bar
    # the lean-P code error bounds the lse error (Mitchell bound + half a code step)
    assert np.abs(lse.cpu().numpy() - lref).max() <= np.log(2) * (0.0861 + 1 / 16) + 1e-3


@pytest.mark.parametrize("B,S,Hq,Hkv,dqk,causal,dist", [
    (1, 384, 2, 1, 128, True, "gaussian"),
    (1, 256, 2, 2, 192, True, "outlier"),
    (2, 256, 2, 1, 128, False, "outlier"),
    (1, 640, 3, 1, 128, True, "outlier"),      # G = 3 (rows mode), five tiles
])
def test_fp8_leanp_codes_bit_exact(B, S, Hq, Hkv, dqk, causal, dist, key_tile):
    _, dev, host = _fp8_inputs(B, S, Hq, Hkv, dqk, 100 + S, dist)
    (q8, dq), (k8, dk), (v8, dv) = dev
    o, lse, ds, dc, dks = pkg.attn_fwd_fp8_dump(q8, k8, v8, dq, dk, dv, causal=causal)
    torch.cuda.synchronize()
    assert pkg.attn_device_status() == pkg.ATTN_OK
    o_n, lse_n = pkg.attn_fwd(q8, k8, v8, causal=causal, descale_q=dq, descale_k=dk, descale_v=dv)
    assert torch.equal(o, o_n) and torch.equal(lse, lse_n)   # the dump changes nothing
    ds, dc, dks = ds.cpu().numpy(), dc.cpu().numpy(), dks.cpu().numpy()
    a = leanp.slope(dqk, host[0][1], host[1][1])
    qd = quantize.dequantize(host[0][0], 1.0)
    kd = quantize.dequantize(host[1][0], 1.0)
    vd = quantize.dequantize(host[2][0], host[2][1])
    G = Hq // Hkv
    o_host = o.float().cpu().numpy()
    worst = 0.0
    for b in range(B):
        for h in range(Hq):
            g = h // G
            for i in range(S):
                nt = (i // 128 + 1) if causal else S // 128
                srow = ds[b, h, i, : nt * 128]
                # the kernel's scores are the tensor-core sums of the e4m3 products
                exact = kd[b, : nt * 128, g, :] @ qd[b, i, h, :]
                if causal:
                    exact = np.where(np.arange(nt * 128) <= i, exact, -np.inf)
                fin = np.isfinite(exact)
                assert np.array_equal(np.isfinite(srow), fin)
                np.testing.assert_allclose(srow[fin], exact[fin], rtol=1e-5, atol=1e-5 * np.abs(exact[fin]).max())
                codes, ks, _ = leanp.encode_row(srow, a, key_tile)
                assert np.array_equal(dc[b, h, i, : nt * 128], codes), (b, h, i)
                assert np.array_equal(dks[b, h, i, : nt * 2], ks), (b, h, i)
            # O from the emulator driven by the kernel's own scores: equal up to fp32
            # accumulation order and the bf16 rounding of the output
            rows = list(range(0, S, 37)) + [S - 1]
            for i in rows:
                nvis = i + 1 if causal else S
                orow = np.zeros(128)
                lrow = np.zeros(1)
                import ctypes
                srow = np.ascontiguousarray(ds[b, h, i, :nvis])
                vv = np.ascontiguousarray(vd[b, :, g, :])
                leanp.lib().leanp_attention_row(
                    srow.ctypes.data_as(ctypes.POINTER(ctypes.c_float)), nvis, key_tile,
                    vv.ctypes.data_as(ctypes.POINTER(ctypes.c_double)), 128, float(a), leanp.KMAX,
                    orow.ctypes.data_as(ctypes.POINTER(ctypes.c_double)),
                    lrow.ctypes.data_as(ctypes.POINTER(ctypes.c_double)))
                err = np.abs(o_host[b, i, h] - orow).max() / max(np.abs(orow).max(), 1e-6)
                worst = max(worst, err)
    assert worst <= 8e-3


@pytest.mark.parametrize("dist", ["gaussian", "outlier"])
def test_fp8_hadamard_rotated(dist):
    B, S, Hq, Hkv = 1, 512, 4, 2
    (q, k, v), dev, host = _fp8_inputs(B, S, Hq, Hkv, 128, 33, dist, rotate=True)
    (q8, dq), (k8, dk), (v8, dv) = dev
    o, _ = pkg.attn_fwd(q8, k8, v8, descale_q=dq, descale_k=dk, descale_v=dv, unrotate=True)
    torch.cuda.synchronize()
    deq = [quantize.dequantize(c, s) for c, s in host]
    ref_rot, _ = attention.causal_attention(*deq)
    ref = hadamard.rotate_fp64(ref_rot)                      # un-rotate along d_v
    got = o.float().cpu().numpy()
    assert rel_rms(got, ref) <= FP8_REL_RMS


def test_bitwise_deterministic_1000_launches():
    B, S, Hq, Hkv = 1, 1024, 4, 2
    q, k, v = [t.cuda() for t in synth.make_qkv(B, S, Hq, Hkv, 128, 128, seed=9)]
    o0, l0 = pkg.attn_fwd(q, k, v)
    (q8, dq), (k8, dk), (v8, dv) = quantize_dev((q.cpu(), k.cpu(), v.cpu()))
    f0, fl0 = pkg.attn_fwd(q8, k8, v8, descale_q=dq, descale_k=dk, descale_v=dv)
    o, l = torch.empty_like(o0), torch.empty_like(l0)
    f, fl = torch.empty_like(f0), torch.empty_like(fl0)
    same = True
    for _ in range(1000):
        pkg.attn_fwd(q, k, v, out=o, lse=l)
        pkg.attn_fwd(q8, k8, v8, descale_q=dq, descale_k=dk, descale_v=dv, out=f, lse=fl)
        same &= bool(torch.equal(o, o0)) and bool(torch.equal(l, l0))
        same &= bool(torch.equal(f, f0)) and bool(torch.equal(fl, fl0))
    assert same
    assert pkg.attn_device_status() == pkg.ATTN_OK
