"""Pins of the exact-P ablation in the oracle (oracle.leanp.exact_*): the probabilities
formed with an exponential and rounded to e4m3, with the lean-P reference max and 64-key
block shifts.  Closed forms at powers of two, the e4m3 rounding bound, monotonicity, masking,
the tile driver against the C driver, and end-to-end accuracy against fp64 attention."""
import numpy as np
import pytest

import synth
from oracle import attention, e4m3, leanp, quantize


@pytest.mark.parametrize("m,kb", [(0, 0), (16, 2), (40, 5), (-24, 0), (8, 16)])
def test_powers_of_two_closed_form(m, kb):
    # a = 8: x = s + (8 (7 + kb) - m) / 8 is an integer for integer s, 2^x is exact and
    # its e4m3 code is 8 (x + 7) over the normal range x in [-6, 8]
    c = (8 * (7 + kb) - m) / 8.0
    x = np.arange(-6, 9, dtype=np.float64)
    s = (x - c).astype(np.float32)
    codes = leanp.exact_codes(s, 8.0, m, kb)
    np.testing.assert_array_equal(codes, (8 * (x + 7)).astype(np.uint8))


def test_rounding_bound_and_relation_to_lean_p():
    rng = np.random.default_rng(1)
    a = np.float32(3.7)
    m, kb = 200, 1
    s = (rng.uniform(-10, 60, 20000)).astype(np.float32)
    x = leanp.exact_arg(s, a, m, kb).astype(np.float64)
    ce = leanp.exact_codes(s, a, m, kb)
    cl = np.array([leanp.code(v, a, m, kb) for v in s[:4000]], dtype=np.uint8)
    normal = (x >= -6) & (x <= 8.7)
    ve = e4m3.e4m3_decode(ce)
    # e4m3 has 3 mantissa bits: relative rounding error at most 2^-4 in the normal range
    assert np.all(np.abs(ve[normal] / np.exp2(x[normal]) - 1) <= 2.0 ** -4 + 1e-12)
    # lean P approximates the same 2^x within the log-linear (Mitchell) bound plus half a
    # code step; the two agree to within the sum of both bounds
    nl = normal[:4000] & (cl > 0)
    vl = e4m3.e4m3_decode(cl)
    assert np.all(np.abs(np.log2(vl[nl]) - x[:4000][nl]) <= 0.0861 + 1 / 16 + 1e-9)
    assert np.all(np.abs(np.log2(vl[nl]) - np.log2(ve[:4000][nl])) <= 0.0861 + 1 / 16 + np.log2(17 / 16))
    # the exponential is the more accurate of the two on average
    err_e = np.abs(np.log2(ve[:4000][nl]) - x[:4000][nl]).mean()
    err_l = np.abs(np.log2(vl[nl]) - x[:4000][nl]).mean()
    assert err_e < err_l


def test_monotone_masked_and_underflow():
    s = np.sort(np.random.default_rng(2).uniform(-40, 40, 5000)).astype(np.float32)
    c = leanp.exact_codes(s, np.float32(2.5), 60, 3)
    assert np.all(np.diff(c.astype(int)) >= 0)
    z = leanp.exact_codes(np.array([-np.inf, -1e30, -5000.0], np.float32), np.float32(2.5), 60, 3)
    np.testing.assert_array_equal(z, [0, 0, 0])
    # saturation never yields the NaN code
    big = leanp.exact_codes(np.array([1e6], np.float32), np.float32(2.5), 0, 0)
    assert big[0] == 126


def test_row_driver_matches_c_driver_on_lean_codes():
    B, S, Hq, Hkv, D = 1, 300, 2, 1, 128
    q, k, v = synth.make_qkv(B, S, Hq, Hkv, D, D, seed=5, dist="outlier")
    (qc, dq), (kc, dk), (vc, dv) = [quantize.quantize_e4m3(t.float().numpy()) for t in (q, k, v)]
    rows = [0, 1, 127, 128, 200, 255, 256, 299]
    o_c, lse_c = leanp.attention_rows(qc, kc, vc, dq, dk, dv, rows, [0, 1])
    o_p, lse_p = leanp.attention_rows_exact(qc, kc, vc, dq, dk, dv, rows, [0, 1], lean=True)
    np.testing.assert_allclose(o_p, o_c, rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(lse_p, lse_c, rtol=0, atol=1e-11)


@pytest.mark.parametrize("dist", ["gaussian", "outlier"])
def test_exact_p_within_fp8_tolerance_of_fp64(dist):
    B, S, Hq, Hkv, D = 1, 384, 4, 2, 128
    q, k, v = synth.make_qkv(B, S, Hq, Hkv, D, D, seed=3, dist=dist)
    (qc, dq), (kc, dk), (vc, dv) = [quantize.quantize_e4m3(t.float().numpy()) for t in (q, k, v)]
    qd, kd, vd = [quantize.dequantize(c, s) for c, s in ((qc, dq), (kc, dk), (vc, dv))]
    o_ref, lse_ref = attention.causal_attention(qd, kd, vd)
    rows = np.arange(S)
    heads = list(range(Hq))
    o_ex, lse_ex = leanp.attention_rows_exact(qc, kc, vc, dq, dk, dv, rows, heads)
    ref = o_ref[0].transpose(1, 0, 2)
    rel = np.sqrt(((o_ex - ref) ** 2).sum() / (ref ** 2).sum())
    assert rel <= 3e-2
    # the normaliser is the sum of the same rounded values: lse within the e4m3 rounding
    assert np.abs(lse_ex - lse_ref[0]).max() <= np.log(17 / 16)
    np.testing.assert_allclose(o_ex[:, 0, :], vd[0, 0, [h // 2 for h in heads], :], rtol=0, atol=1e-12)
