"""Pins of the lean-P emulator: exact rounding, closed forms, the Mitchell bound,
monotonicity, and the end-to-end tile driver against fp64 attention."""
from fractions import Fraction

import numpy as np
import pytest

import synth
from oracle import attention, e4m3, leanp, quantize

MAGIC = 12582912.0


def _round_f32_exact(fr):
    """Nearest float32 to a rational, ties to even, by checking neighbours exactly."""
    c = np.float32(float(fr))
    cands = [c, np.nextafter(c, np.float32(np.inf)), np.nextafter(c, np.float32(-np.inf))]
    best = None
    for v in cands:
        d = abs(Fraction(float(v)) - fr)
        key = (d, int(np.float32(v).view(np.uint32)) & 1)
        if best is None or key < best[0]:
            best = (key, v)
    return np.float32(best[1])


def test_fmaf_single_rounding():
    rng = np.random.default_rng(0)
    for _ in range(3000):
        x = np.float32(rng.standard_normal() * 50)
        y = np.float32(rng.standard_normal() * 20)
        z = np.float32(MAGIC + rng.integers(-500, 500))
        exact = Fraction(float(x)) * Fraction(float(y)) + Fraction(float(z))
        assert leanp.fmaf(x, y, z) == _round_f32_exact(exact)
    # a case where two roundings differ from one: x*y just above a .5 boundary
    x = np.float32(1.0 + 2 ** -23)
    y = np.float32(0.5)
    z = np.float32(MAGIC)
    exact = Fraction(float(x)) * Fraction(float(y)) + Fraction(float(z))
    assert leanp.fmaf(x, y, z) == _round_f32_exact(exact) == np.float32(MAGIC + 1)


def test_closed_form_block_max_code():
    # with a power-of-two slope a*s is exact, so a score equal to the reference max (in
    # code units) codes to 112 = 8*(7+7), i.e. 2^7, and the scale 2^-(7+0) gives weight 1
    checked = 0
    for a in (np.float32(0.25), np.float32(2.0), leanp.slope(128, 1.0, 1.0)):
        for m in (-40, 0, 7, 333):
            s = np.float32(m / float(a))
            if float(np.float32(a * s)) != float(m) or float(a) * float(s) != m:
                continue
            kb = leanp.kshift(s, a, m)
            assert kb == 0
            c = leanp.code(s, a, m, kb)
            assert c == 112 == 8 * (7 + 7)
            assert e4m3.e4m3_decode(np.array([c]))[0] * 2.0 ** -(7 + kb) == 1.0
            # one block (8 codes) below: k = 1 keeps the code at 112 and the weight 2^-1
            s2 = np.float32((m - 8) / float(a))
            if float(a) * float(s2) == m - 8:
                assert leanp.kshift(s2, a, m) == 1
                assert leanp.code(s2, a, m, 1) == 112
            # up to the headroom above the reference: codes 113..126, never NaN (127)
            for up in range(1, 15):
                s3 = np.float32((m + up) / float(a))
                if float(a) * float(s3) == m + up:
                    assert leanp.code(s3, a, m, 0) == 112 + up
            checked += 1
    assert checked >= 8


def test_codes_follow_log_linear_rule_within_mitchell_bound():
    rng = np.random.default_rng(1)
    a = leanp.slope(128, 0.01, 0.02)
    s = (rng.standard_normal(128 * 16) * 300).astype(np.float32)
    codes, ks, mref = leanp.encode_row(s, a)
    for t in range(16):
        m = mref[t]
        for j in range(128):
            idx = t * 128 + j
            c = int(codes[idx])
            kb = int(ks[idx // 64])
            y = (float(a) * float(s[idx]) - m) / 8.0 + 7 + kb     # wanted log2 of the value
            if c >= 8:                                          # normal e4m3 codes
                got = np.log2(e4m3.e4m3_decode(np.array([c]))[0])
                assert abs(got - y) <= 0.0861 + 1.0 / 16 + 1e-6
            elif c == 0:
                assert y < 0.5 / 8 - 6 + 1e-6                   # below the smallest code
            assert c <= 126


def test_block_shift_rule_and_monotonicity():
    rng = np.random.default_rng(2)
    a = leanp.slope(128, 0.02, 0.02)
    for trial in range(50):
        s = (rng.standard_normal(128) * 200 - rng.uniform(0, 3000) * (np.arange(128) >= 64)).astype(np.float32)
        codes, ks, mref = leanp.encode_row(s, a)
        m = mref[0]
        for b in range(2):
            blk = s[b * 64:(b + 1) * 64]
            kb = int(ks[b])
            top = int(codes[b * 64 + int(np.argmax(blk))])
            if 0 < kb < leanp.KMAX:
                assert 104 <= top <= 112
            if kb == 0:
                assert top <= 126
            # monotone within a block
            order = np.argsort(blk, kind="stable")
            assert np.all(np.diff(codes[b * 64:(b + 1) * 64][order].astype(int)) >= 0)
        assert m == int(np.ceil(np.float32(a * s.max())))


def test_masked_scores_code_zero_and_full_mask_shift():
    a = leanp.slope(128, 1.0, 1.0)
    s = np.full(128, -np.inf, dtype=np.float32)
    s[:10] = np.linspace(-5, 5, 10)
    codes, ks, mref = leanp.encode_row(s, a)
    assert not codes[10:].any()
    assert ks[1] == leanp.KMAX


def test_lazy_reference_max():
    a = leanp.slope(128, 1.0, 1.0)
    ca = lambda x: int(np.ceil(np.float32(a * np.float32(x))))
    # a small rise stays within the headroom (no rescale); a large one raises m
    s = np.concatenate([np.full(128, 1.0), np.full(128, 10.0), np.full(128, 40.0),
                        np.full(128, 20.0)]).astype(np.float32)
    _, _, mref = leanp.encode_row(s, a)
    assert ca(10.0) <= ca(1.0) + 14 < ca(40.0)
    assert list(mref) == [ca(1.0), ca(1.0), ca(40.0), ca(40.0)]
    codes, _, _ = leanp.encode_row(s, a)
    assert codes.max() <= 126 and codes[128:256].min() > codes[:128].max()


@pytest.mark.parametrize("dist", ["gaussian", "outlier"])
def test_tile_driver_within_fp8_tolerance_of_fp64(dist):
    B, S, Hq, Hkv, D = 1, 384, 4, 2, 128
    q, k, v = synth.make_qkv(B, S, Hq, Hkv, D, D, seed=3, dist=dist)
    qf, kf, vf = [t.float().numpy() for t in (q, k, v)]
    (qc, dq), (kc, dk), (vc, dv) = [quantize.quantize_e4m3(t) for t in (qf, kf, vf)]
    qd, kd, vd = [quantize.dequantize(c, s) for c, s in ((qc, dq), (kc, dk), (vc, dv))]
    o_ref, lse_ref = attention.causal_attention(qd, kd, vd)
    rows = np.arange(S)
    heads = list(range(Hq))
    o_lp, lse_lp = leanp.attention_rows(qc, kc, vc, dq, dk, dv, rows, heads)
    ref = o_ref[0].transpose(1, 0, 2)
    rel = np.sqrt(((o_lp - ref) ** 2).sum() / (ref ** 2).sum())
    assert rel <= 3e-2
    # lse carries the log-linear code error: at most the Mitchell bound plus half a step
    assert np.abs(lse_lp - lse_ref[0]).max() <= np.log(2) * (0.0861 + 1 / 16)
    # row 0: a single key of weight one -> o = v0 exactly
    np.testing.assert_allclose(o_lp[:, 0, :], vd[0, 0, [h // 2 for h in heads], :], rtol=0, atol=1e-12)


def _quantised_case(S, dist, seed=11):
    q, k, v = synth.make_qkv(1, S, 4, 2, 128, 128, seed=seed, dist=dist)
    qf, kf, vf = [t.float().numpy() for t in (q, k, v)]
    (qc, dq), (kc, dk), (vc, dv) = [quantize.quantize_e4m3(t) for t in (qf, kf, vf)]
    deq = [quantize.dequantize(c, s) for c, s in ((qc, dq), (kc, dk), (vc, dv))]
    o_ref, _ = attention.causal_attention(*deq)
    return (qc, kc, vc, dq, dk, dv), o_ref[0].transpose(1, 0, 2)


def _rel(o, ref):
    return float(np.sqrt(((o - ref) ** 2).sum() / (ref ** 2).sum()))


@pytest.mark.parametrize("dist,S", [("gaussian", 512), ("gaussian", 1024), ("outlier", 512),
                                    ("outlier", 1024)])
def test_lazy_reference_against_eager_reading(dist, S):
    """The kernel raises its reference max lazily (only past a 14-code headroom, block
    maxima at code 112); the eager reading raises it on every tile with block maxima at code
    120.  Both are replayed here on the same quantised inputs against fp64 attention.
    Finding: where the error is at the 3e-2 bar (unit Gaussian rows) the lazy reading is no
    worse (within 1%); on outlier-channel rows, whose weight sits on a few keys, the eager
    reading places the running maximum just under an octave boundary, where the log-linear
    code is exact, and is about 8% more accurate -- both stay below a third of the bar."""
    (qc, kc, vc, dq, dk, dv), ref = _quantised_case(S, dist)
    rows, heads = np.arange(S), list(range(4))
    lazy, _ = leanp.attention_rows(qc, kc, vc, dq, dk, dv, rows, heads)
    eager, _ = leanp.attention_rows(qc, kc, vc, dq, dk, dv, rows, heads, rd=leanp.EAGER)
    r_lazy, r_eager = _rel(lazy, ref), _rel(eager, ref)
    if dist == "gaussian":
        assert r_lazy <= 1.01 * r_eager <= 3e-2
    else:
        assert r_lazy <= 1.12 * r_eager and r_lazy <= 1e-2
    # the two readings differ only in the codes, not in the method: same outputs within
    # the size of the code error itself
    assert _rel(lazy, eager) <= 2 * max(r_lazy, r_eager)


def test_eager_reading_closed_forms():
    """Eager reading: the reference equals ceil(a * running max) after every tile, so each
    tile's maximum codes into (119, 120] and never above 120."""
    rng = np.random.default_rng(5)
    a = leanp.slope(128, 0.02, 0.03)
    s = (rng.standard_normal(128 * 8) * 150 + np.repeat(np.arange(8) * 40.0, 128)).astype(np.float32)
    codes, ks, mref = leanp.encode_row(s, a, rd=leanp.EAGER)
    run = -np.inf
    for t in range(8):
        run = max(run, float(s[t * 128:(t + 1) * 128].max()))
        assert mref[t] == int(np.ceil(np.float32(a * np.float32(run))))
        tile_codes = codes[t * 128:(t + 1) * 128]
        assert tile_codes.max() <= 120 and ks[2 * t:2 * t + 2].min() >= 0
    # the last tile holds the row maximum: its code is 119 or 120 (within one code step)
    assert codes[7 * 128:].max() in (119, 120)
