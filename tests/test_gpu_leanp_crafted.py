"""Lean-P codes bit-exact on crafted inputs that drive the method's edge cases, over ten
key tiles (so the kernel's K/V rings wrap several times):
  * the reference max raised in the middle of a row on several tiles, and a tile maximum
    exactly at the headroom (code 126, no raise);
  * 64-key blocks whose maximum lies more than 16 octaves below the reference: the shift
    clamps at k_b = 16 with codes still live;
  * scores whose code lands exactly on a .5 midpoint of the integer conversion (round to
    nearest even decides).
The inputs are e4m3 codes chosen directly, with descales set so that the lean-P slope a is
exactly 1/4 code per score unit: every score (a sum of e4m3 products) and every code
position is then known exactly, and the test checks that each edge case really occurs in
the emulator's replay before comparing the kernel's codes with it.  Lean P follows
[ZYFA-mb] "Como o motor de atenção FP8 da Zyphra funciona" (multiply-add and integer
conversion, power-of-two scale per 64-key block)."""
import ctypes

import numpy as np
import pytest
import torch

import bf16_causal_prefill_attn_b200 as pkg
from oracle import e4m3, leanp

N_TILES = 10
S = 128 * N_TILES
HKV = 1

# every sum of two finite e4m3 values -> one such pair (the crafted scores are such sums)
_VALS = e4m3.e4m3_decode(np.arange(256, dtype=np.uint8))
_VALS = np.unique(_VALS[np.isfinite(_VALS)])
_PAIRS = {}
for _x in _VALS:
    for _y in _VALS:
        _PAIRS.setdefault(float(_x + _y), (float(_x), float(_y)))


def _pair(target):
    """(x, y) e4m3 values with x + y == the reachable value nearest to target."""
    if target in _PAIRS:
        return _PAIRS[target]
    keys = np.fromiter(_PAIRS.keys(), dtype=np.float64)
    return _PAIRS[float(keys[np.argmin(np.abs(keys - target))])]


def unit_slope_descale_k(d_qk):
    """An fp32 descale_k that makes the kernel's slope a = fp32(8 log2 e / sqrt(d) * 1 * dk)
    exactly 1/4 (searched over neighbouring fp32 values of the ideal quotient)."""
    c = 8.0 * leanp.LOG2E * (1.0 / np.sqrt(np.float64(d_qk)))
    dk = np.float32(0.25 / c)
    for _ in range(64):
        a = leanp.slope(d_qk, 1.0, dk)
        if a == np.float32(0.25):
            return dk
        dk = np.nextafter(dk, np.float32(np.inf) if a < 0.25 else np.float32(-np.inf))
    raise AssertionError("no fp32 descale gives a = 1/4")


def crafted_scores(rng):
    """Target scores (score units; code = 112 + 8 k - m + s / 4) of the crafted key sequence
    for the query pattern q = e_0 + e_1.  With m the reference in code units:
    tile 0 maximum 40 -> m = 10; tile 1 reaches 96 = 4 (m + 14): code 126 without a raise,
    plus .5 ties at 94 and 90; tile 2 reaches 100 -> raise to 25; tile 4 reaches 220 ->
    raise to 55; tile 5's first block lies near -480 (more than 16 octaves below m: k_b
    clamps at 16, codes ~75 stay live); tile 6's first block near -180 (k_b = 11); tile 7
    reaches 280 -> raise to 70; ties (s = 2 mod 4) throughout tiles 3, 6 and 8."""
    s = np.zeros(S)
    t = lambda i: slice(128 * i, 128 * (i + 1))
    s[t(0)] = rng.integers(-60, 40, 128)
    s[5] = 40
    s[t(1)] = rng.integers(-60, 40, 128)
    s[128 + 17], s[128 + 30], s[128 + 31] = 96, 94, 90
    s[t(2)] = rng.integers(-60, 90, 128)
    s[256 + 77] = 100
    s[t(3)] = 4 * rng.integers(-10, 25, 128) + 2
    s[t(4)] = rng.integers(-40, 200, 128)
    s[512 + 3] = 220
    s[640:704] = rng.integers(-520, -480, 64)
    s[704:768] = rng.integers(0, 200, 64)
    s[768:832] = rng.integers(-220, -180, 64)
    s[832:896] = 4 * rng.integers(0, 50, 64) + 2
    s[t(7)] = rng.integers(0, 220, 128)
    s[896 + 100] = 280
    s[t(8)] = 4 * rng.integers(25, 70, 128) + 2
    s[t(9)] = rng.integers(-100, 280, 128)
    return s


def build_inputs(d_qk, seed=0, hq=2):
    """e4m3 codes Q [1,S,hq,d], K [1,S,HKV,d], V [1,S,HKV,128] and fp32 descales.  Query row
    i of head h follows pattern (i + h) mod 4: A = e_0 + e_1 (the crafted sequence),
    B = e_0, C = -(e_0 + e_1) (the sequence reversed in order of size), D = random small
    values over every channel (generic scores)."""
    rng = np.random.default_rng(seed)
    target = crafted_scores(rng)
    k = np.zeros((1, S, HKV, d_qk))
    for j in range(S):
        k[0, j, 0, 0], k[0, j, 0, 1] = _pair(float(target[j]))
    small = _VALS[(np.abs(_VALS) <= 2.0) & (np.abs(_VALS) >= 0.25)]
    k[0, :, 0, 2:] = rng.choice(small, size=(S, d_qk - 2))
    q = np.zeros((1, S, hq, d_qk))
    for h in range(hq):
        for i in range(S):
            pat = (i + h) % 4
            if pat == 0:
                q[0, i, h, :2] = (1.0, 1.0)
            elif pat == 1:
                q[0, i, h, 0] = 1.0
            elif pat == 2:
                q[0, i, h, :2] = (-1.0, -1.0)
            else:
                q[0, i, h, :] = rng.choice(small, size=d_qk) * rng.choice([-1.0, 1.0], size=d_qk)
    v = rng.choice(np.concatenate([small, -small]), size=(1, S, HKV, 128))
    codes = [e4m3.e4m3_encode(x.astype(np.float32)) for x in (q, k, v)]
    for c, x in zip(codes, (q, k, v)):
        assert np.array_equal(e4m3.e4m3_decode(c), x)     # every value is exact in e4m3
    return codes, (np.float32(1.0), unit_slope_descale_k(d_qk), np.float32(1.0))


def exact_scores(codes):
    """fp64 scores of every (head, row, key) from the codes (exact: small dyadic sums)."""
    qd, kd = e4m3.e4m3_decode(codes[0]), e4m3.e4m3_decode(codes[1])
    return np.einsum("ihd,jd->hij", qd[0], kd[0, :, 0, :])


def replay_and_count(scores, a, tile):
    """Replay the emulator on every causal row; return the codes, shifts and counts of the
    edge cases met: rows with two or more mid-row raises, live blocks at k_b = 16, codes at
    126, and live codes formed from an exact .5 midpoint."""
    top = leanp.reading()[0]
    out_codes = np.zeros(scores.shape, dtype=np.uint8)
    out_ks = np.zeros(scores.shape[:2] + (S // 64,), dtype=np.int8)
    n = {"raises2": 0, "k16_live": 0, "code126": 0, "ties": 0}
    for h in range(scores.shape[0]):
        for i in range(S):
            nt = i // 128 + 1
            row = np.full(nt * 128, -np.inf, dtype=np.float32)
            row[: i + 1] = scores[h, i, : i + 1]
            codes, ks, mref = leanp.encode_row(row, a, tile)
            out_codes[h, i, : nt * 128] = codes
            out_ks[h, i, : nt * 2] = ks
            n["raises2"] += int(np.count_nonzero(np.diff(mref)) >= 2)
            for b in range(nt * 2):
                blk = codes[b * 64:(b + 1) * 64]
                if ks[b] == leanp.KMAX and np.isfinite(row[b * 64:(b + 1) * 64]).any() and blk.any():
                    n["k16_live"] += 1
            n["code126"] += int((codes == 126).sum())
            fin = np.isfinite(row)
            x = (np.float64(a) * row[fin].astype(np.float64)
                 + (top + 8 * ks[np.nonzero(fin)[0] // 64].astype(np.float64)
                    - mref[np.nonzero(fin)[0] // tile]))
            live = (x > 0.5) & (x < 126)
            n["ties"] += int(((x - np.floor(x)) == 0.5)[live].sum())
    return out_codes, out_ks, n


@pytest.mark.gpu
@pytest.mark.usefixtures("prefill_kernel")
@pytest.mark.parametrize("d_qk,hq", [(128, 2), (192, 2), (128, 1)])
def test_leanp_codes_bit_exact_on_crafted_edge_cases(d_qk, hq, key_tile):
    """hq = 2: two query heads share the kv head (so the head-pair work unit applies); hq = 1:
    one head (two query tiles per CTA in either setting)."""
    codes, (dq, dk, dv) = build_inputs(d_qk, seed=d_qk, hq=hq)
    a = leanp.slope(d_qk, dq, dk)
    assert a == np.float32(0.25)
    dev = [torch.from_numpy(c).cuda() for c in codes]
    ds = [torch.tensor([x], dtype=torch.float32, device="cuda") for x in (dq, dk, dv)]
    o, lse, d_s, d_c, d_k = pkg.attn_fwd_fp8_dump(*dev, *ds, causal=True)
    torch.cuda.synchronize()
    assert pkg.attn_device_status() == pkg.ATTN_OK
    d_s, d_c, d_k = d_s.cpu().numpy()[0], d_c.cpu().numpy()[0], d_k.cpu().numpy()[0]
    ref = exact_scores(codes)
    causal = np.tril(np.ones((S, S), dtype=bool))
    # the kernel's scores are the exact sums; masked entries are -inf
    assert np.array_equal(d_s[:, causal], ref[:, causal].astype(np.float32))
    for h in range(hq):
        for i in range(S):
            nt = i // 128 + 1
            assert np.isneginf(d_s[h, i, i + 1: nt * 128]).all()
    exp_codes, exp_ks, n = replay_and_count(d_s, a, key_tile)
    # every edge case the inputs were built for occurs
    assert n["raises2"] >= 100 * hq and n["k16_live"] >= 100 * hq and n["code126"] >= 50 * hq
    assert n["ties"] >= 1000, n
    for h in range(hq):
        for i in range(S):
            nt = i // 128 + 1
            assert np.array_equal(d_c[h, i, : nt * 128], exp_codes[h, i, : nt * 128]), (h, i)
            assert np.array_equal(d_k[h, i, : nt * 2].astype(np.int8), exp_ks[h, i, : nt * 2]), (h, i)
    # the output against the emulator's tile driver on the kernel's own scores
    vd = np.ascontiguousarray(e4m3.e4m3_decode(codes[2])[0, :, 0, :])
    o = o.float().cpu().numpy()[0]
    worst = 0.0
    for h in range(hq):
        for i in list(range(0, S, 41)) + [S - 1]:
            srow = np.ascontiguousarray(d_s[h, i, : i + 1])
            orow, lrow = np.zeros(128), np.zeros(1)
            leanp.lib().leanp_attention_row(
                srow.ctypes.data_as(ctypes.POINTER(ctypes.c_float)), i + 1, key_tile,
                vd.ctypes.data_as(ctypes.POINTER(ctypes.c_double)), 128, float(a), leanp.KMAX,
                orow.ctypes.data_as(ctypes.POINTER(ctypes.c_double)),
                lrow.ctypes.data_as(ctypes.POINTER(ctypes.c_double)))
            worst = max(worst, np.abs(o[i, h] - orow).max() / max(np.abs(orow).max(), 1e-6))
    assert worst <= 8e-3
