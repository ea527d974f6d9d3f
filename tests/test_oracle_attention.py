"""Pins of the fp64 attention oracle against brute force, closed forms and invariants."""
import math
import os

import numpy as np
import pytest

from oracle import attention

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _brute(q, k, v, scale, causal=True):
    """Pure-Python loops over the definition (tiny sizes only)."""
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    dv = v.shape[3]
    G = Hq // Hkv
    o = np.zeros((B, S, Hq, dv))
    lse = np.zeros((B, Hq, S))
    for b in range(B):
        for h in range(Hq):
            g = h // G
            for i in range(S):
                keys = range(i + 1) if causal else range(S)
                s = [scale * sum(float(q[b, i, h, c]) * float(k[b, j, g, c]) for c in range(D))
                     for j in keys]
                mx = max(s)
                e = [math.exp(x - mx) for x in s]
                den = sum(e)
                for c in range(dv):
                    o[b, i, h, c] = sum(e[t] * float(v[b, j, g, c]) for t, j in enumerate(keys)) / den
                lse[b, h, i] = mx + math.log(den)
    return o, lse


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def test_golden_2x2():
    rows = np.loadtxt(os.path.join(GOLDEN, "attention_2x2.txt"))
    q = np.array([0.0, math.log(3.0)]).reshape(1, 2, 1, 1)
    k = np.array([1.0, 2.0]).reshape(1, 2, 1, 1)
    v = np.array([4.0, 8.0]).reshape(1, 2, 1, 1)
    o, lse = attention.causal_attention(q, k, v, scale=1.0)
    for r, ov, lv in rows:
        assert abs(o[0, int(r), 0, 0] - ov) < 1e-12
        assert abs(lse[0, 0, int(r)] - lv) < 1e-12


@pytest.mark.parametrize("S,Hq,Hkv,D,dv", [(1, 1, 1, 1, 1), (5, 2, 1, 3, 2), (7, 4, 2, 4, 3), (6, 3, 3, 2, 4)])
def test_brute_force(S, Hq, Hkv, D, dv):
    q = _rand((2, S, Hq, D), 1)
    k = _rand((2, S, Hkv, D), 2)
    v = _rand((2, S, Hkv, dv), 3)
    sc = 1.0 / math.sqrt(D)
    o, lse = attention.causal_attention(q, k, v)
    ob, lb = _brute(q, k, v, sc)
    np.testing.assert_allclose(o, ob, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lb, rtol=0, atol=1e-12)
    o2, l2 = attention.causal_attention(q, k, v, causal=False)
    ob2, lb2 = _brute(q, k, v, sc, causal=False)
    np.testing.assert_allclose(o2, ob2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l2, lb2, rtol=0, atol=1e-12)


def test_zero_query_gives_prefix_mean():
    S, D = 40, 8
    q = np.zeros((1, S, 2, D))
    k = _rand((1, S, 1, D), 5)
    v = _rand((1, S, 1, 3), 6)
    o, lse = attention.causal_attention(q, k, v)
    pref = np.cumsum(v[0, :, 0, :], axis=0) / np.arange(1, S + 1)[:, None]
    for h in range(2):
        np.testing.assert_allclose(o[0, :, h, :], pref, rtol=0, atol=1e-13)
        np.testing.assert_allclose(lse[0, h], np.log(np.arange(1, S + 1)), rtol=0, atol=1e-13)


def test_row0_is_v0_and_rows_sum_to_one():
    S, D = 33, 16
    q = _rand((1, S, 2, D), 7) * 3
    k = _rand((1, S, 2, D), 8) * 3
    v = _rand((1, S, 2, D), 9)
    o, _ = attention.causal_attention(q, k, v)
    assert np.array_equal(o[0, 0], v[0, 0])
    ones = np.ones((1, S, 2, 5))
    o1, _ = attention.causal_attention(q, k, ones)
    np.testing.assert_allclose(o1, 1.0, rtol=0, atol=1e-14)


def test_masked_keys_have_no_influence():
    S, D = 24, 8
    q = _rand((1, S, 1, D), 10)
    k = _rand((1, S, 1, D), 11)
    v = _rand((1, S, 1, D), 12)
    o, lse = attention.causal_attention(q, k, v)
    i = 9
    k2 = k.copy()
    v2 = v.copy()
    k2[0, i + 1:] += 100.0 * _rand(k2[0, i + 1:].shape, 13)
    v2[0, i + 1:] -= 1e6
    o2, lse2 = attention.causal_attention(q, k2, v2)
    np.testing.assert_array_equal(o2[0, : i + 1], o[0, : i + 1])
    np.testing.assert_array_equal(lse2[0, :, : i + 1], lse[0, :, : i + 1])
    assert not np.allclose(o2[0, i + 1:], o[0, i + 1:])


def test_gqa_equals_mha_with_repeated_heads():
    S, D = 20, 8
    Hq, Hkv = 6, 2
    q = _rand((2, S, Hq, D), 14)
    k = _rand((2, S, Hkv, D), 15)
    v = _rand((2, S, Hkv, D), 16)
    o, lse = attention.causal_attention(q, k, v)
    G = Hq // Hkv
    kr = np.repeat(k, G, axis=2)
    vr = np.repeat(v, G, axis=2)
    o2, lse2 = attention.causal_attention(q, kr, vr)
    np.testing.assert_allclose(o, o2, rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse, lse2, rtol=0, atol=1e-14)
    # head h reads kv head h // G (consecutive grouping), not h % Hkv
    assert not np.allclose(o[0, :, 1], attention.causal_attention(q[:, :, 1:2], k[:, :, 1:2], v[:, :, 1:2])[0][0, :, 0])


def test_shift_invariance_in_k():
    S, D = 18, 8
    q = _rand((1, S, 1, D), 17)
    k = _rand((1, S, 1, D), 18)
    v = _rand((1, S, 1, D), 19)
    o, lse = attention.causal_attention(q, k, v)
    c = _rand((D,), 20)
    o2, lse2 = attention.causal_attention(q, k + c, v)
    np.testing.assert_allclose(o2, o, rtol=0, atol=1e-12)
    shift = (q[0, :, 0, :] @ c) / math.sqrt(D)
    np.testing.assert_allclose(lse2[0, 0], lse[0, 0] + shift, rtol=0, atol=1e-12)


def test_rows_variant_matches_full():
    S, D = 50, 8
    q = _rand((2, S, 4, D), 21)
    k = _rand((2, S, 2, D), 22)
    v = _rand((2, S, 2, 6), 23)
    o, lse = attention.causal_attention(q, k, v)
    rows = [0, 1, 17, 49]
    for b in range(2):
        orow, lrow = attention.causal_attention_rows(q, k, v, rows, [0, 3], batch=b)
        for hi, h in enumerate([0, 3]):
            np.testing.assert_allclose(orow[hi], o[b, rows, h, :], rtol=0, atol=1e-13)
            np.testing.assert_allclose(lrow[hi], lse[b, h, rows], rtol=0, atol=1e-13)
