"""Pins of the paged decode oracle: the last row of the prefill oracle on the gathered
sequence, invariance under a permutation of the physical pages, and closed forms."""
import numpy as np

from oracle import attention, decode


def _paged(rng, B, Hq, Hkv, d, lengths, page, n_pages):
    k_cache = rng.standard_normal((n_pages, page, Hkv, d))
    v_cache = rng.standard_normal((n_pages, page, Hkv, d))
    perm = rng.permutation(n_pages)
    max_blocks = max((n + page - 1) // page for n in lengths)
    table = np.zeros((B, max_blocks), dtype=np.int32)
    used = 0
    for b, n in enumerate(lengths):
        nb = (n + page - 1) // page
        table[b, :nb] = perm[used:used + nb]
        used += nb
    q = rng.standard_normal((B, Hq, d))
    return q, k_cache, v_cache, table


def test_last_row_of_prefill_on_the_gathered_sequence():
    rng = np.random.default_rng(0)
    lengths = [1, 5, 16, 37]
    q, kc, vc, table = _paged(rng, 4, 4, 2, 8, lengths, 4, 20)
    o, lse = decode.decode_attention(q, kc, vc, table, lengths, 4)
    for b, n in enumerate(lengths):
        K = decode.gather_pages(kc, table[b], n, 4)
        V = decode.gather_pages(vc, table[b], n, 4)
        Q = np.zeros((1, n, 4, 8))
        Q[0, n - 1] = q[b]
        ref, lref = attention.causal_attention(Q, K[None], V[None])
        np.testing.assert_allclose(o[b], ref[0, n - 1], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(lse[b], lref[0, :, n - 1], rtol=1e-12, atol=1e-12)


def test_page_permutation_invariance_and_gather():
    rng = np.random.default_rng(1)
    lengths = [9, 30]
    q, kc, vc, table = _paged(rng, 2, 2, 1, 16, lengths, 8, 10)
    o1, l1 = decode.decode_attention(q, kc, vc, table, lengths, 8)
    perm = rng.permutation(10)            # move every physical page, fix up the table
    inv = np.argsort(perm)
    o2, l2 = decode.decode_attention(q, kc[perm], vc[perm], inv[table], lengths, 8)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)
    # gather by hand: token 12 of sequence 1 is slot 4 of its second page
    g = decode.gather_pages(kc, table[1], 30, 8)
    np.testing.assert_array_equal(g[12], kc[table[1][1], 4])


def test_closed_forms():
    rng = np.random.default_rng(2)
    lengths = [1, 7, 0]
    q, kc, vc, table = _paged(rng, 3, 4, 4, 8, lengths, 2, 8)
    o, lse = decode.decode_attention(q, kc, vc, table, lengths, 2)
    # one cached token: o = v_0, lse = its scaled score
    v0 = vc[table[0][0], 0]
    np.testing.assert_allclose(o[0], v0, rtol=0, atol=1e-15)
    np.testing.assert_allclose(lse[0], (kc[table[0][0], 0] * q[0]).sum(-1) / np.sqrt(8), rtol=1e-14)
    # q = 0: the mean of the cached values, lse = ln n
    qz = q.copy()
    qz[1] = 0
    oz, lz = decode.decode_attention(qz, kc, vc, table, lengths, 2)
    V = decode.gather_pages(vc, table[1], 7, 2)
    np.testing.assert_allclose(oz[1], V.mean(axis=0), rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(lz[1], np.log(7.0), rtol=1e-14)
    # an empty sequence
    assert np.all(o[2] == 0) and np.all(np.isneginf(lse[2]))
