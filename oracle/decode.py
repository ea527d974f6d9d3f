"""fp64 decode attention over a paged KV cache, the plain definition.  Test infrastructure
(see oracle/__init__.py).

The pages list decode and paged KV caches as work not yet supported by their kernels
([ZYFA-fr] "Ce que couvrent les noyaux").  Reading, the plainest one consistent with the
prefill definition in oracle/attention.py: one new query token per sequence attends to
every cached token of its sequence (the cache includes the token itself), i.e. the last
row of causal attention over the sequence.

    cache layout   k_cache [P, page_size, Hkv, d_qk], v_cache [P, page_size, Hkv, d_v]
    token j of sequence b lives in page block_table[b][j // page_size], slot
    j % page_size
    s_j   = scale * <q_bh, k_j>,  j < seq_lens[b],  scale = 1/sqrt(d_qk)
    o_bh  = sum_j exp(s_j - max s) v_j / sum_j exp(s_j - max s)
    lse_bh = max s + ln sum_j exp(s_j - max s)
with query head h reading key/value head h // (Hq / Hkv).  Inputs are float64 values (for
FP8 caches: decoded codes times the descale).
"""
import numpy as np


def gather_pages(cache, table_row, n_tokens, page_size):
    """Tokens 0 .. n_tokens-1 of one sequence from a paged cache: [n_tokens, H, d]."""
    out = np.zeros((n_tokens,) + cache.shape[2:], dtype=np.float64)
    for j in range(n_tokens):
        out[j] = cache[table_row[j // page_size], j % page_size]
    return out


def decode_attention(q, k_cache, v_cache, block_table, seq_lens, page_size, scale=None):
    """q [B, Hq, d_qk]; returns (o [B, Hq, d_v], lse [B, Hq]) in float64.  A sequence of
    length 0 gives o = 0 and lse = -inf."""
    q = np.asarray(q, dtype=np.float64)
    B, Hq, d_qk = q.shape
    Hkv = k_cache.shape[2]
    d_v = v_cache.shape[3]
    G = Hq // Hkv
    sc = 1.0 / np.sqrt(np.float64(d_qk)) if scale is None else np.float64(scale)
    o = np.zeros((B, Hq, d_v))
    lse = np.full((B, Hq), -np.inf)
    for b in range(B):
        n = int(seq_lens[b])
        if n == 0:
            continue
        K = gather_pages(np.asarray(k_cache, dtype=np.float64), block_table[b], n, page_size)
        V = gather_pages(np.asarray(v_cache, dtype=np.float64), block_table[b], n, page_size)
        for h in range(Hq):
            g = h // G
            s = sc * (K[:, g, :] @ q[b, h])
            m = s.max()
            w = np.exp(s - m)
            o[b, h] = w @ V[:, g, :] / w.sum()
            lse[b, h] = m + np.log(w.sum())
    return o, lse
