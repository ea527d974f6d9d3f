"""fp64 causal (prefill) attention, the plain definition.  Test infrastructure
(see oracle/__init__.py).

What is computed ([ZYFA-fr] "Ce que couvrent les noyaux": forward causal attention, the
prefill phase; [ZYFA-pt] TL;DR: head dim 128 and the MLA shape 192/128):

    s_ij  = scale * <q_i, k_j>            for key j visible from query i (j <= i if causal)
    p_ij  = exp(s_ij - max_j s_ij) / sum_j exp(s_ij - max_j s_ij)
    o_i   = sum_j p_ij v_j
    lse_i = max_j s_ij + ln sum_j exp(s_ij - max_j s_ij)

Readings where the pages are silent: scale = 1/sqrt(d_qk); Sq = Sk with key j visible
iff j <= i (diagonal included); grouped-query heads map query head h to key/value head
h // (Hq / Hkv); lse in natural-log units.  Layout: q [B, S, Hq, d_qk],
k [B, S, Hkv, d_qk], v [B, S, Hkv, d_v] (token-major, head dim innermost); outputs
o [B, S, Hq, d_v] and lse [B, Hq, S].

A library matrix product serves as the dot-product step; nothing is blocked, fused or
reordered beyond the definition.
"""
import numpy as np


def _scale(d_qk, scale):
    return 1.0 / np.sqrt(np.float64(d_qk)) if scale is None else np.float64(scale)


def causal_attention(q, k, v, scale=None, causal=True):
    """Full fp64 attention.  Returns (o fp64 [B,S,Hq,dv], lse fp64 [B,Hq,S])."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, S, Hq, dqk = q.shape
    Hkv = k.shape[2]
    dv = v.shape[3]
    assert Hq % Hkv == 0
    G = Hq // Hkv
    sc = _scale(dqk, scale)
    o = np.zeros((B, S, Hq, dv))
    lse = np.zeros((B, Hq, S))
    visible = np.tril(np.ones((S, S), dtype=bool)) if causal else np.ones((S, S), dtype=bool)
    for b in range(B):
        for h in range(Hq):
            g = h // G
            s = (q[b, :, h, :] @ k[b, :, g, :].T) * sc
            s = np.where(visible, s, -np.inf)
            m = s.max(axis=1, keepdims=True)
            p = np.exp(s - m)
            l = p.sum(axis=1, keepdims=True)
            o[b, :, h, :] = (p @ v[b, :, g, :]) / l
            lse[b, h, :] = (m + np.log(l))[:, 0]
    return o, lse


def causal_attention_rows(q, k, v, rows, heads, batch=0, scale=None, causal=True):
    """The same definition restricted to query rows ``rows`` of heads ``heads`` of one batch
    entry (for sizes where the full problem is too large for the CPU).  Returns
    (o fp64 [len(heads), len(rows), dv], lse fp64 [len(heads), len(rows)])."""
    rows = np.asarray(rows, dtype=np.int64)
    Hq = q.shape[2]
    Hkv = k.shape[2]
    G = Hq // Hkv
    dqk = q.shape[3]
    dv = v.shape[3]
    sc = _scale(dqk, scale)
    S = k.shape[1]
    o = np.zeros((len(heads), len(rows), dv))
    lse = np.zeros((len(heads), len(rows)))
    for hi, h in enumerate(heads):
        g = h // G
        kk = np.asarray(k[batch, :, g, :], dtype=np.float64)
        vv = np.asarray(v[batch, :, g, :], dtype=np.float64)
        qq = np.asarray(q[batch, rows, h, :], dtype=np.float64)
        s = (qq @ kk.T) * sc                                   # [R, S]
        if causal:
            s = np.where(np.arange(S)[None, :] <= rows[:, None], s, -np.inf)
        m = s.max(axis=1, keepdims=True)
        p = np.exp(s - m)
        l = p.sum(axis=1, keepdims=True)
        o[hi] = (p @ vv) / l
        lse[hi] = (m + np.log(l))[:, 0]
    return o, lse


def causal_flops(B, Hq, S, d_qk, d_v):
    """Causal FLOP count used for throughput: 2 * B * Hq * S^2 / 2 * (d_qk + d_v)."""
    return 2.0 * B * Hq * S * S / 2.0 * (d_qk + d_v)
