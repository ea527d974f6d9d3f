"""Splitting one attention problem across GPUs by heads (host logic only).

The forward attention of one (batch, kv head) group is independent of every other group
(no exchange step: the softmax of a query row only involves its own head's keys), so N
GPUs can share one problem by taking disjoint ranges of kv heads, each with the query
heads that read them (query head h reads kv head h / (Hq / Hkv)).  Each GPU runs the
unchanged kernels on its slice; nothing is communicated on the data path, and the full
output is the concatenation of the slices along the head axis.
"""


def head_partition(Hq, Hkv, world, rank):
    """Kv heads [kv_lo, kv_hi) and query heads [q_lo, q_hi) of `rank` out of `world`: kv
    heads dealt in contiguous, near-equal ranges (the first Hkv % world ranks take one
    more).  A rank may get no heads when world > Hkv."""
    if Hq <= 0 or Hkv <= 0 or Hq % Hkv:
        raise ValueError("Hq must be a positive multiple of Hkv")
    if world <= 0 or not 0 <= rank < world:
        raise ValueError("rank out of range")
    G = Hq // Hkv
    base, extra = divmod(Hkv, world)
    kv_lo = rank * base + min(rank, extra)
    kv_hi = kv_lo + base + (1 if rank < extra else 0)
    return kv_lo, kv_hi, kv_lo * G, kv_hi * G


def slice_heads(q, k, v, Hq, Hkv, world, rank):
    """The slices of q [.., S, Hq, d], k and v [.., S, Hkv, d] that `rank` computes, made
    contiguous (the layout the kernels take)."""
    kv_lo, kv_hi, q_lo, q_hi = head_partition(Hq, Hkv, world, rank)
    return (q[..., q_lo:q_hi, :].contiguous(), k[..., kv_lo:kv_hi, :].contiguous(),
            v[..., kv_lo:kv_hi, :].contiguous())
