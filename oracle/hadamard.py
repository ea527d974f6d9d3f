"""Hadamard rotation along the head dimension.  Test infrastructure (oracle/__init__.py).

[ZYFA-mb] "Precisão, estabilidade e efeito na prática": most of the FP8 error comes from
quantising Q, K and V, and a Hadamard rotation of those tensors halves that component.

Readings (the page gives no more):
  * the Sylvester matrix H_n, H_1 = [1], H_2n = [[H_n, H_n], [H_n, -H_n]], n = 128,
    normalised by 1/sqrt(128), applied along d of Q, K and V; no random signs;
  * since H/sqrt(n) is symmetric and orthogonal, Q'K'^T = QK^T and the output of
    attention on rotated V is O H / sqrt(n); O is recovered by applying the same rotation;
  * the rotation of quantiser inputs is computed in float32 by the recursive (butterfly)
    form of the definition, stage h = 1, 2, 4, ..., n/2, each stage mapping a pair
    (u, w) at positions (i, i+h), i & h == 0, to (u + w, u - w), then one float32 multiply
    by float32(1/sqrt(n)).  Fixing the order fixes every rounding, so the e4m3 codes of
    rotated inputs are a defined function of the bf16 inputs.
"""
import numpy as np


def sylvester(n):
    """Explicit Sylvester-Hadamard matrix, entries (-1)^popcount(i & j)."""
    i = np.arange(n)[:, None]
    j = np.arange(n)[None, :]
    bits = np.bitwise_and(i, j)
    pop = np.zeros_like(bits)
    for b in range(int(np.log2(n)) + 1):
        pop += (bits >> b) & 1
    return np.where(pop % 2 == 0, 1.0, -1.0)


def butterfly(x, dtype):
    """Unnormalised transform x -> x H_n along the last axis, by the recursive definition,
    every add/subtract rounded in ``dtype``."""
    y = np.array(x, dtype=dtype, copy=True)
    n = y.shape[-1]
    lead = y.shape[:-1]
    h = 1
    while h < n:
        v = y.reshape(lead + (n // (2 * h), 2, h))
        u = v[..., 0, :].copy()
        w = v[..., 1, :].copy()
        v[..., 0, :] = u + w
        v[..., 1, :] = u - w
        y = v.reshape(lead + (n,))
        h *= 2
    return y


def rotate_fp32(x):
    """x H_n / sqrt(n) along the last axis in float32, in the fixed order above."""
    n = x.shape[-1]
    r = np.float32(1.0 / np.sqrt(np.float64(n)))
    return (butterfly(np.asarray(x, dtype=np.float32), np.float32) * r).astype(np.float32)


def rotate_fp64(x):
    """x H_n / sqrt(n) along the last axis in float64 (used to un-rotate oracle outputs)."""
    n = x.shape[-1]
    return butterfly(np.asarray(x, dtype=np.float64), np.float64) / np.sqrt(np.float64(n))
