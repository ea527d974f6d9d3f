"""Seeded synthetic inputs for causal prefill attention.

Shared by the tests, the smoke check and the bench: it holds none of the attention or
quantisation arithmetic, only random numbers and their shapes.  Everything is generated
on the host (numpy PCG64, one independent stream per (seed, tensor)), rounded to bf16
(round to nearest even, via torch), and then handed to both the CUDA path and the oracle.

Distributions (the pages benchmark "Gaussian" inputs and captured model activations,
[ZYFA-mb] "ZYFA acelera atenção em até 1,76x com menos erro"; captured activations need
model weights and prompts that are not available, so a synthetic outlier-channel scheme
stands in for them):
  gaussian  x ~ N(0, 1) iid.
  outlier   per tensor and head: channel scales c_d = exp(sigma * z_d), z_d ~ N(0, 1),
            sigma = 1, and 4 channels (a seeded permutation) multiplied by 20; x = z * c_d
            with z ~ N(0, 1) iid.
Layout: [B, S, H, d] (token-major, head dim innermost), contiguous.
"""
import numpy as np

STREAM_Q, STREAM_K, STREAM_V, STREAM_SCALES = 0, 1, 2, 3


def _rng(seed, stream, extra=0):
    return np.random.default_rng([int(seed), int(stream), int(extra)])


def normal_f32(shape, seed, stream):
    """iid N(0,1) float32 array from stream (seed, stream)."""
    return _rng(seed, stream).standard_normal(size=shape, dtype=np.float32)


def outlier_scales(H, d, seed, stream, sigma=1.0, n_outliers=4, factor=20.0):
    """Per-head channel scales [H, d] of the outlier scheme (float32)."""
    r = _rng(seed, STREAM_SCALES, 1 + stream)
    c = np.exp(sigma * r.standard_normal(size=(H, d))).astype(np.float32)
    for h in range(H):
        idx = r.permutation(d)[:n_outliers]
        c[h, idx] *= np.float32(factor)
    return c


def make_tensor(shape, seed, stream, dist="gaussian"):
    """float32 array of bf16-representable values, shape [B, S, H, d]."""
    import torch
    x = normal_f32(shape, seed, stream)
    if dist == "outlier":
        H, d = shape[2], shape[3]
        x *= outlier_scales(H, d, seed, stream)[None, None, :, :]
    elif dist != "gaussian":
        raise ValueError(f"unknown distribution {dist!r}")
    t = torch.from_numpy(x).to(torch.bfloat16)
    return t


def make_qkv(B, S, Hq, Hkv, d_qk, d_v, seed=0, dist="gaussian"):
    """(q, k, v) as CPU torch.bfloat16 tensors in [B, S, H, d] layout."""
    q = make_tensor((B, S, Hq, d_qk), seed, STREAM_Q, dist)
    k = make_tensor((B, S, Hkv, d_qk), seed, STREAM_K, dist)
    v = make_tensor((B, S, Hkv, d_v), seed, STREAM_V, dist)
    return q, k, v
