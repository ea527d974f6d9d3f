"""Per-tensor e4m3 quantisation.  Test infrastructure (see oracle/__init__.py).

[ZYFA-mb] "Precisão, estabilidade e efeito na prática": the FP8 path quantises Q, K and
V, optionally after a Hadamard rotation.  The pages give neither granularity nor rounding;
readings (one scale per tensor, float32 descale):
    y       = x                      (or rotate_fp32(x) when rotating)
    amax    = max |y|                (float32; amax == 0 -> scale = descale = 1)
    scale   = float32(448) / amax    (float32, correctly rounded)
    descale = amax / float32(448)    (float32, correctly rounded)
    code    = e4m3_encode(float32(y * scale))   (nearest, ties even, saturating)
and the dequantised value seen by attention is decode(code) * descale.
"""
import numpy as np

from . import e4m3 as _e4m3
from . import hadamard as _had


def quantize_e4m3(x, rotate=False):
    """x: float array (bf16 values widened) of shape [..., d].  Returns (codes uint8, descale
    float32 scalar)."""
    y = np.asarray(x, dtype=np.float32)
    if rotate:
        y = _had.rotate_fp32(y)
    amax = np.float32(np.max(np.abs(y))) if y.size else np.float32(0.0)
    if amax == 0.0 or not np.isfinite(amax):
        scale = np.float32(1.0)
        descale = np.float32(1.0)
    else:
        scale = np.float32(np.float32(448.0) / amax)
        descale = np.float32(amax / np.float32(448.0))
    codes = _e4m3.e4m3_encode((y * scale).astype(np.float32))
    return codes, descale


def dequantize(codes, descale):
    """float64 values decode(code) * descale."""
    return _e4m3.e4m3_decode(codes) * np.float64(descale)
