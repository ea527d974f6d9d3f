"""ctypes front end of the plain-C lean-P emulator (oracle/leanp.c).  Test infrastructure
(see oracle/__init__.py).  The C source documents the reading of the pages it follows.
"""
import ctypes
import os
import subprocess

import numpy as np

from . import e4m3 as _e4m3

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "leanp.c")
_LIB = os.path.join(_HERE, "_leanp.so")

LOG2E = 1.4426950408889634
KMAX = 16
TILE = 128


def build(force=False):
    """Compile oracle/leanp.c into oracle/_leanp.so with gcc (no fp contraction)."""
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-shared",
           "-fPIC", _SRC, "-o", _LIB + ".tmp", "-lm"]
    subprocess.check_call(cmd)
    os.replace(_LIB + ".tmp", _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        f32, i32, u8p = ctypes.c_float, ctypes.c_int, ctypes.POINTER(ctypes.c_uint8)
        fp = ctypes.POINTER(ctypes.c_float)
        dp = ctypes.POINTER(ctypes.c_double)
        _lib.leanp_fmaf.restype = f32
        _lib.leanp_fmaf.argtypes = [f32, f32, f32]
        _lib.leanp_e4m3_decode.restype = ctypes.c_double
        _lib.leanp_e4m3_decode.argtypes = [ctypes.c_uint8]
        _lib.leanp_update_max.restype = i32
        _lib.leanp_update_max.argtypes = [f32, f32, i32, i32]
        _lib.leanp_kshift.restype = i32
        _lib.leanp_kshift.argtypes = [f32, f32, i32, i32]
        _lib.leanp_code.restype = ctypes.c_uint8
        _lib.leanp_code.argtypes = [f32, f32, i32, i32]
        _lib.leanp_encode_row_tile.restype = None
        _lib.leanp_encode_row_tile.argtypes = [fp, i32, f32, i32, i32, u8p, u8p]
        _lib.leanp_encode_row.restype = None
        _lib.leanp_encode_row.argtypes = [fp, i32, i32, f32, i32, u8p, u8p,
                                          ctypes.POINTER(ctypes.c_int)]
        _lib.leanp_attention_row.restype = None
        _lib.leanp_attention_row.argtypes = [fp, i32, i32, dp, i32, f32, i32, dp, dp]
    return _lib


def _ptr(a, ct):
    return a.ctypes.data_as(ctypes.POINTER(ct))


def slope(d_qk, descale_q, descale_k):
    """a = float32(8 log2(e) * (1/sqrt(d_qk)) * dq * dk): byte units per raw-score unit.
    The product is formed in float64, left to right in this order, and rounded once."""
    c = 8.0 * LOG2E * (1.0 / np.sqrt(np.float64(d_qk)))
    return np.float32(c * np.float64(np.float32(descale_q)) * np.float64(np.float32(descale_k)))


def fmaf(x, y, z):
    return np.float32(lib().leanp_fmaf(float(x), float(y), float(z)))


def kshift(mu_b, a, m, kmax=KMAX):
    return lib().leanp_kshift(float(mu_b), float(a), int(m), int(kmax))


def code(s, a, m, kb):
    return lib().leanp_code(float(s), float(a), int(m), int(kb))


def update_max(mu_tile, a, m_old, m_valid):
    return lib().leanp_update_max(float(mu_tile), float(a), int(m_old), int(m_valid))


def encode_row(s_row, a, tile=TILE, kmax=KMAX):
    """Replay the per-row state machine over raw float32 scores ``s_row`` (length a
    multiple of ``tile``; -inf where masked).  Returns (codes uint8 [n], kshift uint8
    [n/64], mref int32 [n/tile])."""
    s = np.ascontiguousarray(s_row, dtype=np.float32)
    n = s.shape[0]
    assert n % tile == 0 and tile % 64 == 0
    codes = np.zeros(n, dtype=np.uint8)
    ks = np.zeros(n // 64, dtype=np.uint8)
    mref = np.zeros(n // tile, dtype=np.int32)
    lib().leanp_encode_row(_ptr(s, ctypes.c_float), n // tile, tile, float(a), int(kmax),
                           _ptr(codes, ctypes.c_uint8), _ptr(ks, ctypes.c_uint8),
                           _ptr(mref, ctypes.c_int))
    return codes, ks, mref


def raw_scores(q_codes_row, k_codes):
    """Raw scores of one query row: float32(exact sum of decoded e4m3 products)."""
    qd = _e4m3.e4m3_decode(q_codes_row)
    kd = _e4m3.e4m3_decode(k_codes)
    return (kd @ qd).astype(np.float32)


def attention_rows(q_codes, k_codes, v_codes, dq, dk, dv, rows, heads, batch=0,
                   causal=True, tile=TILE, kmax=KMAX):
    """End-to-end lean-P prediction for selected rows/heads from e4m3 codes and descales.
    Layout as in oracle.attention (BSHD).  Returns (o [len(heads), len(rows), d_v],
    lse [len(heads), len(rows)])."""
    Hq = q_codes.shape[2]
    Hkv = k_codes.shape[2]
    G = Hq // Hkv
    d_qk = q_codes.shape[3]
    d_v = v_codes.shape[3]
    a = slope(d_qk, dq, dk)
    o = np.zeros((len(heads), len(rows), d_v))
    lse = np.zeros((len(heads), len(rows)))
    L = lib()
    for hi, h in enumerate(heads):
        g = h // G
        kd = _e4m3.e4m3_decode(k_codes[batch, :, g, :])
        vd = np.ascontiguousarray(_e4m3.e4m3_decode(v_codes[batch, :, g, :]) * np.float64(dv))
        for ri, i in enumerate(rows):
            n_vis = i + 1 if causal else kd.shape[0]
            qd = _e4m3.e4m3_decode(q_codes[batch, i, h, :])
            s = np.ascontiguousarray((kd[:n_vis] @ qd).astype(np.float32))
            orow = np.zeros(d_v)
            lrow = np.zeros(1)
            L.leanp_attention_row(_ptr(s, ctypes.c_float), n_vis, tile,
                                  _ptr(vd, ctypes.c_double), d_v, float(a), int(kmax),
                                  _ptr(orow, ctypes.c_double), _ptr(lrow, ctypes.c_double))
            o[hi, ri] = orow
            lse[hi, ri] = lrow[0]
    return o, lse
