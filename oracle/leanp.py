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
        i8p = ctypes.POINTER(ctypes.c_int8)
        fp = ctypes.POINTER(ctypes.c_float)
        dp = ctypes.POINTER(ctypes.c_double)
        ip = ctypes.POINTER(ctypes.c_int)
        sigs = {
            "leanp_fmaf": (f32, [f32, f32, f32]),
            "leanp_e4m3_decode": (ctypes.c_double, [ctypes.c_uint8]),
            "leanp_reading_top": (i32, []),
            "leanp_reading_headroom": (i32, []),
            "leanp_reading_kmin": (i32, []),
            "leanp_update_max": (i32, [f32, f32, i32, i32]),
            "leanp_update_max_ex": (i32, [f32, f32, i32, i32, i32]),
            "leanp_kshift": (i32, [f32, f32, i32, i32]),
            "leanp_kshift_ex": (i32, [f32, f32, i32, i32, i32]),
            "leanp_code": (ctypes.c_uint8, [f32, f32, i32, i32]),
            "leanp_code_ex": (ctypes.c_uint8, [f32, f32, i32, i32, i32]),
            "leanp_encode_row_tile": (None, [fp, i32, f32, i32, i32, u8p, i8p]),
            "leanp_encode_row": (None, [fp, i32, i32, f32, i32, u8p, i8p, ip]),
            "leanp_encode_row_ex": (None, [fp, i32, i32, f32, i32, i32, i32, i32, u8p, i8p,
                                           ip]),
            "leanp_attention_row": (None, [fp, i32, i32, dp, i32, f32, i32, dp, dp]),
            "leanp_attention_row_ex": (None, [fp, i32, i32, dp, i32, f32, i32, i32, i32, i32,
                                              dp, dp]),
            "leanp_exact_arg": (None, [fp, i32, f32, i32, i32, fp]),
        }
        for name, (res, args) in sigs.items():
            fn = getattr(_lib, name)
            fn.restype = res
            fn.argtypes = args
    return _lib


def reading():
    """(T, H, KMIN) of the reading the kernel follows: block maxima code into (T - 8, T],
    the reference max is raised once the tile max exceeds it by more than H codes, and a
    block's shift k_b lies in [KMIN, KMAX]."""
    L = lib()
    return L.leanp_reading_top(), L.leanp_reading_headroom(), L.leanp_reading_kmin()


EAGER = (120, 0, 0)  # the eager reading: reference raised on every tile, block max at 120


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


def unit_exponent():
    """log2 of the weight of code T: weights are decode(code) 2^-(T/8 - 7 + k_b)."""
    return reading()[0] // 8 - 7


def update_max(mu_tile, a, m_old, m_valid):
    return lib().leanp_update_max(float(mu_tile), float(a), int(m_old), int(m_valid))


def encode_row(s_row, a, tile=TILE, kmax=KMAX, rd=None):
    """Replay the per-row state machine over raw float32 scores ``s_row`` (length a
    multiple of ``tile``; -inf where masked) under the reading ``rd`` = (T, H, KMIN)
    (default: the kernel's).  Returns (codes uint8 [n], kshift int8 [n/64],
    mref int32 [n/tile])."""
    s = np.ascontiguousarray(s_row, dtype=np.float32)
    n = s.shape[0]
    assert n % tile == 0 and tile % 64 == 0
    top, hr, kmin = reading() if rd is None else rd
    codes = np.zeros(n, dtype=np.uint8)
    ks = np.zeros(n // 64, dtype=np.int8)
    mref = np.zeros(n // tile, dtype=np.int32)
    lib().leanp_encode_row_ex(_ptr(s, ctypes.c_float), n // tile, tile, float(a), int(kmax),
                              int(top), int(hr), int(kmin), _ptr(codes, ctypes.c_uint8),
                              _ptr(ks, ctypes.c_int8), _ptr(mref, ctypes.c_int))
    return codes, ks, mref


def attention_rows(q_codes, k_codes, v_codes, dq, dk, dv, rows, heads, batch=0,
                   causal=True, tile=TILE, kmax=KMAX, rd=None):
    """End-to-end lean-P prediction for selected rows/heads from e4m3 codes and descales.
    Layout as in oracle.attention (BSHD).  rd = (T, H, KMIN) selects the reading (default:
    the kernel's lazy one; EAGER for the reference raised on every tile).
    Returns (o [len(heads), len(rows), d_v], lse [len(heads), len(rows)])."""
    top, hr, kmin = reading() if rd is None else rd
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
            L.leanp_attention_row_ex(_ptr(s, ctypes.c_float), n_vis, tile,
                                     _ptr(vd, ctypes.c_double), d_v, float(a), int(kmax),
                                     int(top), int(hr), int(kmin), _ptr(orow, ctypes.c_double),
                                     _ptr(lrow, ctypes.c_double))
            o[hi, ri] = orow
            lse[hi, ri] = lrow[0]
    return o, lse


# ----------------------------------------------------------------------------- exact P
# The ablation the pages contrast with lean P: the same reference max and 64-key block
# shifts, but each probability formed by an exponential and rounded to e4m3 (round to
# nearest even, saturating).  See leanp_exact_arg in leanp.c for the reading.

def exact_arg(s, a, m, kb):
    """float32 exponent x = fmaf(s, a/8, (8 (7 + kb) - m)/8) for an array of scores."""
    s = np.ascontiguousarray(s, dtype=np.float32).ravel()
    x = np.zeros_like(s)
    lib().leanp_exact_arg(_ptr(s, ctypes.c_float), s.size, float(a), int(m), int(kb),
                          _ptr(x, ctypes.c_float))
    return x


def exact_codes(s, a, m, kb):
    """e4m3 codes of float32(2^x), x = exact_arg(s, a, m, kb); -inf scores give code 0."""
    x = exact_arg(s, a, m, kb)
    with np.errstate(over="ignore"):
        v = np.exp2(x.astype(np.float64)).astype(np.float32)
    return _e4m3.e4m3_encode(v)


def encode_row_exact(s_row, a, tile=TILE, kmax=KMAX):
    """Exact-P codes of one row: the lean-P state machine (encode_row) fixes the reference
    max per tile and the shift per 64-key block; the codes are then exact_codes.
    Returns (codes uint8 [n], kshift int8 [n/64], mref int32 [n/tile])."""
    s = np.ascontiguousarray(s_row, dtype=np.float32)
    _, ks, mref = encode_row(s, a, tile, kmax)
    codes = np.zeros(s.shape[0], dtype=np.uint8)
    for b in range(s.shape[0] // 64):
        t = (b * 64) // tile
        blk = s[b * 64:(b + 1) * 64]
        if np.all(np.isneginf(blk)):
            continue
        codes[b * 64:(b + 1) * 64] = exact_codes(blk, a, mref[t], int(ks[b]))
    return codes, ks, mref


def combine_row(codes, ks, mref, n_vis, vd, tile=TILE):
    """Normalised output row and lse from the codes of one row, in float64: weight of key j
    = decode(code_j) 2^-(T/8 - 7 + k_b(j)) 2^((m_t(j) - m_final)/8), o = sum w_j v_j / sum w_j,
    lse = ln 2 (m_final/8 + log2 sum w_j) with the weights taken relative to m_final.  This
    is the tile-by-tile online combination with its rescales written out."""
    ntiles = (n_vis + tile - 1) // tile
    m_final = int(mref[ntiles - 1])  # any common reference cancels in o; lse adds it back
    j = np.arange(n_vis)
    w = (_e4m3.e4m3_decode(codes[:n_vis])
         * np.exp2(-(unit_exponent() + ks[j // 64].astype(np.float64)))
         * np.exp2((mref[j // tile].astype(np.float64) - m_final) / 8.0))
    l = w.sum()
    o = (w[:, None] * vd[:n_vis]).sum(axis=0) / l
    return o, np.log(2.0) * (m_final / 8.0 + np.log2(l))


def attention_rows_exact(q_codes, k_codes, v_codes, dq, dk, dv, rows, heads, batch=0,
                         causal=True, tile=TILE, kmax=KMAX, lean=False):
    """End-to-end exact-P prediction for selected rows/heads (layout as attention_rows).
    With lean=True the same driver combines lean-P codes instead (used to pin the driver
    against the C tile driver)."""
    Hq = q_codes.shape[2]
    Hkv = k_codes.shape[2]
    G = Hq // Hkv
    d_qk = q_codes.shape[3]
    d_v = v_codes.shape[3]
    a = slope(d_qk, dq, dk)
    o = np.zeros((len(heads), len(rows), d_v))
    lse = np.zeros((len(heads), len(rows)))
    for hi, h in enumerate(heads):
        g = h // G
        kd = _e4m3.e4m3_decode(k_codes[batch, :, g, :])
        vd = _e4m3.e4m3_decode(v_codes[batch, :, g, :]) * np.float64(dv)
        S = kd.shape[0]
        for ri, i in enumerate(rows):
            n_vis = i + 1 if causal else S
            qd = _e4m3.e4m3_decode(q_codes[batch, i, h, :])
            n_pad = (n_vis + tile - 1) // tile * tile
            s = np.full(n_pad, -np.inf, dtype=np.float32)
            s[:n_vis] = (kd[:n_vis] @ qd).astype(np.float32)
            if lean:
                codes, ks, mref = encode_row(s, a, tile, kmax)
            else:
                codes, ks, mref = encode_row_exact(s, a, tile, kmax)
            o[hi, ri], lse[hi, ri] = combine_row(codes, ks, mref, n_vis, vd, tile)
    return o, lse

