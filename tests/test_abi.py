"""The C-ABI library loads, exports every symbol include/attn.h declares, and rejects bad
arguments before touching the GPU (host logic only: no kernel runs here)."""
import ctypes
import os
import re

import pytest

import bf16_causal_prefill_attn_b200 as pkg
from bf16_causal_prefill_attn_b200 import build as B

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "attn.h")


@pytest.fixture(scope="module")
def L():
    B.build()
    return pkg.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*(attn_[a-z0-9_]+)\s*\(", text, flags=re.M)))


def test_exports_every_declared_symbol(L):
    names = declared_functions()
    assert "attn_fwd" in names and "attn_quantize_e4m3" in names and len(names) >= 9
    for n in names:
        assert hasattr(L, n), n


def test_version_and_status_strings(L):
    assert pkg.version() >= 1
    assert pkg.status_string(0) == "ok"
    assert "timed out" in pkg.status_string(pkg.ATTN_ERR_TIMEOUT)
    assert pkg.status_string(99) == "unknown status"


def _fwd(L, q=1, k=1, v=1, o=1, B=1, Hq=2, Hkv=1, S=128, dqk=128, dv=128, dtype=0, ds=(0, 0, 0),
         causal=1, flags=0):
    vp = ctypes.c_void_p
    p = lambda x: vp(x * 256) if x else None  # fake, aligned, never dereferenced
    return L.attn_fwd_ex(p(q), p(k), p(v), p(o), None, B, Hq, Hkv, S, dqk, dv, dtype,
                         p(ds[0]), p(ds[1]), p(ds[2]), causal, flags, None)


def test_fwd_argument_validation(L):
    assert _fwd(L, Hq=3, Hkv=2) == pkg.ATTN_ERR_INVALID_ARG
    assert _fwd(L, Hkv=0) == pkg.ATTN_ERR_INVALID_ARG
    assert _fwd(L, B=-1) == pkg.ATTN_ERR_INVALID_ARG
    assert _fwd(L, causal=2) == pkg.ATTN_ERR_INVALID_ARG
    assert _fwd(L, flags=8) == pkg.ATTN_ERR_INVALID_ARG
    assert _fwd(L, flags=pkg.ATTN_FLAG_EXACT_P) == pkg.ATTN_ERR_INVALID_ARG  # BF16 + exact P
    assert _fwd(L, dtype=7) == pkg.ATTN_ERR_INVALID_ARG
    assert _fwd(L, dqk=64) == pkg.ATTN_ERR_UNSUPPORTED
    assert _fwd(L, dv=192) == pkg.ATTN_ERR_UNSUPPORTED
    # S % 128 != 0 runs the tail-masking variant, which has no exact-P form
    assert _fwd(L, S=100, dtype=1, ds=(1, 1, 1), flags=pkg.ATTN_FLAG_EXACT_P) == pkg.ATTN_ERR_UNSUPPORTED
    assert _fwd(L, q=0) == pkg.ATTN_ERR_INVALID_ARG
    assert _fwd(L, o=0) == pkg.ATTN_ERR_INVALID_ARG
    assert _fwd(L, dtype=1) == pkg.ATTN_ERR_INVALID_ARG      # FP8 without descales
    # empty problems are no-ops that never touch the device
    assert _fwd(L, S=0, q=0, k=0, v=0, o=0) == pkg.ATTN_OK
    assert _fwd(L, B=0, q=0, k=0, v=0, o=0) == pkg.ATTN_OK
    # misaligned pointers
    vp = ctypes.c_void_p
    st = L.attn_fwd(vp(256 + 8), vp(256), vp(256), vp(256), None, 1, 1, 1, 128, 128, 128, 0,
                    None, None, None, 1, None)
    assert st == pkg.ATTN_ERR_ALIGNMENT


def test_quantize_argument_validation(L):
    vp = ctypes.c_void_p
    ws = L.attn_quantize_workspace_size(10, 2, 128)
    assert ws >= 4
    q = L.attn_quantize_e4m3
    assert q(vp(256), vp(256), vp(256), 10, 2, 100, 0, vp(256), ws, None) == pkg.ATTN_ERR_INVALID_ARG
    assert q(vp(256), vp(256), vp(256), 10, 2, 64, 1, vp(256), ws, None) == pkg.ATTN_ERR_UNSUPPORTED
    assert q(vp(256), vp(256), None, 10, 2, 128, 0, vp(256), ws, None) == pkg.ATTN_ERR_INVALID_ARG
    assert q(vp(256), vp(256), vp(256), 10, 2, 128, 0, None, ws, None) == pkg.ATTN_ERR_INVALID_ARG
    assert q(vp(256), vp(256), vp(256), 10, 2, 128, 0, vp(256), 0, None) == pkg.ATTN_ERR_INVALID_ARG
    assert q(vp(256), vp(256), vp(256), -1, 2, 128, 0, vp(256), ws, None) == pkg.ATTN_ERR_INVALID_ARG
    assert q(vp(256), vp(256), vp(256), 10, 2, 128, 3, vp(256), ws, None) == pkg.ATTN_ERR_INVALID_ARG
    assert q(vp(256), vp(256), vp(258), 10, 2, 128, 0, vp(256), ws, None) == pkg.ATTN_ERR_ALIGNMENT


def test_binding_raises_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(pkg, "_lib", None)
    monkeypatch.setattr(pkg, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="not built"):
        pkg.lib()


def _varlen(L, q=1, k=1, v=1, o=1, cu=1, B=2, max_s=100, T=150, Hq=2, Hkv=1, dtype=0,
            causal=1, flags=0, cu_off=0):
    vp = ctypes.c_void_p
    p = lambda x: vp(x * 256) if x else None  # fake, aligned, never dereferenced
    cu_p = vp(cu * 256 + cu_off) if cu else None
    return L.attn_fwd_varlen(p(q), p(k), p(v), p(o), None, cu_p, B, max_s, T, Hq, Hkv, 128, 128,
                             dtype, None, None, None, causal, flags, None)


def test_varlen_argument_validation(L):
    assert _varlen(L, B=-1) == pkg.ATTN_ERR_INVALID_ARG
    assert _varlen(L, max_s=-1) == pkg.ATTN_ERR_INVALID_ARG
    assert _varlen(L, Hq=3, Hkv=2) == pkg.ATTN_ERR_INVALID_ARG
    assert _varlen(L, cu=0) == pkg.ATTN_ERR_INVALID_ARG
    assert _varlen(L, q=0) == pkg.ATTN_ERR_INVALID_ARG
    assert _varlen(L, cu_off=2) == pkg.ATTN_ERR_ALIGNMENT
    assert _varlen(L, max_s=200, T=150) == pkg.ATTN_ERR_UNSUPPORTED   # longer than the tensor
    assert _varlen(L, T=2 ** 31) == pkg.ATTN_ERR_UNSUPPORTED
    assert _varlen(L, dtype=1, flags=pkg.ATTN_FLAG_EXACT_P) == pkg.ATTN_ERR_UNSUPPORTED
    assert _varlen(L, flags=4) == pkg.ATTN_ERR_INVALID_ARG
    # empty problems are no-ops that never touch the device
    assert _varlen(L, B=0, q=0, k=0, v=0, o=0, cu=0) == pkg.ATTN_OK
    assert _varlen(L, T=0, max_s=0, q=0, k=0, v=0, o=0, cu=0) == pkg.ATTN_OK



def _decode(L, B=2, Hq=8, Hkv=2, dqk=128, dv=128, P=4, page=16, mb=4, msl=64, dtype=0, ws=1,
            ws_bytes=None, cache_off=0, q=1, o=1, table=1, lens=1):
    vp = ctypes.c_void_p
    p = lambda x: vp(x * 256) if x else None  # fake, aligned, never dereferenced
    need = L.attn_decode_workspace_size(B, Hq, Hkv, max(msl, 1))
    return L.attn_decode_paged(p(q), vp(256 + cache_off), vp(512), p(o), None, p(table), p(lens),
                               B, Hq, Hkv, dqk, dv, P, page, mb, msl, dtype, None, None, None,
                               p(ws), need if ws_bytes is None else ws_bytes, None)


def test_decode_workspace_follows_the_split_policy(L):
    """Partials of B x Hq heads x n_splits ranges (128 floats + max and sum each); the split
    count aims at ~16 CTAs per SM of 148 over the B x Hkv pairs, each split at least two
    64-token tiles."""
    def want(B, Hq, Hkv, msl):
        tiles = -(-msl // 64)
        ns = min(-(-(16 * 148) // (B * Hkv)), max(1, tiles // 2))
        return B * Hq * max(ns, 1) * 130 * 4
    for B, Hq, Hkv, msl in [(64, 32, 8, 4096), (16, 32, 8, 32768), (1, 8, 1, 64), (1, 32, 8, 1),
                            (3, 16, 16, 3000), (256, 64, 8, 128), (1, 16, 1, 1 << 20)]:
        assert L.attn_decode_workspace_size(B, Hq, Hkv, msl) == want(B, Hq, Hkv, msl)


def test_decode_argument_validation(L):
    assert L.attn_decode_workspace_size(0, 8, 2, 64) == 0
    assert L.attn_decode_workspace_size(2, 8, 2, 64) > 0
    assert _decode(L, Hq=6, Hkv=4) == pkg.ATTN_ERR_INVALID_ARG
    assert _decode(L, B=-1) == pkg.ATTN_ERR_INVALID_ARG
    assert _decode(L, page=0) == pkg.ATTN_ERR_INVALID_ARG
    assert _decode(L, dtype=5) == pkg.ATTN_ERR_INVALID_ARG
    assert _decode(L, page=24) == pkg.ATTN_ERR_UNSUPPORTED       # not a power of two
    assert _decode(L, dqk=192) == pkg.ATTN_ERR_UNSUPPORTED
    assert _decode(L, Hq=6, Hkv=2) == pkg.ATTN_ERR_UNSUPPORTED   # 3 query heads per kv head
    assert _decode(L, msl=100, mb=4, page=16) == pkg.ATTN_ERR_INVALID_ARG  # beyond the table
    assert _decode(L, ws=0) == pkg.ATTN_ERR_INVALID_ARG
    assert _decode(L, ws_bytes=16) == pkg.ATTN_ERR_INVALID_ARG
    assert _decode(L, dtype=1) == pkg.ATTN_ERR_INVALID_ARG       # FP8 without descales
    assert _decode(L, q=0) == pkg.ATTN_ERR_INVALID_ARG
    assert _decode(L, cache_off=8) == pkg.ATTN_ERR_ALIGNMENT
    assert _decode(L, B=0, q=0, o=0, table=0, lens=0, ws=0) == pkg.ATTN_OK


def test_built_library_is_newer_than_every_source(L):
    """The build's up-to-date check covers every file under csrc/ and the header, so the
    library the tests load is never older than a source it was compiled from."""
    lib_t = os.path.getmtime(B.LIB)
    csrc = os.path.join(os.path.dirname(B.__file__), "csrc")
    files = [os.path.join(csrc, f) for f in os.listdir(csrc)] + [HEADER]
    assert set(B.sources()) >= {f for f in files if f.endswith((".cu", ".cuh", ".h"))} - {HEADER}
    for f in files:
        assert os.path.getmtime(f) <= lib_t, f


def test_prefill_kernel_selection_validated(L):
    """Units, schedules and the BF16 pipeline combine by OR; both schedule flags or both
    pipeline flags at once, or an unknown bit, are rejected (no GPU call is made)."""
    import bf16_causal_prefill_attn_b200 as pkg
    good = [pkg.ATTN_KERNEL_SINGLE, pkg.ATTN_KERNEL_HEADS,
            pkg.ATTN_KERNEL_PERSISTENT, pkg.ATTN_KERNEL_HEADS | pkg.ATTN_KERNEL_PERSISTENT,
            pkg.ATTN_KERNEL_DYNAMIC, pkg.ATTN_KERNEL_HEADS | pkg.ATTN_KERNEL_DYNAMIC,
            pkg.ATTN_KERNEL_AUTO, pkg.ATTN_KERNEL_BF16_S_AHEAD,
            pkg.ATTN_KERNEL_BF16_P_OVER_S | pkg.ATTN_KERNEL_HEADS | pkg.ATTN_KERNEL_DYNAMIC]
    try:
        for k in good:
            assert L.attn_select_prefill_kernel(k) == pkg.ATTN_OK
        for bad in (pkg.ATTN_KERNEL_PERSISTENT | pkg.ATTN_KERNEL_DYNAMIC, 1, 128, -1,
                    pkg.ATTN_KERNEL_AUTO | pkg.ATTN_KERNEL_HEADS,
                    pkg.ATTN_KERNEL_AUTO | pkg.ATTN_KERNEL_BF16_S_AHEAD,
                    pkg.ATTN_KERNEL_BF16_S_AHEAD | pkg.ATTN_KERNEL_BF16_P_OVER_S):
            assert L.attn_select_prefill_kernel(bad) == pkg.ATTN_ERR_INVALID_ARG
    finally:
        L.attn_select_prefill_kernel(pkg.ATTN_KERNEL_AUTO)
