"""Python binding of libattn_b200.so (include/attn.h): argument marshalling only.

Every step of the computation runs in the library's CUDA kernels; this module turns torch
tensors into device pointers and sizes, allocates outputs with torch when the caller
does not pass them, and raises on a non-zero status.  There is no fallback: if the
library is missing or fails to load, the calls raise.
"""
import ctypes
import os

import torch

from .build import LIB as LIB_PATH

ATTN_OK = 0
ATTN_ERR_INVALID_ARG = 1
ATTN_ERR_UNSUPPORTED = 2
ATTN_ERR_ALIGNMENT = 3
ATTN_ERR_CUDA = 4
ATTN_ERR_TIMEOUT = 5
ATTN_BF16 = 0
ATTN_FP8_E4M3 = 1
ATTN_FLAG_UNROTATE_O = 1
ATTN_FLAG_EXACT_P = 2
ATTN_KERNEL_SINGLE = 0
ATTN_KERNEL_HEADS = 2
ATTN_KERNEL_PERSISTENT = 4
ATTN_KERNEL_DYNAMIC = 8
ATTN_KERNEL_AUTO = 16
ATTN_KERNEL_BF16_S_AHEAD = 32
ATTN_KERNEL_BF16_P_OVER_S = 64

_lib = None


class AttnError(RuntimeError):
    def __init__(self, status, what):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} (status {status})")


def lib():
    """Load the shared library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"CUDA library {LIB_PATH} is not built; run "
                "`python -m bf16_causal_prefill_attn_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, u32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_uint
        fwd_args = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, vp, vp, vp, i32]
        L.attn_fwd.argtypes = fwd_args + [vp]
        L.attn_fwd.restype = i32
        L.attn_fwd_ex.argtypes = fwd_args + [u32, vp]
        L.attn_fwd_ex.restype = i32
        L.attn_fwd_varlen.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, ctypes.c_int64, i32,
                                      i32, i32, i32, i32, vp, vp, vp, i32, u32, vp]
        L.attn_fwd_varlen.restype = i32
        L.attn_decode_paged.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32,
                                        i32, i32, i32, i32, i32, vp, vp, vp, vp, ctypes.c_size_t,
                                        vp]
        L.attn_decode_paged.restype = i32
        L.attn_decode_workspace_size.argtypes = [i32, i32, i32, i32]
        L.attn_decode_workspace_size.restype = ctypes.c_size_t
        L.attn_fwd_fp8_dump.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32,
                                        vp, vp, vp, i32, u32, vp, vp, vp, vp]
        L.attn_fwd_fp8_dump.restype = i32
        L.attn_quantize_e4m3.argtypes = [vp, vp, vp, ctypes.c_int64, i32, i32, i32, vp,
                                         ctypes.c_size_t, vp]
        L.attn_quantize_e4m3.restype = i32
        L.attn_quantize_qkv_e4m3.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_int64,
                                             i32, i32, i32, i32, i32, vp, ctypes.c_size_t, vp]
        L.attn_quantize_qkv_e4m3.restype = i32
        L.attn_quantize_qkv_workspace_size.argtypes = []
        L.attn_quantize_qkv_workspace_size.restype = ctypes.c_size_t
        L.attn_quantize_workspace_size.argtypes = [ctypes.c_int64, i32, i32]
        L.attn_quantize_workspace_size.restype = ctypes.c_size_t
        L.attn_device_status.argtypes = [vp]
        L.attn_device_status.restype = i32
        L.attn_set_wait_timeout_ns.argtypes = [ctypes.c_uint64]
        L.attn_set_wait_timeout_ns.restype = None
        L.attn_select_prefill_kernel.argtypes = [i32]
        L.attn_select_prefill_kernel.restype = i32
        L.attn_selftest_stall_tile.argtypes = [i32]
        L.attn_selftest_stall_tile.restype = None
        L.attn_selftest_max_ctas.argtypes = [i32]
        L.attn_selftest_max_ctas.restype = None
        L.attn_selftest_wait_timeout.argtypes = [ctypes.c_uint64, vp]
        L.attn_selftest_wait_timeout.restype = i32
        L.attn_status_string.argtypes = [i32]
        L.attn_status_string.restype = ctypes.c_char_p
        L.attn_version.argtypes = []
        L.attn_version.restype = i32
        _lib = L
    return _lib


def status_string(status):
    return lib().attn_status_string(int(status)).decode()


def version():
    return lib().attn_version()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(status, what):
    if status != ATTN_OK:
        raise AttnError(status, what)


def _codes(t):
    """e4m3 tensors may be passed as uint8 codes or torch.float8_e4m3fn."""
    return t.view(torch.uint8) if t.dtype == torch.float8_e4m3fn else t


def attn_fwd(q, k, v, causal=True, descale_q=None, descale_k=None, descale_v=None, out=None,
             lse=None, return_lse=True, unrotate=False, exact_p=False, stream=None):
    """Causal prefill attention.  q [B,S,Hq,d_qk], k [B,S,Hkv,d_qk], v [B,S,Hkv,d_v] on the
    GPU: bf16, or e4m3 codes (uint8 / float8_e4m3fn) with fp32 descale tensors.
    exact_p (FP8): the exact-P ablation instead of lean P (ATTN_FLAG_EXACT_P).
    Returns (o bf16 [B,S,Hq,d_v], lse fp32 [B,Hq,S] or None)."""
    fp8 = q.dtype in (torch.uint8, torch.float8_e4m3fn)
    q, k, v = (_codes(x) for x in (q, k, v)) if fp8 else (q, k, v)
    for x in (q, k, v):
        if not x.is_contiguous():
            raise ValueError("q, k, v must be contiguous [B, S, H, d]")
    B, S, Hq, d_qk = q.shape
    Hkv = k.shape[2]
    d_v = v.shape[3]
    if out is None:
        out = torch.empty((B, S, Hq, d_v), dtype=torch.bfloat16, device=q.device)
    if lse is None and return_lse:
        lse = torch.empty((B, Hq, S), dtype=torch.float32, device=q.device)
    flags = (ATTN_FLAG_UNROTATE_O if unrotate else 0) | (ATTN_FLAG_EXACT_P if exact_p else 0)
    st = lib().attn_fwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, Hkv, S,
                           d_qk, d_v, ATTN_FP8_E4M3 if fp8 else ATTN_BF16, _ptr(descale_q),
                           _ptr(descale_k), _ptr(descale_v), 1 if causal else 0, flags,
                           _stream(stream))
    _check(st, "attn_fwd")
    return out, lse


def attn_fwd_varlen(q, k, v, cu_seqlens, max_seqlen, causal=True, descale_q=None,
                    descale_k=None, descale_v=None, out=None, lse=None, return_lse=True,
                    unrotate=False, stream=None):
    """Packed variable-length batch: q [T,Hq,d_qk], k/v [T,Hkv,d], cu_seqlens int32 [B+1] on
    the GPU (sequence b = tokens cu_seqlens[b] .. cu_seqlens[b+1]-1).  Returns (o bf16
    [T,Hq,d_v], lse fp32 [Hq,T] or None); tokens outside every sequence are left as
    allocated."""
    fp8 = q.dtype in (torch.uint8, torch.float8_e4m3fn)
    q, k, v = (_codes(x) for x in (q, k, v)) if fp8 else (q, k, v)
    for x in (q, k, v):
        if not x.is_contiguous():
            raise ValueError("q, k, v must be contiguous [T, H, d]")
    if cu_seqlens.dtype != torch.int32 or not cu_seqlens.is_contiguous():
        raise ValueError("cu_seqlens must be a contiguous int32 tensor")
    T, Hq, d_qk = q.shape
    Hkv = k.shape[1]
    d_v = v.shape[2]
    B = cu_seqlens.numel() - 1
    if out is None:
        out = torch.empty((T, Hq, d_v), dtype=torch.bfloat16, device=q.device)
    if lse is None and return_lse:
        lse = torch.empty((Hq, T), dtype=torch.float32, device=q.device)
    st = lib().attn_fwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(cu_seqlens),
                               B, int(max_seqlen), T, Hq, Hkv, d_qk, d_v,
                               ATTN_FP8_E4M3 if fp8 else ATTN_BF16, _ptr(descale_q),
                               _ptr(descale_k), _ptr(descale_v), 1 if causal else 0,
                               ATTN_FLAG_UNROTATE_O if unrotate else 0, _stream(stream))
    _check(st, "attn_fwd_varlen")
    return out, lse


def attn_decode_workspace_size(B, Hq, Hkv, max_seqlen):
    return lib().attn_decode_workspace_size(int(B), int(Hq), int(Hkv), int(max_seqlen))


def attn_decode_paged(q, k_cache, v_cache, block_table, seq_lens, max_seqlen, descale_q=None,
                      descale_k=None, descale_v=None, out=None, lse=None, return_lse=True,
                      workspace=None, stream=None):
    """Decode over a paged cache: q [B,Hq,128], caches [P,page,Hkv,128] (bf16, or e4m3 codes
    with fp32 descale tensors), block_table int32 [B,max_blocks], seq_lens int32 [B], all on
    the GPU.  Returns (o bf16 [B,Hq,128], lse fp32 [B,Hq] or None)."""
    fp8 = q.dtype in (torch.uint8, torch.float8_e4m3fn)
    q, k_cache, v_cache = ((_codes(x) for x in (q, k_cache, v_cache)) if fp8
                           else (q, k_cache, v_cache))
    for x in (q, k_cache, v_cache, block_table, seq_lens):
        if not x.is_contiguous():
            raise ValueError("all tensors must be contiguous")
    if block_table.dtype != torch.int32 or seq_lens.dtype != torch.int32:
        raise ValueError("block_table and seq_lens must be int32")
    B, Hq, d = q.shape
    P, page, Hkv, _ = k_cache.shape
    if out is None:
        out = torch.empty((B, Hq, v_cache.shape[3]), dtype=torch.bfloat16, device=q.device)
    if lse is None and return_lse:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    ws_bytes = attn_decode_workspace_size(B, Hq, Hkv, max(int(max_seqlen), 1))
    if workspace is None:
        workspace = torch.empty((ws_bytes + 15) // 16 * 4, dtype=torch.float32, device=q.device)
    st = lib().attn_decode_paged(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(out), _ptr(lse),
                                 _ptr(block_table), _ptr(seq_lens), B, Hq, Hkv, d,
                                 v_cache.shape[3], P, page, block_table.shape[1], int(max_seqlen),
                                 ATTN_FP8_E4M3 if fp8 else ATTN_BF16, _ptr(descale_q),
                                 _ptr(descale_k), _ptr(descale_v), _ptr(workspace),
                                 workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "attn_decode_paged")
    return out, lse


def attn_fwd_fp8_dump(q, k, v, descale_q, descale_k, descale_v, causal=True, exact_p=False,
                      stream=None):
    """Test-only FP8 forward that also returns the raw scores, P codes (lean, or exact with
    exact_p) and shifts."""
    q, k, v = (_codes(x) for x in (q, k, v))
    B, S, Hq, d_qk = q.shape
    Hkv = k.shape[2]
    d_v = v.shape[3]
    dev = q.device
    out = torch.empty((B, S, Hq, d_v), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, Hq, S), dtype=torch.float32, device=dev)
    ds = torch.full((B, Hq, S, S), float("nan"), dtype=torch.float32, device=dev)
    dc = torch.zeros((B, Hq, S, S), dtype=torch.uint8, device=dev)
    dk = torch.full((B, Hq, S, S // 64), 255, dtype=torch.uint8, device=dev)
    st = lib().attn_fwd_fp8_dump(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, Hkv,
                                 S, d_qk, d_v, _ptr(descale_q), _ptr(descale_k),
                                 _ptr(descale_v), 1 if causal else 0,
                                 ATTN_FLAG_EXACT_P if exact_p else 0, _ptr(ds), _ptr(dc),
                                 _ptr(dk), _stream(stream))
    _check(st, "attn_fwd_fp8_dump")
    return out, lse, ds, dc, dk


def attn_quantize_workspace_size(tokens, H, d):
    return lib().attn_quantize_workspace_size(tokens, H, d)


def attn_quantize_e4m3(x, hadamard=False, out=None, descale=None, workspace=None, stream=None):
    """Per-tensor e4m3 quantisation of a contiguous bf16 tensor [tokens, H, d] (or
    [B, S, H, d]).  Returns (codes uint8 with x's shape, descale fp32 [1])."""
    if x.dtype != torch.bfloat16 or not x.is_contiguous():
        raise ValueError("x must be a contiguous bf16 tensor")
    d = x.shape[-1]
    H = x.shape[-2]
    tokens = x.numel() // (H * d) if x.numel() else 0
    if out is None:
        out = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    if descale is None:
        descale = torch.empty((1,), dtype=torch.float32, device=x.device)
    ws_bytes = attn_quantize_workspace_size(tokens, H, d)
    if workspace is None:
        workspace = torch.empty((ws_bytes + 3) // 4, dtype=torch.int32, device=x.device)
    st = lib().attn_quantize_e4m3(_ptr(x), _ptr(out), _ptr(descale), tokens, H, d,
                                  1 if hadamard else 0, _ptr(workspace),
                                  workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "attn_quantize_e4m3")
    return out, descale


def attn_quantize_qkv_e4m3(q, k, v, hadamard=False, out=None, descales=None, workspace=None,
                           stream=None):
    """Per-tensor e4m3 quantisation of Q, K and V (contiguous bf16 [.., H, d]) in two
    launches.  out: optional (q8, k8, v8) uint8 tensors; descales: optional three fp32 [1]
    tensors.  Returns ((q8, dq), (k8, dk), (v8, dv))."""
    for x in (q, k, v):
        if x.dtype != torch.bfloat16 or not x.is_contiguous():
            raise ValueError("q, k, v must be contiguous bf16 tensors")
    Hq, d_qk = q.shape[-2], q.shape[-1]
    Hkv, d_v = v.shape[-2], v.shape[-1]
    tokens = q.numel() // (Hq * d_qk) if q.numel() else 0
    if k.numel() != tokens * Hkv * d_qk or v.numel() != tokens * Hkv * d_v:
        raise ValueError("q, k, v token counts differ")
    if out is None:
        out = tuple(torch.empty(x.shape, dtype=torch.uint8, device=x.device) for x in (q, k, v))
    if descales is None:
        descales = tuple(torch.empty((1,), dtype=torch.float32, device=q.device) for _ in range(3))
    ws_bytes = lib().attn_quantize_qkv_workspace_size()
    if workspace is None:
        workspace = torch.empty((ws_bytes + 3) // 4, dtype=torch.int32, device=q.device)
    st = lib().attn_quantize_qkv_e4m3(_ptr(q), _ptr(k), _ptr(v), *(_ptr(t) for t in out),
                                      *(_ptr(t) for t in descales), tokens, Hq, Hkv, d_qk, d_v,
                                      1 if hadamard else 0, _ptr(workspace),
                                      workspace.numel() * workspace.element_size(),
                                      _stream(stream))
    _check(st, "attn_quantize_qkv_e4m3")
    return tuple(zip(out, descales))


def attn_device_status(stream=None):
    """Synchronise the stream and return the device status code (ATTN_OK, ATTN_ERR_*)."""
    return lib().attn_device_status(_stream(stream))


def attn_set_wait_timeout_ns(ns):
    lib().attn_set_wait_timeout_ns(int(ns))


def attn_select_prefill_kernel(kernel):
    """Work unit and schedule of the prefill kernel for later calls: ATTN_KERNEL_SINGLE (two
    query tiles of one head per unit) or ATTN_KERNEL_HEADS (one query tile of two heads of
    one kv group), optionally OR one schedule: ATTN_KERNEL_PERSISTENT (one CTA per SM
    running a static list of units) or ATTN_KERNEL_DYNAMIC (one CTA per unit; running CTAs
    take over the units of CTAs not yet started), and for BF16 optionally OR one pipeline:
    ATTN_KERNEL_BF16_S_AHEAD or ATTN_KERNEL_BF16_P_OVER_S (without one: S-ahead when
    Hq > Hkv); or ATTN_KERNEL_AUTO (the default: dynamic, head pairs for FP8, tile pairs for
    BF16, the BF16 pipeline by Hq / Hkv)."""
    _check(lib().attn_select_prefill_kernel(int(kernel)), "attn_select_prefill_kernel")


def attn_selftest_max_ctas(n):
    """Test-only: cap the persistent grid at n CTAs (n <= 0: no cap)."""
    lib().attn_selftest_max_ctas(int(n))


def attn_selftest_stall_tile(tile):
    """Test-only: prefill calls stop loading before key tile `tile` (negative: normal)."""
    lib().attn_selftest_stall_tile(int(tile))


def attn_selftest_wait_timeout(timeout_ns, stream=None):
    """Launch the test-only kernel whose bounded wait is never satisfied."""
    _check(lib().attn_selftest_wait_timeout(int(timeout_ns), _stream(stream)),
           "attn_selftest_wait_timeout")
