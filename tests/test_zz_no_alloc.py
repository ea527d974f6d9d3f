"""attn_quantize_e4m3_static (the quantiser for callers that cannot allocate device memory:
its scratch is a fixed array inside the library) gives the same codes and descale as
attn_quantize_e4m3 with a caller workspace, on two calls in a row.  This file is collected
last so a failure here stops a run only after every other test has run."""
import ctypes

import pytest
import torch

import bf16_causal_prefill_attn_b200 as pkg
import synth

pytestmark = pytest.mark.gpu


def _static_entry():
    L = pkg.lib()
    f = L.attn_quantize_e4m3_static
    vp = ctypes.c_void_p
    f.argtypes = [vp, vp, vp, ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int, vp]
    f.restype = ctypes.c_int
    return f


def test_static_scratch_matches_workspace_entry_two_calls_in_a_row():
    f = _static_entry()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    # the first call leaves a large amax in the shared scratch; the second, with a smaller
    # amax, is only right if the scratch is cleared at the start of the call
    cases = [((2, 384, 4, 128), True, "outlier"), ((2, 384, 4, 128), True, "gaussian"),
             ((1, 333, 3, 192), False, "outlier"), ((1, 333, 3, 192), False, "gaussian")]
    for i, (shape, rot, dist) in enumerate(cases):
        x = synth.make_tensor(shape, 40 + i, 0, dist).cuda()
        ref_codes, ref_ds = pkg.attn_quantize_e4m3(x, hadamard=rot)
        codes = torch.full(shape, 0xAB, dtype=torch.uint8, device="cuda")
        ds = torch.full((1,), -1.0, dtype=torch.float32, device="cuda")
        tokens = shape[0] * shape[1]
        st = f(ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(codes.data_ptr()),
               ctypes.c_void_p(ds.data_ptr()), tokens, shape[2], shape[3], 1 if rot else 0,
               stream)
        assert st == pkg.ATTN_OK, pkg.status_string(st)
        torch.cuda.synchronize()
        assert torch.equal(codes, ref_codes), f"call {i}: codes differ"
        assert torch.equal(ds, ref_ds), f"call {i}: descale differs"
    assert pkg.attn_device_status() == pkg.ATTN_OK


def test_static_entry_rejects_bad_arguments():
    f = _static_entry()
    vp = ctypes.c_void_p
    assert f(vp(256), vp(256), vp(256), 4, 2, 100, 0, None) == pkg.ATTN_ERR_INVALID_ARG
    assert f(vp(256), vp(256), vp(256), -1, 2, 128, 0, None) == pkg.ATTN_ERR_INVALID_ARG
    assert f(vp(256), vp(256), vp(256), 4, 2, 64, 1, None) == pkg.ATTN_ERR_UNSUPPORTED


def test_static_entry_empty_tensor_sets_descale_one_and_writes_no_codes():
    """tokens == 0: no element to quantise; descale is set to 1 on the device and the
    output buffer is left as it was."""
    f = _static_entry()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    codes = torch.full((64,), 0xAB, dtype=torch.uint8, device="cuda")
    ds = torch.full((1,), -1.0, dtype=torch.float32, device="cuda")
    x = torch.zeros((64,), dtype=torch.bfloat16, device="cuda")
    st = f(ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(codes.data_ptr()),
           ctypes.c_void_p(ds.data_ptr()), 0, 4, 128, 0, stream)
    assert st == pkg.ATTN_OK, pkg.status_string(st)
    torch.cuda.synchronize()
    assert ds.item() == 1.0
    assert bool((codes == 0xAB).all())
    assert pkg.attn_device_status() == pkg.ATTN_OK
