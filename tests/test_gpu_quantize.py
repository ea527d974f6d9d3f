"""GPU quantiser against the oracle: codes and descale bit-exact (integer/byte work)."""
import numpy as np
import pytest
import torch

import bf16_causal_prefill_attn_b200 as pkg
import synth
from oracle import quantize

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("shape,rot,dist", [
    ((1, 256, 1, 128), False, "gaussian"),
    ((2, 384, 4, 128), True, "outlier"),
    ((1, 128, 3, 192), False, "outlier"),
    ((1, 77, 5, 128), True, "gaussian"),      # ragged row count
    ((3, 1, 1, 8), False, "gaussian"),         # tiny
    ((1, 4096, 8, 128), True, "outlier"),     # several waves of blocks
])
def test_quantize_bit_exact(shape, rot, dist):
    x = synth.make_tensor(shape, 11, 0, dist)
    codes, ds = pkg.attn_quantize_e4m3(x.cuda(), hadamard=rot)
    ref_codes, ref_ds = quantize.quantize_e4m3(x.float().numpy(), rotate=rot)
    got = codes.cpu().numpy()
    assert got.shape == ref_codes.shape
    mism = np.count_nonzero(got != ref_codes)
    assert mism == 0, f"{mism} codes differ"
    assert ds.item() == float(ref_ds)


def test_quantize_zero_and_empty():
    z = torch.zeros((2, 64, 2, 128), dtype=torch.bfloat16, device="cuda")
    codes, ds = pkg.attn_quantize_e4m3(z)
    assert not codes.any() and ds.item() == 1.0
    e = torch.zeros((0, 4, 128), dtype=torch.bfloat16, device="cuda")
    codes, ds = pkg.attn_quantize_e4m3(e)
    assert codes.numel() == 0 and ds.item() == 1.0


def test_quantize_deterministic():
    x = synth.make_tensor((1, 2048, 8, 128), 5, 1, "outlier").cuda()
    c0, d0 = pkg.attn_quantize_e4m3(x, hadamard=True)
    for _ in range(20):
        c, d = pkg.attn_quantize_e4m3(x, hadamard=True)
        assert torch.equal(c, c0) and torch.equal(d, d0)


@pytest.mark.parametrize("B,S,Hq,Hkv,dqk,rot,dist", [
    (1, 1024, 8, 2, 128, False, "outlier"),
    (2, 384, 4, 4, 128, True, "gaussian"),
    (1, 257, 4, 2, 192, False, "outlier"),    # MLA shape, ragged token count
    (1, 3, 2, 1, 128, True, "outlier"),       # fewer rows than one block
])
def test_quantize_qkv_batched_bit_exact(B, S, Hq, Hkv, dqk, rot, dist):
    """The two-launch Q/K/V quantiser gives the oracle's codes and descales for each
    tensor, bit for bit."""
    q, k, v = synth.make_qkv(B, S, Hq, Hkv, dqk, 128, seed=S, dist=dist)
    res = pkg.attn_quantize_qkv_e4m3(q.cuda(), k.cuda(), v.cuda(), hadamard=rot)
    torch.cuda.synchronize()
    for (codes, ds), x in zip(res, (q, k, v)):
        ref_codes, ref_ds = quantize.quantize_e4m3(x.float().numpy(), rotate=rot)
        assert np.array_equal(codes.cpu().numpy(), ref_codes)
        assert ds.item() == float(ref_ds)
    # an empty batch sets every descale to 1
    e = [torch.zeros((0, h, d), dtype=torch.bfloat16, device="cuda")
         for h, d in ((Hq, dqk), (Hkv, dqk), (Hkv, 128))]
    for codes, ds in pkg.attn_quantize_qkv_e4m3(*e):
        assert codes.numel() == 0 and ds.item() == 1.0
