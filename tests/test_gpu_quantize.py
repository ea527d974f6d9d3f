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
