"""Pins of the Hadamard rotation and the per-tensor quantiser."""
import numpy as np
import torch

from oracle import e4m3, hadamard, quantize


def test_sylvester_orthogonal_and_recursive():
    H = hadamard.sylvester(128)
    assert np.array_equal(H @ H.T, 128 * np.eye(128))
    for n in (1, 2, 4, 8, 16, 32, 64):
        Hn = hadamard.sylvester(n)
        H2 = hadamard.sylvester(2 * n)
        assert np.array_equal(H2, np.block([[Hn, Hn], [Hn, -Hn]]))
    assert np.array_equal(H, H.T)


def test_butterfly_is_the_matrix_product():
    rng = np.random.default_rng(1)
    x = rng.integers(-1000, 1000, size=(37, 128)).astype(np.float64)
    assert np.array_equal(hadamard.butterfly(x, np.float64), x @ hadamard.sylvester(128))
    y = rng.standard_normal((20, 128))
    np.testing.assert_allclose(hadamard.rotate_fp64(y), y @ hadamard.sylvester(128) / np.sqrt(128), rtol=0, atol=1e-13)


def test_round_trip_and_fp32_accuracy():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((64, 128))
    np.testing.assert_allclose(hadamard.rotate_fp64(hadamard.rotate_fp64(x)), x, rtol=0, atol=1e-13)
    y32 = hadamard.rotate_fp32(x.astype(np.float32))
    y64 = hadamard.rotate_fp64(x.astype(np.float32).astype(np.float64))
    assert y32.dtype == np.float32
    np.testing.assert_allclose(y32, y64, rtol=0, atol=5e-6 * np.abs(y64).max())


def test_quantize_against_torch_cast():
    rng = np.random.default_rng(3)
    x = torch.from_numpy(rng.standard_normal((3, 50, 4, 128)).astype(np.float32) * 3).to(torch.bfloat16)
    xf = x.float().numpy()
    codes, ds = quantize.quantize_e4m3(xf)
    amax = np.float32(np.abs(xf).max())
    assert ds == np.float32(amax / np.float32(448.0))
    sc = np.float32(np.float32(448.0) / amax)
    ref = torch.from_numpy(xf * sc).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(codes, ref)
    # the largest magnitude maps to +-448
    i = np.unravel_index(np.argmax(np.abs(xf)), xf.shape)
    assert codes[i] & 0x7F == 0x7E
    # dequantised values are within half a step (relative 2^-4) for normal codes
    deq = quantize.dequantize(codes, ds)
    normal = (codes & 0x78) != 0
    rel = np.abs(deq - xf)[normal] / np.abs(xf)[normal]
    assert rel.max() <= 2.0 ** -4 + 1e-6


def test_quantize_rotated_and_zero():
    rng = np.random.default_rng(4)
    xf = torch.from_numpy(rng.standard_normal((2, 16, 2, 128)).astype(np.float32)).to(torch.bfloat16).float().numpy()
    codes, ds = quantize.quantize_e4m3(xf, rotate=True)
    y = hadamard.rotate_fp32(xf)
    amax = np.float32(np.abs(y).max())
    assert ds == np.float32(amax / np.float32(448.0))
    ref = e4m3.e4m3_encode(y * np.float32(np.float32(448.0) / amax))
    assert np.array_equal(codes, ref)
    z, dz = quantize.quantize_e4m3(np.zeros((4, 128), dtype=np.float32))
    assert dz == 1.0 and not z.any()
