"""Pins of the e4m3 codec against torch.float8_e4m3fn (a library routine)."""
import numpy as np
import torch

from oracle import e4m3


def _torch_decode(codes):
    return torch.from_numpy(codes.astype(np.uint8)).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def _torch_encode(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_decode_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    ours = e4m3.e4m3_decode(codes)
    ref = _torch_decode(codes)
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    m = ~np.isnan(ref)
    assert np.array_equal(ours[m], ref[m])
    assert e4m3.e4m3_decode(np.array([0x7E]))[0] == 448.0
    assert e4m3.e4m3_decode(np.array([0x01]))[0] == 2.0 ** -9
    assert e4m3.e4m3_decode(np.array([0x38]))[0] == 1.0


def test_round_trip_all_finite_codes():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    vals = e4m3.e4m3_decode(codes).astype(np.float32)
    assert np.array_equal(e4m3.e4m3_encode(vals), codes)


def test_midpoints_and_neighbours():
    table = e4m3.e4m3_decode(np.arange(127, dtype=np.uint8))
    mids = ((table[:-1] + table[1:]) / 2).astype(np.float32)
    assert np.array_equal(mids.astype(np.float64), (table[:-1] + table[1:]) / 2)  # exact in fp32
    xs = np.concatenate([mids, np.nextafter(mids, np.float32(np.inf)), np.nextafter(mids, np.float32(0))])
    xs = np.concatenate([xs, -xs])
    ours = e4m3.e4m3_encode(xs)
    ref = _torch_encode(xs)
    assert np.array_equal(ours, ref)
    # ties go to the even code
    tie_codes = e4m3.e4m3_encode(mids)
    assert np.all(tie_codes % 2 == 0)


def test_dense_sweep_and_saturation():
    rng = np.random.default_rng(0)
    x = (rng.standard_normal(400000) * np.exp2(rng.uniform(-14, 9, 400000))).astype(np.float32)
    x = np.concatenate([x, rng.uniform(-463.99, 463.99, 100000).astype(np.float32)])
    inrange = np.abs(x) < 464
    assert np.array_equal(e4m3.e4m3_encode(x[inrange]), _torch_encode(x[inrange]))
    big = np.array([464.0, 465.0, 1e9, -480.0, -1e30, np.inf, -np.inf], dtype=np.float32)
    assert list(e4m3.e4m3_encode(big)) == [126, 126, 126, 254, 254, 126, 254]
    assert e4m3.e4m3_encode(np.array([np.nan], dtype=np.float32))[0] == 0x7F
    assert e4m3.e4m3_encode(np.array([-0.0], dtype=np.float32))[0] == 0x80
    # underflow: below half the smallest subnormal rounds to zero, at it ties to even (0)
    assert list(e4m3.e4m3_encode(np.array([2.0 ** -11, 2.0 ** -10, 2.0 ** -10 * 1.0001], dtype=np.float32))) == [0, 0, 1]
