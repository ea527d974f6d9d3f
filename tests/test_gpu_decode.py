"""GPU decode attention over a paged KV cache against the fp64 oracle: BF16 and FP8 caches,
grouped-query ratios 1 to 16, page sizes, lengths from 0 to several splits, shuffled pages;
bad page ids reported by the device status without a fault."""
import numpy as np
import pytest
import torch

import bf16_causal_prefill_attn_b200 as pkg
import synth
from oracle import decode, quantize

pytestmark = pytest.mark.gpu


def rel_rms(got, ref):
    return float(np.sqrt(((got - ref) ** 2).sum() / (ref ** 2).sum()))


def _cache(B, Hq, Hkv, lengths, page, seed, dist="gaussian", spare_pages=3):
    """Paged K/V caches (bf16) holding every sequence on randomly placed pages."""
    blocks = [(n + page - 1) // page for n in lengths]
    P = sum(blocks) + spare_pages
    rng = np.random.default_rng(seed)
    perm = rng.permutation(P)
    mb = max(max(blocks), 1)
    table = np.zeros((B, mb), dtype=np.int32)
    used = 0
    for b, nb in enumerate(blocks):
        table[b, :nb] = perm[used:used + nb]
        used += nb
    # synthetic K/V of the cache shape and a query per sequence, from the seeded generator
    q, k, v = synth.make_qkv(1, P * page, Hq, Hkv, 128, 128, seed=seed, dist=dist)
    kc = k[0].reshape(P, page, Hkv, 128).contiguous()
    vc = v[0].reshape(P, page, Hkv, 128).contiguous()
    qd = q[0, :B].contiguous()                         # [B, Hq, 128]
    return qd, kc, vc, table, np.array(lengths, dtype=np.int32), mb


CASES = [
    (4, 32, 8, [1, 63, 64, 65], 16),
    (3, 16, 16, [3000, 0, 129], 64),     # G = 1, several splits, an empty sequence
    (2, 16, 2, [2048, 700], 128),        # G = 8
    (2, 16, 1, [513, 1], 16),            # G = 16
    (2, 32, 8, [777, 1500], 256),        # G = 4, tiles inside large pages, ragged tails
    (3, 16, 8, [64, 200, 1], 64),        # G = 2, pages of exactly one tile
]


@pytest.mark.parametrize("B,Hq,Hkv,lengths,page", CASES)
def test_decode_bf16(B, Hq, Hkv, lengths, page):
    qd, kc, vc, table, lens, mb = _cache(B, Hq, Hkv, lengths, page, seed=B + page)
    o, lse = pkg.attn_decode_paged(qd.cuda(), kc.cuda(), vc.cuda(), torch.from_numpy(table).cuda(),
                                   torch.from_numpy(lens).cuda(), max(lengths))
    torch.cuda.synchronize()
    assert pkg.attn_device_status() == pkg.ATTN_OK
    f64 = lambda t: t.float().numpy().astype(np.float64)
    ref, lref = decode.decode_attention(f64(qd), f64(kc), f64(vc), table, lens, page)
    got = o.float().cpu().numpy()
    ok = lens > 0
    assert np.abs(got[ok] - ref[ok]).max() <= 1e-2
    assert rel_rms(got[ok], ref[ok]) <= 5e-3
    np.testing.assert_allclose(lse.cpu().numpy()[ok], lref[ok], rtol=0, atol=1e-3)
    assert np.all(got[~ok] == 0) and np.all(np.isneginf(lse.cpu().numpy()[~ok]))
    # one cached token: o is that token's value row exactly (after bf16 rounding)
    G = Hq // Hkv
    for b in np.nonzero(lens == 1)[0]:
        v0 = vc[table[b, 0], 0, [h // G for h in range(Hq)]]
        assert torch.equal(o[b].cpu(), v0)


@pytest.mark.parametrize("B,Hq,Hkv,lengths,page", CASES)
def test_decode_fp8(B, Hq, Hkv, lengths, page):
    qd, kc, vc, table, lens, mb = _cache(B, Hq, Hkv, lengths, page, seed=7 + B + page, dist="outlier")
    dev = [pkg.attn_quantize_e4m3(t.cuda()) for t in (qd, kc.reshape(-1, Hkv, 128),
                                                       vc.reshape(-1, Hkv, 128))]
    (q8, dq), (k8, dk), (v8, dv) = dev
    k8 = k8.reshape(kc.shape)
    v8 = v8.reshape(vc.shape)
    o, lse = pkg.attn_decode_paged(q8, k8, v8, torch.from_numpy(table).cuda(),
                                   torch.from_numpy(lens).cuda(), max(lengths), descale_q=dq,
                                   descale_k=dk, descale_v=dv)
    torch.cuda.synchronize()
    assert pkg.attn_device_status() == pkg.ATTN_OK
    deq = lambda c, d: quantize.dequantize(c.cpu().numpy(), np.float32(d.item()))
    ref, lref = decode.decode_attention(deq(q8, dq), deq(k8, dk), deq(v8, dv), table, lens, page)
    got = o.float().cpu().numpy()
    ok = lens > 0
    # fp32 arithmetic on exactly dequantised inputs: only the 16-bit rounding of p and the
    # bf16 output rounding remain
    assert rel_rms(got[ok], ref[ok]) <= 5e-3
    np.testing.assert_allclose(lse.cpu().numpy()[ok], lref[ok], rtol=0, atol=1e-3)
    # elementwise: the rounding errors scale with sum_j p_j |v_j| (>= |o|), the attention of
    # |V| -- 1e-2 of it, or 1e-2 absolute where that is below one (as for BF16 prefill)
    mag, _ = decode.decode_attention(deq(q8, dq), deq(k8, dk), np.abs(deq(v8, dv)), table, lens,
                                     page)
    assert (np.abs(got[ok] - ref[ok]) / (1e-2 * np.maximum(1.0, mag[ok]))).max() <= 1.0
    # one cached token: o is that token's dequantised value row, fp32(code * descale_v)
    # rounded to bf16, exactly
    G = Hq // Hkv
    v8h = v8.cpu().numpy()
    for b in np.nonzero(lens == 1)[0]:
        codes = v8h[table[b, 0], 0, [h // G for h in range(Hq)]]
        want = (quantize.dequantize(codes, 1.0).astype(np.float32) * np.float32(dv.item()))
        want = torch.from_numpy(want.astype(np.float32)).to(torch.bfloat16)
        assert torch.equal(o[b].cpu(), want)


def test_bad_page_id_reported_not_faulted():
    qd, kc, vc, table, lens, mb = _cache(2, 8, 2, [100, 40], 16, seed=3)
    bad = table.copy()
    bad[0, 2] = kc.shape[0] + 5                        # outside the cache
    args = (qd.cuda(), kc.cuda(), vc.cuda())
    pkg.attn_decode_paged(*args, torch.from_numpy(bad).cuda(), torch.from_numpy(lens).cuda(), 100)
    assert pkg.attn_device_status() == pkg.ATTN_ERR_INVALID_ARG
    o, _ = pkg.attn_decode_paged(*args, torch.from_numpy(table).cuda(), torch.from_numpy(lens).cuda(), 100)
    assert pkg.attn_device_status() == pkg.ATTN_OK
    assert torch.isfinite(o.float()).all()
