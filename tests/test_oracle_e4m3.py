"""Pins of the oracle's FP8 E4M3 pieces (quantised KV pages).

The pages say only that paging combines with a quantised cache
("pagedattention vllm" §Comparison with Alternatives); the element format is
the OCP FP8 E4M3 ("fn") encoding: sign, 4 exponent bits with bias 7, 3
mantissa bits, no infinities, S.1111.111 = NaN.  These tests hold the
oracle's decoder and encoder to values that follow from that definition by
hand, to torch's independent float8_e4m3fn conversion, and the quantised
decode to the float64 brute force over dequantised values.
"""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import oracle
from oracle import brute
from oracle.cache_ops import e4m3_encode, kv_cache_append, kv_cache_append_e4m3


def _dec(codes):
    return np.array([oracle.lib().pkvo_decode_e4m3(int(c)) for c in codes], dtype=np.float64)


def test_decoder_hand_values():
    # exponent field 7 = 2^0; 0x38 = 1.0, 0x40 = 2.0, 0x3C = 1.5
    assert oracle.lib().pkvo_decode_e4m3(0x38) == 1.0
    assert oracle.lib().pkvo_decode_e4m3(0x40) == 2.0
    assert oracle.lib().pkvo_decode_e4m3(0x3C) == 1.5
    assert oracle.lib().pkvo_decode_e4m3(0xB8) == -1.0
    # largest finite: 2^8 * (1 + 6/8) = 448
    assert oracle.lib().pkvo_decode_e4m3(0x7E) == 448.0
    # smallest normal 2^-6, smallest subnormal 2^-9, largest subnormal 7 * 2^-9
    assert oracle.lib().pkvo_decode_e4m3(0x08) == 2.0 ** -6
    assert oracle.lib().pkvo_decode_e4m3(0x01) == 2.0 ** -9
    assert oracle.lib().pkvo_decode_e4m3(0x07) == 7 * 2.0 ** -9
    assert oracle.lib().pkvo_decode_e4m3(0x00) == 0.0
    assert math.copysign(1.0, oracle.lib().pkvo_decode_e4m3(0x80)) == -1.0
    assert math.isnan(oracle.lib().pkvo_decode_e4m3(0x7F))
    assert math.isnan(oracle.lib().pkvo_decode_e4m3(0xFF))
    # 0x78 (exponent 15, mantissa 0) is a number in this variant: 256
    assert oracle.lib().pkvo_decode_e4m3(0x78) == 256.0


def test_decoder_all_codes_vs_torch():
    codes = np.arange(256, dtype=np.uint8)
    ours = _dec(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])
    # strictly increasing over the positive finite codes
    pos = ours[:0x7F]
    assert np.all(np.diff(pos) > 0)


def test_encoder_round_trip_every_code():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    vals = _dec(codes).astype(np.float32)
    back = e4m3_encode(vals)
    # -0 encodes as 0x80, +0 as 0x00: the round trip is exact on the bits
    assert np.array_equal(back, codes)


def test_encoder_ties_to_even_and_saturation():
    pos = _dec(np.arange(0x7F, dtype=np.uint8))
    mids = ((pos[:-1] + pos[1:]) / 2).astype(np.float32)   # exact in float32
    enc = e4m3_encode(mids)
    lo = np.arange(0x7E, dtype=np.uint8)
    # the tie goes to the code with an even mantissa (last bit 0)
    want = np.where(lo % 2 == 0, lo, lo + 1).astype(np.uint8)
    assert np.array_equal(enc, want)
    # saturation: beyond 448 (and inf) -> 448, sign kept; NaN -> NaN
    big = np.array([448.0, 463.9, 464.0, 500.0, 1e6, np.inf, -1e6, -np.inf], dtype=np.float32)
    assert list(e4m3_encode(big)) == [0x7E] * 6 + [0xFE] * 2
    assert e4m3_encode(np.array([np.nan], dtype=np.float32))[0] & 0x7F == 0x7F


def test_encoder_vs_torch_random():
    rng = np.random.default_rng(7)
    x = np.concatenate([rng.standard_normal(20000) * s for s in (1e-3, 0.05, 1, 30, 200)])
    x = x.astype(np.float32)
    x = x[np.abs(x) < 464]            # torch's cast does not saturate beyond
    ours = e4m3_encode(x)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)


def test_append_e4m3_is_encode_then_append():
    rng = np.random.default_rng(3)
    N, H, bs, D, T = 6, 2, 4, 32, 9
    k = (rng.standard_normal((T, H, D)) * 3).astype(np.float16)
    v = (rng.standard_normal((T, H, D)) * 3).astype(np.float16)
    ks = np.array([0.5, 0.07], dtype=np.float32)
    vs = np.array([0.06, 1.0], dtype=np.float32)
    slots = rng.permutation(N * bs)[:T].astype(np.int64)
    slots[2] = -1
    kc = np.zeros((N, H, bs, D), np.uint8)
    vc = np.zeros_like(kc)
    kv_cache_append_e4m3(kc, vc, k, v, slots, ks, vs, "f16")
    # expected: torch's cast of the float32 quotients (all |y| < 464 here)
    kq = (torch.from_numpy(k.astype(np.float32)) / torch.from_numpy(ks)[None, :, None])
    vq = (torch.from_numpy(v.astype(np.float32)) / torch.from_numpy(vs)[None, :, None])
    assert kq.abs().max() < 464 and vq.abs().max() < 464
    kc2 = np.zeros_like(kc)
    vc2 = np.zeros_like(kc)
    kv_cache_append(kc2, vc2, kq.to(torch.float8_e4m3fn).view(torch.uint8).numpy(),
                    vq.to(torch.float8_e4m3fn).view(torch.uint8).numpy(), slots)
    assert np.array_equal(kc, kc2) and np.array_equal(vc, vc2)


def _tiny_quantised_case(seed, B=3, Hq=4, Hkv=2, D=16, bs=4, N=12):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, Hq, D)).astype(np.float16)
    kc = rng.integers(0, 256, size=(N, Hkv, bs, D)).astype(np.uint8)
    vc = rng.integers(0, 256, size=(N, Hkv, bs, D)).astype(np.uint8)
    # no NaN codes
    kc[(kc & 0x7F) == 0x7F] = 0x3C
    vc[(vc & 0x7F) == 0x7F] = 0x3C
    lens = np.array([0, 5, 11][:B], dtype=np.int32)
    bt = np.stack([rng.permutation(N)[:3] for _ in range(B)]).astype(np.int32)
    ks = np.array([0.01, 0.003], dtype=np.float32)[:Hkv]
    vs = np.array([0.02, 0.5], dtype=np.float32)[:Hkv]
    return q, kc, vc, bt, lens, ks, vs


@pytest.mark.parametrize("window", [0, 3])
def test_quantised_decode_vs_brute(window):
    q, kc, vc, bt, lens, ks, vs = _tiny_quantised_case(11)
    scale = 0.25
    got = oracle.paged_decode(q, kc, vc, bt, lens, scale=scale, dtype="f16", kv_dtype="e4m3",
                              k_scale=ks, v_scale=vs, window=window)
    # brute force over values decoded by torch and scaled in float64
    kd = torch.from_numpy(kc).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    vd = torch.from_numpy(vc).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    kd = kd * ks.astype(np.float64)[None, :, None, None]
    vd = vd * vs.astype(np.float64)[None, :, None, None]
    want = np.array(brute.paged_decode(q.astype(np.float64), kd, vd, bt, lens, scale,
                                       window=window))
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


def test_quantised_decode_power_of_two_scales_equal_f16_decode():
    """With power-of-two scales the dequantised values are exact in fp16, so
    the quantised decode equals the fp16 decode over those values."""
    q, kc, vc, bt, lens, _, _ = _tiny_quantised_case(5)
    ks = np.array([2.0 ** -4, 2.0 ** -7], dtype=np.float32)
    vs = np.array([2.0 ** -2, 1.0], dtype=np.float32)
    got = oracle.paged_decode(q, kc, vc, bt, lens, scale=0.3, dtype="f16", kv_dtype="e4m3",
                              k_scale=ks, v_scale=vs)
    kd = torch.from_numpy(kc).view(torch.float8_e4m3fn).to(torch.float32)
    vd = torch.from_numpy(vc).view(torch.float8_e4m3fn).to(torch.float32)
    k16 = (kd * torch.from_numpy(ks)[None, :, None, None]).to(torch.float16)
    v16 = (vd * torch.from_numpy(vs)[None, :, None, None]).to(torch.float16)
    # exactness of the fp16 copies
    assert torch.equal(k16.float(), kd * torch.from_numpy(ks)[None, :, None, None])
    assert torch.equal(v16.float(), vd * torch.from_numpy(vs)[None, :, None, None])
    want = oracle.paged_decode(q, k16.numpy(), v16.numpy(), bt, lens, scale=0.3, dtype="f16")
    np.testing.assert_array_equal(got, want)


# ---------------------------------------------------------------------------
# per-page scales ([num_blocks, Hkv])

def test_per_page_scales_broadcast_equal_per_head():
    q, kc, vc, bt, lens, ks, vs = _tiny_quantised_case(21)
    N = kc.shape[0]
    a = oracle.paged_decode(q, kc, vc, bt, lens, scale=0.2, dtype="f16", kv_dtype="e4m3",
                            k_scale=ks, v_scale=vs)
    b = oracle.paged_decode(q, kc, vc, bt, lens, scale=0.2, dtype="f16", kv_dtype="e4m3",
                            k_scale=np.tile(ks, (N, 1)), v_scale=np.tile(vs, (N, 1)))
    np.testing.assert_array_equal(a, b)


@pytest.mark.parametrize("window", [0, 4])
def test_per_page_scales_vs_brute(window):
    q, kc, vc, bt, lens, _, _ = _tiny_quantised_case(22)
    N, Hkv = kc.shape[:2]
    g = np.random.default_rng(5)
    ks = g.uniform(0.001, 0.05, size=(N, Hkv)).astype(np.float32)
    vs = g.uniform(0.01, 300.0, size=(N, Hkv)).astype(np.float32)
    got = oracle.paged_decode(q, kc, vc, bt, lens, scale=0.3, dtype="f16", kv_dtype="e4m3",
                              k_scale=ks, v_scale=vs, window=window)
    kd = torch.from_numpy(kc).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    vd = torch.from_numpy(vc).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    kd = kd * ks.astype(np.float64)[:, :, None, None]
    vd = vd * vs.astype(np.float64)[:, :, None, None]
    want = np.array(brute.paged_decode(q.astype(np.float64), kd, vd, bt, lens, 0.3,
                                       window=window))
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


def test_append_per_page_scales():
    rng = np.random.default_rng(9)
    N, H, bs, D, T = 6, 2, 4, 16, 10
    k = (rng.standard_normal((T, H, D))).astype(np.float16)
    v = (rng.standard_normal((T, H, D))).astype(np.float16)
    ks = rng.uniform(0.005, 0.02, size=(N, H)).astype(np.float32)
    vs = rng.uniform(0.005, 0.02, size=(N, H)).astype(np.float32)
    slots = rng.permutation(N * bs)[:T].astype(np.int64)
    slots[1] = -1
    kc = np.zeros((N, H, bs, D), np.uint8)
    vc = np.zeros_like(kc)
    kv_cache_append_e4m3(kc, vc, k, v, slots, ks, vs, "f16")
    for t, s in enumerate(slots):
        if s < 0:
            continue
        blk, off = divmod(int(s), bs)
        for h in range(H):
            want_k = torch.from_numpy(k[t, h].astype(np.float32) / ks[blk, h]) \
                .to(torch.float8_e4m3fn).view(torch.uint8).numpy()
            assert np.array_equal(kc[blk, h, off], want_k)
            want_v = torch.from_numpy(v[t, h].astype(np.float32) / vs[blk, h]) \
                .to(torch.float8_e4m3fn).view(torch.uint8).numpy()
            assert np.array_equal(vc[blk, h, off], want_v)
