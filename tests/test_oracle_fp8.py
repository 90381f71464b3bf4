"""Pins of the oracle's FP8 (e4m3) storage: torch's float8_e4m3fn as an
independent implementation of the format, hand-worked values, saturation."""
import math

import numpy as np
import pytest
import torch

from oracle import fp8
from oracle.cache_ops import reshape_and_cache, reshape_and_cache_fp8
from oracle.paged_attention import paged_attention_decode, paged_attention_decode_fp8


def test_decode_every_code_matches_torch():
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    ours = fp8.decode_array(np.arange(256))
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan) and nan.sum() == 2
    assert np.array_equal(ours[~nan], ref[~nan])
    assert fp8.decode(0x7E) == 448.0 and fp8.decode(0x01) == 2.0 ** -9 and fp8.decode(0x08) == 2.0 ** -6


def test_encode_matches_torch_inside_the_range():
    # every value on a fine grid, every code's midpoint to its neighbours (ties), and random values
    codes = np.arange(256)
    vals = fp8.decode_array(codes)
    finite = np.sort(np.unique(vals[np.isfinite(vals)]))
    mids = (finite[1:] + finite[:-1]) / 2
    rng = np.random.default_rng(0)
    x = np.concatenate([finite, mids, np.nextafter(mids, np.inf), np.nextafter(mids, -np.inf),
                        rng.standard_normal(20000) * 30, rng.uniform(-463, 463, 20000)]).astype(np.float32)
    x = x[np.abs(x) < 464]
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(fp8.encode_array(x), ref)


def test_hand_worked_values_and_saturation():
    assert fp8.encode(1.0) == 0x38
    assert fp8.encode(1.0625) == 0x38              # tie between 1 and 1.125: even mantissa
    assert fp8.encode(1.1875) == 0x3A              # tie between 1.125 and 1.25: even mantissa
    assert fp8.encode(2.0 ** -10) == 0x00          # half of the smallest subnormal: ties to 0
    assert fp8.encode(3 * 2.0 ** -11) == 0x01      # 0.75 of it: rounds up
    assert fp8.encode(-0.0) == 0x80
    for big in (449.0, 464.0, 479.9, 480.0, 1e9, math.inf):
        assert fp8.encode(big) == 0x7E and fp8.encode(-big) == 0xFE
    assert fp8.encode(math.nan) == 0x7F


def test_quantize_uses_float32_products():
    x = np.float32(1.0 / 3.0)
    scale = 0.0123
    inv = np.float32(1.0) / np.float32(scale)
    assert fp8.quantize(np.array([x]), scale)[0] == fp8.encode(float(np.float32(x * inv)))
    # dequantised values are within half a quantum of the input
    xs = np.random.default_rng(1).standard_normal(5000).astype(np.float32)
    d = fp8.dequantize(fp8.quantize(xs, 1 / 64), 1 / 64)
    assert np.all(np.abs(d - xs) <= np.abs(xs) * 2 ** -4 + 2 ** -9 / 64)


def test_fp8_attention_is_attention_over_dequantised_cache():
    rng = np.random.default_rng(2)
    nb, bs, hkv, d = 10, 4, 2, 8
    k = rng.standard_normal((13, hkv, d)).astype(np.float32)
    v = rng.standard_normal((13, hkv, d)).astype(np.float32)
    slots = np.array([5 * 4 + i for i in range(4)] + [2 * 4 + i for i in range(4)] + [7 * 4 + i for i in range(4)]
                     + [1 * 4])
    kc = np.zeros((nb, bs, hkv, d), np.uint8)
    vc = np.zeros((nb, bs, hkv, d), np.uint8)
    reshape_and_cache_fp8(k, v, kc, vc, slots, 1 / 64, 1 / 32)
    kd = np.zeros((nb, bs, hkv, d))
    vd = np.zeros((nb, bs, hkv, d))
    reshape_and_cache(fp8.dequantize(fp8.quantize(k, 1 / 64), 1 / 64), fp8.dequantize(fp8.quantize(v, 1 / 32), 1 / 32),
                      kd, vd, slots)
    q = rng.standard_normal((1, 4, d))
    table = [[5, 2, 7, 1]]
    a = paged_attention_decode_fp8(q, kc, vc, table, [13], 0.35, bs, 1 / 64, 1 / 32)
    b = paged_attention_decode(q, kd, vd, table, [13], 0.35, bs)
    assert np.array_equal(a, b)


@pytest.mark.parametrize("mistake", ["truncate", "bias8", "no_saturate"])
def test_planted_encoder_mistakes_are_caught(mistake):
    def bad(x):
        if mistake == "truncate":
            a = abs(x)
            if a == 0:
                return 0
            e = max(math.floor(math.log2(a)), -6)
            n = int(a / 2.0 ** (e - 3))                    # truncates instead of rounding
            s = 0x80 if x < 0 else 0
            return s | (n if e == -6 and n < 8 else ((e + 7) << 3) | (n - 8))
        if mistake == "bias8":
            c = fp8.encode(x)
            return (c & 0x87) | ((((c >> 3) & 0xF) + 1) & 0xF) << 3 if c & 0x78 else c
        c = fp8.encode(x)
        return 0x7F if abs(x) > 448 else c
    xs = [1.0625, 0.3, -2.7, 500.0, 100.0]
    assert any(bad(x) != fp8.encode(x) for x in xs)


def test_array_encoder_equals_scalar_definition():
    rng = np.random.default_rng(9)
    vals = fp8.decode_array(np.arange(256))
    fin = np.sort(np.unique(vals[np.isfinite(vals)]))
    mids = (fin[1:] + fin[:-1]) / 2
    x = np.concatenate([fin, -fin, mids, -mids, np.nextafter(mids, 0), np.nextafter(mids, 1e9),
                        rng.standard_normal(5000) * 50, [0.0, -0.0, 1e-300, 464.0, 480.0, 1e9, -1e9, math.inf,
                                                          -math.inf, math.nan]])
    assert np.array_equal(fp8.encode_array(x), np.array([fp8.encode(v) for v in x], dtype=np.uint8))
