"""Pins of the oracle's FP8-activation-cache requantization ("FP8 Mixed
Precision: DeepSeek-V3 Training Architecture", section 4: activations cached
in FP8 for the backward pass): the BF16 dequantization step against exact
rational arithmetic, and the whole chain on activations whose 1x128
quantization is lossless, where it must equal the 128x1 quantizer applied to
the original activation.
"""
from fractions import Fraction

import numpy as np

import oracle
import workloads as W


def _bf16_nearest_even(fr: Fraction) -> float:
    """Round a rational to the nearest BF16 (ties to an even significand), by search."""
    if fr == 0:
        return 0.0
    sign = -1 if fr < 0 else 1
    a = abs(fr)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    ulp = Fraction(2) ** (max(e, -126) - 7)
    lo = (a // ulp) * ulp
    hi = lo + ulp
    if a - lo < hi - a:
        r = lo
    elif hi - a < a - lo:
        r = hi
    else:
        r = lo if (lo / ulp) % 2 == 0 else hi
    return sign * float(r)


def test_dequantization_rounds_the_exact_product_once():
    rng = np.random.default_rng(3)
    codes = rng.integers(0, 256, 384).astype(np.uint8)
    codes = codes[(codes & 0x7F) != 0x7F]                      # no NaN codes
    # scales with full 24-bit significands, so fl32(code * s) often differs from the exact product
    s = (rng.uniform(1.0, 2.0, codes.size) * 2.0 ** rng.integers(-30, 10, codes.size)).astype(np.float32)
    # and products whose float32 rounding lands on a BF16 midpoint (rounding twice would go wrong)
    mc, ms = W.midpoint_product_pairs(128)
    codes, s = np.concatenate([mc, codes]), np.concatenate([ms, s])
    T = 128
    q = np.zeros((T, 128 * 4), np.uint8)
    sf = np.zeros((T, 4), np.float32)
    n = min(codes.size, T * 4)
    rows, tiles = np.divmod(np.arange(n), 4)
    q[rows, tiles * 128] = codes[:n]
    sf[rows, tiles] = s[:n]
    sf[sf == 0] = 1.0
    _, _, xh = oracle.requant_1x128_to_128x1(q, sf)
    got = W.bf16_bits_to_f32(xh[rows, tiles * 128]).astype(np.float64)
    dec = oracle.e4m3_decode(codes[:n])
    want = [_bf16_nearest_even(Fraction(float(d)) * Fraction(float(v))) for d, v in zip(dec, s[:n])]
    assert np.array_equal(got, np.array(want))


def test_lossless_cache_gives_the_direct_128x1_quantization():
    """Tiles holding E4M3 values times 2^k with 448 * 2^k among them quantize
    1x128 without loss (s = 2^k), so the cache dequantizes to the activation
    itself and the requantized operand equals the 128x1 quantizer's."""
    rng = np.random.default_rng(5)
    T, C = 256, 384
    codes = rng.integers(0, 0x7F, (T, C)).astype(np.uint8) | (rng.integers(0, 2, (T, C)) << 7).astype(np.uint8)
    codes[:, ::128] = 0x7E                                       # every tile holds +448
    k = rng.integers(-20, 10, (T, C // 128))
    vals = oracle.e4m3_decode(codes).reshape(T, C) * np.repeat(2.0 ** k, 128, axis=1)
    x = (vals.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    q, sf = oracle.quant_act_1x128(x)
    assert np.array_equal(q, codes) and np.array_equal(sf, (2.0 ** k).astype(np.float32))
    qt, sft, xh = oracle.requant_1x128_to_128x1(q, sf)
    assert np.array_equal(xh, x)
    qt_direct, sft_direct = oracle.quant_act_128x1(x)
    assert np.array_equal(qt, qt_direct) and np.array_equal(sft, sft_direct)


def test_zero_cache():
    q = np.zeros((128, 256), np.uint8)
    q[3, 5] = 0x80                                                # -0 stays -0
    sf = np.full((128, 2), np.float32(1e-12), np.float32)
    qt, sft, xh = oracle.requant_1x128_to_128x1(q, sf)
    assert np.all(qt[np.arange(256) != 5] == 0) and qt[5, 3] == 0x80
    assert np.all(sft == np.float32(1e-12)) and xh[3, 5] == 0x8000
