"""Pins for the oracle's FP8 / BF16 codecs (CPU only).

The oracle's E4M3 / E5M2 codecs are written from the OCP "FP8 Formats for Deep
Learning" definition (listed as a primary source by "Online Quantization
During Training" and "Fine-Grained FP8 Quantization in DeepSeek").  They are
pinned here against things other than themselves:
  * brute-force enumeration of all 256 codes and the format facts the pages
    print (E4M3 max 448: "FP8 Mixed Precision: DeepSeek-V3 Training
    Architecture", section 3 "Why Naive FP8 Training Suffers Precision Collapse"),
  * PyTorch's independent float8_e4m3fn / float8_e5m2 dtypes (a library cast),
  * a brute-force nearest-value search over the decoded code table.
"""
import numpy as np
import pytest
import torch

import oracle


def _all_codes():
    return np.arange(256, dtype=np.uint8)


def test_e4m3_enumeration_facts(page_values):
    dec = oracle.e4m3_decode(_all_codes())
    nan = np.isnan(dec)
    assert set(np.nonzero(nan)[0].tolist()) == {0x7F, 0xFF}
    fin = dec[~nan]
    assert fin.size == 254
    assert fin.max() == page_values["e4m3_max"]["value"] == dec[0x7E]
    assert fin.min() == -448.0 == dec[0xFE]
    assert dec[0x08] == 2.0 ** -6        # smallest normal
    assert dec[0x01] == 2.0 ** -9        # smallest subnormal
    assert dec[0x38] == 1.0              # exponent bias 7
    assert dec[0x00] == 0.0 and np.signbit(dec[0x80]) and dec[0x80] == 0.0
    pos = np.sort(dec[1:0x7F])
    assert pos.size == 126 and np.all(np.diff(pos) > 0)  # 126 distinct positive values
    # every positive normal binade holds 8 values with spacing 2^(e-3)
    for e in range(-6, 9):
        binade = pos[(pos >= 2.0 ** e) & (pos < 2.0 ** (e + 1))]
        if e < 8:
            assert binade.size == 8 and np.allclose(np.diff(binade), 2.0 ** (e - 3))
        else:
            assert binade.size == 7     # 256..448, the all-ones code is NaN


def test_e4m3_round_trip_all_codes():
    codes = _all_codes()
    dec = oracle.e4m3_decode(codes)
    ok = ~np.isnan(dec)
    re = oracle.e4m3_encode(dec[ok].astype(np.float32))
    assert np.array_equal(re, codes[ok])


def test_e4m3_decode_matches_torch_dtype():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    t = codes.view(torch.float8_e4m3fn).double().numpy()
    d = oracle.e4m3_decode(_all_codes())
    both_nan = np.isnan(t) & np.isnan(d)
    assert np.array_equal(np.isnan(t), np.isnan(d))
    assert np.array_equal(t[~both_nan], d[~both_nan])
    assert np.array_equal(np.signbit(t[~both_nan]), np.signbit(d[~both_nan]))


def _float_sweep(lo_exp, hi_exp, stride):
    """float32 bit patterns with exponents in [lo_exp, hi_exp], every `stride`-th mantissa, both signs."""
    out = []
    for e in range(lo_exp, hi_exp + 1):
        base = np.uint32((e + 127) << 23)
        mant = np.arange(0, 1 << 23, stride, dtype=np.uint32)
        mant = np.concatenate([mant, np.array([0x3FFFF, 0x40000, 0x40001, 0x7FFFF, 0x80000, 0x80001,
                                               0xBFFFF, 0xC0000, 0xC0001, 0xFFFFF, 0x100000, 0x100001,
                                               0x7FFFFF], np.uint32)])
        out.append(base | mant)
    u = np.concatenate(out)
    u = np.concatenate([u, u | np.uint32(0x80000000)])
    return u.view(np.float32)


def test_e4m3_encode_matches_torch_cast_below_saturation():
    # below 464 torch's RNE cast and the satfinite cast agree by definition
    x = _float_sweep(-20, 8, 97)
    x = x[np.abs(x) <= 464.0]
    ref = torch.from_numpy(x.copy()).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = oracle.e4m3_encode(x)
    bad = np.nonzero(ref != got)[0]
    assert bad.size == 0, (x[bad[:5]], ref[bad[:5]], got[bad[:5]])


def test_e4m3_encode_is_nearest_ties_even_bruteforce():
    codes = np.arange(0x00, 0x7F, dtype=np.uint8)
    vals = oracle.e4m3_decode(codes)
    rng = np.random.default_rng(7)
    x = np.concatenate([rng.uniform(0, 450, 20000), rng.uniform(0, 2.0 ** -5, 20000),
                        (vals[:-1] + vals[1:]) / 2.0]).astype(np.float32)     # include every midpoint
    got = oracle.e4m3_encode(x)
    xd = x.astype(np.float64)
    for xi, gi in zip(xd, got):
        if xi >= 448.0:
            assert gi == 0x7E
            continue
        d = np.abs(vals - xi)
        best = np.nonzero(d == d.min())[0]
        if best.size == 1:
            assert gi == codes[best[0]]
        else:   # tie: the even code (mantissa LSB 0)
            even = [codes[b] for b in best if codes[b] % 2 == 0]
            assert len(even) == 1 and gi == even[0]


def test_e4m3_saturation_and_signs():
    x = np.array([448.0, 449.0, 463.9, 464.0, 470.0, 480.0, 1e30, np.inf,
                  -448.0, -464.0, -1e30, -np.inf, 0.0, -0.0, -1e-30, 1e-30], np.float32)
    got = oracle.e4m3_encode(x)
    assert got.tolist() == [0x7E] * 8 + [0xFE] * 4 + [0x00, 0x80, 0x80, 0x00]
    assert oracle.e4m3_encode(np.array([np.nan], np.float32))[0] & 0x7F == 0x7F


def test_e4m3_ties_to_even_examples():
    # 1.0625 lies between 1.0 (mantissa 0) and 1.125 (mantissa 1): goes to 1.0
    # 1.1875 lies between 1.125 (m=1) and 1.25 (m=2): goes to 1.25
    # 2^-10 lies between 0 and the smallest subnormal 2^-9: goes to 0
    # 3 * 2^-10 lies between 2^-9 (m=1) and 2^-8 (m=2): goes to 2^-8
    x = np.array([1.0625, 1.1875, 2.0 ** -10, 3 * 2.0 ** -10], np.float32)
    assert oracle.e4m3_decode(oracle.e4m3_encode(x)).tolist() == [1.0, 1.25, 0.0, 2.0 ** -8]


def test_outlier_shrink_values_are_exact_e4m3(page_values):
    # "Introduction to LLM Quantization": with an outlier 32 dividing the
    # values, 0.25 and 0.5 shrink to 0.0078 and 0.0156 (printed to 4 places).
    ex = page_values["outlier_shrink"]
    shrunk = np.array(ex["values"], np.float64) / ex["outlier"]
    assert np.allclose(np.round(shrunk, ex["printed_decimals"]), ex["printed_results"])
    codes = oracle.e4m3_encode(shrunk.astype(np.float32))
    assert codes.tolist() == [0x04, 0x08]       # 2^-7 (subnormal) and 2^-6 (smallest normal)
    assert oracle.e4m3_decode(codes).tolist() == shrunk.tolist()
    # the page's point: down there E4M3 has lost its mantissa: the relative
    # spacing at 2^-7 is 2^-9 / 2^-7 = 1/4, versus 1/8 in every normal binade
    vals = np.sort(oracle.e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8)))
    i = np.searchsorted(vals, shrunk[0])
    assert (vals[i + 1] - vals[i]) / vals[i] == 0.25


def test_e5m2_ranges_and_torch():
    codes = _all_codes()
    dec = oracle.e5m2_decode(codes)
    t = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e5m2).double().numpy()
    assert np.array_equal(np.isnan(dec), np.isnan(t))
    m = ~np.isnan(dec)
    assert np.array_equal(dec[m], t[m])
    assert dec[0x7B] == 57344.0 and np.isinf(dec[0x7C]) and np.isnan(dec[0x7D])
    assert dec[0x04] == 2.0 ** -14 and dec[0x01] == 2.0 ** -16
    # wider range, lower precision than E4M3 ("Introduction to LLM Quantization", E4M3 vs E5M2)
    assert dec[0x7B] > oracle.e4m3_decode(np.array([0x7E], np.uint8))[0]
    # relative spacing in a normal binade: 2^-2 for E5M2 vs 2^-3 for E4M3
    assert dec[0x3D] - dec[0x3C] == 0.25 * dec[0x3C]      # 1.25 - 1.0
    x = _float_sweep(-18, 15, 211)
    x = x[np.abs(x) < 57344.0]
    ref = torch.from_numpy(x.copy()).to(torch.float8_e5m2).view(torch.uint8).numpy()
    assert np.array_equal(ref, oracle.e5m2_encode(x))


def test_round_bf16_and_f32_single_rounding():
    rng = np.random.default_rng(3)
    # values exactly representable in float32: torch's f32 -> bf16 cast is a single RNE rounding
    x32 = (rng.standard_normal(100000) * np.exp2(rng.integers(-40, 40, 100000))).astype(np.float32)
    ref = torch.from_numpy(x32).to(torch.bfloat16).double().numpy()
    assert np.array_equal(oracle.round_bf16(x32.astype(np.float64)), ref)
    x64 = rng.standard_normal(100000) * np.exp2(rng.integers(-40, 40, 100000))
    assert np.array_equal(oracle.round_f32(x64), x64.astype(np.float32).astype(np.float64))
    # a double just above a bf16 midpoint must round up (a float32 detour would round to even)
    mid = 1.0 + 2.0 ** -8                    # midpoint between 1 and 1 + 2^-7
    assert oracle.round_bf16(np.array([mid + 2.0 ** -40]))[0] == 1.0 + 2.0 ** -7
    assert oracle.round_bf16(np.array([mid]))[0] == 1.0
