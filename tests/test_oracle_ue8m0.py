"""Pins of the oracle's power-of-two (UE8M0) scale mode -- the throughput
study of hardware block scaling beside the pages' method.

The pages fix s = amax/448 ("FP8 Mixed Precision: DeepSeek-V3 Training
Architecture", section 1, eq. s_W).  Block-scaled MMAs take power-of-two
scales (UE8M0 bytes, 2^(b-127)); the reading pinned here rounds the method's
scale up to the next power of two on the method's own tiles.  Pins: the
closed form of that rounding, the UE8M0 byte round trip, codes against
torch's float8_e4m3fn cast of NumPy float32 quotients, no saturation, the
reduction to the method's quantizer when amax/448 is already a power of two,
transposition invariance of the weight blocks, and the GEMM against a NumPy
FP64 product of the dequantized operands.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W


def _f32(bits):
    return W.bf16_bits_to_f32(bits)


def test_pow2_scale_closed_form():
    rng = np.random.default_rng(0)
    t = np.concatenate([np.exp(rng.uniform(-27, 60, 20000)).astype(np.float32),
                        np.float32(2.0) ** np.arange(-39, 100, dtype=np.float32),
                        np.nextafter(np.float32(2.0) ** np.arange(-39, 100, dtype=np.float32), np.float32(np.inf)),
                        np.nextafter(np.float32(2.0) ** np.arange(-39, 100, dtype=np.float32), np.float32(0))])
    got = np.array([oracle.pow2_scale(v) for v in t], np.float64)
    want = np.exp2(np.ceil(np.log2(t.astype(np.float64))))
    assert np.array_equal(got, want)
    m, _ = np.frexp(got)
    assert np.all(m == 0.5)                                   # a power of two
    assert np.all(got >= t) and np.all(got < 2.0 * t)         # the smallest one >= t


def test_ue8m0_round_trip():
    for b in range(0, 255):
        s = float(np.ldexp(np.float32(1.0), b - 127))
        assert oracle.ue8m0_encode(s) == b
    assert oracle.ue8m0_encode(0.3) == -1 and oracle.ue8m0_encode(3.0) == -1


def test_act_pow2_codes_against_torch_cast():
    x = W.activations_with_outliers(96, 512, seed=11, channel_frac=2 / 512, elem_frac=1e-2)
    q, sf = oracle.quant_act_1x128_pow2(x)
    xf = _f32(x).reshape(96, 4, 128)
    amax = np.abs(xf).max(axis=2)
    t = np.vectorize(oracle.tile_scale, otypes=[np.float32])(amax)
    want_sf = np.exp2(np.ceil(np.log2(t.astype(np.float64)))).astype(np.float32)
    assert np.array_equal(sf, want_sf)
    v = (xf / sf[:, :, None]).astype(np.float32)              # exact: division by a power of two
    assert np.all(np.abs(v) <= 448.0)                         # nothing saturates
    want_q = torch.from_numpy(v.reshape(96, 512)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(q, want_q)
    # amax / s2 lies in (224, 448], so the largest code of each tile decodes to
    # a value in [224, 448] (values just above 224 round to it: spacing 16 there)
    assert np.all(amax / sf > 224.0) and np.all(amax / sf <= 448.0)
    dq = np.abs(oracle.e4m3_decode(q).reshape(96, 4, 128)).max(axis=2)
    assert np.all(dq >= 224.0) and np.all(dq <= 448.0)


def test_act_pow2_reduces_to_the_method_when_the_scale_is_a_power_of_two():
    """amax = 28 gives amax/448 = 2^-4 exactly: both rules pick the same scale
    and the same codes."""
    rng = np.random.default_rng(3)
    v = rng.normal(0, 5, (8, 256)).astype(np.float32)
    v = np.clip(v, -27.0, 27.0)
    v[:, 7] = 28.0
    v[:, 200] = -28.0
    bits = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    q2, s2 = oracle.quant_act_1x128_pow2(bits)
    q1, s1 = oracle.quant_act_1x128(bits)
    assert np.all(s1 == np.float32(2.0 ** -4))
    assert np.array_equal(s2, s1) and np.array_equal(q2, q1)


def test_zero_tile_takes_the_floor():
    x = np.zeros((2, 128), np.uint16)
    x[1, :] = 0x8000                                          # -0
    q, sf = oracle.quant_act_1x128_pow2(x)
    assert np.all(sf == np.float32(2.0 ** -39))               # 2^ceil(log2 1e-12)
    assert np.all(q[0] == 0x00) and np.all(q[1] == 0x80)


def test_weight_pow2_blocks_and_transpose():
    w = W.weights(256, 384, seed=4)
    q, sf = oracle.quant_w_128x128_pow2(w)
    qt, sft = oracle.quant_w_128x128_pow2(np.ascontiguousarray(w.T))
    assert np.array_equal(qt, q.T) and np.array_equal(sft, sf.T)
    wf = _f32(w).reshape(2, 128, 3, 128)
    amax = np.abs(wf).max(axis=(1, 3))
    t = np.vectorize(oracle.tile_scale, otypes=[np.float32])(amax)
    assert np.array_equal(sf, np.exp2(np.ceil(np.log2(t.astype(np.float64)))).astype(np.float32))
    v = (wf / sf[:, None, :, None]).astype(np.float32).reshape(256, 384)
    assert np.array_equal(q, torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy())


def test_gemm_with_pow2_scales_against_numpy_fp64():
    x = W.activations_with_outliers(64, 512, seed=5, channel_frac=1 / 512, elem_frac=1e-3)
    w = W.weights(256, 512, seed=6)
    qa, sa = oracle.quant_act_1x128_pow2(x)
    qb, sb = oracle.quant_w_128x128_pow2(w)
    ref = oracle.gemm_sampled(qa, sa, qb, sb, oracle.SFB_BLOCK128)
    da = oracle.e4m3_decode(qa) * np.repeat(sa.astype(np.float64), 128, axis=1)
    db = oracle.e4m3_decode(qb) * np.repeat(np.repeat(sb.astype(np.float64), 128, axis=1), 128, axis=0)
    want = da @ db.T
    assert np.allclose(ref, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())
    # the dequantized operands stay close to the inputs: within a power-of-two step of E4M3
    rel = np.abs(da - _f32(x)) / np.maximum(np.repeat(sa.astype(np.float64), 128, axis=1), 1e-30)
    assert np.all(rel <= 2.0 ** -4 * 448.0)
