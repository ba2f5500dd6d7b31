"""Pins of the oracle's E5M2 gradient variant ("FP8 Mixed Precision:
DeepSeek-V3 Training Architecture", "2. Universal E4M3"; "Introduction to LLM
Quantization", "E4M3 vs E5M2"): the tile rule with the E5M2 maximum, checked
against NumPy's float32 arithmetic and the codec; the 128x1 quantizer as the
1x128 one on the transpose; the formats' precision ordering the pages state
(E4M3 the finer grid, E5M2 the wider range); and the GEMM on E5M2 operands
against NumPy's FP64 product of the decoded operands.
"""
import numpy as np

import oracle
import workloads as W


def test_e5m2_tile_rule_against_numpy():
    x = W.grad_with_outlier_tokens(24, 512, seed=4)
    q, sf = oracle.quant_act_1x128_e5m2(x)
    xf = W.bf16_bits_to_f32(x).reshape(24, 4, 128)
    amax = np.abs(xf).max(axis=2)
    s_np = np.maximum((amax / np.float32(57344.0)).astype(np.float32), np.float32(1e-12))
    assert np.array_equal(sf, s_np)
    v = (xf / s_np[:, :, None]).astype(np.float32).reshape(24, 512)
    assert np.array_equal(q, oracle.e5m2_encode(v))
    # every tile reaches the format's maximum magnitude exactly at its amax
    dec = np.abs(oracle.e5m2_decode(q).reshape(24, 4, 128)).max(axis=2)
    assert np.all(dec == 57344.0)


def test_e5m2_128x1_is_1x128_of_the_transpose():
    x = W.grad_with_outlier_tokens(256, 384, seed=6)
    qt, sft = oracle.quant_act_128x1_e5m2(x)
    xt = np.ascontiguousarray(x.T)
    q1, sf1 = oracle.quant_act_1x128_e5m2(xt)
    assert np.array_equal(qt, q1) and np.array_equal(sft, sf1.T)


def test_e4m3_is_finer_and_e5m2_wider():
    """On the same gradient tiles the E4M3 round trip has the smaller error
    (3 mantissa bits against 2), while the E5M2 grid reaches far smaller
    magnitudes relative to the tile maximum before flushing to zero."""
    x = W.grad_with_outlier_tokens(64, 1024, seed=2)
    xf = W.bf16_bits_to_f32(x).astype(np.float64)
    q4, s4 = oracle.quant_act_1x128(x)
    q5, s5 = oracle.quant_act_1x128_e5m2(x)
    d4 = oracle.e4m3_decode(q4).reshape(x.shape) * np.repeat(s4, 128, axis=1)
    d5 = oracle.e5m2_decode(q5).reshape(x.shape) * np.repeat(s5, 128, axis=1)
    e4 = np.linalg.norm(d4 - xf) / np.linalg.norm(xf)
    e5 = np.linalg.norm(d5 - xf) / np.linalg.norm(xf)
    assert e4 < e5 < 4 * e4
    # smallest nonzero magnitude relative to the maximum: 2^-9/448 against 2^-16/57344
    assert oracle.e4m3_decode(np.array([1], np.uint8))[0] / 448 > 1e4 * oracle.e5m2_decode(np.array([1], np.uint8))[0] / 57344


def test_gemm_with_e5m2_operand_against_numpy():
    qa, sa = oracle.quant_act_1x128_e5m2(W.grad_with_outlier_tokens(12, 256, seed=1))
    qb, sb = oracle.quant_w_128x128(W.weights(256, 256, seed=1))
    ref = oracle.gemm_sampled(qa, sa, qb, sb, oracle.SFB_BLOCK128, a_fmt=oracle.FMT_E5M2)
    da = oracle.e5m2_decode(qa).reshape(qa.shape) * np.repeat(sa.astype(np.float64), 128, axis=1)
    db = oracle.e4m3_decode(qb).reshape(qb.shape) * np.repeat(np.repeat(sb.astype(np.float64), 128, axis=0), 128, axis=1)
    direct = da @ db.T
    assert np.allclose(ref, direct, rtol=1e-12, atol=1e-12 * np.abs(direct).max())
