"""Pins of the oracle's per-tensor baseline ("FP8 Mixed Precision: DeepSeek-V3
Training Architecture", section 1, the per-tensor scaling of its error
comparison): the codes against NumPy's float32 division and the codec, the
special case of a tensor that is one 1x128 tile (where per-tensor and
fine-grained scaling coincide), the oracle's other per-tensor routine, and the
per-tensor GEMM against NumPy's FP64 matrix product of the decoded operands.
"""
import numpy as np

import oracle
import workloads as W


def test_pertensor_codes_against_numpy():
    x = W.activations_with_outliers(37, 640, seed=2, channel_frac=2 / 640, elem_frac=1e-2)
    q, amax, s = oracle.quant_pertensor(x)
    xf = W.bf16_bits_to_f32(x)
    assert np.float32(amax) == np.abs(xf).max()
    assert np.float32(s) == np.float32(oracle.tile_scale(np.abs(xf).max()))
    assert np.array_equal(q, oracle.e4m3_encode((xf / np.float32(s)).astype(np.float32)))


def test_pertensor_of_one_tile_is_the_tile_quantizer():
    x = W.activations_with_outliers(1, 128, seed=4, channel_frac=0, elem_frac=2e-2)
    q, _, s = oracle.quant_pertensor(x)
    q1, sf1 = oracle.quant_act_1x128(x)
    assert np.array_equal(q, q1) and np.float32(s) == sf1[0, 0]


def test_pertensor_codes_agree_with_the_dequantizing_routine():
    x = W.activations_with_outliers(8, 256, seed=6)
    q, _, s = oracle.quant_pertensor(x)
    deq, s2 = oracle.quant_pertensor_e4m3(x)
    assert np.float32(s) == np.float32(s2)
    assert np.array_equal(oracle.e4m3_decode(q).reshape(deq.shape) * np.float64(np.float32(s)), deq)


def test_pertensor_gemm_against_numpy():
    qa, _, sa = oracle.quant_pertensor(W.activations_with_outliers(20, 384, seed=1))
    qb, _, sb = oracle.quant_pertensor(W.weights(256, 384, seed=1))
    ref = oracle.gemm_pertensor_sampled(qa, sa, qb, sb)
    da = oracle.e4m3_decode(qa).reshape(qa.shape)
    db = oracle.e4m3_decode(qb).reshape(qb.shape)
    direct = (np.float64(np.float32(sa)) * np.float64(np.float32(sb))) * (da @ db.T)
    assert np.allclose(ref, direct, rtol=1e-12, atol=1e-12 * np.abs(direct).max())
    rows, cols = np.array([0, 7, 19]), np.array([3, 255])
    assert np.array_equal(oracle.gemm_pertensor_sampled(qa, sa, qb, sb, rows=rows, cols=cols), ref[np.ix_(rows, cols)])
