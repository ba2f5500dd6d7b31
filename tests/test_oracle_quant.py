"""Pins for the oracle's quantizers (CPU only).

Passages: "Fine-Grained FP8 Quantization in DeepSeek" sections 2-3 and its
worked example; "FP8 Mixed Precision: DeepSeek-V3 Training Architecture",
eq. s_W = max|block|/448 and eq. W_FP8, "Step 1" and "Step 2" listings;
"Introduction to LLM Quantization", "INT8" and "5) Online Quantization".

Pins used (none re-types the oracle's own code):
  * a torch composite of library ops (fp32 max, IEEE fp32 division, PyTorch's
    float8_e4m3fn cast) on the same inputs,
  * closed-form invariants: each tile's largest code decodes to 448, the
    reconstruction error stays within half an E4M3 spacing,
  * structural identities: 128x1 tiles of X equal 1x128 tiles of X^T; weight
    blocks of W^T equal the transposed blocks of W,
  * the pages' worked examples (two tiles near 0.1 vs outlier 20, INT8 with
    alpha = 10.8, per-tensor vs fine-grained error).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W


def torch_quant_1x128(x_bits):
    x = torch.from_numpy(W.bf16_bits_to_f32(x_bits))
    M, K = x.shape
    t = x.reshape(M, K // 128, 128)
    amax = t.abs().amax(dim=-1, keepdim=True)
    s = torch.clamp(amax / 448.0, min=torch.tensor(1e-12, dtype=torch.float32))
    q = (t / s).to(torch.float8_e4m3fn).view(torch.uint8).reshape(M, K)
    return q.numpy(), s.reshape(M, K // 128).numpy()


def _inputs(M, K, seed):
    return W.activations_with_outliers(M, K, seed=seed, channel_frac=3 / K if K >= 384 else 0.0,
                                       elem_frac=4e-4)


@pytest.mark.parametrize("M,K,seed", [(7, 384, 1), (64, 1024, 2), (130, 256, 3)])
def test_quant_1x128_matches_torch_composite(M, K, seed):
    x = _inputs(M, K, seed)
    q, sf = oracle.quant_act_1x128(x)
    tq, tsf = torch_quant_1x128(x)
    assert np.array_equal(sf, tsf)
    assert np.array_equal(q, tq)


def test_quant_1x128_invariants():
    x = _inputs(96, 2048, 5)
    q, sf = oracle.quant_act_1x128(x)
    xf = W.bf16_bits_to_f32(x).astype(np.float64).reshape(96, 16, 128)
    dec = oracle.e4m3_decode(q).reshape(96, 16, 128)
    # the largest code of each (non-zero) tile decodes to exactly 448
    assert np.all(np.abs(dec).max(axis=-1) == 448.0)
    # scale is amax/448 within float rounding
    amax = np.abs(xf).max(axis=-1)
    assert np.allclose(sf, amax / 448.0, rtol=2 ** -23, atol=0)
    # reconstruction: |dec*s - x| <= half spacing*s (+ the fp32 division's rounding)
    y = xf / sf[..., None]
    spacing = np.where(np.abs(y) < 2.0 ** -6, 2.0 ** -9, 2.0 ** (np.floor(np.log2(np.maximum(np.abs(y), 1e-300))) - 3))
    assert np.all(np.abs(dec - y) <= spacing / 2 + np.abs(y) * 2.0 ** -23)


def test_quant_1x128_zero_and_signed_zero_tiles():
    x = np.zeros((2, 256), np.uint16)
    x[1, :128] = 0x8000                       # -0.0 everywhere in tile (1, 0)
    x[1, 128 + 5] = W.f32_to_bf16_bits(np.array([3.0], np.float32))[0]   # a single non-zero value
    q, sf = oracle.quant_act_1x128(x)
    assert sf[0, 0] == np.float32(1e-12) and sf[1, 0] == np.float32(1e-12)
    assert np.all(q[0] == 0x00) and np.all(q[1, :128] == 0x80)
    assert sf[1, 1] == np.float32(3.0) / np.float32(448.0)
    assert q[1, 128 + 5] == 0x7E and np.count_nonzero(q[1, 128:]) == 1


def test_quant_128x1_equals_1x128_of_transpose():
    x = _inputs(256, 384, 9)                   # T=256, C=384
    qt, sf = oracle.quant_act_128x1(x)
    q1, sf1 = oracle.quant_act_1x128(np.ascontiguousarray(x.T))
    assert np.array_equal(qt, q1)              # [C][T]
    assert np.array_equal(sf, sf1.T)           # [T/128][C]


def test_quant_w_blocks_torch_and_transpose():
    w = W.weights(384, 256, seed=4)
    w[5, 7] = W.f32_to_bf16_bits(np.array([1.5], np.float32))[0]     # an outlier in block (0,0)
    q, sf = oracle.quant_w_128x128(w)
    wf = torch.from_numpy(W.bf16_bits_to_f32(w))
    blocks = wf.reshape(3, 128, 2, 128).permute(0, 2, 1, 3)
    s = torch.clamp(blocks.abs().amax(dim=(2, 3), keepdim=True) / 448.0, min=torch.tensor(1e-12))
    tq = (blocks / s).to(torch.float8_e4m3fn).view(torch.uint8).permute(0, 2, 1, 3).reshape(384, 256)
    assert np.array_equal(sf, s.reshape(3, 2).numpy())
    assert np.array_equal(q, tq.numpy())
    qT, sfT = oracle.quant_w_128x128(np.ascontiguousarray(w.T))
    assert np.array_equal(qT, q.T) and np.array_equal(sfT, sf.T)


def test_scale_overhead(page_values):
    # 4 bytes of FP32 scale per 128 FP8 values: 1/32 of the payload (3.125 %)
    ov = page_values["scale_bytes_per_value_fp32_per_128"]
    x = _inputs(8, 1024, 1)
    q, sf = oracle.quant_act_1x128(x)
    assert sf.nbytes / q.size == ov["scale_bytes"] / ov["values"] == 0.03125
    assert sf.nbytes / q.nbytes == 1 / 32
    # the worked example's two tiles: two local scales vs one global scale
    ex = page_values["two_tiles"]
    assert ex["n_local_scales"] * 4 / (2 * ex["tile_len"]) == 0.03125
    assert 4 / (2 * ex["tile_len"]) == 0.015625


def _two_tiles(seed=0):
    ex_rng = np.random.Generator(np.random.Philox(key=[seed, 77]))
    a = 0.1 + 0.01 * ex_rng.standard_normal(128)
    b = ex_rng.standard_normal(128)
    b[17] = 20.0
    return W.f32_to_bf16_bits(np.concatenate([a, b]).astype(np.float32)).reshape(1, 256)


def test_two_tile_worked_example(page_values):
    """Two 128-value tiles, one near 0.1, one holding the outlier 20, under one
    global scale versus two local scales ("Fine-Grained FP8 Quantization in
    DeepSeek", worked example)."""
    ex = page_values["two_tiles"]
    x = _two_tiles()
    xf = W.bf16_bits_to_f32(x).astype(np.float64)[0]
    q_loc, sf_loc = oracle.quant_act_1x128(x)                # two local scales
    deq_glob, s_glob = oracle.quant_pertensor_e4m3(x)        # one scale for both tiles
    deq_loc = oracle.e4m3_decode(q_loc)[0] * np.repeat(sf_loc[0].astype(np.float64), 128)
    # tile B holds the global max, so its local scale is the global one: identical bytes
    assert sf_loc[0, 1] == np.float32(s_glob) == np.float32(ex["tile_b_outlier"]) / np.float32(448)
    assert np.array_equal(deq_loc[128:], deq_glob[0, 128:])
    # tile A (values ~0.1 scaled by 448/20 ~ 2.2) stays in E4M3's normal range
    # under both scales, so both reconstruct within 2^-4 relative
    a = xf[:128]
    for d in (deq_loc[:128], deq_glob[0, :128]):
        assert np.all(np.abs(d - a) <= 2.0 ** -4 * np.abs(a) * (1 + 1e-6))
    # under the integer-grid model of the "Step 1" listing the local scale is far better
    loc_int = oracle.quant_tiles_intgrid(xf, 128)
    glob_int = oracle.quant_tiles_intgrid(xf, 256)
    e_loc = np.linalg.norm(loc_int[:128] - a)
    e_glob = np.linalg.norm(glob_int[:128] - a)
    assert e_loc * 10 <= e_glob
    # an E4M3 case where local scaling must win: a tile near 1e-3 next to an
    # outlier of 120 goes subnormal under the global scale (1e-3*448/120 < 2^-6)
    y = np.concatenate([1e-3 * (1 + 0.1 * np.random.default_rng(1).standard_normal(128)),
                        np.r_[120.0, np.zeros(127)]]).astype(np.float32)
    yb = W.f32_to_bf16_bits(y).reshape(1, 256)
    yf = W.bf16_bits_to_f32(yb).astype(np.float64)[0]
    ql, sl = oracle.quant_act_1x128(yb)
    dl = oracle.e4m3_decode(ql)[0, :128] * float(sl[0, 0])
    dg, _ = oracle.quant_pertensor_e4m3(yb)
    assert np.linalg.norm(dl - yf[:128]) * 2 < np.linalg.norm(dg[0, :128] - yf[:128])


def test_int8_absmax_example(page_values):
    ex = page_values["int8_absmax"]
    x = np.array([ex["alpha"], -ex["alpha"], 0.0, ex["alpha"] / 2, 1.0, -3.3])
    q, s = oracle.int8_absmax(x)
    assert s == ex["alpha"] / ex["multiplier"]
    assert q[:3].tolist() == [127, -127, 0]
    assert q[3] == 64                             # 63.5 rounds half to even -> 64
    assert q[4] == round(1.0 / 10.8 * 127) == 12
    assert q[5] == -39                            # -3.3/10.8*127 = -38.8


def test_p3_fixture_fine_beats_per_tensor(page_values):
    """'Step 2' of the FP8 Mixed Precision page: X 64x512 ~0.4 N(0,1) with
    channel 88 shifted by +35, W 1024x512 ~0.08 N(0,1); fine-grained (1x128 /
    128x128) relative error below per-tensor.  The page prints no output
    values, so only the ordering is pinned; the integer-grid model of its
    listing is used, as is an E4M3 run on the same data."""
    ex = page_values["per_tensor_vs_fine_fixture"]
    rs = np.random.RandomState(ex["seed"])
    X = rs.randn(ex["N"], ex["D"]) * ex["x_sigma"]
    X[:, ex["outlier_column"]] += ex["outlier_add"]
    Wm = rs.randn(ex["M"], ex["D"]) * ex["w_sigma"]
    Y = X @ Wm.T
    # integer-grid model
    Xp = oracle.quant_tiles_intgrid(X, X.size)
    Wp = oracle.quant_tiles_intgrid(Wm, Wm.size)
    Xf = oracle.quant_tiles_intgrid(X, 128)
    Wblk = Wm.reshape(8, 128, 4, 128).transpose(0, 2, 1, 3).reshape(32, 128 * 128)
    Wf = oracle.quant_tiles_intgrid(Wblk, 128 * 128).reshape(8, 4, 128, 128).transpose(0, 2, 1, 3).reshape(1024, 512)
    e_pt = np.linalg.norm(Xp @ Wp.T - Y) / np.linalg.norm(Y)
    e_fg = np.linalg.norm(Xf @ Wf.T - Y) / np.linalg.norm(Y)
    assert e_fg < e_pt
    # E4M3 on the BF16-rounded inputs
    Xb = W.f32_to_bf16_bits(X.astype(np.float32))
    Wb = W.f32_to_bf16_bits(Wm.astype(np.float32))
    qx, sx = oracle.quant_act_1x128(Xb)
    qw, sw = oracle.quant_w_128x128(Wb)
    Yf = oracle.gemm_sampled(qx, sx, qw, sw, oracle.SFB_BLOCK128)
    dxp, _ = oracle.quant_pertensor_e4m3(Xb)
    dwp, _ = oracle.quant_pertensor_e4m3(Wb)
    Yb = W.bf16_bits_to_f32(Xb).astype(np.float64) @ W.bf16_bits_to_f32(Wb).astype(np.float64).T
    e8_fg = np.linalg.norm(Yf - Yb) / np.linalg.norm(Yb)
    e8_pt = np.linalg.norm(dxp @ dwp.T - Yb) / np.linalg.norm(Yb)
    assert e8_fg < e8_pt
