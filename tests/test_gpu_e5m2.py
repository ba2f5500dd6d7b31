"""GPU parity of the E5M2 gradient variant against the oracle ("FP8 Mixed
Precision: DeepSeek-V3 Training Architecture", "2. Universal E4M3";
"Introduction to LLM Quantization", "E4M3 vs E5M2"): the E5M2 1x128 and 128x1
quantizers bit for bit, and the block-scaled GEMM with E5M2 operands (Dgrad
dY x W^T, Wgrad dY^T x X^T, and the B operand in E5M2) within the GEMM
tolerance of tests/common.py, on both dense kernels.
"""
import numpy as np
import pytest

import oracle
import workloads as W
from common import check_gemm, load_fp8q, to_dev_bf16, to_dev_f32, to_dev_u8

pytestmark = pytest.mark.gpu

BLK, ROW = 0, 1
E4, E5 = 0, 1


@pytest.fixture(scope="module")
def fp8q():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return load_fp8q()


@pytest.fixture(params=["single", "pair"])
def dense_kernel(request, fp8q):
    """Run a test on the one-CTA kernel and on the CTA-pair kernel."""
    fp8q.fp8q_debug_force_dense_kernel(fp8q.FP8Q_DENSE_SINGLE if request.param == "single" else fp8q.FP8Q_DENSE_PAIR)
    yield request.param
    fp8q.fp8q_debug_force_dense_kernel(fp8q.FP8Q_DENSE_AUTO)


def _q1(fp8q, x):
    import torch
    M, K = x.shape
    ld = (M + 3) // 4 * 4 + 4
    xd = to_dev_bf16(np.pad(x, ((0, 0), (0, 8))))[:, :K]
    qbuf = torch.full((M + 1, K + 16), 0x5A, dtype=torch.uint8, device="cuda")
    sf = torch.full((K // 128, ld), -1.0, dtype=torch.float32, device="cuda")
    fp8q.fp8q_quant_act_1x128_e5m2(xd, qbuf[:M, :K], sf)
    torch.cuda.synchronize()
    assert fp8q.fp8q_device_status() == 0
    q = qbuf.cpu().numpy()
    assert np.all(q[M] == 0x5A) and np.all(q[:, K:] == 0x5A)
    s = sf.cpu().numpy()
    assert np.all(s[:, M:] == -1.0)
    return q[:M, :K], s[:, :M].T


def _q2(fp8q, x):
    import torch
    T, C = x.shape
    ld = (C + 3) // 4 * 4 + 4
    xd = to_dev_bf16(np.pad(x, ((0, 0), (0, 8))))[:, :C]
    qtbuf = torch.full((C + 1, T + 16), 0x5A, dtype=torch.uint8, device="cuda")
    sf = torch.full((T // 128, ld), -1.0, dtype=torch.float32, device="cuda")
    fp8q.fp8q_quant_act_128x1_e5m2(xd, qtbuf[:C, :T], sf)
    torch.cuda.synchronize()
    assert fp8q.fp8q_device_status() == 0
    qt = qtbuf.cpu().numpy()
    assert np.all(qt[C] == 0x5A) and np.all(qt[:, T:] == 0x5A)
    s = sf.cpu().numpy()
    assert np.all(s[:, C:] == -1.0)
    return qt[:C, :T], s[:, :C]


@pytest.mark.parametrize("M,K", [(1, 128), (65, 384), (200, 1024)])
def test_e5m2_1x128_matches_oracle(fp8q, M, K):
    x = W.grad_with_outlier_tokens(M, K, seed=M + K)
    x[0, :4] = [0x0000, 0x8000, 0x0001, 0x8001]           # signed zeros, BF16 subnormals
    oq, osf = oracle.quant_act_1x128_e5m2(x)
    q, sf = _q1(fp8q, x)
    assert np.array_equal(q, oq)
    assert np.array_equal(sf.view(np.uint32), osf.view(np.uint32))


@pytest.mark.parametrize("T,C", [(128, 8), (256, 200), (384, 1024)])
def test_e5m2_128x1_matches_oracle(fp8q, T, C):
    x = W.grad_with_outlier_tokens(T, C, seed=T + C)
    oqt, osf = oracle.quant_act_128x1_e5m2(x)
    qt, sf = _q2(fp8q, x)
    assert np.array_equal(qt, oqt)
    assert np.array_equal(sf.view(np.uint32), osf.view(np.uint32))


def test_e5m2_quantizers_full_size(fp8q):
    """dY 8192 x 18432 in E5M2, 1x128 (Dgrad) and 128x1 transposed (Wgrad), every tile."""
    dy = W.grad_with_outlier_tokens(8192, 18432, seed=0)
    oq, osf = oracle.quant_act_1x128_e5m2(dy)
    q, sf = _q1(fp8q, dy)
    assert np.array_equal(sf.view(np.uint32), osf.view(np.uint32)) and np.array_equal(q, oq)
    del oq, q
    oqt, osft = oracle.quant_act_128x1_e5m2(dy)
    qt, sft = _q2(fp8q, dy)
    assert np.array_equal(sft.view(np.uint32), osft.view(np.uint32)) and np.array_equal(qt, oqt)


def _kmajor(sf_mk):
    M, KB = sf_mk.shape
    buf = np.full((KB, (M + 3) // 4 * 4), np.nan, np.float32)
    buf[:, :M] = sf_mk.T
    return to_dev_f32(buf)


def _blk(sfb):
    NB, KB = sfb.shape
    buf = np.full((NB, (KB + 3) // 4 * 4), np.nan, np.float32)
    buf[:, :KB] = sfb
    return to_dev_f32(buf)[:, :KB]


def _gemm(fp8q, qa, a_fmt, sa, qb, b_fmt, sb, mode, f32):
    import torch
    M, K = qa.shape
    N = qb.shape[0]
    a, b = to_dev_u8(qa), to_dev_u8(qb)
    sbd = _blk(sb) if mode == BLK else _kmajor(sb)
    dbuf = torch.full((M + 2, N + 8), -3.0, dtype=torch.float32 if f32 else torch.bfloat16, device="cuda")
    d = dbuf[1:M + 1, :N]
    fp8q.fp8q_gemm_blockscaled_fmt(a, a_fmt, _kmajor(sa), b, b_fmt, sbd, mode, d)
    torch.cuda.synchronize()
    assert fp8q.fp8q_device_status() == 0
    full = dbuf.float().cpu().numpy().astype(np.float64)
    assert np.all(full[0] == -3.0) and np.all(full[-1] == -3.0) and np.all(full[1:-1, N:] == -3.0)
    return full[1:-1, :N]


def _rounded(ref, f32):
    return oracle.round_f32(ref) if f32 else oracle.round_bf16(ref)


@pytest.mark.parametrize("M,N,K", [(1, 256, 128), (300, 384, 640), (1000, 1280, 768)])
def test_e5m2_dgrad_matches_oracle(fp8q, dense_kernel, M, N, K):
    """dY (E5M2, 1x128) x W^T (E4M3, 128x128 blocks), BF16 out."""
    qa, sa = oracle.quant_act_1x128_e5m2(W.grad_with_outlier_tokens(M, K, seed=M))
    qb, sb = oracle.quant_w_128x128(W.weights(N, K, seed=N))
    ref = oracle.gemm_sampled(qa, sa, qb, sb, BLK, a_fmt=E5)
    check_gemm(_gemm(fp8q, qa, E5, sa, qb, E4, sb, BLK, False), ref, _rounded(ref, False))


@pytest.mark.parametrize("M,N,K", [(257, 512, 1024), (129, 128, 384)])
def test_e5m2_wgrad_matches_oracle(fp8q, dense_kernel, M, N, K):
    """dY^T (E5M2, 128x1) x X^T (E4M3, 128x1), FP32 out: both operands carry per-row scales."""
    dyt, sdy = oracle.quant_act_128x1_e5m2(W.grad_with_outlier_tokens(K, M, seed=K))
    xt, sx = oracle.quant_act_128x1(W.activations_with_outliers(K, N, seed=N, channel_frac=2 / N, elem_frac=1e-3))
    sa, sb = np.ascontiguousarray(sdy.T), np.ascontiguousarray(sx.T)
    ref = oracle.gemm_sampled(dyt, sa, xt, sb, ROW, a_fmt=E5)
    check_gemm(_gemm(fp8q, dyt, E5, sa, xt, E4, sb, ROW, True), ref, _rounded(ref, True))


def test_e5m2_b_operand(fp8q, dense_kernel):
    """The B operand in E5M2 (A in E4M3), and both in E5M2: the two format fields."""
    M, N, K = 200, 256, 512
    qa4, sa4 = oracle.quant_act_1x128(W.activations_with_outliers(M, K, seed=1, elem_frac=1e-3))
    qa5, sa5 = oracle.quant_act_1x128_e5m2(W.grad_with_outlier_tokens(M, K, seed=2))
    qb5, sb5 = oracle.quant_act_1x128_e5m2(W.grad_with_outlier_tokens(N, K, seed=3))
    for qa, a_fmt, sa in ((qa4, E4, sa4), (qa5, E5, sa5)):
        ref = oracle.gemm_sampled(qa, sa, qb5, sb5, ROW, a_fmt=a_fmt, b_fmt=E5)
        check_gemm(_gemm(fp8q, qa, a_fmt, sa, qb5, E5, sb5, ROW, True), ref, _rounded(ref, True))
