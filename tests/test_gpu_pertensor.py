"""GPU parity of the per-tensor FP8 baseline against the oracle: the quantizer
bit for bit (codes, amax, scale) and the GEMM within the GEMM tolerance of
tests/common.py.  The per-tensor GEMM accumulates the whole K reduction in the
tensor cores' accumulator, so one case checks that this accumulation keeps
FP32 precision over a long K: the pages' Hopper figure (about 14 bits kept in
the tensor-core accumulator) is the reason the fine-grained GEMM promotes
every 128-wide chunk ("Introduction to LLM Quantization", "3. Increasing
accumulation Quantization"; "FP8 Mixed Precision: DeepSeek-V3 Training
Architecture", section 3).
"""
import numpy as np
import pytest

import oracle
import workloads as W
from common import check_gemm, load_fp8q, to_dev_bf16, to_dev_f32, to_dev_u8

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fp8q():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return load_fp8q()


def _quant(fp8q, x):
    import torch
    M, K = x.shape
    xd = to_dev_bf16(np.pad(x, ((0, 0), (0, 8))))[:, :K]
    qbuf = torch.full((M + 1, K + 16), 0x5A, dtype=torch.uint8, device="cuda")
    amax_scale = torch.full((3,), -1.0, dtype=torch.float32, device="cuda")
    fp8q.fp8q_quant_pertensor(xd, qbuf[:M, :K], amax_scale)
    torch.cuda.synchronize()
    assert fp8q.fp8q_device_status() == 0
    q = qbuf.cpu().numpy()
    assert np.all(q[M] == 0x5A) and np.all(q[:, K:] == 0x5A)
    a = amax_scale.cpu().numpy()
    assert a[2] == -1.0
    return q[:M, :K], a[0], a[1]


@pytest.mark.parametrize("M,K", [(1, 128), (1, 8), (70, 384), (130, 1000), (513, 7168)])
def test_pertensor_quantizer_matches_oracle(fp8q, M, K):
    x = W.activations_with_outliers(M, K, seed=M + K, channel_frac=2 / max(K, 128), elem_frac=1e-3)
    oq, oamax, os_ = oracle.quant_pertensor(x)
    q, amax, s = _quant(fp8q, x)
    assert np.array_equal(q, oq)
    assert np.float32(amax) == np.float32(oamax) and np.float32(s) == np.float32(os_)


def test_pertensor_quantizer_zero_and_empty(fp8q):
    import torch
    q, amax, s = _quant(fp8q, np.zeros((3, 256), np.uint16))
    assert amax == 0.0 and np.float32(s) == np.float32(1e-12) and np.all(q == 0)
    amax_scale = torch.full((2,), -1.0, dtype=torch.float32, device="cuda")
    x = torch.empty((0, 128), dtype=torch.bfloat16, device="cuda")
    fp8q.fp8q_quant_pertensor(x, torch.empty((0, 128), dtype=torch.uint8, device="cuda"), amax_scale)
    torch.cuda.synchronize()
    a = amax_scale.cpu().numpy()
    assert a[0] == 0.0 and np.float32(a[1]) == np.float32(1e-12)


def _run_gemm(fp8q, qa, sa, qb, sb, out_f32):
    import torch
    M, K = qa.shape
    N = qb.shape[0]
    a, b = to_dev_u8(qa), to_dev_u8(qb)
    scales = to_dev_f32(np.array([sa, sb], np.float32))
    dt = torch.float32 if out_f32 else torch.bfloat16
    dbuf = torch.full((M + 2, N + 8), -3.0, dtype=dt, device="cuda")
    d = dbuf[1:M + 1, :N]
    fp8q.fp8q_gemm_pertensor(a, scales[0:1], b, scales[1:2], d)
    torch.cuda.synchronize()
    assert fp8q.fp8q_device_status() == 0
    full = dbuf.float().cpu().numpy().astype(np.float64)
    assert np.all(full[0] == -3.0) and np.all(full[-1] == -3.0) and np.all(full[1:-1, N:] == -3.0)
    return full[1:-1, :N]


def _rounded(ref, out_f32):
    return oracle.round_f32(ref) if out_f32 else oracle.round_bf16(ref)


@pytest.mark.parametrize("M,N,K,f32", [
    (1, 128, 128, False), (200, 256, 384, False), (300, 512, 1024, True), (257, 384, 2048, False),
    (513, 256, 4096, True),
])
def test_pertensor_gemm_matches_oracle(fp8q, M, N, K, f32):
    qa, _, sa = oracle.quant_pertensor(W.activations_with_outliers(M, K, seed=M, elem_frac=1e-3))
    qb, _, sb = oracle.quant_pertensor(W.weights(N, K, seed=N))
    d = _run_gemm(fp8q, qa, sa, qb, sb, f32)
    ref = oracle.gemm_pertensor_sampled(qa, sa, qb, sb)
    check_gemm(d, ref, _rounded(ref, f32))


def test_pertensor_accumulator_keeps_fp32_over_long_k(fp8q):
    """Row 0: the product 128 x 128 = 2^14 first, then 18430 products 1 x 1
    and one 1 x 128.  The exact sum, 34942, needs 16 significant bits; every
    partial sum is an integer below 2^24, so an FP32 accumulator gets it
    exactly in any order, while a 14-bit one would drop unit terms.  Row 1:
    the same terms with the large product last."""
    K = 18432
    one, big = 0x38, 0x70          # E4M3 codes of 1.0 and 128.0
    qa = np.full((2, K), one, np.uint8)
    qa[0, 0] = big
    qa[1, K - 1] = big
    qb = np.full((128, K), one, np.uint8)
    qb[:, 0] = big
    qb[:, K - 1] = big
    d = _run_gemm(fp8q, qa, 1.0, qb, 1.0, True)
    ref = oracle.gemm_pertensor_sampled(qa, 1.0, qb, 1.0)
    assert ref[0, 0] == 2.0 ** 14 + 2.0 ** 7 + (K - 2) and np.all(ref == ref[0, 0])
    assert np.array_equal(d, ref), (d[:, :4], ref[0, 0])


def test_pertensor_accumulator_keeps_24_bits(fp8q):
    """Row 0: 128 products 256 x 256 = 2^16 (together 2^23) first, then
    18176 products 1 x 1 and 128 products 1 x 256.  The exact sum, 2^23 +
    2^15 + 18176, needs 24 significant bits and every partial sum is an
    integer below 2^24, so only a full FP32 accumulator returns it exactly.
    Row 1 puts the large products last."""
    K = 18432
    one, big = 0x38, 0x78          # E4M3 codes of 1.0 and 256.0
    qa = np.full((2, K), one, np.uint8)
    qa[0, :128] = big
    qa[1, K - 128:] = big
    qb = np.full((128, K), one, np.uint8)
    qb[:, :128] = big
    qb[:, K - 128:] = big
    d = _run_gemm(fp8q, qa, 1.0, qb, 1.0, True)
    ref = oracle.gemm_pertensor_sampled(qa, 1.0, qb, 1.0)
    assert ref[0, 0] == 2.0 ** 23 + 128 * 256 + (K - 256) and np.all(ref == ref[0, 0])
    assert np.array_equal(d, ref), (d[:, :4], ref[0, 0])


def test_pertensor_gemm_full_size_sampled(fp8q):
    """The Fprop shape, 8192 x 18432 x 7168, per-tensor operands; sampled full rows and columns."""
    import torch
    M, N, K = 8192, 18432, 7168
    qa, _, sa = oracle.quant_pertensor(W.activations_with_outliers(M, K, seed=0))
    qb, _, sb = oracle.quant_pertensor(W.weights(N, K, seed=0))
    a, b = to_dev_u8(qa), to_dev_u8(qb)
    scales = to_dev_f32(np.array([sa, sb], np.float32))
    d = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    fp8q.fp8q_gemm_pertensor(a, scales[0:1], b, scales[1:2], d)
    torch.cuda.synchronize()
    assert fp8q.fp8q_device_status() == 0
    rng = np.random.default_rng(7)
    rows = np.unique(np.r_[0, M - 1, rng.integers(0, M, 22)]).astype(np.int64)
    cols = np.unique(np.r_[0, N - 1, rng.integers(0, N, 22)]).astype(np.int64)
    ref_r = oracle.gemm_pertensor_sampled(qa, sa, qb, sb, rows=rows)
    got_r = d[torch.from_numpy(rows).cuda()].float().cpu().numpy().astype(np.float64)
    check_gemm(got_r, ref_r, _rounded(ref_r, False))
    ref_c = oracle.gemm_pertensor_sampled(qa, sa, qb, sb, cols=cols)
    got_c = d[:, torch.from_numpy(cols).cuda()].float().cpu().numpy().astype(np.float64)
    check_gemm(got_c, ref_c, _rounded(ref_c, False), row_max=np.abs(ref_c).max(axis=1))
