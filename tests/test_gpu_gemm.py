"""GPU parity of the block-scaled FP8 GEMM against the oracle's FP64 result.

Passages: "FP8 Mixed Precision: DeepSeek-V3 Training Architecture", section 3
"Decoupled Accumulation in Tensor Core GEMMs" (eq. C_ij per 128-wide K chunk);
"Introduction to LLM Quantization", "1. Mixed Precision Quantization"
(y = Wx walk-through: x 128x1, W 256x128, FP32 accumulate, BF16 out) and
"3) Backward propagation" (Dgrad, Wgrad).  Tolerance: see tests/common.py.
"""
import numpy as np
import pytest

import oracle
import workloads as W
from common import check_gemm, load_fp8q, to_dev_bf16, to_dev_f32, to_dev_u8

pytestmark = pytest.mark.gpu

BLK, ROW = 0, 1


@pytest.fixture(scope="module")
def fp8q():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return load_fp8q()


def sfa_dev(sf_mk, ld=None):
    """oracle scales [M][K/128] -> device [K/128][ld >= M] (K-chunk-major)."""
    M, KB = sf_mk.shape
    ld = ld or (M + 3) // 4 * 4
    buf = np.full((KB, ld), np.nan, np.float32)
    buf[:, :M] = sf_mk.T
    return to_dev_f32(buf)


def sfb_dev(sfb, pad=True):
    """Block scales [N/128][K/128] on the device; with pad, the row stride is
    rounded up to 4 floats (the layout the CTA-pair kernel loads with TMA)."""
    NB, KB = sfb.shape
    ld = (KB + 3) // 4 * 4 if pad else KB
    buf = np.full((NB, ld), np.nan, np.float32)
    buf[:, :KB] = sfb
    return to_dev_f32(buf)[:, :KB]


def run_gemm(fp8q, qa, sfa, qb, sfb, mode, out_f32=False, lda=None, ldb=None, ldd=None, pad_sfb=True):
    """qa [M][K], sfa [M][K/128]; qb [N][K]; sfb [N/128][K/128] (BLK) or [N][K/128] (ROW)."""
    import torch
    M, K = qa.shape
    N = qb.shape[0]
    lda = lda or K
    ldb = ldb or K
    ldd = ldd or N
    abuf = np.zeros((M, lda), np.uint8); abuf[:, :K] = qa
    bbuf = np.zeros((N, ldb), np.uint8); bbuf[:, :K] = qb
    a = to_dev_u8(abuf)[:, :K]
    b = to_dev_u8(bbuf)[:, :K]
    sa = sfa_dev(sfa)
    sb = sfb_dev(sfb, pad_sfb) if mode == BLK else sfa_dev(sfb)
    dt = torch.float32 if out_f32 else torch.bfloat16
    dbuf = torch.full((M + 2, ldd), -3.0, dtype=dt, device="cuda")
    d = dbuf[1:M + 1, :N]
    fp8q.fp8q_gemm_blockscaled(a, sa, b, sb, mode, d)
    torch.cuda.synchronize()
    assert fp8q.fp8q_device_status() == 0
    full = dbuf.float().cpu().numpy().astype(np.float64)
    assert np.all(full[0] == -3.0) and np.all(full[-1] == -3.0) and np.all(full[1:-1, N:] == -3.0)
    return full[1:-1, :N]


def rounded(ref, out_f32):
    return oracle.round_f32(ref) if out_f32 else oracle.round_bf16(ref)


def test_linear_y_wx_worked_example(fp8q):
    """x 1x128 ~N(0,1) with element 17 = 20.0, W 256x128 ~N(0,0.02): two weight
    blocks, one activation tile, FP32 accumulate, BF16 out."""
    import torch
    x, w = W.linear_1x128_inputs(seed=0)
    qx, sx = oracle.quant_act_1x128(x)
    qw, sw = oracle.quant_w_128x128(w)
    assert sw.shape == (2, 1) and sx.shape == (1, 1)
    ref = oracle.gemm_sampled(qx, sx, qw, sw, BLK)
    d = run_gemm(fp8q, qx, sx, qw, sw, BLK)
    check_gemm(d, ref, rounded(ref, False))
    # the same through the device quantizers (bit-exact, so identical GEMM inputs)
    xd, wd = to_dev_bf16(x), to_dev_bf16(w)
    q1, s1 = fp8q.quant_act_1x128(xd)
    q2, s2 = fp8q.quant_w_128x128(wd)
    y = torch.empty((1, 256), dtype=torch.bfloat16, device="cuda")
    fp8q.fp8q_gemm_blockscaled(q1, s1, q2, s2, BLK, y)
    assert np.array_equal(q1.cpu().numpy(), qx) and np.array_equal(q2.cpu().numpy(), qw)
    check_gemm(y.float().cpu().numpy(), ref, rounded(ref, False))


@pytest.fixture(params=["single", "pair"])
def dense_kernel(request, fp8q):
    """Run a test on the one-CTA kernel and on the CTA-pair kernel."""
    fp8q.fp8q_debug_force_dense_kernel(fp8q.FP8Q_DENSE_SINGLE if request.param == "single" else fp8q.FP8Q_DENSE_PAIR)
    yield request.param
    fp8q.fp8q_debug_force_dense_kernel(fp8q.FP8Q_DENSE_AUTO)


@pytest.mark.parametrize("M,N,K,mode,f32", [
    (1, 256, 128, BLK, False),       # one row (a pair tile with 255 empty rows)
    (128, 256, 128, BLK, False),     # one tile, one chunk
    (300, 384, 640, BLK, False),     # ragged M, half N tile, 5 chunks
    (300, 384, 640, BLK, True),
    (257, 512, 1024, ROW, True),     # Wgrad scale mode
    (129, 128, 384, ROW, False),
    (1000, 1280, 768, BLK, False),   # several tiles per CTA pass
    (2048, 2560, 512, ROW, True),    # more pair tiles than co-resident pairs
])
def test_gemm_parity_small(fp8q, dense_kernel, M, N, K, mode, f32):
    x = W.activations_with_outliers(M, K, seed=M, channel_frac=2 / K, elem_frac=1e-3)
    qa, sa = oracle.quant_act_1x128(x)
    if mode == BLK:
        qb, sb = oracle.quant_w_128x128(W.weights(N, K, seed=N))
    else:
        qb, sb = oracle.quant_act_1x128(W.activations_with_outliers(N, K, seed=N + 1, channel_frac=0, elem_frac=1e-3))
    ref = oracle.gemm_sampled(qa, sa, qb, sb, mode)
    d = run_gemm(fp8q, qa, sa, qb, sb, mode, f32, lda=K + 16, ldb=K + 32, ldd=N + 8)
    check_gemm(d, ref, rounded(ref, f32))


def test_gemm_unaligned_scale_layout(fp8q, dense_kernel):
    """Block scales with a row stride of K/128 = 5 floats: the CTA-pair kernel
    cannot TMA-load them, so even when forced the one-CTA kernel runs."""
    M, N, K = 300, 384, 640
    qa, sa = oracle.quant_act_1x128(W.activations_with_outliers(M, K, seed=7, channel_frac=2 / K, elem_frac=1e-3))
    qb, sb = oracle.quant_w_128x128(W.weights(N, K, seed=8))
    ref = oracle.gemm_sampled(qa, sa, qb, sb, BLK)
    d = run_gemm(fp8q, qa, sa, qb, sb, BLK, pad_sfb=False)
    check_gemm(d, ref, rounded(ref, False))


def test_gemm_integer_exact(fp8q, dense_kernel):
    """Small-integer codes with power-of-two scales: every partial sum is exact
    in FP32, so the device result must equal the oracle exactly."""
    rng = np.random.default_rng(1)
    codes = np.array([0x00, 0x38, 0x40, 0x44, 0x48, 0xB8, 0xC0, 0xC4, 0xC8], np.uint8)
    M, N, K = 200, 256, 512
    qa = codes[rng.integers(0, 9, (M, K))]
    qb = codes[rng.integers(0, 9, (N, K))]
    sa = np.exp2(rng.integers(-3, 3, (M, K // 128))).astype(np.float32)
    sb = np.exp2(rng.integers(-3, 3, (N // 128, K // 128))).astype(np.float32)
    ref = oracle.gemm_sampled(qa, sa, qb, sb, BLK)
    d = run_gemm(fp8q, qa, sa, qb, sb, BLK, out_f32=True)
    assert np.array_equal(d, ref)


def test_gemm_one_hot_rows(fp8q, dense_kernel):
    N, K = 256, 256
    qb, sb = oracle.quant_w_128x128(W.weights(N, K, seed=5))
    qa = np.zeros((3, K), np.uint8)
    qa[0, 0] = 0x38
    qa[1, 255] = 0x38
    qa[2, 129] = 0xC0      # -2
    sa = np.ones((3, 2), np.float32)
    d = run_gemm(fp8q, qa, sa, qb, sb, BLK, out_f32=True)
    ref = oracle.gemm_sampled(qa, sa, qb, sb, BLK)
    assert np.array_equal(d, oracle.round_f32(ref))


def _sample(n, k, rng, must=()):
    idx = np.unique(np.concatenate([np.asarray(must, np.int64), rng.choice(n, size=min(k, n), replace=False)]))
    return idx.astype(np.int64)


def _full_size_check(fp8q, qa, sa, qb, sb, mode, out_f32, seed):
    """Run the full GEMM on the device; compare sampled full rows and full columns with the oracle."""
    import torch
    M, K = qa.shape
    N = qb.shape[0]
    a, b = to_dev_u8(qa), to_dev_u8(qb)
    sad = sfa_dev(sa)
    sbd = to_dev_f32(sb) if mode == BLK else sfa_dev(sb)
    d = torch.empty((M, N), dtype=torch.float32 if out_f32 else torch.bfloat16, device="cuda")
    fp8q.fp8q_gemm_blockscaled(a, sad, b, sbd, mode, d)
    torch.cuda.synchronize()
    assert fp8q.fp8q_device_status() == 0
    rng = np.random.default_rng(seed)
    rows = _sample(M, 24, rng, must=[0, M - 1])
    cols = _sample(N, 24, rng, must=[0, N - 1])
    all_cols = np.arange(N, dtype=np.int64)
    ref_r = oracle.gemm_sampled(qa, sa, qb, sb, mode, rows=rows, cols=all_cols)
    got_r = d[torch.from_numpy(rows).cuda()].float().cpu().numpy().astype(np.float64)
    check_gemm(got_r, ref_r, rounded(ref_r, out_f32))
    all_rows = np.arange(M, dtype=np.int64)
    ref_c = oracle.gemm_sampled(qa, sa, qb, sb, mode, rows=all_rows, cols=cols)
    got_c = d[:, torch.from_numpy(cols).cuda()].float().cpu().numpy().astype(np.float64)
    # the elementwise bound uses each row's max over all N (from the sampled-row pass where known)
    check_gemm(got_c, ref_c, rounded(ref_c, out_f32), row_max=np.abs(ref_c).max(axis=1))


def test_forward_gemm_full_size(fp8q):
    """A 8192x7168 (1x128 tiles of the outlier activations) x B 18432x7168
    (128x128 blocks of N(0,0.02)) -> C 8192x18432 BF16."""
    x = W.activations_with_outliers(8192, 7168, seed=0)
    qa, sa = oracle.quant_act_1x128(x)
    qb, sb = oracle.quant_w_128x128(W.weights(18432, 7168, seed=0))
    _full_size_check(fp8q, qa, sa, qb, sb, BLK, False, seed=3)


@pytest.mark.slow
def test_forward_gemm_full_output(fp8q):
    """Every output of the full-size Fprop (8192 x 18432 = 151 M values) against
    the FP64 oracle, once, in blocks of 512 full rows: about 1.1e12 multiply-adds
    of oracle work, a minute or two on the host cores."""
    import torch
    x = W.activations_with_outliers(8192, 7168, seed=0)
    qa, sa = oracle.quant_act_1x128(x)
    qb, sb = oracle.quant_w_128x128(W.weights(18432, 7168, seed=0))
    M, N = qa.shape[0], qb.shape[0]
    d = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    fp8q.fp8q_gemm_blockscaled(to_dev_u8(qa), sfa_dev(sa), to_dev_u8(qb), to_dev_f32(sb), BLK, d)
    torch.cuda.synchronize()
    assert fp8q.fp8q_device_status() == 0
    got = d.float().cpu().numpy()
    del d
    num = den = 0.0
    for r0 in range(0, M, 512):
        rows = np.arange(r0, min(M, r0 + 512), dtype=np.int64)
        ref = oracle.gemm_sampled(qa, sa, qb, sb, BLK, rows=rows)
        blk = got[r0:r0 + len(rows)].astype(np.float64)
        check_gemm(blk, ref, rounded(ref, False))
        num += float(np.sum((blk - ref) ** 2))
        den += float(np.sum(ref ** 2))
    assert np.sqrt(num / den) <= 2e-3


def test_backward_gemms_full_size(fp8q):
    """Dgrad: dY 8192x18432 (1x128) x W^T (W 18432x7168, 128x128 blocks, K = 18432).
    Wgrad: dY^T x X with both operands in 128x1 tiles along tokens (K = 8192), FP32 out."""
    dy = W.grad_with_outlier_tokens(8192, 18432, seed=0)
    w = W.weights(18432, 7168, seed=0)
    qdy, sdy = oracle.quant_act_1x128(dy)
    qw, sw = oracle.quant_w_128x128(np.ascontiguousarray(w.T))       # W^T blocks = transposed W blocks
    _full_size_check(fp8q, qdy, sdy, qw, sw, BLK, False, seed=4)
    del qdy, sdy, qw, sw
    x = W.activations_with_outliers(8192, 7168, seed=0)
    qdyt, sdyt = oracle.quant_act_128x1(dy)          # [18432][8192], [64][18432]
    qxt, sxt = oracle.quant_act_128x1(x)             # [7168][8192],  [64][7168]
    _full_size_check(fp8q, qdyt, np.ascontiguousarray(sdyt.T), qxt, np.ascontiguousarray(sxt.T), ROW, True, seed=5)
