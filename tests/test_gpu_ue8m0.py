"""GPU parity of the power-of-two (UE8M0) scale study: the quantizers and the
GEMM on the tensor core's block-scaled MMA (tcgen05.mma kind::mxf8f6f4)
against the oracle's power-of-two mode.

Not the pages' method: the pages fix s = amax/448 ("FP8 Mixed Precision:
DeepSeek-V3 Training Architecture", section 1, eq. s_W); this mode rounds that
scale up to a power of two on the same tiles so the tensor core can apply it.
Quantized bytes and scales are compared bit for bit, GEMM outputs with the
GEMM tolerance of every other GEMM test.
"""
import numpy as np
import pytest

import oracle
import workloads as W
from common import check_gemm, load_fp8q, to_dev_bf16, to_dev_u8

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fp8q():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return load_fp8q()


def atoms_from_scales(sf_rows_kb: np.ndarray) -> np.ndarray:
    """Scale-atom words [K/128][ceil(R/128)][128] from power-of-two scales
    [R][K/128] (rows past R padded with the word of 1.0), by the layout's
    definition: row r = 128 rb + r0 + 32 r1 -> word 4 r0 + r1, its UE8M0 byte
    (2^(b-127)) in all four bytes."""
    R, KB = sf_rows_kb.shape
    RB = (R + 127) // 128
    out = np.full((KB, RB, 128), 0x7F7F7F7F, np.uint32)
    for r in range(R):
        for kb in range(KB):
            b = oracle.ue8m0_encode(float(sf_rows_kb[r, kb]))
            assert 0 <= b <= 254
            out[kb, r // 128, 4 * (r % 32) + (r % 128) // 32] = b * 0x01010101
    return out


def scales_from_atoms(words: np.ndarray, R: int) -> np.ndarray:
    """Inverse of atoms_from_scales for the first R rows; checks the four bytes agree."""
    KB = words.shape[0]
    w = words.astype(np.uint32)
    out = np.empty((R, KB), np.float32)
    for r in range(R):
        word = w[:, r // 128, 4 * (r % 32) + (r % 128) // 32]
        b = word & 0xFF
        assert np.all(word == b * 0x01010101)
        out[r] = np.ldexp(np.float32(1.0), b.astype(np.int64) - 127).astype(np.float32)
    return out


@pytest.mark.parametrize("M,K", [(1, 128), (100, 256), (256, 512), (300, 384)])
def test_act_quantizer_bit_exact(fp8q, M, K):
    x = W.activations_with_outliers(M, K, seed=M + K, channel_frac=2 / K, elem_frac=1e-2)
    q, sf = fp8q.quant_act_1x128_ue8m0(to_dev_bf16(x))
    oq, osf = oracle.quant_act_1x128_pow2(x)
    assert np.array_equal(q.cpu().numpy(), oq)
    words = sf.cpu().numpy().view(np.uint32)
    assert np.array_equal(words, atoms_from_scales(osf))
    assert fp8q.fp8q_device_status() == 0


def test_weight_quantizer_bit_exact(fp8q):
    w = W.weights(384, 512, seed=9)
    q, sf = fp8q.quant_w_128x128_ue8m0(to_dev_bf16(w))
    oq, osf = oracle.quant_w_128x128_pow2(w)
    assert np.array_equal(q.cpu().numpy(), oq)
    per_row = np.repeat(osf, 128, axis=0)                  # each row carries its block's scale
    assert np.array_equal(sf.cpu().numpy().view(np.uint32), atoms_from_scales(per_row))


def _run(fp8q, qa, sa, qb, sb):
    """sa [M][K/128], sb [N/K/128] per row: power-of-two scales from the oracle."""
    import torch
    M, N = qa.shape[0], qb.shape[0]
    sfa = torch.from_numpy(atoms_from_scales(sa).view(np.int32)).cuda()
    sfb = torch.from_numpy(atoms_from_scales(sb).view(np.int32)).cuda()
    d = torch.full((M + 1, N), -3.0, dtype=torch.bfloat16, device="cuda")
    fp8q.fp8q_gemm_mxf8_ue8m0(to_dev_u8(qa), sfa, to_dev_u8(qb), sfb, d[:M])
    torch.cuda.synchronize()
    assert fp8q.fp8q_device_status() == 0
    out = d.float().cpu().numpy().astype(np.float64)
    assert np.all(out[M] == -3.0)                          # nothing written past the output
    return out[:M]


@pytest.mark.parametrize("M,N,K", [
    (256, 256, 256),      # two m-tiles, one n-tile, two chunks
    (1, 256, 128),        # one row
    (300, 512, 640),      # ragged M, two n-tiles, five chunks
    (128, 768, 1024),
])
def test_gemm_against_oracle(fp8q, M, N, K):
    x = W.activations_with_outliers(M, K, seed=M * 7 + K, channel_frac=1 / K, elem_frac=1e-3)
    w = W.weights(N, K, seed=N + K)
    qa, sa = oracle.quant_act_1x128_pow2(x)
    qb, sb = oracle.quant_w_128x128_pow2(w)
    d = _run(fp8q, qa, sa, qb, np.repeat(sb, 128, axis=0))
    ref = oracle.gemm_sampled(qa, sa, qb, sb, oracle.SFB_BLOCK128)
    check_gemm(d, ref, oracle.round_bf16(ref))


def test_gemm_distinct_scales_per_row_and_chunk(fp8q):
    """Scales that differ by row, column and K chunk (powers of two 2^-3 ..
    2^3) on the codes 0, +-0.5, +-1, +-2, so a scale taken from the wrong row,
    column or chunk changes the result.  Every product is a multiple of 2^-7
    and every sum stays below 2^17, so an FP32 accumulation is exact and the
    BF16 result must equal the oracle's rounded value bit for bit."""
    rng = np.random.default_rng(1)
    M, N, K = 256, 512, 512
    qa = rng.choice(np.array([0x38, 0xB8, 0x40, 0x00, 0x30], np.uint8), size=(M, K))   # 1, -1, 2, 0, 0.5
    qb = rng.choice(np.array([0x38, 0xB8, 0x40, 0x00], np.uint8), size=(N, K))
    sa = np.ldexp(np.float32(1.0), rng.integers(-3, 4, (M, K // 128))).astype(np.float32)
    sb_rows = np.ldexp(np.float32(1.0), rng.integers(-3, 4, (N, K // 128))).astype(np.float32)
    d = _run(fp8q, qa, sa, qb, sb_rows)
    ref = oracle.gemm_sampled(qa, sa, qb, sb_rows, oracle.SFB_ROW)
    assert np.abs(ref).max() < 2.0 ** 17
    check_gemm(d, ref, oracle.round_bf16(ref))
    assert np.array_equal(d, oracle.round_bf16(ref))


def test_full_size_forward_shape(fp8q):
    """The Fprop shape (8192 x 7168 activations, 18432 x 7168 weights), both
    quantized on the device, checked on sampled full rows and columns."""
    import torch
    x = W.activations_with_outliers(8192, 7168, seed=0)
    w = W.weights(18432, 7168, seed=0)
    qa, sfa = fp8q.quant_act_1x128_ue8m0(to_dev_bf16(x))
    qb, sfb = fp8q.quant_w_128x128_ue8m0(to_dev_bf16(w))
    d = torch.empty((8192, 18432), dtype=torch.bfloat16, device="cuda")
    fp8q.fp8q_gemm_mxf8_ue8m0(qa, sfa, qb, sfb, d)
    torch.cuda.synchronize()
    assert fp8q.fp8q_device_status() == 0
    oqa, osa = oracle.quant_act_1x128_pow2(x)
    oqb, osb = oracle.quant_w_128x128_pow2(w)
    assert np.array_equal(qa.cpu().numpy(), oqa) and np.array_equal(qb.cpu().numpy(), oqb)
    rng = np.random.default_rng(2)
    rows = np.unique(np.concatenate([[0, 8191], rng.choice(8192, 14, replace=False)])).astype(np.int64)
    cols = np.unique(np.concatenate([[0, 18431], rng.choice(18432, 14, replace=False)])).astype(np.int64)
    ref_r = oracle.gemm_sampled(oqa, osa, oqb, osb, oracle.SFB_BLOCK128, rows=rows)
    got_r = d[torch.from_numpy(rows).cuda()].float().cpu().numpy().astype(np.float64)
    check_gemm(got_r, ref_r, oracle.round_bf16(ref_r))
    ref_c = oracle.gemm_sampled(oqa, osa, oqb, osb, oracle.SFB_BLOCK128, cols=cols)
    got_c = d[:, torch.from_numpy(cols).cuda()].float().cpu().numpy().astype(np.float64)
    check_gemm(got_c, ref_c, oracle.round_bf16(ref_c), row_max=np.abs(ref_c).max(axis=1))
