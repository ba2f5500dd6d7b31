"""GPU parity of the fused calls: GEMMs whose epilogue emits the next layer's
1x128 FP8 tiles, and the 1x128 quantizer fused with the MoE dispatch gather.

Passages: "Fine-Grained FP8 Quantization in DeepSeek", section 2 (activations
are quantized online per 1x128 tile, scale = tile max / 448); "FP8 Mixed
Precision: DeepSeek-V3 Training Architecture", section 1 (activations kept in
FP8 between layers) and section 2 (MoE dispatch carries FP8 activations).

What is unique is compared bit for bit.  A fused GEMM must equal the same
GEMM with BF16 output followed by the 1x128 quantizer; the BF16 GEMM itself
is held to the oracle's FP64 result with the tolerance of tests/common.py,
and its BF16 bits are quantized by the oracle to give the expected FP8 bytes
and scales.  The gather must equal the oracle's quantization of the gathered
rows.
"""
import numpy as np
import pytest

import oracle
import workloads as W
from common import check_gemm, load_fp8q, to_dev_bf16, to_dev_f32, to_dev_u8

pytestmark = pytest.mark.gpu

BLK = 0
SENTINEL_Q = 0x5A
SENTINEL_S = -7.0


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


def _sf_kmajor(sf_mk, ld=None):
    """oracle scales [M][K/128] -> device [K/128][ld >= M], rows padded with NaN."""
    M, KB = sf_mk.shape
    ld = ld or (M + 3) // 4 * 4
    buf = np.full((KB, ld), np.nan, np.float32)
    buf[:, :M] = sf_mk.T
    return to_dev_f32(buf)


def _bf16_bits(t):
    import torch
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def _fp8_out(M, N, ld, ld_sf):
    """Output buffers with a guard row, guard columns and guard scale entries."""
    import torch
    qbuf = torch.full((M + 1, ld), SENTINEL_Q, dtype=torch.uint8, device="cuda")
    sbuf = torch.full((N // 128, ld_sf), SENTINEL_S, dtype=torch.float32, device="cuda")
    return qbuf, sbuf


def _check_fp8_out(qbuf, sbuf, M, N, q_ref, sf_ref):
    q = qbuf.cpu().numpy()
    s = sbuf.cpu().numpy()
    assert np.array_equal(q[:M, :N], q_ref)
    assert np.array_equal(s[:, :M].view(np.uint32), np.ascontiguousarray(sf_ref.T).view(np.uint32))
    assert np.all(q[M] == SENTINEL_Q) and np.all(q[:, N:] == SENTINEL_Q)
    assert np.all(s[:, M:] == SENTINEL_S)


@pytest.mark.parametrize("M,N,K", [
    (1, 256, 128),       # one row
    (130, 384, 640),     # ragged M, odd number of 128-column blocks, 5 chunks
    (300, 1280, 768),    # several tiles per CTA pass
    (2048, 2560, 512),   # more pair tiles than co-resident pairs
])
def test_gemm_q1x128_equals_quantized_bf16_gemm(fp8q, dense_kernel, M, N, K):
    import torch
    x = W.activations_with_outliers(M, K, seed=M + 11, channel_frac=2 / K, elem_frac=1e-3)
    x[M // 2] = 0                                  # an all-zero output row: scale 1e-12, codes 0
    qa, sa = oracle.quant_act_1x128(x)
    qb, sb = oracle.quant_w_128x128(W.weights(N, K, seed=N + 3))
    a, b = to_dev_u8(qa), to_dev_u8(qb)
    sad, sbd = _sf_kmajor(sa), to_dev_f32(np.pad(sb, ((0, 0), (0, (-sb.shape[1]) % 4))))[:, :K // 128]
    d = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    fp8q.fp8q_gemm_blockscaled(a, sad, b, sbd, BLK, d)
    ld_sf = (M + 3) // 4 * 4 + 4
    qbuf, sbuf = _fp8_out(M, N, N + 32, ld_sf)
    fp8q.fp8q_gemm_blockscaled_q1x128(a, sad, b, sbd, qbuf[:M, :N], sbuf)
    torch.cuda.synchronize()
    assert fp8q.fp8q_device_status() == 0
    ref = oracle.gemm_sampled(qa, sa, qb, sb, BLK)
    dbits = _bf16_bits(d)
    check_gemm(W.bf16_bits_to_f32(dbits).astype(np.float64), ref, oracle.round_bf16(ref))
    q_ref, sf_ref = oracle.quant_act_1x128(dbits)
    _check_fp8_out(qbuf, sbuf, M, N, q_ref, sf_ref)


def test_gemm_q1x128_saturating_values(fp8q, dense_kernel):
    """Large scales push the BF16 results far beyond 448: the tile scale takes
    them back to [-448, 448] and the tile maximum encodes as +-448 (0x7E/0xFE)."""
    import torch
    M, N, K = 256, 256, 256
    qa, sa = oracle.quant_act_1x128(W.activations_with_outliers(M, K, seed=5, channel_frac=0, elem_frac=0))
    qb, sb = oracle.quant_w_128x128(W.weights(N, K, seed=6))
    sa = (sa * np.float32(2.0 ** 40)).astype(np.float32)
    a, b = to_dev_u8(qa), to_dev_u8(qb)
    sad, sbd = _sf_kmajor(sa), to_dev_f32(np.pad(sb, ((0, 0), (0, 2))))[:, :2]
    d = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    fp8q.fp8q_gemm_blockscaled(a, sad, b, sbd, BLK, d)
    qbuf, sbuf = _fp8_out(M, N, N, M)
    fp8q.fp8q_gemm_blockscaled_q1x128(a, sad, b, sbd, qbuf[:M], sbuf)
    torch.cuda.synchronize()
    assert fp8q.fp8q_device_status() == 0
    dbits = _bf16_bits(d)
    assert np.abs(W.bf16_bits_to_f32(dbits)).max() > 1e6
    q_ref, sf_ref = oracle.quant_act_1x128(dbits)
    _check_fp8_out(qbuf, sbuf, M, N, q_ref, sf_ref)
    assert np.all(np.isin(q_ref.reshape(M, -1, 128), [0x7E, 0xFE]).any(axis=2))


@pytest.mark.parametrize("counts", [
    [3, 0, 1, 130, 0, 257],          # empty experts, a 1-row expert, ragged tiles
    [1] * 9,                         # many one-row experts
    [128, 128, 0, 256],              # exact tile multiples
    [17, 33, 48, 0, 96, 100, 5],     # assorted small experts
])
def test_grouped_q1x128_equals_quantized_bf16_gemm(fp8q, counts):
    import torch
    G, N, K = len(counts), 384, 512
    off = W.ragged_offsets(counts)
    Mt = int(off[-1])
    qa, sa = oracle.quant_act_1x128(W.activations_with_outliers(Mt, K, seed=Mt, channel_frac=1 / K, elem_frac=1e-3))
    wq = np.empty((G, N, K), np.uint8)
    ws = np.empty((G, N // 128, K // 128), np.float32)
    for g in range(G):
        wq[g], ws[g] = oracle.quant_w_128x128(W.weights(N, K, seed=G * 1000 + g))
    a, sad, wd, wsd = to_dev_u8(qa), _sf_kmajor(sa), to_dev_u8(wq), to_dev_f32(ws)
    offd = torch.from_numpy(off.astype(np.int32)).cuda()
    d = torch.empty((Mt, N), dtype=torch.bfloat16, device="cuda")
    fp8q.fp8q_grouped_gemm_blockscaled(a, sad, wd, wsd, offd, d)
    qbuf, sbuf = _fp8_out(Mt, N, N + 16, Mt + 8)
    fp8q.fp8q_grouped_gemm_blockscaled_q1x128(a, sad, wd, wsd, offd, qbuf[:Mt, :N], sbuf)
    torch.cuda.synchronize()
    assert fp8q.fp8q_device_status() == 0
    ref = oracle.grouped_gemm_sampled(qa, sa, wq, ws, off)
    dbits = _bf16_bits(d)
    check_gemm(W.bf16_bits_to_f32(dbits).astype(np.float64), ref, oracle.round_bf16(ref))
    q_ref, sf_ref = oracle.quant_act_1x128(dbits)
    _check_fp8_out(qbuf, sbuf, Mt, N, q_ref, sf_ref)


@pytest.mark.parametrize("M_src,M,K", [
    (5, 1, 128),          # one output row
    (40, 320, 384),       # every token repeated 8 times (top-8 dispatch), ragged row tile
    (300, 77, 1024),      # a subset, several K tiles
])
def test_gather_quant_equals_quant_of_gathered_rows(fp8q, M_src, M, K):
    import torch
    x = W.activations_with_outliers(M_src, K, seed=M_src + K, channel_frac=2 / K, elem_frac=1e-3)
    rng = np.random.default_rng(M)
    rows = rng.integers(0, M_src, M).astype(np.int32)
    rows[0] = M_src - 1
    xd = to_dev_bf16(np.pad(x, ((0, 0), (0, 8))))[:, :K]          # ldx = K + 8
    qbuf = torch.full((M + 1, K + 16), SENTINEL_Q, dtype=torch.uint8, device="cuda")
    sbuf = torch.full((K // 128, M + 4), SENTINEL_S, dtype=torch.float32, device="cuda")
    fp8q.fp8q_quant_act_1x128_gather(xd, torch.from_numpy(rows).cuda(), qbuf[:M, :K], sbuf)
    torch.cuda.synchronize()
    assert fp8q.fp8q_device_status() == 0
    q_ref, sf_ref = oracle.quant_act_1x128(x[rows.astype(np.int64)])
    q = qbuf.cpu().numpy()
    s = sbuf.cpu().numpy()
    assert np.array_equal(q[:M, :K], q_ref)
    assert np.array_equal(s[:, :M].view(np.uint32), np.ascontiguousarray(sf_ref.T).view(np.uint32))
    assert np.all(q[M] == SENTINEL_Q) and np.all(q[:, K:] == SENTINEL_Q) and np.all(s[:, M:] == SENTINEL_S)


def test_gather_bad_index_is_reported_not_faulted(fp8q):
    """Indices outside [0, M_src) quantize a zero row (codes 0, scale 1e-12)
    and set FP8Q_ERR_INVALID_ARG in the device status word; the other rows are
    unaffected."""
    import torch
    M_src, K = 16, 256
    x = W.activations_with_outliers(M_src, K, seed=3, channel_frac=0, elem_frac=0)
    rows = np.array([3, -1, 15, M_src, 1 << 30, 0], np.int32)
    q = torch.full((6, K), SENTINEL_Q, dtype=torch.uint8, device="cuda")
    sf = torch.full((K // 128, 8), SENTINEL_S, dtype=torch.float32, device="cuda")
    fp8q.fp8q_quant_act_1x128_gather(to_dev_bf16(x), torch.from_numpy(rows).cuda(), q, sf)
    torch.cuda.synchronize()
    status = fp8q.fp8q_device_status()
    assert status & 0xFF == fp8q.FP8Q_ERR_INVALID_ARG
    good = np.array([0, 2, 5])
    q_ref, sf_ref = oracle.quant_act_1x128(x[rows[good].astype(np.int64)])
    qh, sh = q.cpu().numpy(), sf.cpu().numpy()
    assert np.array_equal(qh[good], q_ref)
    assert np.array_equal(sh[:, good].T, sf_ref)
    bad = np.array([1, 3, 4])
    assert np.all(qh[bad] == 0)
    assert np.all(sh[:, bad] == np.float32(oracle.tile_scale(0.0)))
    assert fp8q.fp8q_device_status() == 0            # the word was cleared by the read


def test_moe_dispatch_and_up_projection_full_size(fp8q):
    """The MoE step's fused path at full size: 4096 tokens x 7168 gathered into
    the 32768 expert rows of a top-8 of 256 Zipf(1.1) routing (gather-quantize
    checked on every row), then the up projection 7168 -> 2048 with the FP8
    epilogue, checked on sampled rows of every non-empty checked expert against
    the oracle's quantization of the BF16 GEMM's rows."""
    import torch
    route = W.moe_routing(seed=0)
    off = route.offsets
    Mt = int(off[-1])
    x = W.activations_with_outliers(4096, 7168, seed=0)
    rows = torch.from_numpy(route.token_of_row.astype(np.int32)).cuda()
    qa = torch.empty((Mt, 7168), dtype=torch.uint8, device="cuda")
    sa = torch.empty((56, Mt), dtype=torch.float32, device="cuda")
    fp8q.fp8q_quant_act_1x128_gather(to_dev_bf16(x), rows, qa, sa)
    torch.cuda.synchronize()
    assert fp8q.fp8q_device_status() == 0
    oq, osf = oracle.quant_act_1x128(np.ascontiguousarray(x[route.token_of_row]))
    assert np.array_equal(qa.cpu().numpy(), oq)
    assert np.array_equal(sa.cpu().numpy(), np.ascontiguousarray(osf.T))
    del oq, osf
    N, K = 2048, 7168
    wdev = W.expert_weights_device(256, N, K, seed=0, tid=W.TID_EXPERT_UP)
    wq = torch.empty((256, N, K), dtype=torch.uint8, device="cuda")
    ws = torch.empty((256, N // 128, K // 128), dtype=torch.float32, device="cuda")
    for g in range(256):
        fp8q.fp8q_quant_w_128x128(wdev[g], wq[g], ws[g])
    del wdev
    offd = torch.from_numpy(off.astype(np.int32)).cuda()
    d = torch.empty((Mt, N), dtype=torch.bfloat16, device="cuda")
    fp8q.fp8q_grouped_gemm_blockscaled(qa, sa, wq, ws, offd, d)
    hq = torch.empty((Mt, N), dtype=torch.uint8, device="cuda")
    hs = torch.empty((N // 128, Mt), dtype=torch.float32, device="cuda")
    fp8q.fp8q_grouped_gemm_blockscaled_q1x128(qa, sa, wq, ws, offd, hq, hs)
    torch.cuda.synchronize()
    assert fp8q.fp8q_device_status() == 0
    rng = np.random.default_rng(21)
    sample = np.unique(np.concatenate([[0, Mt - 1], rng.integers(0, Mt, 200)])).astype(np.int64)
    idx = torch.from_numpy(sample).cuda()
    q_ref, sf_ref = oracle.quant_act_1x128(_bf16_bits(d[idx]))
    assert np.array_equal(hq[idx].cpu().numpy(), q_ref)
    assert np.array_equal(hs[:, idx].cpu().numpy().T, sf_ref)
