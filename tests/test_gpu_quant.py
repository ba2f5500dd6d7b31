"""GPU parity of the quantizers against the oracle: bytes and scales bit-exact.

Passages: "Fine-Grained FP8 Quantization in DeepSeek", sections 2-3;
"FP8 Mixed Precision: DeepSeek-V3 Training Architecture", section 1 (eq. s_W,
eq. W_FP8); "Introduction to LLM Quantization", "5) Online Quantization".
"""
import numpy as np
import pytest

import oracle
import workloads as W
from common import load_fp8q, to_dev_bf16

pytestmark = pytest.mark.gpu

CANARY = 0xA5


@pytest.fixture(scope="module")
def fp8q():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return load_fp8q()


def _padded_bf16(x_bits, ld):
    M, K = x_bits.shape
    buf = np.full((M, ld), 0x7FC0, np.uint16)      # NaN padding: must never be read
    buf[:, :K] = x_bits
    return buf


def run_q1(fp8q, x_bits, ldx=None, ldq=None, ld_sf=None):
    import torch
    M, K = x_bits.shape
    ldx = ldx or K
    ldq = ldq or K
    ld_sf = ld_sf or M
    xd = to_dev_bf16(_padded_bf16(x_bits, ldx))[:, :K]
    # guard rows before and after every output
    qbuf = torch.full((M + 2, ldq), CANARY, dtype=torch.uint8, device="cuda")
    sfbuf = torch.full((K // 128 + 2, ld_sf), -7.0, dtype=torch.float32, device="cuda")
    q = qbuf[1:M + 1, :K]
    sf = sfbuf[1:K // 128 + 1]
    fp8q.fp8q_quant_act_1x128(xd, q, sf)
    torch.cuda.synchronize()
    assert fp8q.fp8q_device_status() == 0
    qh = qbuf.cpu().numpy()
    sfh = sfbuf.cpu().numpy()
    assert np.all(qh[0] == CANARY) and np.all(qh[M + 1] == CANARY)
    assert np.all(qh[1:M + 1, K:] == CANARY)
    assert np.all(sfh[0] == -7.0) and np.all(sfh[-1] == -7.0) and np.all(sfh[1:-1, M:] == -7.0)
    return qh[1:M + 1, :K], sfh[1:-1, :M].T.copy()


@pytest.mark.parametrize("M,K,ldx,ldq,ld_sf", [
    (1, 128, None, None, 4),
    (7, 384, 392, 400, 12),
    (33, 1024, None, None, None),
    (130, 256, 264, 272, 131),
    (517, 640, None, None, 520),
])
def test_quant_1x128_parity(fp8q, M, K, ldx, ldq, ld_sf):
    x = W.activations_with_outliers(M, K, seed=M + K, channel_frac=2 / K, elem_frac=1e-3)
    q, sf = run_q1(fp8q, x, ldx, ldq, ld_sf)
    oq, osf = oracle.quant_act_1x128(x)
    assert np.array_equal(sf, osf)
    assert np.array_equal(q, oq)


def _edge_rows():
    """Tiles the pages' review advice calls for: zero, -0, a single non-zero,
    exact E4M3 midpoints (ties), subnormal landings, the maximum in every lane."""
    rows = []
    rows.append(np.zeros(128, np.float32))
    rows.append(-np.zeros(128, np.float32))
    one = np.zeros(128, np.float32); one[77] = -3.0; rows.append(one)
    # amax = 448 -> s = 1 exactly, so the cast input is the value itself
    mids = np.array([1.0625, 1.1875, 1.3125, 1.4375, 2.125, 2.375, 2.0 ** -10, 3 * 2.0 ** -10,
                     5 * 2.0 ** -10, 7 * 2.0 ** -10, 15 * 2.0 ** -10, 464.0 / 2, 240.0, 208.0], np.float32)
    t = np.zeros(128, np.float32); t[0] = 448.0; t[1:1 + mids.size] = mids; t[20:20 + mids.size] = -mids
    rows.append(t)
    # amax = 448 * 2^-5 -> s = 2^-5: midpoints scaled
    rows.append(t * np.float32(2.0 ** -5))
    # amax = 1344 -> s = 3 exactly, not a power of two: x = 3*mid (exact in BF16)
    # divides exactly onto the midpoint, while x * fl32(1/3) lands just off it,
    # so these ties must come out of the exact (division) path
    t3 = np.zeros(128, np.float32); t3[0] = 1344.0; t3[1:1 + mids.size] = 3 * mids; t3[20:20 + mids.size] = -3 * mids
    rows.append(t3)
    # values far below the tile max: subnormal codes
    sub = np.linspace(-2e-4, 2e-4, 128).astype(np.float32); sub[5] = 3.0; rows.append(sub)
    for lane in range(0, 128, 9):
        r = np.random.default_rng(lane).standard_normal(128).astype(np.float32)
        r[lane] = 17.5 if lane % 2 else -17.5
        rows.append(r)
    return W.f32_to_bf16_bits(np.stack(rows))


def test_quant_1x128_edge_tiles(fp8q):
    x = _edge_rows()
    x = np.concatenate([x, x], axis=1)           # two chunks per row
    q, sf = run_q1(fp8q, x)
    oq, osf = oracle.quant_act_1x128(x)
    assert np.array_equal(sf, osf) and np.array_equal(q, oq)
    assert np.all(q[0] == 0x00) and np.all(q[1] == 0x80)
    assert sf[0, 0] == np.float32(1e-12)


def test_quant_1x128_full_activation_workload(fp8q):
    """8192 x 7168 BF16 ~N(0,1), 0.1% channels x20, 1e-5 elements -> +-120."""
    x = W.activations_with_outliers(8192, 7168, seed=0)
    q, sf = run_q1(fp8q, x)
    oq, osf = oracle.quant_act_1x128(x)
    assert np.array_equal(sf, osf)
    assert np.array_equal(q, oq)


def run_qt(fp8q, x_bits, ldx=None, ldqt=None, ld_sf=None):
    import torch
    T, C = x_bits.shape
    ldx = ldx or C
    ldqt = ldqt or T
    ld_sf = ld_sf or C
    xd = to_dev_bf16(_padded_bf16(x_bits, ldx))[:, :C]
    qbuf = torch.full((C + 2, ldqt), CANARY, dtype=torch.uint8, device="cuda")
    sfbuf = torch.full((T // 128 + 2, ld_sf), -7.0, dtype=torch.float32, device="cuda")
    fp8q.fp8q_quant_act_128x1(xd, qbuf[1:C + 1, :T], sfbuf[1:T // 128 + 1])
    torch.cuda.synchronize()
    assert fp8q.fp8q_device_status() == 0
    qh = qbuf.cpu().numpy()
    sfh = sfbuf.cpu().numpy()
    assert np.all(qh[0] == CANARY) and np.all(qh[C + 1] == CANARY) and np.all(qh[1:C + 1, T:] == CANARY)
    assert np.all(sfh[0] == -7.0) and np.all(sfh[-1] == -7.0) and np.all(sfh[1:-1, C:] == -7.0)
    return qh[1:C + 1, :T], sfh[1:-1, :C]


@pytest.mark.parametrize("T,C,ldx,ldqt,ld_sf", [
    (128, 8, None, None, None),
    (256, 264, 272, 272, 268),
    (384, 520, None, 400, None),
    (128, 1024, None, None, None),
])
def test_quant_128x1_parity(fp8q, T, C, ldx, ldqt, ld_sf):
    x = W.activations_with_outliers(T, C, seed=T + C, channel_frac=1 / C, elem_frac=1e-3)
    qt, sf = run_qt(fp8q, x, ldx, ldqt, ld_sf)
    oqt, osf = oracle.quant_act_128x1(x)
    assert np.array_equal(sf, osf)
    assert np.array_equal(qt, oqt)


def test_quant_128x1_edge_tiles(fp8q):
    x = np.ascontiguousarray(_edge_rows()[:, :128].T)       # every edge tile as a column
    x = np.concatenate([x, x[:, ::-1]], axis=1)
    C = x.shape[1] // 8 * 8
    x = np.ascontiguousarray(x[:, :C])
    qt, sf = run_qt(fp8q, x)
    oqt, osf = oracle.quant_act_128x1(x)
    assert np.array_equal(sf, osf) and np.array_equal(qt, oqt)


def test_quant_128x1_full_workloads(fp8q):
    """Both Wgrad operands: X 8192x7168 and dY 8192x18432 along the token dimension."""
    x = W.activations_with_outliers(8192, 7168, seed=0)
    qt, sf = run_qt(fp8q, x)
    oqt, osf = oracle.quant_act_128x1(x)
    assert np.array_equal(sf, osf) and np.array_equal(qt, oqt)
    dy = W.grad_with_outlier_tokens(8192, 18432, seed=0)
    qt, sf = run_qt(fp8q, dy)
    oqt, osf = oracle.quant_act_128x1(dy)
    assert np.array_equal(sf, osf) and np.array_equal(qt, oqt)


def run_qw(fp8q, w_bits, transposed=True, ldw=None):
    import torch
    N, K = w_bits.shape
    ldw = ldw or K
    wd = to_dev_bf16(_padded_bf16(w_bits, ldw))[:, :K]
    q = torch.full((N, K), CANARY, dtype=torch.uint8, device="cuda")
    sf = torch.full((N // 128, K // 128), -7.0, dtype=torch.float32, device="cuda")
    qt = sft = None
    if transposed:
        qt = torch.full((K, N), CANARY, dtype=torch.uint8, device="cuda")
        sft = torch.full((K // 128, N // 128), -7.0, dtype=torch.float32, device="cuda")
    fp8q.fp8q_quant_w_128x128(wd, q, sf, qt, sft)
    torch.cuda.synchronize()
    assert fp8q.fp8q_device_status() == 0
    out = [q.cpu().numpy(), sf.cpu().numpy()]
    if transposed:
        out += [qt.cpu().numpy(), sft.cpu().numpy()]
    return out


@pytest.mark.parametrize("N,K,ldw", [(128, 128, None), (384, 256, 264), (256, 1152, None)])
def test_quant_w_parity(fp8q, N, K, ldw):
    w = W.weights(N, K, seed=N + K)
    w[3, 5] = W.f32_to_bf16_bits(np.array([0.9], np.float32))[0]
    q, sf, qt, sft = run_qw(fp8q, w, True, ldw)
    oq, osf = oracle.quant_w_128x128(w)
    assert np.array_equal(sf, osf) and np.array_equal(q, oq)
    assert np.array_equal(sft, osf.T) and np.array_equal(qt, oq.T)
    q2, sf2 = run_qw(fp8q, w, False)
    assert np.array_equal(q2, oq) and np.array_equal(sf2, osf)


def test_quant_w_edge_blocks(fp8q):
    """The edge tiles (zeros, -0, ties at scales 1, 2^-5 and 3, subnormal
    landings) laid out as 128x128 weight blocks."""
    e = _edge_rows()                                   # [rows][128]
    reps = -(-128 // e.shape[0])
    blk = np.concatenate([e] * reps, axis=0)[:128]     # one block per edge set
    w = np.concatenate([blk, e[np.arange(128) % e.shape[0]][:, ::-1]], axis=0)   # two blocks
    for i, row in enumerate(e[:8]):                    # and blocks whose max is one edge row's
        b = np.zeros((128, 128), np.uint16); b[5] = row; b[77] = row[::-1]
        w = np.concatenate([w, b], axis=0)
    q, sf, qt, sft = run_qw(fp8q, np.ascontiguousarray(w), True)
    oq, osf = oracle.quant_w_128x128(w)
    assert np.array_equal(sf, osf) and np.array_equal(q, oq)
    assert np.array_equal(sft, osf.T) and np.array_equal(qt, oq.T)


def test_quant_w_full_weight(fp8q):
    """W 18432 x 7168 ~N(0, 0.02): 144 x 56 blocks, with the transposed copy."""
    w = W.weights(18432, 7168, seed=0)
    q, sf, qt, sft = run_qw(fp8q, w, True)
    oq, osf = oracle.quant_w_128x128(w)
    assert np.array_equal(sf, osf) and np.array_equal(q, oq)
    assert np.array_equal(sft, osf.T) and np.array_equal(qt, oq.T)


def test_device_cast_matches_oracle_encoder_all_fp32(fp8q):
    """Every FP32 bit pattern through the device E4M3 cast (the one the
    quantizers use) against the oracle's encoder written from the OCP format."""
    import torch
    chunk = 1 << 27
    out = torch.empty(chunk, dtype=torch.uint8, device="cuda")
    for start in range(0, 1 << 32, chunk):
        fp8q.fp8q_debug_cast_e4m3_bits(start, chunk, out)
        dev = out.cpu().numpy()
        bits = np.arange(start, start + chunk, dtype=np.uint64).astype(np.uint32)
        x = bits.view(np.float32)
        ref = oracle.e4m3_encode(x)
        nan = np.isnan(x)
        ok = (dev == ref) | (nan & ((dev & 0x7F) == 0x7F))
        if not ok.all():
            bad = np.nonzero(~ok)[0][:8]
            raise AssertionError([(hex(int(bits[i])), float(x[i]), int(dev[i]), int(ref[i])) for i in bad])
    assert fp8q.fp8q_device_status() == 0


def _amax_sweep(n_random=384, seed=0):
    """Rows of 128 BF16 values; each row holds a tile maximum amax first and
    then BF16 inputs with |x| <= amax.  For every amax sampled (all-zero tiles,
    the smallest subnormal, the largest finite value, 448, powers of two and a
    seeded sample of the rest) the rows cover EVERY BF16 x with |x| <= amax,
    both signs and both zeros.  Rows of one amax are padded to a multiple of
    128 so that 128x128 blocks and 128-token columns share it as well."""
    rng = np.random.default_rng(seed)
    specials = [0x0000, 0x0001, 0x007F, 0x0080, 0x3F80, 0x43E0, 0x43E1, 0x7F7F, 0x0100, 0x2000, 0x5F00]
    picks = np.unique(np.concatenate([np.array(specials), rng.integers(1, 0x7F80, n_random)])).astype(np.uint32)
    blocks = []
    for ab in picks:
        mags = np.arange(ab + 1, dtype=np.uint32)
        xs = np.concatenate([mags, mags | 0x8000]).astype(np.uint16)
        rows = -(-xs.size // 127)
        rows = -(-rows // 128) * 128
        body = np.zeros(rows * 127, np.uint16)
        body[:xs.size] = xs
        blk = np.empty((rows, 128), np.uint16)
        blk[:, 0] = ab
        blk[:, 1:] = body.reshape(rows, 127)
        blocks.append(blk)
    return np.concatenate(blocks, axis=0)


def test_quantizers_every_input_under_sampled_tile_maxima(fp8q):
    """The division-free cast on the device: all three quantizers equal the
    oracle's IEEE-quotient codes for every BF16 input under each sampled tile
    maximum."""
    x = _amax_sweep()
    R = x.shape[0]
    oq, osf = oracle.quant_act_1x128(x)
    q, sf = run_q1(fp8q, x)
    assert np.array_equal(sf.view(np.uint32), osf.view(np.uint32))
    assert np.array_equal(q, oq)
    # the same tiles as 128-token columns: x^T is [128 tokens][R channels]
    qt, sft = run_qt(fp8q, np.ascontiguousarray(x.T))
    assert np.array_equal(qt, oq) and np.array_equal(sft[0], osf[:, 0])
    # and as 128x128 blocks (each block's rows share one maximum)
    wq, wsf = run_qw(fp8q, x, transposed=False)
    owq, owsf = oracle.quant_w_128x128(x)
    assert np.array_equal(wsf, owsf) and np.array_equal(wq, owq)
    assert np.array_equal(wq, oq)       # every block's maximum is its rows' maximum
    assert R > 100000
