"""GPU parity of the scale-policy calls against the oracle, bit for bit:
the 1x128 quantizer with given scales (codes, recorded tile maxima, count of
saturated elements) and the per-tile history update; and the drift workload
of "Online Quantization During Training" (worked example) run step by step on
the device under an exponential amax history, against the oracle's run.
"""
import numpy as np
import pytest

import oracle
import workloads as W
from common import load_fp8q, to_dev_bf16, to_dev_f32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fp8q():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return load_fp8q()


def _kmajor(a_mk, ld):
    M, KB = a_mk.shape
    buf = np.full((KB, ld), np.nan, np.float32)
    buf[:, :M] = a_mk.T
    return buf


@pytest.mark.parametrize("M,K,mult", [
    (1, 128, 1.0),        # the online scales: no clipping
    (70, 384, 0.5),       # scales halved: the largest values saturate
    (130, 256, 0.02),     # heavy saturation
    (33, 512, 3.7),       # coarse scales: many codes in the subnormal range
])
def test_scaled_quantizer_matches_oracle(fp8q, M, K, mult):
    import torch
    x = W.activations_with_outliers(M, K, seed=M + K, channel_frac=2 / K, elem_frac=1e-2)
    _, sf_on = oracle.quant_act_1x128(x)
    sf = (sf_on * np.float32(mult)).astype(np.float32)
    oq, oamax, oclip = oracle.quant_act_1x128_scaled(x, sf)
    ld = (M + 3) // 4 * 4 + 4
    xd = to_dev_bf16(np.pad(x, ((0, 0), (0, 8))))[:, :K]
    sfd = to_dev_f32(_kmajor(sf, ld))
    qbuf = torch.full((M + 1, K + 16), 0x5A, dtype=torch.uint8, device="cuda")
    amax = torch.full((K // 128, ld), -1.0, dtype=torch.float32, device="cuda")
    clipped = torch.zeros(1, dtype=torch.int64, device="cuda")
    fp8q.fp8q_quant_act_1x128_scaled(xd, sfd, qbuf[:M, :K], amax, clipped)
    torch.cuda.synchronize()
    assert fp8q.fp8q_device_status() == 0
    q = qbuf.cpu().numpy()
    assert np.array_equal(q[:M, :K], oq)
    assert np.all(q[M] == 0x5A) and np.all(q[:, K:] == 0x5A)
    a = amax.cpu().numpy()
    assert np.array_equal(a[:, :M].T, oamax) and np.all(a[:, M:] == -1.0)
    assert int(clipped.item()) == oclip
    if mult == 1.0:
        assert oclip == 0
    if mult < 1.0:
        assert oclip > 0


def test_scaled_quantizer_overflowing_quotients(fp8q):
    """Given scales far below the tiles' ranges: x / s overflows FP32 to
    infinity for the largest values, and must still saturate to +-448."""
    import torch
    M, K = 4, 256
    rng = np.random.default_rng(5)
    xf = rng.standard_normal((M, K)).astype(np.float32) * 1e30
    xf[0, :8] = [3.0e38, -3.0e38, 1e27, -1e27, 0.0, -0.0, 1e-30, -1e-30]
    x = (xf.view(np.uint32) >> 16).astype(np.uint16)
    sf = np.full((M, K // 128), 1e-12, np.float32)
    sf[1, 1] = 3e-39                                  # a subnormal scale
    oq, oamax, oclip = oracle.quant_act_1x128_scaled(x, sf)
    ld = 8
    xd = to_dev_bf16(x)
    qd = torch.empty((M, K), dtype=torch.uint8, device="cuda")
    amax = torch.empty((K // 128, ld), dtype=torch.float32, device="cuda")
    clipped = torch.zeros(1, dtype=torch.int64, device="cuda")
    fp8q.fp8q_quant_act_1x128_scaled(xd, to_dev_f32(_kmajor(sf, ld)), qd, amax, clipped)
    torch.cuda.synchronize()
    assert np.array_equal(qd.cpu().numpy(), oq)
    assert int(clipped.item()) == oclip and oclip > 0


@pytest.mark.parametrize("policy", [0, 1, 2])
@pytest.mark.parametrize("alpha", [0.0, 0.5, 0.9, 1.0])
def test_history_update_matches_oracle(fp8q, policy, alpha):
    import torch
    rng = np.random.default_rng(policy * 10 + int(alpha * 10))
    n = 1000
    a = np.exp(rng.uniform(-30, 20, n)).astype(np.float32)
    h = np.exp(rng.uniform(-30, 20, n)).astype(np.float32)
    a[:5] = 0.0
    h[5:10] = 0.0
    oh, osf = oracle.scale_history_update(policy, alpha, a, h)
    ad, hd = to_dev_f32(a), to_dev_f32(h)
    sfd = torch.empty(n, dtype=torch.float32, device="cuda")
    fp8q.fp8q_scale_history_update(policy, alpha, ad, hd, sfd)
    torch.cuda.synchronize()
    assert np.array_equal(hd.cpu().numpy().view(np.uint32), oh.view(np.uint32))
    assert np.array_equal(sfd.cpu().numpy().view(np.uint32), osf.view(np.uint32))


def test_drift_workload_under_ema_history(fp8q):
    """100 steps of one 1x128 tile (std doubling, one 20-sigma outlier): the
    device loop -- quantize with the history's scale, record the maximum,
    update the history -- gives the oracle's scales, codes and clip counts."""
    import torch
    tiles, t_out = W.drift_tiles(steps=100, seed=0)
    alpha = 0.9
    sf = torch.empty((1, 4), dtype=torch.float32, device="cuda")     # [K/128][ld = 4]
    q = torch.empty((1, 128), dtype=torch.uint8, device="cuda")
    amax = torch.empty((1, 4), dtype=torch.float32, device="cuda")
    hist = torch.zeros(1, dtype=torch.float32, device="cuda")
    clipped = torch.zeros(1, dtype=torch.int64, device="cuda")
    # step 0 is calibrated on itself (the online quantizer), and starts the history
    x0 = to_dev_bf16(tiles[0:1])
    fp8q.fp8q_quant_act_1x128(x0, q, sf)
    o_sf = oracle.quant_act_1x128(tiles[0:1])[1][0, 0]
    o_hist = np.zeros(1, np.float32)
    dev_clips, o_clips = [], []
    for t in range(100):
        xt = to_dev_bf16(tiles[t:t + 1])
        before = int(clipped.item())
        fp8q.fp8q_quant_act_1x128_scaled(xt, sf, q, amax, clipped)
        if t == 0:
            hist.copy_(amax[0, :1])
        fp8q.fp8q_scale_history_update(oracle.POLICY_EMA, alpha, amax[0, :1], hist, sf[0, :1])
        torch.cuda.synchronize()
        dev_clips.append(int(clipped.item()) - before)
        # the oracle, step by step with the same rules
        oq, oa, oc = oracle.quant_act_1x128_scaled(tiles[t:t + 1], np.array([[o_sf]], np.float32))
        assert np.array_equal(q.cpu().numpy(), oq), t
        o_clips.append(oc)
        if t == 0:
            o_hist[0] = oa[0, 0]
        o_hist, o_next = oracle.scale_history_update(oracle.POLICY_EMA, alpha, oa[0], o_hist)
        o_sf = o_next[0]
        assert sf[0, 0].item() == float(o_sf), t
    assert dev_clips == o_clips
    assert dev_clips[t_out] >= 1
    ref = oracle.scale_policy_drift(tiles, alpha=alpha)["ema"][0]
    assert np.array_equal(np.array(dev_clips) / 128.0, ref)
    assert fp8q.fp8q_device_status() == 0


# ---------------------------------------------------------------- percentile clipping
def _run_percentile(fp8q, x, rank):
    import torch
    M, K = x.shape
    ld = (M + 3) // 4 * 4 + 4
    xd = to_dev_bf16(np.pad(x, ((0, 0), (0, 8))))[:, :K]
    qbuf = torch.full((M + 1, K + 16), 0x5A, dtype=torch.uint8, device="cuda")
    sf = torch.full((K // 128, ld), -1.0, dtype=torch.float32, device="cuda")
    clipped = torch.zeros(1, dtype=torch.int64, device="cuda")
    fp8q.fp8q_quant_act_1x128_percentile(xd, rank, qbuf[:M, :K], sf, clipped)
    torch.cuda.synchronize()
    assert fp8q.fp8q_device_status() == 0
    q = qbuf.cpu().numpy()
    assert np.all(q[M] == 0x5A) and np.all(q[:, K:] == 0x5A)
    s = sf.cpu().numpy()
    assert np.all(s[:, M:] == -1.0)
    return q[:M, :K], s[:, :M].T, int(clipped.item())


@pytest.mark.parametrize("M,K,rank", [
    (1, 128, 1), (70, 384, 2), (130, 256, 3), (65, 512, 8), (33, 128, 64), (40, 256, 128), (200, 1024, 2),
])
def test_percentile_quantizer_matches_oracle(fp8q, M, K, rank):
    x = W.activations_with_outliers(M, K, seed=3 * M + K + rank, channel_frac=2 / K, elem_frac=2e-2)
    oq, osf, oclip = oracle.quant_act_1x128_percentile(x, rank)
    q, sf, clip = _run_percentile(fp8q, x, rank)
    assert np.array_equal(q, oq)
    assert np.array_equal(sf.view(np.uint32), osf.view(np.uint32))
    assert clip == oclip
    if rank == 1:
        assert clip == 0


def _f32_to_bf16_bits(v):
    return (np.asarray(v, np.float32).view(np.uint32) >> 16).astype(np.uint16)


def test_percentile_degenerate_tiles(fp8q):
    """Ties at the top, all-equal and all-zero tiles, signed zeros, BF16
    subnormals, a rank above the number of distinct magnitudes, and a huge
    outlier over tiny values (x / s overflows to infinity in FP32)."""
    rng = np.random.default_rng(11)
    tiles = []
    tiles.append(np.zeros(128, np.float32))                                   # all zero
    t = -np.zeros(128, np.float32); tiles.append(t)                            # all -0
    tiles.append(np.full(128, -3.5, np.float32))                               # all equal
    t = rng.uniform(-1, 1, 128).astype(np.float32); t[[3, 50, 77, 100, 127]] = [9, -9, 9, 9, -9]
    tiles.append(t)                                                            # five-way tie at the top
    t = np.zeros(128, np.float32); t[[0, 64]] = [2.0, -1.0]; tiles.append(t)   # two distinct magnitudes + zeros
    t = (rng.integers(1, 127, 128) * 2.0 ** -133).astype(np.float32); tiles.append(t)  # BF16 subnormals
    t = np.full(128, 1e-30, np.float32); t[9] = -3.0e38; tiles.append(t)      # overflow of x / s
    t = rng.standard_normal(128).astype(np.float32) * 1e-3; t[17] = 5e3; t[90] = -4e3; tiles.append(t)
    x = _f32_to_bf16_bits(np.stack(tiles))
    for rank in (1, 2, 3, 5, 6, 100, 128):
        oq, osf, oclip = oracle.quant_act_1x128_percentile(x, rank)
        q, sf, clip = _run_percentile(fp8q, x, rank)
        assert np.array_equal(q, oq), rank
        assert np.array_equal(sf.view(np.uint32), osf.view(np.uint32)), rank
        assert clip == oclip, rank


def test_percentile_full_size(fp8q):
    """The 8192 x 7168 activation at the 99th percentile (rank 2), every tile."""
    M, K = 8192, 7168
    x = W.activations_with_outliers(M, K, seed=21, channel_frac=4 / K, elem_frac=1e-3)
    rank = oracle.percentile_rank(0.99)
    oq, osf, oclip = oracle.quant_act_1x128_percentile(x, rank)
    q, sf, clip = _run_percentile(fp8q, x, rank)
    assert np.array_equal(sf.view(np.uint32), osf.view(np.uint32))
    assert np.array_equal(q, oq)
    assert clip == oclip and clip > 0
