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
