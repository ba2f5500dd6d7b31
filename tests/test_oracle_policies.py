"""Pins of the oracle's scale-policy functions ("Online Quantization During
Training", section 4 "Max scaling is robust but noisy" and its worked example;
"Introduction to LLM Quantization", "5) Online Quantization", delayed versus
online quantization).

The quantizer with given scales reduces to the online quantizer when it is
given the online scales; its cast and clip count are checked against NumPy's
IEEE float32 division and the codec; the history updates are checked through
their special cases and invariants; the drift simulation through the
behaviour the pages describe.
"""
import numpy as np
import pytest

import oracle
import workloads as W


def test_given_online_scales_reproduce_the_online_quantizer():
    x = W.activations_with_outliers(40, 512, seed=3, channel_frac=2 / 512, elem_frac=1e-2)
    q_on, sf_on = oracle.quant_act_1x128(x)
    q, amax, clipped = oracle.quant_act_1x128_scaled(x, sf_on)
    assert np.array_equal(q, q_on)
    assert clipped == 0                                # the online scale never saturates its tile
    # the recorded maxima are the tiles' maxima: the online rule rebuilds the same scales
    assert np.array_equal(np.vectorize(oracle.tile_scale, otypes=[np.float32])(amax), sf_on)
    xf = W.bf16_bits_to_f32(x).reshape(40, 4, 128)
    assert np.array_equal(amax, np.abs(xf).max(axis=2))


@pytest.mark.parametrize("scale_mult", [1.0, 0.5, 0.01, 7.3])
def test_scaled_cast_and_clip_count_against_numpy(scale_mult):
    """Arbitrary scales: codes = codec(float32(x) / float32(s)) and the clip
    count = #|x/s| > 464 (the saturating cast's threshold), by brute force."""
    x = W.activations_with_outliers(16, 384, seed=5, channel_frac=0, elem_frac=1e-2)
    _, sf_on = oracle.quant_act_1x128(x)
    sf = (sf_on * np.float32(scale_mult)).astype(np.float32)
    q, _, clipped = oracle.quant_act_1x128_scaled(x, sf)
    xf = W.bf16_bits_to_f32(x)
    v = (xf.reshape(16, 3, 128) / sf[:, :, None]).astype(np.float32).reshape(16, 384)
    assert np.array_equal(q, oracle.e4m3_encode(v))
    assert clipped == int((np.abs(v) > 464.0).sum())
    if scale_mult < 1.0:
        assert clipped > 0
    # saturated elements carry the extreme codes
    assert np.all(np.isin(q[np.abs(v) > 464.0], [0x7E, 0xFE]))


def test_history_update_special_cases():
    rng = np.random.default_rng(0)
    a = rng.uniform(0.01, 50.0, 64).astype(np.float32)
    h = rng.uniform(0.01, 50.0, 64).astype(np.float32)
    tile = np.vectorize(oracle.tile_scale, otypes=[np.float32])
    # previous step: the history is the last maximum, whatever alpha
    h0, s0 = oracle.scale_history_update(oracle.POLICY_PREVIOUS, 0.7, a, h)
    assert np.array_equal(h0, a) and np.array_equal(s0, tile(a))
    # EMA with alpha = 0 forgets, alpha = 1 never moves; decayed max with alpha = 0 is the current max
    h1, _ = oracle.scale_history_update(oracle.POLICY_EMA, 0.0, a, h)
    assert np.array_equal(h1, a)
    h2, _ = oracle.scale_history_update(oracle.POLICY_EMA, 1.0, a, h)
    assert np.array_equal(h2, h)
    h3, _ = oracle.scale_history_update(oracle.POLICY_DECAYED_MAX, 0.0, a, h)
    assert np.array_equal(h3, a)
    # EMA of a constant stays at it; decayed max never falls below the current maximum
    hc, _ = oracle.scale_history_update(oracle.POLICY_EMA, 0.9, a, a)
    assert np.allclose(hc, a, rtol=2 ** -22)
    hd, sd = oracle.scale_history_update(oracle.POLICY_DECAYED_MAX, 0.8, a, h)
    assert np.all(hd >= a) and np.all(hd >= (np.float32(0.8) * h).astype(np.float32))
    assert np.array_equal(sd, tile(hd))
    # EMA lies between its two inputs
    he, _ = oracle.scale_history_update(oracle.POLICY_EMA, 0.9, a, h)
    lo, hi = np.minimum(a, h), np.maximum(a, h)
    assert np.all(he >= lo * (1 - 2 ** -22)) and np.all(he <= hi * (1 + 2 ** -22))


ALPHAS = (0.1, 0.37, 0.9, 0.999)


def _ema_pairs(seed, n=4096):
    rng = np.random.default_rng(seed)
    a = np.exp(rng.uniform(-8, 6, n)).astype(np.float32)
    h = np.exp(rng.uniform(-8, 6, n)).astype(np.float32)
    return a, h


@pytest.mark.parametrize("alpha", ALPHAS)
def test_ema_history_bit_exact_against_numpy_float32(alpha):
    """The exponential history rounds every operation to FP32 on its own:
    beta = fl32(1 - alpha), h' = fl32(fl32(alpha * h) + fl32(beta * a))
    ("Online Quantization During Training", section 4 and its worked example:
    an exponential moving history of the tile maxima).  NumPy float32
    arithmetic rounds each operation once, so it states the same value
    independently of the oracle's C++."""
    a, h = _ema_pairs(seed=int(alpha * 1000))
    got, sf = oracle.scale_history_update(oracle.POLICY_EMA, alpha, a, h)
    al = np.float32(alpha)
    beta = np.float32(np.float32(1.0) - al)
    want = (np.float32(al * h) + np.float32(beta * a)).astype(np.float32)
    assert want.dtype == np.float32
    assert np.array_equal(got, want)
    tile = np.vectorize(oracle.tile_scale, otypes=[np.float32])
    assert np.array_equal(sf, tile(want))


def test_ema_pin_separates_plausible_variants():
    """The pin above would catch the plausible mistakes: a fused multiply-add
    (one rounding of alpha*h + r), beta = 1 - alpha kept in double, or the
    whole update in double and rounded once.  Each of them differs from the
    oracle on some of the same inputs."""
    fma_diff = dbl_beta_diff = all_dbl_diff = 0
    for alpha in ALPHAS:
        a, h = _ema_pairs(seed=int(alpha * 1000))
        got, _ = oracle.scale_history_update(oracle.POLICY_EMA, alpha, a, h)
        al = np.float32(alpha)
        beta = np.float32(np.float32(1.0) - al)
        r = (beta * a).astype(np.float32)
        fma = (np.float64(al) * h.astype(np.float64) + r.astype(np.float64)).astype(np.float32)
        beta64 = np.float64(1.0) - np.float64(al)
        dbl_beta = (np.float32(al * h) + (beta64 * a.astype(np.float64)).astype(np.float32)).astype(np.float32)
        all_dbl = (np.float64(al) * h.astype(np.float64) + beta64 * a.astype(np.float64)).astype(np.float32)
        fma_diff += int((fma != got).sum())
        dbl_beta_diff += int((dbl_beta != got).sum())
        all_dbl_diff += int((all_dbl != got).sum())
    assert fma_diff > 0 and dbl_beta_diff > 0 and all_dbl_diff > 0, (fma_diff, dbl_beta_diff, all_dbl_diff)


def test_bad_policy_is_rejected():
    with pytest.raises(Exception):
        oracle.scale_history_update(3, 0.5, np.ones(4, np.float32), np.ones(4, np.float32))


def test_drift_simulation_matches_the_pages_claims():
    """The worked example: std doubling over 100 steps, one 20-sigma outlier.
    Current-max never clips; a fixed calibration clips more and more as the
    distribution widens; every history policy clips the outlier (it lags
    behind a sudden range change) and pays for it in error at that step."""
    tiles, t_out = W.drift_tiles(steps=100, seed=0)
    res = oracle.scale_policy_drift(tiles, alpha=0.9)
    clip_cur, err_cur = res["current_max"]
    assert np.all(clip_cur == 0)
    clip_fix, err_fix = res["fixed"]
    assert clip_fix[:10].mean() < clip_fix[-10:].mean()
    assert clip_fix[-10:].mean() > 0.1
    for name in ("previous", "ema", "decayed_max"):
        clip, err = res[name]
        assert clip[t_out] >= 1 / 128, name                 # the outlier is clamped
        assert err[t_out] > 5 * err_cur[t_out], name
        assert clip.mean() < clip_fix.mean(), name          # but far less clipping than a fixed scale
    # E4M3 is a floating-point grid: a 20-sigma tile maximum leaves the other
    # values well inside the normal range, so current-max loses little there
    neighbours = np.r_[err_cur[t_out - 3:t_out], err_cur[t_out + 1:t_out + 4]]
    assert err_cur[t_out] < 2 * neighbours.mean()


# ---------------------------------------------------------------- percentile clipping
def _nearest_rank_scales(xf_tiles, p):
    """Per tile: v = NumPy's nearest-rank percentile (Hyndman-Fan type 1,
    'inverted_cdf') of the magnitudes, then the online scale rule on v."""
    v = np.percentile(np.abs(xf_tiles), 100.0 * p, axis=-1, method="inverted_cdf")
    return np.vectorize(oracle.tile_scale, otypes=[np.float32])(v.astype(np.float32))


def test_percentile_rank_is_the_nearest_rank_rule():
    assert oracle.percentile_rank(1.0) == 1
    assert oracle.percentile_rank(0.99) == 2          # ceil(126.72) = 127th smallest of 128
    assert oracle.percentile_rank(0.5) == 65
    assert oracle.percentile_rank(1 / 128) == 128     # the smallest value
    vals = np.random.default_rng(1).permutation(128).astype(np.float64)
    for p in (0.9, 0.95, 0.99, 0.999, 0.5, 0.01):
        r = oracle.percentile_rank(p)
        assert np.percentile(vals, 100 * p, method="inverted_cdf") == np.sort(vals)[::-1][r - 1]
    with pytest.raises(ValueError):
        oracle.percentile_rank(0.0)


def test_percentile_rank_one_is_the_online_quantizer():
    x = W.activations_with_outliers(24, 512, seed=8, channel_frac=2 / 512, elem_frac=1e-2)
    q_on, sf_on = oracle.quant_act_1x128(x)
    q, sf, clipped = oracle.quant_act_1x128_percentile(x, 1)
    assert np.array_equal(q, q_on) and np.array_equal(sf, sf_on) and clipped == 0


@pytest.mark.parametrize("p", [0.99, 0.95, 0.9, 0.5])
def test_percentile_against_numpy(p):
    """Scales from NumPy's nearest-rank percentile, codes from NumPy's float32
    division and the codec, the clip count by brute force."""
    M, K = 20, 384
    x = W.activations_with_outliers(M, K, seed=9, channel_frac=0, elem_frac=2e-2)
    r = oracle.percentile_rank(p)
    q, sf, clipped = oracle.quant_act_1x128_percentile(x, r)
    xf = W.bf16_bits_to_f32(x).reshape(M, K // 128, 128)
    s_np = _nearest_rank_scales(xf, p)
    assert np.array_equal(sf, s_np)
    v = (xf / s_np[:, :, None]).astype(np.float32)
    assert np.array_equal(q, oracle.e4m3_encode(v.reshape(M, K)))
    per_tile = (np.abs(v) > 464.0).sum(axis=2)
    assert clipped == int(per_tile.sum())
    assert np.all(per_tile <= r - 1)                  # only values above the r-th largest can saturate


def test_percentile_ties_and_single_outlier():
    # all-equal tile: every rank gives the same scale and nothing clips
    x = np.full((1, 128), 0x3F80, np.uint16)          # 1.0
    for r in (1, 2, 64, 128):
        q, sf, clipped = oracle.quant_act_1x128_percentile(x, r)
        assert sf[0, 0] == oracle.tile_scale(1.0) and clipped == 0 and np.all(q == 0x7E)
    # one 20x outlier among values of magnitude <= 1: rank 2 clamps exactly it
    rng = np.random.default_rng(4)
    xf = rng.uniform(-1.0, 1.0, 128).astype(np.float32)
    xf[37] = -20.0
    xb = (xf.view(np.uint32) >> 16).astype(np.uint16)[None, :]
    q, sf, clipped = oracle.quant_act_1x128_percentile(xb, 2)
    assert clipped == 1 and q[0, 37] == 0xFE
    second = np.sort(np.abs(W.bf16_bits_to_f32(xb)[0]))[-2]
    assert sf[0, 0] == oracle.tile_scale(second)


def test_percentile_in_the_drift_run():
    """Clipping the current tile's top value protects the rest of the tile's
    grid but clamps the 20-sigma outlier itself: on an E4M3 grid that costs
    more than it saves (the online maximum keeps the lower error)."""
    tiles, t_out = W.drift_tiles(steps=100, seed=0)
    res = oracle.scale_policy_drift(tiles, alpha=0.9, percentile=0.99)
    clip, err = res["percentile"]
    _, err_cur = res["current_max"]
    assert clip[t_out] == 1 / 128
    assert err[t_out] > 5 * err_cur[t_out]
    assert err.mean() > err_cur.mean()
    assert np.all(clip <= 1 / 128)                    # rank 2: at most one element per tile
