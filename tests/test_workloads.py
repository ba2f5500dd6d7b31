"""The seeded input generators (workloads/): the recipe's structure -- the
same bytes for the same seed, independent streams per tensor, the outlier
counts and magnitudes it states, the routing's top-k distinct experts and
forced-empty experts, the drift tiles' doubling deviation and their outlier,
and the midpoint pairs' defining property."""
import numpy as np

import workloads as W


def test_generators_are_reproducible_and_seeded():
    a = W.activations_with_outliers(64, 512, seed=3)
    assert np.array_equal(a, W.activations_with_outliers(64, 512, seed=3))
    assert not np.array_equal(a, W.activations_with_outliers(64, 512, seed=4))
    w = W.weights(256, 512, seed=3)
    assert not np.array_equal(a[:, :256], w[:64, :256])     # another tensor id, another stream


def test_activation_outliers_follow_the_recipe():
    M, K = 256, 1024
    x = W.bf16_bits_to_f32(W.activations_with_outliers(M, K, seed=0, channel_frac=4 / K, channel_gain=20.0,
                                                     elem_frac=1e-3, elem_value=120.0))
    assert np.sum(np.abs(x) == 120.0) == round(1e-3 * M * K)
    col_rms = np.sqrt((x ** 2).mean(axis=0))
    assert np.sum(col_rms > 10.0) >= 4                     # the 4 amplified channels stand out


def test_routing_structure():
    r = W.moe_routing(512, 64, 8, n_forced_empty=3, seed=1)
    ids = r.expert_ids
    assert ids.shape == (512, 8)
    assert all(len(set(row)) == 8 for row in ids.tolist())  # distinct experts per token
    assert np.all(r.counts[r.empty_experts] == 0) and r.empty_experts.size == 3
    assert r.offsets[-1] == 512 * 8 and np.array_equal(np.diff(r.offsets), r.counts)
    # packed rows: expert-major, tokens ascending within an expert, and entry_row inverts token_of_row
    assert np.all(r.token_of_row[r.entry_row] == np.arange(512)[:, None])
    exp_of_row = np.repeat(np.arange(64), r.counts)
    assert np.all(exp_of_row[r.entry_row] == ids)


def test_drift_tiles_double_and_hold_one_outlier():
    x, t_out = W.drift_tiles(steps=100, seed=0, outlier_sigmas=20.0)
    xf = W.bf16_bits_to_f32(x).astype(np.float64)
    sd = np.sqrt((np.delete(xf, t_out, axis=0) ** 2).mean(axis=1))
    assert 1.5 < sd[-10:].mean() / sd[:10].mean() < 2.5
    assert 25 <= t_out < 75 and np.abs(xf[t_out]).max() > 10 * np.sqrt((xf[t_out] ** 2).mean()) / 2


def test_midpoint_pairs_are_traps():
    codes, scales = W.midpoint_product_pairs(32)
    assert codes.size == 32
    for c, s in zip(codes, scales):
        v = np.float32(W.MIDPOINT_CODES[int(c)])
        p = np.float32(v * s)
        assert (int(np.array([p]).view(np.uint32)[0]) & 0xFFFF) == 0x8000     # a BF16 midpoint in float32
        assert np.float64(v) * np.float64(s) != np.float64(p)                 # but not the exact product
