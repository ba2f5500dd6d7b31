"""Pins of the oracle's MoE dispatch definitions ("FP8 Mixed Precision:
DeepSeek-V3 Training Architecture", section 4: FP8 all-to-all dispatch): the
layout against a brute-force loop over the experts, and the per-rank result
of the reference against its own parts (one rank: the layout's order of the
quantized tokens; two ranks: the rows split by expert range)."""
import numpy as np

import oracle
import workloads as W


def test_layout_brute_force():
    rng = np.random.default_rng(1)
    ids = rng.integers(0, 5, (9, 3))
    ids[4] = [2, 2, 2]                                     # repeats keep slot order
    rows, pos, off = oracle.moe_layout(ids, 6)
    want_rows = [t for e in range(6) for t in range(9) for j in range(3) if ids[t, j] == e]
    assert rows.tolist() == want_rows
    assert off.tolist() == [0] + np.cumsum([(ids == e).sum() for e in range(6)]).tolist()
    for t in range(9):
        for j in range(3):
            assert rows[pos[t, j]] == t and ids.reshape(-1)[np.argsort(ids.reshape(-1), kind="stable")][pos[t, j]] == ids[t, j]
    assert sorted(pos.reshape(-1).tolist()) == list(range(27))


def test_reference_one_rank_is_layout_then_quantize():
    x = W.activations_with_outliers(40, 256, seed=3)
    ids = W.moe_routing(40, 8, 2, n_forced_empty=2, seed=3).expert_ids
    (q, sf, off), = oracle.moe_dispatch_reference([x], [ids], 8)
    rows, _, off_l = oracle.moe_layout(ids, 8)
    qx, sx = oracle.quant_act_1x128(x)
    assert np.array_equal(q, qx[rows]) and np.array_equal(sf, sx[rows]) and np.array_equal(off, off_l)


def test_reference_two_ranks_partition_the_rows():
    xs = [W.activations_with_outliers(30, 128, seed=s) for s in (5, 6)]
    ids = [W.moe_routing(30, 4, 2, n_forced_empty=0, seed=s).expert_ids for s in (5, 6)]
    out = oracle.moe_dispatch_reference(xs, ids, 4)
    assert sum(o[0].shape[0] for o in out) == 2 * 30 * 2
    # rank 1's first expert (global 2) holds rank 0's then rank 1's rows for it
    q1 = oracle.quant_act_1x128(xs[0])[0]
    t0 = np.nonzero((ids[0] == 2).any(axis=1))[0]
    assert np.array_equal(out[1][0][:t0.size], q1[t0])
