"""Pins for the oracle's block-scaled GEMM and grouped GEMM (CPU only).

Passages: "FP8 Mixed Precision: DeepSeek-V3 Training Architecture", section
"3. Decoupled Accumulation in Tensor Core GEMMs" (eq. C_ij) and the "Step 2"
listing (X_fine @ W_fine.T); "Introduction to LLM Quantization",
"Fine-grained Quantization" Steps 1-4 and "3) Backward propagation".

Pins (independent of the oracle's code):
  * small-integer codes with power-of-two scales: the result is an exact
    integer matmul (numpy int64) times the scale, so it must match exactly;
  * general data: the "Step 2" formulation, a float64 numpy matmul of the
    dequantised operands, to FP64 rounding;
  * a one-hot row reproduces a dequantised column of B;
  * K = 128 (one chunk) against a pure-Python triple loop on a tiny case;
  * grouped GEMM: per-expert numpy matmuls, with empty and one-row experts.
"""
import numpy as np
import pytest

import oracle
import workloads as W

# E4M3 codes of the integers -4..4 (1 = 0x38, 2 = 0x40, 3 = 0x44, 4 = 0x48)
INT_CODES = {0: 0x00, 1: 0x38, 2: 0x40, 3: 0x44, 4: 0x48,
             -1: 0xB8, -2: 0xC0, -3: 0xC4, -4: 0xC8}


def _int_operand(rng, R, K):
    ints = rng.integers(-4, 5, size=(R, K))
    codes = np.vectorize(INT_CODES.get)(ints).astype(np.uint8)
    return ints.astype(np.int64), codes


def test_int_codes_decode():
    for v, c in INT_CODES.items():
        assert oracle.e4m3_decode(np.array([c], np.uint8))[0] == v


@pytest.mark.parametrize("mode", [oracle.SFB_BLOCK128, oracle.SFB_ROW])
def test_gemm_exact_integers_pow2_scales(mode):
    rng = np.random.default_rng(11)
    M, N, K = 5, 256, 384
    ia, qa = _int_operand(rng, M, K)
    ib, qb = _int_operand(rng, N, K)
    ea = rng.integers(-6, 6, size=(M, K // 128))
    sfa = np.exp2(ea).astype(np.float32)
    if mode == oracle.SFB_BLOCK128:
        eb = rng.integers(-6, 6, size=(N // 128, K // 128))
        eb_full = np.repeat(eb, 128, axis=0)
    else:
        eb = rng.integers(-6, 6, size=(N, K // 128))
        eb_full = eb
    sfb = np.exp2(eb).astype(np.float32)
    D = oracle.gemm_sampled(qa, sfa, qb, sfb, mode)
    ref = np.zeros((M, N))
    for kb in range(K // 128):
        part = ia[:, kb * 128:(kb + 1) * 128] @ ib[:, kb * 128:(kb + 1) * 128].T   # exact int64
        ref += part * np.exp2(ea[:, kb][:, None] + eb_full[:, kb][None, :])
    assert np.array_equal(D, ref)


@pytest.mark.parametrize("mode", [oracle.SFB_BLOCK128, oracle.SFB_ROW])
def test_gemm_equals_dequantised_matmul(mode):
    M, N, K = 37, 384, 512
    x = W.activations_with_outliers(M, K, seed=3, channel_frac=2 / K, elem_frac=1e-3)
    qa, sfa = oracle.quant_act_1x128(x)
    if mode == oracle.SFB_BLOCK128:
        qb, sfb = oracle.quant_w_128x128(W.weights(N, K, seed=3))
        sb_full = np.repeat(np.repeat(sfb, 128, axis=0), 128, axis=1)
    else:
        qb, sfb = oracle.quant_act_1x128(W.activations_with_outliers(N, K, seed=4))
        sb_full = np.repeat(sfb, 128, axis=1)
    deq_a = oracle.e4m3_decode(qa) * np.repeat(sfa.astype(np.float64), 128, axis=1)
    deq_b = oracle.e4m3_decode(qb) * sb_full.astype(np.float64)
    ref = deq_a @ deq_b.T
    D = oracle.gemm_sampled(qa, sfa, qb, sfb, mode)
    assert np.allclose(D, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    # sampled rows/cols are the same numbers as the full product
    rows = np.array([0, 5, 36])
    cols = np.array([383, 0, 128, 129])
    Ds = oracle.gemm_sampled(qa, sfa, qb, sfb, mode, rows=rows, cols=cols)
    assert np.array_equal(Ds, D[np.ix_(rows, cols)])


def test_gemm_one_hot_row_gives_dequantised_column():
    M, N, K = 2, 256, 256
    qb, sfb = oracle.quant_w_128x128(W.weights(N, K, seed=8))
    qa = np.zeros((M, K), np.uint8)
    qa[0, 200] = INT_CODES[1]
    qa[1, 3] = INT_CODES[-2]
    sfa = np.array([[1.0, 1.0], [0.5, 1.0]], np.float32)
    D = oracle.gemm_sampled(qa, sfa, qb, sfb, oracle.SFB_BLOCK128)
    col200 = oracle.e4m3_decode(qb[:, 200]) * np.repeat(sfb[:, 1].astype(np.float64), 128)
    col3 = oracle.e4m3_decode(qb[:, 3]) * np.repeat(sfb[:, 0].astype(np.float64), 128)
    assert np.array_equal(D[0], col200)
    assert np.array_equal(D[1], -2.0 * 0.5 * col3)


def test_gemm_single_chunk_python_loops():
    rng = np.random.default_rng(5)
    M, N, K = 3, 128, 128
    qa = rng.integers(0, 256, size=(M, K)).astype(np.uint8)
    qb = rng.integers(0, 256, size=(N, K)).astype(np.uint8)
    qa[(qa & 0x7F) == 0x7F] = 0x01      # no NaN codes
    qb[(qb & 0x7F) == 0x7F] = 0x02
    sfa = rng.uniform(0.01, 2, size=(M, 1)).astype(np.float32)
    sfb = rng.uniform(0.01, 2, size=(1, 1)).astype(np.float32)
    D = oracle.gemm_sampled(qa, sfa, qb, sfb, oracle.SFB_BLOCK128)
    da = oracle.e4m3_decode(qa)
    db = oracle.e4m3_decode(qb)
    for m in range(M):
        for n in range(N):
            s = 0.0
            for k in range(K):
                s += float(da[m, k]) * float(db[n, k])          # exact: see the oracle's header
            assert D[m, n] == (float(sfa[m, 0]) * float(sfb[0, 0])) * s


def test_grouped_gemm_matches_per_expert_products():
    G, N, K = 5, 256, 256
    counts = np.array([3, 0, 1, 130, 0])
    off = W.ragged_offsets(counts)
    Mt = int(off[-1])
    x = W.activations_with_outliers(Mt, K, seed=6, channel_frac=0.0, elem_frac=1e-3)
    qa, sfa = oracle.quant_act_1x128(x)
    wq = np.empty((G, N, K), np.uint8)
    ws = np.empty((G, N // 128, K // 128), np.float32)
    for g in range(G):
        wq[g], ws[g] = oracle.quant_w_128x128(W.weights(N, K, seed=100 + g))
    D = oracle.grouped_gemm_sampled(qa, sfa, wq, ws, off)
    for g in range(G):
        r0, r1 = off[g], off[g + 1]
        if r1 == r0:
            continue
        ref = oracle.gemm_sampled(qa[r0:r1], sfa[r0:r1], wq[g], ws[g], oracle.SFB_BLOCK128)
        assert np.array_equal(D[r0:r1], ref)
        deq_a = oracle.e4m3_decode(qa[r0:r1]) * np.repeat(sfa[r0:r1].astype(np.float64), 128, axis=1)
        deq_w = oracle.e4m3_decode(wq[g]) * np.repeat(np.repeat(ws[g], 128, 0), 128, 1).astype(np.float64)
        assert np.allclose(D[r0:r1], deq_a @ deq_w.T, rtol=1e-12, atol=1e-12)


def test_gemm_rejects_bad_arguments():
    qa = np.zeros((2, 100), np.uint8)
    with pytest.raises(ValueError):
        oracle.gemm_sampled(qa, np.ones((2, 1), np.float32), qa, np.ones((1, 1), np.float32),
                            oracle.SFB_ROW)


def test_moe_routing_structure():
    r = W.moe_routing(tokens=4096, experts=256, top_k=8, seed=0)
    assert r.offsets[-1] == 4096 * 8
    assert np.all(r.counts[r.empty_experts] == 0) and r.empty_experts.size == 8
    assert r.counts.max() <= 4096                # an expert takes a token at most once
    # each token appears top_k times, with distinct experts
    tok_counts = np.bincount(r.token_of_row, minlength=4096)
    assert np.all(tok_counts == 8)
    exp_of_row = np.repeat(np.arange(256), r.counts)
    pairs = set(zip(r.token_of_row.tolist(), exp_of_row.tolist()))
    assert len(pairs) == 4096 * 8
    # Zipf popularity: group sizes are very uneven
    s = np.sort(r.counts)[::-1]
    assert s[0] > 10 * np.median(s)
