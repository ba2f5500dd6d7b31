"""GPU parity of the grouped (MoE expert) block-scaled GEMM.

Per-expert semantics are those of the dense GEMM; group sizes live only on the
device.  MoE context: "FP8 Mixed Precision: DeepSeek-V3 Training
Architecture", sections 2 and 4 (expert routing, FP8 dispatch).
"""
import numpy as np
import pytest

import oracle
import workloads as W
from common import check_gemm, load_fp8q, to_dev_bf16, to_dev_f32, to_dev_u8

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fp8q():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return load_fp8q()


def _sfa_dev(sf_mk):
    M, KB = sf_mk.shape
    ld = (M + 3) // 4 * 4
    buf = np.full((KB, ld), np.nan, np.float32)
    buf[:, :M] = sf_mk.T
    return to_dev_f32(buf)


def run_grouped(fp8q, qa, sa, wq, ws, offsets):
    import torch
    Mt, K = qa.shape
    G, N, _ = wq.shape
    d = torch.full((Mt + 1, N), -5.0, dtype=torch.bfloat16, device="cuda")
    off = torch.from_numpy(np.asarray(offsets, np.int32)).cuda()
    fp8q.fp8q_grouped_gemm_blockscaled(to_dev_u8(qa), _sfa_dev(sa), to_dev_u8(wq), to_dev_f32(ws), off, d[:Mt])
    torch.cuda.synchronize()
    status = fp8q.fp8q_device_status()
    out = d.float().cpu().numpy().astype(np.float64)
    assert np.all(out[Mt] == -5.0)
    return out[:Mt], status


def _experts(G, N, K, seed):
    wq = np.empty((G, N, K), np.uint8)
    ws = np.empty((G, N // 128, K // 128), np.float32)
    for g in range(G):
        wq[g], ws[g] = oracle.quant_w_128x128(W.weights(N, K, seed=seed * 1000 + g))
    return wq, ws


@pytest.mark.parametrize("counts", [
    [3, 0, 1, 130, 0, 257],          # empty experts, a 1-row expert, ragged tiles
    [0, 0, 700, 0],                  # everything in one expert
    [1] * 9,                         # many one-row experts
    [128, 128, 0, 256],              # exact tile multiples
])
def test_grouped_parity(fp8q, counts):
    G, N, K = len(counts), 384, 512
    off = W.ragged_offsets(counts)
    Mt = int(off[-1])
    x = W.activations_with_outliers(Mt, K, seed=Mt, channel_frac=1 / K, elem_frac=1e-3)
    qa, sa = oracle.quant_act_1x128(x)
    wq, ws = _experts(G, N, K, seed=G)
    d, status = run_grouped(fp8q, qa, sa, wq, ws, off)
    assert status == 0
    ref = oracle.grouped_gemm_sampled(qa, sa, wq, ws, off)
    check_gemm(d, ref, oracle.round_bf16(ref))


def test_grouped_bad_offsets_are_reported_not_faulted(fp8q):
    """Offsets beyond M_total are clamped on the device and reported through
    the status word (no out-of-bounds access)."""
    G, N, K = 3, 256, 256
    qa, sa = oracle.quant_act_1x128(W.activations_with_outliers(40, K, seed=2, channel_frac=0, elem_frac=0))
    wq, ws = _experts(G, N, K, seed=7)
    bad = [0, 10, 1 << 30, 40]
    d, status = run_grouped(fp8q, qa, sa, wq, ws, bad)
    assert status & 0xFF == 1            # FP8Q_ERR_INVALID_ARG
    # clamped offsets [0, 10, 40, 40]: experts 0 and 1 computed as usual
    ref = oracle.grouped_gemm_sampled(qa, sa, wq, ws, np.array([0, 10, 40, 40]))
    check_gemm(d, ref, oracle.round_bf16(ref))


def test_non_monotone_offsets_return_invalid_arg_status(fp8q):
    """Decreasing offsets are forced nondecreasing on the device and reported;
    the C entry point fp8q_device_status returns FP8Q_ERR_INVALID_ARG (the code
    held in the word's low byte), not a timeout."""
    import ctypes
    import torch
    G, N, K = 3, 256, 256
    qa, sa = oracle.quant_act_1x128(W.activations_with_outliers(40, K, seed=4, channel_frac=0, elem_frac=0))
    wq, ws = _experts(G, N, K, seed=8)
    d = torch.empty((40, N), dtype=torch.bfloat16, device="cuda")
    off = torch.tensor([0, 30, 12, 40], dtype=torch.int32, device="cuda")
    fp8q.fp8q_grouped_gemm_blockscaled(to_dev_u8(qa), _sfa_dev(sa), to_dev_u8(wq), to_dev_f32(ws), off, d)
    code = ctypes.c_int(0)
    rc = fp8q.lib().fp8q_device_status(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream), ctypes.byref(code))
    assert rc == fp8q.FP8Q_ERR_INVALID_ARG
    assert code.value & 0xFF == fp8q.FP8Q_ERR_INVALID_ARG
    assert fp8q.fp8q_device_status() == 0
    # offsets as the device used them: [0, 30, 30, 40]
    ref = oracle.grouped_gemm_sampled(qa, sa, wq, ws, np.array([0, 30, 30, 40]))
    check_gemm(d.float().cpu().numpy().astype(np.float64), ref, oracle.round_bf16(ref))


def test_moe_full_size(fp8q):
    """4096 tokens x 7168, top-8 of 256 experts with Zipf(1.1) popularity and 8
    forced-empty experts; up 7168 -> 2048 and down 2048 -> 7168 with 128x128-block
    FP8 expert weights.  Weights are drawn on the device by the seeded input
    generator and quantized there; the oracle gets a copy of the same BF16
    weights of every non-empty expert and quantizes them itself.  Each of the
    248 non-empty experts is checked on full rows (its first, its last and one
    between), so a tile-mapping error in any expert's tiles shows."""
    import torch
    fp = fp8q
    route = W.moe_routing(seed=0)
    off = route.offsets
    Mt = int(off[-1])
    x = W.activations_with_outliers(4096, 7168, seed=0)
    xp = np.ascontiguousarray(x[route.token_of_row])           # packed by expert
    h = W.normal_bf16(Mt, 2048, 1.0, seed=0, tid=W.TID_H)       # down-projection input
    offd = torch.from_numpy(off.astype(np.int32)).cuda()
    counts = route.counts
    # every non-empty expert: its first and last rows and one row between
    check_experts = np.nonzero(counts)[0]
    assert len(check_experts) == 248
    rng = np.random.default_rng(9)
    for (K, N, tid, a_bits) in ((7168, 2048, W.TID_EXPERT_UP, xp), (2048, 7168, W.TID_EXPERT_DN, h)):
        wdev = W.expert_weights_device(256, N, K, seed=0, tid=tid)
        wq = torch.empty((256, N, K), dtype=torch.uint8, device="cuda")
        ws = torch.empty((256, N // 128, K // 128), dtype=torch.float32, device="cuda")
        for g in range(256):
            fp.fp8q_quant_w_128x128(wdev[g], wq[g], ws[g])
        qa, sa = fp.quant_act_1x128(to_dev_bf16(a_bits))
        d = torch.empty((Mt, N), dtype=torch.bfloat16, device="cuda")
        fp.fp8q_grouped_gemm_blockscaled(qa, sa, wq, ws, offd, d)
        torch.cuda.synchronize()
        assert fp.fp8q_device_status() == 0
        oqa, osa = oracle.quant_act_1x128(a_bits)
        assert np.array_equal(qa.cpu().numpy(), oqa)
        for g in check_experts:
            wbits = wdev[g].view(torch.int16).cpu().numpy().view(np.uint16)
            oq, osf = oracle.quant_w_128x128(wbits)
            assert np.array_equal(wq[g].cpu().numpy(), oq)
            r0, r1 = int(off[g]), int(off[g + 1])
            rows = np.unique(np.concatenate([[r0, r1 - 1], rng.integers(r0, r1, 1)])).astype(np.int64)
            one = np.array([0, r1 - r0], np.int64)
            ref = oracle.grouped_gemm_sampled(oqa[r0:r1], osa[r0:r1], oq[None], osf[None], one,
                                              rows=rows - r0, cols=np.arange(N, dtype=np.int64))
            got = d[torch.from_numpy(rows).cuda()].float().cpu().numpy().astype(np.float64)
            check_gemm(got, ref, oracle.round_bf16(ref))
        del wdev, wq, ws, d
        torch.cuda.empty_cache()
