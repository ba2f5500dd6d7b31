"""Every output of the step's other full-size GEMMs against the FP64 oracle,
once: Dgrad (8192 x 7168, K = 18432), Wgrad (18432 x 7168, K = 8192, FP32 out)
and the MoE layer's up (32768 x 2048, K = 7168) and down (32768 x 7168,
K = 2048) projections over all 248 non-empty experts.  (The full-size Fprop
is compared in full in test_gpu_gemm.py.)  Each compares the whole output in
blocks of full rows with the GEMM tolerance of tests/common.py; together about
3e12 multiply-adds of oracle work, a few minutes on the host cores.

Passages: "FP8 Mixed Precision: DeepSeek-V3 Training Architecture", section 3
(eq. C_ij per 128-wide K chunk) and section 2 (the MoE layer);
"Introduction to LLM Quantization", "3) Backward propagation" (Dgrad, Wgrad).
"""
import numpy as np
import pytest

import oracle
import workloads as W
from common import check_gemm, load_fp8q, to_dev_bf16, to_dev_f32, to_dev_u8

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

BLK, ROW = 0, 1


@pytest.fixture(scope="module")
def fp8q():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return load_fp8q()


def _sf_dev(sf_mk):
    M, KB = sf_mk.shape
    ld = (M + 3) // 4 * 4
    buf = np.zeros((KB, ld), np.float32)
    buf[:, :M] = sf_mk.T
    return to_dev_f32(buf)


def _compare_full(got, ref_fn, M, block, f32_out):
    """got: host copy of the whole output; ref_fn(rows) -> the oracle's FP64 rows."""
    num = den = 0.0
    for r0 in range(0, M, block):
        rows = np.arange(r0, min(M, r0 + block), dtype=np.int64)
        ref = ref_fn(rows)
        blk = got[r0:r0 + len(rows)].astype(np.float64)
        check_gemm(blk, ref, oracle.round_f32(ref) if f32_out else oracle.round_bf16(ref))
        num += float(np.sum((blk - ref) ** 2))
        den += float(np.sum(ref ** 2))
    assert np.sqrt(num / den) <= 2e-3


def test_dgrad_full_output(fp8q):
    import torch
    dy = W.grad_with_outlier_tokens(8192, 18432, seed=0)
    w = W.weights(18432, 7168, seed=0)
    qa, sa = oracle.quant_act_1x128(dy)
    qb, sb = oracle.quant_w_128x128(np.ascontiguousarray(w.T))      # W^T blocks = transposed W blocks
    d = torch.empty((8192, 7168), dtype=torch.bfloat16, device="cuda")
    fp8q.fp8q_gemm_blockscaled(to_dev_u8(qa), _sf_dev(sa), to_dev_u8(qb), to_dev_f32(sb), BLK, d)
    torch.cuda.synchronize()
    assert fp8q.fp8q_device_status() == 0
    got = d.float().cpu().numpy()
    _compare_full(got, lambda rows: oracle.gemm_sampled(qa, sa, qb, sb, BLK, rows=rows), 8192, 512, False)


def test_wgrad_full_output(fp8q):
    import torch
    dy = W.grad_with_outlier_tokens(8192, 18432, seed=0)
    x = W.activations_with_outliers(8192, 7168, seed=0)
    qa, sa_t = oracle.quant_act_128x1(dy)            # [18432][8192], [64][18432]
    qb, sb_t = oracle.quant_act_128x1(x)             # [7168][8192],  [64][7168]
    sa = np.ascontiguousarray(sa_t.T)
    sb = np.ascontiguousarray(sb_t.T)
    d = torch.empty((18432, 7168), dtype=torch.float32, device="cuda")
    fp8q.fp8q_gemm_blockscaled(to_dev_u8(qa), _sf_dev(sa), to_dev_u8(qb), _sf_dev(sb), ROW, d)
    torch.cuda.synchronize()
    assert fp8q.fp8q_device_status() == 0
    got = d.cpu().numpy()
    _compare_full(got, lambda rows: oracle.gemm_sampled(qa, sa, qb, sb, ROW, rows=rows), 18432, 1024, True)


def test_moe_full_outputs(fp8q):
    """The 4096-token top-8 routing over 256 experts; expert weights drawn and
    quantized on the device, copied back and re-quantized by the oracle (bit
    for bit), then every row of both projections compared."""
    import torch
    route = W.moe_routing(seed=0)
    off = route.offsets.astype(np.int64)
    Mt = int(off[-1])
    offd = torch.from_numpy(off.astype(np.int32)).cuda()
    x = W.activations_with_outliers(4096, 7168, seed=0)
    xp = np.ascontiguousarray(x[route.token_of_row])
    h = W.normal_bf16(Mt, 2048, 1.0, seed=0, tid=W.TID_H)
    for (K, N, tid, a_bits) in ((7168, 2048, W.TID_EXPERT_UP, xp), (2048, 7168, W.TID_EXPERT_DN, h)):
        wdev = W.expert_weights_device(256, N, K, seed=0, tid=tid)
        wq = torch.empty((256, N, K), dtype=torch.uint8, device="cuda")
        ws = torch.empty((256, N // 128, K // 128), dtype=torch.float32, device="cuda")
        for g in range(256):
            fp8q.fp8q_quant_w_128x128(wdev[g], wq[g], ws[g])
        qa, sa = fp8q.quant_act_1x128(to_dev_bf16(a_bits))
        d = torch.empty((Mt, N), dtype=torch.bfloat16, device="cuda")
        fp8q.fp8q_grouped_gemm_blockscaled(qa, sa, wq, ws, offd, d)
        torch.cuda.synchronize()
        assert fp8q.fp8q_device_status() == 0
        got = d.float().cpu().numpy()
        oqa, osa = oracle.quant_act_1x128(a_bits)
        assert np.array_equal(qa.cpu().numpy(), oqa)
        owq = np.empty((256, N, K), np.uint8)
        ows = np.empty((256, N // 128, K // 128), np.float32)
        for g in range(256):
            owq[g], ows[g] = oracle.quant_w_128x128(wdev[g].view(torch.int16).cpu().numpy().view(np.uint16))
        assert np.array_equal(wq.cpu().numpy(), owq) and np.array_equal(ws.cpu().numpy(), ows)
        del wdev, wq, ws, d
        torch.cuda.empty_cache()
        _compare_full(got, lambda rows: oracle.grouped_gemm_sampled(oqa, osa, owq, ows, off, rows=rows), Mt, 2048,
                      False)
