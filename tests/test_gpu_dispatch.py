"""GPU parity of the FP8 MoE dispatch's device steps against the oracle
("FP8 Mixed Precision: DeepSeek-V3 Training Architecture", section 4: FP8
all-to-all dispatch): the layout kernel (a stable counting sort by expert, bit
for bit), the gather quantizer with row-major scales, the quantize-once scatter
quantizer, the regroup of received FP8 rows, and the whole dispatch on one GPU
-- without a process group, and through a one-rank NCCL group (the
all_to_all_single path).
"""
import os
import socket

import numpy as np
import pytest

import oracle
import workloads as W
from common import load_fp8q, to_dev_bf16, to_dev_f32, to_dev_u8

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fp8q():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return load_fp8q()


def _ids_dev(ids):
    import torch
    return torch.from_numpy(np.ascontiguousarray(ids, np.int32)).cuda()


@pytest.mark.parametrize("T,k,E", [(4096, 8, 256), (1, 1, 1), (300, 3, 7), (1000, 4, 1024), (64, 8, 16)])
def test_layout_matches_oracle(fp8q, T, k, E):
    ids = W.moe_routing(T, E, k, n_forced_empty=min(2, E - k), seed=T + E).expert_ids
    rows, pos, off = fp8q.moe_dispatch_layout(_ids_dev(ids), E)
    assert fp8q.fp8q_device_status() == 0
    orows, opos, ooff = oracle.moe_layout(ids, E)
    assert np.array_equal(off.cpu().numpy(), ooff)
    assert np.array_equal(rows.cpu().numpy(), orows)
    assert np.array_equal(pos.cpu().numpy(), opos)


def test_layout_all_one_expert_and_bad_ids(fp8q):
    ids = np.full((700, 2), 3, np.int64)                      # every entry ties on one expert
    rows, pos, off = fp8q.moe_dispatch_layout(_ids_dev(ids), 4)
    assert fp8q.fp8q_device_status() == 0
    orows, opos, ooff = oracle.moe_layout(ids, 4)
    assert np.array_equal(rows.cpu().numpy(), orows) and np.array_equal(pos.cpu().numpy(), opos)
    assert off.cpu().numpy().tolist() == ooff.tolist()
    bad = ids.copy()
    bad[5, 1] = 4                                             # outside [0, E): dropped, status recorded
    bad[9, 0] = -2
    rows, pos, off = fp8q.moe_dispatch_layout(_ids_dev(bad), 4)
    assert fp8q.fp8q_device_status() != 0
    p = pos.cpu().numpy()
    assert p[5, 1] == -1 and p[9, 0] == -1 and off.cpu().numpy()[-1] == 1398
    keep = np.ones(bad.size, bool)
    keep[[5 * 2 + 1, 9 * 2]] = False
    assert np.array_equal(np.sort(p.reshape(-1)[keep]), np.arange(1398))


def test_gather_rowscales_matches_oracle(fp8q):
    import torch
    x = W.activations_with_outliers(500, 768, seed=9, channel_frac=2 / 768, elem_frac=1e-3)
    rows = np.random.default_rng(2).integers(0, 500, 1234).astype(np.int32)
    q = torch.full((1234, 768 + 16), 0x5A, dtype=torch.uint8, device="cuda")
    sf = torch.full((1234, 8), -1.0, dtype=torch.float32, device="cuda")
    fp8q.fp8q_quant_act_1x128_gather_rowscales(to_dev_bf16(x), torch.from_numpy(rows).cuda(), q[:, :768], sf)
    assert fp8q.fp8q_device_status() == 0
    oq, osf = oracle.quant_act_1x128(x)
    qh, sh = q.cpu().numpy(), sf.cpu().numpy()
    assert np.array_equal(qh[:, :768], oq[rows]) and np.all(qh[:, 768:] == 0x5A)
    assert np.array_equal(sh[:, :6], osf[rows]) and np.all(sh[:, 6:] == -1.0)


@pytest.mark.parametrize("K,packed", [(512, False), (4224, True), (7168, True)])
def test_regroup_matches_numpy(fp8q, K, packed):
    """Separate code and scale arrays, and the dispatch's packed receive rows
    (codes then scales in one row); K = 4224 ends in a partial batch of
    16-byte copies."""
    import torch
    from fine_grained_fp8_x128_b200.moe_dispatch import send_row_bytes, split_send_rows
    rng = np.random.default_rng(4 + K)
    M_in, M_out = 777, 1500
    q_in = rng.integers(0, 256, (M_in, K)).astype(np.uint8)
    sf_in = rng.random((M_in, K // 128)).astype(np.float32)
    rows = rng.integers(0, M_in, M_out).astype(np.int32)
    ld = M_out + 4
    q_out = torch.full((M_out, K), 0x5A, dtype=torch.uint8, device="cuda")
    sf_out = torch.full((K // 128, ld), -1.0, dtype=torch.float32, device="cuda")
    if packed:
        buf = np.zeros((M_in, send_row_bytes(K)), np.uint8)
        buf[:, :K] = q_in
        buf[:, K:K + 4 * (K // 128)] = sf_in.view(np.uint8)
        qd, sd = split_send_rows(to_dev_u8(buf), K)
    else:
        qd, sd = to_dev_u8(q_in), to_dev_f32(sf_in)
    fp8q.fp8q_gather_rows_fp8(qd, sd, torch.from_numpy(rows).cuda(), q_out, sf_out)
    assert fp8q.fp8q_device_status() == 0
    assert np.array_equal(q_out.cpu().numpy(), q_in[rows])
    s = sf_out.cpu().numpy()
    assert np.array_equal(s[:, :M_out], sf_in[rows].T) and np.all(s[:, M_out:] == -1.0)


def _offsets_table(counts_all):
    """Every source rank's layout offsets over all experts, rank-major."""
    world, E = counts_all.shape
    off = np.zeros((world, E + 1), np.int32)
    off[:, 1:] = np.cumsum(counts_all, axis=1)
    return off


def test_regroup_order_kernel_matches_host(fp8q):
    """The device order from the all-gathered offsets table against the host
    statement (regroup_order) on random tables: 1 to 8 ranks, empty sources
    and experts, every rank of the group, up to 1024 experts."""
    import torch
    from fine_grained_fp8_x128_b200.moe_dispatch import regroup_order
    rng = np.random.default_rng(11)
    cases = [(1, 256), (2, 8), (4, 64), (8, 1024), (3, 9), (8, 8)]
    for world, E in cases:
        el = E // world
        counts_all = rng.integers(0, 40, (world, E))
        counts_all[rng.random((world, E)) < 0.25] = 0
        if world > 2:
            counts_all[1, :] = 0                        # a source that sends nothing
        off = torch.from_numpy(_offsets_table(counts_all).reshape(-1)).cuda()
        for rank in range(world):
            recv = counts_all[:, rank * el:(rank + 1) * el]
            want_rows, want_off = regroup_order(recv)
            M = int(recv.sum())
            rows = torch.full((M,), -7, dtype=torch.int32, device="cuda")
            eo = torch.full((el + 1,), -7, dtype=torch.int32, device="cuda")
            fp8q.fp8q_moe_regroup_order(off, world, rank, E, rows, eo)
            assert fp8q.fp8q_device_status() == 0
            assert np.array_equal(rows.cpu().numpy(), want_rows), (world, E, rank)
            assert np.array_equal(eo.cpu().numpy(), want_off), (world, E, rank)


def test_regroup_order_kernel_reports_a_bad_table(fp8q):
    """M_recv larger than the table's total: the extra rows get -1 and the
    status word records FP8Q_ERR_INVALID_ARG; a decreasing table too."""
    import torch
    counts_all = np.array([[3, 0, 2, 1], [1, 4, 0, 2]])
    off = torch.from_numpy(_offsets_table(counts_all).reshape(-1)).cuda()
    rows = torch.full((8 + 3,), -7, dtype=torch.int32, device="cuda")
    eo = torch.empty(3, dtype=torch.int32, device="cuda")
    fp8q.fp8q_moe_regroup_order(off, 2, 0, 4, rows, eo)        # rank 0 receives 3+0+1+4 = 8 rows
    assert fp8q.fp8q_device_status() & 0xFF == fp8q.FP8Q_ERR_INVALID_ARG
    r = rows.cpu().numpy()
    assert np.all(r[8:] == -1) and np.array_equal(np.sort(r[:8]), np.arange(8))
    bad = _offsets_table(counts_all)
    bad[1, 2] = bad[1, 1] - 1                                   # a decreasing offset
    rows = torch.empty(8, dtype=torch.int32, device="cuda")
    fp8q.fp8q_moe_regroup_order(torch.from_numpy(bad.reshape(-1)).cuda(), 2, 0, 4, rows, eo)
    assert fp8q.fp8q_device_status() & 0xFF == fp8q.FP8Q_ERR_INVALID_ARG
    assert fp8q.fp8q_device_status() == 0


def _check_dispatch(res, x, ids, E):
    (q, sf, off), = oracle.moe_dispatch_reference([x], [ids], E)
    M = q.shape[0]
    assert np.array_equal(res.q.cpu().numpy(), q)
    assert np.array_equal(res.sf.cpu().numpy()[:, :M].T, sf)
    assert np.array_equal(res.expert_offsets.cpu().numpy(), off)


def test_dispatch_one_gpu(fp8q):
    """The 4096-token top-8 routing over 256 experts, no process group."""
    import torch
    from fine_grained_fp8_x128_b200.moe_dispatch import dispatch
    x = W.activations_with_outliers(4096, 1024, seed=1, channel_frac=2 / 1024, elem_frac=1e-3)
    ids = W.moe_routing(4096, 256, 8, seed=1).expert_ids
    res = dispatch(to_dev_bf16(x), _ids_dev(ids), 256)
    torch.cuda.synchronize()
    assert fp8q.fp8q_device_status() == 0
    _check_dispatch(res, x, ids, 256)


def test_dispatch_through_a_one_rank_nccl_group(fp8q):
    import torch
    import torch.distributed as dist
    from fine_grained_fp8_x128_b200.moe_dispatch import dispatch
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda:0"))
    try:
        x = W.activations_with_outliers(1000, 512, seed=2)
        ids = W.moe_routing(1000, 64, 6, seed=2).expert_ids
        res = dispatch(to_dev_bf16(x), _ids_dev(ids), 64)
        torch.cuda.synchronize()
        assert fp8q.fp8q_device_status() == 0
        _check_dispatch(res, x, ids, 64)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("T,k,E,H", [(4096, 8, 256, 7168), (300, 3, 7, 384), (1, 1, 1, 128)])
def test_scatter_quantizer_matches_oracle(fp8q, T, k, E, H):
    """Each token quantized once and written to its k layout rows: equal to the
    oracle's 1x128 quantization of the token for every row, rows untouched
    elsewhere, dropped entries (position -1) skipped."""
    import torch
    x = W.activations_with_outliers(T, H, seed=T + k, channel_frac=2 / H, elem_frac=1e-3)
    ids = W.moe_routing(T, E, k, n_forced_empty=min(2, E - k), seed=T).expert_ids
    rows, pos, off = oracle.moe_layout(ids, E)
    pos = pos.copy()
    if T > 1:
        pos[0, 0] = -1                                    # a dropped entry: its row stays untouched
    M = rows.size + 3                                     # three rows that no entry names
    q = torch.full((M, H + 16), 0x5A, dtype=torch.uint8, device="cuda")
    ld = (M + 3) // 4 * 4
    sf = torch.full((H // 128, ld), -1.0, dtype=torch.float32, device="cuda")
    fp8q.fp8q_quant_act_1x128_scatter(to_dev_bf16(x), torch.from_numpy(pos.astype(np.int32)).cuda(), q[:, :H], sf)
    assert fp8q.fp8q_device_status() == 0
    oq, osf = oracle.quant_act_1x128(x)
    qh, sh = q.cpu().numpy(), sf.cpu().numpy()
    written = np.zeros(M, bool)
    written[pos[pos >= 0]] = True
    tok_of = np.full(M, -1)
    tok_of[pos[pos >= 0]] = np.nonzero(pos >= 0)[0]
    assert np.array_equal(qh[written, :H], oq[tok_of[written]])
    assert np.array_equal(sh[:, :M][:, written], osf[tok_of[written]].T)
    assert np.all(qh[~written] == 0x5A) and np.all(sh[:, :M][:, ~written] == -1.0) and np.all(qh[:, H:] == 0x5A)


def test_scatter_rowscales_matches_oracle(fp8q):
    """The send-buffer form: scales row-major, sf[row][kb]."""
    import torch
    T, k, E, H = 500, 4, 16, 512
    x = W.activations_with_outliers(T, H, seed=7, channel_frac=2 / H, elem_frac=1e-3)
    ids = W.moe_routing(T, E, k, n_forced_empty=2, seed=7).expert_ids
    rows, pos, off = oracle.moe_layout(ids, E)
    M = rows.size
    q = torch.full((M, H), 0x5A, dtype=torch.uint8, device="cuda")
    sf = torch.full((M, H // 128 + 2), -1.0, dtype=torch.float32, device="cuda")
    fp8q.fp8q_quant_act_1x128_scatter_rowscales(to_dev_bf16(x), torch.from_numpy(pos.astype(np.int32)).cuda(), q,
                                                sf[:, :H // 128])
    assert fp8q.fp8q_device_status() == 0
    oq, osf = oracle.quant_act_1x128(x)
    sh = sf.cpu().numpy()
    assert np.array_equal(q.cpu().numpy(), oq[rows])
    assert np.array_equal(sh[:, :H // 128], osf[rows]) and np.all(sh[:, H // 128:] == -1.0)
