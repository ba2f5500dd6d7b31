"""Host logic of the FP8 MoE dispatch ("FP8 Mixed Precision: DeepSeek-V3
Training Architecture", section 4: FP8 all-to-all dispatch), on the CPU: the
regroup order from per-expert counts, and the whole dispatch over two gloo
ranks with the device steps done by the oracle, compared with the oracle's
definition of what each rank must hold afterwards.
"""
import os
import socket

import numpy as np
import pytest

import oracle
import workloads as W
from fine_grained_fp8_x128_b200.moe_dispatch import dispatch, regroup_order, send_row_bytes


def test_regroup_order_small():
    # 2 sources x 3 local experts; receive buffer: source 0 rows (e0: 2, e1: 0, e2: 1), source 1 rows (e0: 1, e1: 2, e2: 0)
    rows, off = regroup_order(np.array([[2, 0, 1], [1, 2, 0]]))
    # expected output order: e0 (s0 rows 0,1; s1 row 3), e1 (s1 rows 4,5), e2 (s0 row 2)
    assert rows.tolist() == [0, 1, 3, 4, 5, 2]
    assert off.tolist() == [0, 3, 5, 6]


def test_regroup_order_is_a_permutation():
    rng = np.random.default_rng(0)
    counts = rng.integers(0, 5, (4, 8))
    counts[1, :] = 0                                  # a source that sends nothing
    counts[:, 3] = 0                                  # an expert that receives nothing
    rows, off = regroup_order(counts)
    assert np.array_equal(np.sort(rows), np.arange(counts.sum()))
    assert off[-1] == counts.sum() and np.array_equal(np.diff(off), counts.sum(axis=0))


def test_regroup_order_against_a_loop():
    """Random count tables (empty sources and experts included) against the
    order written out piece by piece."""
    rng = np.random.default_rng(3)
    for _ in range(200):
        world, el = int(rng.integers(1, 9)), int(rng.integers(1, 40))
        counts = rng.integers(0, 6, (world, el))
        counts[rng.random((world, el)) < 0.3] = 0
        base = np.concatenate([[0], np.cumsum(counts.sum(axis=1))])
        want = []
        for e in range(el):
            for s in range(world):
                first = base[s] + counts[s, :e].sum()
                want.extend(range(first, first + counts[s, e]))
        rows, off = regroup_order(counts)
        assert rows.tolist() == want
        assert off.tolist() == [0] + np.cumsum(counts.sum(axis=0)).tolist()


class OracleOps:
    """The dispatch's device steps done by the oracle, on CPU tensors."""

    def layout(self, expert_ids, num_experts):
        import torch
        rows, pos, off = oracle.moe_layout(expert_ids.numpy(), num_experts)
        return torch.from_numpy(rows), torch.from_numpy(pos), torch.from_numpy(off)

    def quant_send(self, x, pos, M):
        """Packed send rows: the codes, then the row's scales as bytes."""
        import torch
        qx, sx = oracle.quant_act_1x128(x.numpy())
        K = qx.shape[1]
        p = pos.numpy()
        tok = np.nonzero(p >= 0)[0]
        buf = np.zeros((M, send_row_bytes(K)), np.uint8)
        buf[p[p >= 0], :K] = qx[tok]
        buf[p[p >= 0], K:K + 4 * (K // 128)] = np.ascontiguousarray(sx[tok]).view(np.uint8)
        return torch.from_numpy(buf)

    def regroup_order(self, all_off, world, rank, num_experts, M):
        """The host statement of the order, from the same offsets table."""
        import torch
        el = num_experts // world
        per_expert = np.diff(all_off.numpy().astype(np.int64).reshape(world, num_experts + 1), axis=1)
        rows, off = regroup_order(per_expert[:, rank * el:(rank + 1) * el])
        assert rows.size == M
        return torch.from_numpy(rows), torch.from_numpy(off)

    def regroup(self, recv, K, rows):
        import torch
        r = np.asarray(rows)
        b = recv.numpy()[r]
        sf = np.ascontiguousarray(b[:, K:K + 4 * (K // 128)]).view(np.float32)
        return torch.from_numpy(np.ascontiguousarray(b[:, :K])), torch.from_numpy(np.ascontiguousarray(sf.T))

    def quant_grouped(self, x, pos, M):
        K = x.shape[1]
        return self.regroup(self.quant_send(x, pos, M), K, np.arange(M, dtype=np.int32))


def test_dispatch_without_a_process_group():
    """One process, all experts local: no exchange, the layout order is the
    grouped GEMM's, and the result equals the one-rank reference."""
    import torch
    x, ids = _inputs(0, 80, 256, 4, 8)
    res = dispatch(torch.from_numpy(x), torch.from_numpy(ids.astype(np.int32)), 8, ops=OracleOps())
    (q, sf, off), = oracle.moe_dispatch_reference([x], [ids], 8)
    assert np.array_equal(res.q.numpy(), q) and np.array_equal(res.sf.numpy().T, sf)
    assert np.array_equal(res.expert_offsets.numpy(), off)
    assert res.send_counts is None and res.recv_counts is None


def _inputs(rank, T, H, k, E):
    x = W.activations_with_outliers(T, H, seed=100 + rank, channel_frac=2 / H, elem_frac=1e-3)
    ids = W.moe_routing(T, E, k, n_forced_empty=1, seed=200 + rank).expert_ids
    return x, ids


def _rank_main(rank, world, port, T_list, H, k, E, result_q):
    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        x, ids = _inputs(rank, T_list[rank], H, k, E)
        res = dispatch(torch.from_numpy(x), torch.from_numpy(ids.astype(np.int32)), E, ops=OracleOps())
        ref = oracle.moe_dispatch_reference([_inputs(r, T_list[r], H, k, E)[0] for r in range(world)],
                                            [_inputs(r, T_list[r], H, k, E)[1] for r in range(world)], E)[rank]
        ok = (np.array_equal(res.q.numpy(), ref[0]) and np.array_equal(res.sf.numpy().T, ref[1])
              and np.array_equal(res.expert_offsets.numpy(), ref[2]))
        result_q.put((rank, ok, int(res.q.shape[0]), res.send_counts.tolist()))
    finally:
        dist.destroy_process_group()


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


@pytest.mark.parametrize("T_list", [(64, 64), (96, 40), (50, 0, 70, 33)])
def test_dispatch_gloo_ranks(T_list):
    """Two and four ranks; one rank of four has no tokens at all."""
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    world, H, k, E = len(T_list), 256, 4, 8
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, T_list, H, k, E, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    codes = [p.exitcode for p in procs]
    results = sorted(q.get(timeout=5) for _ in range(world))
    assert codes == [0] * world, codes
    assert all(ok for _, ok, _, _ in results), results
    # every routed entry was sent and received exactly once
    total_sent = sum(sum(s) for _, _, _, s in results)
    assert total_sent == sum(T_list) * k == sum(m for _, _, m, _ in results)


def test_send_row_layout():
    """A packed exchange row holds K codes then K/128 FP32 scales, padded to a
    multiple of 16 bytes (the exchange and the GPU copies move 16-byte units),
    and the two views read back what was written."""
    import torch
    from fine_grained_fp8_x128_b200.moe_dispatch import split_send_rows
    for K in (128, 256, 384, 512, 2048, 4224, 7168):
        w = send_row_bytes(K)
        assert w % 16 == 0 and K + 4 * (K // 128) <= w < K + 4 * (K // 128) + 16
        buf = torch.zeros((5, w), dtype=torch.uint8)
        q, sf = split_send_rows(buf, K)
        assert q.shape == (5, K) and sf.shape == (5, K // 128) and sf.dtype == torch.float32
        assert q.stride(0) == w and sf.stride(0) * 4 == w
        q[3] = 7
        sf[3] = 2.5
        row = buf[3].numpy()
        assert np.all(row[:K] == 7) and np.all(row[K:K + 4 * (K // 128)].view(np.float32) == 2.5)
        assert np.all(row[K + 4 * (K // 128):] == 0)
