"""FP8 MoE dispatch across expert-parallel ranks.

"FP8 Mixed Precision: DeepSeek-V3 Training Architecture", section 4: tokens
sent to their experts' GPUs are quantized to FP8 on the fly, which halves the
all-to-all traffic.  One process per GPU; the experts are split into equal
contiguous ranges over the ranks of the process group.  One call:

  1. layout (device): a stable counting sort of the (token, slot) entries by
     expert, giving the send order -- expert-major, hence rank-major;
  2. all_gather of every rank's expert offsets, copied to the host
     asynchronously;
  3. quantize (device): each token's 1x128 FP8 codes and scales, computed once
     and written straight to its rows of the send buffer; a send row holds the
     codes and then the row's scales, so one exchange moves both.  It is queued
     behind the copy of step 2, and the host waits only for that copy (the one
     synchronisation of a call: the collective needs the split sizes), so the
     quantizer runs while the host works out the splits.  The offsets table
     gives both what this rank sends to each rank and what it receives per
     (source rank, local expert).  Without a process group nothing is
     exchanged: each token is quantized once and scattered to its rows of the
     grouped GEMM's input, and the host never waits;
  4. all_to_all_single of the packed rows (NCCL over NVLink on GPUs);
  5. regroup (device): the received rows from (source, expert) order into
     (expert, source) order, the scales into the grouped GEMM's K-chunk-major
     layout, so that the grouped GEMM runs on the result directly.  The order
     is index arithmetic on the offsets table, done on the device from the
     all-gathered table itself (`regroup_order` is its host statement).

The device steps are this package's kernels (`CudaDispatchOps`).  The
collectives are torch.distributed's.  The host part -- split sizes and the
regroup order -- is plain index arithmetic on per-expert counts.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np


class CudaDispatchOps:
    """The device steps of a dispatch, on this package's CUDA kernels."""

    def layout(self, expert_ids, num_experts):
        from . import moe_dispatch_layout
        return moe_dispatch_layout(expert_ids, num_experts)

    def quant_send(self, x, pos, M):
        """The send buffer, uint8 [M][send_row_bytes(K)]: each token quantized
        once and written to its M-row layout positions; a row holds the K codes
        and then the row's K/128 FP32 scales, so they travel together."""
        import torch
        from . import fp8q_quant_act_1x128_scatter_rowscales
        K = x.shape[1]
        buf = torch.empty((M, send_row_bytes(K)), dtype=torch.uint8, device=x.device)
        q, sf = split_send_rows(buf, K)
        if M > 0 and x.shape[0] > 0:
            fp8q_quant_act_1x128_scatter_rowscales(x, pos, q, sf)
        return buf

    def quant_grouped(self, x, pos, M):
        """Without an exchange: the grouped GEMM's input directly (scales K-chunk-major),
        each token quantized once and written to its M-row layout positions."""
        import torch
        from . import fp8q_quant_act_1x128_scatter, sf_ld
        K = x.shape[1]
        q = torch.empty((M, K), dtype=torch.uint8, device=x.device)
        sf = torch.empty((K // 128, sf_ld(M)), dtype=torch.float32, device=x.device)
        if M > 0 and x.shape[0] > 0:
            fp8q_quant_act_1x128_scatter(x, pos, q, sf)
        return q, sf

    def regroup_order(self, all_off, world, rank, num_experts, M):
        """Device form of regroup_order from the all-gathered offsets table:
        (rows int32 [M], local expert offsets int32 [el + 1])."""
        import torch
        from . import fp8q_moe_regroup_order
        rows = torch.empty(M, dtype=torch.int32, device=all_off.device)
        off = torch.empty(num_experts // world + 1, dtype=torch.int32, device=all_off.device)
        fp8q_moe_regroup_order(all_off, world, rank, num_experts, rows, off)
        return rows, off

    def regroup(self, recv, K, rows):
        import torch
        from . import fp8q_gather_rows_fp8, sf_ld
        q, sf = split_send_rows(recv, K)
        M = rows.numel()
        q_out = torch.empty((M, K), dtype=torch.uint8, device=recv.device)
        sf_out = torch.empty((K // 128, sf_ld(M)), dtype=torch.float32, device=recv.device)
        if M > 0:
            fp8q_gather_rows_fp8(q, sf, rows, q_out, sf_out)
        return q_out, sf_out


def send_row_bytes(K: int) -> int:
    """Bytes of one exchanged row: K FP8 codes, then K/128 FP32 scales, padded
    to a multiple of 16 bytes."""
    return (K + 4 * (K // 128) + 15) // 16 * 16


def split_send_rows(buf, K: int):
    """Views of a packed row buffer: the codes uint8 [M][K] and the scales
    float32 [M][K/128] (both with the packed row stride)."""
    import torch
    return buf[:, :K], buf[:, K:K + 4 * (K // 128)].view(torch.float32)


def regroup_order(recv_counts: np.ndarray):
    """Received rows arrive source-major, each source's rows expert-major.
    Returns (rows, expert_offsets): the receive-buffer row of every output row
    in (local expert, source) order, and the local experts' row ranges."""
    recv_counts = np.asarray(recv_counts, np.int64)
    world, el = recv_counts.shape
    src_base = np.zeros(world + 1, np.int64)
    src_base[1:] = np.cumsum(recv_counts.sum(axis=1))
    within = np.zeros((world, el + 1), np.int64)
    within[:, 1:] = np.cumsum(recv_counts, axis=1)
    # piece (e, s) -- expert-major, source-minor -- is a run of receive rows
    # starting at src_base[s] + within[s, e]; output row i of a piece that
    # begins at output row o maps to its start + (i - o)
    cnt = recv_counts.T.reshape(-1)
    start = (src_base[:world, None] + within[:, :el]).T.reshape(-1)
    out_start = np.zeros(cnt.size, np.int64)
    out_start[1:] = np.cumsum(cnt)[:-1]
    total = int(cnt.sum())
    rows = (np.repeat(start - out_start, cnt) + np.arange(total, dtype=np.int64)).astype(np.int32)
    offsets = np.zeros(el + 1, np.int32)
    offsets[1:] = np.cumsum(recv_counts.sum(axis=0))
    return rows, offsets


@dataclass
class DispatchResult:
    q: object               # uint8 [M][H]: this rank's expert rows, expert-major then source rank
    sf: object              # float32 [H/128][ld >= M]: their 1x128 scales (grouped GEMM layout)
    expert_offsets: object  # int32 [E_local + 1] on the device: the grouped GEMM's group offsets
    pos: object             # int32 [T][k]: where each local (token, slot) entry went in the send order
    send_counts: np.ndarray  # int64 [world]: rows sent to each rank (None without a process group)
    recv_counts: np.ndarray  # int64 [world][E_local]: rows received per source rank and local expert (idem)


_HOST = {}


def _to_host(t):
    """Copies a small int32 device tensor to the host without waiting: returns
    (host tensor, wait), where wait() blocks until the copy is done.  The host
    buffer is pinned and kept per device; a dispatch reads it before it
    returns, so calls from one thread never overlap on it (concurrent
    dispatches from several host threads on one device would)."""
    import torch
    if t.device.type != "cuda":
        return t, lambda: None
    key = str(t.device)
    buf = _HOST.get(key)
    if buf is None or buf.numel() < t.numel():
        buf = torch.empty(max(t.numel(), 4096), dtype=t.dtype, pin_memory=True)
        _HOST[key] = buf
    out = buf[:t.numel()]
    out.copy_(t, non_blocking=True)
    ev = torch.cuda.Event()
    ev.record()
    return out, ev.synchronize


def dispatch(x, expert_ids, num_experts: int, group=None, ops=None) -> DispatchResult:
    """x: bf16 [T][H] (H % 128 == 0) on this rank's device; expert_ids: int32
    [T][k] on the same device.  Collective over `group`: every rank calls it."""
    import torch
    import torch.distributed as dist
    ops = ops or CudaDispatchOps()
    collective = dist.is_initialized()
    world = dist.get_world_size(group) if collective else 1
    if num_experts % world != 0:
        raise ValueError("num_experts must be a multiple of the group size")
    el = num_experts // world
    H = x.shape[1]
    rows, pos, offsets = ops.layout(expert_ids, num_experts)
    if not collective:
        # one process, all experts local: the layout order is the grouped GEMM's
        # order, so each token is quantized once and written to its rows of the
        # GEMM input, and nothing waits on the host
        q, sf = ops.quant_grouped(x, pos, expert_ids.numel())
        return DispatchResult(q=q, sf=sf, expert_offsets=offsets, pos=pos, send_counts=None, recv_counts=None)
    rank = dist.get_rank(group)
    all_off = torch.empty(world * (num_experts + 1), dtype=offsets.dtype, device=offsets.device)
    dist.all_gather_into_tensor(all_off, offsets, group=group)
    off_host, wait = _to_host(all_off)
    send = ops.quant_send(x, pos, expert_ids.numel())                  # runs while the host waits
    wait()                                                              # the one host sync: every rank's offsets
    off_all = off_host.numpy().astype(np.int64).reshape(world, num_experts + 1)
    per_expert = np.diff(off_all, axis=1)                               # [source rank][expert]
    send_counts = per_expert[rank].reshape(world, el).sum(axis=1)
    recv_counts = np.ascontiguousarray(per_expert[:, rank * el:(rank + 1) * el])
    recv_rows = recv_counts.sum(axis=1)
    M = int(recv_rows.sum())
    order, exp_off = ops.regroup_order(all_off, world, rank, num_experts, M)   # on the device, from the table
    recv = torch.empty((M, send.shape[1]), dtype=torch.uint8, device=x.device)
    dist.all_to_all_single(recv, send, recv_rows.tolist(), send_counts.tolist(), group=group)
    q, sf = ops.regroup(recv, H, order)
    return DispatchResult(q=q, sf=sf, expert_offsets=exp_off, pos=pos,
                          send_counts=send_counts, recv_counts=recv_counts)
