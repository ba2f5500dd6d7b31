"""FP8 MoE dispatch across expert-parallel ranks.

"FP8 Mixed Precision: DeepSeek-V3 Training Architecture", section 4: tokens
sent to their experts' GPUs are quantized to FP8 on the fly, which halves the
all-to-all traffic.  One process per GPU; the experts are split into equal
contiguous ranges over the ranks of the process group.  One call:

  1. layout (device): a stable counting sort of the (token, slot) entries by
     expert, giving the send order -- expert-major, hence rank-major;
  2. quantize (device): each token's 1x128 FP8 codes and row-major scales,
     computed once and written straight to its rows of the send buffer --
     queued at once, since it needs only the layout's positions;
  3. all_gather of every rank's expert offsets, read on the host once (the
     one synchronisation of a call: the collective needs the split sizes);
     that one table gives both what this rank sends to each rank and what it
     receives per (source rank, local expert).  Without a process group
     nothing is exchanged: each token is quantized once and scattered to its
     rows of the grouped GEMM's input, and the host never waits;
  4. all_to_all_single of the codes and of the scales (NCCL over NVLink on
     GPUs);
  5. regroup (device): the received rows from (source, expert) order into
     (expert, source) order, the scales into the grouped GEMM's K-chunk-major
     layout, so that the grouped GEMM runs on the result directly.  The order
     is index arithmetic on the count table, uploaded from pinned memory
     without another synchronisation.

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
        """The send buffer: each token quantized once and written to its M-row
        layout positions, scales row-major so that they travel with their rows."""
        import torch
        from . import fp8q_quant_act_1x128_scatter_rowscales
        K = x.shape[1]
        q = torch.empty((M, K), dtype=torch.uint8, device=x.device)
        sf = torch.empty((M, K // 128), dtype=torch.float32, device=x.device)
        if M > 0 and x.shape[0] > 0:
            fp8q_quant_act_1x128_scatter_rowscales(x, pos, q, sf)
        return q, sf

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

    def regroup(self, q, sf, rows):
        import torch
        from . import fp8q_gather_rows_fp8, sf_ld
        M, K = rows.numel(), q.shape[1]
        q_out = torch.empty((M, K), dtype=torch.uint8, device=q.device)
        sf_out = torch.empty((K // 128, sf_ld(M)), dtype=torch.float32, device=q.device)
        if M > 0:
            fp8q_gather_rows_fp8(q, sf, rows, q_out, sf_out)
        return q_out, sf_out


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


_PINNED = {}


def _upload(a: np.ndarray, device):
    """int32 host array -> device, through a cached pinned buffer (no host
    synchronisation; the buffer is reused once its previous copy is done)."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a, np.int32))
    if torch.device(device).type != "cuda":
        return t.clone()
    buf, ev = _PINNED.get(str(device), (None, None))
    if buf is None or buf.numel() < t.numel():
        buf = torch.empty(max(t.numel(), 1 << 16), dtype=torch.int32, pin_memory=True)
        ev = None
    if ev is not None:
        ev.synchronize()                    # the last copy out of this buffer has finished
    buf[:t.numel()].copy_(t)
    out = buf[:t.numel()].to(device, non_blocking=True)
    ev = torch.cuda.Event()
    ev.record()
    _PINNED[str(device)] = (buf, ev)
    return out


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
    KB = H // 128
    rows, pos, offsets = ops.layout(expert_ids, num_experts)
    if not collective:
        # one process, all experts local: the layout order is the grouped GEMM's
        # order, so each token is quantized once and written to its rows of the
        # GEMM input, and nothing waits on the host
        q, sf = ops.quant_grouped(x, pos, expert_ids.numel())
        return DispatchResult(q=q, sf=sf, expert_offsets=offsets, pos=pos, send_counts=None, recv_counts=None)
    rank = dist.get_rank(group)
    q_send, sf_send = ops.quant_send(x, pos, expert_ids.numel())       # queued before the host waits
    gathered = [torch.empty_like(offsets) for _ in range(world)]
    dist.all_gather(gathered, offsets, group=group)
    off_all = torch.stack(gathered).cpu().numpy().astype(np.int64)     # the one host sync: every rank's offsets
    per_expert = np.diff(off_all, axis=1)                               # [source rank][expert]
    send_counts = per_expert[rank].reshape(world, el).sum(axis=1)
    recv_counts = np.ascontiguousarray(per_expert[:, rank * el:(rank + 1) * el])
    recv_rows = recv_counts.sum(axis=1)
    M = int(recv_rows.sum())
    q_recv = torch.empty((M, H), dtype=torch.uint8, device=x.device)
    sf_recv = torch.empty((M, KB), dtype=torch.float32, device=x.device)
    dist.all_to_all_single(q_recv, q_send, recv_rows.tolist(), send_counts.tolist(), group=group)
    dist.all_to_all_single(sf_recv, sf_send, recv_rows.tolist(), send_counts.tolist(), group=group)
    order, exp_off = regroup_order(recv_counts)
    both = _upload(np.concatenate([order, exp_off]), x.device)
    q, sf = ops.regroup(q_recv, sf_recv, both[:order.size])
    return DispatchResult(q=q, sf=sf, expert_offsets=both[order.size:], pos=pos,
                          send_counts=send_counts, recv_counts=recv_counts)
