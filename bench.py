"""Benchmark: one training step of the fine-grained FP8 hot path on B200.

A step is one pass of every hot-path operation over one batch of synthetic,
seeded, outlier-injected input:
  dense linear layer, 8192 tokens x 7168 -> 18432 (forward and backward):
    quant_w_128x128(W, with W^T)           weights re-quantized once per step
    quant_act_dual(X): 1x128 and 128x1 from one read  -> Fprop  Y  = X W^T   (BF16 out)
    quant_act_dual(dY): 1x128 and 128x1 from one read -> Dgrad  dX = dY W    (BF16 out)
    Wgrad dW = dY^T X on both 128x1 quantizations     (FP32 out)
  MoE layer, 4096 tokens, top-8 of 256 experts (Zipf 1.1), hidden 7168, expert 2048:
    quant_act_1x128 of each token once, scattered to its 8 expert rows (the dispatch)
    grouped up-projection, epilogue emitting H as 1x128 FP8 tiles
    grouped down-projection (BF16 out)
Expert weights are resident FP8 (quantized once at set-up); the dense weight is
re-quantized inside every step.

value = GEMM FLOPs of the step / step time (TFLOP/s, whole job over all ranks).
With --gpus N (torchrun), every rank runs the same step on its own seeded batch
(weak scaling, no data-path collective); time = max over ranks.

--impl reference times the CPU oracle (the plain C++ statement of the method)
on a bounded sample of the same step; it is the deliberately slow baseline.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
LOG_DIR = os.environ.get("FP8Q_BENCH_LOG_DIR", os.path.join(ROOT, "bench_logs"))   # nvidia-smi clock samples
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "FP8 block-scaled GEMM TFLOP/s & % FP8 peak; quantizer GB/s & % HBM BW (1 B200)"
UNIT = "TFLOP/s"

# dense layer and MoE shapes
TOK, HID, OUT = 8192, 7168, 18432
MOE_TOK, MOE_E, MOE_K, MOE_FF = 4096, 256, 8, 2048

# fallbacks when MEASURED_PEAKS.json is absent (earlier measurement on this machine)
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
FP8_OVER_BF16 = 2.0          # nominal dense FP8 : BF16 tensor throughput (4.5 : 2.25 PFLOP/s)
# the problem statement's denominators, reported beside the measured ones
SPEC_HBM_GBS = 8000.0
SPEC_FP8_TFLOPS = 4500.0
# the problem statement's bars: quantizers >= 70 % of HBM, large GEMMs >= 60 % of dense FP8
BAR_QUANT_HBM = 0.70
BAR_GEMM_FP8 = 0.60


def gemm_flops():
    f = {
        "fprop": 2.0 * TOK * OUT * HID,
        "dgrad": 2.0 * TOK * HID * OUT,
        "wgrad": 2.0 * OUT * HID * TOK,
        "moe_up": 2.0 * MOE_TOK * MOE_K * MOE_FF * HID,
        "moe_down": 2.0 * MOE_TOK * MOE_K * HID * MOE_FF,
    }
    return f


def quant_bytes():
    """Algorithmic bytes of each quantizer launch: read BF16 + write E4M3 + write FP32 scales."""
    def act(m, k):
        return m * k * 2 + m * k + (m * k // 128) * 4
    def dual(m, k):   # one read, both orientations written (codes and scales twice)
        return m * k * 2 + 2 * m * k + 2 * (m * k // 128) * 4
    return {
        "quant_w": OUT * HID * 2 + 2 * OUT * HID + 2 * (OUT // 128) * (HID // 128) * 4,
        "quant_x": act(TOK, HID),
        "quant_dy": act(TOK, OUT),
        "quant_dy_t": act(TOK, OUT),
        "quant_x_t": act(TOK, HID),
        "quant_x_dual": dual(TOK, HID),
        "quant_dy_dual": dual(TOK, OUT),
        # the gather reads each token once from HBM (the 59 MB of tokens stay
        # in the L2 across their top-k copies) and writes every expert row
        "quant_moe_x": MOE_TOK * HID * 2 + MOE_TOK * MOE_K * HID + (MOE_TOK * MOE_K * HID // 128) * 4,
    }


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return dict(hbm=float(p["hbm_gbs"]), bf16=float(p["bf16_tflops"]),
                    bf16_sus=float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), src="measured")
    except Exception:
        return dict(hbm=FALLBACK_HBM_GBS, bf16=FALLBACK_BF16_TFLOPS, bf16_sus=1400.0, src="fallback")


def kernel_source_hash():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "fine_grained_fp8_x128_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel_key):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel sources (profiles/dram_traffic.txt: `key bytes srchash`)."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(path):
        return None
    cur = kernel_source_hash()
    for line in open(path):
        parts = line.split()
        if len(parts) >= 3 and not line.startswith("#") and parts[0] == kernel_key and parts[2] == cur:
            return float(parts[1])
    return None


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join(LOG_DIR, f"clocks_rank_gpu{gpu_index}.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "20"], stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
            return
        # nvidia-smi takes a few hundred ms to print its first sample: wait for it
        # (up to 2 s), so that the samples cover the whole timed region
        t_end = time.time() + 2.0
        while time.time() < t_end and self.proc.poll() is None:
            if os.path.getsize(self.path) > 0:
                break
            time.sleep(0.01)

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        sm, pw, smax, reasons = [], [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                clk, mx, w = float(parts[1]), float(parts[2]), float(parts[3])
            except ValueError:
                continue
            sm.append(clk)
            pw.append(w)
            smax = max(smax, mx)
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        # the median over the samples taken under load (power draw at least half the
        # run's peak): the samples before and after the timed kernels are idle
        sm, pw = np.array(sm), np.array(pw)
        load = pw >= 0.5 * pw.max()
        return {"sm_mhz": float(np.median(sm[load])), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": int(sm.size), "samples_under_load": int(load.sum()),
                "sm_mhz_min_under_load": float(sm[load].min()), "power_w_max": float(pw.max())}


# ----------------------------------------------------------------------------- distributed helpers
def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def init_dist(world, backend):
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Max of a per-rank float over all ranks (identity when world == 1)."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world, device=None):
    if world > 1:
        import torch.distributed as dist
        if device is not None and str(device).startswith("cuda"):
            dist.barrier(device_ids=[int(str(device).split(":")[1])])
        else:
            dist.barrier()


def rank_seed(rank: int) -> int:
    """Each rank draws its own batch (weak scaling): seed = rank."""
    return int(rank)


# ----------------------------------------------------------------------------- CPU oracle sample
class CpuSample:
    """A bounded sample of the step for the oracle: R full output rows of every
    GEMM of the step, with every quantization those rows need (the dense weight
    and W^T in full, X^T in full for Wgrad, the owning experts' weights)."""

    def __init__(self, rows: int, seed: int):
        self.R = rows
        self.seed = seed
        self.x_rows = W.activations_with_outliers(rows, HID, seed=seed + 100)
        self.w = W.weights(OUT, HID, seed=seed)
        self.wt = np.ascontiguousarray(self.w.T)
        self.dy_rows = W.grad_with_outlier_tokens(rows, OUT, seed=seed + 100)
        self.x_full = W.activations_with_outliers(TOK, HID, seed=seed)
        self.dy_cols = W.grad_with_outlier_tokens(TOK, 128, seed=seed + 200)[:, :rows].copy() \
            if rows <= 128 else W.grad_with_outlier_tokens(TOK, rows, seed=seed + 200)
        route = W.moe_routing(seed=seed)
        pick = np.random.default_rng(seed).choice(int(route.offsets[-1]), size=rows, replace=False)
        exp_of_row = np.searchsorted(route.offsets, pick, side="right") - 1
        self.experts = np.unique(exp_of_row)
        self.moe_x = W.activations_with_outliers(rows, HID, seed=seed + 300)
        self.exp_local = np.searchsorted(self.experts, exp_of_row)
        self.w_up = W.expert_weights(len(self.experts), MOE_FF, HID, seed=seed, tid=W.TID_EXPERT_UP,
                                     experts=self.experts)
        self.w_dn = W.expert_weights(len(self.experts), HID, MOE_FF, seed=seed, tid=W.TID_EXPERT_DN,
                                     experts=self.experts)
        # rows sorted by expert so each expert owns a contiguous range
        order = np.argsort(self.exp_local, kind="stable")
        self.moe_x, self.exp_local = self.moe_x[order], self.exp_local[order]
        self.moe_off = W.ragged_offsets(np.bincount(self.exp_local, minlength=len(self.experts)))

    def flops(self):
        R = self.R
        return 2.0 * R * (OUT * HID + HID * OUT + HID * TOK + MOE_FF * HID + HID * MOE_FF)

    def description(self):
        return (f"{self.R} full output rows of each of the 5 GEMMs of the step (Fprop, Dgrad, Wgrad, MoE up, "
                f"MoE down) with the quantizations they need (W and W^T 18432x7168 in full, X^T 8192x7168 in "
                f"full for Wgrad, {len(self.experts)} experts' up/down weights, the up projection's BF16 rows "
                f"re-quantized 1x128 as the down projection's input)")

    def run(self):
        import oracle
        R = self.R
        qx, sx = oracle.quant_act_1x128(self.x_rows)
        qw, sw = oracle.quant_w_128x128(self.w)
        oracle.gemm_sampled(qx, sx, qw, sw, oracle.SFB_BLOCK128)
        qdy, sdy = oracle.quant_act_1x128(self.dy_rows)
        qwt, swt = oracle.quant_w_128x128(self.wt)
        oracle.gemm_sampled(qdy, sdy, qwt, swt, oracle.SFB_BLOCK128)
        qdyt, sdyt = oracle.quant_act_128x1(self.dy_cols)
        qxt, sxt = oracle.quant_act_128x1(self.x_full)
        oracle.gemm_sampled(qdyt, np.ascontiguousarray(sdyt.T), qxt, np.ascontiguousarray(sxt.T), oracle.SFB_ROW)
        qa, sa = oracle.quant_act_1x128(self.moe_x)
        G = len(self.experts)
        wq = np.empty((G, MOE_FF, HID), np.uint8); ws = np.empty((G, MOE_FF // 128, HID // 128), np.float32)
        for g in range(G):
            wq[g], ws[g] = oracle.quant_w_128x128(self.w_up[g])
        h = oracle.grouped_gemm_sampled(qa, sa, wq, ws, self.moe_off)
        qh, sh = oracle.quant_act_1x128(W.f32_to_bf16_bits(oracle.round_bf16(h).astype(np.float32)))
        wq = np.empty((G, HID, MOE_FF), np.uint8); ws = np.empty((G, HID // 128, MOE_FF // 128), np.float32)
        for g in range(G):
            wq[g], ws[g] = oracle.quant_w_128x128(self.w_dn[g])
        oracle.grouped_gemm_sampled(qh, sh, wq, ws, self.moe_off)
        return R


def time_cpu_sample(sample: CpuSample):
    import oracle
    oracle.reset_threads_used()
    t0 = time.perf_counter()
    sample.run()
    dt = time.perf_counter() - t0
    return {"value": sample.flops() / dt / 1e12, "unit": UNIT, "cores": oracle.threads_used(), "kind": "oracle",
            "sample": sample.description(), "seconds": dt, "host_threads": oracle.host_threads()}


# ----------------------------------------------------------------------------- the device step
class DeviceStep:
    """All buffers of one step, resident on the device; step() launches the 9
    kernels of the hot path on the current stream."""

    KERNELS = ("quant_w", "quant_x_dual", "fprop", "quant_dy_dual", "dgrad", "wgrad", "quant_moe_x", "moe_up",
               "moe_down")

    def __init__(self, fp8q, seed: int, device):
        import torch
        self.fp8q = fp8q
        self.dev = device
        bf = torch.bfloat16
        u8 = torch.uint8
        f32 = torch.float32
        ld = fp8q.sf_ld

        def dev_bf16(bits):
            return torch.from_numpy(bits.view(np.int16)).to(device).view(bf)

        # host inputs of the step (pinned) and their device copies
        self.h_x = torch.from_numpy(W.activations_with_outliers(TOK, HID, seed=seed).view(np.int16)).view(bf).pin_memory()
        self.h_dy = torch.from_numpy(W.grad_with_outlier_tokens(TOK, OUT, seed=seed).view(np.int16)).view(bf).pin_memory()
        route = W.moe_routing(tokens=MOE_TOK, experts=MOE_E, top_k=MOE_K, seed=seed)
        self.mt = int(route.offsets[-1])
        xt = W.activations_with_outliers(MOE_TOK, HID, seed=seed, tid=W.TID_MISC)
        self.h_xm = torch.from_numpy(xt.view(np.int16)).view(bf).pin_memory()       # MoE tokens, token order
        self.h_pos = torch.from_numpy(route.entry_row.astype(np.int32)).pin_memory()   # (token, pick) -> expert row
        self.h_off = torch.from_numpy(route.offsets.astype(np.int32)).pin_memory()
        self.w = dev_bf16(W.weights(OUT, HID, seed=seed))                      # model state, resident
        self.x = torch.empty((TOK, HID), dtype=bf, device=device)
        self.dy = torch.empty((TOK, OUT), dtype=bf, device=device)
        self.xm = torch.empty((MOE_TOK, HID), dtype=bf, device=device)
        self.pos = torch.empty((MOE_TOK, MOE_K), dtype=torch.int32, device=device)
        self.off = torch.empty((MOE_E + 1,), dtype=torch.int32, device=device)
        self.upload()
        # quantized operands and outputs
        self.wq = torch.empty((OUT, HID), dtype=u8, device=device)
        self.sw = torch.empty((OUT // 128, HID // 128), dtype=f32, device=device)
        self.wqt = torch.empty((HID, OUT), dtype=u8, device=device)
        self.swt = torch.empty((HID // 128, OUT // 128), dtype=f32, device=device)
        self.xq = torch.empty((TOK, HID), dtype=u8, device=device)
        self.sx = torch.empty((HID // 128, ld(TOK)), dtype=f32, device=device)
        self.y = torch.empty((TOK, OUT), dtype=bf, device=device)
        self.dyq = torch.empty((TOK, OUT), dtype=u8, device=device)
        self.sdy = torch.empty((OUT // 128, ld(TOK)), dtype=f32, device=device)
        self.dx = torch.empty((TOK, HID), dtype=bf, device=device)
        self.dyqt = torch.empty((OUT, TOK), dtype=u8, device=device)
        self.sdyt = torch.empty((TOK // 128, ld(OUT)), dtype=f32, device=device)
        self.xqt = torch.empty((HID, TOK), dtype=u8, device=device)
        self.sxt = torch.empty((TOK // 128, ld(HID)), dtype=f32, device=device)
        self.dw = torch.empty((OUT, HID), dtype=f32, device=device)
        # MoE: resident FP8 expert weights, quantized once here with the library
        self.wup_q = torch.empty((MOE_E, MOE_FF, HID), dtype=u8, device=device)
        self.wup_s = torch.empty((MOE_E, MOE_FF // 128, HID // 128), dtype=f32, device=device)
        self.wdn_q = torch.empty((MOE_E, HID, MOE_FF), dtype=u8, device=device)
        self.wdn_s = torch.empty((MOE_E, HID // 128, MOE_FF // 128), dtype=f32, device=device)
        for (q, s, n, k, tid) in ((self.wup_q, self.wup_s, MOE_FF, HID, W.TID_EXPERT_UP),
                                  (self.wdn_q, self.wdn_s, HID, MOE_FF, W.TID_EXPERT_DN)):
            wb = W.expert_weights_device(MOE_E, n, k, seed=seed, tid=tid, device=device)
            for g in range(MOE_E):
                fp8q.fp8q_quant_w_128x128(wb[g], q[g], s[g])
            del wb
        self.xpq = torch.empty((self.mt, HID), dtype=u8, device=device)
        self.sxp = torch.empty((HID // 128, ld(self.mt)), dtype=f32, device=device)
        self.hq = torch.empty((self.mt, MOE_FF), dtype=u8, device=device)
        self.sh = torch.empty((MOE_FF // 128, ld(self.mt)), dtype=f32, device=device)
        self.out = torch.empty((self.mt, HID), dtype=bf, device=device)
        # pinned host outputs for the end-to-end leg
        self.h_y = torch.empty_like(self.y, device="cpu").pin_memory()
        self.h_dx = torch.empty_like(self.dx, device="cpu").pin_memory()
        self.h_dw = torch.empty_like(self.dw, device="cpu").pin_memory()
        self.h_out = torch.empty_like(self.out, device="cpu").pin_memory()
        # the end-to-end leg double-buffers the step's inputs and outputs so that
        # the copies of neighbouring steps overlap this step's kernels
        self.slots = [self._slot_tensors()]
        self.slots.append({k: torch.empty_like(v) for k, v in self.slots[0].items()})
        torch.cuda.synchronize()

    _SLOT = ("x", "dy", "xm", "pos", "off", "y", "dx", "dw", "out")

    def _slot_tensors(self):
        return {k: getattr(self, k) for k in self._SLOT}

    def use_slot(self, b):
        for k, v in self.slots[b].items():
            setattr(self, k, v)

    def h2d_bytes(self):
        return sum(t.numel() * t.element_size() for t in (self.h_x, self.h_dy, self.h_xm, self.h_pos, self.h_off))

    def d2h_bytes(self):
        return sum(t.numel() * t.element_size() for t in (self.h_y, self.h_dx, self.h_dw, self.h_out))

    def upload(self):
        self.x.copy_(self.h_x, non_blocking=True)
        self.dy.copy_(self.h_dy, non_blocking=True)
        self.xm.copy_(self.h_xm, non_blocking=True)
        self.pos.copy_(self.h_pos, non_blocking=True)
        self.off.copy_(self.h_off, non_blocking=True)

    def download(self):
        self.h_y.copy_(self.y, non_blocking=True)
        self.h_dx.copy_(self.dx, non_blocking=True)
        self.h_dw.copy_(self.dw, non_blocking=True)
        self.h_out.copy_(self.out, non_blocking=True)

    def step(self, events=None):
        """Launch the 9 kernels; if `events` is a list, append (name, start, end) CUDA events."""
        import torch
        f = self.fp8q
        ops = (
            ("quant_w", lambda: f.fp8q_quant_w_128x128(self.w, self.wq, self.sw, self.wqt, self.swt)),
            # X in 1x128 tiles (Fprop) and 128x1 tiles (Wgrad) from one read
            ("quant_x_dual", lambda: f.fp8q_quant_act_dual(self.x, self.xq, self.sx, self.xqt, self.sxt)),
            ("fprop", lambda: f.fp8q_gemm_blockscaled(self.xq, self.sx, self.wq, self.sw, f.FP8Q_SFB_BLOCK128, self.y)),
            # dY in 1x128 tiles (Dgrad) and 128x1 tiles (Wgrad) from one read
            ("quant_dy_dual", lambda: f.fp8q_quant_act_dual(self.dy, self.dyq, self.sdy, self.dyqt, self.sdyt)),
            ("dgrad", lambda: f.fp8q_gemm_blockscaled(self.dyq, self.sdy, self.wqt, self.swt, f.FP8Q_SFB_BLOCK128,
                                                      self.dx)),
            ("wgrad", lambda: f.fp8q_gemm_blockscaled(self.dyqt, self.sdyt, self.xqt, self.sxt, f.FP8Q_SFB_ROW,
                                                      self.dw)),
            ("quant_moe_x", lambda: f.fp8q_quant_act_1x128_scatter(self.xm, self.pos, self.xpq, self.sxp)),
            ("moe_up", lambda: f.fp8q_grouped_gemm_blockscaled_q1x128(self.xpq, self.sxp, self.wup_q, self.wup_s,
                                                                      self.off, self.hq, self.sh)),
            ("moe_down", lambda: f.fp8q_grouped_gemm_blockscaled(self.hq, self.sh, self.wdn_q, self.wdn_s, self.off,
                                                                 self.out)),
        )
        for name, fn in ops:
            if events is None:
                fn()
            else:
                s = torch.cuda.Event(enable_timing=True)
                e = torch.cuda.Event(enable_timing=True)
                s.record()
                fn()
                e.record()
                events.append((name, s, e))
        return len(ops)


# ----------------------------------------------------------------------------- reporting
def config_block(world):
    return {
        "workload": ("one training step of a 8192-token linear layer 7168->18432 (weight quant with W^T, "
                     "X and dY each quantized 1x128 and 128x1 from one read, Fprop, Dgrad, Wgrad with "
                     "1x128 / 128x1 / 128x128 quantization) plus a 4096-token MoE "
                     "layer (top-8 of 256 experts, Zipf 1.1, 8 empty; dispatch gather fused into the 1x128 "
                     "quantizer, grouped up 7168->2048 with FP8 epilogue, grouped down 2048->7168)"),
        "tokens": TOK, "hidden": HID, "out_features": OUT,
        "moe_tokens": MOE_TOK, "experts": MOE_E, "top_k": MOE_K, "expert_ffn": MOE_FF,
        "tile": "1x128 activations, 128x1 (Wgrad), 128x128 weights; promotion every 128 of K",
        "l2": "inputs larger than L2: every step streams > 9 GB (7.5 GB of FP8 expert weights alone)",
        "ranks": world,
    }


def kernel_stats(events, K):
    import collections
    tot = collections.defaultdict(float)
    cnt = collections.defaultdict(int)
    for name, s, e in events:
        tot[name] += s.elapsed_time(e) * 1e-3
        cnt[name] += 1
    return {n: (tot[n] / cnt[n], tot[n]) for n in tot}


def fp8_peak_for_clock(pk, clk, kernel_mhz=None):
    """The measured FP8 denominator that matches the run's clock record: the
    burst figure (2 x the burst BF16 GEMM) when the SM clock stayed at its
    maximum, the sustained one (2 x the seconds-long BF16 loop at the power
    cap) otherwise.  The clock taken is the one measured inside the GEMM
    kernels (kernel_mhz, cycles over global-timer nanoseconds) when there is
    one -- under FP8 load the clock drops to the power limit between
    nvidia-smi's samples -- else the sampled median.  Returns (TFLOP/s,
    description)."""
    smax = (clk or {}).get("sm_max_mhz") or 0.0
    if kernel_mhz is not None:
        mhz, what = kernel_mhz, "SM clock inside the GEMM kernels"
    elif clk is not None:
        mhz, what = clk["sm_mhz"], "median sampled SM clock"
    else:
        mhz, what = None, None
    if mhz is not None and smax and mhz >= 0.97 * smax:
        return pk["bf16"] * FP8_OVER_BF16, (f"{pk['src']} MEASURED_PEAKS.json burst BF16 TFLOP/s x 2 (nominal "
                                            f"FP8:BF16 ratio); {what} {mhz:.0f} MHz = max")
    why = "no clock record" if mhz is None else f"{what} {mhz:.0f} MHz below the {smax:.0f} MHz max"
    return pk["bf16_sus"] * FP8_OVER_BF16, (f"{pk['src']} MEASURED_PEAKS.json sustained BF16 TFLOP/s x 2 "
                                            f"(nominal FP8:BF16 ratio); {why}")


def gemm_kernel_mhz(name, kclk):
    """The in-kernel SM clock of the kernel kind that runs a step GEMM."""
    if not kclk:
        return None
    kind = "one_cta" if name.startswith("moe") else "pair"
    return kclk.get(kind, {}).get("mhz")


def build_breakdown(stats, pk, moe_w_bytes, moe_other_bytes, clk=None, kclk=None):
    fl = gemm_flops()
    qb = quant_bytes()
    out = {}
    for name, (avg, total) in stats.items():
        ent = {"avg_us": round(avg * 1e6, 2), "share": None}
        if name in qb:
            gbs = qb[name] / avg / 1e9
            ent.update(bytes=qb[name], gbps=round(gbs, 1), frac_hbm=round(gbs / pk["hbm"], 3),
                       frac_hbm_spec=round(gbs / SPEC_HBM_GBS, 3),
                       bar_70pct_hbm_spec=bool(gbs / SPEC_HBM_GBS >= BAR_QUANT_HBM))
        if name in fl:
            tf = fl[name] / avg / 1e12
            fp8_peak, _ = fp8_peak_for_clock(pk, clk, gemm_kernel_mhz(name, kclk))
            ent.update(flops=fl[name], tflops=round(tf, 1), frac_fp8=round(tf / fp8_peak, 3),
                       frac_fp8_burst=round(tf / (pk["bf16"] * FP8_OVER_BF16), 3),
                       frac_fp8_spec=round(tf / SPEC_FP8_TFLOPS, 3))
            if gemm_kernel_mhz(name, kclk) is not None:
                ent.update(kernel_sm_mhz=gemm_kernel_mhz(name, kclk))
            if name.startswith("moe"):
                b = moe_w_bytes + moe_other_bytes[name]
                ent.update(bytes=b, gbps=round(b / avg / 1e9, 1), frac_hbm=round(b / avg / 1e9 / pk["hbm"], 3),
                           frac_hbm_spec=round(b / avg / 1e9 / SPEC_HBM_GBS, 3))
            else:
                ent.update(bar_60pct_fp8_spec=bool(tf / SPEC_FP8_TFLOPS >= BAR_GEMM_FP8))
        out[name] = ent
    grand = sum(t for _, t in stats.values())
    for name, (avg, total) in stats.items():
        out[name]["share"] = round(total / grand, 4)
    return out


def roofline_for(name, stats, pk, breakdown, clk=None, kclk=None):
    avg, _ = stats[name]
    ent = breakdown[name]
    if name.startswith("moe") or name.startswith("quant"):
        achieved = ent["bytes"] / avg / 1e9
        peak, spec = pk["hbm"], SPEC_HBM_GBS
        bound, unit = "hbm", "GB/s"
        src = f"{pk['src']} MEASURED_PEAKS.json: HBM copy GB/s"
    else:
        achieved = ent["flops"] / avg / 1e12
        peak, src = fp8_peak_for_clock(pk, clk, gemm_kernel_mhz(name, kclk))
        spec = SPEC_FP8_TFLOPS
        bound, unit = "tensor", "TFLOP/s"
    out = {"kernel": name, "bound": bound, "achieved": round(achieved, 1), "peak": round(peak, 1), "unit": unit,
           "frac": round(achieved / peak, 4), "traffic": recorded_traffic(name), "peak_source": src,
           "spec_peak": spec, "frac_spec": round(achieved / spec, 4)}
    if bound == "tensor":
        out["frac_burst"] = round(achieved / (pk["bf16"] * FP8_OVER_BF16), 4)
    return out


def linear_y_wx_latency(fp8q, device, reps=50):
    """The single linear layer y = Wx of "Introduction to LLM Quantization",
    "1. Mixed Precision Quantization" (x 1x128 with the outlier 20.0 at index
    17, W 256x128): median microseconds of the whole path on the device -- x
    quantized in one 1x128 tile, W in two 128x128 blocks, the block-scaled GEMM
    with BF16 out (three launches), inputs resident, CUDA events."""
    import torch
    x, w = W.linear_1x128_inputs(seed=0)

    def dev_bf16(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device).view(torch.bfloat16)

    xd, wd = dev_bf16(x), dev_bf16(w)
    qx = torch.empty((1, 128), dtype=torch.uint8, device=device)
    sx = torch.empty((1, fp8q.sf_ld(1)), dtype=torch.float32, device=device)
    qw = torch.empty((256, 128), dtype=torch.uint8, device=device)
    sw = torch.empty((2, 1), dtype=torch.float32, device=device)
    y = torch.empty((1, 256), dtype=torch.bfloat16, device=device)

    def path():
        fp8q.fp8q_quant_act_1x128(xd, qx, sx)
        fp8q.fp8q_quant_w_128x128(wd, qw, sw)
        fp8q.fp8q_gemm_blockscaled(qx, sx, qw, sw, fp8q.FP8Q_SFB_BLOCK128, y)

    for _ in range(5):
        path()
    torch.cuda.synchronize()
    times = []
    for _ in range(reps):
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        path()
        e.record()
        torch.cuda.synchronize()
        times.append(s.elapsed_time(e) * 1e3)
    return round(float(np.median(times)), 2)


def run_fp8q(args):
    import torch
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    device = f"cuda:{local}"
    init_dist(world, "nccl")
    if rank == 0:
        import importlib.util
        spec = importlib.util.spec_from_file_location(
            "fp8q_build", os.path.join(ROOT, "fine_grained_fp8_x128_b200", "build.py"))
        _b = importlib.util.module_from_spec(spec)
        spec.loader.exec_module(_b)
        _b.build()
    barrier(world, device)
    import fine_grained_fp8_x128_b200 as fp8q

    pk = peaks()
    st = DeviceStep(fp8q, rank_seed(rank), device)
    flops_step = sum(gemm_flops().values())
    for _ in range(args.warmup):
        st.step()
    torch.cuda.synchronize()
    code = fp8q.fp8q_device_status()
    if code != 0:
        raise RuntimeError(f"device status 0x{code:x} after warm-up")

    # ---- device-resident timed region
    fp8q.fp8q_kernel_clock_counters(reset=True)
    uuid = "GPU-" + str(torch.cuda.get_device_properties(local).uuid)
    clocks = ClockSampler(uuid)
    clocks.path = os.path.join(LOG_DIR, f"clocks_rank{rank}.csv")
    barrier(world, device)
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    events = []
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    launches = 0
    t0.record()
    for _ in range(args.steps):
        launches += st.step(events)
    t1.record()
    torch.cuda.synchronize()
    clk = clocks.stop()
    kclk = fp8q.fp8q_kernel_clock_counters(reset=True)   # the SM clock inside the GEMM kernels
    if clk is not None:
        clk["gemm_kernel_sm_mhz"] = {k: v["mhz"] for k, v in kclk.items()}
    barrier(world, device)
    elapsed = t0.elapsed_time(t1) * 1e-3
    t_max = max_over_ranks(elapsed, world, device)
    value = world * flops_step * args.steps / t_max / 1e12
    stats = kernel_stats(events, args.steps)

    # ---- end-to-end: host inputs in, host outputs back, through the public API.
    # Every step uploads its inputs and downloads its outputs inside the timed
    # region; with two buffer sets, step i+1's upload and step i-1's download
    # run on their own streams while step i's kernels run.
    barrier(world, device)
    torch.cuda.synchronize()
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()
    in_ready, comp_done, out_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(comp)

    def upload_into(b, after=None):
        with torch.cuda.stream(s_in):
            s_in.wait_event(e0)
            if after is not None:
                s_in.wait_event(after)      # the slot's previous step has finished reading it
            st.use_slot(b)
            st.upload()
            in_ready[b].record(s_in)

    upload_into(0)
    for i in range(args.steps):
        b = i % 2
        if i + 1 < args.steps:
            upload_into(b ^ 1, comp_done[b ^ 1] if i >= 1 else None)
        comp.wait_event(in_ready[b])
        if i >= 2:
            comp.wait_event(out_done[b])    # step i-2's outputs have left this slot
        st.use_slot(b)
        st.step()
        comp_done[b].record(comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(comp_done[b])
            st.download()
            out_done[b].record(s_out)
    comp.wait_event(out_done[(args.steps - 1) % 2])
    if args.steps >= 2:
        comp.wait_event(out_done[args.steps % 2])
    e1.record(comp)
    torch.cuda.synchronize()
    st.use_slot(0)
    e2e_t = max_over_ranks(e0.elapsed_time(e1) * 1e-3, world, device)
    e2e_value = world * flops_step * args.steps / e2e_t / 1e12
    code = fp8q.fp8q_device_status()
    if code != 0:
        raise RuntimeError(f"device status 0x{code:x} after the timed region")

    nz = int((st.h_off[1:] - st.h_off[:-1] > 0).sum())
    moe_w = nz * MOE_FF * HID + nz * (MOE_FF // 128) * (HID // 128) * 4
    mt = st.mt
    moe_other = {"moe_up": mt * HID + (HID // 128) * mt * 4 + mt * MOE_FF + (MOE_FF // 128) * mt * 4,
                 "moe_down": mt * MOE_FF + (MOE_FF // 128) * mt * 4 + mt * HID * 2}
    breakdown = build_breakdown(stats, pk, moe_w, moe_other, clk, kclk)
    dominant = max(stats, key=lambda n: stats[n][1])
    roof = roofline_for(dominant, stats, pk, breakdown, clk, kclk)
    latency = {"linear_y_wx_us": linear_y_wx_latency(fp8q, device)}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = time_cpu_sample(CpuSample(args.cpu_rows, seed=0))

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(t_max / args.steps * 1e3, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "fp8_e4m3", "data": "synthetic",
            "config": config_block(world),
            "roofline": roof,
            "cpu_baseline": cpu,
            "e2e": {"value": round(e2e_value, 3), "unit": UNIT, "h2d_bytes_per_step": st.h2d_bytes(),
                    "d2h_bytes_per_step": st.d2h_bytes()},
            "gpu_launches": launches,
            "clocks": clk,
            "breakdown": breakdown,
            "latency": latency,
            "impl": "fp8q",
        }
        print(json.dumps(line), flush=True)
    del st
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_reference(args):
    rank, world, local = dist_env()
    if rank != 0:
        return
    sample = CpuSample(args.ref_rows, seed=0)
    for _ in range(args.warmup):
        sample.run()
    import oracle
    oracle.reset_threads_used()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        sample.run()
    dt = time.perf_counter() - t0
    value = sample.flops() * args.steps / dt / 1e12
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_block(world), "impl": "reference",
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.threads_used(), "kind": "oracle",
                         "sample": "each step: " + sample.description()},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- single-kernel timing
SINGLE_KERNELS = ("linear_y_wx", "mx_fprop", "fprop_single", "quant_x_dual", "quant_dy_dual", "quant_dy",
                  "quant_dy_t", "quant_x_ue8m0", "quant_w_ue8m0", "quant_x", "quant_x_scaled", "quant_x_pct", "quant_x_pt", "pt_fprop", "quant_x_t", "requant_x_t", "quant_dy_e5m2", "dgrad_e5m2", "moe_dispatch", "moe_dispatch_nccl", "moe_layout", "quant_w", "fprop", "dgrad", "wgrad", "quant_moe_x", "quant_moe_x_gather", "moe_up", "moe_up_q",
                  "moe_down")


def run_single(args):
    """Time one kernel of the step in isolation (for A/B comparisons and ncu
    captures): --tokens scales the token dimension; weights keep their sizes."""
    import torch
    import fine_grained_fp8_x128_b200 as fp8q
    dev = "cuda:0"
    torch.cuda.set_device(0)
    gen = torch.Generator(device=dev)
    gen.manual_seed(1234)
    T = args.tokens

    def randn(*shape, sigma=1.0):
        return (torch.randn(shape, generator=gen, device=dev) * sigma).to(torch.bfloat16)

    name = args.single
    ld = fp8q.sf_ld
    u8, f32, bf = torch.uint8, torch.float32, torch.bfloat16
    work = None
    if name == "linear_y_wx":
        # the y = Wx worked example: quantize x (one 1x128 tile) and W (two 128x128 blocks), GEMM, BF16 out
        x, w = W.linear_1x128_inputs(seed=0)
        xd = torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).to(dev).view(bf)
        wd = torch.from_numpy(np.ascontiguousarray(w).view(np.int16)).to(dev).view(bf)
        qx = torch.empty((1, 128), dtype=u8, device=dev); sx = torch.empty((1, ld(1)), dtype=f32, device=dev)
        qw = torch.empty((256, 128), dtype=u8, device=dev); sw = torch.empty((2, 1), dtype=f32, device=dev)
        y = torch.empty((1, 256), dtype=bf, device=dev)

        def fn():
            fp8q.fp8q_quant_act_1x128(xd, qx, sx)
            fp8q.fp8q_quant_w_128x128(wd, qw, sw)
            fp8q.fp8q_gemm_blockscaled(qx, sx, qw, sw, fp8q.FP8Q_SFB_BLOCK128, y)
        work = ("flops", 2.0 * 256 * 128)
    elif name == "mx_fprop":
        # power-of-two (UE8M0) scale study: the Fprop shape on the block-scaled MMA, all of K in TMEM
        M, N, K = T, OUT, HID
        qa, sfa = fp8q.quant_act_1x128_ue8m0(randn(M, K))
        qb, sfb = fp8q.quant_w_128x128_ue8m0(randn(N, K, sigma=0.02))
        d = torch.empty((M, N), dtype=bf, device=dev)
        fn = lambda: fp8q.fp8q_gemm_mxf8_ue8m0(qa, sfa, qb, sfb, d)
        work = ("flops", 2.0 * M * N * K)
    elif name in ("quant_x_ue8m0", "quant_w_ue8m0"):
        # power-of-two (UE8M0) scale study: the quantizers writing scale atoms
        if name == "quant_x_ue8m0":
            x = randn(T, HID)
            q = torch.empty((T, HID), dtype=u8, device=dev)
            sf = torch.empty((HID // 128, (T + 127) // 128, 128), dtype=torch.int32, device=dev)
            fn = lambda: fp8q.fp8q_quant_act_1x128_ue8m0(x, q, sf)
            work = ("bytes", T * HID * 3 + T * HID // 128 * 4)
        else:
            w = randn(OUT, HID, sigma=0.02)
            q = torch.empty((OUT, HID), dtype=u8, device=dev)
            sf = torch.empty((HID // 128, OUT // 128, 128), dtype=torch.int32, device=dev)
            fn = lambda: fp8q.fp8q_quant_w_128x128_ue8m0(w, q, sf)
            work = ("bytes", OUT * HID * 3 + OUT * HID // 128 * 4)
    elif name in ("quant_x_dual", "quant_dy_dual", "quant_dy", "quant_dy_t"):
        # both orientations from one read (dual), or the gradient's single-orientation passes
        C = HID if name == "quant_x_dual" else OUT
        x = randn(T, C) if name == "quant_x_dual" else randn(T, C, sigma=1e-3)
        q = torch.empty((T, C), dtype=u8, device=dev); sf = torch.empty((C // 128, ld(T)), dtype=f32, device=dev)
        qt = torch.empty((C, T), dtype=u8, device=dev); sft = torch.empty((T // 128, ld(C)), dtype=f32, device=dev)
        if name == "quant_dy":
            fn = lambda: fp8q.fp8q_quant_act_1x128(x, q, sf)
            work = ("bytes", T * C * 3 + T * C // 128 * 4)
        elif name == "quant_dy_t":
            fn = lambda: fp8q.fp8q_quant_act_128x1(x, qt, sft)
            work = ("bytes", T * C * 3 + T * C // 128 * 4)
        else:
            fn = lambda: fp8q.fp8q_quant_act_dual(x, q, sf, qt, sft)
            work = ("bytes", T * C * 4 + 2 * (T * C // 128) * 4)
    elif name == "quant_x_pt":
        # per-tensor baseline quantizer: amax pass + cast pass (reads x twice)
        x = randn(T, HID)
        q = torch.empty((T, HID), dtype=u8, device=dev)
        amax_scale = torch.empty(2, dtype=f32, device=dev)
        fn = lambda: fp8q.fp8q_quant_pertensor(x, q, amax_scale)
        work = ("bytes", T * HID * 3)
    elif name in ("moe_dispatch", "moe_dispatch_nccl", "moe_layout"):
        # FP8 MoE dispatch on one GPU: without a process group (layout + gather-quantize
        # into the grouped GEMM's input), through a one-rank NCCL group (layout, host sync
        # for the split sizes, gather-quantize, all_to_all_single, regroup), or the layout alone
        from fine_grained_fp8_x128_b200.moe_dispatch import dispatch
        moe_tokens = MOE_TOK if T == TOK else T
        xm = randn(moe_tokens, HID)
        ids = torch.from_numpy(W.moe_routing(tokens=moe_tokens, experts=MOE_E, top_k=MOE_K, seed=0).expert_ids
                               .astype(np.int32)).to(dev)
        if name == "moe_layout":
            fn = lambda: fp8q.moe_dispatch_layout(ids, MOE_E)
            work = ("bytes", moe_tokens * MOE_K * 4 * 4)
        else:
            if name == "moe_dispatch_nccl":
                import socket
                import torch.distributed as dist
                sock = socket.socket()
                sock.bind(("127.0.0.1", 0))
                os.environ["MASTER_ADDR"] = "127.0.0.1"
                os.environ["MASTER_PORT"] = str(sock.getsockname()[1])
                sock.close()
                dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device(dev))
            fn = lambda: dispatch(xm, ids, MOE_E)
            rows_out = moe_tokens * MOE_K
            # tokens read once (repeats hit the L2), codes and scales written; the exchange path
            # also reads and writes them again (all_to_all_single) and once more (regroup)
            passes = 1 if name == "moe_dispatch" else 5
            work = ("bytes", moe_tokens * HID * 2 + passes * (rows_out * HID + rows_out * (HID // 128) * 4))
    elif name == "quant_dy_e5m2":
        # E5M2 gradient variant of the dY quantizer (1x128, s = amax / 57344)
        dy = randn(T, OUT, sigma=1e-3)
        q = torch.empty((T, OUT), dtype=u8, device=dev); sf = torch.empty((OUT // 128, ld(T)), dtype=f32, device=dev)
        fn = lambda: fp8q.fp8q_quant_act_1x128_e5m2(dy, q, sf)
        work = ("bytes", T * OUT * 3 + T * OUT // 128 * 4)
    elif name == "dgrad_e5m2":
        # E5M2 gradient variant of Dgrad: dY (E5M2) x W^T (E4M3)
        M, N, K = T, HID, OUT
        qa = torch.empty((M, K), dtype=u8, device=dev); sa = torch.empty((K // 128, ld(M)), dtype=f32, device=dev)
        fp8q.fp8q_quant_act_1x128_e5m2(randn(M, K, sigma=1e-3), qa, sa)
        qb, sb = fp8q.quant_w_128x128(randn(N, K, sigma=0.02))
        d = torch.empty((M, N), dtype=bf, device=dev)
        fn = lambda: fp8q.fp8q_gemm_blockscaled_fmt(qa, fp8q.FP8Q_FMT_E5M2, sa, qb, fp8q.FP8Q_FMT_E4M3, sb,
                                                    fp8q.FP8Q_SFB_BLOCK128, d)
        work = ("flops", 2.0 * M * N * K)
    elif name == "requant_x_t":
        # FP8 activation cache -> Wgrad operand: 1x128 codes + scales in, 128x1 transposed codes + scales out
        q, sf_in = fp8q.quant_act_1x128(randn(T, HID))
        qt = torch.empty((HID, T), dtype=u8, device=dev); sf = torch.empty((T // 128, ld(HID)), dtype=f32, device=dev)
        fn = lambda: fp8q.fp8q_requant_1x128_to_128x1(q, sf_in, qt, sf)
        work = ("bytes", 2 * T * HID + 2 * T * HID // 128 * 4)
    elif name == "pt_fprop":
        # per-tensor baseline GEMM at the Fprop shape: one TMEM accumulation over K, no promotion
        M, N, K = T, OUT, HID
        qa, sa = fp8q.quant_pertensor(randn(M, K))
        qb, sb = fp8q.quant_pertensor(randn(N, K, sigma=0.02))
        d = torch.empty((M, N), dtype=bf, device=dev)
        fn = lambda: fp8q.fp8q_gemm_pertensor(qa, sa[1:2], qb, sb[1:2], d)
        work = ("flops", 2.0 * M * N * K)
    elif name in ("quant_x", "quant_x_scaled", "quant_x_pct", "quant_x_t"):
        x = randn(T, HID)
        if name == "quant_x_scaled":
            # a scale policy's pass: given scales (here the online ones), tile maxima and clip count out
            q = torch.empty((T, HID), dtype=u8, device=dev); sf = torch.empty((HID // 128, ld(T)), dtype=f32, device=dev)
            fp8q.fp8q_quant_act_1x128(x, q, sf)
            amax = torch.empty_like(sf)
            clipped = torch.zeros(1, dtype=torch.int64, device=dev)
            fn = lambda: fp8q.fp8q_quant_act_1x128_scaled(x, sf, q, amax, clipped)
        elif name == "quant_x_pct":
            # percentile clipping: the scale from each tile's rank-th largest magnitude
            q = torch.empty((T, HID), dtype=u8, device=dev); sf = torch.empty((HID // 128, ld(T)), dtype=f32, device=dev)
            clipped = torch.zeros(1, dtype=torch.int64, device=dev)
            fn = lambda: fp8q.fp8q_quant_act_1x128_percentile(x, args.rank, q, sf, clipped)
        elif name == "quant_x":
            q = torch.empty((T, HID), dtype=u8, device=dev); sf = torch.empty((HID // 128, ld(T)), dtype=f32, device=dev)
            fn = lambda: fp8q.fp8q_quant_act_1x128(x, q, sf)
        else:
            q = torch.empty((HID, T), dtype=u8, device=dev); sf = torch.empty((T // 128, ld(HID)), dtype=f32, device=dev)
            fn = lambda: fp8q.fp8q_quant_act_128x1(x, q, sf)
        work = ("bytes", T * HID * 3 + T * HID // 128 * (8 if name == "quant_x_scaled" else 4))
    elif name == "quant_w":
        w = randn(OUT, HID, sigma=0.02)
        q, sf, qt, sft = fp8q.quant_w_128x128(w, transposed=True)
        fn = lambda: fp8q.fp8q_quant_w_128x128(w, q, sf, qt, sft)
        work = ("bytes", OUT * HID * 4 + 2 * (OUT // 128) * (HID // 128) * 4)
    elif name in ("fprop", "fprop_single", "dgrad", "wgrad"):
        if name == "fprop_single":
            # the one-CTA (128 x 256 tile) kernel at the Fprop shape, beside the one-CTA UE8M0 kernel
            fp8q.fp8q_debug_force_dense_kernel(fp8q.FP8Q_DENSE_SINGLE)
        if name in ("fprop", "fprop_single"):
            M, N, K = T, OUT, HID
        elif name == "dgrad":
            M, N, K = T, HID, OUT
        else:
            M, N, K = OUT, HID, T
        qa, sa = fp8q.quant_act_1x128(randn(M, K))
        if name == "wgrad":
            qb, sb = fp8q.quant_act_1x128(randn(N, K))
            d = torch.empty((M, N), dtype=f32, device=dev)
            mode = fp8q.FP8Q_SFB_ROW
        else:
            qb, sb = fp8q.quant_w_128x128(randn(N, K, sigma=0.02))
            d = torch.empty((M, N), dtype=bf, device=dev)
            mode = fp8q.FP8Q_SFB_BLOCK128
        fn = lambda: fp8q.fp8q_gemm_blockscaled(qa, sa, qb, sb, mode, d)
        work = ("flops", 2.0 * M * N * K)
    elif name in ("quant_moe_x", "quant_moe_x_gather", "moe_up", "moe_up_q", "moe_down"):
        moe_tokens = MOE_TOK if T == TOK else T          # --tokens counts MoE tokens before top-k
        route = W.moe_routing(tokens=moe_tokens, experts=MOE_E, top_k=MOE_K, seed=0)
        mt = int(route.offsets[-1])
        if name in ("quant_moe_x", "quant_moe_x_gather"):
            xm = randn(moe_tokens, HID)
            q = torch.empty((mt, HID), dtype=u8, device=dev)
            sf = torch.empty((HID // 128, ld(mt)), dtype=f32, device=dev)
            if name == "quant_moe_x":       # each token quantized once, scattered to its expert rows
                pos = torch.from_numpy(route.entry_row.astype(np.int32)).to(dev)
                fn = lambda: fp8q.fp8q_quant_act_1x128_scatter(xm, pos, q, sf)
            else:                           # each expert row gathers and quantizes its token
                rows = torch.from_numpy(route.token_of_row.astype(np.int32)).to(dev)
                fn = lambda: fp8q.fp8q_quant_act_1x128_gather(xm, rows, q, sf)
            work = ("bytes", moe_tokens * HID * 2 + mt * HID + mt * HID // 128 * 4)
        else:
            K, N = (MOE_FF, HID) if name == "moe_down" else (HID, MOE_FF)
            qa, sa = fp8q.quant_act_1x128(randn(mt, K))
            wq = torch.randint(0, 0x7E, (MOE_E, N, K), generator=gen, device=dev, dtype=u8)
            ws = torch.rand((MOE_E, N // 128, K // 128), generator=gen, device=dev) * 1e-3
            off = torch.from_numpy(route.offsets.astype(np.int32)).to(dev)
            if name == "moe_up_q":
                dq = torch.empty((mt, N), dtype=u8, device=dev)
                sfd = torch.empty((N // 128, ld(mt)), dtype=f32, device=dev)
                fn = lambda: fp8q.fp8q_grouped_gemm_blockscaled_q1x128(qa, sa, wq, ws, off, dq, sfd)
            else:
                d = torch.empty((mt, N), dtype=bf, device=dev)
                fn = lambda: fp8q.fp8q_grouped_gemm_blockscaled(qa, sa, wq, ws, off, d)
            work = ("flops", 2.0 * mt * N * K)
    else:
        raise SystemExit(f"unknown kernel {name}; choose from {SINGLE_KERNELS}")
    scrub = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    clocks = ClockSampler("GPU-" + str(torch.cuda.get_device_properties(0).uuid))
    clocks.path = os.path.join(LOG_DIR, f"clocks_single_{name}.csv")
    clocks.start()
    time.sleep(0.2)
    fp8q.fp8q_kernel_clock_counters(reset=True)
    times = []
    for _ in range(args.steps):
        scrub.zero_()                       # evict the inputs from L2 between launches
        s = torch.cuda.Event(enable_timing=True)
        e = torch.cuda.Event(enable_timing=True)
        s.record(); fn(); e.record()
        torch.cuda.synchronize()
        times.append(s.elapsed_time(e) * 1e-3)
    clk = clocks.stop()
    kclk = fp8q.fp8q_kernel_clock_counters(reset=True)
    if clk is not None:
        clk["gemm_kernel_sm_mhz"] = {k: v["mhz"] for k, v in kclk.items()}
    code = fp8q.fp8q_device_status()
    t = float(np.median(times))
    out = {"kernel": name, "tokens": T, "median_us": round(t * 1e6, 2), "min_us": round(min(times) * 1e6, 2),
           "status": code, "clocks": clk}
    if work[0] == "bytes":
        out["GBps"] = round(work[1] / t / 1e9, 1)
    else:
        out["TFLOPs"] = round(work[1] / t / 1e12, 1)
    print(json.dumps(out), flush=True)
    import torch.distributed as dist
    if dist.is_initialized():
        dist.destroy_process_group()
    if code != 0:
        raise SystemExit(1)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("fp8q", "reference"), default="fp8q")
    ap.add_argument("--cpu-rows", type=int, default=256,
                    help="rows per GEMM in the oracle's CPU-baseline sample (10-15 s on a 16-core host)")
    ap.add_argument("--ref-rows", type=int, default=4, help="rows per GEMM per step of the reference arm")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--single", choices=SINGLE_KERNELS, help="time one kernel alone (not the bench line)")
    ap.add_argument("--tokens", type=int, default=TOK, help="token count for --single")
    ap.add_argument("--rank", type=int, default=2, help="rank for --single quant_x_pct (2 = 99th percentile)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.single:
        run_single(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_fp8q(args)


if __name__ == "__main__":
    main()
