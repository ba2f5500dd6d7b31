"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module holds no arithmetic of the method (no scales, no FP8 casts, no
GEMM): only random numbers, the outlier injection and the MoE routing that the
workloads call for, rounded to BF16.  Both the CUDA path and the CPU oracle are
fed from here, so they always see identical bytes.

Generator: numpy's Philox4x32-10 bit generator, one independent key per
(seed, tensor id, row block), so large tensors are filled by several threads and
the bytes do not depend on the thread count.  Normals come from numpy's
``standard_normal`` in float32 and are rounded to bfloat16 with
round-half-to-even on the bit pattern.
"""
from __future__ import annotations

import concurrent.futures as _cf
import os
from dataclasses import dataclass

import numpy as np

# tensor ids (one Philox key space per logical tensor)
TID_X = 1          # activations X [tokens][hidden]
TID_W = 2          # dense weight W [out][in]
TID_DY = 3         # output gradient dY [tokens][out]
TID_OUTLIER = 4    # outlier placement draws
TID_ROUTE = 5      # MoE routing draws
TID_EXPERT_UP = 6  # per-expert up-projection weights
TID_EXPERT_DN = 7  # per-expert down-projection weights
TID_H = 8          # MoE down-projection input (stand-in for the up output)
TID_MISC = 9

_ROWS_PER_BLOCK = 256


def _rng(seed: int, tid: int, block: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.Philox(key=[(seed << 32) | tid, block]))


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (RNE on the bit pattern); finite inputs only."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> 16) & 1
    return ((u + np.uint32(0x7FFF) + lsb) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _threads() -> int:
    return max(1, min(16, os.cpu_count() or 1))


def normal_f32(rows: int, cols: int, sigma: float, seed: int, tid: int) -> np.ndarray:
    """float32 [rows][cols] ~ N(0, sigma^2); row blocks drawn from independent keys."""
    out = np.empty((rows, cols), np.float32)
    nblk = (rows + _ROWS_PER_BLOCK - 1) // _ROWS_PER_BLOCK

    def fill(b):
        r0 = b * _ROWS_PER_BLOCK
        r1 = min(rows, r0 + _ROWS_PER_BLOCK)
        g = _rng(seed, tid, b)
        blk = g.standard_normal((r1 - r0, cols), dtype=np.float32)
        if sigma != 1.0:
            blk *= np.float32(sigma)
        out[r0:r1] = blk

    if nblk <= 1:
        for b in range(nblk):
            fill(b)
    else:
        with _cf.ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(fill, range(nblk)))
    return out


def normal_bf16(rows: int, cols: int, sigma: float, seed: int, tid: int) -> np.ndarray:
    """BF16 bits uint16 [rows][cols] ~ N(0, sigma^2)."""
    return f32_to_bf16_bits(normal_f32(rows, cols, sigma, seed, tid))


# --------------------------------------------------------------------------
# Workload recipes.  Sizes and distributions are those of the five workloads:
#   1. y = Wx: x 1x128 ~N(0,1) with element 17 = 20.0; W 256x128 ~N(0, 0.02)
#   2. X 8192x7168 ~N(0,1), 0.1% of channels x20, 1e-5 of elements -> +-120
#   3. forward GEMM: X as in 2, W 18432x7168 ~N(0, 0.02)
#   4. backward: dY 8192x18432 ~N(0, 1e-3) with 0.1% of tokens x50
#   5. MoE: 4096 tokens x 7168 ~N(0,1); top-8 of 256 experts, Zipf(1.1)
#      popularity over a seeded permutation, 8 experts forced empty;
#      up 7168->2048, down 2048->7168, expert weights ~N(0, 0.02).
# --------------------------------------------------------------------------
def linear_1x128_inputs(seed: int = 0):
    x = normal_f32(1, 128, 1.0, seed, TID_X)
    x[0, 17] = 20.0
    w = normal_f32(256, 128, 0.02, seed, TID_W)
    return f32_to_bf16_bits(x), f32_to_bf16_bits(w)


def activations_with_outliers(M: int, K: int, seed: int = 0, channel_frac: float = 1e-3,
                              channel_gain: float = 20.0, elem_frac: float = 1e-5,
                              elem_value: float = 120.0, tid: int = TID_X) -> np.ndarray:
    """BF16 [M][K] ~N(0,1); round(channel_frac*K) seeded channels scaled by
    channel_gain; round(elem_frac*M*K) seeded elements replaced by +-elem_value."""
    x = normal_f32(M, K, 1.0, seed, tid)
    g = _rng(seed, TID_OUTLIER, tid)
    n_ch = int(round(channel_frac * K))
    if n_ch:
        ch = g.choice(K, size=n_ch, replace=False)
        x[:, ch] *= np.float32(channel_gain)
    n_el = int(round(elem_frac * M * K))
    if n_el:
        flat = g.choice(M * K, size=n_el, replace=False)
        sign = np.where(g.random(n_el) < 0.5, -1.0, 1.0).astype(np.float32)
        x.reshape(-1)[flat] = sign * np.float32(elem_value)
    return f32_to_bf16_bits(x)


def weights(N: int, K: int, seed: int = 0, sigma: float = 0.02, tid: int = TID_W) -> np.ndarray:
    return normal_bf16(N, K, sigma, seed, tid)


def grad_with_outlier_tokens(M: int, N: int, seed: int = 0, sigma: float = 1e-3,
                             token_frac: float = 1e-3, gain: float = 50.0) -> np.ndarray:
    """BF16 dY [M][N] ~N(0, sigma^2) with round(token_frac*M) seeded tokens x gain."""
    y = normal_f32(M, N, sigma, seed, TID_DY)
    g = _rng(seed, TID_OUTLIER, TID_DY)
    n_tok = int(round(token_frac * M))
    if n_tok:
        rows = g.choice(M, size=n_tok, replace=False)
        y[rows] *= np.float32(gain)
    return f32_to_bf16_bits(y)


@dataclass
class Routing:
    """Tokens packed by expert: packed row r holds token token_of_row[r];
    expert g owns packed rows [offsets[g], offsets[g+1])."""
    offsets: np.ndarray      # int64 [G+1]
    token_of_row: np.ndarray  # int64 [T*top_k]
    counts: np.ndarray       # int64 [G]
    empty_experts: np.ndarray
    expert_ids: np.ndarray = None   # int64 [T][top_k]: each token's experts, in its pick order
    entry_row: np.ndarray = None    # int64 [T][top_k]: the packed row of each (token, pick)


def moe_routing(tokens: int = 4096, experts: int = 256, top_k: int = 8, zipf_s: float = 1.1,
                n_forced_empty: int = 8, seed: int = 0) -> Routing:
    """Zipf(s) popularity over a seeded expert permutation, n_forced_empty
    experts given zero weight, each token picking top_k distinct experts
    without replacement in proportion to the weights (Gumbel top-k)."""
    g = _rng(seed, TID_ROUTE)
    perm = g.permutation(experts)
    pop = np.empty(experts, np.float64)
    pop[perm] = np.arange(1, experts + 1, dtype=np.float64) ** (-zipf_s)
    empty = np.sort(g.choice(experts, size=n_forced_empty, replace=False)) if n_forced_empty else np.zeros(0, np.int64)
    pop[empty] = 0.0
    with np.errstate(divide="ignore"):
        logw = np.log(pop)
    gumbel = -np.log(-np.log(g.random((tokens, experts))))
    keys = logw[None, :] + gumbel
    choice = np.argsort(-keys, axis=1, kind="stable")[:, :top_k]   # [T][top_k]
    tok = np.repeat(np.arange(tokens, dtype=np.int64), top_k)
    exp = choice.reshape(-1).astype(np.int64)
    order = np.lexsort((tok, exp))       # by expert, then token
    counts = np.bincount(exp, minlength=experts).astype(np.int64)
    offsets = np.zeros(experts + 1, np.int64)
    offsets[1:] = np.cumsum(counts)
    entry_row = np.empty(tok.size, np.int64)
    entry_row[order] = np.arange(tok.size, dtype=np.int64)
    return Routing(offsets=offsets, token_of_row=tok[order], counts=counts, empty_experts=empty,
                   expert_ids=choice.astype(np.int64), entry_row=entry_row.reshape(tokens, top_k))


def expert_weights(G: int, N: int, K: int, seed: int = 0, sigma: float = 0.02,
                   tid: int = TID_EXPERT_UP, experts=None) -> np.ndarray:
    """BF16 [G][N][K]; expert g drawn from key (seed, tid*1024+g) so any subset
    of experts can be regenerated alone."""
    ids = range(G) if experts is None else experts
    ids = list(ids)
    out = np.empty((len(ids), N, K), np.uint16)

    def fill(i):
        out[i] = normal_bf16(N, K, sigma, seed, tid * 1024 + ids[i])

    with _cf.ThreadPoolExecutor(min(_threads(), max(1, len(ids)))) as ex:
        list(ex.map(fill, range(len(ids))))
    return out


def ragged_offsets(counts) -> np.ndarray:
    counts = np.asarray(counts, np.int64)
    off = np.zeros(counts.size + 1, np.int64)
    off[1:] = np.cumsum(counts)
    return off


def expert_weights_device(G: int, N: int, K: int, seed: int = 0, sigma: float = 0.02,
                          tid: int = TID_EXPERT_UP, device="cuda"):
    """BF16 [G][N][K] ~N(0, sigma^2) drawn on the device with torch's seeded
    generator (one generator per (seed, tid), experts drawn in order), for
    sizes too large to draw on the host.  A test that needs some experts on the
    host copies those bytes back."""
    import torch
    gen = torch.Generator(device=device)
    gen.manual_seed((seed << 20) + tid)
    out = torch.empty((G, N, K), dtype=torch.bfloat16, device=device)
    for g in range(G):
        out[g] = (torch.randn((N, K), generator=gen, device=device, dtype=torch.float32) * sigma).to(torch.bfloat16)
    return out


def drift_tiles(steps: int = 100, seed: int = 0, outlier_sigmas: float = 20.0):
    """The scale-policy drift workload: one 1x128 tile per step whose standard
    deviation doubles over the steps (sigma_t = 2^(t / (steps - 1))), with one
    element of one seeded step (in the middle half) replaced by an outlier of
    outlier_sigmas * sigma_t.  Returns (bf16 bits [steps][128], outlier step)."""
    g = _rng(seed, TID_MISC, 1)
    sig = np.exp2(np.arange(steps, dtype=np.float64) / max(steps - 1, 1))
    x = (g.standard_normal((steps, 128)) * sig[:, None]).astype(np.float32)
    t_out = int(g.integers(steps // 4, 3 * steps // 4))
    x[t_out, int(g.integers(0, 128))] = np.float32(outlier_sigmas * sig[t_out])
    return f32_to_bf16_bits(x), t_out


# E4M3 bytes of a few values with odd significands (3, 5, 7, 3.25, 1.875, 0.4375)
MIDPOINT_CODES = {0x44: 3.0, 0x4A: 5.0, 0x4E: 7.0, 0x45: 3.25, 0x3F: 1.875, 0x2E: 0.4375}


def midpoint_product_pairs(count: int = 64, seed: int = 0):
    """(code, scale) pairs whose float32 product fl32(c * s) lies exactly on a
    BF16 rounding midpoint while the exact product does not: the inputs on
    which rounding c * s to BF16 through float32 (twice) and rounding the exact
    product once disagree.  Found by walking float32 scales near m / c for
    midpoints m in [8, 16); returns (codes uint8 [n], scales float32 [n]),
    both directions of the exact product's offset included."""
    g = _rng(seed, TID_MISC, 2)
    codes, scales = [], []
    for code, c in MIDPOINT_CODES.items():
        for j in range(128):
            m = (1.0 + (2 * j + 1) / 256.0) * 8.0
            s0 = np.float32(m / c)
            for step in (-2, -1, 1, 2):
                s = s0
                for _ in range(abs(step)):
                    s = np.nextafter(s, np.float32(np.inf) if step > 0 else np.float32(0.0))
                p = np.float32(np.float32(c) * s)
                if (int(np.array([p], np.float32).view(np.uint32)[0]) & 0xFFFF) != 0x8000:
                    continue
                if np.float64(c) * np.float64(s) == np.float64(p):      # exact products are no trap
                    continue
                codes.append(code)
                scales.append(s)
    idx = g.permutation(len(codes))[:count]
    return np.array(codes, np.uint8)[idx], np.array(scales, np.float32)[idx]
