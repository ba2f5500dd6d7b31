"""CPU oracle for the fine-grained FP8 path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
(and its ``--impl reference`` arm) may import this package.  The product path
(``fine_grained_fp8_x128_b200``) never imports it and shares no code with it.

The arithmetic lives in ``fp8q_oracle.cpp`` (plain C++, FP64 where the method
allows it); this module only builds that file with g++ and marshals numpy
arrays through ctypes.  Each wrapped function names the page passage it follows;
the C++ source states the readings taken where the pages are silent.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fp8q_oracle.cpp")
_LIB = os.path.join(_HERE, "libfp8q_oracle.so")
_CFLAGS = ["-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared", "-pthread"]

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with g++ (IEEE float, no contraction).  Returns the .so path."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", *_CFLAGS, "-o", tmp, _SRC])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    P = ctypes.c_void_p
    I64 = ctypes.c_int64
    lib.orc_version.restype = ctypes.c_int
    lib.orc_threads_used.restype = ctypes.c_int
    lib.orc_host_threads.restype = ctypes.c_int
    lib.orc_e4m3_encode.argtypes = [ctypes.c_float]
    lib.orc_e4m3_encode.restype = ctypes.c_uint8
    lib.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
    lib.orc_e4m3_decode.restype = ctypes.c_double
    lib.orc_e5m2_encode.argtypes = [ctypes.c_float]
    lib.orc_e5m2_encode.restype = ctypes.c_uint8
    lib.orc_e5m2_decode.argtypes = [ctypes.c_uint8]
    lib.orc_e5m2_decode.restype = ctypes.c_double
    lib.orc_e4m3_encode_array.argtypes = [P, I64, P]
    lib.orc_e5m2_encode_array.argtypes = [P, I64, P]
    lib.orc_round_bf16.argtypes = [P, I64, P]
    lib.orc_round_f32.argtypes = [P, I64, P]
    lib.orc_tile_scale.argtypes = [ctypes.c_float]
    lib.orc_tile_scale.restype = ctypes.c_float
    lib.orc_quant_act_1x128.argtypes = [P, I64, I64, I64, P, I64, P]
    lib.orc_quant_act_1x128_scaled.argtypes = [P, I64, I64, I64, P, P, I64, P, P]
    lib.orc_scale_history_update.argtypes = [ctypes.c_int, ctypes.c_float, P, P, P, I64]
    lib.orc_quant_act_1x128_percentile.argtypes = [P, I64, I64, I64, ctypes.c_int, P, I64, P, P]
    lib.orc_quant_act_128x1.argtypes = [P, I64, I64, I64, P, I64, P]
    lib.orc_quant_w_128x128.argtypes = [P, I64, I64, I64, P, I64, P]
    lib.orc_quant_tiles_intgrid.argtypes = [P, I64, I64, P]
    lib.orc_int8_absmax.argtypes = [P, I64, P, P]
    lib.orc_gemm_sampled.argtypes = [P, I64, P, P, I64, P, ctypes.c_int, I64, I64, I64,
                                     P, I64, P, I64, P]
    lib.orc_grouped_gemm_sampled.argtypes = [P, I64, P, P, P, P, I64, I64, I64,
                                             P, I64, P, I64, P]
    lib.orc_quant_pertensor_e4m3.argtypes = [P, I64, P, P]
    lib.orc_quant_pertensor.argtypes = [P, I64, I64, I64, P, I64, P, P]
    lib.orc_quant_act_1x128_e5m2.argtypes = [P, I64, I64, I64, P, I64, P]
    lib.orc_quant_act_128x1_e5m2.argtypes = [P, I64, I64, I64, P, I64, P]
    lib.orc_tile_scale_e5m2.argtypes = [ctypes.c_float]
    lib.orc_tile_scale_e5m2.restype = ctypes.c_float
    lib.orc_gemm_sampled_fmt.argtypes = [P, I64, P, P, I64, P, ctypes.c_int, I64, I64, I64,
                                         P, I64, P, I64, ctypes.c_int, ctypes.c_int, P]
    lib.orc_pow2_scale.argtypes = [ctypes.c_float]
    lib.orc_pow2_scale.restype = ctypes.c_float
    lib.orc_ue8m0_encode.argtypes = [ctypes.c_float]
    lib.orc_ue8m0_encode.restype = ctypes.c_int
    lib.orc_quant_act_1x128_pow2.argtypes = [P, I64, I64, I64, P, I64, P]
    lib.orc_quant_w_128x128_pow2.argtypes = [P, I64, I64, I64, P, I64, P]
    for name in ("orc_quant_act_1x128", "orc_quant_act_128x1", "orc_quant_w_128x128",
                 "orc_gemm_sampled", "orc_grouped_gemm_sampled", "orc_quant_act_1x128_pow2",
                 "orc_quant_w_128x128_pow2"):
        getattr(lib, name).restype = ctypes.c_int
    _lib = lib
    return lib


def _p(arr: np.ndarray):
    assert arr.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return arr.ctypes.data_as(ctypes.c_void_p)


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"oracle {what}: invalid arguments (rc={rc})")


def threads_used() -> int:
    """Most host threads any oracle call used since reset_threads_used()."""
    return _load().orc_threads_used()


def reset_threads_used() -> None:
    _load().orc_reset_threads_used()


def host_threads() -> int:
    return _load().orc_host_threads()


# ---------------------------------------------------------------- codecs
def e4m3_encode(x) -> np.ndarray:
    """E4M3 RNE + satfinite encode of float32 values (OCP FP8 definition)."""
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    out = np.empty(x.shape, dtype=np.uint8)
    _load().orc_e4m3_encode_array(_p(x), x.size, _p(out))
    return out


def e4m3_decode(codes) -> np.ndarray:
    """Exact value of each E4M3 code as float64 (NaN for S.1111.111)."""
    lib = _load()
    codes = np.asarray(codes, dtype=np.uint8)
    table = np.array([lib.orc_e4m3_decode(c) for c in range(256)], dtype=np.float64)
    return table[codes]


def e5m2_encode(x) -> np.ndarray:
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    out = np.empty(x.shape, dtype=np.uint8)
    _load().orc_e5m2_encode_array(_p(x), x.size, _p(out))
    return out


def e5m2_decode(codes) -> np.ndarray:
    lib = _load()
    codes = np.asarray(codes, dtype=np.uint8)
    table = np.array([lib.orc_e5m2_decode(c) for c in range(256)], dtype=np.float64)
    return table[codes]


def round_bf16(x) -> np.ndarray:
    """Single RNE rounding of float64 values to bfloat16 (returned as float64)."""
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    out = np.empty_like(x)
    _load().orc_round_bf16(_p(x), x.size, _p(out))
    return out


def round_f32(x) -> np.ndarray:
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    out = np.empty_like(x)
    _load().orc_round_f32(_p(x), x.size, _p(out))
    return out


def tile_scale(amax: float) -> float:
    """s = max(fl32(amax / 448), fl32(1e-12))."""
    return float(_load().orc_tile_scale(float(amax)))


# ---------------------------------------------------------------- quantizers
def quant_act_1x128(x_bf16: np.ndarray):
    """1x128 tiles along K.  x: uint16 bf16 bits [M][K] -> (q uint8 [M][K], sf float32 [M][K/128])."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    M, K = x.shape
    q = np.empty((M, K), np.uint8)
    sf = np.empty((M, K // 128), np.float32)
    _check(_load().orc_quant_act_1x128(_p(x), M, K, K, _p(q), K, _p(sf)), "quant_act_1x128")
    return q, sf


def quant_act_128x1(x_bf16: np.ndarray):
    """128x1 tiles along T, transposed.  x [T][C] -> (qt uint8 [C][T], sf float32 [T/128][C])."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    T, C = x.shape
    qt = np.empty((C, T), np.uint8)
    sf = np.empty((T // 128, C), np.float32)
    _check(_load().orc_quant_act_128x1(_p(x), T, C, C, _p(qt), T, _p(sf)), "quant_act_128x1")
    return qt, sf


def requant_1x128_to_128x1(q: np.ndarray, sf: np.ndarray):
    """FP8 activation caching ([P3] section 4: activations cached in FP8 for
    the backward pass).  From a 1x128 quantization (q uint8 [T][C], sf float32
    [T][C/128]) rebuild Wgrad's operand: the BF16 dequantization xh =
    RN_bf16(decode(q) * s) -- the product of a 4-bit and a 24-bit significand
    is exact in FP64, so one rounding -- then the 128x1 quantizer on xh.
    Returns (qt [C][T], sf_t [T/128][C], xh_bits uint16 [T][C])."""
    q = np.ascontiguousarray(q, np.uint8)
    T, C = q.shape
    sf = np.ascontiguousarray(sf, np.float32)
    assert sf.shape == (T, C // 128)
    deq = e4m3_decode(q).reshape(T, C) * np.repeat(sf.astype(np.float64), 128, axis=1)
    xh = round_bf16(deq)
    bits = (xh.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)   # exact: xh is a BF16 value
    qt, sft = quant_act_128x1(bits)
    return qt, sft, bits


FMT_E4M3 = 0
FMT_E5M2 = 1


def tile_scale_e5m2(amax: float) -> float:
    """E5M2 gradient variant: s = max(fl32(amax / 57344), fl32(1e-12))."""
    return float(_load().orc_tile_scale_e5m2(float(amax)))


def quant_act_1x128_e5m2(x_bf16: np.ndarray):
    """E5M2 gradient variant of quant_act_1x128: (q [M][K], sf [M][K/128])."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    M, K = x.shape
    q = np.empty((M, K), np.uint8)
    sf = np.empty((M, K // 128), np.float32)
    _check(_load().orc_quant_act_1x128_e5m2(_p(x), M, K, K, _p(q), K, _p(sf)), "quant_act_1x128_e5m2")
    return q, sf


def quant_act_128x1_e5m2(x_bf16: np.ndarray):
    """E5M2 gradient variant of quant_act_128x1: (qt [C][T], sf [T/128][C])."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    T, C = x.shape
    qt = np.empty((C, T), np.uint8)
    sf = np.empty((T // 128, C), np.float32)
    _check(_load().orc_quant_act_128x1_e5m2(_p(x), T, C, C, _p(qt), T, _p(sf)), "quant_act_128x1_e5m2")
    return qt, sf


def quant_w_128x128(w_bf16: np.ndarray):
    """128x128 blocks.  w [N][K] -> (q uint8 [N][K], sf float32 [N/128][K/128])."""
    w = np.ascontiguousarray(w_bf16, dtype=np.uint16)
    N, K = w.shape
    q = np.empty((N, K), np.uint8)
    sf = np.empty((N // 128, K // 128), np.float32)
    _check(_load().orc_quant_w_128x128(_p(w), N, K, K, _p(q), K, _p(sf)), "quant_w_128x128")
    return q, sf


# ---------------------------------------------------------------- power-of-two (UE8M0) scales
# Not the pages' method (which fixes s = amax/448): a reading for the study of
# hardware block scaling, which takes power-of-two scales.  The method's scale
# is rounded up to the next power of two; the tiles stay 1x128 / 128x128.
def pow2_scale(t: float) -> float:
    """Smallest power of two >= t (t > 0, a float32 value)."""
    return float(_load().orc_pow2_scale(float(t)))


def ue8m0_encode(s: float) -> int:
    """UE8M0 byte (biased exponent, 2^(b-127)) of a power of two; -1 otherwise."""
    return int(_load().orc_ue8m0_encode(float(s)))


def quant_act_1x128_pow2(x_bf16: np.ndarray):
    """1x128 tiles, s2 = 2^ceil(log2 tile_scale(amax)): (q uint8 [M][K], sf float32 [M][K/128])."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    M, K = x.shape
    q = np.empty((M, K), np.uint8)
    sf = np.empty((M, K // 128), np.float32)
    _check(_load().orc_quant_act_1x128_pow2(_p(x), M, K, K, _p(q), K, _p(sf)), "quant_act_1x128_pow2")
    return q, sf


def quant_w_128x128_pow2(w_bf16: np.ndarray):
    """128x128 blocks with power-of-two scales: (q uint8 [N][K], sf float32 [N/128][K/128])."""
    w = np.ascontiguousarray(w_bf16, dtype=np.uint16)
    N, K = w.shape
    q = np.empty((N, K), np.uint8)
    sf = np.empty((N // 128, K // 128), np.float32)
    _check(_load().orc_quant_w_128x128_pow2(_p(w), N, K, K, _p(q), K, _p(sf)), "quant_w_128x128_pow2")
    return q, sf


def quant_tiles_intgrid(x: np.ndarray, tile: int) -> np.ndarray:
    """P3 listing's integer-grid model over rows of `tile` values; returns q*s."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    assert x.size % tile == 0
    out = np.empty_like(x)
    _load().orc_quant_tiles_intgrid(_p(x), x.size // tile, tile, _p(out))
    return out


def int8_absmax(x):
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    q = np.empty(x.shape, np.int8)
    s = ctypes.c_double()
    _load().orc_int8_absmax(_p(x), x.size, _p(q), ctypes.cast(ctypes.pointer(s), ctypes.c_void_p))
    return q, s.value


def quant_pertensor_e4m3(x_bf16: np.ndarray):
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    deq = np.empty(x.shape, np.float64)
    s = ctypes.c_float()
    _load().orc_quant_pertensor_e4m3(_p(x), x.size, _p(deq), ctypes.cast(ctypes.pointer(s), ctypes.c_void_p))
    return deq, s.value


def quant_pertensor(x_bf16: np.ndarray):
    """Per-tensor E4M3 codes of a BF16 matrix: (q uint8 [M][K], amax, s)."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    M, K = x.shape
    q = np.empty((M, K), np.uint8)
    a = ctypes.c_float()
    s = ctypes.c_float()
    _check(_load().orc_quant_pertensor(_p(x), M, K, K, _p(q), K, ctypes.cast(ctypes.pointer(a), ctypes.c_void_p),
                                       ctypes.cast(ctypes.pointer(s), ctypes.c_void_p)), "quant_pertensor")
    return q, a.value, s.value


def gemm_pertensor_sampled(a, sa: float, b, sb: float, rows=None, cols=None) -> np.ndarray:
    """D = (sa * sb) * sum_k decode(a[m,k]) decode(b[n,k]) at the sampled
    entries, FP64.  This is the block-scaled GEMM with every block scale equal:
    it calls gemm_sampled with constant scale arrays."""
    M, K = a.shape
    N = b.shape[0]
    sfa = np.full((M, K // 128), sa, np.float32)
    sfb = np.full((N // 128, K // 128), sb, np.float32)
    return gemm_sampled(a, sfa, b, sfb, SFB_BLOCK128, rows, cols)


# ---------------------------------------------------------------- scale policies
POLICY_PREVIOUS = 0     # delayed: the previous step's tile maximum
POLICY_EMA = 1          # exponential amax history
POLICY_DECAYED_MAX = 2  # running maximum that decays by alpha per step


def quant_act_1x128_scaled(x_bf16: np.ndarray, sf: np.ndarray):
    """1x128 tiles cast with GIVEN scales sf [M][K/128] (a scale policy's).
    Returns (q uint8 [M][K], amax float32 [M][K/128] of the current tiles,
    clipped = number of elements the saturating cast clamps, |fl32(x / s)| > 464)."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    M, K = x.shape
    sf = np.ascontiguousarray(sf, dtype=np.float32)
    assert sf.shape == (M, K // 128)
    q = np.empty((M, K), np.uint8)
    amax = np.empty((M, K // 128), np.float32)
    clipped = ctypes.c_int64(0)
    _check(_load().orc_quant_act_1x128_scaled(_p(x), M, K, K, _p(sf), _p(q), K, _p(amax),
                                              ctypes.cast(ctypes.pointer(clipped), ctypes.c_void_p)),
           "quant_act_1x128_scaled")
    return q, amax, int(clipped.value)


def percentile_rank(p: float, n: int = 128) -> int:
    """The nearest-rank p-th percentile (0 < p <= 1) of n values is the
    ceil(p*n)-th smallest, i.e. the r-th largest with r = n - ceil(p*n) + 1."""
    if not 0.0 < p <= 1.0:
        raise ValueError("percentile must lie in (0, 1]")
    return n - int(np.ceil(p * n)) + 1


def quant_act_1x128_percentile(x_bf16: np.ndarray, rank: int):
    """Percentile clipping per 1x128 tile: s from the rank-th largest magnitude
    (rank 1 = the online rule).  Returns (q uint8 [M][K], sf float32 [M][K/128],
    clipped = number of saturated elements, |fl32(x / s)| > 464)."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    M, K = x.shape
    q = np.empty((M, K), np.uint8)
    sf = np.empty((M, K // 128), np.float32)
    clipped = ctypes.c_int64(0)
    _check(_load().orc_quant_act_1x128_percentile(_p(x), M, K, K, int(rank), _p(q), K, _p(sf),
                                                  ctypes.cast(ctypes.pointer(clipped), ctypes.c_void_p)),
           "quant_act_1x128_percentile")
    return q, sf, int(clipped.value)


def scale_history_update(policy: int, alpha: float, amax: np.ndarray, hist: np.ndarray):
    """One history step for each tile: returns (new history, next scales), float32."""
    a = np.ascontiguousarray(amax, dtype=np.float32)
    h = np.array(hist, dtype=np.float32, copy=True)
    sf = np.empty_like(a)
    _check(_load().orc_scale_history_update(int(policy), float(alpha), _p(a), _p(h), _p(sf), a.size),
           "scale_history_update")
    return h, sf


def scale_policy_drift(tiles_bf16: np.ndarray, alpha: float = 0.9, percentile: float = 0.99):
    """The [P1] worked example on the oracle: one 1x128 tile per step
    (tiles_bf16 [steps][128], e.g. a standard deviation doubling over the steps
    with a rare outlier) quantized under six policies -- current-max (online),
    fixed calibration (the first step's scale), previous-step delayed, EMA
    history, decaying maximum and percentile clipping of the current tile.  Returns {policy: (clip_rate [steps],
    mean_rel_err [steps])}: the fraction of clipped elements, and
    mean |dequant - x| / mean |x| of each step's tile."""
    x = np.ascontiguousarray(tiles_bf16, dtype=np.uint16)
    steps = x.shape[0]
    xf = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    table = e4m3_decode(np.arange(256, dtype=np.uint8))

    def measure(row, s):
        q, amax, clipped = quant_act_1x128_scaled(x[row:row + 1], np.array([[s]], np.float32))
        deq = table[q[0]] * float(s)
        err = np.abs(deq - xf[row]).mean() / max(np.abs(xf[row]).mean(), 1e-300)
        return clipped / 128.0, err, float(amax[0, 0])

    out = {}
    # current-max: each step's own tile maximum
    cr, er = np.zeros(steps), np.zeros(steps)
    for t in range(steps):
        _, s = quant_act_1x128(x[t:t + 1])
        cr[t], er[t], _ = measure(t, s[0, 0])
    out["current_max"] = (cr, er)
    # percentile clipping: each step's own tile, scaled from an upper percentile
    r = percentile_rank(percentile)
    cr, er = np.zeros(steps), np.zeros(steps)
    for t in range(steps):
        _, s, _ = quant_act_1x128_percentile(x[t:t + 1], r)
        cr[t], er[t], _ = measure(t, s[0, 0])
    out["percentile"] = (cr, er)
    # fixed calibration: the first step's scale for every step
    _, s0 = quant_act_1x128(x[0:1])
    cr, er = np.zeros(steps), np.zeros(steps)
    for t in range(steps):
        cr[t], er[t], _ = measure(t, s0[0, 0])
    out["fixed"] = (cr, er)
    # history policies: step 0 is calibrated on itself, step t uses the history after step t-1
    for name, pol in (("previous", POLICY_PREVIOUS), ("ema", POLICY_EMA), ("decayed_max", POLICY_DECAYED_MAX)):
        cr, er = np.zeros(steps), np.zeros(steps)
        _, s = quant_act_1x128(x[0:1])
        hist = np.zeros(1, np.float32)
        first = True
        for t in range(steps):
            cr[t], er[t], a = measure(t, s[0, 0] if first else s[0])
            if first:
                hist[0] = a            # the history starts at the calibration step's maximum
                first = False
            hist, s = scale_history_update(pol, alpha, np.array([a], np.float32), hist)
        out[name] = (cr, er)
    return out


# ---------------------------------------------------------------- MoE dispatch
def moe_layout(expert_ids: np.ndarray, num_experts: int):
    """[P3] section 4, FP8 MoE dispatch: the (token, slot) entries i = t*k + j
    in expert-major order, ties in entry order (a stable sort by expert id).
    Returns (rows [n]: token of output row m, pos [T][k]: output row of each
    entry, offsets [E+1]: the rows of expert e are offsets[e] .. offsets[e+1]-1)."""
    ids = np.ascontiguousarray(expert_ids, np.int64)
    T, k = ids.shape
    flat = ids.reshape(-1)
    assert np.all((flat >= 0) & (flat < num_experts))
    order = np.argsort(flat, kind="stable")
    rows = (order // k).astype(np.int32)
    pos = np.empty(flat.size, np.int32)
    pos[order] = np.arange(flat.size, dtype=np.int32)
    offsets = np.zeros(num_experts + 1, np.int32)
    offsets[1:] = np.cumsum(np.bincount(flat, minlength=num_experts))
    return rows, pos.reshape(T, k), offsets


def moe_dispatch_reference(xs, expert_ids_list, num_experts: int):
    """What each rank holds after an FP8 MoE dispatch over len(xs) ranks with
    experts split into equal contiguous ranges: for every local expert (in
    order), the rows from every source rank (in rank order), each source's
    rows in entry order -- every row the 1x128 FP8 quantization of its token.
    xs[s]: bf16 bits [T_s][H]; expert_ids_list[s]: int [T_s][k].
    Returns per rank (q [M][H], sf [M][H/128], expert offsets [E_local+1])."""
    world = len(xs)
    assert num_experts % world == 0
    el = num_experts // world
    quant = [quant_act_1x128(x) for x in xs]
    out = []
    for r in range(world):
        q_rows, s_rows, counts = [], [], np.zeros(el, np.int64)
        for e in range(r * el, (r + 1) * el):
            for s_ in range(world):
                ids = np.asarray(expert_ids_list[s_])
                ent = np.nonzero(ids.reshape(-1) == e)[0]
                toks = ent // ids.shape[1]
                q_rows.append(quant[s_][0][toks])
                s_rows.append(quant[s_][1][toks])
                counts[e - r * el] += toks.size
        H = xs[0].shape[1]
        q = np.concatenate(q_rows) if q_rows else np.zeros((0, H), np.uint8)
        sf = np.concatenate(s_rows) if s_rows else np.zeros((0, H // 128), np.float32)
        off = np.zeros(el + 1, np.int32)
        off[1:] = np.cumsum(counts)
        out.append((q, sf, off))
    return out


# ---------------------------------------------------------------- GEMMs
SFB_BLOCK128 = 0
SFB_ROW = 1


def gemm_sampled(a, sfa, b, sfb, sfb_mode, rows=None, cols=None, a_fmt=0, b_fmt=0) -> np.ndarray:
    """FP64 block-scaled GEMM D = A . B^T on the requested rows x cols.

    a: uint8 [M][K]; sfa: float32 [M][K/128]; b: uint8 [N][K];
    sfb: [N/128][K/128] (SFB_BLOCK128) or [N][K/128] (SFB_ROW).
    a_fmt, b_fmt: operand formats, FMT_E4M3 (the method's) or FMT_E5M2.
    """
    a = np.ascontiguousarray(a, np.uint8)
    b = np.ascontiguousarray(b, np.uint8)
    sfa = np.ascontiguousarray(sfa, np.float32)
    sfb = np.ascontiguousarray(sfb, np.float32)
    M, K = a.shape
    N = b.shape[0]
    rows = np.arange(M, dtype=np.int64) if rows is None else np.ascontiguousarray(rows, np.int64)
    cols = np.arange(N, dtype=np.int64) if cols is None else np.ascontiguousarray(cols, np.int64)
    out = np.empty((rows.size, cols.size), np.float64)
    rc = _load().orc_gemm_sampled_fmt(_p(a), K, _p(sfa), _p(b), K, _p(sfb), int(sfb_mode),
                                      M, N, K, _p(rows), rows.size, _p(cols), cols.size, int(a_fmt), int(b_fmt),
                                      _p(out))
    _check(rc, "gemm_sampled")
    return out


def grouped_gemm_sampled(a, sfa, w, sfw, offsets, rows=None, cols=None) -> np.ndarray:
    """FP64 grouped GEMM: row m of expert g (offsets[g] <= m < offsets[g+1]) times w[g]^T."""
    a = np.ascontiguousarray(a, np.uint8)
    sfa = np.ascontiguousarray(sfa, np.float32)
    w = np.ascontiguousarray(w, np.uint8)
    sfw = np.ascontiguousarray(sfw, np.float32)
    offsets = np.ascontiguousarray(offsets, np.int64)
    G, N, K = w.shape
    Mt = int(offsets[-1])
    rows = np.arange(Mt, dtype=np.int64) if rows is None else np.ascontiguousarray(rows, np.int64)
    cols = np.arange(N, dtype=np.int64) if cols is None else np.ascontiguousarray(cols, np.int64)
    out = np.empty((rows.size, cols.size), np.float64)
    rc = _load().orc_grouped_gemm_sampled(_p(a), K, _p(sfa), _p(w), _p(sfw), _p(offsets), G, N, K,
                                          _p(rows), rows.size, _p(cols), cols.size, _p(out))
    _check(rc, "grouped_gemm_sampled")
    return out
