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
    lib.orc_quant_act_128x1.argtypes = [P, I64, I64, I64, P, I64, P]
    lib.orc_quant_w_128x128.argtypes = [P, I64, I64, I64, P, I64, P]
    lib.orc_quant_tiles_intgrid.argtypes = [P, I64, I64, P]
    lib.orc_int8_absmax.argtypes = [P, I64, P, P]
    lib.orc_gemm_sampled.argtypes = [P, I64, P, P, I64, P, ctypes.c_int, I64, I64, I64,
                                     P, I64, P, I64, P]
    lib.orc_grouped_gemm_sampled.argtypes = [P, I64, P, P, P, P, I64, I64, I64,
                                             P, I64, P, I64, P]
    lib.orc_quant_pertensor_e4m3.argtypes = [P, I64, P, P]
    for name in ("orc_quant_act_1x128", "orc_quant_act_128x1", "orc_quant_w_128x128",
                 "orc_gemm_sampled", "orc_grouped_gemm_sampled"):
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


def quant_w_128x128(w_bf16: np.ndarray):
    """128x128 blocks.  w [N][K] -> (q uint8 [N][K], sf float32 [N/128][K/128])."""
    w = np.ascontiguousarray(w_bf16, dtype=np.uint16)
    N, K = w.shape
    q = np.empty((N, K), np.uint8)
    sf = np.empty((N // 128, K // 128), np.float32)
    _check(_load().orc_quant_w_128x128(_p(w), N, K, K, _p(q), K, _p(sf)), "quant_w_128x128")
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


# ---------------------------------------------------------------- GEMMs
SFB_BLOCK128 = 0
SFB_ROW = 1


def gemm_sampled(a, sfa, b, sfb, sfb_mode, rows=None, cols=None) -> np.ndarray:
    """FP64 block-scaled GEMM D = A . B^T on the requested rows x cols.

    a: uint8 [M][K]; sfa: float32 [M][K/128]; b: uint8 [N][K];
    sfb: [N/128][K/128] (SFB_BLOCK128) or [N][K/128] (SFB_ROW).
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
    rc = _load().orc_gemm_sampled(_p(a), K, _p(sfa), _p(b), K, _p(sfb), int(sfb_mode),
                                  M, N, K, _p(rows), rows.size, _p(cols), cols.size, _p(out))
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
