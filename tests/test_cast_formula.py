"""The quantizers cast without a division: x / s is replaced by a product with
the negated reciprocal plus one FMA correction step (Markstein).  This CPU test
walks every BF16 input against every BF16 tile maximum that can contain it and
checks that the codes equal those of the IEEE quotient fl32(x / s) that the
scaling rule defines ("Fine-Grained FP8 Quantization in DeepSeek", section 2;
"FP8 Mixed Precision: DeepSeek-V3 Training Architecture", section 1, eq. s =
max|tile| / 448).  The GPU tests then compare the kernels with the oracle.
"""
import ctypes
import os
import subprocess
import tempfile

import numpy as np
import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "cast_formula_check.c")


@pytest.fixture(scope="module")
def harness():
    d = tempfile.mkdtemp(prefix="cfc_")
    so = os.path.join(d, "cfc.so")
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fPIC", "-shared", "-o", so, SRC, "-lm"])
    lib = ctypes.CDLL(so)
    lib.cfc_encode.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p]
    lib.cfc_check.argtypes = [ctypes.POINTER(ctypes.c_longlong), ctypes.POINTER(ctypes.c_longlong)]
    lib.cfc_check.restype = ctypes.c_longlong
    lib.cfc_encode_e5m2.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p]
    lib.cfc_check_e5m2.argtypes = [ctypes.POINTER(ctypes.c_longlong), ctypes.POINTER(ctypes.c_longlong)]
    lib.cfc_check_e5m2.restype = ctypes.c_longlong
    return lib


def test_harness_encoder_matches_oracle(harness):
    """The harness's own E4M3 encoder agrees with the oracle's on the values
    the check feeds it: every BF16 value scaled into the cast's range, the
    E4M3 midpoints and their float neighbours, signed zeros and saturation."""
    bf = (np.arange(0x7F80, dtype=np.uint32) << 16).view(np.float32)
    vals = [bf * np.float32(2.0 ** k) for k in (-120, -20, -9, 0, 3)]
    codes = np.arange(0x7F, dtype=np.uint8)
    grid = oracle.e4m3_decode(codes).astype(np.float32)
    mids = ((grid[:-1].astype(np.float64) + grid[1:]) / 2).astype(np.float32)
    vals += [grid, mids, np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(1e9)),
             np.array([0.0, -0.0, 448.0, 463.9, 464.0, 1e30], np.float32)]
    v = np.concatenate(vals).astype(np.float32)
    v = np.concatenate([v, -v])
    v = v[np.isfinite(v)]
    out = np.empty(v.size, np.uint8)
    harness.cfc_encode(v.ctypes.data, v.size, out.ctypes.data)
    assert np.array_equal(out, oracle.e4m3_encode(v))


def test_division_free_cast_is_exact_for_every_bf16_pair(harness):
    pairs = ctypes.c_longlong(0)
    plain = ctypes.c_longlong(0)
    bad = harness.cfc_check(ctypes.byref(pairs), ctypes.byref(plain))
    # sum over amax patterns a = 0..0x7F7F of 2(a+1) signed inputs
    assert pairs.value == 0x7F80 * (0x7F80 + 1)
    assert plain.value > 0          # the uncorrected product differs somewhere: the walk sees it
    assert bad == 0


def test_harness_e5m2_encoder_matches_oracle(harness):
    """The E5M2 gradient variant: the harness's E5M2 encoder against the
    oracle's on BF16 values scaled into the cast's range, the E5M2 grid, its
    midpoints and their neighbours, signed zeros and saturation."""
    bf = (np.arange(0x7F80, dtype=np.uint32) << 16).view(np.float32)
    vals = [bf * np.float32(2.0 ** k) for k in (-120, -30, -16, 0, 10)]
    codes = np.arange(0x7C, dtype=np.uint8)                      # finite magnitudes
    grid = oracle.e5m2_decode(codes).astype(np.float32)
    mids = ((grid[:-1].astype(np.float64) + grid[1:]) / 2).astype(np.float32)
    vals += [grid, mids, np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(1e9)),
             np.array([0.0, -0.0, 57344.0, 61439.0, 61440.0, 1e30], np.float32)]
    v = np.concatenate(vals).astype(np.float32)
    v = np.concatenate([v, -v])
    v = v[np.isfinite(v)]
    out = np.empty(v.size, np.uint8)
    harness.cfc_encode_e5m2(v.ctypes.data, v.size, out.ctypes.data)
    assert np.array_equal(out, oracle.e5m2_encode(v))


def test_division_free_e5m2_cast_is_exact_for_every_bf16_pair(harness):
    pairs = ctypes.c_longlong(0)
    plain = ctypes.c_longlong(0)
    bad = harness.cfc_check_e5m2(ctypes.byref(pairs), ctypes.byref(plain))
    assert pairs.value == 0x7F80 * (0x7F80 + 1)
    assert plain.value > 0
    assert bad == 0
