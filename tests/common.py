"""Shared helpers for the test suite: library loading, host<->device transfer
of the seeded inputs, and the GEMM tolerance rule.

GEMM tolerance (the GEMM results are not unique: summation order differs):
  * normwise   ||D - D_ref||_F / ||D_ref||_F <= 2e-3
  * elementwise |D - D_ref| <= ulp_bf16(D_ref) + 1e-3 * max_n |D_ref[m, n]|
with D_ref the oracle's FP64 result rounded once to the output type and
ulp_bf16(r) = 2^(max(floor(log2|r|), -126) - 7).  Quantized bytes and scales
are unique and compared bit for bit.
"""
from __future__ import annotations

import numpy as np

NORMWISE_TOL = 2e-3
ROW_REL_TOL = 1e-3


def load_fp8q():
    """Import the CUDA binding, building libfp8q.so in-tree first if needed
    (build.py is loaded by path: importing the package would load the old library)."""
    import importlib.util
    import os
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    spec = importlib.util.spec_from_file_location("fp8q_build", os.path.join(root, "fine_grained_fp8_x128_b200", "build.py"))
    _b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(_b)
    _b.build()
    import fine_grained_fp8_x128_b200 as fp8q
    return fp8q


def to_dev_bf16(bits: np.ndarray, device="cuda"):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device)
    return t.view(torch.bfloat16)


def to_dev_u8(a: np.ndarray, device="cuda"):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, np.uint8)).to(device)


def to_dev_f32(a: np.ndarray, device="cuda"):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(device)


def ulp_bf16(r: np.ndarray) -> np.ndarray:
    a = np.abs(np.asarray(r, np.float64))
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.where(a > 0, np.maximum(e, -126), -126)
    return np.exp2(e - 7)


def check_gemm(d: np.ndarray, d_exact: np.ndarray, d_ref_rounded: np.ndarray, row_max: np.ndarray = None):
    """d: device result (float64 view); d_exact: oracle FP64; d_ref_rounded: oracle rounded to the
    output type.  row_max: max_n |D_ref[m, n]| per sampled row (defaults to the sample's own rows)."""
    d = np.asarray(d, np.float64)
    num = np.linalg.norm(d - d_exact)
    den = np.linalg.norm(d_exact)
    normwise = num / den if den > 0 else num
    if row_max is None:
        row_max = np.abs(d_exact).max(axis=1)
    bound = ulp_bf16(d_ref_rounded) + ROW_REL_TOL * row_max[:, None]
    err = np.abs(d - d_ref_rounded)
    bad = err > bound
    info = dict(normwise=float(normwise), max_err=float(err.max()) if err.size else 0.0,
                n_bad=int(bad.sum()), max_ratio=float((err / np.maximum(bound, 1e-300)).max()) if err.size else 0.0)
    assert normwise <= NORMWISE_TOL, info
    assert not bad.any(), (info, np.argwhere(bad)[:5])
    return info
