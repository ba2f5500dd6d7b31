"""The checked build on the GPU: libfp8q_checks.so is the library compiled
with -DFP8Q_CHECKS, where every instrumented kernel compares the computed
global index of each store (and the dispatch's row maps) with the extent its
arguments give and records FP8Q_ERR_BOUNDS instead of writing outside it.
The quantizer, GEMM, grouped-GEMM, fusion, E5M2, FP8-cache and dispatch parity
suites run against it in a child process: every case keeps a clean status
word (each test reads it) and still matches the oracle, so no computed index
of those shapes -- ragged tails, empty experts, one-row groups, 1024 experts
included -- leaves its buffer."""
import importlib.util
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SUITES = ["tests/test_gpu_quant.py", "tests/test_gpu_quant_dual.py", "tests/test_gpu_gemm.py",
          "tests/test_gpu_grouped.py", "tests/test_gpu_fused.py", "tests/test_gpu_e5m2.py",
          "tests/test_gpu_requant.py", "tests/test_gpu_dispatch.py"]


def _checked_library():
    spec = importlib.util.spec_from_file_location("fp8q_build", os.path.join(ROOT, "fine_grained_fp8_x128_b200", "build.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    b.build()
    return b.build(checks=True)


def test_parity_suites_under_the_checked_build():
    env = dict(os.environ, FP8Q_LIBRARY=_checked_library())
    probe = subprocess.run([sys.executable, "-c", "import fine_grained_fp8_x128_b200 as f; print(f.fp8q_build_checks())"],
                           cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert probe.returncode == 0 and probe.stdout.strip() == "True", probe.stdout + probe.stderr
    r = subprocess.run([sys.executable, "-m", "pytest", *SUITES, "-m", "gpu and not slow", "-q", "-x",
                        "-p", "no:cacheprovider"], cwd=ROOT, env=env, capture_output=True, text=True, timeout=3000)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
