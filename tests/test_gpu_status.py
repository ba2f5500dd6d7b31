"""Failure detection without a GPU fault: a bounded device-side wait that runs
out records FP8Q_ERR_TIMEOUT in the status word, the kernel returns, and the
context stays usable.  Every pipeline wait in the GEMM uses the same wait."""
import numpy as np
import pytest

import oracle
import workloads as W
from common import load_fp8q, to_dev_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fp8q():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return load_fp8q()


def test_bounded_wait_expires_and_reports(fp8q):
    import torch
    assert fp8q.fp8q_device_status() == 0
    fp8q.fp8q_debug_wait_timeout(1 << 20)          # ~0.5 ms of SM clocks
    code = fp8q.fp8q_device_status()
    assert code & 0xFF == fp8q.FP8Q_ERR_TIMEOUT
    assert code >> 8 == 6                          # the debug wait site
    assert fp8q.fp8q_device_status() == 0          # reading clears it
    # the context is still usable
    x = W.activations_with_outliers(64, 256, seed=1, channel_frac=0, elem_frac=0)
    q, sf = fp8q.quant_act_1x128(to_dev_bf16(x))
    oq, osf = oracle.quant_act_1x128(x)
    assert np.array_equal(q.cpu().numpy(), oq)
    assert fp8q.fp8q_device_status() == 0


def test_gemm_clock_record(fp8q):
    """Every GEMM CTA adds its SM cycles and global-timer nanoseconds on exit;
    the ratio is the effective SM clock inside the kernels, and the CTA count
    is the launch's grid."""
    import torch
    x = W.activations_with_outliers(512, 512, seed=2, channel_frac=0, elem_frac=0)
    qa, sa = fp8q.quant_act_1x128(to_dev_bf16(x))
    qb, sb = fp8q.quant_w_128x128(to_dev_bf16(W.weights(512, 512, seed=3)))
    d = torch.empty((512, 512), dtype=torch.bfloat16, device="cuda")
    fp8q.fp8q_kernel_clock_counters(reset=True)
    fp8q.fp8q_gemm_blockscaled(qa, sa, qb, sb, fp8q.FP8Q_SFB_BLOCK128, d)      # M > 128: the CTA-pair kernel
    rec = fp8q.fp8q_kernel_clock_counters(reset=True)
    assert set(rec) == {"pair"}
    assert rec["pair"]["ctas"] == 8                  # 2 m-pairs x 2 n-tiles, two CTAs each
    assert 300.0 < rec["pair"]["mhz"] < 3000.0
    assert fp8q.fp8q_kernel_clock_counters(reset=True) == {}
    assert fp8q.fp8q_device_status() == 0
