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
