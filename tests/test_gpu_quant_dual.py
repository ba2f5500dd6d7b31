"""GPU parity of fp8q_quant_act_dual: both tile orientations of one tensor
from a single read ("Introduction to LLM Quantization", "3) Backward
propagation"; "Fine-Grained FP8 Quantization in DeepSeek", section 2 and
section 4).  Its two outputs must equal, bit for bit, the oracle's 1x128 and
128x1 quantizations of the same BF16 tensor (the definitions the single-
orientation quantizers are held to), including the edge tiles (zeros, -0,
ties, subnormal landings) and the full activation and gradient workloads.
"""
import numpy as np
import pytest

import oracle
import workloads as W
from common import load_fp8q, to_dev_bf16

pytestmark = pytest.mark.gpu

CANARY = 0xA5


@pytest.fixture(scope="module")
def fp8q():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return load_fp8q()


def run_dual(fp8q, x_bits, ldx=None):
    import torch
    T, C = x_bits.shape
    ldx = ldx or C
    buf = np.full((T, ldx), 0x7FC0, np.uint16)        # NaN padding: must never be read
    buf[:, :C] = x_bits
    xd = to_dev_bf16(buf)[:, :C]
    q = torch.full((T, C + 16), CANARY, dtype=torch.uint8, device="cuda")
    qt = torch.full((C, T + 16), CANARY, dtype=torch.uint8, device="cuda")
    sf = torch.full((C // 128, T + 4), -7.0, dtype=torch.float32, device="cuda")
    sft = torch.full((T // 128, C + 4), -7.0, dtype=torch.float32, device="cuda")
    fp8q.fp8q_quant_act_dual(xd, q[:, :C], sf, qt[:, :T], sft)
    torch.cuda.synchronize()
    assert fp8q.fp8q_device_status() == 0
    qh, qth, sfh, sfth = q.cpu().numpy(), qt.cpu().numpy(), sf.cpu().numpy(), sft.cpu().numpy()
    # nothing written outside the outputs
    assert np.all(qh[:, C:] == CANARY) and np.all(qth[:, T:] == CANARY)
    assert np.all(sfh[:, T:] == -7.0) and np.all(sfth[:, C:] == -7.0)
    return qh[:, :C], sfh[:, :T], qth[:, :T], sfth[:, :C]


def _check(fp8q, x, ldx=None):
    q, sf, qt, sft = run_dual(fp8q, x, ldx)
    oq, osf = oracle.quant_act_1x128(x)
    oqt, osft = oracle.quant_act_128x1(x)
    assert np.array_equal(q, oq) and np.array_equal(sf, osf.T)
    assert np.array_equal(qt, oqt) and np.array_equal(sft, osft)


@pytest.mark.parametrize("T,C,ldx", [(128, 128, None), (256, 384, 392), (640, 1024, None)])
def test_dual_parity(fp8q, T, C, ldx):
    x = W.activations_with_outliers(T, C, seed=T + C, channel_frac=2 / C, elem_frac=1e-2)
    _check(fp8q, x, ldx)


def test_dual_edge_tiles(fp8q):
    """Zero and -0 tiles, a single non-zero, exact ties at non-power-of-two
    scales and values that land on E4M3 subnormals, in both orientations."""
    rng = np.random.default_rng(4)
    v = rng.normal(0, 1, (256, 256)).astype(np.float32)
    v[:128, :128] = 0.0
    v[:128, 128:] = -0.0
    v[5, 131] = -3.0
    v[128:, :128] *= np.float32(2.0 ** -14)           # lands on subnormal codes next to a larger tile maximum
    v[200, 7] = 448.0 * 3.0                           # scale 3: ties at its multiples
    v[201, :128] = np.float32(3.0) * np.float32(1.0625)
    x = W.f32_to_bf16_bits(v)
    _check(fp8q, x)


def test_dual_full_workloads(fp8q):
    """The bench's activation X 8192 x 7168 and gradient dY 8192 x 18432."""
    _check(fp8q, W.activations_with_outliers(8192, 7168, seed=0))
    _check(fp8q, W.grad_with_outlier_tokens(8192, 18432, seed=0))
