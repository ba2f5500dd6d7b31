"""GPU parity of the FP8-activation-cache requantizer against the oracle, bit
for bit ("FP8 Mixed Precision: DeepSeek-V3 Training Architecture", section 4:
activations cached in FP8 for the backward pass): the 1x128 cache of an
activation is turned into Wgrad's 128x1 transposed operand.  Inputs include
products that fall on BF16 rounding midpoints after float32 rounding.
"""
import numpy as np
import pytest

import oracle
import workloads as W
from common import load_fp8q, to_dev_f32, to_dev_u8

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fp8q():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return load_fp8q()


def _run(fp8q, q, sf):
    import torch
    T, C = q.shape
    ld_in = (T + 3) // 4 * 4 + 4
    sbuf = np.full((C // 128, ld_in), np.nan, np.float32)
    sbuf[:, :T] = sf.T
    qd = to_dev_u8(np.pad(q, ((0, 0), (0, 16))))[:, :C]
    qtbuf = torch.full((C + 1, T + 16), 0x5A, dtype=torch.uint8, device="cuda")
    ld = (C + 3) // 4 * 4 + 4
    sft = torch.full((T // 128, ld), -1.0, dtype=torch.float32, device="cuda")
    fp8q.fp8q_requant_1x128_to_128x1(qd, to_dev_f32(sbuf), qtbuf[:C, :T], sft)
    torch.cuda.synchronize()
    assert fp8q.fp8q_device_status() == 0
    qt = qtbuf.cpu().numpy()
    assert np.all(qt[C] == 0x5A) and np.all(qt[:, T:] == 0x5A)
    s = sft.cpu().numpy()
    assert np.all(s[:, C:] == -1.0)
    return qt[:C, :T], s[:, :C]


@pytest.mark.parametrize("T,C", [(128, 128), (256, 384), (640, 1024)])
def test_requant_matches_oracle(fp8q, T, C):
    x = W.activations_with_outliers(T, C, seed=T + C, channel_frac=2 / C, elem_frac=1e-3)
    q, sf = oracle.quant_act_1x128(x)
    oqt, osft, _ = oracle.requant_1x128_to_128x1(q, sf)
    qt, sft = _run(fp8q, q, sf)
    assert np.array_equal(qt, oqt)
    assert np.array_equal(sft.view(np.uint32), osft.view(np.uint32))


def test_requant_midpoint_products_and_signed_zeros(fp8q):
    """Arbitrary caches: random codes (no NaN codes) with per-tile scales,
    plus products that land on BF16 midpoints after float32 rounding."""
    rng = np.random.default_rng(8)
    T, C = 256, 256
    q = rng.integers(0, 256, (T, C)).astype(np.uint8)
    q[(q & 0x7F) == 0x7F] = 0x80                                # NaN codes -> -0
    sf = (rng.uniform(1.0, 2.0, (T, C // 128)) * 2.0 ** rng.integers(-40, 20, (T, C // 128))).astype(np.float32)
    mc, ms = W.midpoint_product_pairs(T * 2)
    rows = np.arange(mc.size) // 2
    tiles = np.arange(mc.size) % 2
    q[rows, tiles * 128 + 7] = mc
    sf[rows, tiles] = ms
    q[:, 200] = 0x80
    oqt, osft, _ = oracle.requant_1x128_to_128x1(q, sf)
    qt, sft = _run(fp8q, q, sf)
    assert np.array_equal(qt, oqt)
    assert np.array_equal(sft.view(np.uint32), osft.view(np.uint32))


def test_requant_full_size(fp8q):
    """The cached 8192 x 7168 forward activation -> the Wgrad operand, every tile."""
    x = W.activations_with_outliers(8192, 7168, seed=0)
    q, sf = oracle.quant_act_1x128(x)
    oqt, osft, _ = oracle.requant_1x128_to_128x1(q, sf)
    qt, sft = _run(fp8q, q, sf)
    assert np.array_equal(sft.view(np.uint32), osft.view(np.uint32))
    assert np.array_equal(qt, oqt)
