"""The no-allocation dispatch layout, fp8q_moe_dispatch_layout_noalloc.

Some callers cannot allocate device memory at the moment they call -- a plugin
enqueued by a host framework that owns all device memory and hands it no
workspace, a runtime whose memory budget was reserved at start-up, a path where
cudaMalloc's implicit synchronisation is not allowed.  For them the library
offers the MoE dispatch layout with its scratch in a fixed device array of its
own.  This file checks, through the C ABI, that the entry point returns exactly
what the workspace entry point fp8q_moe_dispatch_layout returns (the layout is
integer work: equal bit for bit) on two calls in a row, the second after the
first has left its contents in the shared array, and that a request larger
than the array is refused without a launch.

The file is named to be collected last, so that a run stopping at the first
failure has run every other test already.
"""
import ctypes

import numpy as np
import pytest

import workloads as W
from common import load_fp8q

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fp8q():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return load_fp8q()


def _ids_dev(ids):
    import torch
    return torch.from_numpy(np.ascontiguousarray(ids, np.int32)).cuda()


def _with_workspace(fp8q, ids_d, E):
    """The existing entry point, with a caller-allocated workspace."""
    import torch
    n, k = ids_d.numel(), ids_d.shape[1]
    rows = torch.full((n,), -7, dtype=torch.int32, device="cuda")
    pos = torch.full(tuple(ids_d.shape), -7, dtype=torch.int32, device="cuda")
    off = torch.full((E + 1,), -7, dtype=torch.int32, device="cuda")
    ws = torch.empty(max(1, fp8q.lib().fp8q_moe_dispatch_layout_workspace(n, E)), dtype=torch.int32, device="cuda")
    fp8q.fp8q_moe_dispatch_layout(ids_d, E, rows, pos, off, ws)
    return rows, pos, off


def _no_alloc_raw(fp8q, ids_d, E):
    """The new entry point called through the C ABI with raw pointers."""
    import torch
    n, k = ids_d.numel(), ids_d.shape[1]
    rows = torch.full((n,), -7, dtype=torch.int32, device="cuda")
    pos = torch.full(tuple(ids_d.shape), -7, dtype=torch.int32, device="cuda")
    off = torch.full((E + 1,), -7, dtype=torch.int32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = fp8q.lib().fp8q_moe_dispatch_layout_noalloc(
        ctypes.c_void_p(ids_d.data_ptr()), n, k, E, ctypes.c_void_p(rows.data_ptr()),
        ctypes.c_void_p(pos.data_ptr()), ctypes.c_void_p(off.data_ptr()), stream)
    assert rc == fp8q.FP8Q_OK, fp8q.fp8q_status_string(rc)
    return rows, pos, off


def test_no_alloc_layout_equals_workspace_layout_on_two_calls(fp8q):
    import torch
    # call 1: the MoE workload's routing (4096 tokens, top-8 of 256 experts);
    # call 2: another shape (1000 tokens, top-4 of 1024 experts) that reuses
    # the scratch array with a different chunk count and expert count
    cases = [(W.moe_routing(4096, 256, 8, n_forced_empty=8, seed=0).expert_ids, 256),
             (W.moe_routing(1000, 1024, 4, n_forced_empty=2, seed=5).expert_ids, 1024)]
    for ids, E in cases:
        ids_d = _ids_dev(ids)
        want = _with_workspace(fp8q, ids_d, E)
        got = _no_alloc_raw(fp8q, ids_d, E)
        torch.cuda.synchronize()
        assert fp8q.fp8q_device_status() == 0
        for g, w in zip(got, want):
            assert torch.equal(g, w)
        # a complete permutation: every entry placed, expert counts summing to all entries
        off = got[2].cpu().numpy()
        assert off[0] == 0 and off[-1] == ids.size and np.all(np.diff(off) >= 0)


def test_no_alloc_layout_refuses_requests_beyond_the_array(fp8q):
    """1024 experts need 2 x chunks x 1024 scratch words; 32769 entries take
    129 chunks, beyond the 262144-word array: refused before any launch, and
    the next call in bounds still matches the workspace entry point."""
    import torch
    assert fp8q.FP8Q_LAYOUT_NOALLOC_SCRATCH_INTS == 262144
    E, k, n = 1024, 1, 32769
    assert fp8q.lib().fp8q_moe_dispatch_layout_workspace(n, E) > fp8q.FP8Q_LAYOUT_NOALLOC_SCRATCH_INTS
    ids_d = torch.zeros((n, k), dtype=torch.int32, device="cuda")
    rows = torch.empty(n, dtype=torch.int32, device="cuda")
    pos = torch.empty((n, k), dtype=torch.int32, device="cuda")
    off = torch.full((E + 1,), -7, dtype=torch.int32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = fp8q.lib().fp8q_moe_dispatch_layout_noalloc(
        ctypes.c_void_p(ids_d.data_ptr()), n, k, E, ctypes.c_void_p(rows.data_ptr()),
        ctypes.c_void_p(pos.data_ptr()), ctypes.c_void_p(off.data_ptr()), stream)
    assert rc == fp8q.FP8Q_ERR_SCRATCH_LIMIT
    torch.cuda.synchronize()
    assert torch.all(off == -7)                       # nothing was launched
    ids_ok = ids_d[:32768]
    want = _with_workspace(fp8q, ids_ok, E)
    got = _no_alloc_raw(fp8q, ids_ok, E)
    torch.cuda.synchronize()
    assert fp8q.fp8q_device_status() == 0
    for g, w in zip(got, want):
        assert torch.equal(g, w)
