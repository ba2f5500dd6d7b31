"""fine_grained_fp8_x128_b200: fine-grained FP8 training matmuls on B200.

Python binding of the C ABI in include/fp8q.h (libfp8q.so, built in-tree by
``build.py``).  Argument marshalling only: every step runs in the library's
sm_100a kernels, on the caller's current CUDA stream.  There is no CPU path;
if the shared library is missing, importing this package raises.

Each function has the C entry point's name and takes torch CUDA tensors for the
device buffers (torch is used only for memory and streams).  Sizes and leading
dimensions are taken from the tensors' shapes and row strides.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# FP8Q_LIBRARY may name another build of the same library (A/B timing).
LIB_PATH = os.environ.get("FP8Q_LIBRARY") or os.path.join(_HERE, "libfp8q.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"libfp8q.so is not built ({LIB_PATH}); run `python fine_grained_fp8_x128_b200/build.py`")

_lib = ctypes.CDLL(LIB_PATH)

FP8Q_OK = 0
FP8Q_ERR_INVALID_ARG = 1
FP8Q_ERR_ALIGNMENT = 2
FP8Q_ERR_UNSUPPORTED = 3
FP8Q_ERR_CUDA = 4
FP8Q_ERR_TIMEOUT = 5
FP8Q_ERR_SCRATCH_LIMIT = 6
FP8Q_ERR_BOUNDS = 7
FP8Q_LAYOUT_NOALLOC_SCRATCH_INTS = 262144
FP8Q_SFB_BLOCK128 = 0
FP8Q_SFB_ROW = 1
FP8Q_POLICY_PREVIOUS = 0
FP8Q_POLICY_EMA = 1
FP8Q_POLICY_DECAYED_MAX = 2
FP8Q_OUT_BF16 = 0
FP8Q_OUT_F32 = 1
FP8Q_FMT_E4M3 = 0
FP8Q_FMT_E5M2 = 1
FP8Q_DENSE_AUTO = 0
FP8Q_DENSE_SINGLE = 1
FP8Q_DENSE_PAIR = 2

EXPORTS = (
    "fp8q_version", "fp8q_status_string", "fp8q_device_status",
    "fp8q_quant_act_1x128", "fp8q_quant_act_1x128_gather", "fp8q_quant_act_1x128_scaled",
    "fp8q_quant_act_1x128_percentile", "fp8q_scale_history_update", "fp8q_quant_act_128x1", "fp8q_quant_w_128x128",
    "fp8q_gemm_blockscaled", "fp8q_gemm_blockscaled_q1x128",
    "fp8q_grouped_gemm_blockscaled", "fp8q_grouped_gemm_blockscaled_q1x128",
    "fp8q_quant_pertensor", "fp8q_gemm_pertensor", "fp8q_requant_1x128_to_128x1",
    "fp8q_quant_act_1x128_e5m2", "fp8q_quant_act_128x1_e5m2", "fp8q_gemm_blockscaled_fmt",
    "fp8q_moe_dispatch_layout_workspace", "fp8q_moe_dispatch_layout", "fp8q_quant_act_1x128_gather_rowscales",
    "fp8q_gather_rows_fp8", "fp8q_quant_act_1x128_scatter", "fp8q_quant_act_1x128_scatter_rowscales",
    "fp8q_debug_cast_e4m3_bits", "fp8q_debug_wait_timeout", "fp8q_debug_force_dense_kernel",
    "fp8q_moe_dispatch_layout_noalloc",
    "fp8q_quant_act_1x128_ue8m0", "fp8q_quant_w_128x128_ue8m0", "fp8q_gemm_mxf8_ue8m0",
    "fp8q_kernel_clock_counters", "fp8q_quant_act_dual", "fp8q_moe_regroup_order", "fp8q_build_checks",
)

_P = ctypes.c_void_p
_I = ctypes.c_int64
_lib.fp8q_version.restype = ctypes.c_int
_lib.fp8q_build_checks.restype = ctypes.c_int
_lib.fp8q_status_string.argtypes = [ctypes.c_int]
_lib.fp8q_status_string.restype = ctypes.c_char_p
_lib.fp8q_device_status.argtypes = [_P, ctypes.POINTER(ctypes.c_int)]
_lib.fp8q_quant_act_1x128.argtypes = [_P, _I, _I, _I, _P, _I, _P, _I, _P]
_lib.fp8q_quant_act_1x128_gather.argtypes = [_P, _I, _I, _I, _P, _I, _P, _I, _P, _I, _P]
_lib.fp8q_quant_act_1x128_scaled.argtypes = [_P, _I, _I, _I, _P, _I, _P, _I, _P, _I, _P, _P]
_lib.fp8q_quant_act_1x128_percentile.argtypes = [_P, _I, _I, _I, ctypes.c_int, _P, _I, _P, _I, _P, _P]
_lib.fp8q_requant_1x128_to_128x1.argtypes = [_P, _I, _I, _I, _P, _I, _P, _I, _P, _I, _P]
_lib.fp8q_quant_act_1x128_e5m2.argtypes = [_P, _I, _I, _I, _P, _I, _P, _I, _P]
_lib.fp8q_quant_act_128x1_e5m2.argtypes = [_P, _I, _I, _I, _P, _I, _P, _I, _P]
_lib.fp8q_gemm_blockscaled_fmt.argtypes = [_P, ctypes.c_int, _I, _P, _I, _P, ctypes.c_int, _I, _P, _I, ctypes.c_int,
                                           _P, _I, ctypes.c_int, _I, _I, _I, _P]
_lib.fp8q_moe_dispatch_layout_workspace.argtypes = [_I, ctypes.c_int]
_lib.fp8q_moe_dispatch_layout_workspace.restype = ctypes.c_int64
_lib.fp8q_moe_dispatch_layout.argtypes = [_P, _I, ctypes.c_int, ctypes.c_int, _P, _P, _P, _P, _I, _P]
_lib.fp8q_moe_dispatch_layout_noalloc.argtypes = [_P, _I, ctypes.c_int, ctypes.c_int, _P, _P, _P, _P]
_lib.fp8q_quant_act_1x128_gather_rowscales.argtypes = [_P, _I, _I, _I, _P, _I, _P, _I, _P, _I, _P]
_lib.fp8q_quant_act_1x128_scatter.argtypes = [_P, _I, _I, _I, _P, ctypes.c_int, _I, _P, _I, _P, _I, _P]
_lib.fp8q_quant_act_1x128_scatter_rowscales.argtypes = [_P, _I, _I, _I, _P, ctypes.c_int, _I, _P, _I, _P, _I, _P]
_lib.fp8q_gather_rows_fp8.argtypes = [_P, _I, _P, _I, _I, _P, _I, _I, _P, _I, _P, _I, _P]
_lib.fp8q_moe_regroup_order.argtypes = [_P, ctypes.c_int, ctypes.c_int, ctypes.c_int, _I, _P, _P, _P]
_lib.fp8q_quant_pertensor.argtypes = [_P, _I, _I, _I, _P, _I, _P, _P]
_lib.fp8q_gemm_pertensor.argtypes = [_P, _I, _P, _P, _I, _P, _P, _I, ctypes.c_int, _I, _I, _I, _P]
_lib.fp8q_scale_history_update.argtypes = [ctypes.c_int, ctypes.c_float, _P, _P, _P, _I, _P]
_lib.fp8q_quant_act_128x1.argtypes = [_P, _I, _I, _I, _P, _I, _P, _I, _P]
_lib.fp8q_quant_w_128x128.argtypes = [_P, _I, _I, _I, _P, _I, _P, _I, _P, _I, _P, _I, _P]
_lib.fp8q_gemm_blockscaled.argtypes = [_P, _I, _P, _I, _P, _I, _P, _I, ctypes.c_int, _P, _I, ctypes.c_int,
                                       _I, _I, _I, _P]
_lib.fp8q_gemm_blockscaled_q1x128.argtypes = [_P, _I, _P, _I, _P, _I, _P, _I, _P, _I, _P, _I, _I, _I, _I, _P]
_lib.fp8q_grouped_gemm_blockscaled.argtypes = [_P, _I, _P, _I, _P, _P, _P, _I, _I, _P, _I, _I, _I, _P]
_lib.fp8q_grouped_gemm_blockscaled_q1x128.argtypes = [_P, _I, _P, _I, _P, _P, _P, _I, _I, _P, _I, _P, _I, _I, _I,
                                                      _P]
_lib.fp8q_debug_cast_e4m3_bits.argtypes = [ctypes.c_uint32, _I, _P, _P]
_lib.fp8q_debug_wait_timeout.argtypes = [_I, _P]
_lib.fp8q_debug_force_dense_kernel.argtypes = [ctypes.c_int]
_lib.fp8q_kernel_clock_counters.argtypes = [_P, ctypes.c_int]
_lib.fp8q_quant_act_dual.argtypes = [_P, _I, _I, _I, _P, _I, _P, _I, _P, _I, _P, _I, _P]
_lib.fp8q_quant_act_1x128_ue8m0.argtypes = [_P, _I, _I, _I, _P, _I, _P, _P]
_lib.fp8q_quant_w_128x128_ue8m0.argtypes = [_P, _I, _I, _I, _P, _I, _P, _P]
_lib.fp8q_gemm_mxf8_ue8m0.argtypes = [_P, _I, _P, _P, _I, _P, _P, _I, _I, _I, _I, _P]
for _n in EXPORTS[2:]:
    getattr(_lib, _n).restype = ctypes.c_int


class FP8QError(RuntimeError):
    def __init__(self, status: int, call: str):
        self.status = status
        super().__init__(f"{call}: {fp8q_status_string(status)} (status {status})")


def lib() -> ctypes.CDLL:
    return _lib


def fp8q_version() -> int:
    return _lib.fp8q_version()


def fp8q_status_string(status: int) -> str:
    return _lib.fp8q_status_string(int(status)).decode()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _ptr(t):
    return None if t is None else t.data_ptr()


def _ld(t):
    """Row stride (elements) of a 2D tensor whose last dimension is contiguous."""
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError("expected a 2D tensor with a contiguous last dimension")
    return t.stride(0)


def _check(rc: int, call: str):
    if rc != FP8Q_OK:
        raise FP8QError(rc, call)


def fp8q_build_checks() -> bool:
    """True for the checked build (device-side bounds checks, libfp8q_checks.so)."""
    return bool(_lib.fp8q_build_checks())


def fp8q_device_status(stream=None) -> int:
    """Synchronise the stream; return and clear the device status word (0 = clean)."""
    code = ctypes.c_int(0)
    rc = _lib.fp8q_device_status(_stream(stream), ctypes.byref(code))
    if rc not in (FP8Q_OK, FP8Q_ERR_TIMEOUT, FP8Q_ERR_INVALID_ARG, FP8Q_ERR_BOUNDS):
        raise FP8QError(rc, "fp8q_device_status")
    return code.value


def fp8q_quant_act_1x128(x, q, sf, stream=None):
    """x bf16 [M][K] -> q uint8 [M][K], sf float32 [K/128][ld_sf >= M] (sf[kb][m])."""
    M, K = x.shape
    _check(_lib.fp8q_quant_act_1x128(_ptr(x), M, K, _ld(x), _ptr(q), _ld(q), _ptr(sf), _ld(sf) if sf.dim() == 2 else M,
                                     _stream(stream)), "fp8q_quant_act_1x128")


def fp8q_quant_act_1x128_gather(x, rows, q, sf, stream=None):
    """q[m] / sf[:, m] = 1x128 quantization of x[rows[m]]; rows int32 [M] on device."""
    M_src, K = x.shape
    M = rows.shape[0]
    _check(_lib.fp8q_quant_act_1x128_gather(_ptr(x), M_src, K, _ld(x), _ptr(rows), M, _ptr(q), _ld(q), _ptr(sf),
                                            _ld(sf), _stream(stream)), "fp8q_quant_act_1x128_gather")


def fp8q_quant_act_1x128_scaled(x, sf, q, amax=None, clipped=None, stream=None):
    """q = e4m3(x / sf) per 1x128 tile with given scales sf [K/128][ld >= M];
    optional amax [K/128][ld] (tile maxima out) and clipped (int64 device
    counter, += saturated elements)."""
    M, K = x.shape
    _check(_lib.fp8q_quant_act_1x128_scaled(_ptr(x), M, K, _ld(x), _ptr(sf), _ld(sf), _ptr(q), _ld(q), _ptr(amax),
                                            _ld(amax) if amax is not None else 0, _ptr(clipped), _stream(stream)),
           "fp8q_quant_act_1x128_scaled")


def fp8q_quant_act_1x128_percentile(x, rank, q, sf, clipped=None, stream=None):
    """Percentile clipping per 1x128 tile: sf [K/128][ld >= M] from each tile's
    rank-th largest magnitude (rank 1 = the online rule), q = e4m3(x / sf);
    optional clipped (int64 device counter, += saturated elements)."""
    M, K = x.shape
    _check(_lib.fp8q_quant_act_1x128_percentile(_ptr(x), M, K, _ld(x), int(rank), _ptr(q), _ld(q), _ptr(sf), _ld(sf),
                                                _ptr(clipped), _stream(stream)), "fp8q_quant_act_1x128_percentile")


def fp8q_scale_history_update(policy, alpha, amax, hist, sf, stream=None):
    """Elementwise over n = amax.numel() tiles: hist <- policy(hist, amax), sf <- tile scale of hist."""
    _check(_lib.fp8q_scale_history_update(int(policy), float(alpha), _ptr(amax), _ptr(hist), _ptr(sf), amax.numel(),
                                          _stream(stream)), "fp8q_scale_history_update")


def fp8q_quant_act_128x1(x, qt, sf, stream=None):
    """x bf16 [T][C] -> qt uint8 [C][T], sf float32 [T/128][ld_sf >= C]."""
    T, C = x.shape
    _check(_lib.fp8q_quant_act_128x1(_ptr(x), T, C, _ld(x), _ptr(qt), _ld(qt), _ptr(sf), _ld(sf), _stream(stream)),
           "fp8q_quant_act_128x1")


def fp8q_quant_act_dual(x, q, sf, qt, sft, stream=None):
    """Both orientations from one read: x bf16 [T][C] -> q uint8 [T][C] with sf [C/128][ld >= T]
    (1x128 tiles) and qt uint8 [C][T] with sft [T/128][ld >= C] (128x1 tiles)."""
    T, C = x.shape
    _check(_lib.fp8q_quant_act_dual(_ptr(x), T, C, _ld(x), _ptr(q), _ld(q), _ptr(sf), _ld(sf), _ptr(qt), _ld(qt),
                                    _ptr(sft), _ld(sft), _stream(stream)), "fp8q_quant_act_dual")


def fp8q_quant_w_128x128(w, q, sf, qt=None, sft=None, stream=None):
    """w bf16 [N][K] -> q [N][K], sf [N/128][K/128]; optional qt [K][N], sft [K/128][N/128]."""
    N, K = w.shape
    _check(_lib.fp8q_quant_w_128x128(_ptr(w), N, K, _ld(w), _ptr(q), _ld(q), _ptr(sf), _ld(sf),
                                     _ptr(qt), _ld(qt) if qt is not None else 0,
                                     _ptr(sft), _ld(sft) if sft is not None else 0, _stream(stream)),
           "fp8q_quant_w_128x128")


def fp8q_gemm_blockscaled(a, sfa, b, sfb, sfb_mode, d, stream=None):
    """d[M][N] = block-scaled a[M][K] . b[N][K]^T; d is bf16 or float32."""
    M, K = a.shape
    N = b.shape[0]
    dt = FP8Q_OUT_F32 if d.dtype == torch.float32 else FP8Q_OUT_BF16
    _check(_lib.fp8q_gemm_blockscaled(_ptr(a), _ld(a), _ptr(sfa), _ld(sfa), _ptr(b), _ld(b), _ptr(sfb), _ld(sfb),
                                      int(sfb_mode), _ptr(d), _ld(d), dt, M, N, K, _stream(stream)),
           "fp8q_gemm_blockscaled")


def fp8q_requant_1x128_to_128x1(q, sf_in, qt, sf, stream=None):
    """FP8 activation cache -> Wgrad operand: q uint8 [T][C] with sf_in [C/128][ld >= T]
    (a 1x128 quantization) -> qt uint8 [C][T], sf [T/128][ld >= C] (128x1 tiles of the
    BF16 dequantization)."""
    T, C = q.shape
    _check(_lib.fp8q_requant_1x128_to_128x1(_ptr(q), T, C, _ld(q), _ptr(sf_in), _ld(sf_in), _ptr(qt), _ld(qt),
                                            _ptr(sf), _ld(sf), _stream(stream)), "fp8q_requant_1x128_to_128x1")


def fp8q_quant_act_1x128_e5m2(x, q, sf, stream=None):
    """E5M2 gradient variant of fp8q_quant_act_1x128 (s = amax / 57344)."""
    M, K = x.shape
    _check(_lib.fp8q_quant_act_1x128_e5m2(_ptr(x), M, K, _ld(x), _ptr(q), _ld(q), _ptr(sf), _ld(sf), _stream(stream)),
           "fp8q_quant_act_1x128_e5m2")


def fp8q_quant_act_128x1_e5m2(x, qt, sf, stream=None):
    """E5M2 gradient variant of fp8q_quant_act_128x1 (s = amax / 57344)."""
    T, C = x.shape
    _check(_lib.fp8q_quant_act_128x1_e5m2(_ptr(x), T, C, _ld(x), _ptr(qt), _ld(qt), _ptr(sf), _ld(sf),
                                          _stream(stream)), "fp8q_quant_act_128x1_e5m2")


def fp8q_gemm_blockscaled_fmt(a, a_fmt, sfa, b, b_fmt, sfb, sfb_mode, d, stream=None):
    """fp8q_gemm_blockscaled with operand formats FP8Q_FMT_E4M3 / FP8Q_FMT_E5M2."""
    M, K = a.shape
    N = b.shape[0]
    dt = FP8Q_OUT_F32 if d.dtype == torch.float32 else FP8Q_OUT_BF16
    _check(_lib.fp8q_gemm_blockscaled_fmt(_ptr(a), int(a_fmt), _ld(a), _ptr(sfa), _ld(sfa), _ptr(b), int(b_fmt), _ld(b),
                                          _ptr(sfb), _ld(sfb), int(sfb_mode), _ptr(d), _ld(d), dt, M, N, K,
                                          _stream(stream)), "fp8q_gemm_blockscaled_fmt")


def fp8q_moe_dispatch_layout(expert_ids, num_experts, rows, pos, offsets, workspace, stream=None):
    """Stable counting sort of the (token, slot) entries by expert (expert_ids int32 [T][k])."""
    T, k = expert_ids.shape
    _check(_lib.fp8q_moe_dispatch_layout(_ptr(expert_ids), T * k, k, int(num_experts), _ptr(rows), _ptr(pos),
                                         _ptr(offsets), _ptr(workspace), workspace.numel(), _stream(stream)),
           "fp8q_moe_dispatch_layout")


def fp8q_moe_dispatch_layout_noalloc(expert_ids, num_experts, rows, pos, offsets, stream=None):
    """fp8q_moe_dispatch_layout with no workspace argument: the library's fixed
    scratch array (FP8Q_LAYOUT_NOALLOC_SCRATCH_INTS int32) is used instead, so
    the call allocates nothing.  For callers that cannot allocate device memory
    when they call; calls that overlap on the GPU race on the shared array."""
    T, k = expert_ids.shape
    _check(_lib.fp8q_moe_dispatch_layout_noalloc(_ptr(expert_ids), T * k, k, int(num_experts), _ptr(rows), _ptr(pos),
                                                 _ptr(offsets), _stream(stream)),
           "fp8q_moe_dispatch_layout_noalloc")


def moe_dispatch_layout(expert_ids, num_experts, stream=None):
    """Returns (rows int32 [T*k], pos int32 [T][k], offsets int32 [E+1]) on expert_ids' device."""
    T, k = expert_ids.shape
    dev = expert_ids.device
    rows = torch.empty(T * k, dtype=torch.int32, device=dev)
    pos = torch.empty((T, k), dtype=torch.int32, device=dev)
    offsets = torch.empty(num_experts + 1, dtype=torch.int32, device=dev)
    ws = torch.empty(max(1, _lib.fp8q_moe_dispatch_layout_workspace(T * k, int(num_experts))), dtype=torch.int32,
                     device=dev)
    fp8q_moe_dispatch_layout(expert_ids, num_experts, rows, pos, offsets, ws, stream)
    return rows, pos, offsets


def fp8q_quant_act_1x128_gather_rowscales(x, rows, q, sf, stream=None):
    """Gather-quantize: q row m = 1x128 FP8 of x row rows[m]; sf row-major [M][ld >= K/128]."""
    M_src, K = x.shape
    M = rows.numel()
    _check(_lib.fp8q_quant_act_1x128_gather_rowscales(_ptr(x), M_src, K, _ld(x), _ptr(rows), M, _ptr(q), _ld(q),
                                                      _ptr(sf), _ld(sf), _stream(stream)),
           "fp8q_quant_act_1x128_gather_rowscales")


def fp8q_quant_act_1x128_scatter(x, pos, q, sf, stream=None):
    """Quantize each row of x once and write it to output rows pos[row][j] (pos int32 [M_src][k])."""
    M_src, K = x.shape
    k = pos.shape[1]
    _check(_lib.fp8q_quant_act_1x128_scatter(_ptr(x), M_src, K, _ld(x), _ptr(pos), k, q.shape[0], _ptr(q), _ld(q),
                                             _ptr(sf), _ld(sf), _stream(stream)), "fp8q_quant_act_1x128_scatter")


def fp8q_quant_act_1x128_scatter_rowscales(x, pos, q, sf, stream=None):
    """fp8q_quant_act_1x128_scatter with row-major scales sf [M_out][ld >= K/128]."""
    M_src, K = x.shape
    k = pos.shape[1]
    _check(_lib.fp8q_quant_act_1x128_scatter_rowscales(_ptr(x), M_src, K, _ld(x), _ptr(pos), k, q.shape[0], _ptr(q),
                                                       _ld(q), _ptr(sf), _ld(sf), _stream(stream)),
           "fp8q_quant_act_1x128_scatter_rowscales")


def fp8q_gather_rows_fp8(q_in, sf_in, rows, q_out, sf_out, stream=None):
    """q_out row m = q_in row rows[m]; scales row-major in, [K/128][ld >= M_out] out."""
    M_in, K = q_in.shape
    _check(_lib.fp8q_gather_rows_fp8(_ptr(q_in), _ld(q_in), _ptr(sf_in), _ld(sf_in), M_in, _ptr(rows), rows.numel(), K,
                                     _ptr(q_out), _ld(q_out), _ptr(sf_out), _ld(sf_out), _stream(stream)),
           "fp8q_gather_rows_fp8")


def fp8q_moe_regroup_order(all_offsets, world, rank, num_experts, rows, expert_offsets, stream=None):
    """rows int32 [M_recv] <- received row of each output row (local expert, then
    source rank); expert_offsets int32 [num_experts/world + 1].  all_offsets:
    int32 [world * (num_experts + 1)], every rank's layout offsets."""
    _check(_lib.fp8q_moe_regroup_order(_ptr(all_offsets), int(world), int(rank), int(num_experts), rows.numel(),
                                       _ptr(rows), _ptr(expert_offsets), _stream(stream)),
           "fp8q_moe_regroup_order")


def fp8q_quant_pertensor(x, q, amax_scale, stream=None):
    """Per-tensor baseline: amax_scale float32 [2] <- {max|x|, s}, q = e4m3(x / s)."""
    M, K = x.shape
    _check(_lib.fp8q_quant_pertensor(_ptr(x), M, K, _ld(x), _ptr(q), _ld(q), _ptr(amax_scale), _stream(stream)),
           "fp8q_quant_pertensor")


def fp8q_gemm_pertensor(a, scale_a, b, scale_b, d, stream=None):
    """d[M][N] = (*scale_a * *scale_b) * a[M][K] . b[N][K]^T, one TMEM accumulation over K."""
    M, K = a.shape
    N = b.shape[0]
    dt = FP8Q_OUT_F32 if d.dtype == torch.float32 else FP8Q_OUT_BF16
    _check(_lib.fp8q_gemm_pertensor(_ptr(a), _ld(a), _ptr(scale_a), _ptr(b), _ld(b), _ptr(scale_b), _ptr(d), _ld(d),
                                    dt, M, N, K, _stream(stream)), "fp8q_gemm_pertensor")


def fp8q_gemm_blockscaled_q1x128(a, sfa, b, sfb, dq, sfd, stream=None):
    """dq[M][N] uint8, sfd [N/128][ld >= M]: 1x128 quantization of the bf16 GEMM result."""
    M, K = a.shape
    N = b.shape[0]
    _check(_lib.fp8q_gemm_blockscaled_q1x128(_ptr(a), _ld(a), _ptr(sfa), _ld(sfa), _ptr(b), _ld(b), _ptr(sfb),
                                             _ld(sfb), _ptr(dq), _ld(dq), _ptr(sfd), _ld(sfd), M, N, K,
                                             _stream(stream)), "fp8q_gemm_blockscaled_q1x128")


def fp8q_grouped_gemm_blockscaled(a, sfa, w, sfw, group_offsets, d, stream=None):
    """Per-expert block-scaled GEMM; w [G][N][K], sfw [G][N/128][K/128], offsets int32 [G+1] on device."""
    M_total, K = a.shape
    G, N, _ = w.shape
    _check(_lib.fp8q_grouped_gemm_blockscaled(_ptr(a), _ld(a), _ptr(sfa), _ld(sfa), _ptr(w), _ptr(sfw),
                                              _ptr(group_offsets), G, M_total, _ptr(d), _ld(d), N, K,
                                              _stream(stream)), "fp8q_grouped_gemm_blockscaled")


def fp8q_grouped_gemm_blockscaled_q1x128(a, sfa, w, sfw, group_offsets, dq, sfd, stream=None):
    """Grouped GEMM whose per-expert rows come out as 1x128 E4M3 tiles (dq uint8 [M_total][N]) and scales."""
    M_total, K = a.shape
    G, N, _ = w.shape
    _check(_lib.fp8q_grouped_gemm_blockscaled_q1x128(_ptr(a), _ld(a), _ptr(sfa), _ld(sfa), _ptr(w), _ptr(sfw),
                                                     _ptr(group_offsets), G, M_total, _ptr(dq), _ld(dq), _ptr(sfd),
                                                     _ld(sfd), N, K, _stream(stream)),
           "fp8q_grouped_gemm_blockscaled_q1x128")


def fp8q_debug_cast_e4m3_bits(start: int, count: int, out, stream=None):
    _check(_lib.fp8q_debug_cast_e4m3_bits(ctypes.c_uint32(start & 0xFFFFFFFF), count, _ptr(out), _stream(stream)),
           "fp8q_debug_cast_e4m3_bits")


def fp8q_quant_act_1x128_ue8m0(x, q, sf_mx, stream=None):
    """Power-of-two scale study: x bf16 [M][K] -> q uint8 [M][K], sf_mx int32 [K/128][ceil(M/128)][128] atoms."""
    M, K = x.shape
    _check(_lib.fp8q_quant_act_1x128_ue8m0(_ptr(x), M, K, _ld(x), _ptr(q), _ld(q), _ptr(sf_mx), _stream(stream)),
           "fp8q_quant_act_1x128_ue8m0")


def fp8q_quant_w_128x128_ue8m0(w, q, sf_mx, stream=None):
    """Power-of-two scale study: w bf16 [N][K] -> q uint8 [N][K], sf_mx int32 [K/128][N/128][128] atoms."""
    N, K = w.shape
    _check(_lib.fp8q_quant_w_128x128_ue8m0(_ptr(w), N, K, _ld(w), _ptr(q), _ld(q), _ptr(sf_mx), _stream(stream)),
           "fp8q_quant_w_128x128_ue8m0")


def fp8q_gemm_mxf8_ue8m0(a, sfa_mx, b, sfb_mx, d, stream=None):
    """d bf16 [M][N] = a . b^T on the block-scaled MMA with UE8M0 scale atoms (study)."""
    M, K = a.shape
    N = b.shape[0]
    _check(_lib.fp8q_gemm_mxf8_ue8m0(_ptr(a), _ld(a), _ptr(sfa_mx), _ptr(b), _ld(b), _ptr(sfb_mx), _ptr(d), _ld(d),
                                     M, N, K, _stream(stream)), "fp8q_gemm_mxf8_ue8m0")


GEMM_CLOCK_KINDS = ("pair", "one_cta", "pertensor", "mx")


def fp8q_kernel_clock_counters(reset: bool = True) -> dict:
    """Effective SM clock inside the GEMM kernels since the last reset:
    {kind: {"cycles", "ns", "ctas", "mhz"}} for the kinds that ran."""
    buf = (ctypes.c_ulonglong * 12)()
    _check(_lib.fp8q_kernel_clock_counters(ctypes.cast(buf, ctypes.c_void_p), 1 if reset else 0),
           "fp8q_kernel_clock_counters")
    out = {}
    for i, kind in enumerate(GEMM_CLOCK_KINDS):
        cyc, ns, ctas = buf[3 * i], buf[3 * i + 1], buf[3 * i + 2]
        if ctas:
            out[kind] = {"cycles": cyc, "ns": ns, "ctas": ctas, "mhz": round(cyc / ns * 1e3, 1)}
    return out


def fp8q_debug_force_dense_kernel(choice: int):
    """FP8Q_DENSE_AUTO / FP8Q_DENSE_SINGLE / FP8Q_DENSE_PAIR for later dense GEMM calls."""
    _check(_lib.fp8q_debug_force_dense_kernel(int(choice)), "fp8q_debug_force_dense_kernel")


def fp8q_debug_wait_timeout(budget_cycles: int, stream=None):
    _check(_lib.fp8q_debug_wait_timeout(int(budget_cycles), _stream(stream)), "fp8q_debug_wait_timeout")


# ---------------------------------------------------------------- allocation helpers
def sf_ld(rows: int) -> int:
    """Leading dimension used for [K/128][ld] scale arrays (rows rounded up to 4)."""
    return (rows + 3) // 4 * 4


def quant_act_1x128(x, stream=None):
    M, K = x.shape
    q = torch.empty((M, K), dtype=torch.uint8, device=x.device)
    sf = torch.empty((K // 128, sf_ld(M)), dtype=torch.float32, device=x.device)
    fp8q_quant_act_1x128(x, q, sf, stream)
    return q, sf


def quant_act_1x128_ue8m0(x, stream=None):
    M, K = x.shape
    q = torch.empty((M, K), dtype=torch.uint8, device=x.device)
    sf = torch.empty((K // 128, (M + 127) // 128, 128), dtype=torch.int32, device=x.device)
    fp8q_quant_act_1x128_ue8m0(x, q, sf, stream)
    return q, sf


def quant_w_128x128_ue8m0(w, stream=None):
    N, K = w.shape
    q = torch.empty((N, K), dtype=torch.uint8, device=w.device)
    sf = torch.empty((K // 128, N // 128, 128), dtype=torch.int32, device=w.device)
    fp8q_quant_w_128x128_ue8m0(w, q, sf, stream)
    return q, sf


def quant_pertensor(x, stream=None):
    """Returns (q uint8 [M][K], amax_scale float32 [2] = {amax, s}) on x's device."""
    M, K = x.shape
    q = torch.empty((M, K), dtype=torch.uint8, device=x.device)
    amax_scale = torch.empty(2, dtype=torch.float32, device=x.device)
    fp8q_quant_pertensor(x, q, amax_scale, stream)
    return q, amax_scale


def quant_act_dual(x, stream=None):
    """Returns (q, sf, qt, sft): the 1x128 and the 128x1 quantizations of x from one read."""
    T, C = x.shape
    q = torch.empty((T, C), dtype=torch.uint8, device=x.device)
    sf = torch.empty((C // 128, sf_ld(T)), dtype=torch.float32, device=x.device)
    qt = torch.empty((C, T), dtype=torch.uint8, device=x.device)
    sft = torch.empty((T // 128, sf_ld(C)), dtype=torch.float32, device=x.device)
    fp8q_quant_act_dual(x, q, sf, qt, sft, stream)
    return q, sf, qt, sft


def quant_act_128x1(x, stream=None):
    T, C = x.shape
    qt = torch.empty((C, T), dtype=torch.uint8, device=x.device)
    sf = torch.empty((T // 128, sf_ld(C)), dtype=torch.float32, device=x.device)
    fp8q_quant_act_128x1(x, qt, sf, stream)
    return qt, sf


def quant_w_128x128(w, transposed: bool = False, stream=None):
    N, K = w.shape
    q = torch.empty((N, K), dtype=torch.uint8, device=w.device)
    sf = torch.empty((N // 128, K // 128), dtype=torch.float32, device=w.device)
    qt = sft = None
    if transposed:
        qt = torch.empty((K, N), dtype=torch.uint8, device=w.device)
        sft = torch.empty((K // 128, N // 128), dtype=torch.float32, device=w.device)
    fp8q_quant_w_128x128(w, q, sf, qt, sft, stream)
    return (q, sf, qt, sft) if transposed else (q, sf)
