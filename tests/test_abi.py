"""The C-ABI boundary on the host (no GPU needed): the library loads, exports
every entry point include/fp8q.h declares, and rejects invalid arguments with
the documented status codes before touching a device."""
import ctypes
import os
import re

import pytest

from common import load_fp8q

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fp8q.h")

FAKE = 1 << 20        # 16-byte aligned fake device address (never dereferenced)


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fp8q_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def fp8q():
    return load_fp8q()


def test_header_declares_the_five_entry_points():
    syms = declared_symbols()
    for name in ("fp8q_quant_act_1x128", "fp8q_quant_act_128x1", "fp8q_quant_w_128x128",
                 "fp8q_gemm_blockscaled", "fp8q_grouped_gemm_blockscaled"):
        assert name in syms


def test_library_exports_every_declared_symbol(fp8q):
    lib = ctypes.CDLL(fp8q.LIB_PATH)
    for name in declared_symbols():
        assert hasattr(lib, name), name
    assert set(fp8q.EXPORTS) == set(declared_symbols())


def test_version_and_status_strings(fp8q):
    assert fp8q.fp8q_version() >= 100
    for code in range(8):
        assert fp8q.fp8q_status_string(code) != "unknown status"
    assert fp8q.fp8q_status_string(99) == "unknown status"


def test_quant_act_validation(fp8q):
    L = fp8q.lib()
    INV, ALN = fp8q.FP8Q_ERR_INVALID_ARG, fp8q.FP8Q_ERR_ALIGNMENT
    assert L.fp8q_quant_act_1x128(FAKE, 4, 100, 100, FAKE, 112, FAKE, 4, None) == INV    # K % 128
    assert L.fp8q_quant_act_1x128(FAKE, 4, 128, 64, FAKE, 128, FAKE, 4, None) == INV     # ldx < K
    assert L.fp8q_quant_act_1x128(FAKE, 4, 128, 128, FAKE, 128, FAKE, 3, None) == INV    # ld_sf < M
    assert L.fp8q_quant_act_1x128(FAKE, -1, 128, 128, FAKE, 128, FAKE, 4, None) == INV
    assert L.fp8q_quant_act_1x128(FAKE + 8, 4, 128, 128, FAKE, 128, FAKE, 4, None) == ALN
    assert L.fp8q_quant_act_1x128(FAKE, 4, 128, 132, FAKE, 128, FAKE, 4, None) == ALN    # ldx % 8
    assert L.fp8q_quant_act_1x128(FAKE, 4, 128, 128, FAKE, 136, FAKE, 4, None) == ALN    # ldq % 16
    assert L.fp8q_quant_act_1x128(None, 4, 128, 128, FAKE, 128, FAKE, 4, None) == INV
    assert L.fp8q_quant_act_1x128(None, 0, 128, 128, None, 128, None, 0, None) == 0     # empty: nothing launched
    assert L.fp8q_quant_act_128x1(FAKE, 100, 8, 8, FAKE, 128, FAKE, 8, None) == INV      # T % 128
    assert L.fp8q_quant_act_128x1(FAKE, 128, 12, 16, FAKE, 128, FAKE, 12, None) == INV   # C % 8
    assert L.fp8q_quant_act_128x1(FAKE, 128, 8, 8, FAKE, 120, FAKE, 8, None) == INV      # ldqt < T
    assert L.fp8q_quant_act_128x1(FAKE, 128, 8, 8, FAKE + 4, 128, FAKE, 8, None) == ALN
    assert L.fp8q_quant_act_128x1(None, 0, 8, 8, None, 0, None, 8, None) == 0


def test_quant_dual_validation(fp8q):
    L = fp8q.lib()
    INV, ALN = fp8q.FP8Q_ERR_INVALID_ARG, fp8q.FP8Q_ERR_ALIGNMENT

    def qd(x=FAKE, T=256, C=256, ldx=256, q=FAKE, ldq=256, sf=FAKE, ld_sf=256, qt=FAKE, ldqt=256, sft=FAKE,
           ld_sft=256):
        return L.fp8q_quant_act_dual(x, T, C, ldx, q, ldq, sf, ld_sf, qt, ldqt, sft, ld_sft, None)

    assert qd(T=200) == INV and qd(C=200) == INV and qd(T=-128) == INV          # whole 128 x 128 tiles
    assert qd(ldx=128) == INV and qd(ldq=128) == INV and qd(ldqt=128) == INV
    assert qd(ld_sf=128) == INV and qd(ld_sft=128) == INV
    assert qd(x=None) == INV and qd(qt=None) == INV and qd(sft=None) == INV
    assert qd(x=FAKE + 8) == ALN and qd(qt=FAKE + 8) == ALN and qd(ldx=260) == ALN and qd(ldq=264) == ALN
    assert qd(ldqt=264) == ALN and qd(sf=FAKE + 2) == ALN
    assert qd(T=0, x=None, q=None, sf=None, qt=None, sft=None) == 0          # empty: nothing launched


def test_quant_gather_validation(fp8q):
    L = fp8q.lib()
    INV, ALN = fp8q.FP8Q_ERR_INVALID_ARG, fp8q.FP8Q_ERR_ALIGNMENT

    def qg(x=FAKE, Ms=16, K=256, ldx=256, rows=FAKE, M=8, q=FAKE, ldq=256, sf=FAKE, ld_sf=8):
        return L.fp8q_quant_act_1x128_gather(x, Ms, K, ldx, rows, M, q, ldq, sf, ld_sf, None)

    assert qg(Ms=-1) == INV and qg(M=-1) == INV and qg(K=200) == INV
    assert qg(ldx=128) == INV and qg(ldq=128) == INV and qg(ld_sf=4) == INV
    assert qg(rows=None) == INV and qg(x=None) == INV
    assert qg(rows=FAKE + 2) == ALN and qg(x=FAKE + 8) == ALN and qg(ldq=264) == ALN
    assert qg(M=0, rows=None, q=None, sf=None, ld_sf=0) == 0    # no output rows: nothing launched


def test_scale_policy_validation(fp8q):
    L = fp8q.lib()
    INV, ALN = fp8q.FP8Q_ERR_INVALID_ARG, fp8q.FP8Q_ERR_ALIGNMENT

    def qs(M=8, K=256, ldx=256, sf=FAKE, ld_sf=8, q=FAKE, ldq=256, amax=FAKE, ld_amax=8, clipped=FAKE):
        return L.fp8q_quant_act_1x128_scaled(FAKE, M, K, ldx, sf, ld_sf, q, ldq, amax, ld_amax, clipped, None)

    assert qs(K=200) == INV and qs(ld_sf=4) == INV and qs(ld_amax=4) == INV and qs(ldq=128) == INV
    assert qs(sf=None) == INV and qs(q=None) == INV
    assert qs(sf=FAKE + 2) == ALN and qs(clipped=FAKE + 4) == ALN and qs(ldq=264) == ALN
    assert qs(M=0, sf=None, q=None, amax=None, clipped=None, ld_sf=0, ld_amax=0) == 0
    def qp(M=64, K=256, ldx=256, rank=2, q=FAKE, ldq=256, sf=FAKE, ld_sf=64, clipped=None):
        return L.fp8q_quant_act_1x128_percentile(FAKE, M, K, ldx, rank, q, ldq, sf, ld_sf, clipped, None)

    assert qp(rank=0) == INV and qp(rank=129) == INV and qp(rank=-3) == INV
    assert qp(K=200) == INV and qp(ld_sf=4) == INV and qp(ldq=128) == INV and qp(sf=None) == INV
    assert qp(ldq=264) == ALN and qp(clipped=FAKE + 4) == ALN and qp(sf=FAKE + 2) == ALN
    assert qp(M=0, q=None, sf=None, ld_sf=0) == 0
    assert L.fp8q_quant_act_1x128_e5m2(FAKE, 4, 200, 256, FAKE, 256, FAKE, 4, None) == INV     # K % 128
    assert L.fp8q_quant_act_1x128_e5m2(FAKE, 4, 256, 256, FAKE, 264, FAKE, 4, None) == ALN     # ldq % 16
    assert L.fp8q_quant_act_128x1_e5m2(FAKE, 100, 8, 8, FAKE, 128, FAKE, 8, None) == INV       # T % 128
    assert L.fp8q_quant_act_128x1_e5m2(FAKE, 0, 8, 8, None, 128, None, 8, None) == 0
    F = L.fp8q_gemm_blockscaled_fmt
    assert F(FAKE, 2, 256, FAKE, 256, FAKE, 0, 256, FAKE, 2, 0, FAKE, 256, 0, 256, 256, 256, None) == INV   # a_fmt
    assert F(FAKE, 1, 256, FAKE, 256, FAKE, -1, 256, FAKE, 2, 0, FAKE, 256, 0, 256, 256, 256, None) == INV  # b_fmt
    assert F(FAKE, 1, 256, FAKE, 256, FAKE, 0, 256, FAKE, 2, 0, FAKE, 256, 3, 256, 256, 256, None) == INV   # dtype
    assert F(FAKE, 1, 256, FAKE, 256, FAKE, 0, 256, FAKE, 2, 0, FAKE, 256, 0, 256, 200, 256, None) == INV   # N % 128
    R = L.fp8q_requant_1x128_to_128x1
    assert R(FAKE, 100, 256, 256, FAKE, 128, FAKE, 128, FAKE, 256, None) == INV     # T % 128
    assert R(FAKE, 128, 200, 256, FAKE, 128, FAKE, 128, FAKE, 256, None) == INV     # C % 128
    assert R(FAKE, 128, 256, 256, FAKE, 64, FAKE, 128, FAKE, 256, None) == INV      # ld_sf_in < T
    assert R(FAKE, 128, 256, 256, FAKE + 4, 128, FAKE, 128, FAKE, 256, None) == ALN  # sf_in 16-byte
    assert R(FAKE, 128, 256, 256, FAKE, 130, FAKE, 128, FAKE, 256, None) == ALN     # ld_sf_in % 4
    assert R(FAKE, 128, 256, 264, FAKE, 128, FAKE, 128, FAKE, 256, None) == ALN     # ldq % 16
    assert R(FAKE, 0, 256, 256, None, 0, None, 0, None, 256, None) == 0
    P = L.fp8q_quant_pertensor
    assert P(FAKE, 4, 100, 128, FAKE, 128, FAKE, None) == INV                       # K % 8
    assert P(FAKE, 4, 128, 120, FAKE, 128, FAKE, None) == INV                       # ldx < K
    assert P(FAKE, 4, 128, 128, FAKE, 128, None, None) == INV                       # no scale output
    assert P(FAKE, 4, 128, 128, FAKE + 4, 128, FAKE, None) == ALN
    assert P(FAKE, 4, 128, 128, FAKE, 128, FAKE + 2, None) == ALN
    G = L.fp8q_gemm_pertensor
    assert G(FAKE, 256, FAKE, FAKE, 256, FAKE, FAKE, 256, 0, 0, 256, 256, None) == INV        # M = 0
    assert G(FAKE, 256, FAKE, FAKE, 256, FAKE, FAKE, 256, 0, 8, 200, 256, None) == INV        # N % 128
    assert G(FAKE, 256, FAKE, FAKE, 256, FAKE, FAKE, 256, 2, 8, 256, 256, None) == INV        # dtype
    assert G(FAKE, 256, None, FAKE, 256, FAKE, FAKE, 256, 0, 8, 256, 256, None) == INV        # no scale
    assert G(FAKE, 264, FAKE, FAKE, 256, FAKE, FAKE, 256, 0, 8, 256, 256, None) == ALN        # lda % 16
    assert G(FAKE, 256, FAKE + 2, FAKE, 256, FAKE, FAKE, 256, 0, 8, 256, 256, None) == ALN
    U = L.fp8q_scale_history_update
    assert U(3, 0.5, FAKE, FAKE, FAKE, 16, None) == INV and U(-1, 0.5, FAKE, FAKE, FAKE, 16, None) == INV
    assert U(1, 1.5, FAKE, FAKE, FAKE, 16, None) == INV and U(1, -0.1, FAKE, FAKE, FAKE, 16, None) == INV
    assert U(1, float("nan"), FAKE, FAKE, FAKE, 16, None) == INV
    assert U(1, 0.5, None, FAKE, FAKE, 16, None) == INV and U(1, 0.5, FAKE + 2, FAKE, FAKE, 16, None) == ALN
    assert U(2, 0.5, None, None, None, 0, None) == 0


def test_quant_w_validation(fp8q):
    L = fp8q.lib()
    INV, ALN = fp8q.FP8Q_ERR_INVALID_ARG, fp8q.FP8Q_ERR_ALIGNMENT
    assert L.fp8q_quant_w_128x128(FAKE, 100, 128, 128, FAKE, 128, FAKE, 1, None, 0, None, 0, None) == INV
    assert L.fp8q_quant_w_128x128(FAKE, 128, 256, 256, FAKE, 256, FAKE, 1, None, 0, None, 0, None) == INV  # ld_sf
    assert L.fp8q_quant_w_128x128(FAKE, 128, 128, 128, FAKE, 128, FAKE, 1, FAKE, 64, None, 0, None) == INV  # ldqt
    assert L.fp8q_quant_w_128x128(FAKE, 128, 128, 128, FAKE, 128, FAKE, 1, FAKE + 1, 128, None, 0, None) == ALN
    assert L.fp8q_quant_w_128x128(FAKE, 256, 128, 128, FAKE, 128, FAKE, 1, None, 0, FAKE, 1, None) == INV  # ld_sft


def test_gemm_validation(fp8q):
    L = fp8q.lib()
    INV, ALN = fp8q.FP8Q_ERR_INVALID_ARG, fp8q.FP8Q_ERR_ALIGNMENT
    BLK, ROW, BF, F32 = 0, 1, 0, 1

    def g(M=8, N=256, K=256, lda=256, ldb=256, ld_sfa=8, ld_sfb=2, mode=BLK, ldd=256, dt=BF,
          a=FAKE, b=FAKE, d=FAKE, sfa=FAKE, sfb=FAKE):
        return L.fp8q_gemm_blockscaled(a, lda, sfa, ld_sfa, b, ldb, sfb, ld_sfb, mode, d, ldd, dt, M, N, K, None)

    assert g(M=0) == INV
    assert g(N=192) == INV and g(K=100) == INV and g(N=0) == INV and g(K=0) == INV
    assert g(lda=128) == INV and g(ldb=128) == INV and g(ldd=128) == INV and g(ld_sfa=4) == INV
    assert g(mode=2) == INV and g(dt=7) == INV
    assert g(ld_sfb=1) == INV                      # block mode needs ld_sfb >= K/128
    assert g(mode=ROW, ld_sfb=128) == INV          # row mode needs ld_sfb >= N
    assert g(a=FAKE + 8) == ALN and g(b=FAKE + 8) == ALN and g(d=FAKE + 8) == ALN
    assert g(lda=264) == ALN and g(ldb=264) == ALN
    assert g(ldd=260) == ALN                       # 260 bf16 = 520 bytes, not a multiple of 16
    assert g(mode=ROW, ld_sfb=258) == ALN          # row-mode scales are bulk-copied: ld % 4
    assert g(sfa=FAKE + 2) == ALN
    assert g(a=None) == INV


def test_gemm_q1x128_validation(fp8q):
    L = fp8q.lib()
    INV, ALN = fp8q.FP8Q_ERR_INVALID_ARG, fp8q.FP8Q_ERR_ALIGNMENT

    def gq(M=8, N=256, K=256, ldd=256, sfd=FAKE, ld_sfd=8, d=FAKE, ld_sfb=2):
        return L.fp8q_gemm_blockscaled_q1x128(FAKE, K, FAKE, 8, FAKE, K, FAKE, ld_sfb, d, ldd, sfd, ld_sfd, M, N, K,
                                              None)

    assert gq(M=0) == INV and gq(N=200) == INV and gq(ldd=128) == INV
    assert gq(ld_sfd=4) == INV and gq(sfd=None) == INV and gq(ld_sfb=1) == INV
    assert gq(ldd=264) == ALN                       # FP8 rows: ld % 16
    assert gq(sfd=FAKE + 2) == ALN and gq(d=FAKE + 8) == ALN

    def ggq(G=4, Mt=64, ldd=256, sfd=FAKE, ld_sfd=64):
        return L.fp8q_grouped_gemm_blockscaled_q1x128(FAKE, 256, FAKE, 64, FAKE, FAKE, FAKE, G, Mt, FAKE, ldd, sfd,
                                                      ld_sfd, 256, 256, None)

    assert ggq(G=0) == INV and ggq(ld_sfd=32) == INV and ggq(sfd=None) == INV and ggq(ldd=128) == INV
    assert ggq(ldd=264) == ALN and ggq(sfd=FAKE + 1) == ALN
    assert ggq(Mt=0, sfd=None, ld_sfd=0) == 0


def test_grouped_validation(fp8q):
    L = fp8q.lib()
    INV, UNS = fp8q.FP8Q_ERR_INVALID_ARG, fp8q.FP8Q_ERR_UNSUPPORTED

    def gg(G=4, Mt=64, N=256, K=256, lda=256, ld_sfa=64, ldd=256):
        return L.fp8q_grouped_gemm_blockscaled(FAKE, lda, FAKE, ld_sfa, FAKE, FAKE, FAKE, G, Mt, FAKE, ldd, N, K, None)

    assert gg(G=0) == INV and gg(Mt=-1) == INV and gg(N=200) == INV and gg(K=64) == INV
    assert gg(G=4096) == UNS
    assert gg(ld_sfa=32) == INV and gg(lda=128) == INV and gg(ldd=128) == INV
    assert gg(Mt=0, ld_sfa=0) == 0                # no rows: nothing launched


def test_debug_entry_validation(fp8q):
    L = fp8q.lib()
    INV = fp8q.FP8Q_ERR_INVALID_ARG
    assert L.fp8q_debug_cast_e4m3_bits(0, -1, FAKE, None) == INV
    assert L.fp8q_debug_cast_e4m3_bits(0, (1 << 32) + 1, FAKE, None) == INV
    assert L.fp8q_debug_cast_e4m3_bits(0, 0, None, None) == 0
    assert L.fp8q_debug_wait_timeout(0, None) == INV
    assert L.fp8q_debug_wait_timeout((1 << 34) + 1, None) == INV


def test_regroup_order_validation(fp8q):
    L = fp8q.lib()
    INV, UNS, ALN = fp8q.FP8Q_ERR_INVALID_ARG, fp8q.FP8Q_ERR_UNSUPPORTED, fp8q.FP8Q_ERR_ALIGNMENT

    def ro(off=FAKE, world=2, rank=0, E=16, M=100, rows=FAKE, eo=FAKE):
        return L.fp8q_moe_regroup_order(off, world, rank, E, M, rows, eo, None)

    assert ro(world=0) == INV and ro(rank=2) == INV and ro(rank=-1) == INV
    assert ro(E=0) == INV and ro(E=2048, world=1) == INV and ro(E=15) == INV     # 15 % 2 != 0
    assert ro(M=-1) == INV and ro(M=1 << 31) == UNS
    assert ro(off=None) == INV and ro(eo=None) == INV and ro(rows=None) == INV
    assert ro(off=FAKE + 2) == ALN and ro(rows=FAKE + 1) == ALN and ro(eo=FAKE + 3) == ALN


def test_checked_build_exports_the_same_symbols(fp8q):
    """The checked build (-DFP8Q_CHECKS) is the same C ABI and says so; the
    default build says it is not checked."""
    import importlib.util
    spec = importlib.util.spec_from_file_location("fp8q_build", os.path.join(ROOT, "fine_grained_fp8_x128_b200", "build.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    checked = ctypes.CDLL(b.build(checks=True))
    for name in declared_symbols():
        assert hasattr(checked, name), name
    assert checked.fp8q_build_checks() == 1
    assert ctypes.CDLL(b.LIB).fp8q_build_checks() == 0
    assert fp8q.fp8q_status_string(fp8q.FP8Q_ERR_BOUNDS) != "unknown status"
