"""The C ABI library loads and exports every symbol include/dbf.h declares;
host-side argument checks (which return before any CUDA call) behave."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dbf.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(dbf_[a-z_0-9]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    import double_binary_rank_b200 as dbf
    return dbf._lib


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("dbf_pack_signs", "dbf_forward", "dbf_forward_segmented", "dbf_unpack_signs",
              "dbf_workspace_bytes", "dbf_packed_bytes", "dbf_status_string"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_binding_covers_header():
    import double_binary_rank_b200 as dbf
    assert sorted(dbf.EXPORTED) == declared_functions()


def test_packed_bytes(lib):
    import double_binary_rank_b200 as dbf
    assert dbf.packed_bytes(3, 33) == 3 * 2 * 4
    assert dbf.packed_bytes(11008, 5888) == 8101888
    assert dbf.packed_bytes(5888, 4096) == 3014656
    assert dbf.packed_bytes(0, 5) == 0


def test_status_strings(lib):
    import double_binary_rank_b200 as dbf
    assert dbf.status_string(dbf.OK) == "ok"
    assert "workspace" in dbf.status_string(dbf.ERR_WORKSPACE)
    assert dbf.version().startswith("dbf-b200")


def _layer(M=64, N=48, R=32, ell=1, p=0x1000):
    import double_binary_rank_b200 as dbf
    return dbf.DbfLayerC(M, N, R, ell, p, p, p, p, p)


def test_forward_rejects_bad_arguments_without_launch(lib):
    import double_binary_rank_b200 as dbf
    L = _layer()
    f = lib.dbf_forward
    by = ctypes.byref
    assert f(None, 0x1000, dbf.F32, 0x1000, dbf.F32, 4, 0, 0, 0x1000, 1 << 20, None) == dbf.ERR_INVALID_ARG
    assert f(by(_layer(ell=0)), 0x1000, dbf.F32, 0x1000, dbf.F32, 4, 0, 0, 0x1000, 1 << 20, None) == dbf.ERR_INVALID_ARG
    assert f(by(_layer(ell=9)), 0x1000, dbf.F32, 0x1000, dbf.F32, 4, 0, 0, 0x1000, 1 << 20, None) == dbf.ERR_INVALID_ARG
    assert f(by(_layer(R=-1)), 0x1000, dbf.F32, 0x1000, dbf.F32, 4, 0, 0, 0x1000, 1 << 20, None) == dbf.ERR_INVALID_ARG
    assert f(by(L), 0x1000, dbf.F16, 0x1000, dbf.F32, 4, 0, 0, 0x1000, 1 << 20, None) == dbf.ERR_INVALID_ARG
    assert f(by(L), 0x1000, dbf.F32, 0x1000, dbf.I8, 4, 0, 0, 0x1000, 1 << 20, None) == dbf.ERR_INVALID_ARG
    assert f(by(L), 0x1000, dbf.F32, 0x1000, dbf.F32, 4, 0, 7, 0x1000, 1 << 20, None) == dbf.ERR_INVALID_ARG
    assert f(by(L), 0x1000, dbf.F32, 0x1000, dbf.F32, 4, 4, 0, 0x1000, 1 << 20, None) == dbf.ERR_INVALID_ARG
    assert f(by(L), 0x1008, dbf.F32, 0x1000, dbf.F32, 4, 0, 0, 0x1000, 1 << 20, None) == dbf.ERR_ALIGNMENT
    assert f(by(L), 0x1000, dbf.F32, 0x1004, dbf.F32, 4, 0, 0, 0x1000, 1 << 20, None) == dbf.ERR_ALIGNMENT
    assert f(by(_layer(p=0x1004)), 0x1000, dbf.F32, 0x1000, dbf.F32, 4, 0, 0, 0x1000, 1 << 20, None) == dbf.ERR_ALIGNMENT
    assert f(by(L), 0x1000, dbf.F32, 0x1000, dbf.F32, 4, 0, 0, None, 0, None) == dbf.ERR_WORKSPACE
    assert f(by(L), 0x1000, dbf.F32, 0x1000, dbf.F32, 4, 0, 0, 0x1000, 16, None) == dbf.ERR_WORKSPACE
    # GEMM path needs M % 128 == 0 and R % 128 == 0
    assert f(by(L), 0x1000, dbf.F32, 0x1000, dbf.F32, 4, 0, dbf.PATH_GEMM, 0x1000, 1 << 30, None) == dbf.ERR_UNSUPPORTED
    # T == 0 is a no-op
    assert f(by(L), None, dbf.F32, None, dbf.F32, 0, 0, 0, None, 0, None) == dbf.OK


def test_workspace_query(lib):
    import double_binary_rank_b200 as dbf
    L = _layer(M=64, N=48, R=32, ell=2)
    ws = lib.dbf_workspace_bytes(ctypes.byref(L), 5, dbf.PATH_GEMV)
    assert ws >= 5 * 2 * 32 * 4 and ws % 256 == 0
    assert lib.dbf_workspace_bytes(None, 5, dbf.PATH_GEMV) == 0
    assert lib.dbf_segmented_workspace_bytes(32, 2, 256) >= 256 * 2 * 32 * 4


def test_pack_rejects_bad_arguments(lib):
    import double_binary_rank_b200 as dbf
    f = lib.dbf_pack_signs
    assert f(None, dbf.I8, 4, 4, 0x1000, 16, None, None) == dbf.ERR_INVALID_ARG
    assert f(0x1000, dbf.I8, 0, 4, 0x1000, 16, None, None) == dbf.ERR_INVALID_ARG
    assert f(0x1000, dbf.I8, 4, 40, 0x1000, 16, None, None) == dbf.ERR_INVALID_ARG   # dst too small
    assert f(0x1000, 9, 4, 4, 0x1000, 16, None, None) == dbf.ERR_INVALID_ARG
    assert f(0x1002, dbf.F32, 4, 4, 0x1000, 16, None, None) == dbf.ERR_ALIGNMENT
    assert f(0x1000, dbf.I8, 4, 4, 0x1002, 16, None, None) == dbf.ERR_ALIGNMENT


def test_segmented_rejects_bad_arguments(lib):
    import double_binary_rank_b200 as dbf
    f = lib.dbf_forward_segmented
    a = 0x1000
    assert f(a, 4, a, a, 3, 0, 1, 64, 64, a, dbf.F32, a, dbf.F32, 8, 0, a, 1 << 20, None, None) == dbf.ERR_INVALID_ARG
    assert f(a, 4, a, a, 3, 32, 9, 64, 64, a, dbf.F32, a, dbf.F32, 8, 0, a, 1 << 20, None, None) == dbf.ERR_INVALID_ARG
    assert f(a, 4, a, a, 3, 32, 1, 64, 64, a, dbf.F32, a, dbf.F32, 8, 0, None, 0, None, None) == dbf.ERR_WORKSPACE
    assert f(a, 4, a + 2, a, 3, 32, 1, 64, 64, a, dbf.F32, a, dbf.F32, 8, 0, a, 1 << 20, None, None) == dbf.ERR_ALIGNMENT
    assert f(a, 4, a, a, 0, 32, 1, 64, 64, a, dbf.F32, a, dbf.F32, 8, 0, None, 0, None, None) == dbf.OK


def test_forward_launch_count(lib):
    # host-side query, no launch: GEMM path = pre-pass + one launch of both
    # stages when both are at least 32 K steps deep (M >= 2048, ell R >= 2048),
    # else pre-pass + two stages; GEMV path = one kernel whenever M <= 8192 (any
    # token count: the columns are cut into chunks), else two
    import double_binary_rank_b200 as dbf
    by = ctypes.byref
    L = _layer(M=4096, N=11008, R=5888, ell=1)
    assert lib.dbf_forward_launches(by(L), 2048, dbf.PATH_AUTO) == 2
    assert lib.dbf_forward_launches(by(_layer(M=1024, N=4096, R=4096, ell=1)), 2048, dbf.PATH_GEMM) == 3
    assert lib.dbf_forward_launches(by(_layer(M=2048, N=512, R=1024, ell=1)), 2048, dbf.PATH_GEMM) == 3
    assert lib.dbf_forward_launches(by(_layer(M=2048, N=512, R=1024, ell=2)), 2048, dbf.PATH_GEMM) == 2
    assert lib.dbf_forward_launches(by(L), 1, dbf.PATH_AUTO) == 1
    for T in (7, 8, 64, 2048):
        assert lib.dbf_forward_launches(by(L), T, dbf.PATH_GEMV) == 1
    L1 = _layer(M=4096, N=4096, R=64, ell=1)
    for T in (8, 9, 64):
        assert lib.dbf_forward_launches(by(L1), T, dbf.PATH_GEMV) == 1
    L2 = _layer(M=256, N=256, R=16, ell=3)
    assert lib.dbf_forward_launches(by(L2), 3, dbf.PATH_GEMV) == 1
    L3 = _layer(M=8224, N=256, R=96, ell=1)   # M above 8192
    assert lib.dbf_forward_launches(by(L3), 1, dbf.PATH_GEMV) == 2
    assert lib.dbf_forward_launches(by(L), 0, dbf.PATH_AUTO) == 0
    assert lib.dbf_forward_launches(None, 1, dbf.PATH_AUTO) == 0


def test_backward_rejects_bad_arguments_without_launch(lib):
    import double_binary_rank_b200 as dbf
    by = ctypes.byref
    L = _layer(M=256, N=384, R=128, ell=2)
    f = lib.dbf_backward
    p = 0x1000
    # flags other than ACCUMULATE, bad dtypes, null operands
    assert f(by(L), p, p, p, dbf.F32, p, dbf.F32, 4, p, p, p, p, None, None, 2, p, 1 << 30, None) == dbf.ERR_INVALID_ARG
    assert f(by(L), p, p, p, dbf.I8, p, dbf.F32, 4, p, p, p, p, None, None, 0, p, 1 << 30, None) == dbf.ERR_INVALID_ARG
    assert f(by(L), None, p, p, dbf.F32, p, dbf.F32, 4, p, p, p, p, None, None, 0, p, 1 << 30, None) == dbf.ERR_INVALID_ARG
    # shapes off the 128 grid are not served
    L2 = _layer(M=200, N=384, R=128)
    assert f(by(L2), p, p, p, dbf.F32, p, dbf.F32, 4, p, p, p, p, None, None, 0, p, 1 << 30, None) == dbf.ERR_UNSUPPORTED
    assert lib.dbf_backward_workspace_bytes(by(L2), 4, 0) == 0
    # alignment and workspace
    assert f(by(L), p, p, p + 4, dbf.F32, p, dbf.F32, 4, p, p, p, p, None, None, 0, p, 1 << 30, None) == dbf.ERR_ALIGNMENT
    need = lib.dbf_backward_workspace_bytes(by(L), 4, 0)
    assert lib.dbf_backward_workspace_bytes(by(L), 4, 1) > need
    assert need >= 256 + 2 * 4 * (256 + 384) * 2 + 2 * 4 * 128 * 8
    assert f(by(L), p, p, p, dbf.F32, p, dbf.F32, 4, p, p, p, p, None, None, 0, p, need - 1, None) == dbf.ERR_WORKSPACE
    # T == 0 is a no-op
    assert f(by(L), p, p, p, dbf.F32, p, dbf.F32, 0, p, p, p, p, None, None, 0, None, 0, None) == dbf.OK


def test_transpose_rejects_bad_arguments(lib):
    import double_binary_rank_b200 as dbf
    t = lib.dbf_transpose_signs
    assert t(None, 4, 4, 0x1000, 1 << 20, None) == dbf.ERR_INVALID_ARG
    assert t(0x1000, 40, 64, 0x1000, lib.dbf_packed_bytes(64, 40) - 1, None) == dbf.ERR_INVALID_ARG
    assert t(0x1002, 40, 64, 0x1000, 1 << 20, None) == dbf.ERR_ALIGNMENT


def test_ste_rejects_bad_arguments(lib):
    import double_binary_rank_b200 as dbf
    st = lib.dbf_ste_backward
    assert st(0x1000, 0x1000, dbf.I8, 16, 1.0, 0x1000, 0, None) == dbf.ERR_INVALID_ARG
    assert st(0x1000, 0x1000, dbf.F32, 16, float("nan"), 0x1000, 0, None) == dbf.ERR_INVALID_ARG
    assert st(0x1000, 0x1000, dbf.F32, 16, 1.0, 0x1000, 4, None) == dbf.ERR_INVALID_ARG
    assert st(0x1002, 0x1000, dbf.F32, 16, 1.0, 0x1000, 0, None) == dbf.ERR_ALIGNMENT
    assert st(None, None, dbf.F32, 0, 1.0, None, 0, None) == dbf.OK


def test_mbok_rejects_bad_arguments(lib):
    import double_binary_rank_b200 as dbf
    by = ctypes.byref
    p = 0x1000
    L = dbf.DbfMbokLayerC(256, 100, 3, p, p, p)
    f = lib.dbf_mbok_forward
    need = lib.dbf_mbok_workspace_bytes(by(L), 8)
    assert need >= 256 + 8 * 3 * 256 * 2
    assert f(by(L), p, dbf.F32, p, dbf.F32, 8, 2, p, need, None) == dbf.ERR_INVALID_ARG
    assert f(by(L), p, dbf.I8, p, dbf.F32, 8, 0, p, need, None) == dbf.ERR_INVALID_ARG
    assert f(by(dbf.DbfMbokLayerC(200, 100, 3, p, p, p)), p, dbf.F32, p, dbf.F32, 8, 0, p, need, None) == dbf.ERR_UNSUPPORTED
    assert lib.dbf_mbok_workspace_bytes(by(dbf.DbfMbokLayerC(200, 100, 3, p, p, p)), 8) == 0
    assert f(by(L), p + 8, dbf.F32, p, dbf.F32, 8, 0, p, need, None) == dbf.ERR_ALIGNMENT
    assert f(by(L), p, dbf.F32, p, dbf.F32, 8, 0, p, need - 1, None) == dbf.ERR_WORKSPACE
    assert f(by(L), None, dbf.F32, None, dbf.F32, 0, 0, None, 0, None) == dbf.OK


def test_segmented_planned_rejects_bad_tables(lib):
    import numpy as np
    import double_binary_rank_b200 as dbf
    arr = (dbf.DbfLayerC * 2)(_layer(M=64, N=48, R=32), _layer(M=64, N=48, R=128))
    f = lib.dbf_forward_segmented_planned
    q = lib.dbf_forward_segmented_planned_workspace_bytes
    offs = np.array([0, 5, 9], dtype=np.int32)
    ok_ids = np.array([0, 1], dtype=np.int32)
    need = q(arr, 2, offs.ctypes.data, ok_ids.ctypes.data, 2, 64, 48, 9)
    assert need >= 256
    for bad_offs, bad_ids in (([0, 5, 10], [0, 1]), ([0, 6, 5], [0, 1]), ([0, 5, 9], [0, 2]), ([0, 5, 9], [-2, 0])):
        o = np.array(bad_offs, dtype=np.int32)
        i = np.array(bad_ids, dtype=np.int32)
        assert q(arr, 2, o.ctypes.data, i.ctypes.data, 2, 64, 48, 9) == 0
        assert f(arr, 2, o.ctypes.data, i.ctypes.data, 2, 64, 48, 0x1000, dbf.F32, 0x1000, dbf.F32, 9, 0,
                 0x1000, 1 << 30, None) == dbf.ERR_INVALID_ARG
    # a descriptor whose N differs from the call's
    assert f(arr, 2, offs.ctypes.data, ok_ids.ctypes.data, 2, 64, 40, 0x1000, dbf.F32, 0x1000, dbf.F32, 9, 0,
             0x1000, 1 << 30, None) == dbf.ERR_INVALID_ARG
    # rows of a segment must stay 16-byte aligned: M = 60 bf16 rows are 120 bytes
    arr2 = (dbf.DbfLayerC * 1)(_layer(M=60, N=48, R=32))
    z = np.array([0], dtype=np.int32)
    assert f(arr2, 1, np.array([0, 4], dtype=np.int32).ctypes.data, z.ctypes.data, 1, 60, 48, 0x1000, dbf.BF16,
             0x1000, dbf.F32, 4, 0, 0x1000, 1 << 30, None) == dbf.ERR_ALIGNMENT


def test_factorize_rejects_bad_arguments(lib):
    import double_binary_rank_b200 as dbf
    f = lib.dbf_factorize
    q = lib.dbf_factorize_workspace_bytes
    p = 0x1000
    n, m, k = 96, 80, 40
    need = q(n, m, k, 3, 24)
    assert need > 4 * (n * k + k * m + 4 * max(n * k, k * m) + k * k)
    assert q(n, m, k, 3, 0) == 0 and q(0, m, k, 3, 24) == 0 and q(n, m, k, -1, 24) == 0
    assert q(1 << 24, m, k, 1, 24) == 0
    args = lambda **kw: dict(dict(W=p, n=n, m=m, k=k, U0=p, V0=p, outer=3, admm=4, svid=24, rho=1.0, A=p, B=p,
                                  al=p, be=p, ga=p, obj=p, ws=p, wsb=need), **kw)
    call = lambda a: f(a["W"], a["n"], a["m"], a["k"], a["U0"], a["V0"], a["outer"], a["admm"], a["svid"], a["rho"],
                       a["A"], a["B"], a["al"], a["be"], a["ga"], a["obj"], a["ws"], a["wsb"], None)
    assert call(args(W=None)) == dbf.ERR_INVALID_ARG
    assert call(args(admm=0)) == dbf.ERR_INVALID_ARG
    assert call(args(svid=0)) == dbf.ERR_INVALID_ARG
    assert call(args(rho=0.0)) == dbf.ERR_INVALID_ARG
    assert call(args(rho=float("nan"))) == dbf.ERR_INVALID_ARG
    assert call(args(rho=float("inf"))) == dbf.ERR_INVALID_ARG
    assert call(args(outer=-1)) == dbf.ERR_INVALID_ARG
    assert call(args(n=1 << 24)) == dbf.ERR_UNSUPPORTED
    assert call(args(W=p + 2)) == dbf.ERR_ALIGNMENT
    assert call(args(obj=p + 2)) == dbf.ERR_ALIGNMENT
    assert call(args(wsb=need - 1)) == dbf.ERR_WORKSPACE
    assert call(args(ws=None)) == dbf.ERR_WORKSPACE
    assert call(args(ws=p + 16)) == dbf.ERR_ALIGNMENT


def test_gemm_min_tokens(lib):
    # AUTO's crossover per shape (host-side model fit to B200 sweeps): the
    # measured crossovers were between 8 and 16 tokens on the DBF MLP layer and
    # between 64 and 128 on a 4096 x 4096 rank-1024 layer; small adapter ranks
    # stay on the decode kernels at any T; shapes outside the GEMM path never
    # take it
    by = ctypes.byref
    assert 8 < lib.dbf_gemm_min_tokens(by(_layer(M=4096, N=11008, R=5888, ell=1))) <= 16
    assert 64 < lib.dbf_gemm_min_tokens(by(_layer(M=4096, N=4096, R=1024, ell=1))) <= 128
    assert lib.dbf_gemm_min_tokens(by(_layer(M=4096, N=4096, R=128, ell=1))) > 256
    assert lib.dbf_gemm_min_tokens(by(_layer(M=4096, N=4096, R=64, ell=1))) == -1     # R % 128 != 0
    assert lib.dbf_gemm_min_tokens(by(_layer(M=8192, N=8192, R=8192, ell=1))) < 64
    assert lib.dbf_gemm_min_tokens(None) == -1
