"""Host-side checks of the C ABI (no GPU compute): the library loads, exports
exactly the functions declared in include/metis.h, and the host-only helpers
and the argument checks behave as documented."""
import ctypes
import subprocess

import numpy as np
import pytest
import torch

from oracle import fp4
from spectral_domain_quantization_b200 import api


def test_library_exports_exactly_the_declared_symbols():
    L = api.lib()
    names = api.header_functions()
    assert {"metis_split", "metis_quantize_fp4", "metis_linear_fwd", "metis_linear_bwd",
            "averis_split"} <= set(names)
    for n in names:
        assert hasattr(L, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", api.LIB_PATH], capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    # the internal C++ launchers and kernels stay hidden
    assert exported == set(names)


@pytest.mark.parametrize("fmt", ["mx", "nv"])
@pytest.mark.parametrize("outer,inner", [(1, 32), (300, 1024 + 256), (128, 256), (129, 96)])
def test_buffer_sizes_match_layout(fmt, outer, inner):
    L = api.lib()
    bs = 32 if fmt == "mx" else 16
    rows, cols = fp4.tc_scale_shape(outer, inner, bs)
    assert L.metis_fp4_scales_bytes(api.FMT[fmt], outer, inner) == rows * cols
    assert L.metis_fp4_codes_bytes(outer, inner) == outer * inner // 2


def test_status_strings():
    L = api.lib()
    assert L.metis_status_string(0) == b"ok"
    assert L.metis_status_string(2) == b"invalid shape"
    assert L.metis_status_string(99) == b"unknown status"


def _fake_fp4(fmt, outer, inner):
    s = api.FP4Struct()
    s.fmt, s.outer, s.inner = fmt, outer, inner
    s.codes, s.scales, s.tensor_scale = 0x10000, 0x20000, 0x30000
    return s


def _quant(X, dtype, rows, cols, ld, axis, out, ws=None, wsb=None):
    L = api.lib()
    size = ctypes.c_size_t(0 if wsb is None else wsb)
    st = L.metis_quantize_fp4(X, dtype, rows, cols, ld, axis, None,
                              ctypes.byref(out) if out is not None else None, ws, ctypes.byref(size), None)
    return st, size.value


def test_quantize_argument_checks_and_workspace_query():
    X = ctypes.c_void_p(0x40000)
    ok = _fake_fp4(api.NVFP4, 64, 128)
    st, need = _quant(X, api.BF16, 64, 128, 128, 1, ok)
    assert st == api.OK and need >= 256
    assert _quant(X, api.BF16, 64, 128, 128, 1, None)[0] == 1           # NULL out
    assert _quant(None, api.BF16, 64, 128, 128, 1, ok)[0] == 1            # NULL X
    assert _quant(X, 7, 64, 128, 128, 1, ok)[0] == 7                      # bad dtype
    assert _quant(X, api.BF16, 64, 128, 128, 2, ok)[0] == 7               # bad axis
    assert _quant(X, api.BF16, 64, 128, 100, 1, ok)[0] == 2               # ld < cols
    assert _quant(X, api.BF16, 64, 128, 132, 1, ok)[0] == 3               # ld*2 not 16B
    assert _quant(ctypes.c_void_p(0x40002), api.BF16, 64, 128, 128, 1, ok)[0] == 3
    bad = _fake_fp4(api.NVFP4, 64, 96 + 16)                                # inner % 32
    assert _quant(X, api.BF16, 64, 112, 112 + 8, 1, bad)[0] == 2
    wrong = _fake_fp4(api.NVFP4, 128, 64)                                  # shape mismatch
    assert _quant(X, api.BF16, 64, 128, 128, 1, wrong)[0] == 2
    # axis 0: outer = cols, inner = rows
    t0 = _fake_fp4(api.MXFP4, 128, 64)
    assert _quant(X, api.F32, 64, 128, 128, 0, t0)[0] == api.OK
    # too-small workspace with a real (fake) pointer
    st, _ = _quant(X, api.BF16, 64, 128, 128, 1, ok, ws=ctypes.c_void_p(0x50000), wsb=8)
    assert st == 5


def test_unbuilt_entry_points_report_instead_of_crashing():
    # argument errors are returned before any device work even without a GPU
    L = api.lib()
    size = ctypes.c_size_t(0)
    st = L.metis_linear_fwd(None, None, 1, 1, 32, None, api.F32, 1, None, ctypes.byref(size), None, None)
    assert st != api.OK


ERR_NULL, ERR_ARG = 1, 7  # metis_status codes of include/metis.h


def test_selftest_wait_argument_checks():
    L = api.lib()
    assert L.metis_selftest_wait_timeout(1000, None, None) == ERR_NULL
    fake = ctypes.c_int32(0)
    assert L.metis_selftest_wait_timeout(0, ctypes.addressof(fake), None) == ERR_ARG
    assert L.metis_selftest_wait_timeout(2_000_000_000, ctypes.addressof(fake), None) == ERR_ARG


def test_fp4_tensor_and_operand_layouts_match_the_header():
    # the library asserts the same sizes and offsets at compile time
    T, O = api.FP4Struct, api.OperandStruct
    assert ctypes.sizeof(T) == 64
    assert [T.fmt.offset, T.outer.offset, T.inner.offset, T.codes.offset, T.scales.offset,
            T.scales_linear.offset, T.tensor_scale.offset, T.inner_sum.offset] == [0, 8, 16, 24, 32, 40, 48, 56]
    assert ctypes.sizeof(O) == 48
    assert [O.R.offset, O.k.offset, O.P.offset, O.F.offset, O.S.offset, O.flags.offset] == [0, 8, 16, 24, 32, 40]
    # the flag bit the header defines
    hdr = open(api.HEADER).read()
    assert "#define METIS_REQUANT_LOWRANK 1" in hdr and api.REQUANT_LOWRANK == 1


def test_split_params_layout_matches_the_header():
    # the library asserts sizeof(metis_split_params) == 56 at compile time;
    # the ctypes mirror must have the same size and field offsets
    import ctypes
    P = api.SplitParams
    assert ctypes.sizeof(P) == 56
    assert [P.k.offset, P.p.offset, P.power_iters.offset, P.seed.offset, P.sketch.offset, P.sparse_nnz.offset,
            P.sample_rows.offset, P.fmt.offset, P.max_core_iters.offset, P.compensate.offset] == \
        [0, 4, 8, 16, 24, 28, 32, 40, 44, 48]


# ---------------------------------------------------------------------------
# argument checks of the split, product and Averis entry points: every case
# returns before any device work (workspace query or a rejected argument), so
# the pointers below are never dereferenced.  The one call that passes every
# check with a workspace runs only without a GPU (where it must report
# METIS_ERR_UNSUPPORTED); on a GPU it would launch on these fake pointers.
# ---------------------------------------------------------------------------

ERR_SHAPE, ERR_ALIGN, ERR_UNSUPPORTED, ERR_WORKSPACE = 2, 3, 4, 5
_A, _U, _S, _V, _ST, _WS = 0x40000, 0x50000, 0x58000, 0x60000, 0x68000, 0x70000


def _params(k=8, p=8, q=1, sketch=0, nnz=4, sample_rows=0, fmt=api.NVFP4, iters=64, compensate=0):
    prm = api.SplitParams()
    prm.k, prm.p, prm.power_iters, prm.seed = k, p, q, 0
    prm.sketch, prm.sparse_nnz, prm.sample_rows = sketch, nnz, sample_rows
    prm.fmt, prm.max_core_iters, prm.compensate = fmt, iters, compensate
    return prm


def _split(m=256, n=128, lda=None, prm=None, A=_A, U_q=None, V_q=None, R_rows=None, R_cols=None, ws=None,
           wsb=None, dtype=None):
    L = api.lib()
    size = ctypes.c_size_t(0 if wsb is None else wsb)
    prm = _params() if prm is None else prm
    ref = lambda t: ctypes.byref(t) if t is not None else None
    st = L.metis_split(A, api.BF16 if dtype is None else dtype, m, n, n if lda is None else lda,
                       ctypes.byref(prm) if prm is not False else None, _U, _S, _V,
                       ref(U_q), ref(V_q), ref(R_rows), ref(R_cols), None, None, ws, ctypes.byref(size),
                       _ST, None)
    return st, size.value


def test_split_argument_checks_and_workspace_query():
    st, need = _split()
    assert st == api.OK and need > 0
    assert _split(R_rows=_fake_fp4(api.NVFP4, 256, 128), R_cols=_fake_fp4(api.NVFP4, 128, 256))[0] == api.OK
    assert _split(prm=False)[0] == ERR_NULL
    assert _split(A=None)[0] == ERR_NULL
    assert _split(m=0)[0] == ERR_SHAPE
    assert _split(lda=100)[0] == ERR_SHAPE                        # lda < n
    assert _split(A=0x40002)[0] == ERR_ALIGN
    assert _split(lda=132)[0] == ERR_ALIGN                        # rows not on 16-byte boundaries
    assert _split(dtype=9)[0] == ERR_ARG
    assert _split(prm=_params(fmt=5))[0] == ERR_ARG
    assert _split(prm=_params(sketch=3))[0] == ERR_ARG
    assert _split(prm=_params(k=0))[0] == ERR_ARG
    assert _split(prm=_params(q=-1))[0] == ERR_ARG
    assert _split(prm=_params(iters=0))[0] == ERR_ARG
    assert _split(prm=_params(sketch=1, nnz=0))[0] == ERR_ARG
    assert _split(prm=_params(sketch=1, nnz=17))[0] == ERR_ARG
    assert _split(prm=_params(compensate=2))[0] == ERR_ARG
    assert _split(prm=_params(compensate=1))[0] == ERR_NULL       # compensation needs U_q and V_q
    assert _split(prm=_params(k=64, p=64))[0] == ERR_SHAPE       # l = k + p above the core's limit
    assert _split(prm=_params(k=6))[0] == ERR_SHAPE              # k not a multiple of 4
    assert _split(n=64, prm=_params(k=40, p=40))[0] == ERR_SHAPE  # l > n
    assert _split(prm=_params(sample_rows=512))[0] == ERR_SHAPE   # more sampled rows than rows
    assert _split(prm=_params(k=40, p=40, sample_rows=64))[0] == ERR_SHAPE  # l > sampled rows
    assert _split(m=96 + 8, n=128)[0] == ERR_SHAPE               # m not a multiple of 32
    assert _split(R_rows=_fake_fp4(api.NVFP4, 128, 256))[0] == ERR_SHAPE   # rows tensor must be m x n
    assert _split(R_rows=_fake_fp4(api.MXFP4, 256, 128))[0] == ERR_ARG     # format differs from the params
    assert _split(U_q=_fake_fp4(api.NVFP4, 8, 256))[0] == api.OK          # U_q: outer k, inner m
    assert _split(U_q=_fake_fp4(api.NVFP4, 256, 8))[0] == ERR_SHAPE
    assert _split(ws=ctypes.c_void_p(_WS), wsb=need - 1)[0] == ERR_WORKSPACE
    assert _split(ws=ctypes.c_void_p(_WS + 8), wsb=need)[0] == ERR_WORKSPACE  # not 256-byte aligned
    if not torch.cuda.is_available():
        assert _split(ws=ctypes.c_void_p(_WS), wsb=need)[0] == ERR_UNSUPPORTED


def _operand(fmt, outer, inner, k=0, P=None, F=None, inner_sum=False):
    R = _fake_fp4(fmt, outer, inner)
    if inner_sum:
        R.inner_sum = 0x78000
    op = api.OperandStruct()
    op.R = ctypes.pointer(R)
    op.k = k
    op.P = ctypes.pointer(P) if P is not None else None
    op.F = ctypes.pointer(F) if F is not None else None
    op.S = 0x7C000 if k else None
    op._keep = (R, P, F)
    return op


def _fwd(X, W, M, N, K, Y=0x80000, ydt=None, ldy=None, ws=None, wsb=None):
    L = api.lib()
    size = ctypes.c_size_t(0 if wsb is None else wsb)
    st = L.metis_linear_fwd(ctypes.byref(X) if X is not None else None, ctypes.byref(W) if W is not None else None,
                            M, N, K, Y, api.F32 if ydt is None else ydt, N if ldy is None else ldy, ws,
                            ctypes.byref(size), _ST, None)
    return st, size.value


def test_linear_argument_checks_and_workspace_query():
    nv, mx = api.NVFP4, api.MXFP4
    M, N, K = 256, 128, 512
    X, W = _operand(nv, M, K), _operand(nv, N, K)
    assert _fwd(X, W, M, N, K)[0] == api.OK
    assert _fwd(None, W, M, N, K)[0] == ERR_NULL
    assert _fwd(X, W, M, N, K, Y=None)[0] == ERR_NULL
    assert _fwd(X, W, 0, N, K)[0] == ERR_SHAPE
    assert _fwd(X, W, M, N, K + 16)[0] == ERR_SHAPE                 # K not a multiple of 32
    big = 1 << 31                                                   # rows past 32-bit indexing
    assert _fwd(_operand(nv, big, K), W, big, N, K)[0] == ERR_SHAPE
    assert _fwd(X, W, M + 1, N, K)[0] == ERR_SHAPE                  # X is not M x K
    assert _fwd(X, _operand(mx, N, K), M, N, K)[0] == ERR_ARG       # formats differ
    assert _fwd(X, W, M, N, K, ydt=9)[0] == ERR_ARG
    assert _fwd(X, W, M, N, K, ldy=N - 1)[0] == ERR_SHAPE
    # split right operand: P (k x K) and F (k x N) quantized along K and N
    P, F = _fake_fp4(nv, 8, K), _fake_fp4(nv, 8, N)
    st, need = _fwd(X, _operand(nv, N, K, 8, P, F), M, N, K)
    assert st == api.OK and need > 0
    assert _fwd(X, _operand(nv, N, K, 8, _fake_fp4(nv, 8, N), F), M, N, K)[0] == ERR_SHAPE   # P must be k x K
    assert _fwd(X, _operand(nv, N, K, 200, P, F), M, N, K)[0] == ERR_ARG                     # k above 128
    assert _fwd(X, _operand(nv, N, K, 2), M, N, K)[0] == ERR_ARG        # only k = 1 may omit P and F (ones)
    bad = _operand(nv, N, K, 8, P, F)
    bad.flags = 2                                                       # an undefined flag bit
    assert _fwd(X, bad, M, N, K)[0] == ERR_ARG
    # an all-ones P (the Averis rank-1 form) needs the other operand's inner sums
    ones = _operand(nv, N, K, 1, None, _fake_fp4(nv, 1, N))
    assert _fwd(X, ones, M, N, K)[0] == ERR_NULL
    assert _fwd(_operand(nv, M, K, inner_sum=True), ones, M, N, K)[0] == api.OK
    st, need = _fwd(X, _operand(nv, N, K, 8, P, F), M, N, K)
    assert _fwd(X, _operand(nv, N, K, 8, P, F), M, N, K, ws=ctypes.c_void_p(_WS), wsb=need - 1)[0] == ERR_WORKSPACE
    # backward: at least one output
    L = api.lib()
    size = ctypes.c_size_t(0)
    assert L.metis_linear_bwd(ctypes.byref(X), ctypes.byref(W), ctypes.byref(X), ctypes.byref(W), M, N, K,
                              None, K, None, N, api.F32, None, ctypes.byref(size), _ST, None) == ERR_NULL


def _averis(m=256, n=128, ld=None, fmt=api.NVFP4, mean=0x90000, mean_q=None, R_rows=None, R_cols=None, X=_A,
            ws=None, wsb=None):
    L = api.lib()
    size = ctypes.c_size_t(0 if wsb is None else wsb)
    ref = lambda t: ctypes.byref(t) if t is not None else None
    st = L.averis_split(X, api.BF16, m, n, n if ld is None else ld, fmt, mean, ref(mean_q), ref(R_rows),
                        ref(R_cols), None, ws, ctypes.byref(size), _ST, None)
    return st, size.value


def test_averis_argument_checks_and_workspace_query():
    st, need = _averis(mean_q=_fake_fp4(api.NVFP4, 1, 128), R_rows=_fake_fp4(api.NVFP4, 256, 128),
                       R_cols=_fake_fp4(api.NVFP4, 128, 256))
    assert st == api.OK and need > 0
    assert _averis(mean=None)[0] == ERR_NULL
    assert _averis(X=None)[0] == ERR_NULL
    assert _averis(mean=0x90004)[0] == ERR_ALIGN
    assert _averis(fmt=5)[0] == ERR_ARG
    assert _averis(m=0)[0] == ERR_SHAPE
    assert _averis(mean_q=_fake_fp4(api.NVFP4, 2, 128))[0] == ERR_SHAPE      # the mean is one row
    assert _averis(R_rows=_fake_fp4(api.MXFP4, 256, 128))[0] == ERR_ARG
    assert _averis(R_cols=_fake_fp4(api.NVFP4, 256, 128))[0] == ERR_SHAPE    # blocks along m: outer n
    st, need1 = _averis(mean_q=_fake_fp4(api.NVFP4, 1, 128))
    assert st == api.OK and 0 < need1 < need
    assert _averis(ws=ctypes.c_void_p(_WS), wsb=need1 - 1,
                   mean_q=_fake_fp4(api.NVFP4, 1, 128))[0] == ERR_WORKSPACE


def _scale(G=_A, K=256, N=128, ldg=128, U=_U, S=_S, V=_V, k=8, cap=4.0, out=0x90000, ws=None, wsb=0):
    size = ctypes.c_size_t(wsb)
    st = api.lib().metis_spectral_scale(G, K, N, ldg, U, S, V, k, ctypes.c_float(cap), out, ws, ctypes.byref(size),
                                        _ST, None)
    return st, size.value


def test_spectral_scale_argument_checks_and_workspace_query():
    st, need = _scale()
    assert st == api.OK and need > 0
    for kw in (dict(G=None), dict(U=None), dict(S=None), dict(V=None), dict(out=None)):
        assert _scale(**kw)[0] == ERR_NULL
    assert _scale(k=0)[0] == ERR_ARG and _scale(k=65)[0] == ERR_ARG           # 1 <= k <= 64
    assert _scale(cap=0.5)[0] == ERR_ARG and _scale(cap=float("nan"))[0] == ERR_ARG
    assert _scale(K=100)[0] == ERR_SHAPE and _scale(N=96 + 8, ldg=104)[0] == ERR_SHAPE
    assert _scale(ldg=130)[0] == ERR_ALIGN and _scale(out=0x90004)[0] == ERR_ALIGN
    assert _scale(ws=ctypes.c_void_p(_WS), wsb=need - 1)[0] == ERR_WORKSPACE
