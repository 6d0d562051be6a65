"""Host-side checks of the C ABI (no GPU compute): the library loads, exports
exactly the functions declared in include/metis.h, and the host-only helpers
and the argument checks behave as documented."""
import ctypes
import subprocess

import numpy as np
import pytest

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


def test_split_params_layout_matches_the_header():
    # the library asserts sizeof(metis_split_params) == 56 at compile time;
    # the ctypes mirror must have the same size and field offsets
    import ctypes
    P = api.SplitParams
    assert ctypes.sizeof(P) == 56
    assert [P.k.offset, P.p.offset, P.power_iters.offset, P.seed.offset, P.sketch.offset, P.sparse_nnz.offset,
            P.sample_rows.offset, P.fmt.offset, P.max_core_iters.offset, P.compensate.offset] == \
        [0, 4, 8, 16, 24, 28, 32, 40, 44, 48]
