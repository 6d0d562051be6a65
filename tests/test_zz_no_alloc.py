"""The quantizer variant without a workspace (metis_quantize_fp4_noalloc).

Some callers cannot hand the library scratch memory (they may not allocate
where they quantize, or hold no spare device buffer), so this entry point keeps
its scratch in a fixed array inside the library.  This file checks, through the
C ABI, that it gives exactly what metis_quantize_fp4 gives, on two calls in a
row (the second call must not see leftovers of the first), that its bytes are
the oracle quantizer's on the same float32 values, and that a request larger
than the fixed array is refused.  The file is named so that pytest collects it
last."""
import ctypes

import numpy as np
import pytest
import torch

from oracle import fp4
from spectral_domain_quantization_b200 import api

from gpu_helpers import assert_fp4_equal

pytestmark = pytest.mark.gpu


def _same(a, b):
    assert torch.equal(a.codes, b.codes)
    assert torch.equal(a.scales, b.scales)
    assert torch.equal(a.tensor_scale, b.tensor_scale)
    if a.inner_sum is not None:
        # identical kernels, identical reduction order
        assert torch.allclose(a.inner_sum, b.inner_sum, rtol=1e-6, atol=0)


def test_noalloc_matches_workspace_entry_point_twice():
    rng = np.random.default_rng(123)
    cases = [("nv", 0, (1056, 304)), ("mx", 1, (300, 1024))]
    for fmt, axis, shape in cases:           # two calls in a row, different shapes
        x = (rng.standard_normal(shape) * np.exp2(rng.integers(-4, 4, (shape[0], 1)))).astype(np.float32)
        X = torch.from_numpy(x).cuda().to(torch.bfloat16)
        ref = api.quantize_fp4(X, fmt, axis, inner_sum=True)
        got = api.quantize_fp4_noalloc(X, fmt, axis, inner_sum=True)
        torch.cuda.synchronize()
        _same(got, ref)
        # and directly against the oracle on the bf16 values both sides saw
        assert_fp4_equal(got, fp4.quantize(X.float().cpu().numpy(), fmt, axis), check_linear=False)
    # a second call on the same inputs as the first (scratch reused)
    x = (rng.standard_normal((1056, 304)) * 3).astype(np.float32)
    X = torch.from_numpy(x).cuda()
    ref = api.quantize_fp4(X, "nv", 0, inner_sum=True)
    got1 = api.quantize_fp4_noalloc(X, "nv", 0, inner_sum=True)
    got2 = api.quantize_fp4_noalloc(X, "nv", 0, inner_sum=True)
    torch.cuda.synchronize()
    _same(got1, ref)
    _same(got2, ref)


def test_noalloc_refuses_oversized_scratch():
    L = api.lib()
    cap = L.metis_noalloc_scratch_bytes()
    assert cap == 2 << 20
    # fits: 128 outer x 64 groups of inner-sum partials = 32 KiB
    X = torch.zeros((4096, 128), dtype=torch.bfloat16, device="cuda")
    q = api.QTensor("nv", 128, 4096, "cuda", inner_sum=True)          # blocks along rows
    s = q.struct()
    assert L.metis_quantize_fp4_noalloc(ctypes.c_void_p(X.data_ptr()), api.BF16, 4096, 128, 128, 0, None,
                                        ctypes.byref(s), None) == api.OK
    # too big: 32 outer x 20000 groups x 4 bytes = 2.56 MB of partials > 2 MiB
    rows = 64 * 20000
    Xh = torch.zeros((rows, 32), dtype=torch.bfloat16, device="cuda")
    qh = api.QTensor("nv", 32, rows, "cuda", inner_sum=True)
    sh = qh.struct()
    st = L.metis_quantize_fp4_noalloc(ctypes.c_void_p(Xh.data_ptr()), api.BF16, rows, 32, 32, 0, None,
                                      ctypes.byref(sh), None)
    assert st == 5                                                     # METIS_ERR_WORKSPACE
    assert b"2 MiB" in L.metis_last_error()
    torch.cuda.synchronize()
