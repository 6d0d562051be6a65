"""Failure detection without a fault: every spin in the library's kernels is
a bounded barrier wait that ends with METIS_DEV_TIMEOUT instead of hanging.
The self-test entry point runs that same wait on a phase that nothing
completes; the GPU must report the timeout, return within the limit's order
of magnitude, and stay usable."""
import time

import numpy as np
import pytest
import torch

from oracle import fp4
from spectral_domain_quantization_b200 import api

from gpu_helpers import assert_fp4_equal

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("limit_ns", [100_000, 5_000_000])
def test_bounded_wait_reports_timeout(limit_ns):
    t0 = time.perf_counter()
    st = api.selftest_wait_timeout(limit_ns)
    elapsed = time.perf_counter() - t0
    assert st & api.DEV_TIMEOUT
    assert elapsed < 2.0   # the wait ended by itself
    # the context is still usable: an ordinary call gives the exact result
    x = np.random.default_rng(5).standard_normal((64, 128)).astype(np.float32)
    q = api.quantize_fp4(torch.from_numpy(x).cuda(), "nv", 1)
    torch.cuda.synchronize()
    assert_fp4_equal(q, fp4.quantize(x, "nv", 1), check_linear=False)
