"""GPU parity of the sketch Omega itself, read back from the split's
workspace (the sketch tap documented with metis_split in metis.h).

Gaussian Omega (Philox4x32-10 + Box-Muller in float64, rounded to bf16,
reading R3): equal to the oracle's except at most 1e-4 of the entries, and
those by one bf16 unit in the last place (the device's and numpy's float64
log / cos / sin may differ in their last bit, which moves a value across a
bf16 rounding boundary only when it lies within that bit of one).
Sparse sign Omega (reading R4): bit-exact.  Rows past l and columns past n
of the stored Omega^T are zero."""
import numpy as np
import pytest
import torch

from oracle import sketch
from spectral_domain_quantization_b200 import api

pytestmark = pytest.mark.gpu

WS_BYTES = 256 << 20


def _run(n, k, p, seed, kind, nnz=4, m=128, sample_rows=0):
    g = torch.Generator().manual_seed(n + k + p)
    A = torch.randn((m, n), generator=g).to(torch.bfloat16).cuda()
    ws = torch.empty(WS_BYTES, dtype=torch.uint8, device="cuda")
    res = api.split(A, k, p, 1 if kind == "gaussian" else 0, seed, "nv", sketch=kind, nnz=nnz,
                    sample_rows=sample_rows, rows=False, cols=False, factors=False, workspace=ws)
    torch.cuda.synchronize()
    assert int(res.dev_status.item()) == 0
    omt, om = api.sketch_tap(ws, n, k, p)
    omt = omt.float().cpu().numpy()
    l = k + p
    assert not omt[l:].any() and not omt[:, n:].any()
    return om.cpu().numpy().astype(np.float64)


def _bf16_ulp(x):
    a = np.abs(x)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.exp2(np.maximum(e, -126) - 7)


@pytest.mark.parametrize("n,k,p,seed", [(4096, 64, 16, 0), (256, 8, 8, 0), (14336, 64, 16, 3),
                                        (512, 20, 13, 77)])
def test_gaussian_omega_matches_oracle(n, k, p, seed):
    got = _run(n, k, p, seed, "gaussian")
    want = sketch.gaussian_omega(n, k + p, seed)
    diff = got != want
    frac = diff.mean()
    assert frac <= 1e-4, (int(diff.sum()), got.size)
    if diff.any():
        assert np.all(np.abs(got[diff] - want[diff]) <= _bf16_ulp(want[diff]) * (1 + 1e-12))


@pytest.mark.parametrize("n,k,p,nnz,seed", [(4096, 32, 16, 4, 0), (256, 8, 8, 3, 5), (14336, 64, 16, 4, 1)])
def test_sparse_sign_omega_bit_exact(n, k, p, nnz, seed):
    got = _run(n, k, p, seed, "sparse_sign", nnz=nnz)
    want = sketch.sparse_sign_omega(n, k + p, nnz, seed)
    assert np.array_equal(got, want)


def test_sampled_split_uses_the_same_sketch():
    # the sampled variant sketches the gathered rows with the same Omega
    n, k, p, seed = 4096, 32, 16, 0
    got = _run(n, k, p, seed, "sparse_sign", m=1024, sample_rows=256)
    assert np.array_equal(got, sketch.sparse_sign_omega(n, k + p, 4, seed))
