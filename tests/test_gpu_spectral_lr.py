"""GPU parity of adaptive spectral learning (metis_spectral_scale, reading
R32) against the oracle's float64 G' = P_L G P_R, fed the same float32
gradient and the GPU split's own factors.

Tolerance: the library forms the rank-2k update with bf16 hi / lo
tensor-core products (each about 2^-16 relative to the update), adds it to G
in float32 and rounds once to float32, so G' carries a relative Frobenius
error of a few 2^-16 of the update plus 2^-24; 1e-4 of ||G'|| bounds both with
margin for the gains up to cap."""
import numpy as np
import pytest
import torch

from oracle import spectral_lr
from spectral_domain_quantization_b200 import api, inputs

from gpu_helpers import rel_fro, to_device

pytestmark = pytest.mark.gpu

TOL = 1e-4


@pytest.mark.parametrize("K,N,k,cap", [(512, 768, 64, 8.0), (256, 256, 8, 4.0), (1024, 384, 32, 100.0),
                                       (384, 512, 16, 1.0)])
def test_spectral_scale_matches_oracle(K, N, k, cap):
    d = inputs.make("layer_4096", scale=dict(K=K, N=N, M=128), keys=("W",))
    W = to_device(d["W"])
    s = api.split(W, k, 16, 1, 0, "nv", rows=False, cols=False, factors=False)
    rng = np.random.default_rng(K + N + k)
    G = (rng.standard_normal((K, N)) * 1e-3).astype(np.float32)
    Gt = torch.from_numpy(G).cuda()
    out = api.spectral_scale(Gt, s.U, s.S, s.V, cap)
    torch.cuda.synchronize()
    assert int(s.dev_status.item()) == 0
    U = s.U.cpu().numpy().astype(np.float64)
    S = s.S.cpu().numpy().astype(np.float64)
    V = s.V.cpu().numpy().astype(np.float64)
    want = spectral_lr.scale(G.astype(np.float64), U, S, V, cap)
    got = out.cpu().numpy()
    assert rel_fro(got, want) < TOL
    # the gradient moves where the gains are above one, and not at cap 1
    if cap == 1.0:
        assert rel_fro(got, G) < TOL
    else:
        assert rel_fro(got, G) > 10 * TOL


def test_spectral_scale_full_size_layer_weight():
    # the 4096 x 4096 layer weight's split (k = 64) and a gradient with a
    # component in its dominant subspaces
    d = inputs.make("layer_4096", keys=("W",))
    W = to_device(d["W"])
    s = api.split(W, 64, 16, 1, 0, "nv", rows=False, cols=False, factors=False)
    rng = np.random.default_rng(7)
    U = s.U.cpu().numpy().astype(np.float64)
    V = s.V.cpu().numpy().astype(np.float64)
    S = s.S.cpu().numpy().astype(np.float64)
    G = (rng.standard_normal((4096, 4096)) * 1e-3 + U @ rng.standard_normal((64, 64)) @ V.T * 1e-2).astype(np.float32)
    out = api.spectral_scale(torch.from_numpy(G).cuda(), s.U, s.S, s.V, 16.0)
    torch.cuda.synchronize()
    rows = np.sort(rng.choice(4096, 64, replace=False))
    L = np.sqrt(spectral_lr.gains(S, 16.0))
    # rows of P_L G P_R from the factors, row by row
    PL_rows = np.eye(4096)[rows] + (U[rows] * (L - 1.0)) @ U.T
    want = (PL_rows @ G.astype(np.float64)) @ (np.eye(4096) + (V * (L - 1.0)) @ V.T)
    assert rel_fro(out.cpu().numpy()[rows], want) < TOL
