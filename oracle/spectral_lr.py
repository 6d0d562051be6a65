"""Adaptive spectral learning: the gradient of a split weight rescaled along
the weight's singular directions (oracle side).

Test infrastructure only (see ``oracle/__init__.py``).

Sources: SII release on Metis, section 2.4 item 2 (learning along the large
singular values is strong by nature while the small ones are easily
neglected; in the spectral space the gradients along the mid and low
singular-value directions are scaled by an inverse normalisation, which
strengthens their updates so that long-tail features are not drowned out,
while avoiding amplified noise); "Metis: Training Large Language Models with
Advanced Low-Bit Quantization", abstract item (ii) (adaptive learning rates in
the spectral domain amplify under-represented directions).

Reading R32.  The pages give no formula.  Plain reading: the weight W (K x N)
has the split W = U diag(S) V^T + R with U (K x k), V (N x k) orthonormal and
S descending.  Normalising the singular values by the largest one gives
s_i = S_i / S_1 in (0, 1]; its inverse is the gain of direction i, capped so
that noise is not amplified without bound:

    lambda_i = min(S_1 / S_i, cap)          (lambda_i = 1 where S_i <= 0),

so the top direction keeps gain 1 and the mid and low ones are amplified.
The gain is a learning rate per singular direction: the gradient G (K x N) is
preconditioned on both sides,

    G' = P_L G P_R,   P_L = I + U (L - I) U^T,   P_R = I + V (L - I) V^T,

with L = diag(sqrt(lambda)).  Then u_i^T G' v_j = sqrt(lambda_i lambda_j)
u_i^T G v_j (the component along u_i v_i^T is scaled by lambda_i), the
components with one side in a split direction are scaled by that side's
sqrt(lambda), and the part outside both subspaces (the long tail) is left as
it is.  Expanded with a = L - I, C = U^T G V:

    G' = G + U a (U^T G) + (G V) a V^T + U a C a V^T,

a rank-2k update of G, which is how the library forms it.
"""

import numpy as np


def gains(S, cap):
    """lambda_i = min(S_1 / S_i, cap) for the descending singular values S;
    1 where S_i <= 0 (a dropped direction)."""
    S = np.asarray(S, dtype=np.float64)
    if cap < 1:
        raise ValueError("cap must be >= 1")
    lam = np.ones_like(S)
    if S.size and S[0] > 0:
        pos = S > 0
        lam[pos] = np.minimum(S[0] / S[pos], cap)
    return lam


def scale(G, U, S, V, cap):
    """G' = P_L G P_R of reading R32 (float64), from the preconditioners."""
    G = np.asarray(G, dtype=np.float64)
    U = np.asarray(U, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    L = np.sqrt(gains(S, cap))
    K, N = G.shape
    PL = np.eye(K) + (U * (L - 1.0)) @ U.T
    PR = np.eye(N) + (V * (L - 1.0)) @ V.T
    return PL @ G @ PR
