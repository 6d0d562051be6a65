"""Mean + spectral composite split (oracle side).

Test infrastructure only (see ``oracle/__init__.py``).

Sources: the Averis paragraphs of the retelling of arXiv 2603.10444 (take the
column mean over all rows, subtract it, quantize mean and residual separately)
and the SII release on Metis, section 2.4 item 1 (split a matrix into its
dominant low-rank part and the long tail by a randomized decomposition).  The
retelling treats the mean as one more component beside the dominant and the
long-tail ones, so the composite removes the mean first and then splits the
mean-free matrix spectrally:

    A = 1 mu^T + U diag(S) V^T + R2.

Reading R28: the rank-1 mean term and the rank-k spectral term form one
rank-(k + 1) low-rank part, F diag(S') P^T with F = [1 | U] (m x (k+1)),
P = [mu | V] (n x (k+1)) and S' = [1, S].  Each factor is quantized as one FP4
tensor along its long axis (one NVFP4 tensor scale per factor).  The ones
column dequantizes to exactly 1 in MXFP4 and, in NVFP4, to
2688 fl32(1 / 2688) (its block scale is 448 and its tensor scale fl32 of
1 / 2688 while no factor entry exceeds 1), which is 1 within 2^-24.  The
mean-free matrix is the float32 residual
fl32(a_ij - mu_j) that the Averis split forms (reading R17), and R2 is the
spectral split's residual of it (readings R1-R10).
"""

import numpy as np

from . import averis, fp4
from . import split as spectral


def split(A32, k, p, power_iters, seed, kind="gaussian", nnz=4, mu32=None):
    """Composite split of A (float32 values).  mu32 (the float32 column mean)
    defaults to the float64 mean rounded to float32.

    Returns dict(mu, R1, U, S, V, R2, F, P, S1)."""
    A32 = np.asarray(A32, dtype=np.float32)
    m, n = A32.shape
    if mu32 is None:
        mu32 = averis.column_mean(A32).astype(np.float32)
    mu32 = np.asarray(mu32, dtype=np.float32)
    R1 = averis.residual_f32(A32, mu32)
    sp = spectral.split(R1.astype(np.float64), k, p, power_iters, seed, kind, nnz)
    F = np.concatenate([np.ones((m, 1)), sp["U"]], axis=1)
    P = np.concatenate([mu32.astype(np.float64)[:, None], sp["V"]], axis=1)
    S1 = np.concatenate([[1.0], sp["S"]])
    return dict(mu=mu32, R1=R1, U=sp["U"], S=sp["S"], V=sp["V"], R2=sp["R"], F=F, P=P, S1=S1)


def factors_fp4(F32, P32, fmt):
    """FP4 factors of the composite from float32 F (m x (k+1)) and P
    (n x (k+1)): blocks along m and n (outer = k + 1)."""
    return (fp4.quantize(np.asarray(F32, dtype=np.float32), fmt, 0),
            fp4.quantize(np.asarray(P32, dtype=np.float32), fmt, 0))


def reconstruct(parts):
    """1 mu^T + F diag(S') P^T + R2 in float64 (= the input up to rounding)."""
    return (parts["F"] * parts["S1"]) @ parts["P"].T + parts["R2"]
