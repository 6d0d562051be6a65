"""Averis mean/residual split (oracle side).

Test infrastructure only (see ``oracle/__init__.py``).

Source: retelling of arXiv 2603.10444 (the curse and blessing of mean bias in
FP4-quantized LLM training), Averis paragraphs: take the mean over all rows of
the activation matrix (one value per column), subtract it from every row
(broadcast), and quantize the mean vector and the mean-free residual
separately; the backward pass splits the output gradient the same way.  The
method costs two mean vectors and two subtractions.  Reading R17 fixes "mean
over all rows" (tokens) and quantizes the mean vector to FP4 too.
"""

import numpy as np


def column_mean(X):
    """mu_j = (1/M) sum_i X_ij in float64."""
    X = np.asarray(X, dtype=np.float64)
    return X.sum(axis=0) / X.shape[0]


def split(X):
    """Returns (mu, R) with X = 1 mu^T + R (float64)."""
    X = np.asarray(X, dtype=np.float64)
    mu = column_mean(X)
    return mu, X - mu[None, :]


def residual_f32(X32, mu32):
    """The float32 residual the quantizer sees: fl32(x_ij - mu_j)."""
    X32 = np.asarray(X32, dtype=np.float32)
    mu32 = np.asarray(mu32, dtype=np.float32)
    return (X32 - mu32[None, :]).astype(np.float32)


def residual_amax_from_columns(X32, mu32):
    """max |fl32(x_ij - mu_j)| computed from the column minimum and maximum
    alone: rounding is monotonic, so the extreme residual of column j is
    fl32(max_i x_ij - mu_j) or -fl32(min_i x_ij - mu_j)."""
    X32 = np.asarray(X32, dtype=np.float32)
    mu32 = np.asarray(mu32, dtype=np.float32)
    hi = (X32.max(axis=0) - mu32).astype(np.float32)
    lo = (X32.min(axis=0) - mu32).astype(np.float32)
    return np.float32(max(np.max(hi), np.max(-lo)))
