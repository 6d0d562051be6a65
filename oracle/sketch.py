"""Random sketch matrices and row sampling (oracle side).

Test infrastructure only (see ``oracle/__init__.py``).

Sources: "Metis: Training LLMs with FP4 Quantization" (arXiv 2509.00404v4
summary), abstract and "technical framework": the dominant spectral subspace is
preserved under sparse random sampling and under random projection.  SII
release, section 2.4 item 1: randomized dimension reduction makes the spectral
decomposition cheap.  The pages fix neither distribution nor scale; the
readings used here are R3 (Gaussian entries from Philox + Box-Muller, rounded to
bf16, unscaled), R4 (sparse sign embedding: every input coordinate feeds
``nnz`` distinct sketch columns with random signs) and R5 (uniform sampling
without replacement: the rows with the smallest Philox keys).
"""

import numpy as np

from .philox import philox4x32_10, seed_key, STREAM_OMEGA, STREAM_SPARSE, STREAM_SAMPLE

TWO_PI = 2.0 * np.pi


def round_to_bf16(x):
    """Round float64 values to the nearest bfloat16 value, ties to even.

    bfloat16 keeps 8 significant bits; the result is returned as float64
    (every bfloat16 value is exact in float64).  Works directly from float64
    (no intermediate float32 rounding).  Subnormal bfloat16 values use the
    fixed quantum 2**-133.
    """
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    _, e2 = np.frexp(a)                    # a = m * 2**e2, m in [0.5, 1)
    e = e2.astype(np.int64) - 1            # floor(log2 a) for a > 0
    e = np.maximum(e, -126)                # subnormal range shares one quantum
    quantum = np.ldexp(1.0, e - 7)
    r = np.round(a / quantum) * quantum    # np.round: half to even; a/quantum exact
    r = np.where(a == 0, 0.0, r)
    return np.copysign(r, x)


def gaussian_omega(n, l, seed):
    """Gaussian sketch Omega (n x l), entries N(0, 1) rounded to bfloat16.

    Entry (i, j) uses the Philox block at counter (j // 2, i, STREAM_OMEGA, 0)
    under key = seed.  Its first two words give u1 = (x0 + 1) * 2**-32 in
    (0, 1] and u2 = x1 * 2**-32 in [0, 1); Box-Muller gives
    r = sqrt(-2 ln u1), theta = 2 pi u2, and the entry is r cos(theta) for even
    j and r sin(theta) for odd j, computed in float64 and rounded to bfloat16.
    """
    k0, k1 = seed_key(seed)
    i = np.arange(n, dtype=np.uint64)[:, None]
    j = np.arange(l, dtype=np.uint64)[None, :]
    x0, x1, _, _ = philox4x32_10(j >> np.uint64(1), i, STREAM_OMEGA, 0, k0, k1)
    u1 = (x0.astype(np.float64) + 1.0) * 2.0 ** -32
    u2 = x1.astype(np.float64) * 2.0 ** -32
    r = np.sqrt(-2.0 * np.log(u1))
    theta = TWO_PI * u2
    z = np.where((j % np.uint64(2)) == 0, r * np.cos(theta), r * np.sin(theta))
    return round_to_bf16(z)


def sparse_sign_omega(n, l, nnz, seed):
    """Sparse sign embedding Omega (n x l) with ``nnz`` entries of +-1 per row.

    Row i (one input coordinate) draws Philox blocks at counters
    (t, i, STREAM_SPARSE, 0) for t = 0, 1, 2, ...; each block offers two
    candidates, (x0, x1) then (x2, x3).  A candidate (a, b) proposes column
    c = floor(a * l / 2**32) with sign -1 if the top bit of b is set, else +1;
    a column already taken by this row is skipped (redraw on collision).  The
    row is complete once ``nnz`` distinct columns are taken.
    """
    if not (0 < nnz <= l):
        raise ValueError("need 0 < nnz <= l")
    k0, k1 = seed_key(seed)
    om = np.zeros((n, l), dtype=np.float64)
    tmax = 64
    rows = np.arange(n, dtype=np.uint64)
    words = [philox4x32_10(t, rows, STREAM_SPARSE, 0, k0, k1) for t in range(tmax)]
    for i in range(n):
        taken = []
        t = 0
        while len(taken) < nnz:
            if t >= tmax:
                raise RuntimeError("sparse sign draw did not finish")
            w = [int(words[t][q][i]) for q in range(4)]
            for a, b in ((w[0], w[1]), (w[2], w[3])):
                if len(taken) == nnz:
                    break
                c = (a * l) >> 32
                if c in taken:
                    continue
                taken.append(c)
                om[i, c] = -1.0 if (b >> 31) else 1.0
            t += 1
    return om


def row_keys(m, seed):
    """64-bit sampling key of each row r: Philox block at (r, 0, STREAM_SAMPLE, 0),
    key = (x1 << 32) | x0."""
    k0, k1 = seed_key(seed)
    r = np.arange(m, dtype=np.uint64)
    x0, x1, _, _ = philox4x32_10(r, 0, STREAM_SAMPLE, 0, k0, k1)
    return (x1.astype(np.uint64) << np.uint64(32)) | x0.astype(np.uint64)


def sample_rows(m, s, seed):
    """Indices of ``s`` distinct rows out of ``m``: the rows with the ``s``
    smallest keys (ties broken by the lower row index), returned in ascending
    row order."""
    if not (0 < s <= m):
        raise ValueError("need 0 < s <= m")
    key = row_keys(m, seed)
    order = np.lexsort((np.arange(m), key))   # primary: key, secondary: row
    return np.sort(order[:s]).astype(np.int64)
