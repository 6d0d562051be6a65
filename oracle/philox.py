"""Philox4x32-10 counter-based random number generator (oracle side).

Test infrastructure only (see ``oracle/__init__.py``).

Definition followed: J. K. Salmon, M. A. Moraes, R. O. Dror, D. E. Shaw,
"Parallel random numbers: as easy as 1, 2, 3", SC'11, section 3 (the Philox
S-box: two 32x32->64 multiplies per round, a Weyl sequence on the key, ten
rounds for the 4x32 variant).  The pages name no generator; this one is the
reading chosen for "seeded random sketch" (reading R3).

One round maps counter (c0, c1, c2, c3) and key (k0, k1) to
    (hi(M1*c2) ^ c1 ^ k0,  lo(M1*c2),  hi(M0*c0) ^ c3 ^ k1,  lo(M0*c0))
and the key is advanced by the Weyl constants (W0, W1) between rounds.

Stream layout used by the method (reading R3/R4/R5): the counter's third word
selects what the draw is for, so that the three uses never share a counter.
"""

import numpy as np

M0 = 0xD2511F53
M1 = 0xCD9E8D57
W0 = 0x9E3779B9
W1 = 0xBB67AE85
_MASK = np.uint64(0xFFFFFFFF)

STREAM_OMEGA = 1    # Gaussian sketch entries
STREAM_SPARSE = 2   # sparse-sign sketch positions and signs
STREAM_SAMPLE = 3   # row-sampling keys


def philox4x32_10(c0, c1, c2, c3, k0, k1):
    """Ten Philox rounds, vectorised over broadcastable uint32 inputs.

    Returns four uint32 arrays (the output block).  All arithmetic is done in
    uint64 so that the 32x32-bit products are exact.
    """
    c0, c1, c2, c3 = (np.asarray(v, dtype=np.uint64) & _MASK for v in (c0, c1, c2, c3))
    shape = np.broadcast_shapes(c0.shape, c1.shape, c2.shape, c3.shape)
    c0, c1, c2, c3 = (np.broadcast_to(v, shape).copy() for v in (c0, c1, c2, c3))
    k0 = np.uint64(int(k0) & 0xFFFFFFFF)
    k1 = np.uint64(int(k1) & 0xFFFFFFFF)
    m0 = np.uint64(M0)
    m1 = np.uint64(M1)
    for rnd in range(10):
        if rnd > 0:
            k0 = np.uint64((int(k0) + W0) & 0xFFFFFFFF)
            k1 = np.uint64((int(k1) + W1) & 0xFFFFFFFF)
        p0 = m0 * c0          # < 2**64: exact in uint64
        p1 = m1 * c2
        hi0, lo0 = p0 >> np.uint64(32), p0 & _MASK
        hi1, lo1 = p1 >> np.uint64(32), p1 & _MASK
        c0, c1, c2, c3 = hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0
    return tuple(v.astype(np.uint32) for v in (c0, c1, c2, c3))


def seed_key(seed):
    """Split a 64-bit seed into the Philox key words (low word first)."""
    seed = int(seed) & 0xFFFFFFFFFFFFFFFF
    return seed & 0xFFFFFFFF, seed >> 32
