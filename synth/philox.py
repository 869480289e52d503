"""Philox4x32-10 counter-based generator, vectorised in numpy.

Written from the published definition (Salmon, Moraes, Dror, Shaw, "Parallel
random numbers: as easy as 1, 2, 3", SC'11): a 4x32-bit counter and a 2x32-bit
key go through ten rounds of two 32x32->64 multiplies with the round
constants 0xD2511F53 / 0xCD9E8D57, the key being bumped by the Weyl constants
0x9E3779B9 / 0xBB67AE85 between rounds.

This module holds no arithmetic of the FP4 method: it only turns
(key, counter) into 32-bit words. The device-side twin lives in
``synth/csrc/synth_gen.cu``; both must produce identical words, which
``tests/test_synth.py`` checks against known-answer vectors.
"""
from __future__ import annotations

import numpy as np

M0 = np.uint64(0xD2511F53)
M1 = np.uint64(0xCD9E8D57)
W0 = np.uint32(0x9E3779B9)
W1 = np.uint32(0xBB67AE85)
_MASK32 = np.uint64(0xFFFFFFFF)
_SH32 = np.uint64(32)


def philox4x32_10(c0, c1, c2, c3, k0, k1):
    """Return the four 32-bit output words for counters (c0..c3) and key (k0, k1).

    Every argument is broadcast; counters are uint32 arrays, keys uint32 scalars
    or arrays. Returns a tuple of four uint32 arrays.
    """
    c0 = np.asarray(c0, dtype=np.uint32)
    c1 = np.asarray(c1, dtype=np.uint32)
    c2 = np.asarray(c2, dtype=np.uint32)
    c3 = np.asarray(c3, dtype=np.uint32)
    k0 = np.asarray(k0, dtype=np.uint32)
    k1 = np.asarray(k1, dtype=np.uint32)
    c0, c1, c2, c3 = np.broadcast_arrays(c0, c1, c2, c3)
    c0 = c0.copy(); c1 = c1.copy(); c2 = c2.copy(); c3 = c3.copy()
    for rnd in range(10):
        if rnd:
            k0 = ((k0.astype(np.uint64) + np.uint64(W0)) & _MASK32).astype(np.uint32)
            k1 = ((k1.astype(np.uint64) + np.uint64(W1)) & _MASK32).astype(np.uint32)
        p0 = M0 * c0.astype(np.uint64)
        p1 = M1 * c2.astype(np.uint64)
        hi0 = (p0 >> _SH32).astype(np.uint32)
        lo0 = (p0 & _MASK32).astype(np.uint32)
        hi1 = (p1 >> _SH32).astype(np.uint32)
        lo1 = (p1 & _MASK32).astype(np.uint32)
        c0, c1, c2, c3 = hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0
    return c0, c1, c2, c3
