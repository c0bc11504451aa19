"""Philox4x32-10 counter-based generator, vectorised over numpy arrays.

Follows the published definition of Philox4x32 with 10 rounds (Salmon, Moraes,
Dror and Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3", SC 2011): a
128-bit counter and a 64-bit key; each round multiplies counter words 0 and 2
by two fixed 32-bit multipliers, recombines the high and low halves with the
key, and bumps the key by two Weyl constants between rounds.

The device-side twin lives in ``synth/csrc/synth_gen.cu``. Both compute the
same integer function, so host and device produce identical words for the same
(counter, key).
"""
import numpy as np

PHILOX_M0 = 0xD2511F53
PHILOX_M1 = 0xCD9E8D57
PHILOX_W0 = 0x9E3779B9
PHILOX_W1 = 0xBB67AE85
MASK32 = 0xFFFFFFFF


def philox4x32_10(c0, c1, c2, c3, k0, k1):
    """Return the four 32-bit output words for counters (c0..c3) and key (k0, k1).

    Arguments broadcast against each other; all are treated as uint32.
    Returns four uint32 arrays.
    """
    u64 = np.uint64
    m32 = u64(MASK32)
    c0, c1, c2, c3 = np.broadcast_arrays(*(np.asarray(x, dtype=np.uint64) & m32
                                           for x in (c0, c1, c2, c3)))
    c0, c1, c2, c3 = c0.copy(), c1.copy(), c2.copy(), c3.copy()
    k0 = np.asarray(k0, dtype=np.uint64) & m32
    k1 = np.asarray(k1, dtype=np.uint64) & m32
    M0, M1 = u64(PHILOX_M0), u64(PHILOX_M1)
    W0, W1 = u64(PHILOX_W0), u64(PHILOX_W1)
    s32 = u64(32)
    for r in range(10):
        p0 = c0 * M0            # exact: 32x32 -> 64 bit fits uint64
        p1 = c2 * M1
        n0 = (p1 >> s32) ^ c1 ^ k0
        n1 = p1 & m32
        n2 = (p0 >> s32) ^ c3 ^ k1
        n3 = p0 & m32
        c0, c1, c2, c3 = n0, n1, n2, n3
        if r != 9:
            k0 = (k0 + W0) & m32
            k1 = (k1 + W1) & m32
    return (c0.astype(np.uint32), c1.astype(np.uint32),
            c2.astype(np.uint32), c3.astype(np.uint32))
