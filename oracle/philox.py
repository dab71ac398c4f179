"""Philox4x32-10 and the canvas's uniform vocabulary draws (oracle side).

[philox] defines Philox4x32-R: a 128-bit counter (four 32-bit words) and a 64-bit
key (two words).  Each round multiplies counter words 0 and 2 by two fixed
32-bit multipliers, keeping both halves of each 64-bit product, and recombines:

    (hi0, lo0) = mulhilo(0xD2511F53, c0)
    (hi1, lo1) = mulhilo(0xCD9E8D57, c2)
    c' = (hi1 ^ c1 ^ k0,  lo1,  hi0 ^ c3 ^ k1,  lo0)

after which the key is bumped by the Weyl constants (0x9E3779B9, 0xBB67AE85).
Ten rounds are applied (the key bump happens between rounds).

The canvas uses one Philox block per (seed, block, step, position) ([canvas]
step 2 and step 3: the initial canvas and re-noised positions are ids drawn
uniformly from the whole vocabulary).  Counter = (position, step, block, tag),
key = (seed & 0xffffffff, seed >> 32); tag 0 is the initial fill (step 0),
tag 1 a re-noise at step t >= 1.  The id is floor(r0 * V / 2**32) with r0 the
first output word, which is exactly uniform whenever V is a power of two.

Vectorised over numpy uint64 arrays: every 32x32-bit product fits in 64 bits.
"""
import numpy as np

MUL0 = 0xD2511F53
MUL1 = 0xCD9E8D57
WEYL0 = 0x9E3779B9
WEYL1 = 0xBB67AE85
MASK32 = 0xFFFFFFFF

TAG_INIT = 0
TAG_RENOISE = 1


def philox4x32_10(c0, c1, c2, c3, k0, k1, rounds=10):
    """Return the four output words for counters (c0..c3) and key (k0, k1).

    Inputs may be Python ints or integer arrays (broadcast together); outputs are
    uint64 arrays holding 32-bit values.
    """
    c0, c1, c2, c3 = (np.asarray(c, dtype=np.uint64) & np.uint64(MASK32) for c in (c0, c1, c2, c3))
    k0 = np.asarray(k0, dtype=np.uint64) & np.uint64(MASK32)
    k1 = np.asarray(k1, dtype=np.uint64) & np.uint64(MASK32)
    m32 = np.uint64(MASK32)
    for r in range(rounds):
        p0 = np.uint64(MUL0) * c0
        p1 = np.uint64(MUL1) * c2
        hi0, lo0 = p0 >> np.uint64(32), p0 & m32
        hi1, lo1 = p1 >> np.uint64(32), p1 & m32
        c0, c1, c2, c3 = (hi1 ^ c1 ^ k0) & m32, lo1, (hi0 ^ c3 ^ k1) & m32, lo0
        if r != rounds - 1:
            k0 = (k0 + np.uint64(WEYL0)) & m32
            k1 = (k1 + np.uint64(WEYL1)) & m32
    return c0, c1, c2, c3


def uniform_ids(seed, block, step, positions, tag, vocab):
    """Ids drawn uniformly from [0, vocab) for the given canvas positions.

    One Philox block per position; counter (position, step, block, tag), key
    from the 64-bit seed; id = floor(r0 * vocab / 2**32).
    """
    seed = int(seed)
    pos = np.asarray(positions, dtype=np.uint64)
    r0, _, _, _ = philox4x32_10(pos, step, block, tag, seed & MASK32, (seed >> 32) & MASK32)
    return ((r0 * np.uint64(vocab)) >> np.uint64(32)).astype(np.int64)
