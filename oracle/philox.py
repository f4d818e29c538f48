"""Counter-based Philox4x32-10 and the round's uniforms, for the CPU oracle.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / reference leg of ``bench.py`` may import this package.

Philox4x32-10 follows Salmon, Moraes, Dror and Shaw, "Parallel random
numbers: as easy as 1, 2, 3" (SC'11), section 4: a 4-word counter and a
2-word key; each of the ten rounds multiplies counter words 0 and 2 by the
two round multipliers, swaps the 64-bit products' halves into the output
with the key XORed in, and the key is bumped by the two Weyl constants
between rounds.

How the speculative round draws its uniforms is not fixed by the pages
(they only require that rejection sampling uses fresh uniforms); the reading
used here, shared with the CUDA path by definition only:

* key      = (lo32(seed), hi32(seed))
* counter  = (request b, (purpose << 24) | position, lo32(round_id), hi32(round_id))
* purpose  = 0 draft sample, 1 acceptance test, 2 residual sample, 3 bonus sample
* position = 1-based draft position k for purposes 0 and 1; for 2 and 3 the
             1-based block position of the emitted correction/bonus token (a+1)
* u        = (word0 >> 8) * 2**-24, a 24-bit uniform in [0, 1) that is exact
             in both fp32 and fp64.
"""
from __future__ import annotations

import numpy as np

PHILOX_M0 = 0xD2511F53
PHILOX_M1 = 0xCD9E8D57
PHILOX_W0 = 0x9E3779B9
PHILOX_W1 = 0xBB67AE85

PURPOSE_DRAFT = 0
PURPOSE_ACCEPT = 1
PURPOSE_RESIDUAL = 2
PURPOSE_BONUS = 3

_MASK32 = np.uint64(0xFFFFFFFF)


def philox4x32_10(ctr, key):
    """Philox4x32 with 10 rounds on arrays of counters.

    ``ctr`` is a sequence of four uint32-valued arrays (broadcastable),
    ``key`` a sequence of two. Returns the four output words as uint64
    arrays holding 32-bit values.
    """
    c0, c1, c2, c3 = (np.asarray(c, dtype=np.uint64) & _MASK32 for c in ctr)
    k0, k1 = (np.asarray(k, dtype=np.uint64) & _MASK32 for k in key)
    m0 = np.uint64(PHILOX_M0)
    m1 = np.uint64(PHILOX_M1)
    for rnd in range(10):
        if rnd:
            k0 = (k0 + np.uint64(PHILOX_W0)) & _MASK32
            k1 = (k1 + np.uint64(PHILOX_W1)) & _MASK32
        p0 = m0 * c0  # < 2**64: exact in uint64
        p1 = m1 * c2
        hi0, lo0 = p0 >> np.uint64(32), p0 & _MASK32
        hi1, lo1 = p1 >> np.uint64(32), p1 & _MASK32
        c0, c1, c2, c3 = hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0
    return c0, c1, c2, c3


def uniform(seed: int, request, position, purpose: int, round_id: int):
    """The 24-bit uniform u(seed, request, position, purpose, round) in [0, 1)."""
    seed = int(seed) & 0xFFFFFFFFFFFFFFFF
    round_id = int(round_id) & 0xFFFFFFFFFFFFFFFF
    req = np.asarray(request, dtype=np.uint64)
    pos = np.asarray(position, dtype=np.uint64)
    w1 = (np.uint64(purpose) << np.uint64(24)) | pos
    out0, _, _, _ = philox4x32_10(
        (req, w1, np.uint64(round_id & 0xFFFFFFFF), np.uint64(round_id >> 32)),
        (np.uint64(seed & 0xFFFFFFFF), np.uint64(seed >> 32)),
    )
    return (out0 >> np.uint64(8)).astype(np.float64) * 2.0 ** -24
