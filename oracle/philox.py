"""Philox4x32-10 and the shared Gumbel noise of coupled-noise verification (oracle).

Test infrastructure only (see the package docstring).

[SPOT] section 1, "Coupled-Noise Verification": at temperature T > 0 the
drafter and the target draw the *same* Gumbel noise, so that, given the noise,
the target's choice is a deterministic function of its logits and the output
distribution is preserved. The pages do not say which generator produces the
noise; we take Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel Random
Numbers: As Easy as 1, 2, 3", SC'11), a counter-based generator, so that any
(candidate, position, vocabulary entry) can be drawn independently.

Our reading of the counter layout (the pages give none):
  key     = (seed mod 2^32, seed >> 32)
  counter = (v >> 2, position, candidate/batch index b, step mod 2^32)
  word    = output word (v & 3) of that counter
  U       = (2 * (word >> 9) + 1) * 2^-24      -- 23 random bits, exact in fp32, U in (0, 1)
  g       = -ln(-ln U)                           -- standard Gumbel
"""
from __future__ import annotations

import numpy as np

# Philox4x32 round multipliers and key-schedule (Weyl) increments, from the SC'11 paper.
PHILOX4x32_M = (0xD2511F53, 0xCD9E8D57)
PHILOX4x32_W = (0x9E3779B9, 0xBB67AE85)
# The 64-bit instance, used only to check the round structure against numpy.
PHILOX4x64_M = (0xD2E7470EE14C6C93, 0xCA5A826395121157)
PHILOX4x64_W = (0x9E3779B97F4A7C15, 0xBB67AE8584CAA73B)


def philox_generic(x, key, width, multipliers, weyl, rounds=10):
    """Philox4xW: `rounds` applications of the Philox S-box to the 4-word counter x.

    One round with key (k0, k1): multiply word 0 by M0 and word 2 by M1 into
    (hi, lo) halves; the new words are
        (hi(M1*x2) ^ x1 ^ k0,  lo(M1*x2),  hi(M0*x0) ^ x3 ^ k1,  lo(M0*x0)),
    then the key is bumped by the Weyl increments. Works on Python ints, object
    arrays, or (for width 32) uint64 numpy arrays holding 32-bit words.
    """
    mask = (1 << width) - 1
    x0, x1, x2, x3 = x
    k0, k1 = int(key[0]), int(key[1])
    for _ in range(rounds):
        p0 = x0 * multipliers[0]
        p1 = x2 * multipliers[1]
        hi0, lo0 = p0 >> width, p0 & mask
        hi1, lo1 = p1 >> width, p1 & mask
        x0, x1, x2, x3 = hi1 ^ x1 ^ k0, lo1, hi0 ^ x3 ^ k1, lo0
        k0 = (k0 + weyl[0]) & mask
        k1 = (k1 + weyl[1]) & mask
    return x0, x1, x2, x3


def philox4x32_10(counter, key):
    """Philox4x32-10 on arrays. counter: 4 integer arrays (32-bit words), key: (k0, k1).
    Returns 4 uint32 arrays."""
    x = tuple(np.asarray(c, dtype=np.uint64) & np.uint64(0xFFFFFFFF) for c in counter)
    out = philox_generic(x, (int(key[0]) & 0xFFFFFFFF, int(key[1]) & 0xFFFFFFFF), 32,
                         PHILOX4x32_M, PHILOX4x32_W)
    return tuple(o.astype(np.uint32) for o in out)


def uniform_from_word(word):
    """U = (2*(word >> 9) + 1) * 2^-24 in fp64 (exactly representable in fp32)."""
    w = np.asarray(word, dtype=np.uint64)
    return (2.0 * (w >> np.uint64(9)).astype(np.float64) + 1.0) * 2.0 ** -24


def noise_words(seed: int, step: int, b: int, pos, v):
    """The Philox output word for each (pos, v) pair (broadcast) of batch entry b."""
    pos = np.asarray(pos, dtype=np.uint64)
    v = np.asarray(v, dtype=np.uint64)
    pos, v = np.broadcast_arrays(pos, v)
    key = (seed & 0xFFFFFFFF, (seed >> 32) & 0xFFFFFFFF)
    ctr = (v >> np.uint64(2), pos, np.full_like(v, b), np.full_like(v, step & 0xFFFFFFFF))
    words = philox4x32_10(ctr, key)
    lane = (v & np.uint64(3)).astype(np.int64)
    stacked = np.stack(words, axis=0)
    return np.take_along_axis(stacked, lane[None], axis=0)[0]


def gumbel(seed: int, step: int, b: int, pos, v):
    """Standard Gumbel noise g = -ln(-ln U) in fp64 for (b, pos, v)."""
    u = uniform_from_word(noise_words(seed, step, b, pos, v))
    return -np.log(-np.log(u))


# Counter word 0 of the decision draws: above every vocabulary counter (v >> 2 < 2^30
# for any int32 vocabulary index), so a decision draw never reuses sampling noise.
DECISION_COUNTER = 0x80000000


def decision_uniform(seed: int, step: int, b: int, pos: int) -> float:
    """U of the stochastic decisions at (b, pos): word 0 of Philox4x32-10 at counter
    (2^31, pos, b, step), mapped like the sampling noise, U = (2 (w >> 9) + 1) 2^-24."""
    key = (seed & 0xFFFFFFFF, (seed >> 32) & 0xFFFFFFFF)
    ctr = tuple(np.array([c], dtype=np.uint64) for c in
                (DECISION_COUNTER, pos, b, step & 0xFFFFFFFF))
    w = philox4x32_10(ctr, key)[0][0]
    return float(uniform_from_word(w))
