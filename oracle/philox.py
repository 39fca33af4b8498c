"""Philox4x32-10 and the Gumbel noise the temperature sampler draws from it.

Test infrastructure only: part of the CPU oracle.

Philox4x32 is defined in J. K. Salmon, M. A. Moraes, R. O. Dror and
D. E. Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3" (SC'11), section 3:
a 128-bit counter (four 32-bit words) is transformed by R rounds keyed by a
64-bit key (two words). One round multiplies words 0 and 2 by the constants
0xD2511F53 and 0xCD9E8D57, keeping both halves of each 64-bit product; the
new words are (hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0). Between rounds the key
is advanced by the Weyl constants 0x9E3779B9 (golden ratio) and 0xBB67AE85
(sqrt(3) - 1). Philox4x32-10 uses ten rounds.

Counter layout for the sampler's noise (keyed (seed, b, k, v)); the method's
pages do not fix one, so this is the chosen reading:
    key     = (seed & 0xFFFFFFFF, seed >> 32)
    counter = (v >> 2, k, b, 0)
and output word ``v & 3`` is the draw for vocabulary id ``v``: one Philox call
serves four consecutive ids.
"""
from __future__ import annotations

import numpy as np

PHILOX_M0 = 0xD2511F53
PHILOX_M1 = 0xCD9E8D57
PHILOX_W0 = 0x9E3779B9
PHILOX_W1 = 0xBB67AE85
MASK32 = 0xFFFFFFFF


def _mulhilo(a: np.ndarray, m: int):
    p = a.astype(np.uint64) * np.uint64(m)
    return (p >> np.uint64(32)).astype(np.uint32), (p & np.uint64(MASK32)).astype(np.uint32)


def philox4x32(counter, key, rounds: int = 10):
    """Philox4x32-R over arrays. ``counter`` is four broadcastable uint32
    arrays, ``key`` two integers. Returns the four output words."""
    c0, c1, c2, c3 = np.broadcast_arrays(*(np.asarray(c, dtype=np.uint32) for c in counter))
    k0, k1 = int(key[0]) & MASK32, int(key[1]) & MASK32
    for _ in range(rounds):
        hi0, lo0 = _mulhilo(c0, PHILOX_M0)
        hi1, lo1 = _mulhilo(c2, PHILOX_M1)
        c0, c1, c2, c3 = hi1 ^ c1 ^ np.uint32(k0), lo1, hi0 ^ c3 ^ np.uint32(k1), lo0
        k0 = (k0 + PHILOX_W0) & MASK32
        k1 = (k1 + PHILOX_W1) & MASK32
    return c0, c1, c2, c3


def noise_words(seed: int, b: int, k: int, vocab: int) -> np.ndarray:
    """The 32-bit draw for every vocabulary id of row b at step k."""
    v = np.arange(vocab, dtype=np.int64)
    blocks = np.arange((vocab + 3) // 4, dtype=np.uint32)
    key = (seed & MASK32, (seed >> 32) & MASK32)
    w = philox4x32((blocks, np.uint32(k), np.uint32(b), np.uint32(0)), key)
    words = np.stack(w, axis=1).reshape(-1)  # word j of block i is id 4i + j
    return words[v]


def uniform_from_word(w: np.ndarray) -> np.ndarray:
    """u = (2 * (w >> 9) + 1) * 2^-24: the top 23 bits as an odd multiple of
    2^-24, so u lies strictly inside (0, 1) and is exact in binary32."""
    w = np.asarray(w, dtype=np.uint32)
    return (2.0 * (w >> np.uint32(9)).astype(np.float64) + 1.0) * 2.0 ** -24


def gumbel_from_uniform(u: np.ndarray) -> np.ndarray:
    """Standard Gumbel variate by inversion: g = -log(-log u)."""
    return -np.log(-np.log(np.asarray(u, dtype=np.float64)))


def gumbel_noise(seed: int, b: int, k: int, vocab: int) -> np.ndarray:
    return gumbel_from_uniform(uniform_from_word(noise_words(seed, b, k, vocab)))
