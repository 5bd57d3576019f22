"""Philox4x32-10, written from its published definition (test infrastructure only).

Salmon, Moraes, Dror & Shaw, "Parallel random numbers: as easy as 1, 2, 3"
(SC'11), section 5 (the Philox S-box): a 4x32-bit counter and a 2x32-bit key;
each of the 10 rounds multiplies counter words 0 and 2 by fixed 32-bit
multipliers, splits each 64-bit product into high and low halves, and mixes the
high halves with the other two counter words and the round key; the key is
bumped by fixed Weyl constants between rounds.

The denoising method's random draws use it as:
  key     = (seed mod 2^32, seed >> 32)
  counter = (position, step, sequence, tag)   tag 0 initial canvas, 1 re-noise,
                                              2 forward noising
  token   = floor(word * V / 2^32) with word = output lane 0  (exactly uniform
            for power-of-two V; bias below V / 2^32 otherwise)
"""
import numpy as np

PHILOX_M0 = 0xD2511F53
PHILOX_M1 = 0xCD9E8D57
PHILOX_W0 = 0x9E3779B9
PHILOX_W1 = 0xBB67AE85
_MASK = np.uint64(0xFFFFFFFF)

TAG_INIT, TAG_RENOISE, TAG_FORWARD = 0, 1, 2


def philox4x32_10(counter, key):
    """counter: (..., 4) unsigned ints < 2^32; key: (2,) or (..., 2).  Returns (..., 4) uint32."""
    c = np.asarray(counter, dtype=np.uint64)
    k = np.asarray(key, dtype=np.uint64)
    x0, x1, x2, x3 = c[..., 0], c[..., 1], c[..., 2], c[..., 3]
    k0, k1 = k[..., 0] & _MASK, k[..., 1] & _MASK
    m0, m1 = np.uint64(PHILOX_M0), np.uint64(PHILOX_M1)
    for r in range(10):
        if r > 0:
            k0 = (k0 + np.uint64(PHILOX_W0)) & _MASK
            k1 = (k1 + np.uint64(PHILOX_W1)) & _MASK
        p0 = m0 * x0          # < 2^64: exact in uint64
        p1 = m1 * x2
        hi0, lo0 = p0 >> np.uint64(32), p0 & _MASK
        hi1, lo1 = p1 >> np.uint64(32), p1 & _MASK
        x0, x1, x2, x3 = hi1 ^ x1 ^ k0, lo1, hi0 ^ x3 ^ k1, lo0
    return np.stack([x0, x1, x2, x3], axis=-1).astype(np.uint32)


def seed_key(seed: int):
    seed = int(seed) & 0xFFFFFFFFFFFFFFFF
    return np.array([seed & 0xFFFFFFFF, seed >> 32], dtype=np.uint64)


def draw(seed: int, pos, step, seq, tag):
    """Philox words for counters (pos, step, seq, tag), broadcast over the inputs."""
    pos, step, seq, tag = np.broadcast_arrays(np.asarray(pos), np.asarray(step), np.asarray(seq), np.asarray(tag))
    ctr = np.stack([pos, step, seq, tag], axis=-1).astype(np.uint64)
    return philox4x32_10(ctr, seed_key(seed))


def uniform_index(word, V: int):
    """floor(word * V / 2^32) -- multiply-shift map of a 32-bit word to [0, V)."""
    return ((np.asarray(word, dtype=np.uint64) * np.uint64(V)) >> np.uint64(32)).astype(np.int64)
