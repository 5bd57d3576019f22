"""Elementwise and row operations of the decoder, fp64 (test infrastructure only).

The pages fix none of these details ("RMSNorm + RoPE, gated-GELU" is all the
workload descriptions say); the readings taken are the plainest standard ones:
RMSNorm with a (1 + g) gain and eps 1e-6, rotate-half RoPE with base 10000,
the tanh form of GELU (Hendrycks & Gimpel 2016), no embedding scale.
"""
import contextlib

import numpy as np

# When False, bf16_round is the identity: the pure-fp64 reading of the method,
# used to pin the oracle against library implementations that do not round.
ROUND_TO_BF16 = True


@contextlib.contextmanager
def pure_fp64():
    global ROUND_TO_BF16
    old, ROUND_TO_BF16 = ROUND_TO_BF16, False
    try:
        yield
    finally:
        ROUND_TO_BF16 = old


def bf16_round(x):
    """Round fp64 values to the nearest bf16 value (ties to even), returned as fp64.

    x = m * 2^e with 0.5 <= |m| < 1; bf16 keeps 8 significant bits, so the
    result is rint(m * 256) * 2^(e-8) (np.rint rounds halves to even).  Values
    below bf16's normal range (|x| < 2^-126) do not occur on this path.
    """
    if not ROUND_TO_BF16:
        return np.asarray(x, dtype=np.float64)
    m, e = np.frexp(np.asarray(x, dtype=np.float64))
    return np.ldexp(np.rint(m * 256.0), e - 8)


def bf16_bits_to_f64(bits):
    """Widen bf16 bit patterns (uint16) to float64 exactly."""
    return (np.asarray(bits).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def rmsnorm(x, g, eps):
    """x / sqrt(mean(x^2) + eps) * (1 + g) over the last axis."""
    x = np.asarray(x, dtype=np.float64)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * (1.0 + g)


def rope_angles(pos, head_dim, base):
    """angle[p, j] = pos[p] * base^(-2j / head_dim), j < head_dim / 2."""
    j = np.arange(head_dim // 2, dtype=np.float64)
    inv_freq = base ** (-2.0 * j / head_dim)
    return np.asarray(pos, dtype=np.float64)[:, None] * inv_freq[None, :]


def rope(x, pos, base):
    """Rotate-half rotary embedding of x[..., n, hd] at absolute positions pos[n]:
    pairs (j, j + hd/2) are rotated by angle pos * base^(-2j/hd)."""
    hd = x.shape[-1]
    ang = rope_angles(pos, hd, base)
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., : hd // 2], x[..., hd // 2:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def gelu_tanh(x):
    return 0.5 * x * (1.0 + np.tanh(np.sqrt(2.0 / np.pi) * (x + 0.044715 * x ** 3)))


def softmax(x, axis=-1):
    m = np.max(x, axis=axis, keepdims=True)
    e = np.exp(x - m)
    return e / np.sum(e, axis=axis, keepdims=True)
