"""FP8 (E4M3) expert weights and activations, fp64 (test infrastructure only).

The pages' throughput figures are for FP8 (hyper.ai digest of the DiffusionGemma
paper, Experiment: speed conditions), and the model is said to be quantized to
FP8 or NVFP4 for deployment (alphasignal.ai article, "Architecture").  The pages
fix no format details; the readings taken:

* format: OCP FP8 E4M3 ("fn": 4 exponent bits, 3 mantissa bits, bias 7, no
  infinities, largest finite value 448, smallest subnormal 2^-9), rounding to
  nearest with ties to even;
* scaling: one power-of-two scale per row -- per output row of every expert (and
  shared-FFN) weight matrix as stored, per token row of the activations that
  enter the expert GEMMs (the normed input of the MoE block, and the gated
  activation GELU(W_g x) * (W_u x) after its bf16 rounding) -- the smallest
  2^e with max |row| / 2^e <= 448 (a zero row takes 2^0), as in the shared
  exponents of the OCP microscaling formats.  Dividing by a power of two is
  exact, so every implementation quantizes a given row to the same values;
* arithmetic: the products of quantized values are summed and then multiplied
  by the two row scales; everything else (router, gates, GELU, combine) is
  unchanged from the bf16 path.
"""
import numpy as np

E4M3_MAX = 448.0


def e4m3_round(x):
    """Round fp64 values with |x| <= 448 to the nearest E4M3 value (ties to even),
    returned as fp64.  Normal range (|x| >= 2^-6): 4 significant bits,
    x = m 2^e with 0.5 <= |m| < 1 -> rint(16 m) 2^(e - 4); below it the quantum
    is 2^-9."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)
    normal = np.ldexp(np.rint(m * 16.0), e - 4)
    sub = np.rint(x * 512.0) / 512.0
    return np.where(np.abs(x) >= 2.0 ** -6, normal, sub)


def row_scale(x):
    """Per row (last axis): the smallest power of two s with max|row| / s <= 448
    (1 for a zero row)."""
    a = np.max(np.abs(np.asarray(x, dtype=np.float64)), axis=-1)
    m, e = np.frexp(a / E4M3_MAX)              # a / 448 = m 2^e, 0.5 <= m < 1
    k = np.where(m == 0.5, e - 1, e)           # ceil(log2(a / 448))
    return np.where(a > 0, np.ldexp(1.0, k), 1.0)


def quant_rows(x):
    """(q, s): q = E4M3(x / s) with s = row_scale(x) broadcast over the last axis."""
    s = row_scale(x)
    return e4m3_round(np.asarray(x, dtype=np.float64) / s[..., None]), s


def expert_ffn_fp8(xq, sx, gate_up, down):
    """Gated-GELU FFN in FP8: xq, sx the quantized token rows and their scales;
    gate_up = (q, s) of the stored [2w][d] gate/up tensor (rows interleaved in
    blocks of 16), down = (q, s) of [d][w].  Returns fp64 [n][d]."""
    from .decoder import split_gate_up
    from .numerics import bf16_round, gelu_tanh
    q_gu, s_gu = gate_up
    w_g, w_u = split_gate_up(q_gu)
    s_g, s_u = split_gate_up(s_gu[:, None])
    g = (xq @ w_g.T) * sx[:, None] * s_g[:, 0][None, :]
    u = (xq @ w_u.T) * sx[:, None] * s_u[:, 0][None, :]
    a = bf16_round(gelu_tanh(g) * u)
    aq, sa = quant_rows(a)
    q_d, s_d = down
    return (aq @ q_d.T) * sa[:, None] * s_d[None, :]
