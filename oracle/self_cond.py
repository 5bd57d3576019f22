"""Self-conditioning of the decoder, fp64 (test infrastructure only).

hyper.ai digest of the DiffusionGemma paper, Method: the decoder takes a
continuous self-conditioning signal z_t in R^{C x d} that feeds the model's
previous predictions back into itself (eq. 3: L_t = Decoder(x_t, z_t, H)); after
each step z_{t - dt} = FFW(p0_hat E) with p0_hat = Softmax(L_t / tau_t) (eq. 4,
second line), E the token embedding and FFW "a standard feedforward network";
Dataset: the model is trained with a zero state for half of the batch.
Experiment: the self-conditioning block adds little overhead.

Readings where the pages are silent:
* z enters by addition to the canvas token embedding at the decoder's input,
  h_0 = E[x_t] + z_t; z = 0 at the first step of a block (and with teacher
  forcing unless given); the prompt pass and the canvas append do not use it;
* p0_hat uses the step's own temperature (the sampler's tau_s); it is rounded
  to bf16 before the product with E (a GEMM operand);
* FFW is the model's FFN form with its own weights: a pre-RMSNorm (gain
  applied as 1 + g) gated-GELU FFN of width w_sc, d -> w_sc -> d, with the
  gate/up rows interleaved in blocks of 16 like the experts'; the normed input
  and the activation are rounded to bf16 (GEMM operands), z stays fp64.
"""
import numpy as np

from .numerics import bf16_round, rmsnorm, softmax
from .decoder import expert_ffn


def probs_times_embedding(W, logits, tau):
    """p0_hat E for logits [n][V] (fp64): softmax of L / tau, rounded to bf16,
    times the embedding, accumulated over vocabulary chunks."""
    L = np.asarray(logits, dtype=np.float64).reshape(-1, W.wl.vocab)
    p = bf16_round(softmax(L / tau, axis=-1))
    u = np.zeros((L.shape[0], W.wl.d_model))
    for r0, E in W.embed_chunks():
        u += p[:, r0:r0 + E.shape[0]] @ E
    return u


def ffw(W, u):
    """FFW(u) = W_d (GELU(W_g n) * (W_u n)), n = bf16(RMSNorm(u) (1 + g))."""
    wl = W.wl
    n = bf16_round(rmsnorm(u, W.get("sc_norm"), wl.rms_eps))
    return expert_ffn(n, W.get("w_sc_gate_up"), W.get("w_sc_down"))


def next_state(W, logits, tau):
    """z for the next step: FFW(p0_hat E), shaped [B][C][d]."""
    wl = W.wl
    z = ffw(W, probs_times_embedding(W, logits, tau))
    return z.reshape(-1, wl.canvas, wl.d_model)
