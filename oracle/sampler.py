"""The sampler side of one denoising step, fp64 (test infrastructure only).

Follows:
* hyper.ai digest of the DiffusionGemma paper, Method, eq. 1 -- the forward
  process q(x_t | x_0) = prod_i [kappa_t delta(x_t^i, x_0^i) + (1 - kappa_t)/V],
  kappa decreasing from 1 at t = 0 to 0 at t = 1 (linear here, as the workloads
  state: kappa(t) = 1 - t);
* same page, Method, eq. 4 first line -- p0_hat = Softmax(L_t / tau_t);
* same page, Method (sampler paragraph) and Experiment (sampler settings) --
  tau annealed linearly from 0.8 to 0.4 over the fractional time, and "all
  other tokens are renoised uniformly at random";
* alphasignal.ai, "How text diffusion actually works", step 2 -- locking in
  the high-confidence tokens on each pass.

Readings taken where the pages leave a step open:
* step s of T sits at time t_s = 1 - s/T; tau_s = tau_min + (tau_max - tau_min) t_s;
* confidence of a position = log of its largest tempered probability,
  conf = -log sum_v exp((L_v - L_max) / tau);
* on each step the m_s = min(ceil(C/T), #uncommitted) uncommitted positions of
  highest confidence (ties: lower position first) are committed to argmax_v L_v
  (ties: lower v) and frozen; on the last step (s = T-1) every uncommitted
  position is committed; every other uncommitted position is redrawn uniformly
  from Philox(seed; position, s, sequence, tag 1);
* the initial canvas is uniform from Philox(seed; position, 0, sequence, tag 0);
* the blocks after the first of a sequence (block-autoregressive generation,
  hyper.ai digest, Method) draw at positions offset by (block index) x C, so
  every block of a sequence gets fresh Philox words.
"""
import math

import numpy as np

from .philox import draw, uniform_index, TAG_INIT, TAG_RENOISE, TAG_FORWARD


def time_of_step(s: int, T: int) -> float:
    return 1.0 - s / T


def kappa(t: float) -> float:
    """Linear schedule: kappa_0 = 1 (clean), kappa_1 = 0 (uniform noise)."""
    return 1.0 - t


def tau_of_step(s: int, T: int, tau_max: float = 0.8, tau_min: float = 0.4) -> float:
    return tau_min + (tau_max - tau_min) * time_of_step(s, T)


def commit_count(s: int, T: int, C: int, n_uncommitted: int, commit_per_step: int = 0) -> int:
    m = commit_per_step if commit_per_step > 0 else math.ceil(C / T)
    if s >= T - 1:
        return n_uncommitted
    return min(m, n_uncommitted)


def row_stats(logits, tau):
    """Per row: (argmax, confidence) of Softmax(L / tau); argmax ties -> lowest index."""
    L = np.asarray(logits, dtype=np.float64)
    arg = np.argmax(L, axis=-1)            # first occurrence of the maximum
    lmax = np.max(L, axis=-1, keepdims=True)
    conf = -np.log(np.sum(np.exp((L - lmax) / tau), axis=-1))
    return arg.astype(np.int64), conf


def init_canvas(seed: int, B: int, C: int, V: int, pos_offset: int = 0):
    pos = pos_offset + np.arange(C)[None, :]
    seq = np.arange(B)[:, None]
    w = draw(seed, pos, 0, seq, TAG_INIT)[..., 0]
    return uniform_index(w, V)


def forward_noise(x0, kap: float, seed: int, step: int = 0):
    """Sample x_t ~ q(x_t | x_0) (eq. 1) at schedule value kappa: keep x0 with
    probability kappa (Philox lane 1 below floor(kappa * 2^32)), else a uniform
    token from lane 0, which may itself equal x0."""
    x0 = np.asarray(x0)
    B, C = x0.shape
    threshold = int(math.floor(kap * 2.0 ** 32))
    pos = np.arange(C)[None, :]
    seq = np.arange(B)[:, None]
    w = draw(seed, pos, step, seq, TAG_FORWARD)
    keep = w[..., 1].astype(np.uint64) < np.uint64(threshold)
    return keep, w


def forward_noise_tokens(x0, kap: float, seed: int, V: int, step: int = 0):
    keep, w = forward_noise(x0, kap, seed, step)
    return np.where(keep, np.asarray(x0), uniform_index(w[..., 0], V))


def sample_commit(logits, tok, committed, s: int, T: int, seed: int, tau: float, commit_per_step: int = 0,
                  pos_offset: int = 0):
    """One sampler step over B canvases.

    logits [B][C][V]; tok [B][C] int; committed [B][C] bool.  Returns
    (new_tok, new_committed, info) where info carries argmax, conf, the
    committed-this-step mask and, per canvas, the confidence margin between the
    last committed and the first passed-over position (inf if none)."""
    L = np.asarray(logits, dtype=np.float64)
    B, C, V = L.shape
    tok = np.array(tok, dtype=np.int64, copy=True)
    committed = np.array(committed, dtype=bool, copy=True)
    arg, conf = row_stats(L, tau)
    new_mask = np.zeros((B, C), dtype=bool)
    margins = np.full(B, np.inf)
    for b in range(B):
        open_pos = [i for i in range(C) if not committed[b, i]]
        order = sorted(open_pos, key=lambda i: (-conf[b, i], i))
        m = commit_count(s, T, C, len(open_pos), commit_per_step)
        chosen = order[:m]
        if 0 < m < len(order):
            margins[b] = conf[b, order[m - 1]] - conf[b, order[m]]
        for i in chosen:
            tok[b, i] = arg[b, i]
            committed[b, i] = True
            new_mask[b, i] = True
        rest = np.array([i for i in order[m:]], dtype=np.int64)
        if rest.size:
            w = draw(seed, pos_offset + rest, s, b, TAG_RENOISE)[..., 0]
            tok[b, rest] = uniform_index(w, V)
    return tok, committed, {"argmax": arg, "conf": conf, "new": new_mask, "margin": margins}
