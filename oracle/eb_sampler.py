"""The pages' own sampler: entropy-bounded acceptance with adaptive stopping, fp64.

TEST INFRASTRUCTURE ONLY (like the rest of oracle/): the reference the device
kernels of this sampler will be checked against; nothing on the product path
imports it.

Follows the hyper.ai digest of the DiffusionGemma paper:
* Method, sampler paragraph -- tokens are accepted in rank order from lowest to
  highest entropy while their mutual-information bound stays strictly below an
  error tolerance; once the tolerance is reached every other token is renoised
  uniformly at random; probabilities are tempered with tau annealed linearly
  from 0.8 to 0.4 over the fractional denoising time;
* Method, adaptive stopping -- denoising halts when the mean predictive entropy
  over the canvas falls below a threshold and the deterministic (argmax)
  predictions of two consecutive steps are identical;
* Experiment, sampler settings -- at most 48 steps (about 12 on average), with
  separate entropy thresholds for stopping and for token selection.

Readings taken where the pages leave a step open:
* entropy of a position: H = -sum_v p_v log p_v of p = Softmax(L / tau) (natural log);
* the mutual-information bound of an accepted set S is the one of entropy-bounded
  unmasking (Ben-Hamu et al. 2025): sum_{i in S} H_i - max_{i in S} H_i.  In
  ascending-entropy order the bound of the first k positions is the sum of the
  k - 1 smallest entropies, non-decreasing in k, so "accept in rank order while
  the bound stays below gamma" accepts the longest such prefix; the first
  position is always accepted (bound 0), so every step makes progress;
* accepted positions are committed to argmax_v L_v (ties: lower v) and frozen;
  ties in entropy rank by lower position;
* time of step s is t_s = 1 - s / T_max (T_max = the step budget, 48);
  tau_s = tau_min + (tau_max - tau_min) t_s;
* the stop test runs after a step's commit: mean entropy over all C positions of
  each canvas below the stop threshold, and the argmax canvas equal to the
  previous step's; on a stop (or on the last allowed step) every uncommitted
  position takes its argmax;
* re-noise draws come from the same Philox stream as the fixed-count sampler
  (position, step, sequence, tag 1).
"""
import numpy as np

from .philox import draw, uniform_index, TAG_RENOISE
from .sampler import tau_of_step


def entropy_rows(logits, tau):
    """Per row: (entropy of Softmax(L / tau), argmax of L with ties to the lowest index)."""
    L = np.asarray(logits, dtype=np.float64) / tau
    L = L - np.max(L, axis=-1, keepdims=True)
    e = np.exp(L)
    Z = np.sum(e, axis=-1, keepdims=True)
    p = e / Z
    # -sum p log p with log p = L - log Z (exact for p = 0 terms, which contribute 0)
    H = -np.sum(p * (L - np.log(Z)), axis=-1)
    arg = np.argmax(np.asarray(logits, dtype=np.float64), axis=-1)
    return H, arg.astype(np.int64)


def accept_count(h_sorted, gamma: float) -> int:
    """How many of the entropies h_sorted (ascending) are accepted: walk the rank
    order and stop before the first position whose admission would make the
    bound (sum of the admitted entropies minus their largest) reach gamma."""
    n = len(h_sorted)
    if n == 0:
        return 0
    total, largest, k = 0.0, 0.0, 0
    for h in h_sorted:
        if k > 0 and (total + h) - max(largest, h) >= gamma:
            break
        total += h
        largest = max(largest, h)
        k += 1
    return k


def sample_commit_eb(logits, tok, committed, s: int, T_max: int, seed: int, tau: float, gamma: float,
                     commit_all: bool = False):
    """One step of the entropy-bounded sampler over B canvases.

    logits [B][C][V]; tok [B][C] int; committed [B][C] bool.  Returns
    (new_tok, new_committed, info) with info["entropy"] [B][C],
    info["argmax"] [B][C] and info["new"] (positions committed this step).
    commit_all: commit every open position (stop or last step)."""
    L = np.asarray(logits, dtype=np.float64)
    B, C, V = L.shape
    tok = np.array(tok, dtype=np.int64, copy=True)
    committed = np.array(committed, dtype=bool, copy=True)
    H, arg = entropy_rows(L, tau)
    new_mask = np.zeros((B, C), dtype=bool)
    for b in range(B):
        open_pos = [i for i in range(C) if not committed[b, i]]
        order = sorted(open_pos, key=lambda i: (H[b, i], i))
        k = len(order) if (commit_all or s >= T_max - 1) else accept_count([H[b, i] for i in order], gamma)
        for i in order[:k]:
            tok[b, i] = arg[b, i]
            committed[b, i] = True
            new_mask[b, i] = True
        rest = np.array(order[k:], dtype=np.int64)
        if rest.size:
            w = draw(seed, rest, s, b, TAG_RENOISE)[..., 0]
            tok[b, rest] = uniform_index(w, V)
    return tok, committed, {"entropy": H, "argmax": arg, "new": new_mask}


def should_stop(entropy, argmax_now, argmax_prev, threshold: float):
    """Per canvas: mean entropy over its C positions < threshold and the argmax
    canvas identical to the previous step's (False when there is none)."""
    H = np.asarray(entropy, dtype=np.float64)
    if argmax_prev is None:
        return np.zeros(H.shape[0], dtype=bool)
    same = np.all(np.asarray(argmax_now) == np.asarray(argmax_prev), axis=-1)
    return (H.mean(axis=-1) < threshold) & same


def generate_block_eb(step_logits, tok0, seed: int, gamma: float, stop_threshold: float, T_max: int = 48,
                      tau_max: float = 0.8, tau_min: float = 0.4):
    """Denoise one block with the entropy-bounded sampler and adaptive stopping.

    step_logits(s, tok) -> logits [B][C][V] (the decoder on the current canvas).
    Returns (tokens [B][C], steps used per canvas).  A canvas is finished when
    all of its positions are committed or its stop test holds; finished canvases
    are left unchanged by later steps."""
    tok = np.array(tok0, dtype=np.int64, copy=True)
    B, C = tok.shape
    committed = np.zeros((B, C), dtype=bool)
    done = np.zeros(B, dtype=bool)
    steps = np.zeros(B, dtype=np.int64)
    prev_arg = None
    for s in range(T_max):
        if done.all():
            break
        tau = tau_of_step(s, T_max, tau_max, tau_min)
        L = step_logits(s, tok)
        new_tok, new_com, info = sample_commit_eb(L, tok, committed, s, T_max, seed, tau, gamma)
        stop = should_stop(info["entropy"], info["argmax"], prev_arg, stop_threshold)
        for b in range(B):
            if done[b]:
                continue
            steps[b] = s + 1
            if stop[b]:   # halt: every open position takes its argmax
                open_b = ~committed[b]
                new_tok[b, open_b] = info["argmax"][b, open_b]
                new_com[b] = True
            tok[b], committed[b] = new_tok[b], new_com[b]
            done[b] = committed[b].all()
        prev_arg = info["argmax"]
    return tok, steps
