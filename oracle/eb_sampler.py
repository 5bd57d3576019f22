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
* the sampler paragraph renoises "all other tokens" and never speaks of freezing;
  the variant freeze=False takes that literally: every position is a candidate
  at every step (earlier choices can be revised -- the self-correction the
  digest's Key Contributions mention), the accepted prefix takes its argmax and
  every other position is redrawn;
* time of step s is t_s = 1 - s / T_max (T_max = the step budget, 48);
  tau_s = tau_min + (tau_max - tau_min) t_s;
* the stop test runs after a step's commit: mean entropy over all C positions of
  each canvas below the stop threshold, and the argmax canvas equal to the
  previous step's; on a stop (or on the last allowed step) every candidate
  position takes its argmax; a canvas that stopped (or, frozen, has every
  position committed) is done and keeps its tokens for the rest of the block;
* re-noise draws come from the same Philox stream as the fixed-count sampler
  (position offset + position, step, sequence, tag 1).
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
                     commit_all=False, freeze: bool = True, pos_offset: int = 0, active=None):
    """One step of the entropy-bounded sampler over B canvases.

    logits [B][C][V]; tok [B][C] int; committed [B][C] bool.  Returns
    (new_tok, new_committed, info) with info["entropy"] [B][C],
    info["argmax"] [B][C] and info["new"] (positions accepted this step).
    commit_all (bool, or one bool per canvas): every candidate takes its argmax
    (stop or last step).  freeze: candidates are the uncommitted positions (True)
    or all positions.  active (one bool per canvas, default all): canvases not
    active are left unchanged."""
    L = np.asarray(logits, dtype=np.float64)
    B, C, V = L.shape
    tok = np.array(tok, dtype=np.int64, copy=True)
    committed = np.array(committed, dtype=bool, copy=True)
    H, arg = entropy_rows(L, tau)
    new_mask = np.zeros((B, C), dtype=bool)
    all_b = np.broadcast_to(np.asarray(commit_all, dtype=bool), (B,))
    act = np.ones(B, dtype=bool) if active is None else np.asarray(active, dtype=bool)
    for b in range(B):
        if not act[b]:
            continue
        cand = [i for i in range(C) if not (freeze and committed[b, i])]
        order = sorted(cand, key=lambda i: (H[b, i], i))
        k = len(order) if (all_b[b] or s >= T_max - 1) else accept_count([H[b, i] for i in order], gamma)
        for i in order[:k]:
            tok[b, i] = arg[b, i]
            committed[b, i] = True
            new_mask[b, i] = True
        rest = np.array(order[k:], dtype=np.int64)
        if rest.size:
            w = draw(seed, pos_offset + rest, s, b, TAG_RENOISE)[..., 0]
            tok[b, rest] = uniform_index(w, V)
            committed[b, rest] = False
    return tok, committed, {"entropy": H, "argmax": arg, "new": new_mask}


def should_stop(entropy, argmax_now, argmax_prev, threshold: float):
    """Per canvas: mean entropy over its C positions < threshold and the argmax
    canvas identical to the previous step's (False when there is none)."""
    H = np.asarray(entropy, dtype=np.float64)
    if argmax_prev is None:
        return np.zeros(H.shape[0], dtype=bool)
    same = np.all(np.asarray(argmax_now) == np.asarray(argmax_prev), axis=-1)
    return (H.mean(axis=-1) < threshold) & same


def block_step_eb(logits, tok, committed, done, prev_arg, s: int, T_max: int, seed: int, tau: float, gamma: float,
                  stop_threshold: float, freeze: bool = True, pos_offset: int = 0):
    """One step of a block: the stop test (s > 0) decides commit_all per canvas;
    canvases done earlier in the block are left unchanged.  Returns (tok,
    committed, done, stop, info); a canvas is done once it stops, at the last
    step, or (frozen) once every position is committed."""
    B = np.asarray(logits).shape[0]
    prev_done = np.asarray(done, dtype=bool) if s > 0 else np.zeros(B, dtype=bool)
    H, arg = entropy_rows(logits, tau)
    stop = should_stop(H, arg, prev_arg, stop_threshold) if s > 0 else np.zeros(B, dtype=bool)
    tok, committed, info = sample_commit_eb(logits, tok, committed, s, T_max, seed, tau, gamma, commit_all=stop,
                                            freeze=freeze, pos_offset=pos_offset, active=~prev_done)
    now = stop | (s >= T_max - 1) | (committed.all(axis=1) if freeze else np.zeros(B, dtype=bool))
    done = prev_done | now
    return tok, committed, done, stop, info


def generate_block_eb(step_logits, tok0, seed: int, gamma: float, stop_threshold: float, T_max: int = 48,
                      tau_max: float = 0.8, tau_min: float = 0.4, freeze: bool = True, pos_offset: int = 0):
    """Denoise one block with the entropy-bounded sampler and adaptive stopping.

    step_logits(s, tok) -> logits [B][C][V] (the decoder on the current canvas).
    Returns (tokens [B][C], steps used per canvas).  Done canvases (see
    block_step_eb) are left unchanged by later steps; the block ends when every
    canvas is done."""
    tok = np.array(tok0, dtype=np.int64, copy=True)
    B, C = tok.shape
    committed = np.zeros((B, C), dtype=bool)
    done = np.zeros(B, dtype=bool)
    steps = np.zeros(B, dtype=np.int64)
    prev_arg = None
    for s in range(T_max):
        if s > 0 and done.all():
            break
        tau = tau_of_step(s, T_max, tau_max, tau_min)
        was = done.copy()
        tok, committed, done, _, info = block_step_eb(step_logits(s, tok), tok, committed, done, prev_arg, s, T_max,
                                                      seed, tau, gamma, stop_threshold, freeze, pos_offset)
        steps[done & ~was] = s + 1
        prev_arg = info["argmax"]
    return tok, steps
