"""One denoising step and one whole block, composed from the oracle's parts (test infrastructure only).

hyper.ai digest of the DiffusionGemma paper, Method, three-stage pipeline:
stage 1 (causal prompt pass -> cache) and stage 2 (iterative refinement of a
noisy canvas); each refinement step computes L_t (eq. 3), p0_hat (eq. 4) and
the next canvas through the sampler.
"""
import numpy as np

from . import decoder, sampler


def prompt_cache(W: decoder.Weights, prompt=None):
    wl = W.wl
    if wl.prompt_kv_given:
        return decoder.given_prompt_cache(wl)
    import synth
    return decoder.prefill(W, synth.prompt_tokens(wl) if prompt is None else prompt)


def denoise_step(W: decoder.Weights, cache, tok, committed, s: int, T: int, seed: int, pos_offset: int = 0,
                 z=None):
    """One step; with self-conditioning (self_cond_width > 0) z is this step's
    state (None: zero) and info["z_next"] the next step's."""
    wl = W.wl
    logits, diag = decoder.decoder_logits(W, tok, cache, z=z)
    tau = sampler.tau_of_step(s, T, wl.tau_max, wl.tau_min)
    new_tok, new_committed, info = sampler.sample_commit(logits, tok, committed, s, T, seed, tau,
                                                         wl.commit_per_step, pos_offset)
    info["router_margin"] = diag["margin"]
    if wl.self_cond_width:
        from . import self_cond
        info["z_next"] = self_cond.next_state(W, logits, tau)
    return logits, new_tok, new_committed, info


def generate_block(W: decoder.Weights, T: int, seed: int, prompt=None, cache=None, keep_logits=False,
                   pos_offset: int = 0):
    wl = W.wl
    if cache is None:
        cache = prompt_cache(W, prompt)
    tok = sampler.init_canvas(seed, wl.batch, wl.canvas, wl.vocab, pos_offset)
    committed = np.zeros_like(tok, dtype=bool)
    trace = []
    z = None
    for s in range(T):
        logits, tok, committed, info = denoise_step(W, cache, tok, committed, s, T, seed, pos_offset, z)
        z = info.get("z_next")
        trace.append({"tok": tok.copy(), "committed": committed.copy(), "info": info,
                      "logits": logits if keep_logits else None})
    return tok, committed, trace


def generate(W: decoder.Weights, n_blocks: int, T: int, seed: int, prompt=None, routing=None):
    """Block-autoregressive generation (hyper.ai digest, Method: one 256-token
    canvas at a time; stage 3 of the three-stage pipeline re-encodes each
    finished canvas causally and appends it to the cache).  Block j draws its
    Philox words at positions offset by j x C.  Returns the blocks [B][n_blocks*C]
    and the final cache.  routing: optional list receiving each causal pass's
    per-layer top-k ids (the prompt pass, then each append)."""
    wl = W.wl
    import synth
    p_routing = [] if routing is not None else None
    cache = decoder.prefill(W, synth.prompt_tokens(wl) if prompt is None else prompt, routing=p_routing)
    if routing is not None:
        routing.append(p_routing)
    out = []
    for j in range(n_blocks):
        tok, _, _ = generate_block(W, T, seed, cache=cache, pos_offset=j * wl.canvas)
        out.append(tok)
        if j + 1 < n_blocks:
            a_routing = [] if routing is not None else None
            cache = decoder.prefill(W, tok, routing=a_routing, prefix=cache)
            if routing is not None:
                routing.append(a_routing)
    return np.concatenate(out, axis=1), cache
