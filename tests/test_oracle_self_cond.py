"""Pins of the self-conditioning path of the oracle (oracle/self_cond.py), no GPU."""
import numpy as np
import torch

import synth
from oracle import decoder, numerics, pipeline, sampler, self_cond

WL = synth.WORKLOADS["tiny"].replace(n_layers=2, canvas=16, prompt_len=8, self_cond_width=128)


def test_a_zero_state_is_the_plain_decoder():
    W = decoder.Weights(WL)
    cache = decoder.prefill(W, synth.prompt_tokens(WL))
    tok = sampler.init_canvas(3, WL.batch, WL.canvas, WL.vocab)
    a, _ = decoder.decoder_logits(W, tok, cache)
    b, _ = decoder.decoder_logits(W, tok, cache, z=np.zeros((WL.batch, WL.canvas, WL.d_model)))
    assert np.array_equal(a, b)
    c, _ = decoder.decoder_logits(W, tok, cache, z=np.full((WL.batch, WL.canvas, WL.d_model), 0.01))
    assert not np.allclose(a, c)


def test_one_hot_predictions_feed_back_the_predicted_embeddings():
    """Logits far apart: p0_hat is one-hot (exactly, after bf16 rounding), so
    p0_hat E is the embedding row of each position's argmax."""
    W = decoder.Weights(WL)
    rng = np.random.default_rng(1)
    target = rng.integers(0, WL.vocab, size=WL.canvas)
    L = np.full((WL.canvas, WL.vocab), -1e4)
    L[np.arange(WL.canvas), target] = 0.0
    u = self_cond.probs_times_embedding(W, L, tau=0.6)
    assert np.array_equal(u, W.embed_rows(target))


def test_uniform_predictions_feed_back_the_mean_embedding():
    """Equal logits: p0_hat = 1/V exactly (V a power of two), so p0_hat E is the
    mean embedding row."""
    W = decoder.Weights(WL)
    u = self_cond.probs_times_embedding(W, np.zeros((3, WL.vocab)), tau=0.8)
    E = W.embed_rows(np.arange(WL.vocab))
    assert np.allclose(u, np.broadcast_to(E.mean(axis=0), u.shape), rtol=1e-12, atol=1e-15)


def test_ffw_matches_a_torch_evaluation():
    """FFW = gated-GELU FFN of the bf16-rounded RMSNorm of its input, evaluated
    here with torch's rms_norm and tanh GELU in fp64 (gate/up rows interleaved in
    blocks of 16), with the same two bf16 roundings."""
    W = decoder.Weights(WL)
    u = np.random.default_rng(2).normal(0, 0.05, size=(5, WL.d_model))
    g = torch.from_numpy(W.get("sc_norm"))
    n = torch.nn.functional.rms_norm(torch.from_numpy(u), (WL.d_model,), eps=WL.rms_eps) * (1.0 + g)
    n = torch.from_numpy(numerics.bf16_round(n.numpy()))
    gu = torch.from_numpy(W.get("w_sc_gate_up")).reshape(-1, 2, 16, WL.d_model)
    wg, wu = gu[:, 0].reshape(-1, WL.d_model), gu[:, 1].reshape(-1, WL.d_model)
    a = torch.nn.functional.gelu(n @ wg.T, approximate="tanh") * (n @ wu.T)
    a = torch.from_numpy(numerics.bf16_round(a.numpy()))
    ref = (a @ torch.from_numpy(W.get("w_sc_down")).T).numpy()
    assert np.allclose(self_cond.ffw(W, u), ref, rtol=1e-10, atol=1e-13)


def test_a_block_threads_the_state_through_its_steps():
    """In a block the first step runs with z = 0 and every later step with the
    state its previous step produced."""
    W = decoder.Weights(WL)
    cache = decoder.prefill(W, synth.prompt_tokens(WL))
    T, seed = 3, 7
    tok, com, trace = pipeline.generate_block(W, T, seed, cache=cache)
    t = sampler.init_canvas(seed, WL.batch, WL.canvas, WL.vocab)
    c = np.zeros_like(t, dtype=bool)
    z = None
    for s in range(T):
        _, t, c, info = pipeline.denoise_step(W, cache, t, c, s, T, seed, z=z)
        assert np.array_equal(t, trace[s]["tok"])
        z = info["z_next"]
        assert z.shape == (WL.batch, WL.canvas, WL.d_model) and np.all(np.isfinite(z))
