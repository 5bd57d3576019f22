"""Full-scale model parity, single canvas (the full-scale workload's model: 30
layers, d 2816, 16/8 heads x 256, 128 experts top-8 of width 704, shared FFN
2112, V 262144).

* The whole 30-layer step against the oracle, with the oracle's routing forced
  (every row) and with the device's own routing (flips at near-ties counted).
  The oracle regenerates the 25 B weights for each pass, so the prompt is kept
  at 256 tokens there (the oracle's prompt pass is its most expensive part).
* At the benchmarked shape (P = 2048, the same attention split count as the
  bench, V = 262144) with the model cut to two layers: the attention output
  against the softmax formula, and the production sampler's inputs (the LM-head
  epilogue's statistics) against the oracle's row statistics of the same logits.
* A whole block at the full sizes: determinism and the block invariants.
"""
import numpy as np
import pytest

import synth
from oracle import decoder, sampler as osamp
from tests.helpers import (make_denoiser, load_prompt_cache, rel_l2, gpu_step, gpu_step_forced, routing_flips,
                           oracle_prompt_routing)
from tests.test_gpu_step import attention_vs_formula
from tests.helpers import end_to_end_bar, flip_margin_bar

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def full30():
    """The 30-layer full-scale model (prompt capacity 2048); each test runs its own prompt pass."""
    wl = synth.WORKLOADS["full"]
    den = make_denoiser(wl)
    yield wl, den
    den.close()


def test_full_model_step_matches_oracle(full30):
    """Forced: the device is given the oracle's routing for the prompt pass and
    the step (the gates still come from its own router logits), so every row's
    arithmetic is compared: logits relative L2 <= 1e-2 over all rows.  Own
    routing: over 30 layers the flips at near-ties reach most rows through
    attention, so this checks that each flip starts at an oracle margin below the
    fixed bar (tests.helpers.flip_margin_bar) and that the rows without a flip match."""
    wl = synth.WORKLOADS["full"].replace(prompt_len=256)
    den = full30[1]
    B, C, V = wl.batch, wl.canvas, wl.vocab
    tok = osamp.init_canvas(wl.seed, B, C, V)
    W = decoder.Weights(wl)
    cache, p_ids = oracle_prompt_routing(W, synth.prompt_tokens(wl))
    ref, diag = decoder.decoder_logits(W, tok, cache)
    ref = ref.reshape(B * C, V)
    del W, cache

    from synth.device import device_prompt
    load_prompt_cache(den, wl)
    got, ids, rl = gpu_step(den, wl, tok, 0)
    usage = den.expert_usage()
    flipped, first, dr_max = routing_flips(ids, rl, diag)
    keep = ~flipped
    err_unforced = rel_l2(got[keep], ref[keep]) if keep.any() else 0.0
    oracle_used = [len(np.unique(diag["ids"][l])) for l in range(wl.n_layers)]

    den.force_routing(torch.from_numpy(p_ids.reshape(-1)).cuda(), None)
    den.prefill_prompt(device_prompt(wl))
    den.synchronize()
    c_ids = np.stack(diag["ids"]).astype(np.int32)
    forced, f_ids, f_rl = gpu_step_forced(den, wl, tok, 0, c_ids)
    den.force_routing(None, None)
    err_forced = rel_l2(forced, ref)
    err_forced_rows = np.linalg.norm(forced - ref, axis=1) / np.linalg.norm(ref, axis=1)
    margins = [m for _, _, m in first]
    print(f"full model (P=256): forced routing: rel-L2 {err_forced:.2e} over all {B * C} rows (worst row "
          f"{err_forced_rows.max():.2e}); own routing: flips in {flipped.sum()}/{C} rows, first-flip margins max "
          f"{max(margins) if margins else 0:.1e}, rel-L2 {err_unforced:.2e} on {keep.sum()} unflipped rows; experts "
          f"routed to: device {usage[:5]}.. oracle {oracle_used[:5]}..")
    assert np.isfinite(got).all() and np.isfinite(forced).all()
    assert np.array_equal(np.sort(f_ids, axis=2), np.sort(c_ids, axis=2))
    assert err_forced <= end_to_end_bar("full")
    assert err_unforced <= end_to_end_bar("full")
    assert all(m < flip_margin_bar("full") for m in margins), first


def test_full_model_each_layer_matches_the_oracle(full30):
    """Layer-wise teacher forcing at the benchmarked sizes (P = 2048, all 30
    layers, V = 262144): each layer's update of the residual stream and the
    logits, computed by the oracle from the device's own input to that layer,
    agree with the device's to relative L2 <= 1e-2."""
    from tests.helpers import layerwise_parity
    wl, den = full30
    load_prompt_cache(den, wl)
    tok = osamp.init_canvas(wl.seed, wl.batch, wl.canvas, wl.vocab)
    upd, full, err_logits = layerwise_parity(den, wl, tok, 0)
    print(f"full (P=2048) layer-wise: update rel-L2 max {max(upd):.2e} (per layer "
          f"{[f'{e:.1e}' for e in upd]}), residual max {max(full):.2e}, logits {err_logits:.2e}")
    assert max(upd) <= 1e-2 and err_logits <= 1e-2


@pytest.fixture(scope="module")
def full2():
    """The full-scale shapes at the benchmarked prompt length (P = 2048), model cut to 2 layers."""
    wl = synth.WORKLOADS["full"].replace(n_layers=2)
    den = make_denoiser(wl)
    load_prompt_cache(den, wl)
    den.synchronize()
    yield wl, den
    den.close()


def test_full_shape_attention_matches_the_formula(full2):
    """hd 256, GQA 16/8, 2048 prompt keys + 256 canvas keys, the automatic key
    split count of the bench (tcgen05 kernel)."""
    wl, den = full2
    tok = osamp.init_canvas(wl.seed, wl.batch, wl.canvas, wl.vocab)
    attention_vs_formula(den, wl, tok, 0, 0, "full (P=2048)")


def sampler_inputs_vs_oracle(den, wl, s, T, label):
    """After a step that also stores its fp32 logits: the production sampler's
    confidence (within 1e-5) and argmax (exact), read from the LM-head epilogue's
    statistics, against the oracle's row statistics of those logits; commit sets
    and tokens against the oracle sampler on them (differences only at a
    confidence margin below 1e-3); and the entropy the epilogue's statistics give
    against the oracle's (relative 1e-4)."""
    from oracle import eb_sampler as eb
    B, C, V = wl.batch, wl.canvas, wl.vocab
    seed = 1234 + s
    tok = osamp.init_canvas(seed, B, C, V)
    committed = np.zeros((B, C), dtype=bool)
    committed[:, 1::5] = True
    den.set_canvas(torch.from_numpy(tok.reshape(-1).astype(np.int32)).cuda(),
                   torch.from_numpy(committed.reshape(-1).astype(np.uint8)).cuda())
    logits = torch.empty(B * C * V, dtype=torch.float32, device="cuda")
    den.denoise_step(s, T, logits)
    conf = torch.empty(B * C, dtype=torch.float32, device="cuda")
    den.sample_commit(s, T, seed, conf)
    amax = torch.empty(B * C, dtype=torch.int32, device="cuda")
    den.debug_read(6, 0, amax)
    t = torch.empty(B * C, dtype=torch.int32, device="cuda")
    c = torch.empty(B * C, dtype=torch.uint8, device="cuda")
    den.get_canvas(t, c)
    den.synchronize()
    L = logits.cpu().numpy().reshape(B, C, V).astype(np.float64)
    del logits
    tau = osamp.tau_of_step(s, T, wl.tau_max, wl.tau_min)
    arg, ref_conf = osamp.row_stats(L, tau)
    rt, rc, info = osamp.sample_commit(L, tok, committed, s, T, seed, tau)
    got_conf = conf.cpu().numpy().reshape(B, C)
    dconf = float(np.max(np.abs(got_conf - ref_conf)))
    assert dconf < 1e-5
    assert np.array_equal(amax.cpu().numpy().reshape(B, C), arg)
    t, c = t.cpu().numpy().reshape(B, C), c.cpu().numpy().reshape(B, C).astype(bool)
    near = 0
    for b in range(B):
        if np.array_equal(c[b], rc[b]):
            assert np.array_equal(t[b], rt[b])
        else:
            assert info["margin"][b] < 1e-3, (b, info["margin"][b])
            near += 1
    # the entropy-bounded sampler's statistics from the same epilogue (no stored logits)
    H_ref, _ = eb.entropy_rows(L, tau)
    ent = torch.empty(B * C, dtype=torch.float32, device="cuda")
    den.set_canvas(torch.from_numpy(tok.reshape(-1).astype(np.int32)).cuda(), None)
    den.sample_commit_eb(None, s, T, seed, 0.0, 0.0, ent)
    den.synchronize()
    H = ent.cpu().numpy().reshape(B, C)
    dH = float(np.max(np.abs(H - H_ref) / np.maximum(1.0, H_ref)))
    print(f"{label} s={s} T={T}: max |conf diff| {dconf:.1e}, argmax exact, near-tie commit differences "
          f"{near}/{B}; entropy max rel diff {dH:.1e} (mean entropy {H_ref.mean():.3f} nats)")
    assert dH < 1e-4


@pytest.mark.parametrize("s,T", [(0, 12), (11, 12)])
def test_full_shape_sampler_inputs_match_oracle(full2, s, T):
    wl, den = full2
    sampler_inputs_vs_oracle(den, wl, s, T, "full (V=262144, N=256)")


@pytest.mark.parametrize("T", [12])
def test_full_size_block_properties(full30, T):
    """At the full single-canvas sizes: a whole block (prompt pass, T steps) is
    deterministic, every position is committed after T steps, committed tokens
    never change, logits are finite."""
    block_properties(synth.WORKLOADS["full"].replace(steps=T), T, full30[1])


def block_properties(wl, T, den=None):
    own = den is None
    if own:
        den = make_denoiser(wl)
    from synth.device import device_prompt
    prompt = device_prompt(wl)
    B, C = wl.batch, wl.canvas
    outs = []
    for rep in range(2):
        den.prefill_prompt(prompt)
        den.init_canvas(wl.seed)
        prev_t = prev_c = None
        t = torch.empty(B * C, dtype=torch.int32, device="cuda")
        c = torch.empty(B * C, dtype=torch.uint8, device="cuda")
        for s in range(T):
            logits = torch.empty(B * C * wl.vocab, dtype=torch.float32, device="cuda") if s == 0 else None
            den.denoise_step(s, T, logits)
            if logits is not None:
                den.synchronize()
                assert bool(torch.isfinite(logits).all())
                del logits
            den.sample_commit(s, T, wl.seed)
            den.get_canvas(t, c)
            den.synchronize()
            tt, ccm = t.cpu().numpy(), c.cpu().numpy().astype(bool)
            if prev_c is not None:
                assert np.array_equal(tt[prev_c], prev_t[prev_c]) and ccm[prev_c].all()
                newly = ccm.reshape(B, C).sum(axis=1) - prev_c.reshape(B, C).sum(axis=1)
                m = -(-C // T)
                expect = np.minimum(m, C - prev_c.reshape(B, C).sum(axis=1)) if s < T - 1 else \
                    C - prev_c.reshape(B, C).sum(axis=1)
                assert np.array_equal(newly, expect)
            prev_t, prev_c = tt, ccm
        assert prev_c.all()
        outs.append(prev_t)
    assert np.array_equal(outs[0], outs[1])
    if own:
        den.close()
