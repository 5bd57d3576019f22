"""Pins of the fp64 oracle to things other than itself (no GPU).

Each test checks one oracle function against what the pages or mathematics fix:
published known-answer vectors, closed forms, library routines that implement
the same textbook operation independently, invariants and brute force.
"""
import math
import os

import numpy as np
import pytest
import scipy.special
import scipy.stats
import torch

import synth
from oracle import decoder, numerics, philox, pipeline, sampler

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------- Philox4x32-10

def test_philox_known_answer_vectors():
    """Random123 known-answer vectors of Philox4x32-10 (SC'11 reference implementation)."""
    rows = [l.split() for l in open(os.path.join(GOLDEN, "philox4x32_10_kat.txt")) if l.strip() and l[0] != "#"]
    assert len(rows) == 3
    for r in rows:
        v = [int(x, 16) for x in r]
        out = philox.philox4x32_10(np.array(v[0:4]), np.array(v[4:6]))
        assert [int(x) for x in out] == v[6:10]


def test_philox_broadcast_matches_scalar():
    seed = 0x123456789ABCDEF
    w = philox.draw(seed, np.arange(5), 3, 2, 1)
    for i in range(5):
        one = philox.philox4x32_10(np.array([i, 3, 2, 1]), np.array([seed & 0xFFFFFFFF, seed >> 32]))
        assert np.array_equal(w[i], one)


def test_uniform_index_is_a_shift_for_power_of_two_vocab():
    w = synth.words(7, 1, 0, 10000).astype(np.uint64) & np.uint64(0xFFFFFFFF)
    for V in (4096, 32768, 262144):
        assert np.array_equal(philox.uniform_index(w, V), (w >> np.uint64(32 - int(math.log2(V)))).astype(np.int64))
    assert philox.uniform_index(np.array([0xFFFFFFFF]), 10)[0] == 9
    assert philox.uniform_index(np.array([0]), 10)[0] == 0


# ----------------------------------------------------------------- forward process (eq. 1)

@pytest.mark.parametrize("kap", [0.0, 0.25, 0.5, 0.9, 1.0])
def test_forward_marginal_monte_carlo(kap):
    """P(x_t = x0) = kappa + (1 - kappa)/V, 10^6 draws, within 5 sigma."""
    V, B, C = 4096, 1000, 1000
    x0 = synth.uniform_i32(11, 99, 0, B * C, V).reshape(B, C)
    xt = sampler.forward_noise_tokens(x0, kap, seed=5, V=V)
    p = kap + (1 - kap) / V
    hits = int(np.sum(xt == x0))
    n = B * C
    if kap == 1.0:
        assert hits == n
        return
    sigma = math.sqrt(n * p * (1 - p))
    assert abs(hits - n * p) < 5 * sigma, (hits, n * p, sigma)


def test_forward_process_at_kappa_zero_is_uniform():
    V, B, C = 4096, 1000, 1000
    x0 = np.zeros((B, C), dtype=np.int64)
    xt = sampler.forward_noise_tokens(x0, 0.0, seed=9, V=V)
    counts = np.bincount(xt.reshape(-1), minlength=V)
    chi2 = float(np.sum((counts - B * C / V) ** 2 / (B * C / V)))
    dof = V - 1
    assert abs(chi2 - dof) < 5 * math.sqrt(2 * dof)


def test_forward_process_factorises_over_positions():
    """Keep/replace indicators of two positions are independent (chi-square, 2x2)."""
    V, B, C = 64, 20000, 8
    x0 = np.zeros((B, C), dtype=np.int64)
    xt = sampler.forward_noise_tokens(x0, 0.5, seed=3, V=V)
    same = xt == x0
    for i, j in [(0, 1), (2, 7), (3, 4)]:
        table = np.array([[np.sum(same[:, i] & same[:, j]), np.sum(same[:, i] & ~same[:, j])],
                          [np.sum(~same[:, i] & same[:, j]), np.sum(~same[:, i] & ~same[:, j])]])
        _, pval, _, _ = scipy.stats.chi2_contingency(table)
        assert pval > 1e-6


def test_schedule_endpoints():
    assert sampler.kappa(0.0) == 1.0 and sampler.kappa(1.0) == 0.0
    T = 12
    assert sampler.tau_of_step(0, T) == pytest.approx(0.8)
    assert sampler.tau_of_step(T - 1, T) == pytest.approx(0.4 + 0.4 / T)
    taus = [sampler.tau_of_step(s, T) for s in range(T)]
    assert np.allclose(np.diff(taus), -0.4 / T)


# ----------------------------------------------------------------- numerics

def test_bf16_round_matches_torch_on_float32_inputs():
    x = synth.normal_f32(1, 2, 0, 200000, 3.0).astype(np.float64)
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(numerics.bf16_round(x), ref)


def test_bf16_round_ties_to_even():
    assert numerics.bf16_round(1 + 2 ** -8) == 1.0
    assert numerics.bf16_round(1 + 3 * 2 ** -8) == 1 + 2 ** -6
    assert numerics.bf16_round(-(1 + 2 ** -8 + 2 ** -30)) == -(1 + 2 ** -7)


def test_rmsnorm_matches_torch_and_constant_vector():
    x = np.random.default_rng(0).normal(size=(5, 64)) * 3
    g = np.random.default_rng(1).normal(size=64) * 0.1
    ref = torch.nn.functional.rms_norm(torch.from_numpy(x), (64,), torch.from_numpy(1 + g), eps=1e-6).numpy()
    assert np.allclose(numerics.rmsnorm(x, g, 1e-6), ref, rtol=1e-12, atol=1e-12)
    c = np.full((1, 16), -2.5)
    assert np.allclose(numerics.rmsnorm(c, np.zeros(16), 0.0), -1.0)


def test_gelu_tanh_matches_torch_and_erf_form():
    x = np.linspace(-6, 6, 1001)
    ref = torch.nn.functional.gelu(torch.from_numpy(x), approximate="tanh").numpy()
    assert np.allclose(numerics.gelu_tanh(x), ref, rtol=1e-12, atol=1e-14)
    exact = 0.5 * x * (1 + scipy.special.erf(x / math.sqrt(2)))
    assert np.max(np.abs(numerics.gelu_tanh(x) - exact)) < 1e-3


def test_rope_is_complex_rotation_per_frequency():
    rng = np.random.default_rng(2)
    hd, base = 8, 10000.0
    x = rng.normal(size=(3, hd))
    pos = np.array([0, 5, 1234])
    y = numerics.rope(x, pos, base)
    for p_i, p in enumerate(pos):
        for j in range(hd // 2):
            z = complex(x[p_i, j], x[p_i, j + hd // 2]) * np.exp(1j * p * base ** (-2 * j / hd))
            assert y[p_i, j] == pytest.approx(z.real, abs=1e-12)
            assert y[p_i, j + hd // 2] == pytest.approx(z.imag, abs=1e-12)
    assert np.allclose(y[0], x[0])


def test_rope_matches_transformers_rotate_half():
    from transformers.models.llama.modeling_llama import apply_rotary_pos_emb
    rng = np.random.default_rng(3)
    hd, base, n = 16, 10000.0, 7
    q = rng.normal(size=(1, 2, n, hd))
    k = rng.normal(size=(1, 2, n, hd))
    pos = np.arange(100, 100 + n)
    ang = pos[:, None] * base ** (-np.arange(0, hd, 2) / hd)[None, :]
    emb = np.concatenate([ang, ang], axis=-1)
    cos = torch.from_numpy(np.cos(emb))[None]
    sin = torch.from_numpy(np.sin(emb))[None]
    rq, rk = apply_rotary_pos_emb(torch.from_numpy(q), torch.from_numpy(k), cos, sin)
    assert np.allclose(numerics.rope(q, pos, base), rq.numpy(), atol=1e-12)
    assert np.allclose(numerics.rope(k, pos, base), rk.numpy(), atol=1e-12)


def test_rope_scores_depend_only_on_relative_position():
    rng = np.random.default_rng(4)
    q, k = rng.normal(size=(1, 32)), rng.normal(size=(1, 32))
    s1 = numerics.rope(q, np.array([10]), 1e4) @ numerics.rope(k, np.array([3]), 1e4).T
    s2 = numerics.rope(q, np.array([1007]), 1e4) @ numerics.rope(k, np.array([1000]), 1e4).T
    assert s1 == pytest.approx(s2, rel=1e-9)


# ----------------------------------------------------------------- attention

def _sdpa_ref(q, k, v, causal):
    Hq, Hkv = q.shape[1], k.shape[1]
    rep = Hq // Hkv
    kk = torch.from_numpy(k).repeat_interleave(rep, dim=1)
    vv = torch.from_numpy(v).repeat_interleave(rep, dim=1)
    return torch.nn.functional.scaled_dot_product_attention(torch.from_numpy(q), kk, vv, is_causal=causal).numpy()


@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (4, 2), (4, 1)])
def test_attention_matches_torch_sdpa(Hq, Hkv):
    rng = np.random.default_rng(5)
    q = rng.normal(size=(2, Hq, 9, 8))
    k = rng.normal(size=(2, Hkv, 13, 8))
    v = rng.normal(size=(2, Hkv, 13, 8))
    assert np.allclose(decoder.attention(q, k, v), _sdpa_ref(q, k, v, False), atol=1e-12)
    k2, v2 = k[:, :, :9], v[:, :, :9]
    assert np.allclose(decoder.attention(q, k2, v2, causal_offset=0), _sdpa_ref(q, k2, v2, True), atol=1e-12)


def test_attention_two_key_closed_form():
    """hd = 1: weights of two keys are sigmoid((b1 - b2) a)."""
    a, b1, b2, v1, v2 = 1.7, 0.3, -1.1, 2.0, -5.0
    q = np.array([[[[a]]]])
    k = np.array([[[[b1], [b2]]]])
    v = np.array([[[[v1], [v2]]]])
    p1 = 1 / (1 + math.exp(-(b1 - b2) * a))
    assert decoder.attention(q, k, v)[0, 0, 0, 0] == pytest.approx(p1 * v1 + (1 - p1) * v2, rel=1e-12)


def test_canvas_attention_is_non_causal_and_permutation_invariant():
    rng = np.random.default_rng(6)
    P, C, hd = 3, 5, 4
    q = rng.normal(size=(1, 2, C, hd))
    k = rng.normal(size=(1, 2, P + C, hd))
    v = rng.normal(size=(1, 2, P + C, hd))
    base = decoder.attention(q, k, v)
    k2 = k.copy()
    k2[0, :, P + C - 1] += 1.0          # a LATER canvas key changes an EARLIER canvas row
    assert not np.allclose(decoder.attention(q, k2, v)[0, :, 0], base[0, :, 0])
    perm = np.r_[np.arange(P), P + rng.permutation(C)]
    assert np.allclose(decoder.attention(q, k[:, :, perm], v[:, :, perm]), base, atol=1e-12)


# ----------------------------------------------------------------- MoE

def _tiny_moe_workload(E, k):
    return synth.WORKLOADS["tiny"].replace(n_layers=1, d_model=32, n_experts=E, top_k=k, expert_width=16,
                                           shared_width=0)


def _moe_arrays(wl, seed):
    rng = np.random.default_rng(seed)
    d, E, w = wl.d_model, wl.n_experts, wl.expert_width
    return {("w_router", 0): rng.normal(size=(E, d)), ("w_gate_up", 0): rng.normal(size=(E, 2 * w, d)) * 0.3,
            ("w_down", 0): rng.normal(size=(E, d, w)) * 0.3}


@pytest.mark.parametrize("E,k", [(8, 2), (8, 8), (4, 1)])
def test_routed_moe_equals_dense_masked_evaluation(E, k):
    wl = _tiny_moe_workload(E, k)
    W = decoder.Weights(wl, _moe_arrays(wl, E * 10 + k))
    x = np.random.default_rng(7).normal(size=(40, wl.d_model))
    with numerics.pure_fp64():
        y, info = decoder.moe(x, W, 0)
        r = x @ W.get("w_router", 0).T
        dense = np.stack([decoder.expert_ffn(x, W.get("w_gate_up", 0, e), W.get("w_down", 0, e))
                          for e in range(E)], axis=1)                                 # [n][E][d]
    # gates from scratch: the k largest logits by value, softmax over them
    mask = np.zeros_like(r)
    for t in range(r.shape[0]):
        top = np.argsort(-r[t], kind="stable")[:k]
        mask[t, top] = scipy.special.softmax(r[t, top])
    assert np.allclose(y, np.einsum("te,ted->td", mask, dense), atol=1e-10)
    if k == E:   # fully dense soft mixture
        assert np.allclose(y, np.einsum("te,ted->td", scipy.special.softmax(r, axis=1), dense), atol=1e-10)


def test_router_ties_go_to_lower_expert_id():
    r_w = np.zeros((6, 4))
    r_w[5] = 1.0          # expert 5 strictly best; experts 0..4 tie at zero
    _, ids, gates, margin = decoder.route(np.ones((1, 4)), r_w, 3)
    assert list(ids[0]) == [5, 0, 1]
    assert margin[0] == 0.0


# ----------------------------------------------------------------- sampler

def test_confidence_closed_forms():
    V = 4096
    arg, conf = sampler.row_stats(np.zeros((1, V)), 0.7)
    assert conf[0] == pytest.approx(-math.log(V)) and arg[0] == 0
    one_hot = np.zeros((1, V))
    one_hot[0, 17] = 1e4
    arg, conf = sampler.row_stats(one_hot, 0.5)
    assert arg[0] == 17 and conf[0] == pytest.approx(0.0, abs=1e-300)
    two = np.array([[0.0, 1.0, 1.0]])
    arg, conf = sampler.row_stats(two, 1.0)
    assert arg[0] == 1 and conf[0] == pytest.approx(math.log(math.e / (1 + 2 * math.e)))


@pytest.mark.parametrize("T", [4, 12, 32])
def test_one_hot_logits_recover_target_and_invariants(T):
    B, C, V, seed = 2, 256, 4096, 77
    target = synth.uniform_i32(1, 5, 0, B * C, V).reshape(B, C)
    tok = sampler.init_canvas(seed, B, C, V)
    committed = np.zeros((B, C), dtype=bool)
    rng = np.random.default_rng(T)
    m = math.ceil(C / T)
    for s in range(T):
        # one-hot at the target with a position-dependent height: distinct confidences
        logits = np.zeros((B, C, V))
        heights = rng.uniform(1.0, 20.0, size=(B, C))
        np.put_along_axis(logits, target[..., None], heights[..., None], axis=2)
        before_tok, before_c = tok.copy(), committed.copy()
        tok, committed, info = sampler.sample_commit(logits, tok, committed, s, T, seed, sampler.tau_of_step(s, T))
        assert np.array_equal(tok[before_c], before_tok[before_c])          # frozen
        assert np.all(committed[before_c])
        newly = committed & ~before_c
        expect = min(m, C - before_c[0].sum()) if s < T - 1 else C - before_c[0].sum()
        assert np.all(newly.sum(axis=1) == expect)
        # committed ones are the highest-height (highest-confidence) open positions
        for b in range(B):
            open_h = heights[b][~before_c[b]]
            if newly[b].any() and (~newly[b] & ~before_c[b]).any():
                assert heights[b][newly[b]].min() >= heights[b][~newly[b] & ~before_c[b]].max()
    assert committed.all()
    assert np.array_equal(tok, target)


def test_renoise_draws_are_the_philox_stream():
    B, C, V, seed, s, T = 1, 16, 4096, 5, 0, 4
    tok = np.zeros((B, C), dtype=np.int64)
    committed = np.zeros((B, C), dtype=bool)
    logits = np.zeros((B, C, V))
    logits[0, :, 3] = np.arange(C)     # confidence increases with position
    new_tok, new_c, info = sampler.sample_commit(logits, tok, committed, s, T, seed, 0.8)
    assert list(np.nonzero(new_c[0])[0]) == list(range(C - 4, C))
    rest = np.arange(C - 4)
    w = [int(philox.philox4x32_10(np.array([i, s, 0, 1]), np.array([seed, 0]))[0]) for i in rest]
    assert list(new_tok[0, rest]) == [(x * V) >> 32 for x in w]
    assert np.all(new_tok[0, C - 4:] == 3)


def test_confidence_ties_commit_lower_position_first():
    B, C, V = 1, 8, 32
    logits = np.zeros((B, C, V))
    logits[0, :, 1] = 5.0                       # all rows identical -> equal confidence
    _, committed, _ = sampler.sample_commit(logits, np.zeros((B, C), int), np.zeros((B, C), bool), 0, 4, 1, 0.8)
    assert list(np.nonzero(committed[0])[0]) == [0, 1]


# ----------------------------------------------------------------- decoder composition

def _hf_gemma_logits(wl, arrays, prompt, canvas):
    """Same model as a one-expert special case, run by transformers' Gemma layers
    over [prompt ; canvas] with a mask that is causal on prompt rows and full on
    canvas rows (prompt rows never see the canvas)."""
    from transformers.models.gemma import modeling_gemma as mg
    cfg = mg.GemmaConfig(vocab_size=wl.vocab, hidden_size=wl.d_model, intermediate_size=wl.expert_width,
                         num_hidden_layers=wl.n_layers, num_attention_heads=wl.n_q_heads,
                         num_key_value_heads=wl.n_kv_heads, head_dim=wl.head_dim, rms_norm_eps=wl.rms_eps,
                         rope_theta=wl.rope_base, hidden_act="gelu_pytorch_tanh", attention_bias=False,
                         attention_dropout=0.0)
    cfg._attn_implementation = "eager"
    model = mg.GemmaModel(cfg).double().eval()
    Hq, Hkv, hd, w = wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.expert_width
    with torch.no_grad():
        for l, layer in enumerate(model.layers):
            qkv = torch.from_numpy(arrays[("w_qkv", l)])
            layer.self_attn.q_proj.weight.copy_(qkv[:Hq * hd])
            layer.self_attn.k_proj.weight.copy_(qkv[Hq * hd:(Hq + Hkv) * hd])
            layer.self_attn.v_proj.weight.copy_(qkv[(Hq + Hkv) * hd:])
            layer.self_attn.o_proj.weight.copy_(torch.from_numpy(arrays[("w_o", l)]))
            layer.input_layernorm.weight.copy_(torch.from_numpy(arrays[("attn_norm", l)]))
            layer.post_attention_layernorm.weight.copy_(torch.from_numpy(arrays[("ffn_norm", l)]))
            g_rows, u_rows = decoder.split_gate_up(arrays[("w_gate_up", l)][0])
            layer.mlp.gate_proj.weight.copy_(torch.from_numpy(g_rows))
            layer.mlp.up_proj.weight.copy_(torch.from_numpy(u_rows))
            layer.mlp.down_proj.weight.copy_(torch.from_numpy(arrays[("w_down", l)][0]))
        model.norm.weight.copy_(torch.from_numpy(arrays[("final_norm", None)]))
        E = torch.from_numpy(arrays[("embed", None)])
        seq = np.concatenate([prompt, canvas], axis=1)
        B, S = seq.shape
        P = prompt.shape[1]
        allow = np.tril(np.ones((S, S), dtype=bool))
        allow[P:, :] = True
        mask = torch.from_numpy(np.where(allow, 0.0, -np.inf))[None, None].expand(B, 1, S, S)
        pos = torch.arange(S)[None]
        h = E[torch.from_numpy(seq)]
        pe = model.rotary_emb(h, position_ids=pos)
        for layer in model.layers:
            h = layer(h, attention_mask=mask, position_ids=pos, position_embeddings=pe)
        h = model.norm(h)
        return (h[:, P:] @ E.T).numpy()


def test_gate_up_storage_interleaves_blocks_of_16():
    w, d = 64, 3
    stored = np.arange(2 * w * d, dtype=np.float64).reshape(2 * w, d)
    g, u = decoder.split_gate_up(stored)
    assert np.array_equal(g[0:16], stored[0:16]) and np.array_equal(u[0:16], stored[16:32])
    assert np.array_equal(g[16:32], stored[32:48]) and np.array_equal(u[48:64], stored[112:128])


def _one_expert_arrays(wl, seed):
    rng = np.random.default_rng(seed)
    d, w = wl.d_model, wl.expert_width
    a = {("embed", None): rng.normal(size=(wl.vocab, d)), ("final_norm", None): rng.normal(size=d) * 0.2}
    for l in range(wl.n_layers):
        a[("attn_norm", l)] = rng.normal(size=d) * 0.2
        a[("ffn_norm", l)] = rng.normal(size=d) * 0.2
        a[("w_qkv", l)] = rng.normal(size=(wl.qkv_rows, d)) * 0.3
        a[("w_o", l)] = rng.normal(size=(d, wl.n_q_heads * wl.head_dim)) * 0.2
        a[("w_router", l)] = rng.normal(size=(1, d))
        a[("w_gate_up", l)] = rng.normal(size=(1, 2 * w, d)) * 0.2
        a[("w_down", l)] = rng.normal(size=(1, d, w)) * 0.2
    return a


def test_decoder_matches_transformers_gemma_one_expert_special_case():
    """Prompt pass + canvas pass == one Gemma forward over [prompt ; canvas] with the
    prompt causal and the canvas bidirectional; E = 1, k = 1 makes the MoE a plain
    gated-GELU MLP.  Pins norm placement, residuals, RoPE positions (canvas at
    P + i), the GQA head map, the one joint softmax and the tied LM head."""
    wl = synth.WORKLOADS["tiny"].replace(n_layers=2, d_model=32, n_q_heads=4, n_kv_heads=2, head_dim=8,
                                         n_experts=1, top_k=1, expert_width=32, vocab=50, batch=2,
                                         prompt_len=6, canvas=5)
    arrays = _one_expert_arrays(wl, 8)
    rng = np.random.default_rng(9)
    prompt = rng.integers(0, wl.vocab, size=(wl.batch, wl.prompt_len))
    canvas = rng.integers(0, wl.vocab, size=(wl.batch, wl.canvas))
    W = decoder.Weights(wl, arrays)
    with numerics.pure_fp64():
        cache = decoder.prefill(W, prompt)
        logits, _ = decoder.decoder_logits(W, canvas, cache)
    ref = _hf_gemma_logits(wl, arrays, prompt, canvas)
    # transformers' Gemma RMSNorm computes in fp32, hence the tolerance
    assert np.allclose(logits, ref, rtol=1e-4, atol=1e-4 * np.abs(ref).max())


def test_prefill_is_causal_and_canvas_pass_is_not():
    wl = synth.WORKLOADS["tiny"].replace(n_layers=2, d_model=32, n_q_heads=2, n_kv_heads=2, head_dim=8,
                                         n_experts=1, top_k=1, expert_width=32, vocab=50, batch=1,
                                         prompt_len=6, canvas=5)
    W = decoder.Weights(wl, _one_expert_arrays(wl, 10))
    prompt = np.array([[1, 2, 3, 4, 5, 6]])
    p2 = prompt.copy()
    p2[0, -1] = 7
    c1, c2 = decoder.prefill(W, prompt), decoder.prefill(W, p2)
    for (k1, v1), (k2, v2) in zip(c1, c2):
        assert np.array_equal(k1[:, :, :-1], k2[:, :, :-1]) and np.array_equal(v1[:, :, :-1], v2[:, :, :-1])
    canvas = np.array([[9, 8, 7, 6, 5]])
    cv2 = canvas.copy()
    cv2[0, -1] = 0
    l1, _ = decoder.decoder_logits(W, canvas, c1)
    l2, _ = decoder.decoder_logits(W, cv2, c1)
    assert not np.allclose(l1[0, 0], l2[0, 0])


def test_oracle_step_on_tiny_workload_runs_and_is_deterministic():
    wl = synth.WORKLOADS["tiny"].replace(n_layers=1, canvas=32, prompt_len=16)
    W = decoder.Weights(wl)
    cache = pipeline.prompt_cache(W)
    tok = sampler.init_canvas(wl.seed, wl.batch, wl.canvas, wl.vocab)
    committed = np.zeros_like(tok, dtype=bool)
    a = pipeline.denoise_step(W, cache, tok, committed, 0, 4, wl.seed)
    b = pipeline.denoise_step(W, cache, tok, committed, 0, 4, wl.seed)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    assert a[2].sum() == 8


def test_shared_ffn_equals_the_sum_of_its_feature_slices():
    """The device runs the shared FFN as ceil(ws / w) pseudo-experts, feature
    slices J_j of width w (the last one ragged is padded with zero rows), whose
    down outputs are summed.  The gated FFN is a sum over its hidden features,
    so W_d (GELU(W_g x) * W_u x) = sum_j W_d[:, J_j] (GELU(W_g[J_j] x) * W_u[J_j] x)
    holds exactly up to the order of the sums, here checked in fp64 (with the
    bf16 rounding of the activation, which is per feature, on both sides)."""
    from oracle import decoder
    rng = np.random.default_rng(8)
    d, ws, w, n = 64, 96, 32, 7                       # three slices of 32 features
    x = rng.normal(size=(n, d))
    w_g, w_u = rng.normal(size=(ws, d)) * 0.2, rng.normal(size=(ws, d)) * 0.2
    w_d = rng.normal(size=(d, ws)) * 0.2

    def interleave(g, u):   # the stored [2 ws][d] layout: 16 gate rows, then the 16 matching up rows
        blocks = np.stack([g.reshape(-1, 16, d), u.reshape(-1, 16, d)], axis=1)
        return blocks.reshape(-1, d)

    whole = decoder.expert_ffn(x, interleave(w_g, w_u), w_d)
    parts = sum(decoder.expert_ffn(x, interleave(w_g[j:j + w], w_u[j:j + w]), w_d[:, j:j + w])
                for j in range(0, ws, w))
    assert np.allclose(whole, parts, rtol=1e-12, atol=1e-12)


def test_appending_a_canvas_equals_one_causal_pass_over_the_concatenation():
    """Stage 3 of the pipeline (re-encode the finished canvas causally and append
    it to the cache): a causal pass over prompt + canvas in one go gives the same
    K / V at every position as the prompt pass followed by the append pass,
    because no position sees a later one.  A wrong RoPE position offset or a
    wrong causal offset in the append breaks the equality."""
    wl = synth.WORKLOADS["tiny"].replace(n_layers=3, d_model=64, n_q_heads=4, n_kv_heads=2, head_dim=16,
                                         n_experts=4, top_k=2, expert_width=64, vocab=97, batch=2,
                                         prompt_len=7, canvas=5)
    W = decoder.Weights(wl)
    rng = np.random.default_rng(21)
    prompt = rng.integers(0, wl.vocab, size=(2, 7))
    canvas = rng.integers(0, wl.vocab, size=(2, 5))
    whole = decoder.prefill(W, np.concatenate([prompt, canvas], axis=1))
    appended = decoder.prefill(W, canvas, prefix=decoder.prefill(W, prompt))
    for (k1, v1), (k2, v2) in zip(whole, appended):
        assert k1.shape == k2.shape == (2, 2, 12, 16)
        assert np.allclose(k1, k2, rtol=0, atol=1e-12) and np.allclose(v1, v2, rtol=0, atol=1e-12)
    shifted = decoder.prefill(W, canvas)            # the same tokens at positions 0.. instead of 7..
    assert not np.allclose(shifted[0][0], appended[0][0][:, :, 7:])


def test_later_blocks_draw_at_offset_positions():
    """Block j of a sequence draws its initial canvas at positions j*C + i: the
    same words as positions j*C.. of one long canvas, distinct from block 0."""
    B, C, V = 2, 16, 4096
    long = sampler.init_canvas(5, B, 3 * C, V)
    for j in range(3):
        assert np.array_equal(sampler.init_canvas(5, B, C, V, pos_offset=j * C), long[:, j * C:(j + 1) * C])
    assert not np.array_equal(long[:, :C], long[:, C:2 * C])


def test_forced_routing_with_the_oracle_s_own_choice_changes_nothing():
    """Teacher forcing of the routing with the ids the router itself picks gives
    the same layer output (gates from the same logits)."""
    wl = synth.WORKLOADS["tiny"].replace(n_layers=2, canvas=16, prompt_len=8)
    W = decoder.Weights(wl)
    cache = decoder.prefill(W, synth.prompt_tokens(wl))
    tok = sampler.init_canvas(1, wl.batch, wl.canvas, wl.vocab)
    ref, diag = decoder.decoder_logits(W, tok, cache)
    dp = decoder.DecoderPass(W, tok, cache, forced_ids=diag["ids"])
    for i in range(dp.n_pieces):
        dp.run_piece(i)
    assert np.array_equal(dp.logits, ref)
    other = [np.roll(ids, 1, axis=1) for ids in diag["ids"]]      # same sets, other slot order
    dp2 = decoder.DecoderPass(W, tok, cache, forced_ids=other)
    for i in range(dp2.n_pieces):
        dp2.run_piece(i)
    assert np.allclose(dp2.logits, ref, rtol=1e-12, atol=1e-12)
