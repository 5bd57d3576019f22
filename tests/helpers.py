"""Shared test plumbing: building a device model from a workload and comparing with the oracle."""
import math

import numpy as np

import synth


def rel_l2(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def make_denoiser(wl, prompt_max=None, device="cuda", weights=None):
    """A Denoiser of workload wl (weights: reuse the (embed, final_norm, layers)
    device tensors of another handle of the same model)."""
    import torch
    import block_denoising_step_b200 as dg
    from synth.device import device_weights, device_self_cond_weights, config_fields
    embed, final_norm, layers = weights if weights is not None else device_weights(wl, device)
    cfg = dg.ModelConfig(**config_fields(wl, prompt_max))
    stream = torch.cuda.current_stream().cuda_stream
    sc = device_self_cond_weights(wl, device) if wl.self_cond_width else None
    return dg.Denoiser(cfg, embed, final_norm, layers, stream=stream, self_cond=sc)


def oracle_prompt_routing(W, prompt):
    """(cache, forced prompt routing [L][B*P][k] int32) of the oracle's prompt pass;
    the last layer of a prompt pass has no MoE, its ids stay 0."""
    from oracle import decoder
    wl = W.wl
    routing = []
    cache = decoder.prefill(W, prompt, routing=routing)
    B, P = np.asarray(prompt).shape
    ids = np.zeros((wl.n_layers, B * P, wl.top_k), dtype=np.int32)
    for l, r in enumerate(routing):
        ids[l] = r
    return cache, ids


def load_prompt_cache(den, wl, device="cuda"):
    """Prompt pass on the device, or the workload's given cache."""
    from synth.device import device_prompt, device_prompt_kv
    if wl.prompt_kv_given:
        for l in range(wl.n_layers):
            k, v = device_prompt_kv(wl, l, device)
            den.set_prompt_kv(l, k, v, wl.prompt_len)
            den.synchronize()
    else:
        den.prefill_prompt(device_prompt(wl, device))


def commit_mismatch_allowed(oracle_info, b, tol=1e-3):
    """A commit-set difference in canvas b is allowed only at a confidence near-tie."""
    return oracle_info["margin"][b] < tol


def near_tie_rows(router_margins, tol=1e-3):
    """(b*C + i) rows whose routing had a near-tie (k-th vs (k+1)-th logit) in any layer."""
    m = np.min(np.stack(router_margins), axis=0)
    return m < tol


def gpu_step(den, wl, tok, s, committed=None):
    """One device step on a teacher-forced canvas with the routing captured.
    Returns (logits [B*C][V] float64, ids [L][B*C][k], router logits [L][B*C][E])."""
    import torch
    R, L, k, E, V = wl.batch * wl.canvas, wl.n_layers, wl.top_k, wl.n_experts, wl.vocab
    ids = torch.empty(L * R * k, dtype=torch.int32, device="cuda")
    rl = torch.empty(L * R * E, dtype=torch.float32, device="cuda")
    den.capture_routing(ids, rl)
    com = None if committed is None else torch.from_numpy(committed.reshape(-1).astype(np.uint8)).cuda()
    den.set_canvas(torch.from_numpy(np.asarray(tok).reshape(-1).astype(np.int32)).cuda(), com)
    logits = torch.empty(R * V, dtype=torch.float32, device="cuda")
    den.denoise_step(s, wl.steps, logits)
    den.synchronize()
    den.capture_routing(None, None)
    return (logits.cpu().numpy().reshape(R, V).astype(np.float64), ids.cpu().numpy().reshape(L, R, k),
            rl.cpu().numpy().reshape(L, R, E))


def gpu_step_forced(den, wl, tok, s, canvas_ids):
    """gpu_step with the decoder pass's routing forced to canvas_ids [L][B*C][k]
    (the gates still come from the device's own router logits)."""
    import torch
    ids_dev = torch.from_numpy(np.ascontiguousarray(canvas_ids, dtype=np.int32).reshape(-1)).cuda()
    den.force_routing(None, ids_dev)
    try:
        return gpu_step(den, wl, tok, s)
    finally:
        den.force_routing(None, None)


def routing_flips(ids, router_logits, diag):
    """Compare device routing with the oracle's, layer by layer.

    Returns (flipped rows mask, first flips [(layer, row, oracle margin)],
    max |router logit difference| over rows not yet flipped, per layer)."""
    L, R, _ = ids.shape
    flipped = np.zeros(R, dtype=bool)
    first, dr_max = [], []
    for l in range(L):
        differ = np.any(np.sort(ids[l], axis=1) != np.sort(diag["ids"][l], axis=1), axis=1)
        dr = np.abs(router_logits[l] - diag["router_logits"][l])
        dr_max.append(float(dr[~flipped].max()) if (~flipped).any() else 0.0)
        for r in np.nonzero(differ & ~flipped)[0]:
            first.append((l, int(r), float(diag["margin"][l][r])))
        flipped |= differ
    return flipped, first, dr_max


def ceil_div(a, b):
    return -(-a // b)


def bf16_dev_to_f64(t):
    """bf16 device tensor -> float64 numpy (exact)."""
    import torch
    return t.view(torch.int16).cpu().numpy().astype(np.uint16).astype(np.uint32).__lshift__(16).view(np.float32) \
        .astype(np.float64)


def layerwise_parity(den, wl, tok, s, n_seq=None):
    """Layer-wise teacher forcing: the device runs one step with its own routing,
    and its residual stream after every layer, its expert ids and its prompt
    cache are captured; the oracle then computes each layer l from the device's
    input to that layer (the residual h_l, the prompt K / V of layer l, the
    device's expert ids of layer l; the canvas's own q / k / v and everything
    else are computed by the oracle) and the final norm + LM head from the
    device's last residual.  Only the first n_seq sequences are compared (they
    are independent).  Returns (per-layer relative L2 of the layer's update
    h_{l+1} - h_l, relative L2 of h_{l+1}, relative L2 of the logits)."""
    import torch
    from oracle import decoder
    B, C, V, L, k, d = wl.batch, wl.canvas, wl.vocab, wl.n_layers, wl.top_k, wl.d_model
    nb = B if n_seq is None else n_seq
    R = B * C
    P = den_prompt_len(wl)
    S_max = den.cfg.prompt_max + C
    ids = torch.empty(L * R * k, dtype=torch.int32, device="cuda")
    hcap = torch.empty(L * R * d, dtype=torch.float32, device="cuda")
    den.capture_routing(ids, None)
    den.capture_residual(hcap)
    den.set_canvas(torch.from_numpy(np.asarray(tok).reshape(-1).astype(np.int32)).cuda(), None)
    logits = torch.empty(R * V, dtype=torch.float32, device="cuda")
    den.denoise_step(s, wl.steps, logits)
    den.synchronize()
    den.capture_routing(None, None)
    den.capture_residual(None)
    ids = ids.cpu().numpy().reshape(L, B, C, k)[:, :nb].reshape(L, nb * C, k)
    hs = hcap.view(L, B, C, d)[:, :nb].cpu().numpy().astype(np.float64)
    got_logits = logits.view(B, C, V)[:nb].cpu().numpy().astype(np.float64)
    del logits, hcap
    kc = torch.empty(B * wl.n_kv_heads * S_max * wl.head_dim, dtype=torch.bfloat16, device="cuda")
    vc = torch.empty_like(kc)
    cache = []
    for l in range(L):
        den.debug_read(4, l, kc)
        den.debug_read(5, l, vc)
        den.synchronize()
        kf = bf16_dev_to_f64(kc).reshape(B, wl.n_kv_heads, S_max, wl.head_dim)[:nb, :, :P]
        vf = bf16_dev_to_f64(vc).reshape(B, wl.n_kv_heads, S_max, wl.head_dim)[:nb, :, :P]
        cache.append((kf, vf))
    wl_o = wl.replace(batch=nb)
    W = decoder.Weights(wl_o)
    dp = decoder.DecoderPass(W, np.asarray(tok)[:nb], cache, forced_ids=list(ids))
    upd, full = [], []
    for l in range(L):
        h_in = dp.h.copy()
        dp.run_piece(2 * l)
        dp.run_piece(2 * l + 1)
        dev = hs[l]
        upd.append(rel_l2(dev - h_in, dp.h - h_in))
        full.append(rel_l2(dev, dp.h))
        dp.h = dev.copy()                 # the next layer starts from the device's residual
    dp.run_piece(2 * L)
    err_logits = rel_l2(got_logits, dp.logits)
    return upd, full, err_logits


def den_prompt_len(wl):
    return wl.prompt_len


def oracle_sensitivity(name):
    """The oracle's own sensitivity for workload `name` (tests/golden/oracle_sensitivity.json,
    written by tests/golden/make_oracle_sensitivity.py from the oracle alone), or None."""
    import json
    import os
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "oracle_sensitivity.json")
    if not os.path.exists(path):
        return None
    return json.load(open(path)).get(name)


def end_to_end_bar(name, base=1e-2):
    """Relative-L2 bar of an end-to-end step comparison: the benchmark spec's 1e-2, or the
    oracle's own logits sensitivity to fp32-sized perturbations of its residual
    stream when that is larger (no fp32 implementation can come closer)."""
    sens = oracle_sensitivity(name)
    return max(base, sens["logits_rel_l2"]) if sens else base


def flip_margin_bar(name, base=5e-2):
    """Largest oracle router margin at which a row's first routing flip is
    accepted: a fixed 5e-2 (router-logit units), or twice the largest first-flip
    margin the oracle itself shows under fp32-sized perturbations when larger."""
    sens = oracle_sensitivity(name)
    return max(base, 2.0 * sens["first_flip_margin_max"]) if sens else base


GELU_SLOPE_MAX = 1.13   # max |d/dx GELU_tanh(x)| (about 1.129, at x near 1.5)


def gated_activation_check(act, g, u, g_abs, u_abs, K):
    """Device bf16 activations act = bf16(GELU(g) * u) against the fp64 g, u of the
    same GEMM inputs.  fp32 accumulation of K products (each exact in fp32) is
    within K 2^-24 of the sum of their magnitudes (g_abs, u_abs: the same GEMMs on
    |operands|), which moves a by at most max|GELU'| |u| dg + |GELU(g)| du; the
    rest is the two sides' bf16 roundings (one ulp, 2^-7 of the value).  Asserts
    every element within that bound; returns the share of elements that differ
    at all."""
    from oracle import numerics
    a_ref = numerics.bf16_round(numerics.gelu_tanh(g) * u)
    gam = K * 2.0 ** -24
    bound = 2.0 ** -7 * np.abs(a_ref) + GELU_SLOPE_MAX * np.abs(u) * gam * g_abs + \
        np.abs(numerics.gelu_tanh(g)) * gam * u_abs
    diff = np.abs(act - a_ref)
    bad = diff > bound
    assert not bad.any(), (int(bad.sum()), float(np.max(diff / (np.abs(a_ref) + 1e-30))))
    return float(np.mean(diff > 0))
