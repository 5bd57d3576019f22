"""Shared test plumbing: building a device model from a workload and comparing with the oracle."""
import math

import numpy as np

import synth


def rel_l2(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def make_denoiser(wl, prompt_max=None, device="cuda"):
    import torch
    import block_denoising_step_b200 as dg
    from synth.device import device_weights, config_fields
    embed, final_norm, layers = device_weights(wl, device)
    cfg = dg.ModelConfig(**config_fields(wl, prompt_max))
    stream = torch.cuda.current_stream().cuda_stream
    return dg.Denoiser(cfg, embed, final_norm, layers, stream=stream)


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
