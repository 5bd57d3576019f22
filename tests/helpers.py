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


def ceil_div(a, b):
    return -(-a // b)
