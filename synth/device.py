"""Upload a workload's synthetic inputs to a CUDA device as torch tensors.

Input plumbing only (no arithmetic of the method): the bf16 bit patterns from
the generator are copied into torch.bfloat16 device tensors in the layouts the
C ABI documents (each GEMM weight [out][in], expert tensors [E][...]).
"""
from __future__ import annotations

import numpy as np
import torch

from . import Workload, LAYER_KINDS, weight_bf16, prompt_tokens, prompt_kv_bf16, tensor_shape


def _to_dev(bits: np.ndarray, device) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.to(device, non_blocking=False)


def _tensor_to_dev(w: Workload, kind: str, layer, device) -> torch.Tensor:
    shape = tensor_shape(w, kind)
    if len(shape) == 3:   # expert tensors: one expert at a time keeps host memory small
        out = torch.empty(shape, dtype=torch.bfloat16, device=device)
        for e in range(shape[0]):
            out[e].copy_(_to_dev(weight_bf16(w, kind, layer, expert=e), device))
        return out
    return _to_dev(weight_bf16(w, kind, layer), device)


def device_self_cond_weights(w: Workload, device="cuda"):
    """(sc_norm, w_sc_gate_up, w_sc_down) bf16 device tensors of the self-conditioning FFW, or Nones."""
    if not w.self_cond_width:
        return None, None, None
    return tuple(_tensor_to_dev(w, k, None, device) for k in ("sc_norm", "w_sc_gate_up", "w_sc_down"))


def device_weights(w: Workload, device="cuda"):
    """(embed, final_norm, [per-layer dict]) of bf16 device tensors."""
    embed = _tensor_to_dev(w, "embed", None, device)
    final_norm = _tensor_to_dev(w, "final_norm", None, device)
    layers = []
    for l in range(w.n_layers):
        d = {}
        for kind in LAYER_KINDS:
            if kind.startswith("w_shared") and w.shared_width == 0:
                d[kind] = None
                continue
            d[kind] = _tensor_to_dev(w, kind, l, device)
        layers.append(d)
    return embed, final_norm, layers


def config_fields(w: Workload, prompt_max: int | None = None) -> dict:
    return dict(n_layers=w.n_layers, d_model=w.d_model, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads,
                head_dim=w.head_dim, n_experts=w.n_experts, top_k=w.top_k, expert_width=w.expert_width,
                shared_width=w.shared_width, vocab=w.vocab, batch=w.batch,
                prompt_max=w.prompt_len if prompt_max is None else prompt_max, canvas=w.canvas,
                commit_per_step=w.commit_per_step, tau_max=w.tau_max, tau_min=w.tau_min, rms_eps=w.rms_eps,
                rope_base=w.rope_base, expert_fp8=int(w.expert_fp8), self_cond_width=w.self_cond_width)


def device_prompt(w: Workload, device="cuda", P=None) -> torch.Tensor:
    return torch.from_numpy(prompt_tokens(w, P)).to(device)


def device_prompt_kv(w: Workload, layer: int, device="cuda", P=None):
    k = _to_dev(prompt_kv_bf16(w, layer, "k", P), device)
    v = _to_dev(prompt_kv_bf16(w, layer, "v", P), device)
    return k, v
