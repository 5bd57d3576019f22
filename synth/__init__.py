"""Seeded synthetic inputs shared by the CPU oracle and the CUDA path.

This package holds no arithmetic of the denoising method.  It names the five
workloads (model shapes, batch, prompt length, canvas length, steps, seed) and
regenerates, element by element, the random-init bf16 weights, the prompt
tokens, the precomputed prompt KV caches of the long-prompt workload and the
synthetic fp32 logits used by sampler tests.  Values come from ``synth.c``
(a counter-based hash + an Irwin-Hall map), so any slice of any tensor can be
produced without materialising the others.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB_PATH = os.path.join(_HERE, "libsynth.so")
_lib = None

WEIGHT_STD = 0.02          # "Weights are bf16 drawn N(0,0.02)"
NORM_GAIN_STD = 0.02       # gains g of the (1+g) RMSNorm form, same law


def build(force: bool = False) -> str:
    """Compile synth.c into libsynth.so next to it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        u64, p = ctypes.c_uint64, ctypes.c_void_p
        lib.synth_normal_bf16.argtypes = [u64, u64, u64, u64, ctypes.c_double, p]
        lib.synth_normal_f32.argtypes = [u64, u64, u64, u64, ctypes.c_double, p]
        lib.synth_uniform_i32.argtypes = [u64, u64, u64, u64, ctypes.c_uint32, p]
        lib.synth_words.argtypes = [u64, u64, u64, u64, p]
        lib.synth_bf16_from_double.argtypes = [ctypes.c_double]
        lib.synth_bf16_from_double.restype = ctypes.c_uint16
        for f in (lib.synth_normal_bf16, lib.synth_normal_f32, lib.synth_uniform_i32, lib.synth_words):
            f.restype = None
        _lib = lib
    return _lib


def normal_bf16(seed: int, tid: int, first: int, n: int, std: float, out: Optional[np.ndarray] = None) -> np.ndarray:
    """bf16 bit patterns (uint16) of elements first..first+n-1 of stream (seed, tid)."""
    if out is None:
        out = np.empty(n, dtype=np.uint16)
    assert out.dtype == np.uint16 and out.flags.c_contiguous and out.size == n
    _load().synth_normal_bf16(seed, tid, first, n, std, out.ctypes.data)
    return out


def normal_f32(seed: int, tid: int, first: int, n: int, std: float) -> np.ndarray:
    out = np.empty(n, dtype=np.float32)
    _load().synth_normal_f32(seed, tid, first, n, std, out.ctypes.data)
    return out


def uniform_i32(seed: int, tid: int, first: int, n: int, V: int) -> np.ndarray:
    out = np.empty(n, dtype=np.int32)
    _load().synth_uniform_i32(seed, tid, first, n, V, out.ctypes.data)
    return out


def words(seed: int, tid: int, first: int, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.uint64)
    _load().synth_words(seed, tid, first, n, out.ctypes.data)
    return out


def bf16_from_double(x: float) -> int:
    return int(_load().synth_bf16_from_double(float(x)))


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float64 (bit placement only)."""
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# --------------------------------------------------------------------------- workloads

@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    n_layers: int
    d_model: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    n_experts: int
    top_k: int
    expert_width: int
    shared_width: int
    vocab: int
    batch: int
    prompt_len: int
    canvas: int
    steps: int
    seed: int
    prompt_kv_given: bool = False      # the long-prompt workload's cache is an input
    tau_max: float = 0.8
    tau_min: float = 0.4
    rms_eps: float = 1e-6
    rope_base: float = 10000.0
    commit_per_step: int = 0           # 0 -> ceil(C / T)
    expert_fp8: bool = False           # expert and shared-FFN GEMMs in FP8 E4M3 with per-row scales
    self_cond_width: int = 0           # width of the self-conditioning FFW (0: z_t = 0 throughout)

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    @property
    def qkv_rows(self) -> int:
        return (self.n_q_heads + 2 * self.n_kv_heads) * self.head_dim

    def param_count(self) -> int:
        d, L = self.d_model, self.n_layers
        per_layer = (2 * d + self.qkv_rows * d + d * self.n_q_heads * self.head_dim + self.n_experts * d
                     + self.n_experts * 3 * self.expert_width * d + 3 * self.shared_width * d)
        sc = d + 3 * self.self_cond_width * d if self.self_cond_width else 0
        return self.vocab * d + d + L * per_layer + sc


_MEDIUM_MODEL = dict(n_layers=8, d_model=1024, n_q_heads=16, n_kv_heads=4, head_dim=64, n_experts=32,
                     top_k=4, expert_width=1024, shared_width=0, vocab=32768)
_FULL_MODEL = dict(n_layers=30, d_model=2816, n_q_heads=16, n_kv_heads=8, head_dim=256, n_experts=128,
                   top_k=8, expert_width=704, shared_width=2112, vocab=262144)

WORKLOADS = {
    # tiny oracle-scale denoiser
    "tiny": Workload("tiny", n_layers=2, d_model=256, n_q_heads=4, n_kv_heads=4, head_dim=64, n_experts=8,
                     top_k=2, expert_width=512, shared_width=0, vocab=4096, batch=1, prompt_len=64, canvas=256,
                     steps=12, seed=0),
    # medium denoiser (GQA 16/4, 32 experts top-4)
    "medium": Workload("medium", **_MEDIUM_MODEL, batch=1, prompt_len=1024, canvas=256, steps=12, seed=1),
    # long prompt: the medium model over a 32768-token precomputed bf16 prompt cache
    "long_prompt": Workload("long_prompt", **_MEDIUM_MODEL, batch=1, prompt_len=32768, canvas=256, steps=12,
                            seed=2, prompt_kv_given=True),
    # full scale, one canvas: 128 experts top-8 + shared FFN, V = 262144 tied
    "full": Workload("full", **_FULL_MODEL, batch=1, prompt_len=2048, canvas=256, steps=12, seed=3),
    # full scale, 8 independent canvases (T swept over 4, 12, 32)
    "full_batched": Workload("full_batched", **_FULL_MODEL, batch=8, prompt_len=4096, canvas=256, steps=12,
                             seed=4),
}

# --------------------------------------------------------------------------- tensor streams

EMBED_ID, FINAL_NORM_ID, PROMPT_ID, LOGITS_ID, TARGET_ID = 1, 2, 10, 20, 30
SC_NORM_ID, SC_GATE_UP_ID, SC_DOWN_ID = 3, 4, 5      # the self-conditioning FFW
LAYER_KINDS = ("attn_norm", "w_qkv", "w_o", "ffn_norm", "w_router", "w_gate_up", "w_down",
               "w_shared_gate_up", "w_shared_down")


def tensor_id(kind: str, layer: Optional[int] = None) -> int:
    if kind == "embed":
        return EMBED_ID
    if kind == "final_norm":
        return FINAL_NORM_ID
    if kind in ("sc_norm", "w_sc_gate_up", "w_sc_down"):
        return {"sc_norm": SC_NORM_ID, "w_sc_gate_up": SC_GATE_UP_ID, "w_sc_down": SC_DOWN_ID}[kind]
    return 1000 + 16 * int(layer) + LAYER_KINDS.index(kind)


def tensor_shape(w: Workload, kind: str) -> tuple:
    d, E, we, ws = w.d_model, w.n_experts, w.expert_width, w.shared_width
    return {
        "embed": (w.vocab, d), "final_norm": (d,), "attn_norm": (d,), "ffn_norm": (d,),
        "w_qkv": (w.qkv_rows, d), "w_o": (d, w.n_q_heads * w.head_dim), "w_router": (E, d),
        "w_gate_up": (E, 2 * we, d), "w_down": (E, d, we),
        "w_shared_gate_up": (2 * ws, d), "w_shared_down": (d, ws),
        "sc_norm": (d,), "w_sc_gate_up": (2 * w.self_cond_width, d), "w_sc_down": (d, w.self_cond_width),
    }[kind]


def tensor_std(kind: str) -> float:
    return NORM_GAIN_STD if kind.endswith("norm") else WEIGHT_STD


def weight_bf16(w: Workload, kind: str, layer: Optional[int] = None, expert: Optional[int] = None) -> np.ndarray:
    """bf16 bit patterns of a weight tensor (or of one expert's slice of an expert tensor)."""
    shape = tensor_shape(w, kind)
    if expert is not None:
        shape = shape[1:]
        n = int(np.prod(shape))
        first = int(expert) * n
    else:
        n = int(np.prod(shape))
        first = 0
    return normal_bf16(w.seed, tensor_id(kind, layer), first, n, tensor_std(kind)).reshape(shape)


def weight_rows_bf16(w: Workload, kind: str, row0: int, nrows: int, layer: Optional[int] = None) -> np.ndarray:
    """Rows row0..row0+nrows-1 of a 2-D weight tensor (e.g. a slice of the embedding)."""
    shape = tensor_shape(w, kind)
    cols = shape[-1]
    return normal_bf16(w.seed, tensor_id(kind, layer), row0 * cols, nrows * cols,
                       tensor_std(kind)).reshape(nrows, cols)


def prompt_tokens(w: Workload, P: Optional[int] = None) -> np.ndarray:
    P = w.prompt_len if P is None else P
    return uniform_i32(w.seed, PROMPT_ID, 0, w.batch * P, w.vocab).reshape(w.batch, P)


# Precomputed prompt caches: K and V entries drawn with the spread a canvas
# projection has at init, sqrt(d) * 0.02 (x has unit RMS after the norm).
def prompt_kv_std(w: Workload) -> float:
    return float(np.sqrt(w.d_model) * WEIGHT_STD)


def prompt_kv_bf16(w: Workload, layer: int, which: str, P: Optional[int] = None) -> np.ndarray:
    """[B][Hkv][P][hd] bf16 bits of a precomputed prompt K (which='k', post-RoPE) or V cache."""
    P = w.prompt_len if P is None else P
    n = w.batch * w.n_kv_heads * P * w.head_dim
    tid = 3000 + 2 * layer + (0 if which == "k" else 1)
    return normal_bf16(w.seed, tid, 0, n, prompt_kv_std(w)).reshape(w.batch, w.n_kv_heads, P, w.head_dim)


def target_canvas(w: Workload, stream: int = 0) -> np.ndarray:
    """A random clean canvas x0 [B][C] (for forward-noised teacher-forced inputs)."""
    return uniform_i32(w.seed, TARGET_ID + stream, 0, w.batch * w.canvas, w.vocab).reshape(w.batch, w.canvas)


def logits_f32(seed: int, stream: int, rows: int, V: int, std: float = 1.0) -> np.ndarray:
    return normal_f32(seed, LOGITS_ID + stream, 0, rows * V, std).reshape(rows, V)
