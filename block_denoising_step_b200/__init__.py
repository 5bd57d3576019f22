"""Python binding of the dgen C ABI (include/dgen.h): argument marshalling only.

Every step of the denoising path runs in the CUDA library ``lib/libdgen.so``;
this module only converts torch tensors / ints to the C call's pointers and
sizes and turns non-zero status codes into exceptions.  Importing it fails
loudly when the library has not been built.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass, fields

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "lib", "libdgen.so")
PROBE_LIB_PATH = os.path.join(_HERE, "lib", "libdgen_probe.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"block_denoising_step_b200: CUDA library not built ({LIB_PATH} missing); "
                      "run `python -c 'import __graft_entry__ as g; g.build()'` from the repository root")

_lib = ctypes.CDLL(LIB_PATH)

DGEN_OK, DGEN_EINVAL, DGEN_ENOMEM, DGEN_ECAP, DGEN_ECUDA, DGEN_EDEVICE, DGEN_ESTATE, DGEN_ESCRATCH = \
    0, -1, -2, -3, -4, -5, -6, -7

EXPORTED = ("dgen_create", "dgen_destroy", "dgen_prefill_prompt", "dgen_set_prompt_kv", "dgen_init_canvas",
            "dgen_set_canvas", "dgen_get_canvas", "dgen_denoise_step", "dgen_sample_commit", "dgen_sample_commit_eb",
            "dgen_set_logits",
            "dgen_generate_block", "dgen_generate_block_host", "dgen_forward_noise", "dgen_synchronize",
            "dgen_launch_count", "dgen_status_str", "dgen_gemm_bf16", "dgen_set_timing", "dgen_get_timing",
            "dgen_capture_routing", "dgen_debug_read", "dgen_sample_from_logits_noalloc",
            "dgen_set_flags", "dgen_expert_usage", "dgen_force_routing", "dgen_set_tuning",
            "dgen_generate_block_eb", "dgen_append_canvas", "dgen_generate", "dgen_capture_residual",
            "dgen_gemm_e4m3", "dgen_set_self_cond", "dgen_gemm_bf16_pair")
PROBE_EXPORTED = ("dgen_gemm_rowsum_variant",)

K_QKV, K_ATTENTION, K_OPROJ, K_ROUTER, K_EXPERT_GATE_UP, K_EXPERT_DOWN, K_SHARED_FFN, K_LM_HEAD, K_SAMPLER, \
    K_OTHER, K_SELF_COND = range(11)
KERNEL_CLASSES = ("qkv", "attention", "oproj", "router", "expert_gate_up", "expert_down", "shared_ffn", "lm_head",
                  "sampler", "other", "self_cond")


class Config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "n_layers", "d_model", "n_q_heads", "n_kv_heads", "head_dim", "n_experts", "top_k", "expert_width",
        "shared_width", "vocab", "batch", "prompt_max", "canvas", "commit_per_step")] + \
        [(n, ctypes.c_float) for n in ("tau_max", "tau_min", "rms_eps", "rope_base")] + \
        [("expert_fp8", ctypes.c_int32), ("self_cond_width", ctypes.c_int32)]


class LayerWeights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "attn_norm", "w_qkv", "w_o", "ffn_norm", "w_router", "w_gate_up", "w_down", "w_shared_gate_up",
        "w_shared_down")]


class Weights(ctypes.Structure):
    _fields_ = [("embed", ctypes.c_void_p), ("final_norm", ctypes.c_void_p),
                ("layers", ctypes.POINTER(LayerWeights)),
                ("sc_norm", ctypes.c_void_p), ("w_sc_gate_up", ctypes.c_void_p), ("w_sc_down", ctypes.c_void_p)]


_P, _I32, _I64, _U64, _F = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64, ctypes.c_float
_SIGS = {
    "dgen_create": [ctypes.POINTER(Config), ctypes.POINTER(Weights), _P, ctypes.POINTER(_P)],
    "dgen_destroy": [_P],
    "dgen_prefill_prompt": [_P, _P, _I32],
    "dgen_set_prompt_kv": [_P, _I32, _P, _P, _I32],
    "dgen_init_canvas": [_P, _U64],
    "dgen_set_canvas": [_P, _P, _P],
    "dgen_get_canvas": [_P, _P, _P],
    "dgen_denoise_step": [_P, _I32, _I32, _P],
    "dgen_sample_commit": [_P, _I32, _I32, _U64, _P],
    "dgen_sample_commit_eb": [_P, _P, _I32, _I32, _U64, _F, _F, _I32, _P, _P],
    "dgen_generate_block_eb": [_P, _P, _I32, _I32, _U64, _F, _F, _I32, _P, _P],
    "dgen_append_canvas": [_P],
    "dgen_capture_residual": [_P, _P],
    "dgen_set_self_cond": [_P, _P],
    "dgen_generate": [_P, _P, _I32, _I32, _I32, _U64, _P],
    "dgen_set_logits": [_P, _P, _I32, _I32],
    "dgen_generate_block": [_P, _P, _I32, _I32, _U64, _P],
    "dgen_generate_block_host": [_P, _P, _I32, _I32, _U64, _P],
    "dgen_forward_noise": [_P, _P, _F, _U64, _I32, _P],
    "dgen_synchronize": [_P],
    "dgen_launch_count": [_P],
    "dgen_status_str": [ctypes.c_int],
    "dgen_gemm_bf16": [_P, _P, _P, _I32, _I32, _I32, _P],
    "dgen_gemm_bf16_pair": [_P, _P, _P, _I32, _I32, _I32, _P],
    "dgen_gemm_e4m3": [_P, _P, _P, _I32, _I32, _I32, _P],
    "dgen_set_timing": [_P, ctypes.c_uint32],
    "dgen_set_flags": [_P, ctypes.c_uint32],
    "dgen_expert_usage": [_P, _P],
    "dgen_force_routing": [_P, _P, _P],
    "dgen_set_tuning": [_P, _I32, _I32],
    "dgen_capture_routing": [_P, _P, _P],
    "dgen_debug_read": [_P, _I32, _I32, _P, _U64],
    "dgen_sample_from_logits_noalloc": [_P, _P, _P, _I32, _I32, _I32, _I32, _I32, _U64, _F, _F, _I32, _P, _P],
    "dgen_get_timing": [_P, _I32, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(_I64)],
}
for _name, _args in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.argtypes = _args
    _f.restype = ctypes.c_int
_lib.dgen_status_str.restype = ctypes.c_char_p
_lib.dgen_launch_count.restype = ctypes.c_int64


class DgenError(RuntimeError):
    def __init__(self, call: str, status: int):
        super().__init__(f"{call}: {status} ({_lib.dgen_status_str(status).decode()})")
        self.status = status


def _check(call: str, status: int) -> None:
    if status != DGEN_OK:
        raise DgenError(call, status)


def _ptr(t) -> int | None:
    """Device address of a torch tensor (or None / an int address)."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


@dataclass
class ModelConfig:
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
    prompt_max: int
    canvas: int
    commit_per_step: int = 0
    tau_max: float = 0.8
    tau_min: float = 0.4
    rms_eps: float = 1e-6
    rope_base: float = 10000.0
    expert_fp8: int = 0
    self_cond_width: int = 0

    def to_c(self) -> Config:
        return Config(**{f.name: getattr(self, f.name) for f in fields(self)})


LAYER_FIELDS = [f[0] for f in LayerWeights._fields_]


_probe_lib = None


def probe_lib():
    """The measurement library (include/dgen_probe.h), loaded on first use."""
    global _probe_lib
    if _probe_lib is None:
        if not os.path.exists(PROBE_LIB_PATH):
            raise ImportError(f"{PROBE_LIB_PATH} missing; build with block_denoising_step_b200/build.py")
        lib = ctypes.CDLL(PROBE_LIB_PATH)
        lib.dgen_gemm_rowsum_variant.argtypes = [_P, _P, _P, _I32, _I32, _I32, _I32, _P]
        lib.dgen_gemm_rowsum_variant.restype = ctypes.c_int
        _probe_lib = lib
    return _probe_lib


def gemm_e4m3(a, b, d, stream: int = 0) -> None:
    """d[M][N] (fp32) = a[M][K] @ b[N][K]^T with E4M3 operands (uint8 tensors of the
    encodings) through the library's tcgen05 kind::f8f6f4 path."""
    M, K = a.shape
    N = b.shape[0]
    _check("dgen_gemm_e4m3", _lib.dgen_gemm_e4m3(_ptr(a), _ptr(b), _ptr(d), M, N, K, stream))


def gemm_bf16_pair(a, b, d, stream: int = 0) -> None:
    """gemm_bf16 on CTA pairs (tcgen05.mma.cta_group::2, 256 x 256 tiles)."""
    M, K = a.shape
    N = b.shape[0]
    _check("dgen_gemm_bf16_pair", _lib.dgen_gemm_bf16_pair(_ptr(a), _ptr(b), _ptr(d), M, N, K, stream))


def gemm_bf16(a, b, d, stream: int = 0) -> None:
    """d[M][N] (fp32) = a[M][K] @ b[N][K]^T through the library's tcgen05 GEMM core."""
    M, K = a.shape
    N = b.shape[0]
    _check("dgen_gemm_bf16", _lib.dgen_gemm_bf16(_ptr(a), _ptr(b), _ptr(d), M, N, K, stream))


def sample_from_logits_noalloc(logits, tok, committed, batch: int, canvas: int, vocab: int, s: int, T: int,
                               seed: int, tau_max: float = 0.8, tau_min: float = 0.4, commit_per_step: int = 0,
                               conf=None, stream: int = 0) -> None:
    """The sampler step on given logits without a handle and without any device
    allocation (see dgen_sample_from_logits_noalloc); tok / committed are
    updated in place."""
    _check("dgen_sample_from_logits_noalloc",
           _lib.dgen_sample_from_logits_noalloc(_ptr(logits), _ptr(tok), _ptr(committed), batch, canvas, vocab, s,
                                                T, seed, tau_max, tau_min, commit_per_step, _ptr(conf), stream))


class Denoiser:
    """One dgen handle.  `weights` maps names to device tensors (bf16):
    'embed', 'final_norm' and per layer a dict with LAYER_FIELDS keys;
    self_cond: (sc_norm, w_sc_gate_up, w_sc_down) when cfg.self_cond_width > 0."""

    def __init__(self, cfg: ModelConfig, embed, final_norm, layers, stream: int = 0, self_cond=None):
        self.cfg = cfg
        self._keep = (embed, final_norm, layers, self_cond)
        arr = (LayerWeights * cfg.n_layers)()
        for i, lw in enumerate(layers):
            for name in LAYER_FIELDS:
                setattr(arr[i], name, _ptr(lw.get(name)))
        self._layers = arr
        sc = tuple(self_cond) if self_cond is not None else (None, None, None)
        w = Weights(_ptr(embed), _ptr(final_norm), ctypes.cast(arr, ctypes.POINTER(LayerWeights)),
                    _ptr(sc[0]), _ptr(sc[1]), _ptr(sc[2]))
        c = cfg.to_c()
        h = _P()
        _check("dgen_create", _lib.dgen_create(ctypes.byref(c), ctypes.byref(w), stream, ctypes.byref(h)))
        self._h = h

    def close(self) -> None:
        if self._h:
            _lib.dgen_destroy(self._h)
            self._h = _P()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def prefill_prompt(self, prompt) -> None:
        _check("dgen_prefill_prompt", _lib.dgen_prefill_prompt(self._h, _ptr(prompt), prompt.shape[-1]))

    def set_prompt_kv(self, layer: int, k, v, P: int) -> None:
        _check("dgen_set_prompt_kv", _lib.dgen_set_prompt_kv(self._h, layer, _ptr(k), _ptr(v), P))

    def init_canvas(self, seed: int) -> None:
        _check("dgen_init_canvas", _lib.dgen_init_canvas(self._h, seed))

    def set_canvas(self, tok, committed=None) -> None:
        _check("dgen_set_canvas", _lib.dgen_set_canvas(self._h, _ptr(tok), _ptr(committed)))

    def get_canvas(self, tok=None, committed=None) -> None:
        _check("dgen_get_canvas", _lib.dgen_get_canvas(self._h, _ptr(tok), _ptr(committed)))

    def denoise_step(self, s: int, T: int, logits=None) -> None:
        _check("dgen_denoise_step", _lib.dgen_denoise_step(self._h, s, T, _ptr(logits)))

    def set_self_cond(self, z=None) -> None:
        """The self-conditioning state [B][C][d] fp32 the next denoise step adds
        to the canvas embeddings (None: zero)."""
        _check("dgen_set_self_cond", _lib.dgen_set_self_cond(self._h, _ptr(z)))

    def sample_commit(self, s: int, T: int, seed: int, conf=None) -> None:
        _check("dgen_sample_commit", _lib.dgen_sample_commit(self._h, s, T, seed, _ptr(conf)))

    def sample_commit_eb(self, logits, s: int, T_max: int, seed: int, gamma: float, stop_threshold: float,
                         entropy=None, stop=None, freeze: bool = True) -> None:
        """Entropy-bounded sampler step (see dgen_sample_commit_eb): on given fp32
        logits, or, with logits None, on the last denoise step's LM-head statistics."""
        _check("dgen_sample_commit_eb",
               _lib.dgen_sample_commit_eb(self._h, _ptr(logits), s, T_max, seed, gamma, stop_threshold,
                                          1 if freeze else 0, _ptr(entropy), _ptr(stop)))

    def generate_block_eb(self, prompt, T_max: int, seed: int, gamma: float, stop_threshold: float, out,
                          freeze: bool = True):
        """One block with the entropy-bounded sampler and adaptive stopping (prompt None:
        continue from the current cache); returns the steps each canvas took (list of B ints)."""
        steps = (ctypes.c_int32 * self.cfg.batch)()
        P = 0 if prompt is None else prompt.shape[-1]
        _check("dgen_generate_block_eb",
               _lib.dgen_generate_block_eb(self._h, _ptr(prompt), P, T_max, seed, gamma,
                                           stop_threshold, 1 if freeze else 0, _ptr(out), ctypes.cast(steps, _P)))
        return list(steps)

    def append_canvas(self) -> None:
        """Re-encode the current canvas causally and append its K/V to the cache."""
        _check("dgen_append_canvas", _lib.dgen_append_canvas(self._h))

    def generate(self, prompt, n_blocks: int, T: int, seed: int, out) -> None:
        """Block-autoregressive generation of n_blocks canvases; out [B][n_blocks * C]."""
        _check("dgen_generate", _lib.dgen_generate(self._h, _ptr(prompt), prompt.shape[-1], n_blocks, T, seed,
                                                   _ptr(out)))

    def set_logits(self, logits, s: int, T: int) -> None:
        _check("dgen_set_logits", _lib.dgen_set_logits(self._h, _ptr(logits), s, T))

    def generate_block(self, prompt, T: int, seed: int, out) -> None:
        _check("dgen_generate_block",
               _lib.dgen_generate_block(self._h, _ptr(prompt), prompt.shape[-1], T, seed, _ptr(out)))

    def generate_block_host(self, prompt_host, T: int, seed: int, out_host) -> None:
        """prompt_host / out_host: CPU torch tensors (int32, contiguous; pinned for speed)."""
        _check("dgen_generate_block_host",
               _lib.dgen_generate_block_host(self._h, prompt_host.data_ptr(), prompt_host.shape[-1], T, seed,
                                             out_host.data_ptr()))

    def forward_noise(self, x0, kappa: float, seed: int, step: int, xt) -> None:
        _check("dgen_forward_noise", _lib.dgen_forward_noise(self._h, _ptr(x0), kappa, seed, step, _ptr(xt)))

    def synchronize(self) -> None:
        _check("dgen_synchronize", _lib.dgen_synchronize(self._h))

    def launch_count(self) -> int:
        return int(_lib.dgen_launch_count(self._h))

    FLAG_NO_GRAPH, FLAG_NO_PDL = 1, 2

    TUNE_EXPERT_CHUNK, TUNE_ATTN_SPLITS, TUNE_ROUTER_SPLITS, TUNE_QKV_SPLITS, TUNE_ATTN_KERNEL = 0, 1, 2, 3, 4
    TUNE_ROUTE_BARRIER_EXTRA = 5
    TUNE_SEPARATE_EXPERTS = 6
    TUNE_STATIC_ITEMS = 7
    TUNE_PAIRS = 8
    TUNE_CHUNK_ORDER = 9

    def set_tuning(self, key: int, value: int) -> None:
        _check("dgen_set_tuning", _lib.dgen_set_tuning(self._h, key, value))

    def force_routing(self, prompt_ids=None, canvas_ids=None) -> None:
        """Teacher-force the routing of the prompt pass ([L][B*P][k] int32) and/or of
        the decoder pass ([L][B*C][k]); None releases."""
        self._force = (prompt_ids, canvas_ids)
        _check("dgen_force_routing", _lib.dgen_force_routing(self._h, _ptr(prompt_ids), _ptr(canvas_ids)))

    def expert_usage(self):
        """Per layer, the number of experts routed to in the last pass."""
        out = (ctypes.c_int32 * self.cfg.n_layers)()
        _check("dgen_expert_usage", _lib.dgen_expert_usage(self._h, ctypes.cast(out, _P)))
        return list(out)

    def set_flags(self, flags: int) -> None:
        _check("dgen_set_flags", _lib.dgen_set_flags(self._h, flags))

    def capture_routing(self, ids=None, logits=None) -> None:
        """Record each layer's top-k ids [L][B*C][k] (and router logits [L][B*C][E])
        during subsequent denoise steps; None, None stops."""
        self._cap = (ids, logits)
        _check("dgen_capture_routing", _lib.dgen_capture_routing(self._h, _ptr(ids), _ptr(logits)))

    def capture_residual(self, h=None) -> None:
        """Record the residual stream after every layer [L][B*C][d] fp32 during
        subsequent denoise steps; None stops."""
        self._cap_h = h
        _check("dgen_capture_residual", _lib.dgen_capture_residual(self._h, _ptr(h)))

    def debug_read(self, which: int, layer: int, dst) -> None:
        """Copy an internal buffer (see dgen_debug_read) into the device tensor dst."""
        _check("dgen_debug_read", _lib.dgen_debug_read(self._h, which, layer, _ptr(dst),
                                                        dst.numel() * dst.element_size()))

    def set_timing(self, classes) -> None:
        mask = 0
        for c in classes:
            mask |= 1 << c
        _check("dgen_set_timing", _lib.dgen_set_timing(self._h, mask))

    def get_timing(self, cls: int):
        """(total ms, launches) of class cls since the last call; synchronizes."""
        ms, n = ctypes.c_double(), _I64()
        _check("dgen_get_timing", _lib.dgen_get_timing(self._h, cls, ctypes.byref(ms), ctypes.byref(n)))
        return ms.value, n.value
