"""Decoder logits of one canvas step, and the causal prompt pass (test infrastructure only).

Follows the hyper.ai digest of the DiffusionGemma paper, Method:
* the model is one transformer used both as a causal encoder (builds the KV
  cache from the prompt) and as the denoising decoder (three-stage pipeline
  paragraph);
* the decoder sees the noisy canvas x_t, the cache H and a self-conditioning
  state z_t and returns logits L_t in R^{C x V} (eq. 3), with bidirectional
  attention over the canvas and attention to the cache;
* E in R^{V x d} is the token embedding (text after eq. 4); the LM head is tied
  to it (full-scale workload description, applied to every workload).

Readings where the pages are silent (each is the plainest standard choice):
* z_t = 0 (the self-conditioning state is zero, a regime the model is trained
  in for half the batch; its injection point is not stated);
* pre-norm blocks h += Attn(RMSNorm(h)); h += MoE(RMSNorm(h)) [+ shared FFN of
  the same normed input];
* canvas queries at absolute positions P..P+C-1 attend, with ONE softmax, over
  keys [prompt cache (positions 0..P-1) ; canvas], no mask; scale 1/sqrt(hd);
  GQA: query head h reads KV head floor(h * Hkv / Hq);
* router: logits r = x W_r^T; the k largest (ties: lower expert id); gates =
  softmax over those k logits; expert e computes W_d,e (GELU(W_g,e x) * (W_u,e x)).
Storage convention (not a reading of the pages): the [2w][d] gate-up tensor
interleaves gate and up rows in blocks of 16 (split_gate_up).
"""
import math

import numpy as np

import synth

from . import fp8, numerics
from .numerics import bf16_bits_to_f64, rmsnorm, rope, gelu_tanh, softmax

_CACHE_LIMIT_BYTES = 4 << 30


class Weights:
    """fp64 views of the synthetic bf16 weights of a workload, regenerated on demand
    (cached as bf16 bits when the whole model is small)."""

    def __init__(self, wl: synth.Workload, arrays=None):
        """arrays: optional {(kind, layer): fp64 array} replacing the synthetic
        weights (for pins with hand-made weights)."""
        self.wl = wl
        self._arrays = arrays
        self._cache = {} if 2 * wl.param_count() <= _CACHE_LIMIT_BYTES else None

    def bits(self, kind, layer=None, expert=None):
        if self._cache is None:
            return synth.weight_bf16(self.wl, kind, layer, expert)
        key = (kind, layer)
        if key not in self._cache:
            self._cache[key] = synth.weight_bf16(self.wl, kind, layer)
        t = self._cache[key]
        return t if expert is None else t[expert]

    def get(self, kind, layer=None, expert=None):
        if self._arrays is not None:
            t = self._arrays[(kind, layer)]
            return t if expert is None else t[expert]
        return bf16_bits_to_f64(self.bits(kind, layer, expert))

    def get_fp8(self, kind, layer=None, expert=None):
        """(q, s): the weight quantized to E4M3 with one power-of-two scale per
        stored row (oracle.fp8.quant_rows)."""
        return fp8.quant_rows(self.get(kind, layer, expert))

    def embed_rows(self, tok):
        tok = np.asarray(tok)
        if self._arrays is not None:
            return self._arrays[("embed", None)][tok]
        if self._cache is not None:
            return bf16_bits_to_f64(self.bits("embed")[tok])
        flat = tok.reshape(-1)
        out = np.empty((flat.size, self.wl.d_model))
        for n, t in enumerate(flat):
            out[n] = bf16_bits_to_f64(synth.weight_rows_bf16(self.wl, "embed", int(t), 1)[0])
        return out.reshape(tok.shape + (self.wl.d_model,))

    def embed_chunks(self, chunk_rows=16384):
        V = self.wl.vocab
        for r0 in range(0, V, chunk_rows):
            n = min(chunk_rows, V - r0)
            if self._arrays is not None:
                yield r0, self._arrays[("embed", None)][r0:r0 + n]
            elif self._cache is not None:
                yield r0, bf16_bits_to_f64(self.bits("embed")[r0:r0 + n])
            else:
                yield r0, bf16_bits_to_f64(synth.weight_rows_bf16(self.wl, "embed", r0, n))


def attention(q, k, v, causal_offset=None):
    """Scaled dot-product attention, one softmax per query row over all keys.

    q [B][Hq][n][hd]; k, v [B][Hkv][S][hd].  causal_offset=None: no mask (the
    canvas pass).  causal_offset=o: query i may see key j only if j <= i + o
    (the causal prompt pass, o = 0)."""
    B, Hq, n, hd = q.shape
    Hkv, S = k.shape[1], k.shape[2]
    out = np.empty_like(q)
    for b in range(B):
        for h in range(Hq):
            kvh = (h * Hkv) // Hq
            s = q[b, h] @ k[b, kvh].T / math.sqrt(hd)
            if causal_offset is not None:
                i = np.arange(n)[:, None]
                j = np.arange(S)[None, :]
                s = np.where(j <= i + causal_offset, s, -np.inf)
            out[b, h] = softmax(s, axis=-1) @ v[b, kvh]
    return out


def route(xn, w_router, top_k, forced_ids=None):
    """Router logits, top-k expert ids (ties: lower id), gates, and per-token
    margin between the k-th and (k+1)-th logit (inf when k = E).

    forced_ids [n][k]: use these experts instead of the top-k (teacher forcing
    of the routing, to compare the arithmetic of a layer with another
    implementation's choices); the gates are still the softmax of this router's
    logits over the given ids, and the margins are inf."""
    r = xn @ w_router.T
    n, E = r.shape
    ids = np.empty((n, top_k), dtype=np.int64)
    margin = np.full(n, np.inf)
    for t in range(n):
        if forced_ids is not None:
            ids[t] = forced_ids[t]
            continue
        order = np.lexsort((np.arange(E), -r[t]))    # by -logit, then by id
        ids[t] = order[:top_k]
        if top_k < E:
            margin[t] = r[t, order[top_k - 1]] - r[t, order[top_k]]
    gates = softmax(np.take_along_axis(r, ids, axis=1), axis=1)
    return r, ids, gates, margin


def split_gate_up(w_gate_up):
    """(W_g, W_u) from the stored [2w][d] tensor, whose rows interleave gate and up
    in blocks of 16: rows 32j..32j+15 are gate rows 16j..16j+15, rows 32j+16..32j+31
    the matching up rows."""
    two_w, d = w_gate_up.shape
    blocks = w_gate_up.reshape(two_w // 32, 2, 16, d)
    return blocks[:, 0].reshape(two_w // 2, d), blocks[:, 1].reshape(two_w // 2, d)


def expert_ffn(x, w_gate_up, w_down):
    """Gated-GELU FFN: W_d (GELU(W_g x) * (W_u x)).  The activation entering W_d
    is rounded to bf16 (a GEMM input)."""
    w_g, w_u = split_gate_up(w_gate_up)
    g = x @ w_g.T
    u = x @ w_u.T
    a = numerics.bf16_round(gelu_tanh(g) * u)
    return a @ w_down.T


def moe(xn, W: Weights, layer: int, forced_ids=None):
    """Routed MoE output for rows xn [n][d] (plus the shared FFN, when present);
    forced_ids as in route.  With the workload's expert_fp8 set, the expert and
    shared-FFN GEMMs run in FP8 (oracle.fp8): the rows xn are quantized once per
    token, the weights per stored row."""
    wl = W.wl
    r, ids, gates, margin = route(xn, W.get("w_router", layer), wl.top_k, forced_ids)
    y = np.zeros_like(xn)
    if wl.expert_fp8:
        xq, sx = fp8.quant_rows(xn)

        def ffn(rows, gu_kind, d_kind, e=None):
            return fp8.expert_ffn_fp8(xq[rows], sx[rows], W.get_fp8(gu_kind, layer, e), W.get_fp8(d_kind, layer, e))
    else:
        def ffn(rows, gu_kind, d_kind, e=None):
            return expert_ffn(xn[rows], W.get(gu_kind, layer, e), W.get(d_kind, layer, e))
    for e in range(wl.n_experts):
        rows, slot = np.nonzero(ids == e)
        if rows.size == 0:
            continue
        ye = ffn(rows, "w_gate_up", "w_down", e)
        y[rows] += gates[rows, slot][:, None] * ye
    if wl.shared_width > 0:
        y += ffn(np.arange(xn.shape[0]), "w_shared_gate_up", "w_shared_down")
    return y, {"router_logits": r, "ids": ids, "gates": gates, "margin": margin}


def _split_heads(x, H, hd):
    B, n, _ = x.shape
    return x.reshape(B, n, H, hd).transpose(0, 2, 1, 3)


def _qkv(xn, W: Weights, layer, pos):
    wl = W.wl
    Hq, Hkv, hd = wl.n_q_heads, wl.n_kv_heads, wl.head_dim
    qkv = xn @ W.get("w_qkv", layer).T
    q = _split_heads(qkv[..., : Hq * hd], Hq, hd)
    k = _split_heads(qkv[..., Hq * hd:(Hq + Hkv) * hd], Hkv, hd)
    v = _split_heads(qkv[..., (Hq + Hkv) * hd:], Hkv, hd)
    q = numerics.bf16_round(rope(q, pos, wl.rope_base))
    k = numerics.bf16_round(rope(k, pos, wl.rope_base))
    return q, k, numerics.bf16_round(v)


def _attn_out(o, W: Weights, layer):
    B, Hq, n, hd = o.shape
    o = numerics.bf16_round(o).transpose(0, 2, 1, 3).reshape(B, n, Hq * hd)
    return o @ W.get("w_o", layer).T


def prefill(W: Weights, prompt, routing=None, prefix=None):
    """Causal pass of the encoder: returns per layer (K, V), each [B][Hkv][P][hd]
    (bf16 values).  routing: optional list that receives each layer's top-k ids
    [B*P][k].

    prefix: an existing cache (per layer (K, V) over P0 positions).  The tokens
    then sit at positions P0..P0+P-1, query i sees the prefix and the new keys up
    to position P0 + i, and the returned cache is the prefix followed by the new
    positions -- stage 3 of the three-stage pipeline (hyper.ai digest, Method:
    the finished canvas goes back through the causal encoder and is appended to
    the KV cache)."""
    wl = W.wl
    prompt = np.asarray(prompt)
    B, P = prompt.shape
    P0 = 0 if prefix is None else prefix[0][0].shape[2]
    pos = P0 + np.arange(P)
    h = W.embed_rows(prompt)
    cache = []
    for layer in range(wl.n_layers):
        xn = numerics.bf16_round(rmsnorm(h, W.get("attn_norm", layer), wl.rms_eps))
        q, k, v = _qkv(xn, W, layer, pos)
        if prefix is not None:
            k = np.concatenate([prefix[layer][0], k], axis=2)
            v = np.concatenate([prefix[layer][1], v], axis=2)
        cache.append((k, v))
        if layer == wl.n_layers - 1:
            break                      # the last layer's output never reaches the cache
        h = h + _attn_out(attention(q, k, v, causal_offset=P0), W, layer)
        xn = numerics.bf16_round(rmsnorm(h, W.get("ffn_norm", layer), wl.rms_eps))
        y, info = moe(xn.reshape(B * P, -1), W, layer)
        if routing is not None:
            routing.append(info["ids"])
        h = h + y.reshape(B, P, -1)
    return cache


def given_prompt_cache(wl: synth.Workload, P=None):
    """The precomputed bf16 prompt cache of a workload whose cache is an input."""
    return [(bf16_bits_to_f64(synth.prompt_kv_bf16(wl, layer, "k", P)),
             bf16_bits_to_f64(synth.prompt_kv_bf16(wl, layer, "v", P))) for layer in range(wl.n_layers)]


class DecoderPass:
    """L_t = Decoder(x_t, z_t = 0, H) for canvases tok [B][C] given the prompt
    cache, as a sequence of pieces run in order: piece 2l is layer l's attention
    block (h += Attn(RMSNorm(h))), piece 2l + 1 its MoE block (h += MoE(RMSNorm(h))),
    piece 2L the final norm and the tied LM head.  Running every piece in order
    is exactly decoder_logits; the pieces exist so that a bounded share of one
    pass can be timed on its own."""

    def __init__(self, W: Weights, tok, cache, rows=None, forced_ids=None, z=None):
        self.W = W
        self.wl = W.wl
        self.tok = np.asarray(tok)
        self.B, self.C = self.tok.shape
        self.cache = cache
        self.P = cache[0][0].shape[2]
        self.pos = self.P + np.arange(self.C)
        self.rows = rows
        self.forced_ids = forced_ids    # optional per-layer [B*C][k] expert ids (see route)
        self.h = W.embed_rows(self.tok)
        if z is not None:               # self-conditioning state z_t (oracle.self_cond), added to the embedding
            self.h = self.h + np.asarray(z, dtype=np.float64).reshape(self.h.shape)
        self.margins, self.route_ids, self.route_logits = [], [], []
        self.logits = None
        self.hn = None

    @property
    def n_pieces(self) -> int:
        return 2 * self.wl.n_layers + 1

    def run_piece(self, i: int) -> None:
        wl, W = self.wl, self.W
        if i == 2 * wl.n_layers:
            self._head()
            return
        layer = i // 2
        if i % 2 == 0:
            xn = numerics.bf16_round(rmsnorm(self.h, W.get("attn_norm", layer), wl.rms_eps))
            q, k, v = _qkv(xn, W, layer, self.pos)
            k_all = np.concatenate([self.cache[layer][0], k], axis=2)
            v_all = np.concatenate([self.cache[layer][1], v], axis=2)
            self.h = self.h + _attn_out(attention(q, k_all, v_all, causal_offset=None), W, layer)
        else:
            xn = numerics.bf16_round(rmsnorm(self.h, W.get("ffn_norm", layer), wl.rms_eps))
            forced = None if self.forced_ids is None else self.forced_ids[layer]
            y, info = moe(xn.reshape(self.B * self.C, -1), W, layer, forced)
            self.margins.append(info["margin"])
            self.route_ids.append(info["ids"])
            self.route_logits.append(info["router_logits"])
            self.h = self.h + y.reshape(self.B, self.C, -1)

    def _head(self) -> None:
        wl, W = self.wl, self.W
        hn = numerics.bf16_round(rmsnorm(self.h, W.get("final_norm"), wl.rms_eps))
        self.hn = hn
        if self.rows is None:
            flat = hn.reshape(self.B * self.C, -1)
        else:
            flat = np.stack([hn[b, i] for b, i in self.rows])
        logits = np.empty((flat.shape[0], wl.vocab))
        for r0, E in W.embed_chunks():
            logits[:, r0:r0 + E.shape[0]] = flat @ E.T
        if self.rows is None:
            logits = logits.reshape(self.B, self.C, wl.vocab)
        self.logits = logits

    def diag(self, final_hidden=False):
        d = {"margin": self.margins, "ids": self.route_ids, "router_logits": self.route_logits}
        if final_hidden:
            d["hn"] = self.hn
        return d


def decoder_logits(W: Weights, tok, cache, rows=None, final_hidden=False, z=None):
    """L_t = Decoder(x_t, z_t = 0, H) for canvases tok [B][C] given the prompt cache.

    rows: optional list of (b, i) canvas positions whose logits are returned
    (the LM head is per row); default all, as [B][C][V].  Returns (logits, diag)
    with, per layer, diag['margin'] (router k-th minus (k+1)-th logit [B*C]),
    diag['ids'] (top-k expert ids [B*C][k]) and diag['router_logits'] [B*C][E]."""
    dp = DecoderPass(W, tok, cache, rows, z=z)
    for i in range(dp.n_pieces):
        dp.run_piece(i)
    return dp.logits, dp.diag(final_hidden)
