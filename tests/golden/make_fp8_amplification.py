"""Writes tests/golden/fp8_amplification.json: how much more the FP8 expert path
of the oracle amplifies a small input difference than its bf16 path.

For each workload, one step on a fixed canvas is run by the oracle (oracle/
only) and, layer by layer from the same layer input (teacher forcing, the same
expert choices), once more with the attention output multiplied by
(1 + 2^-16 z), z ~ N(0, 1) (numpy seed 0) before its bf16 rounding -- the
precision of a P.V product that keeps about 16 significant bits of P.  The
largest relative L2 change of a layer's update of the residual stream is
recorded for the bf16 path and for the FP8 path (E4M3 experts, oracle/fp8.py),
and their ratio: each E4M3 rounding point turns a difference into one about
sqrt(2^-4 / 2^-8) = 4 times larger than a bf16 rounding point does, and the
measured ratio says how much that compounds through a layer.  The FP8 device
comparisons scale their bf16 bars by this ratio.

Usage: python tests/golden/make_fp8_amplification.py [tiny medium full2]
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import synth  # noqa: E402
from oracle import decoder, sampler  # noqa: E402

OUT = os.path.join(HERE, "fp8_amplification.json")
WORKLOADS = {"tiny": synth.WORKLOADS["tiny"], "medium": synth.WORKLOADS["medium"],
             "full2": synth.WORKLOADS["full"].replace(n_layers=2, prompt_len=256)}


def layer_change(wl) -> float:
    W = decoder.Weights(wl)
    cache = decoder.prefill(W, synth.prompt_tokens(wl))
    tok = sampler.init_canvas(wl.seed + 5, wl.batch, wl.canvas, wl.vocab)
    dp = decoder.DecoderPass(W, tok, cache)
    h_in, upd = [], []
    for layer in range(wl.n_layers):
        h_in.append(dp.h.copy())
        dp.run_piece(2 * layer)
        dp.run_piece(2 * layer + 1)
        upd.append(dp.h - h_in[-1])
    rng = np.random.default_rng(0)
    plain = decoder.attention

    def perturbed(q, k, v, causal_offset=None):
        o = plain(q, k, v, causal_offset)
        return o * (1.0 + 2.0 ** -16 * rng.standard_normal(o.shape)) if causal_offset is None else o

    decoder.attention = perturbed
    try:
        worst = 0.0
        for layer in range(wl.n_layers):
            dq = decoder.DecoderPass(W, tok, cache, forced_ids=dp.route_ids)
            dq.h = h_in[layer].copy()
            dq.run_piece(2 * layer)
            dq.run_piece(2 * layer + 1)
            worst = max(worst, float(np.linalg.norm((dq.h - h_in[layer]) - upd[layer]) / np.linalg.norm(upd[layer])))
    finally:
        decoder.attention = plain
    return worst


def main(names):
    data = json.load(open(OUT)) if os.path.exists(OUT) else {}
    for n in names:
        b = layer_change(WORKLOADS[n])
        f = layer_change(WORKLOADS[n].replace(expert_fp8=True))
        data[n] = {"bf16_layer_change": b, "fp8_layer_change": f, "ratio": f / b}
        print(n, data[n], flush=True)
        with open(OUT, "w") as fh:
            json.dump(data, fh, indent=1, sort_keys=True)


if __name__ == "__main__":
    main(sys.argv[1:] or list(WORKLOADS))
