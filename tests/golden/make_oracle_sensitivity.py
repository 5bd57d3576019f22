"""Writes tests/golden/oracle_sensitivity.json: how far the fp64 oracle's own
logits move when its residual stream is perturbed at fp32 rounding level.

For each workload, one teacher-forced step on the initial canvas (s = 0) is run
twice by the oracle (oracle/ only): as it stands, and with the residual stream
h multiplied by (1 + 2^-24 z), z ~ N(0, 1) drawn per element (numpy seed 0),
after every attention block and every MoE block -- the size of one fp32
rounding of h, which an fp32 implementation incurs at every residual add.  The
relative L2 distance between the two runs' logits measures how much the
workload's chain of bf16 rounding points, router gates and attention over many
nearly uniform random keys amplifies perturbations of that size: no
implementation that keeps h in fp32 can be expected to come closer to the fp64
oracle than about this.  The file also records, for the same pair of runs, the
largest router-logit difference over rows whose routing has not flipped yet,
the largest oracle margin at which a row's routing first flips, and how many
rows flip.  The batched workload uses sequence 0 (its sequences
are independent); workloads with a given cache use it, the others the oracle's
prompt pass.

Usage: python tests/golden/make_oracle_sensitivity.py [workload ...]
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import synth  # noqa: E402
from oracle import decoder, sampler  # noqa: E402

OUT = os.path.join(HERE, "oracle_sensitivity.json")


def sensitivity(name: str) -> dict:
    """{'logits_rel_l2', 'router_logit_diff_max', 'first_flip_margin_max', 'flipped_rows', 'rows'}
    of the perturbed run against the plain one (router-logit differences over
    the rows whose routing has not flipped yet, layer by layer)."""
    wl = synth.WORKLOADS[name]
    if wl.batch > 1:
        wl = wl.replace(batch=1, prompt_kv_given=True)
    W = decoder.Weights(wl)
    cache = decoder.given_prompt_cache(wl) if wl.prompt_kv_given else decoder.prefill(W, synth.prompt_tokens(wl))
    tok = sampler.init_canvas(wl.seed, wl.batch, wl.canvas, wl.vocab)
    ref, diag = decoder.decoder_logits(W, tok, cache)
    rng = np.random.default_rng(0)
    dp = decoder.DecoderPass(W, tok, cache)
    for i in range(dp.n_pieces):
        dp.run_piece(i)
        if i < 2 * wl.n_layers:
            dp.h = dp.h * (1.0 + 2.0 ** -24 * rng.standard_normal(dp.h.shape))
    a, b = dp.logits.reshape(-1, wl.vocab), ref.reshape(-1, wl.vocab)
    flipped = np.zeros(a.shape[0], dtype=bool)
    dr, margins = 0.0, []
    for l in range(wl.n_layers):
        differ = np.any(np.sort(dp.route_ids[l], axis=1) != np.sort(diag["ids"][l], axis=1), axis=1)
        keep = ~flipped
        if keep.any():
            dr = max(dr, float(np.abs(dp.route_logits[l] - diag["router_logits"][l])[keep].max()))
        margins += [float(diag["margin"][l][r]) for r in np.nonzero(differ & ~flipped)[0]]
        flipped |= differ
    return {"logits_rel_l2": float(np.linalg.norm(a - b) / np.linalg.norm(b)), "router_logit_diff_max": dr,
            "first_flip_margin_max": max(margins) if margins else 0.0, "flipped_rows": int(flipped.sum()),
            "rows": int(a.shape[0])}


def main(names):
    data = json.load(open(OUT)) if os.path.exists(OUT) else {}
    for n in names:
        data[n] = sensitivity(n)
        print(n, data[n], flush=True)
        with open(OUT, "w") as f:
            json.dump(data, f, indent=1, sort_keys=True)


if __name__ == "__main__":
    main(sys.argv[1:] or ["tiny", "medium", "long_prompt", "full", "full_batched"])
