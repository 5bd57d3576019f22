"""FP8 (E4M3) experts through the C ABI (dgen_config.expert_fp8 = 1) against the
oracle's FP8 path (oracle/fp8.py: E4M3 with power-of-two row scales for the
expert and shared-FFN weights, the expert inputs and the gated activations).

* Given identical quantized operands (read back from the device), the FP8
  expert GEMMs equal the oracle's FP8 formulas up to fp32 summation, and the
  quantizations are bit-exact: the arithmetic of the FP8 path itself.
* Layer-wise teacher forcing and the forced-routing step: E4M3 rounding points
  turn a small difference of their inputs (a bf16 rounding that goes the other
  way upstream) into a jump on a grid 16 times coarser than bf16's, so the
  oracle's own FP8 path moves several times more than its bf16 path under the
  same small perturbation (tests/golden/fp8_amplification.json, written by
  tests/golden/make_fp8_amplification.py from the oracle alone); the bf16 bars
  are scaled by that measured ratio."""
import numpy as np
import pytest

import synth
from oracle import decoder, sampler as osamp
from oracle import numerics
from tests.helpers import (make_denoiser, load_prompt_cache, rel_l2, gpu_step_forced, oracle_prompt_routing,
                           layerwise_parity, end_to_end_bar, gated_activation_check)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

CASES = {
    "tiny": synth.WORKLOADS["tiny"].replace(expert_fp8=True),
    "medium": synth.WORKLOADS["medium"].replace(expert_fp8=True),
    # the full-scale shapes (shared FFN of three expert widths, 128 experts top-8), cut to 2 layers
    "full2": synth.WORKLOADS["full"].replace(n_layers=2, prompt_len=256, expert_fp8=True),
}
SENS = {"tiny": "tiny", "medium": "medium", "full2": "full"}


def amplification(name):
    import json
    import os
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "fp8_amplification.json")
    return json.load(open(path))[name]["ratio"]


@pytest.mark.parametrize("name", list(CASES))
def test_fp8_step_matches_the_fp8_oracle(name):
    import block_denoising_step_b200 as dg
    wl = CASES[name]
    B, C, V = wl.batch, wl.canvas, wl.vocab
    W = decoder.Weights(wl)
    cache, p_ids = oracle_prompt_routing(W, synth.prompt_tokens(wl))
    tok = osamp.init_canvas(wl.seed, B, C, V)
    ref, diag = decoder.decoder_logits(W, tok, cache)
    den = make_denoiser(wl)
    from synth.device import device_prompt
    den.force_routing(torch.from_numpy(p_ids.reshape(-1)).cuda(), None)
    den.prefill_prompt(device_prompt(wl))
    den.synchronize()
    den.force_routing(None, None)
    got, ids, _ = gpu_step_forced(den, wl, tok, 0, np.stack(diag["ids"]))
    # the routed chunks in expert id order instead of largest expert first (the
    # automatic order of the two-launch E4M3 experts): the same logits bit for bit
    den.set_tuning(dg.Denoiser.TUNE_CHUNK_ORDER, 1)
    got_id, _, _ = gpu_step_forced(den, wl, tok, 0, np.stack(diag["ids"]))
    den.set_tuning(dg.Denoiser.TUNE_CHUNK_ORDER, 0)
    assert np.array_equal(got, got_id)
    err = rel_l2(got, ref.reshape(B * C, V))
    upd, full, err_logits = layerwise_parity(den, wl, osamp.init_canvas(wl.seed + 5, B, C, V), 2)
    amp = amplification(name)
    print(f"fp8 {name}: forced-routing step rel-L2 {err:.2e} (bar {amp * end_to_end_bar(SENS[name]):.1e}); layer-wise "
          f"update rel-L2 max {max(upd):.2e} (bar {amp * 1e-2:.1e}), logits {err_logits:.2e}; FP8/bf16 amplification "
          f"{amp:.1f}")
    den.close()
    assert np.isfinite(got).all()
    assert err <= amp * end_to_end_bar(SENS[name])
    assert max(upd) <= amp * 1e-2 and err_logits <= 1e-2


def test_fp8_block_runs_and_commits_everything():
    """A whole block with FP8 experts at the full-scale single-canvas sizes: every
    position committed, committed tokens frozen, deterministic."""
    from tests.test_gpu_fullscale import block_properties
    block_properties(synth.WORKLOADS["full"].replace(expert_fp8=True), 12)


def _rd(den, which, n, dtype):
    t = torch.empty(n, dtype=dtype, device="cuda")
    den.debug_read(which, 0, t)
    den.synchronize()
    return t


def _e4m3(t):
    return t.view(torch.float8_e4m3fn).to(torch.float64).cpu().numpy()


def _bf16(t):
    return t.view(torch.int16).cpu().numpy().astype(np.uint16).astype(np.uint32).__lshift__(16).view(np.float32) \
        .astype(np.float64)


@pytest.mark.parametrize("name", ["tiny", "full2"])
def test_fp8_expert_gemms_are_exact_given_their_quantized_inputs(name):
    """The FP8 analogue of "given identical bf16-rounded inputs": the quantized
    operands the device fed its expert GEMMs in the last layer (E4M3 token rows
    and scales, the routed and shared gated activations) are read back; the
    quantizations of the activations are bit-exact against oracle.fp8.quant_rows
    of the device's own bf16 activations, and every GEMM output -- the routed
    gate-up activations, the routed down outputs (gated), the shared FFN's
    activations and slice outputs -- equals the oracle's FP8 formulas on those
    operands up to fp32 summation: fp32 outputs within relative L2 1e-5, bf16
    activations elementwise within one bf16 ulp plus the fp32 summation bound of
    their gate and up sums (tests.helpers.gated_activation_check: where a sum
    cancels, an fp32 vs fp64 difference may move a small activation by more than
    its ulp), with differing elements at most 1 in 100."""
    from oracle import fp8
    wl = CASES[name]
    W = decoder.Weights(wl)
    B, C, V, L, k, w, d, E = wl.batch, wl.canvas, wl.vocab, wl.n_layers, wl.top_k, wl.expert_width, wl.d_model, \
        wl.n_experts
    R = B * C
    den = make_denoiser(wl)
    from synth.device import device_prompt
    den.prefill_prompt(device_prompt(wl))
    tok = osamp.init_canvas(wl.seed + 5, B, C, V)
    ids = torch.empty(L * R * k, dtype=torch.int32, device="cuda")
    den.capture_routing(ids, None)
    den.set_canvas(torch.from_numpy(tok.reshape(-1).astype(np.int32)).cuda(), None)
    logits = torch.empty(R * V, dtype=torch.float32, device="cuda")
    den.denoise_step(0, wl.steps, logits)
    den.synchronize()
    den.capture_routing(None, None)
    last = ids.cpu().numpy().reshape(L, R, k)[L - 1]
    act = _bf16(_rd(den, 8, R * k * w, torch.bfloat16)).reshape(R * k, w)
    act8 = _e4m3(_rd(den, 9, R * k * w, torch.uint8)).reshape(R * k, w)
    sact = _rd(den, 10, R * k, torch.float32).cpu().numpy().astype(np.float64)
    xp8 = _e4m3(_rd(den, 11, R * k * d, torch.uint8)).reshape(R * k, d)
    sxp = _rd(den, 12, R * k, torch.float32).cpu().numpy().astype(np.float64)
    ptok = _rd(den, 13, R * k, torch.int32).cpu().numpy()
    y = _rd(den, 14, R * k * d, torch.float32).cpu().numpy().astype(np.float64).reshape(R * k, d)
    gate = _rd(den, 15, R * k, torch.float32).cpu().numpy().astype(np.float64)
    q, s = fp8.quant_rows(act)
    assert np.array_equal(act8, q) and np.array_equal(sact, s)
    cnt = np.bincount(last.reshape(-1), minlength=E)
    off = np.concatenate([[0], np.cumsum(cnt)])
    ea, ey = 0.0, 0.0
    for e in range(E):
        rows = np.arange(off[e], off[e + 1])
        if rows.size == 0:
            continue
        assert all(e in last[t] for t in ptok[rows])
        gq, gs = W.get_fp8("w_gate_up", L - 1, e)
        dq, ds = W.get_fp8("w_down", L - 1, e)
        wg, wu = decoder.split_gate_up(gq)
        sg, su = decoder.split_gate_up(gs[:, None])
        sc_g = sxp[rows][:, None] * sg[:, 0][None, :]
        sc_u = sxp[rows][:, None] * su[:, 0][None, :]
        g, u = (xp8[rows] @ wg.T) * sc_g, (xp8[rows] @ wu.T) * sc_u
        ga, ua = (np.abs(xp8[rows]) @ np.abs(wg).T) * sc_g, (np.abs(xp8[rows]) @ np.abs(wu).T) * sc_u
        ea = max(ea, gated_activation_check(act[rows], g, u, ga, ua, d))
        y_ref = (act8[rows] @ dq.T) * sact[rows][:, None] * ds[None, :] * gate[rows][:, None]
        ey = max(ey, rel_l2(y[rows], y_ref))
    msg = (f"fp8 {name} exact-input check: routed gate-up {ea:.1e} of elements off by one bf16 ulp, routed down "
           f"rel-L2 {ey:.1e}")
    if wl.shared_width:
        ws, nsh = wl.shared_width, -(-wl.shared_width // w)
        wp = -(-w // 128) * 128
        ash = _bf16(_rd(den, 16, R * ws, torch.bfloat16)).reshape(R, ws)
        ash8 = _e4m3(_rd(den, 17, R * nsh * wp, torch.uint8)).reshape(R, nsh, wp)
        sash = _rd(den, 18, R, torch.float32).cpu().numpy().astype(np.float64)
        xn8 = _e4m3(_rd(den, 19, R * d, torch.uint8)).reshape(R, d)
        sxn = _rd(den, 20, R, torch.float32).cpu().numpy().astype(np.float64)
        ysh = _rd(den, 21, nsh * R * d, torch.float32).cpu().numpy().astype(np.float64).reshape(nsh, R, d)
        qs, ss = fp8.quant_rows(ash)
        assert np.array_equal(ash8[:, :, :w].reshape(R, nsh * w)[:, :ws], qs) and np.array_equal(sash, ss)
        assert not ash8[:, :, w:].any()                                   # the padding stays zero
        gq, gs = W.get_fp8("w_shared_gate_up", L - 1)
        dq, ds = W.get_fp8("w_shared_down", L - 1)
        wg, wu = decoder.split_gate_up(gq)
        sg, su = decoder.split_gate_up(gs[:, None])
        sc_g, sc_u = sxn[:, None] * sg[:, 0][None, :], sxn[:, None] * su[:, 0][None, :]
        g, u = (xn8 @ wg.T) * sc_g, (xn8 @ wu.T) * sc_u
        ga, ua = (np.abs(xn8) @ np.abs(wg).T) * sc_g, (np.abs(xn8) @ np.abs(wu).T) * sc_u
        esa = gated_activation_check(ash, g, u, ga, ua, d)
        esy = max(rel_l2(ysh[j], (qs[:, j * w:(j + 1) * w] @ dq[:, j * w:(j + 1) * w].T) * ss[:, None] * ds[None, :])
                  for j in range(nsh))
        msg += f", shared gate-up {esa:.1e} of elements off by one bf16 ulp, shared down slices {esy:.1e}"
        assert esa <= 1e-2 and esy <= 1e-5
    print(msg)
    den.close()
    assert ea <= 1e-2 and ey <= 1e-5
