"""Self-conditioning on the device against the oracle (hyper.ai digest of the
DiffusionGemma paper, Method, eqs. 3-4: L_t = Decoder(x_t, z_t, H), z_{t-dt} =
FFW(p0_hat E), p0_hat = Softmax(L_t / tau_t)).

* Each stage given its identical inputs (the device's own intermediates, read
  back): p0_hat from the pass's own logits (bf16, elementwise within one ulp,
  elements rounded the other way at most 5 in 1000: exp2 and the row sum in
  fp32 against fp64), u = p0_hat E (the K-split
  GEMM over the vocabulary with the embedding read MN-major; relative L2
  1e-4), the normed u (bf16 within one ulp) and the FFW activations (within
  one ulp plus the fp32 summation bound of their gate and up sums,
  tests.helpers.gated_activation_check), z = act W_d^T (relative L2 1e-5).
* The whole state: z from the device's own logits against
  oracle.self_cond.next_state of those logits (relative L2 within max(1e-3,
  twice the oracle's own sensitivity to an fp32 rounding of the logits)).
* A step with a given state: the oracle's z for a canvas, given to both sides
  (dgen_set_self_cond), with the oracle's routing forced: the logits within
  tests.helpers.end_to_end_bar.
* Two steps threaded: step 0 from z = 0, the device commits; the state the
  device carries out of step 0 against the oracle on its step-0 logits, and
  step 1 on the device's canvas with that carried state against the oracle's
  step 1 given the same state: logits within the end-to-end bar.
* State semantics: the canvas calls clear z (a step after dgen_set_canvas or
  dgen_set_self_cond(NULL) reproduces the z = 0 logits bit for bit), z changes
  the next step, whole blocks are deterministic and keep the block invariants.
"""
import numpy as np
import pytest

import synth
from oracle import decoder, numerics, sampler as osamp, self_cond as osc
from tests.helpers import make_denoiser, rel_l2, oracle_prompt_routing, end_to_end_bar, gated_activation_check

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

CASES = {
    "tiny": synth.WORKLOADS["tiny"].replace(self_cond_width=512),
    # ragged row count (2 x 200 canvas rows), narrow FFW
    "tiny_ragged": synth.WORKLOADS["tiny"].replace(batch=2, canvas=200, prompt_len=50, self_cond_width=256),
    # the full-scale shapes (d 2816, V 262144, FFW width 2112 = the shared FFN's), two layers
    "full2": synth.WORKLOADS["full"].replace(n_layers=2, self_cond_width=2112),
}
SENS = {"tiny": "tiny", "tiny_ragged": "tiny", "full2": "full"}


def _bf16(t):
    return t.view(torch.int16).cpu().numpy().astype(np.uint16).astype(np.uint32).__lshift__(16).view(np.float32) \
        .astype(np.float64)


def _read(den, which, n, dtype, part=0):
    t = torch.empty(n, dtype=dtype, device="cuda")
    den.debug_read(which, part, t)
    den.synchronize()
    return t


def _sum_parts(den, which, n):
    """Sum (in index order) of the K-split partials `which` (23: u, 26: z)."""
    import block_denoising_step_b200 as dg
    acc, i = None, 0
    while True:
        try:
            t = _read(den, which, n, torch.float32, i)
        except dg.DgenError:
            break
        acc = t.clone() if acc is None else acc + t
        i += 1
    assert i >= 1
    return acc.cpu().numpy().astype(np.float64), i


def _close_bf16(got, ref, atol):
    """Share of elements that differ; asserts none differs by more than one bf16
    ulp (2^-7 of the value) plus atol."""
    diff = np.abs(got - ref)
    bad = diff > 2.0 ** -7 * np.abs(ref) + atol
    assert not bad.any(), (int(bad.sum()), float(np.max(diff - 2.0 ** -7 * np.abs(ref))))
    return float(np.mean(diff > 0))


@pytest.fixture(scope="module", params=list(CASES))
def case(request):
    name = request.param
    wl = CASES[name]
    from synth.device import device_prompt
    W = decoder.Weights(wl)
    prompt = synth.prompt_tokens(wl)
    cache, p_ids = oracle_prompt_routing(W, prompt)
    den = make_denoiser(wl)
    den.force_routing(torch.from_numpy(p_ids.reshape(-1)).cuda(), None)
    den.prefill_prompt(device_prompt(wl))
    den.synchronize()
    den.force_routing(None, None)
    yield name, wl, W, cache, den
    den.close()


def _step(den, wl, tok, s, z=None, ids=None, keep_z=False):
    """One device step on canvas tok with state z (None: zero; keep_z: the
    handle's current state) and optionally forced canvas routing; fp32 logits."""
    R, V = wl.batch * wl.canvas, wl.vocab
    if not keep_z:
        den.set_canvas(torch.from_numpy(np.asarray(tok).reshape(-1).astype(np.int32)).cuda(), None)
        if z is not None:
            den.set_self_cond(torch.from_numpy(np.ascontiguousarray(z, dtype=np.float32).reshape(-1)).cuda())
    if ids is not None:
        den.force_routing(None, torch.from_numpy(np.ascontiguousarray(ids, dtype=np.int32).reshape(-1)).cuda())
    logits = torch.empty(R * V, dtype=torch.float32, device="cuda")
    den.denoise_step(s, wl.steps, logits)
    den.synchronize()
    if ids is not None:
        den.force_routing(None, None)
    return logits.cpu().numpy().reshape(R, V).astype(np.float64)


def test_each_stage_given_its_device_inputs(case):
    name, wl, W, cache, den = case
    B, C, V, d, w = wl.batch, wl.canvas, wl.vocab, wl.d_model, wl.self_cond_width
    R = B * C
    s, T = 3, wl.steps
    tok = osamp.init_canvas(wl.seed + 11, B, C, V)
    L = _step(den, wl, tok, s)
    tau = osamp.tau_of_step(s, T, wl.tau_max, wl.tau_min)
    p = _bf16(_read(den, 22, R * V, torch.bfloat16)).reshape(R, V)
    u, ks = _sum_parts(den, 23, R * d)
    u = u.reshape(R, d)
    n = _bf16(_read(den, 24, R * d, torch.bfloat16)).reshape(R, d)
    act = _bf16(_read(den, 25, R * w, torch.bfloat16)).reshape(R, w)
    z, kz = _sum_parts(den, 26, R * d)
    z = z.reshape(R, d)
    # p0_hat of the device's own logits
    p_ref = numerics.bf16_round(numerics.softmax(L / tau, axis=-1))
    fp = _close_bf16(p, p_ref, 0.0)
    # u = p0_hat E on the device's p0_hat
    u_ref = np.zeros((R, d))
    for r0, E in W.embed_chunks():
        u_ref += p[:, r0:r0 + E.shape[0]] @ E
    eu = rel_l2(u, u_ref)
    # the FFW's pre-norm on the device's u, its activations on the device's n, z on the device's activations
    n_ref = numerics.bf16_round(numerics.rmsnorm(u, W.get("sc_norm"), wl.rms_eps))
    fn = _close_bf16(n, n_ref, 0.0)
    w_g, w_u = decoder.split_gate_up(W.get("w_sc_gate_up"))
    fa = gated_activation_check(act, n @ w_g.T, n @ w_u.T, np.abs(n) @ np.abs(w_g).T, np.abs(n) @ np.abs(w_u).T, d)
    ez = rel_l2(z, act @ W.get("w_sc_down").T)
    print(f"self-cond {name}: p0_hat {fp:.1e} of elements one bf16 ulp off; u ({ks} K splits) rel-L2 {eu:.1e}; "
          f"norm {fn:.1e}, activations {fa:.1e} of elements one ulp off; z ({kz} K splits) rel-L2 {ez:.1e}")
    assert fp <= 5e-3 and eu <= 1e-4 and fn <= 1e-3 and fa <= 1e-2 and ez <= 1e-5
    # the whole state against the oracle on the device's logits
    ez_all, bar = state_vs_oracle(W, L, tau, z)
    print(f"self-cond {name}: z against oracle next_state of the device logits: rel-L2 {ez_all:.1e} (bar {bar:.1e})")
    assert ez_all <= bar


def state_vs_oracle(W, L, tau, z):
    """(relative L2 of the device state z against oracle.self_cond.next_state of
    the logits L, its bar).  The bar is max(1e-3, 2 s_z), s_z being the oracle's
    own sensitivity: how far its next_state moves when L is multiplied by
    (1 + 2^-24 xi), one fp32 rounding (xi standard normal, seeded); the device
    works in fp32 before each of the chain's bf16 roundings (p0_hat, the normed
    u, the activations), so its state cannot be expected closer than that."""
    ref = osc.next_state(W, L, tau).reshape(z.shape)
    xi = np.random.default_rng(12345).standard_normal(L.shape)
    moved = osc.next_state(W, L * (1.0 + 2.0 ** -24 * xi), tau).reshape(z.shape)
    return rel_l2(z, ref), max(1e-3, 2.0 * rel_l2(moved, ref))


def test_step_with_a_given_state_matches_oracle(case):
    name, wl, W, cache, den = case
    B, C, V = wl.batch, wl.canvas, wl.vocab
    tok0 = osamp.init_canvas(wl.seed + 12, B, C, V)
    tau0 = osamp.tau_of_step(0, wl.steps, wl.tau_max, wl.tau_min)
    L0, _ = decoder.decoder_logits(W, tok0, cache)
    z = osc.next_state(W, L0.reshape(B * C, V), tau0)
    tok1 = osamp.init_canvas(wl.seed + 13, B, C, V)
    ref, diag = decoder.decoder_logits(W, tok1, cache, z=z)
    ref = ref.reshape(B * C, V)
    got = _step(den, wl, tok1, 1, z=z, ids=np.stack(diag["ids"]))
    err = rel_l2(got, ref)
    # how far z moves the logits (the device's z = 0 step on the same canvas and routing)
    moved = rel_l2(_step(den, wl, tok1, 1, ids=np.stack(diag["ids"])), ref)
    print(f"self-cond {name}: step with the oracle's z (forced routing): rel-L2 {err:.2e}; the same step without "
          f"z differs by {moved:.2e}")
    assert err <= end_to_end_bar(SENS[name])
    assert moved > 1e-3  # the state is not negligible


def test_two_threaded_steps_match_oracle(case):
    """Step 0 from z = 0 (forced routing), the device commits; the state the
    device carried out of step 0 (read back) against the oracle's next_state of
    the device's step-0 logits (state_vs_oracle); then step 1 on the device's
    committed canvas with the device's own carried state against the oracle's
    step 1 given that same state: the state is carried, and used, as the pages
    say.  (Each side on its own state would add the two sides' step-0 logit
    difference, amplified by the tempered softmax, to the step-1 comparison.)"""
    name, wl, W, cache, den = case
    B, C, V, T, d = wl.batch, wl.canvas, wl.vocab, wl.steps, wl.d_model
    R = B * C
    seed = wl.seed + 14
    tok0 = osamp.init_canvas(seed, B, C, V)
    L0_ref, d0 = decoder.decoder_logits(W, tok0, cache)
    L0_ref = L0_ref.reshape(R, V)
    L0 = _step(den, wl, tok0, 0, ids=np.stack(d0["ids"]))
    z1, _ = _sum_parts(den, 26, R * d)
    den.sample_commit(0, T, seed)
    t1 = torch.empty(R, dtype=torch.int32, device="cuda")
    den.get_canvas(t1, None)
    den.synchronize()
    tok1 = t1.cpu().numpy().reshape(B, C)
    ez, bar_z = state_vs_oracle(W, L0, osamp.tau_of_step(0, T, wl.tau_max, wl.tau_min), z1.reshape(R, d))
    ref, d1 = decoder.decoder_logits(W, tok1, cache, z=z1.reshape(B, C, d))
    ref = ref.reshape(R, V)
    got = _step(den, wl, tok1, 1, ids=np.stack(d1["ids"]), keep_z=True)   # the device's own carried state
    e0, e1 = rel_l2(L0, L0_ref), rel_l2(got, ref)
    print(f"self-cond {name}: threaded steps (forced routing): step 0 rel-L2 {e0:.2e}; carried state against the "
          f"oracle on the device's step-0 logits {ez:.1e} (bar {bar_z:.1e}); step 1 with that state {e1:.2e}")
    assert e0 <= end_to_end_bar(SENS[name]) and e1 <= end_to_end_bar(SENS[name]) and ez <= bar_z


def test_state_is_cleared_by_the_canvas_calls(case):
    name, wl, W, cache, den = case
    B, C, V = wl.batch, wl.canvas, wl.vocab
    tok = osamp.init_canvas(wl.seed + 15, B, C, V)
    a = _step(den, wl, tok, 2)                 # set_canvas: z = 0
    b = _step(den, wl, tok, 2, keep_z=True)    # z from the step before
    c = _step(den, wl, tok, 2)                 # set_canvas clears it again
    den.set_self_cond(None)
    d = _step(den, wl, tok, 2, keep_z=True)
    assert np.array_equal(a, c) and np.array_equal(a, d)
    assert rel_l2(b, a) > 1e-4


@pytest.mark.parametrize("T", [12])
def test_blocks_with_self_conditioning(case, T):
    """Whole blocks (prompt pass, T steps with z threaded): deterministic, every
    position committed, committed tokens never change."""
    from tests.test_gpu_fullscale import block_properties
    name, wl, W, cache, den = case
    block_properties(wl.replace(steps=T), T, den)
