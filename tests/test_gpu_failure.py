"""Failure detection and checkpoint / resume, on the GPU, without a fault.

* A bounded device wait that runs out: a test hook raises the target of the
  routing launch's grid barrier by one, so the barrier can never complete; its
  wait gives up after its time limit (about 2 s), records the error and leaves
  every buffer index in bounds.  dgen_synchronize must report DGEN_EDEVICE, and
  the next step (hook cleared) must run normally and give the same logits as
  before, bit for bit: the context stays usable.
* Checkpoint / resume: a block interrupted after step 5, its canvas state
  (tokens, committed flags) exported to the host and loaded into a fresh handle
  that ran the same prompt pass, finishes with the same canvas as the block run
  without interruption.
"""
import numpy as np
import pytest

import synth
from oracle import sampler as osamp
from tests.helpers import make_denoiser

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

WL = synth.WORKLOADS["tiny"]


def _step_logits(den, tok):
    B, C, V = WL.batch, WL.canvas, WL.vocab
    den.set_canvas(torch.from_numpy(tok.reshape(-1).astype(np.int32)).cuda(), None)
    logits = torch.empty(B * C * V, dtype=torch.float32, device="cuda")
    den.denoise_step(0, WL.steps, logits)
    return logits


def test_a_wait_that_runs_out_is_reported_and_the_context_stays_usable():
    import block_denoising_step_b200 as dg
    from synth.device import device_prompt
    den = make_denoiser(WL)
    den.prefill_prompt(device_prompt(WL))
    tok = osamp.init_canvas(WL.seed, WL.batch, WL.canvas, WL.vocab)
    ref = _step_logits(den, tok)
    den.synchronize()
    ref = ref.cpu().numpy()
    den.set_tuning(dg.Denoiser.TUNE_ROUTE_BARRIER_EXTRA, 1)
    _step_logits(den, tok)
    with pytest.raises(dg.DgenError) as e:
        den.synchronize()
    assert e.value.status == dg.DGEN_EDEVICE
    den.set_tuning(dg.Denoiser.TUNE_ROUTE_BARRIER_EXTRA, 0)
    again = _step_logits(den, tok)
    den.synchronize()                      # no error left behind
    assert np.array_equal(again.cpu().numpy(), ref)
    den.close()


def test_checkpoint_and_resume_in_a_fresh_handle():
    from synth.device import device_weights, device_prompt
    B, C, T = WL.batch, WL.canvas, WL.steps
    weights = device_weights(WL, "cuda")
    prompt = device_prompt(WL)
    t = torch.empty(B * C, dtype=torch.int32, device="cuda")
    c = torch.empty(B * C, dtype=torch.uint8, device="cuda")

    a = make_denoiser(WL, weights=weights)
    a.prefill_prompt(prompt)
    a.init_canvas(WL.seed)
    for s in range(T):
        a.denoise_step(s, T, None)
        a.sample_commit(s, T, WL.seed)
    a.get_canvas(t, None)
    a.synchronize()
    whole = t.cpu().numpy().copy()

    a.prefill_prompt(prompt)
    a.init_canvas(WL.seed)
    for s in range(6):
        a.denoise_step(s, T, None)
        a.sample_commit(s, T, WL.seed)
    a.get_canvas(t, c)
    a.synchronize()
    saved_tok, saved_com = t.cpu().numpy().copy(), c.cpu().numpy().copy()     # host checkpoint
    a.close()

    b = make_denoiser(WL, weights=weights)
    b.prefill_prompt(prompt)
    b.set_canvas(torch.from_numpy(saved_tok).cuda(), torch.from_numpy(saved_com).cuda())
    for s in range(6, T):
        b.denoise_step(s, T, None)
        b.sample_commit(s, T, WL.seed)
    b.get_canvas(t, c)
    b.synchronize()
    assert np.array_equal(t.cpu().numpy(), whole)
    assert c.cpu().numpy().all()
    b.close()
