"""The entropy-bounded sampler with adaptive stopping (dgen_sample_commit_eb)
against the oracle (oracle/eb_sampler.py) on the same fp32 logits.

Inputs are built so that the outcome is decided far from rounding: every row
gets a peak of a different height over N(0, 1) logits, so the entropies are
spread out, and gamma sits in the middle of a gap between two consecutive
prefix bounds of every canvas.  Then entropies agree to fp32 accuracy and the
integer outputs (tokens, commit flags, stop flags) are equal."""
import numpy as np
import pytest

import synth
from oracle import eb_sampler as eb
from oracle.sampler import tau_of_step

WL = synth.WORKLOADS["tiny"].replace(batch=2, canvas=200)   # two canvases, ragged C
T_MAX, SEED = 48, 2024


def make_logits(step: int):
    B, C, V = WL.batch, WL.canvas, WL.vocab
    L = synth.logits_f32(SEED, 300 + step, B * C, V, std=1.0)
    rng = np.random.default_rng(step)
    heights = 1.0 + 11.0 * rng.permutation(B * C) / (B * C)          # distinct peak heights
    cols = synth.uniform_i32(SEED, 40 + step, 0, B * C, V)
    L[np.arange(B * C), cols] += heights.astype(np.float32)
    return L.astype(np.float32)


def pick_gamma(H, committed, margin=1e-3):
    """A gamma between two consecutive prefix bounds of every canvas, at least
    `margin` from each; None if no such value exists."""
    bounds = []
    for b in range(H.shape[0]):
        h = np.sort(H[b][~committed[b]])
        bounds.append(np.concatenate([[0.0], np.cumsum(h)]))
    for j in range(6, 60):
        lo, hi = bounds[0][j - 1], bounds[0][j]
        g = 0.5 * (lo + hi)
        if all(np.min(np.abs(bd - g)) > margin for bd in bounds):
            return float(g)
    return None


def test_inputs_decide_far_from_rounding():
    """Premise of the GPU test (no GPU): entropies of each canvas differ by more than
    fp32 error and a robust gamma exists at each step."""
    B, C = WL.batch, WL.canvas
    committed = np.zeros((B, C), dtype=bool)
    committed[:, ::7] = True
    for s in range(3):
        H, _ = eb.entropy_rows(make_logits(s).astype(np.float64).reshape(B, C, -1), tau_of_step(s, T_MAX))
        for b in range(B):   # the order that decides acceptance: the lowest open entropies
            h = np.sort(H[b][~committed[b]])[:64]
            assert np.min(np.diff(h)) > 1e-5
        assert pick_gamma(H, committed) is not None


@pytest.mark.gpu
def test_eb_steps_match_the_oracle_and_stop_on_an_unchanged_canvas():
    torch = pytest.importorskip("torch")
    from tests.helpers import make_denoiser
    B, C, V = WL.batch, WL.canvas, WL.vocab
    den = make_denoiser(WL)
    tok = synth.uniform_i32(SEED, 7, 0, B * C, V).reshape(B, C).astype(np.int64)
    committed = np.zeros((B, C), dtype=bool)
    committed[:, ::7] = True
    tok[committed] = 5
    den.set_canvas(torch.from_numpy(tok.reshape(-1).astype(np.int32)).cuda(),
                   torch.from_numpy(committed.reshape(-1).astype(np.uint8)).cuda())
    ent = torch.empty(B * C, dtype=torch.float32, device="cuda")
    stop = torch.empty(B, dtype=torch.uint8, device="cuda")
    t_dev = torch.empty(B * C, dtype=torch.int32, device="cuda")
    c_dev = torch.empty(B * C, dtype=torch.uint8, device="cuda")
    prev_arg = None
    for s in range(3):
        L = make_logits(s)
        tau = tau_of_step(s, T_MAX)
        H64, arg = eb.entropy_rows(L.astype(np.float64).reshape(B, C, V), tau)
        gamma = pick_gamma(H64, committed)
        ref_tok, ref_com, info = eb.sample_commit_eb(L.astype(np.float64).reshape(B, C, V), tok, committed, s,
                                                     T_MAX, SEED, tau, gamma)
        ref_stop = eb.should_stop(info["entropy"], info["argmax"], prev_arg, 0.0)
        den.sample_commit_eb(torch.from_numpy(L.reshape(-1)).cuda(), s, T_MAX, SEED, gamma, 0.0, ent, stop)
        den.get_canvas(t_dev, c_dev)
        den.synchronize()
        h = ent.cpu().numpy().reshape(B, C)
        assert np.max(np.abs(h - H64) / (1.0 + H64)) < 1e-4, f"step {s}: entropy"
        assert np.array_equal(t_dev.cpu().numpy().reshape(B, C), ref_tok), f"step {s}: tokens"
        assert np.array_equal(c_dev.cpu().numpy().reshape(B, C).astype(bool), ref_com), f"step {s}: commits"
        assert np.array_equal(stop.cpu().numpy().astype(bool), ref_stop)
        assert info["new"].sum(axis=1).min() >= 6           # gamma admits more than the first position
        tok, committed, prev_arg = ref_tok, ref_com, info["argmax"]
    # the same logits again with a stop threshold above the mean entropy: argmax unchanged -> stop,
    # every open position takes its argmax
    L = make_logits(2)
    tau = tau_of_step(3, T_MAX)
    H64, arg = eb.entropy_rows(L.astype(np.float64).reshape(B, C, V), tau)
    den.sample_commit_eb(torch.from_numpy(L.reshape(-1)).cuda(), 3, T_MAX, SEED, 1e-6, float(H64.mean()) + 1.0,
                         ent, stop)
    den.get_canvas(t_dev, c_dev)
    den.synchronize()
    assert stop.cpu().numpy().all()
    assert c_dev.cpu().numpy().all()
    want = np.where(committed, tok, arg)
    assert np.array_equal(t_dev.cpu().numpy().reshape(B, C), want)
    den.close()


def _device_state(den, B, C):
    t = torch_mod().empty(B * C, dtype=torch_mod().int32, device="cuda")
    c = torch_mod().empty(B * C, dtype=torch_mod().uint8, device="cuda")
    den.get_canvas(t, c)
    den.synchronize()
    return t.cpu().numpy().reshape(B, C).astype(np.int64), c.cpu().numpy().reshape(B, C).astype(bool)


def torch_mod():
    import torch
    return torch


@pytest.mark.gpu
@pytest.mark.parametrize("freeze", [True, False])
def test_hot_path_eb_steps_match_the_oracle_on_the_device_logits(freeze):
    """The production entropy-bounded step reads the LM-head epilogue's statistics
    (no stored logits).  Teacher-forced on the device's own state at every step,
    its entropies (relative 1e-4), tokens, commit flags and stop flags equal the
    oracle's block step on the fp32 logits the same step stored, except where an
    accepted prefix's bound lies within 1e-3 of gamma (a near-tie, counted; the
    step is then not compared further)."""
    torch = torch_mod()
    from tests.helpers import make_denoiser
    from synth.device import device_prompt
    B, C, V = WL.batch, WL.canvas, WL.vocab
    den = make_denoiser(WL)
    den.prefill_prompt(device_prompt(WL))
    den.init_canvas(SEED)
    gamma, thr = 40.0, 0.5
    ent = torch.empty(B * C, dtype=torch.float32, device="cuda")
    stop = torch.empty(B, dtype=torch.uint8, device="cuda")
    logits = torch.empty(B * C * V, dtype=torch.float32, device="cuda")
    done = np.zeros(B, dtype=bool)
    prev_arg = None
    near = 0
    for s in range(6):
        tok, committed = _device_state(den, B, C)
        den.denoise_step(s, T_MAX, logits)
        den.sample_commit_eb(None, s, T_MAX, SEED, gamma, thr, ent, stop, freeze=freeze)
        t_dev, c_dev = _device_state(den, B, C)
        L = logits.cpu().numpy().astype(np.float64).reshape(B, C, V)
        tau = tau_of_step(s, T_MAX)
        ref_tok, ref_com, ref_done, ref_stop, info = eb.block_step_eb(L, tok, committed, done, prev_arg, s, T_MAX,
                                                                      SEED, tau, gamma, thr, freeze)
        H = ent.cpu().numpy().reshape(B, C)
        assert np.max(np.abs(H - info["entropy"]) / np.maximum(1.0, info["entropy"])) < 1e-4
        assert np.array_equal(stop.cpu().numpy().astype(bool), ref_stop)
        for b in range(B):
            if np.array_equal(c_dev[b], ref_com[b]):
                assert np.array_equal(t_dev[b], ref_tok[b]), (s, b)
            else:   # only at a near-tie of a prefix bound with gamma
                cand = ~committed[b] if freeze else np.ones(C, dtype=bool)
                h = np.sort(info["entropy"][b][cand])
                bounds = np.concatenate([[0.0], np.cumsum(h)])
                assert np.min(np.abs(bounds - gamma)) < 1e-3, (s, b)
                near += 1
        done, prev_arg = ref_done, info["argmax"]
    print(f"hot-path entropy-bounded steps (freeze={freeze}): near-tie differences {near}")
    den.close()


@pytest.mark.gpu
@pytest.mark.parametrize("freeze", [True, False])
def test_block_loop_equals_the_step_by_step_calls(freeze):
    """dgen_generate_block_eb (device stop flags read by the host loop) gives the
    same canvas, bit for bit, and the same step counts as driving
    dgen_denoise_step + dgen_sample_commit_eb from the host."""
    torch = torch_mod()
    from tests.helpers import make_denoiser
    from synth.device import device_prompt
    B, C = WL.batch, WL.canvas
    den = make_denoiser(WL)
    prompt = device_prompt(WL)
    gamma, thr, t_max = 300.0, 0.5, 10
    out = torch.empty(B * C, dtype=torch.int32, device="cuda")
    steps = den.generate_block_eb(prompt, t_max, SEED, gamma, thr, out, freeze=freeze)
    den.synchronize()
    # the same calls from the host
    den.prefill_prompt(prompt)
    den.init_canvas(SEED)
    stop = torch.empty(B, dtype=torch.uint8, device="cuda")
    done = np.zeros(B, dtype=bool)
    want = np.zeros(B, dtype=np.int64)
    for s in range(t_max):
        den.denoise_step(s, t_max, None)
        den.sample_commit_eb(None, s, t_max, SEED, gamma, thr, None, stop, freeze=freeze)
        _, c = _device_state(den, B, C)
        now = stop.cpu().numpy().astype(bool) | (s == t_max - 1) | (c.all(axis=1) if freeze else False)
        want[now & ~done] = s + 1
        done |= now
        if done.all():
            break
    tok, _ = _device_state(den, B, C)
    assert np.array_equal(out.cpu().numpy().reshape(B, C), tok)
    assert list(want) == steps
    print(f"block loop (freeze={freeze}, gamma={gamma}): steps per canvas {steps}")
    den.close()


@pytest.mark.gpu
def test_given_logits_leave_the_step_statistics_alone():
    """dgen_sample_commit_eb on given logits, called between dgen_denoise_step and
    dgen_sample_commit (even with another step budget), changes nothing that
    dgen_sample_commit reads: its confidences and canvas are the same as without it."""
    torch = torch_mod()
    from tests.helpers import make_denoiser
    from synth.device import device_prompt
    B, C, V = WL.batch, WL.canvas, WL.vocab
    den = make_denoiser(WL)
    den.prefill_prompt(device_prompt(WL))
    tok = synth.uniform_i32(SEED, 8, 0, B * C, V).astype(np.int32)
    tok_d = torch.from_numpy(tok).cuda()
    results = []
    for interpose in (False, True):
        den.set_canvas(tok_d, None)
        den.denoise_step(4, 12, None)
        if interpose:
            den.sample_commit_eb(torch.from_numpy(make_logits(1).reshape(-1)).cuda(), 30, 48, SEED, 5.0, 0.0)
            den.set_canvas(tok_d, None)
        conf = torch.empty(B * C, dtype=torch.float32, device="cuda")
        den.sample_commit(4, 12, SEED, conf)
        results.append((conf.cpu().numpy(), _device_state(den, B, C)[0]))
    assert np.array_equal(results[0][0], results[1][0]) and np.array_equal(results[0][1], results[1][1])
    # a misaligned logits pointer is rejected before any launch
    import block_denoising_step_b200 as dg
    L = torch.empty(B * C * V + 4, dtype=torch.float32, device="cuda")
    with pytest.raises(dg.DgenError) as e:
        den.sample_commit_eb(L.data_ptr() + 4, 0, 48, SEED, 1.0, 0.0)
    assert e.value.status == dg.DGEN_EINVAL
    den.close()
