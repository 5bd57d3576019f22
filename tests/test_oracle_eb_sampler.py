"""Pins of the oracle's entropy-bounded sampler (the pages' own sampler; no GPU).

Each pin checks the oracle against something other than itself: closed forms
of the entropy, scipy's entropy routine, the cumulative-sum form of the
acceptance rule, the one-hot special case, and the invariants the hyper.ai
digest's Method section states (rank order by entropy, frozen commits,
stopping only on two identical consecutive argmax canvases)."""
import math

import numpy as np
import pytest

from oracle import eb_sampler as eb


def test_entropy_closed_forms():
    V = 4096
    H, _ = eb.entropy_rows(np.zeros((3, V)), tau=0.7)          # uniform
    assert np.allclose(H, math.log(V), rtol=0, atol=1e-12)
    L = np.zeros((1, V))
    L[0, 17] = 1e4                                               # one-hot in the limit
    H, arg = eb.entropy_rows(L, tau=0.5)
    assert H[0] < 1e-12 and arg[0] == 17
    # one logit a above V-1 equal ones: p1 = e^(a/tau) / (e^(a/tau) + V - 1)
    a, tau, V = 3.0, 0.8, 1000
    L = np.zeros((1, V))
    L[0, 5] = a
    p1 = math.exp(a / tau) / (math.exp(a / tau) + V - 1)
    q = (1 - p1) / (V - 1)
    want = -p1 * math.log(p1) - (V - 1) * q * math.log(q)
    H, _ = eb.entropy_rows(L, tau)
    assert abs(H[0] - want) < 1e-12


def test_entropy_matches_scipy():
    scipy_stats = pytest.importorskip("scipy.stats")
    rng = np.random.default_rng(3)
    L = rng.normal(0, 3, size=(16, 257))
    tau = 0.55
    H, arg = eb.entropy_rows(L, tau)
    z = L / tau
    p = np.exp(z - z.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    assert np.allclose(H, scipy_stats.entropy(p, axis=1), rtol=1e-12, atol=1e-12)
    assert np.array_equal(arg, np.argmax(L, axis=1))


def test_accept_count_is_the_longest_prefix_whose_smaller_entropies_sum_below_gamma():
    rng = np.random.default_rng(7)
    for trial in range(200):
        n = int(rng.integers(1, 40))
        h = np.sort(rng.exponential(0.5, size=n))
        gamma = float(rng.uniform(0.01, 5.0))
        # bound of the first k = sum of the k - 1 smallest; longest k with bound < gamma
        prefix = np.concatenate([[0.0], np.cumsum(h)])[:n]   # bound of k = 1..n
        want = int(np.max(np.nonzero(prefix < gamma)[0])) + 1
        assert eb.accept_count(list(h), gamma) == want
    assert eb.accept_count([], 1.0) == 0
    assert eb.accept_count([0.3, 0.4, 2.0], 1e-9) == 1          # the first is always accepted
    assert eb.accept_count([0.3, 0.4, 2.0], 1e9) == 3


def test_accept_count_grows_with_gamma():
    h = list(np.sort(np.random.default_rng(1).exponential(1.0, size=30)))
    counts = [eb.accept_count(h, g) for g in np.linspace(0.01, 20, 50)]
    assert all(a <= b for a, b in zip(counts, counts[1:]))


def test_step_accepts_in_entropy_order_and_freezes_commits():
    rng = np.random.default_rng(11)
    B, C, V, T = 2, 64, 97, 48
    tok = rng.integers(0, V, size=(B, C))
    committed = np.zeros((B, C), dtype=bool)
    for s in range(6):
        L = rng.normal(0, 2, size=(B, C, V)) * rng.uniform(0.2, 4, size=(B, C, 1))
        prev_tok, prev_com = tok.copy(), committed.copy()
        tok, committed, info = eb.sample_commit_eb(L, tok, committed, s, T, seed=5, tau=0.6, gamma=0.8)
        assert np.array_equal(tok[prev_com], prev_tok[prev_com])          # frozen
        assert np.all(committed[prev_com])
        for b in range(B):
            new = info["new"][b]
            assert new.sum() >= 1 or prev_com[b].all()
            assert np.array_equal(tok[b, new], info["argmax"][b, new])
            open_prev = ~prev_com[b]
            rest = open_prev & ~new
            if new.any() and rest.any():                                   # rank order
                assert info["entropy"][b, new].max() <= info["entropy"][b, rest].min()
            h = np.sort(info["entropy"][b, new])
            assert h[:-1].sum() < 0.8                                      # the bound holds


def test_one_hot_logits_finish_in_one_step_and_stop_on_the_second():
    B, C, V = 1, 32, 64
    target = np.random.default_rng(2).integers(0, V, size=(B, C))
    calls = []

    def step_logits(s, tok):
        calls.append(s)
        L = np.full((B, C, V), -50.0)
        np.put_along_axis(L, target[..., None], 50.0, axis=2)
        return L

    tok0 = np.zeros((B, C), dtype=np.int64)
    out, steps = eb.generate_block_eb(step_logits, tok0, seed=1, gamma=0.5, stop_threshold=0.1)
    assert np.array_equal(out, target)
    assert steps[0] == 1 and calls == [0]       # every entropy ~0: all accepted at once


def test_stop_needs_low_entropy_and_two_equal_argmax_canvases():
    H = np.array([[0.1, 0.2], [0.1, 0.2]])
    a = np.array([[1, 2], [3, 4]])
    assert not eb.should_stop(H, a, None, 1.0).any()
    assert eb.should_stop(H, a, a.copy(), 1.0).all()
    b = a.copy()
    b[1, 0] = 9
    assert list(eb.should_stop(H, a, b, 1.0)) == [True, False]
    assert not eb.should_stop(H, a, a.copy(), 0.15).any()      # mean 0.15 is not below 0.15


def test_adaptive_stop_halts_before_the_step_budget():
    """Constant, peaked-but-not-one-hot logits: entropies are low and equal, the
    argmax canvas does not change, so the block stops on the second step with
    every open position set to its argmax."""
    rng = np.random.default_rng(4)
    B, C, V = 2, 40, 50
    L0 = rng.normal(0, 1, size=(B, C, V))
    L0[np.arange(B)[:, None], np.arange(C)[None, :], rng.integers(0, V, size=(B, C))] += 12.0
    out, steps = eb.generate_block_eb(lambda s, tok: L0, rng.integers(0, V, size=(B, C)), seed=3,
                                      gamma=1e-6, stop_threshold=0.5, T_max=48)
    assert np.all(steps == 2)
    assert np.array_equal(out, np.argmax(L0, axis=2))


def test_unfrozen_step_can_revise_an_earlier_choice():
    """freeze=False (every position a candidate each step): a position accepted at
    step 0 whose entropy rises at step 1 drops out of the accepted prefix and is
    redrawn, while with freeze=True it stays committed."""
    B, C, V, T = 1, 8, 32, 48
    rng = np.random.default_rng(3)
    peaks = rng.integers(0, V, size=C)
    L0 = np.zeros((B, C, V))
    L0[0, np.arange(C), peaks] = np.linspace(30, 2, C)          # position 0 most confident
    tok0 = rng.integers(0, V, size=(B, C))
    com0 = np.zeros((B, C), dtype=bool)
    t1, c1, i1 = eb.sample_commit_eb(L0, tok0, com0, 0, T, seed=9, tau=0.6, gamma=1e-3, freeze=False)
    assert c1[0, 0] and t1[0, 0] == peaks[0]
    L1 = L0.copy()
    L1[0, 0] = 0.0                                                # position 0 now uniform: highest entropy
    t2, c2, i2 = eb.sample_commit_eb(L1, t1, c1, 1, T, seed=9, tau=0.6, gamma=1e-3, freeze=False)
    assert not c2[0, 0]                                           # revised: redrawn
    tf, cf, _ = eb.sample_commit_eb(L1, t1, c1, 1, T, seed=9, tau=0.6, gamma=1e-3, freeze=True)
    assert cf[0, 0] and tf[0, 0] == peaks[0]                      # frozen: kept


def test_unfrozen_block_on_one_hot_logits_stops_on_the_second_step():
    """With every entropy ~0 all positions are accepted at step 0; unfrozen, the
    block is done only by the stop test, which holds at step 1 (unchanged
    argmax canvas, mean entropy below the threshold)."""
    B, C, V = 2, 24, 64
    target = np.random.default_rng(6).integers(0, V, size=(B, C))
    L = np.full((B, C, V), -50.0)
    np.put_along_axis(L, target[..., None], 50.0, axis=2)
    out, steps = eb.generate_block_eb(lambda s, tok: L, np.zeros((B, C), dtype=np.int64), seed=1, gamma=0.5,
                                      stop_threshold=0.1, freeze=False)
    assert np.array_equal(out, target) and np.all(steps == 2)


def test_a_done_canvas_is_left_unchanged():
    """Canvas 0 stops at step 1 (constant peaked logits); canvas 1's logits keep
    changing, so it goes on; canvas 0's tokens never change afterwards."""
    rng = np.random.default_rng(12)
    B, C, V = 2, 20, 40
    base = rng.normal(0, 1, size=(B, C, V))
    base[0, np.arange(C), rng.integers(0, V, size=C)] += 15.0

    def step_logits(s, tok):
        L = base.copy()
        L[1] = rng.normal(0, 1, size=(C, V))                      # canvas 1: new noise every step
        return L

    seen = []

    def spy(s, tok):
        seen.append(np.array(tok[0]))
        return step_logits(s, tok)

    out, steps = eb.generate_block_eb(spy, rng.integers(0, V, size=(B, C)), seed=2, gamma=0.05,
                                      stop_threshold=0.5, freeze=False, T_max=8)
    assert steps[0] == 2 and steps[1] == 8
    for t in seen[2:]:
        assert np.array_equal(t, seen[2])
    assert np.array_equal(out[0], np.argmax(base[0], axis=1))
