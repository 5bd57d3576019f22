"""Pins of the FP8 (E4M3) expert path of the oracle (oracle/fp8.py), no GPU."""
import numpy as np
import pytest
import torch

import synth
from oracle import decoder, fp8, numerics


def _all_bf16_within(limit):
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    v = numerics.bf16_bits_to_f64(bits)
    return v[np.isfinite(v) & (np.abs(v) <= limit)]


def test_e4m3_rounding_matches_torch_float8_e4m3fn():
    """Every finite bf16 value in [-448, 448], and random fp64 values, round to the
    same E4M3 value as torch's float8_e4m3fn conversion (round to nearest even)."""
    v = np.concatenate([_all_bf16_within(448.0),
                        np.random.default_rng(0).uniform(-448, 448, 200000),
                        np.random.default_rng(1).normal(0, 1e-2, 200000)])
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(fp8.e4m3_round(v), ref)


def test_row_scales_are_the_smallest_fitting_powers_of_two():
    rng = np.random.default_rng(2)
    x = rng.normal(0, 1, size=(64, 300)) * np.exp2(rng.integers(-20, 20, size=(64, 1)))
    x[3] = 0.0
    x[5, 7] = 448.0 * 2.0 ** -3          # max exactly 448 * 2^-3 -> scale 2^-3
    x[5, 8:] = 0.0
    x[5, :7] = 1.0
    q, s = fp8.quant_rows(x)
    assert np.array_equal(np.log2(s), np.round(np.log2(s)))            # powers of two
    assert s[3] == 1.0 and s[5] == 2.0 ** -3
    amax = np.max(np.abs(q), axis=1)
    live = np.max(np.abs(x), axis=1) > 0
    assert np.all(amax <= 448.0) and np.all(amax[live] >= 224.0)        # half the range at least
    # reconstruction within half an E4M3 ulp (relative 2^-4) for normal values
    rec = q * s[:, None]
    big = np.abs(x / s[:, None]) >= 2.0 ** -6
    assert np.all(np.abs(rec - x)[big] <= 2.0 ** -4 * np.abs(x)[big] + 1e-300)


def test_fp8_ffn_places_the_scales_like_a_dequantized_evaluation():
    """The FP8 FFN equals the plain fp64 evaluation on dequantized operands, with
    every quantization step done by torch's float8_e4m3fn conversion instead of
    oracle.fp8 (a transposed or misplaced scale breaks it)."""
    rng = np.random.default_rng(3)
    n, d, w = 5, 64, 32
    x = numerics.bf16_round(rng.normal(0, 1, size=(n, d)))
    gu = numerics.bf16_round(rng.normal(0, 0.05, size=(2 * w, d)) * np.exp2(rng.integers(-3, 3, size=(2 * w, 1))))
    dn = numerics.bf16_round(rng.normal(0, 0.05, size=(d, w)))

    def tq(a, s):
        return torch.from_numpy(a / s[:, None]).to(torch.float8_e4m3fn).to(torch.float64).numpy() * s[:, None]

    sx, sgu, sdn = fp8.row_scale(x), fp8.row_scale(gu), fp8.row_scale(dn)
    xd, gud, dnd = tq(x, sx), tq(gu, sgu), tq(dn, sdn)
    w_g, w_u = decoder.split_gate_up(gud)
    a = numerics.bf16_round(numerics.gelu_tanh(xd @ w_g.T) * (xd @ w_u.T))
    ref = tq(a, fp8.row_scale(a)) @ dnd.T
    got = fp8.expert_ffn_fp8(*fp8.quant_rows(x), fp8.quant_rows(gu), fp8.quant_rows(dn))
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_fp8_ffn_stays_within_its_quantization_noise_of_the_bf16_ffn():
    """Relative L2 distance to the bf16 FFN of the same weights: three E4M3
    roundings (input, weights, activation), each about 2^-4 / sqrt(3) relative
    RMS, give several percent -- far below the O(1) error of a wrong scale -- and
    not zero (quantization happens)."""
    rng = np.random.default_rng(4)
    n, d, w = 16, 256, 128
    x = numerics.bf16_round(rng.normal(0, 1, size=(n, d)))
    gu = numerics.bf16_round(rng.normal(0, 0.02, size=(2 * w, d)))
    dn = numerics.bf16_round(rng.normal(0, 0.02, size=(d, w)))
    ref = decoder.expert_ffn(x, gu, dn)
    got = fp8.expert_ffn_fp8(*fp8.quant_rows(x), fp8.quant_rows(gu), fp8.quant_rows(dn))
    err = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert 1e-3 < err < 0.12


def test_fp8_moe_equals_dense_masked_fp8_evaluation():
    """The routed FP8 MoE equals evaluating every expert in FP8 on every row and
    masking by the gates (routing is the same as on the bf16 path)."""
    wl = synth.WORKLOADS["tiny"].replace(n_layers=1, d_model=128, n_experts=4, top_k=2, expert_width=64,
                                         shared_width=64, expert_fp8=True)
    W = decoder.Weights(wl)
    xn = numerics.bf16_round(np.random.default_rng(5).normal(0, 1, size=(12, 128)))
    y, info = decoder.moe(xn, W, 0)
    xq, sx = fp8.quant_rows(xn)
    dense = np.zeros_like(xn)
    for e in range(4):
        ye = fp8.expert_ffn_fp8(xq, sx, W.get_fp8("w_gate_up", 0, e), W.get_fp8("w_down", 0, e))
        g = np.zeros(12)
        for j in range(2):
            g += np.where(info["ids"][:, j] == e, info["gates"][:, j], 0.0)
        dense += g[:, None] * ye
    dense += fp8.expert_ffn_fp8(xq, sx, W.get_fp8("w_shared_gate_up", 0), W.get_fp8("w_shared_down", 0))
    assert np.allclose(y, dense, rtol=1e-12, atol=1e-12)
    y16, _ = decoder.moe(xn, decoder.Weights(wl.replace(expert_fp8=False)), 0)
    assert not np.allclose(y, y16)
