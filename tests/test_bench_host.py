"""Host-side arithmetic of bench.py (no GPU): byte and flop accounting of the
roofline objects, and the bounded oracle sample's scaling."""
import math

import synth


def test_lm_head_tensor_figure():
    import bench
    wl = synth.WORKLOADS["full"]
    flop = 2 * 256 * 262144 * 2816
    r = bench.lm_head_tensor(wl, lm_ms=0.5 * 3, lm_n=3, peak_tflops=1000.0)
    assert r["flop_per_launch"] == flop
    assert math.isclose(r["achieved"], flop / 0.5e-3 / 1e12)
    assert math.isclose(r["frac"], r["achieved"] / 1000.0)
    assert bench.lm_head_tensor(wl, 0.0, 0, 1000.0) is None


def test_gate_up_bytes_count_touched_experts_and_the_shared_ffn():
    import bench
    wl = synth.WORKLOADS["full"]
    n, k, d, w, ws = 256, 8, 2816, 704, 2112
    touched = 50.0
    want = (touched * 2 * w * d * 2 + n * k * d * 2 + n * k * w * 2) + (2 * ws * d * 2 + n * d * 2 + n * ws * 2)
    assert math.isclose(bench.expert_gate_up_bytes(wl, touched), want)
    med = synth.WORKLOADS["medium"]                    # no shared FFN
    n, k, d, w = 256, 4, 1024, 1024
    assert math.isclose(bench.expert_gate_up_bytes(med, 32.0), 32 * 2 * w * d * 2 + n * k * d * 2 + n * k * w * 2)


def test_step_bytes_with_every_expert_touched_are_the_weights_plus_the_prompt_kv():
    import bench
    wl = synth.WORKLOADS["full"]
    kv = wl.n_layers * wl.batch * wl.n_kv_heads * (wl.prompt_len + wl.canvas) * wl.head_dim * 2 * 2
    assert bench.step_bytes(wl, float(wl.n_experts)) == 2 * wl.param_count() + kv


def test_job_throughput_counts_every_replica():
    import bench
    wl = synth.WORKLOADS["full"]
    assert math.isclose(bench.job_tokens_per_s(1, wl, 600, 5.6), 256 * 600 / 12 / 5.6)
    assert math.isclose(bench.job_tokens_per_s(4, wl, 600, 5.6), 4 * 256 * 600 / 12 / 5.6)


def test_uniform_routing_spreads_rows_evenly_with_distinct_experts_per_row():
    import numpy as np
    import bench
    wl = synth.WORKLOADS["full"]
    ids = bench.uniform_routing(wl)
    assert ids.shape == (wl.n_layers, 256, 8)
    assert all(len(set(r)) == 8 for r in ids[0])
    counts = np.bincount(ids[0].reshape(-1), minlength=wl.n_experts)
    assert counts.min() == counts.max() == 256 * 8 // 128


def test_oracle_step_pieces_are_the_oracle_step():
    """The reference arm's pieces, run in order, are exactly the oracle's step
    (decoder pass + sampler) on the same canvas and cache."""
    import numpy as np
    import bench
    from oracle import decoder, pipeline, sampler
    wl = synth.WORKLOADS["tiny"].replace(n_layers=2, canvas=32, prompt_len=16, steps=4)
    st = bench.OracleStep(wl)
    W = decoder.Weights(wl)
    cache = decoder.given_prompt_cache(wl)
    tok = sampler.init_canvas(wl.seed, wl.batch, wl.canvas, wl.vocab)
    com = np.zeros_like(tok, dtype=bool)
    for s in range(2):
        _, tok, com, _ = pipeline.denoise_step(W, cache, tok, com, s, wl.steps, wl.seed)
        finished = [st.run_piece() for _ in range(st.pieces_per_step)]
        assert finished == [False] * (st.pieces_per_step - 1) + [True]
        assert np.array_equal(st.tok, tok) and np.array_equal(st.committed, com)


def test_reference_arm_reports_the_requested_steps(capsys):
    import json
    import bench

    class Args:
        gpus, steps, warmup = 1, 3, 2

    wl = synth.WORKLOADS["tiny"].replace(n_layers=1, canvas=32, prompt_len=16)
    bench.reference_arm(Args(), wl, rank=0)
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["steps"] == 3 and line["warmup"] == 2
    assert line["value"] > 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert "1 whole oracle step" in line["cpu_baseline"]["sample"]


def test_down_bytes_and_step_flops():
    import bench
    wl = synth.WORKLOADS["full"]
    n, k, d, w, ws = 256, 8, 2816, 704, 2112
    want = (50 * d * w * 2 + n * k * w * 2 + n * k * d * 4) + (d * ws * 2 + n * ws * 2 + 3 * n * d * 4)
    assert math.isclose(bench.expert_down_bytes(wl, 50.0), want)
    f = bench.step_flops(wl)
    assert 2.0e12 < f < 2.4e12            # about 2.2 TFLOP per full-scale step


def test_fp8_byte_accounting_halves_the_expert_weights():
    import bench
    wl = synth.WORKLOADS["full"]
    w8 = wl.replace(expert_fp8=True)
    kv = wl.n_layers * wl.batch * wl.n_kv_heads * (wl.prompt_len + wl.canvas) * wl.head_dim * 2 * 2
    expert_params = wl.n_layers * (128 * 3 * 704 + 3 * 2112) * 2816
    assert bench.step_bytes(w8, 128.0) == 2 * wl.param_count() - expert_params + kv
    assert bench.expert_gate_up_bytes(w8, 50.0) < 0.6 * bench.expert_gate_up_bytes(wl, 50.0)


def test_self_cond_line_counts_the_logits_probabilities_embedding_and_ffw():
    """The self-conditioning block's algorithmic bytes: the fp32 logits read, p0_hat
    written and read in bf16, the embedding read once by p0_hat E, the FFW's three
    weight matrices; flops: p0_hat E and the FFW's three GEMMs (2 per multiply-add)."""
    import bench
    wl = synth.WORKLOADS["full"].replace(self_cond_width=2112)
    n, V, d, w = 256, 262144, 2816, 2112
    line = bench.self_cond_line(wl, {"ms": 0.5, "launches": 6}, 6534.5, 1631.9, 8.5)
    assert line["hbm_bytes"] == 4 * n * V + 4 * n * V + 2 * V * d + 6 * w * d
    assert line["flops"] == 2 * n * V * d + 6 * n * w * d
    assert math.isclose(line["share_of_step"], 0.5 / 8.5)
    assert math.isclose(line["hbm_frac"], line["hbm_bytes"] / 0.5e-3 / 1e9 / 6534.5)
    # no self-conditioning, or no timed launch: no line
    assert bench.self_cond_line(synth.WORKLOADS["full"], {"ms": 0.5, "launches": 6}, 1, 1, 1) is None
    assert bench.self_cond_line(wl, {"ms": 0.0, "launches": 0}, 1, 1, 1) is None
