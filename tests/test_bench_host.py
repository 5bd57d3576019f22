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
