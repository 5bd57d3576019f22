"""Benchmark of the block denoising step: canvas tokens/s per 256-token block (T = 12).

One bench step = one pass of the whole hot path over the workload's batch: a
decoder pass (dgen_denoise_step: attention over [prompt cache ; canvas], routed
MoE, LM head with fused softmax statistics) followed by the sampler
(dgen_sample_commit).  Steps cycle s = 0..T-1 through the canvas state machine
(a fresh Philox canvas at s = 0), so K steps process K / T blocks:

    value = n_gpus * B * C * K / (T * t_max)      [canvas tokens/s, whole job]

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]
N > 1 runs under torch.distributed.run, one replica per GPU (independent
canvases, no collective on the data path; the barrier and the max over ranks
of the elapsed time are the only collectives).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "canvas tokens/s per 256-token block (T=12)"
UNIT = "tokens/s"
DEFAULT_WORKLOAD = "full"


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=600)
    p.add_argument("--warmup", type=int, default=24)
    p.add_argument("--workload", default=DEFAULT_WORKLOAD)
    p.add_argument("--layers", type=int, default=0,
                   help="profiling aid: cut the workload's model to this many layers (named in config)")
    p.add_argument("--prompt", type=int, default=0, help="profiling aid: prompt length override")
    p.add_argument("--impl", default="native", choices=["native", "reference"])
    p.add_argument("--e2e-blocks", type=int, default=3)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--breakdown", action="store_true",
                   help="after the timed region, time every kernel class over one more step "
                        "(events around each launch) and report ms and launches per class")
    p.add_argument("--flags", type=int, default=0, help="dgen_set_flags value (1 no graph, 2 no PDL)")
    p.add_argument("--gemm-per-sm", action="store_true",
                   help="per-SM streaming rate and fixed cost of the GEMM core (one JSON line per case)")
    p.add_argument("--gemm-streaming", action="store_true",
                   help="measure the GEMM core's weight-streaming rate (tile variants) and cuBLAS on the same shapes")
    return p.parse_args()


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the timed region runs."""

    FIELDS = "timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown," \
             "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown," \
             "clocks_event_reasons.sw_power_cap"

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        """Starts sampling (every 50 ms); call well before the timed region."""
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        self.t0 = self.t1 = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark_start(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    def stop(self):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for t, l in self.lines:
            if self.t0 is not None and not (self.t0 <= t <= (self.t1 or t)):
                continue                    # only samples taken during the timed region
            f = [x.strip() for x in l.split(",")]
            if len(f) < 8:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------- accounting

# ----------------------------------------------------------------------------- replicas (N > 1)
# Each rank is an independent replica: its own canvases (Philox seed offset by
# the rank), no collective on the data path.  The only collectives are the
# barriers around the timed region and the max over ranks of elapsed times.

def replica_seed(wl, rank: int) -> int:
    """Philox seed of rank `rank`'s canvases (distinct per rank)."""
    return wl.seed + 1000 * rank


def max_over_ranks(x: float, world: int, device=None) -> float:
    """Max of x over the ranks of the default process group (x itself when
    world == 1).  device: where the reduction tensor lives (the rank's GPU for
    NCCL, None = CPU for gloo)."""
    if world <= 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(world: int, wl, steps: int, elapsed_max: float) -> float:
    """Whole-job canvas tokens/s: every rank processes B*C tokens per block,
    one block per T steps; time = the slowest rank's."""
    return world * wl.batch * wl.canvas * steps / (wl.steps * elapsed_max)


def lm_head_tensor(wl, lm_ms: float, lm_n: int, peak_tflops: float):
    """Tensor-pipe figure of the LM-head GEMM (N = B*C rows x V x d, 2 flop per
    multiply-add) from its CUDA-event time: achieved TFLOP/s and the fraction of
    the measured dense bf16 peak; None when the launch was not timed."""
    if not lm_n or lm_ms <= 0.0:
        return None
    flop = 2.0 * wl.batch * wl.canvas * wl.vocab * wl.d_model
    achieved = flop / (lm_ms / lm_n / 1e3) / 1e12
    return {"kernel": "LM head (tcgen05 GEMM + softmax-statistics epilogue)", "bound": "tensor",
            "achieved": achieved, "peak": peak_tflops, "unit": "TFLOP/s", "frac": achieved / peak_tflops,
            "flop_per_launch": flop}


def expert_gate_up_bytes(wl, touched: float) -> float:
    """Algorithmic HBM bytes of one grouped gate-up launch: the gate and up
    weights of the experts routed to (touched, averaged over the layers, read
    from the library), the routed token rows in, the activations out; plus the
    shared FFN's gate and up weights, its token rows and activations (the
    shared FFN runs inside the same launch)."""
    n = wl.batch * wl.canvas
    nk = n * wl.top_k
    routed = touched * 2 * wl.expert_width * wl.d_model * 2 + nk * wl.d_model * 2 + nk * wl.expert_width * 2
    shared = (2 * wl.shared_width * wl.d_model * 2 + n * wl.d_model * 2 + n * wl.shared_width * 2
              if wl.shared_width else 0)
    return routed + shared


def step_bytes(wl, touched: float) -> float:
    """Algorithmic HBM bytes of one step: every weight read once, experts only
    if routed to (touched of E, averaged over layers), plus the prompt KV."""
    kv = wl.n_layers * wl.batch * wl.n_kv_heads * (wl.prompt_len + wl.canvas) * wl.head_dim * 2 * 2
    untouched = (wl.n_experts - touched) * 3 * wl.expert_width * wl.d_model * 2 * wl.n_layers
    return 2 * wl.param_count() - untouched + kv


# DRAM bytes / algorithmic bytes of one expert gate-up launch, from an ncu capture of
# the current kernel at the full-scale shape cut to one layer
# (profiles/expert_gemms_full.md); None once the kernel changes.
GATE_UP_TRAFFIC_RATIO = 1.044


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, 1590.0, "fallback"


# ----------------------------------------------------------------------------- CPU oracle

def oracle_step_seconds(wl, n_steps: int):
    """Times the fp64 oracle's denoising step (decoder pass + sampler) on this
    host; weight generation and the prompt pass are outside the timed region."""
    import numpy as np
    from oracle import decoder, pipeline, sampler
    W = decoder.Weights(wl)
    cache = pipeline.prompt_cache(W)
    tok = sampler.init_canvas(wl.seed, wl.batch, wl.canvas, wl.vocab)
    com = np.zeros_like(tok, dtype=bool)
    pipeline.denoise_step(W, cache, tok, com, 0, wl.steps, wl.seed)      # weights generated + cached here
    times = []
    for i in range(n_steps):
        t0 = time.perf_counter()
        _, tok, com, _ = pipeline.denoise_step(W, cache, tok, com, i % wl.steps, wl.steps, wl.seed)
        times.append(time.perf_counter() - t0)
    return times


class OracleSample:
    """A bounded sample of the oracle's step for workloads too large to run whole
    on the host.  The oracle's denoising step (decoder pass + sampler over every
    canvas row, with its per-pass weight generation, as it always runs at this
    size) is timed on the same workload cut to 1 and to 2 layers, and scaled to
    one full step as t1 + (L - 1) (t2 - t1).  The prompt cache is the workload's
    synthetic one (the step's cost does not depend on its values), so no prompt
    pass runs."""

    def __init__(self, wl):
        from oracle import decoder, sampler
        self.wl = wl
        self.parts = []
        for n in (1, 2):
            w = wl.replace(n_layers=n)
            self.parts.append((decoder.Weights(w), decoder.given_prompt_cache(w)))
        self.tok = sampler.init_canvas(wl.seed, wl.batch, wl.canvas, wl.vocab)

    def step(self) -> float:
        import numpy as np
        from oracle import pipeline
        t = []
        for W, cache in self.parts:
            t0 = time.perf_counter()
            pipeline.denoise_step(W, cache, self.tok, np.zeros_like(self.tok, dtype=bool), 0, self.wl.steps,
                                  self.wl.seed)
            t.append(time.perf_counter() - t0)
        return t[0] + (self.wl.n_layers - 1) * max(0.0, t[1] - t[0])

    def describe(self, n) -> str:
        wl = self.wl
        return (f"{n} bounded samples of the oracle's {wl.name} step (B={wl.batch}, C={wl.canvas}, P={wl.prompt_len}): "
                f"the whole step (decoder pass + sampler, all rows) of the model cut to 1 and to 2 of its "
                f"{wl.n_layers} layers, scaled as t1 + {wl.n_layers - 1} (t2 - t1)")


def oracle_baseline(wl, budget_s: float, max_steps: int):
    """(seconds per step, steps timed, description) for the oracle on this host."""
    if 2 * wl.param_count() <= (4 << 30):
        t_one = oracle_step_seconds(wl, 1)[0]
        k = max(1, min(max_steps, int(budget_s / max(t_one, 1e-3))))
        times = oracle_step_seconds(wl, k)
        return sum(times) / len(times), len(times), (
            f"{len(times)} full oracle denoising steps (decoder pass + sampler) of the {wl.name} workload, "
            f"after one untimed step")
    smp = OracleSample(wl)
    t0 = time.perf_counter()
    times = [smp.step()]
    while len(times) < min(max_steps, 3) and (time.perf_counter() - t0) * (len(times) + 1) / len(times) < budget_s:
        times.append(smp.step())
    return sum(times) / len(times), len(times), smp.describe(len(times))


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def reference_arm(args, wl, rank):
    if rank != 0:
        return
    per_step, n, sample = oracle_baseline(wl, budget_s=150.0, max_steps=args.steps)
    value = wl.batch * wl.canvas / (wl.steps * per_step)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": n, "warmup": 1, "ms_per_step": per_step * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": wl.name, "batch": wl.batch, "canvas": wl.canvas, "prompt": wl.prompt_len,
                       "T": wl.steps, "layers": wl.n_layers},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- native arm

def native_arm(args, wl, rank, world, local_rank):
    import numpy as np
    import torch
    import torch.distributed as dist
    import block_denoising_step_b200 as dg
    import synth
    from synth.device import device_weights, config_fields, device_prompt, device_prompt_kv

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(device=dev)
    embed, final_norm, layers = device_weights(wl, dev)
    torch.cuda.synchronize(dev)
    cfg = dg.ModelConfig(**config_fields(wl))
    den = dg.Denoiser(cfg, embed, final_norm, layers, stream=stream.cuda_stream)
    den.set_flags(args.flags)
    seed = replica_seed(wl, rank)
    with torch.cuda.stream(stream):
        if wl.prompt_kv_given:
            for l in range(wl.n_layers):
                k, v = device_prompt_kv(wl, l, dev)
                den.set_prompt_kv(l, k, v, wl.prompt_len)
                den.synchronize()
        else:
            den.prefill_prompt(device_prompt(wl, dev))
    den.synchronize()
    T = wl.steps

    def run_steps(n, s0):
        s = s0
        for _ in range(n):
            if s == 0:
                den.init_canvas(seed)
            den.denoise_step(s, T, None)
            den.sample_commit(s, T, seed)
            s = (s + 1) % T
        return s

    # kernel-class timing: CUDA events recorded on the library's stream around
    # each launch of these classes (captured into the step graph, so the
    # durations read after the timed region are those of its last step)
    timed_classes = [dg.K_EXPERT_GATE_UP, dg.K_EXPERT_DOWN, dg.K_LM_HEAD]
    den.set_timing(timed_classes)
    s = run_steps(max(args.warmup, 3), 0)
    den.synchronize()
    for c in timed_classes:
        den.get_timing(c)                                    # reset
    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.5)                                          # let the sampler start
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    clocks.mark_start()
    launches0 = den.launch_count()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    s = run_steps(args.steps, s)
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    clocks.mark_end()
    elapsed = ev0.elapsed_time(ev1) / 1e3
    launches = den.launch_count() - launches0
    clk = clocks.stop()
    den.set_timing([])
    ktimes = {dg.KERNEL_CLASSES[c]: den.get_timing(c) for c in timed_classes}
    den.synchronize()
    usage = den.expert_usage()                              # last timed step, per layer
    breakdown = None
    if args.breakdown:                                      # outside the timed region
        every = list(range(len(dg.KERNEL_CLASSES)))
        den.set_timing(every)                               # re-captures the step graph with events
        s = run_steps(2, s)
        den.synchronize()
        for c in every:
            den.get_timing(c)
        s = run_steps(1, s)                                 # graph classes report their last replay
        den.synchronize()
        den.set_timing([])
        breakdown = {}
        for c in every:
            ms, n = den.get_timing(c)
            breakdown[dg.KERNEL_CLASSES[c]] = {"ms": ms, "launches": n}
    touched = sum(usage) / len(usage)
    elapsed = max_over_ranks(elapsed, world, dev)

    # end to end through the host-buffer entry point: prompt H2D, prompt pass,
    # T steps, canvas D2H, per block
    e2e = None
    if args.e2e_blocks > 0 and not wl.prompt_kv_given:
        prompt_h = torch.from_numpy(synth.prompt_tokens(wl)).contiguous().pin_memory()
        out_h = torch.empty(wl.batch, wl.canvas, dtype=torch.int32).pin_memory()
        den.generate_block_host(prompt_h, T, seed, out_h)                 # warm
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.e2e_blocks):
            den.generate_block_host(prompt_h, T, seed, out_h)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        t_e2e = e0.elapsed_time(e1) / 1e3
        t_e2e = max_over_ranks(t_e2e, world, dev)
        e2e = {"value": world * wl.batch * wl.canvas * args.e2e_blocks / t_e2e, "unit": UNIT,
               "h2d_bytes_per_step": prompt_h.numel() * 4, "d2h_bytes_per_step": out_h.numel() * 4,
               "step": "one block through dgen_generate_block_host (prompt H2D, prompt pass, T steps, canvas D2H)"}

    hbm, bf16, peak_kind = peaks()
    gu_ms, gu_n = ktimes["expert_gate_up"]
    roof = None
    if gu_n:
        per_launch_s = gu_ms / gu_n / 1e3
        achieved = expert_gate_up_bytes(wl, touched) / per_launch_s / 1e9
        roof = {"kernel": "expert_gate_up (grouped tcgen05 GEMM + GELU*up epilogue; routed experts and the "
                          "shared FFN in one launch)", "bound": "hbm",
                "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                "peak_kind": peak_kind,
                "traffic": (GATE_UP_TRAFFIC_RATIO * expert_gate_up_bytes(wl, touched)
                            if GATE_UP_TRAFFIC_RATIO and wl.name.startswith("full") else None),
                "traffic_source": "ncu dram__bytes_read.sum + dram__bytes_write.sum of this kernel at the "
                                  "full-scale shape cut to 1 layer (ratio to algorithmic bytes 1.044), "
                                  "scaled to this launch's algorithmic bytes",
                "launches_timed": gu_n,
                "bytes_per_launch": expert_gate_up_bytes(wl, touched),
                "experts_touched_per_layer": touched}
    value = job_tokens_per_s(world, wl, args.steps, elapsed)
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": elapsed / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": wl.name, "batch": wl.batch, "canvas": wl.canvas, "prompt": wl.prompt_len,
                       "T": wl.steps, "layers": wl.n_layers, "d_model": wl.d_model, "experts": wl.n_experts,
                       "top_k": wl.top_k, "vocab": wl.vocab, "parallelism": f"replicas x{world}", "flags": args.flags,
                       "l2": f"inputs larger than L2: {step_bytes(wl, touched) / 1e9:.2f} GB of weights+KV "
                             f"streamed per step"},
            "roofline": roof,
            "kernel_us_per_launch": {k: (v[0] / v[1] * 1e3 if v[1] else None) for k, v in ktimes.items()},
            "breakdown": breakdown,
            "step_hbm_gbs": step_bytes(wl, touched) / (elapsed / args.steps) / 1e9,
            "lm_head_tensor": lm_head_tensor(wl, ktimes["lm_head"][0], ktimes["lm_head"][1], bf16),
            "experts_touched": {"mean_per_layer": touched, "of": wl.n_experts, "min": min(usage), "max": max(usage)},
            "e2e": e2e, "gpu_launches": launches, "clocks": clk}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        per, n, sample = oracle_baseline(wl, budget_s=20.0, max_steps=2)
        line["cpu_baseline"] = {"value": wl.batch * wl.canvas / (wl.steps * per), "unit": UNIT,
                                "cores": blas_threads(), "kind": "oracle", "seconds_per_step": per,
                                "sample": sample}
    if rank == 0:
        print(json.dumps(line), flush=True)
    den.close()


def gemm_per_sm():
    """Per-CTA streaming rate of the GEMM core (G CTAs, one 128-row A tile of
    K = 32768 each) and the fixed cost of a launch whose 148 CTAs stream one
    item each (growing K).  L2 flushed before every timed launch."""
    import torch
    import block_denoising_step_b200 as dg
    st = torch.cuda.current_stream().cuda_stream
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    bn_of = {0: 64, 4: 128, 5: 256}

    def run(G, K, v, reps=10):
        M = 128 * G
        a = torch.randn(M, K, device="cuda").to(torch.bfloat16)
        b = torch.randn(bn_of[v], K, device="cuda").to(torch.bfloat16)
        out = torch.empty(M, device="cuda")
        call = lambda: dg._check("dgen_gemm_rowsum_variant", dg._lib.dgen_gemm_rowsum_variant(
            a.data_ptr(), b.data_ptr(), out.data_ptr(), M, bn_of[v], K, v, st))
        for _ in range(3):
            call()
        ts = []
        for _ in range(reps):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            call()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1) * 1e3)
        t = sorted(ts)[reps // 2]
        print(json.dumps({"G": G, "K": K, "variant": v, "us": round(t, 2),
                          "a_GBs_total": round(M * K * 2 / t / 1e3, 1),
                          "a_GBs_per_cta": round(K * 128 * 2 / t / 1e3, 2)}), flush=True)

    for v in (0, 4, 5):
        for G in (1, 16, 64, 128, 148):
            run(G, 32768, v)
    for K in (704, 1408, 2816, 5632, 11264):
        run(148, K, 0)


def gemm_streaming():
    """Streaming rate of the tcgen05 GEMM core: A = 256 MB of bf16 "weights"
    [M][K], B = BN token rows, each thread writing only a row sum per tile, so
    the time is that of streaming A once.  cuBLAS (torch.matmul) on [M][K] x
    [K][64] is timed beside it."""
    import torch
    import block_denoising_step_b200 as dg
    variants = {0: ("BN64 stages8 1box", 64), 1: ("BN64 stages8 8box", 64), 2: ("BN64 stages4 1box", 64),
                3: ("BN32 stages8 1box", 32), 4: ("BN128 stages6 1box", 128), 5: ("BN256 stages4 1box", 256)}
    st = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for K in (64, 256, 1024, 2816):
        M = (2 ** 27 // K) // 128 * 128
        a = torch.randn(M, K, device="cuda").to(torch.bfloat16)
        res = {}
        for v, (name, bn) in variants.items():
            b = torch.randn(bn, K, device="cuda").to(torch.bfloat16)
            out = torch.empty(M, device="cuda")
            call = lambda: dg._check("dgen_gemm_rowsum_variant", dg._lib.dgen_gemm_rowsum_variant(
                a.data_ptr(), b.data_ptr(), out.data_ptr(), M, bn, K, v, st.cuda_stream))
            for _ in range(3):
                call()
            e0.record()
            for _ in range(10):
                call()
            e1.record()
            torch.cuda.synchronize()
            t = e0.elapsed_time(e1) / 10 / 1e3
            res[name] = M * K * 2 / t / 1e9
        bb = torch.randn(64, K, device="cuda").to(torch.bfloat16)
        for _ in range(3):
            c = a @ bb.T
        e0.record()
        for _ in range(10):
            c = a @ bb.T
        e1.record()
        torch.cuda.synchronize()
        res["cuBLAS N=64"] = M * K * 2 / (e0.elapsed_time(e1) / 10 / 1e3) / 1e9
        print(json.dumps({"K": K, "M": M, "GB/s": {k: round(v) for k, v in res.items()}}), flush=True)
        del a


def main():
    args = parse()
    if args.gemm_per_sm:
        gemm_per_sm()
        return
    if args.gemm_streaming:
        gemm_streaming()
        return
    import synth
    wl = synth.WORKLOADS[args.workload]
    if args.layers > 0 or args.prompt > 0:
        wl = wl.replace(name=f"{wl.name}-cut", n_layers=args.layers or wl.n_layers,
                        prompt_len=args.prompt or wl.prompt_len)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        reference_arm(args, wl, rank)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        native_arm(args, wl, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
