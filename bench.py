"""Benchmark of the block denoising step: canvas tokens/s per 256-token block (T = 12).

One bench step = one pass of the whole hot path over the workload's batch: a
decoder pass (dgen_denoise_step: attention over [prompt cache ; canvas], routed
MoE, LM head with fused softmax statistics) followed by the sampler
(dgen_sample_commit).  Steps cycle s = 0..T-1 through the canvas state machine
(a fresh Philox canvas at s = 0), so K steps process K / T blocks:

    value = n_gpus * B * C * K / (T * t_max)      [canvas tokens/s, whole job]

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--T T]
                       [--routing own|uniform] [--impl reference]
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

UNIT = "tokens/s"
DEFAULT_WORKLOAD = "full"


def metric_for(wl) -> str:
    """The metric's name at the workload's T (the default workloads use T = 12)."""
    return f"canvas tokens/s per 256-token block (T={wl.steps})"


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=None,
                   help="timed steps (default 600; reference arm: one oracle step's pieces, 61 at full scale)")
    p.add_argument("--warmup", type=int, default=24)
    p.add_argument("--workload", default=DEFAULT_WORKLOAD)
    p.add_argument("--T", type=int, default=0, help="steps per block override (the batched workload sweeps 4, 12, 32)")
    p.add_argument("--expert-fp8", action="store_true",
                   help="routed experts and shared FFN in FP8 E4M3 (power-of-two row scales); the rest bf16")
    p.add_argument("--self-cond", type=int, default=0, metavar="W",
                   help="self-conditioning with an FFW of width W (the shared FFN's 2112 at full scale); 0 = off")
    p.add_argument("--routing", default="own", choices=["own", "uniform"],
                   help="uniform: force every layer's routing to spread the rows evenly over all experts")
    p.add_argument("--eb-blocks", type=int, default=2, help="blocks timed with the entropy-bounded sampler")
    p.add_argument("--eb-tmax", type=int, default=48)
    p.add_argument("--eb-gamma", type=float, default=250.0)
    p.add_argument("--eb-stop", type=float, default=0.5)
    p.add_argument("--layers", type=int, default=0,
                   help="profiling aid: cut the workload's model to this many layers (named in config)")
    p.add_argument("--prompt", type=int, default=0, help="profiling aid: prompt length override")
    p.add_argument("--impl", default="native", choices=["native", "reference"])
    p.add_argument("--e2e-blocks", type=int, default=3)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--flags", type=int, default=0, help="dgen_set_flags value (1 no graph, 2 no PDL)")
    p.add_argument("--static-items", action="store_true",
                   help="measurement: the one-launch expert GEMMs take their items in a fixed stride")
    p.add_argument("--chunk-order", default="auto", choices=["auto", "id", "size"],
                   help="measurement: order of the routed experts' chunks (auto: largest expert first for the "
                        "two-launch E4M3 experts, id order for the one-launch bf16 experts)")
    p.add_argument("--pairs", default="auto", choices=["auto", "none", "all"],
                   help="measurement: dense GEMMs on CTA pairs (auto: LM head and p0_hat E; all: also QKV and O "
                        "projection)")
    p.add_argument("--gemm-per-sm", action="store_true",
                   help="per-SM streaming rate and fixed cost of the GEMM core (one JSON line per case)")
    p.add_argument("--attn-splits-sweep", action="store_true",
                   help="time the attention launch class (split combine included) at key split counts 1-8 "
                        "(one JSON line)")
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

# Nominal B200 figures, beside the measured ones (MEASURED_PEAKS.json).
NOMINAL_HBM_GBS = 8000.0
NOMINAL_BF16_TFLOPS = 2250.0

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
    the measured dense bf16 peak (and of the nominal 2.25 PFLOP/s); None when
    the launch was not timed."""
    if not lm_n or lm_ms <= 0.0:
        return None
    flop = 2.0 * wl.batch * wl.canvas * wl.vocab * wl.d_model
    achieved = flop / (lm_ms / lm_n / 1e3) / 1e12
    return {"kernel": "LM head (tcgen05 GEMM + softmax-statistics epilogue)", "bound": "tensor",
            "achieved": achieved, "peak": peak_tflops, "unit": "TFLOP/s", "frac": achieved / peak_tflops,
            "frac_nominal": achieved / NOMINAL_BF16_TFLOPS, "flop_per_launch": flop,
            "us_per_launch": lm_ms / lm_n * 1e3}


def expert_gate_up_bytes(wl, touched: float) -> float:
    """Algorithmic HBM bytes of one grouped gate-up launch: the gate and up
    weights of the experts routed to (touched, averaged over the layers, read
    from the library), the routed token rows in, the activations out; plus the
    shared FFN's gate and up weights, its token rows and activations (the
    shared FFN runs inside the same launch).  With E4M3 experts the weights and
    token rows are one byte per element plus a 4-byte scale per row."""
    n = wl.batch * wl.canvas
    nk = n * wl.top_k
    b = 1 if wl.expert_fp8 else 2
    sc = 4 if wl.expert_fp8 else 0
    routed = (touched * 2 * wl.expert_width * (wl.d_model * b + sc) + nk * (wl.d_model * b + sc)
              + nk * wl.expert_width * 2)
    shared = (2 * wl.shared_width * (wl.d_model * b + sc) + n * (wl.d_model * b + sc) + n * wl.shared_width * 2
              if wl.shared_width else 0)
    return routed + shared


def expert_down_bytes(wl, touched: float) -> float:
    """Algorithmic HBM bytes of one grouped down launch: the down weights of the
    touched experts and of the shared FFN, the activations in, the gated fp32
    output rows (routed slots and shared-FFN slices)."""
    n = wl.batch * wl.canvas
    nk = n * wl.top_k
    parts = -(-wl.shared_width // wl.expert_width) if wl.shared_width else 0
    b = 1 if wl.expert_fp8 else 2
    routed = touched * wl.d_model * wl.expert_width * b + nk * wl.expert_width * b + nk * wl.d_model * 4
    shared = (wl.d_model * wl.shared_width * b + n * wl.shared_width * b + parts * n * wl.d_model * 4
              if wl.shared_width else 0)
    return routed + shared


def step_bytes(wl, touched: float) -> float:
    """Algorithmic HBM bytes of one step: every weight read once, experts only
    if routed to (touched of E, averaged over layers), plus the prompt KV."""
    kv = wl.n_layers * wl.batch * wl.n_kv_heads * (wl.prompt_len + wl.canvas) * wl.head_dim * 2 * 2
    b = 1 if wl.expert_fp8 else 2
    untouched = (wl.n_experts - touched) * 3 * wl.expert_width * wl.d_model * b * wl.n_layers
    expert_params = wl.n_layers * (wl.n_experts * 3 * wl.expert_width + 3 * wl.shared_width) * wl.d_model
    return 2 * wl.param_count() - (2 - b) * expert_params - untouched + kv


def self_cond_line(wl, cls, hbm, bf16, ms_step):
    """The self-conditioning block's share of a step: its device time (class
    timing), algorithmic HBM bytes (the logits read, p0_hat written and read,
    the embedding read by p0_hat E, the FFW weights) and flops (p0_hat E and
    the FFW), each against its peak."""
    if not wl.self_cond_width or not cls["launches"]:
        return None
    n, V, d, w = wl.batch * wl.canvas, wl.vocab, wl.d_model, wl.self_cond_width
    nbytes = 4 * n * V + 2 * 2 * n * V + 2 * V * d + 2 * 3 * w * d
    flops = 2 * n * V * d + 2 * n * 3 * w * d
    t = cls["ms"] / 1e3
    return {"ms_per_step": cls["ms"], "share_of_step": cls["ms"] / ms_step, "launches_per_step": cls["launches"],
            "hbm_bytes": nbytes, "hbm_frac": nbytes / t / 1e9 / hbm, "flops": flops,
            "tensor_frac": flops / t / 1e12 / bf16,
            "note": "p0_hat = Softmax(L / tau) in bf16, u = p0_hat E (K-split tcgen05 GEMM, E read MN-major), "
                    "RMSNorm, gated-GELU FFW; z added to the next step's embeddings"}


def step_flops(wl) -> float:
    """Algorithmic flops of one step (2 per multiply-add): projections, attention
    over P + C keys, the k routed experts and the shared FFN per row, the LM head."""
    n = wl.batch * wl.canvas
    d, hd = wl.d_model, wl.head_dim
    proj = 2 * n * d * (wl.qkv_rows + wl.n_q_heads * hd + wl.n_experts)
    attn = 2 * 2 * n * wl.n_q_heads * (wl.prompt_len + wl.canvas) * hd
    moe = 2 * n * 3 * d * (wl.top_k * wl.expert_width + wl.shared_width)
    return wl.n_layers * (proj + attn + moe) + 2 * n * d * wl.vocab


# DRAM bytes (read + write) / algorithmic bytes of the one-launch expert GEMMs,
# from an ncu capture of the current kernel at the full-scale shapes cut to two
# layers (profiles/expert_fused_full_2layer.md: 1.491 and 1.463 GB for 1.498 GB);
# the weights of the touched experts dominate both, so the ratio carries to the
# 30-layer launch.  None once the kernel changes.
FUSED_TRAFFIC_RATIO = 0.986


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, 1590.0, "fallback"


def uniform_routing(wl):
    """Expert ids [L][B*C][k] that spread the canvas rows evenly over all experts:
    row r, slot j -> (r k + j) mod E (distinct within a row when k <= E), the
    load-balanced routing a trained router aims for; every layer the same."""
    import numpy as np
    n = wl.batch * wl.canvas
    ids = (np.arange(n)[:, None] * wl.top_k + np.arange(wl.top_k)[None, :]) % wl.n_experts
    return np.broadcast_to(ids, (wl.n_layers, n, wl.top_k)).astype(np.int32).copy()


# ----------------------------------------------------------------------------- CPU oracle

def host_cpu():
    """(logical CPUs, CPU model name) of this host."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return os.cpu_count(), model


class OracleStep:
    """The fp64 oracle's denoising step of a workload (decoder pass + sampler over
    every canvas row, with the oracle's per-pass weight regeneration, as it always
    runs at this size), cut into pieces that run in order: for each layer its
    attention block and its MoE block, then the final norm + LM head + sampler
    (oracle.decoder.DecoderPass, oracle.sampler.sample_commit).  Consecutive steps
    continue the canvas state machine (s = 0, 1, ...).  The prompt cache is the
    workload's synthetic bf16 cache (a step costs the same whatever the cache
    holds), so no prompt pass runs.  n_seq < B keeps only the first n_seq of
    the independent sequences (a bounded sample of a batched workload)."""

    def __init__(self, wl, n_seq=None):
        import numpy as np
        from oracle import decoder, sampler
        self.n_seq = wl.batch if n_seq is None else n_seq
        self.wl = wl.replace(batch=self.n_seq)
        self.W = decoder.Weights(self.wl)
        self.cache = decoder.given_prompt_cache(self.wl)
        self.tok = sampler.init_canvas(wl.seed, self.n_seq, wl.canvas, wl.vocab)
        self.committed = np.zeros_like(self.tok, dtype=bool)
        self.s = 0
        self.dp = None
        self.next_piece = 0

    @property
    def pieces_per_step(self) -> int:
        return 2 * self.wl.n_layers + 1

    def run_piece(self) -> bool:
        """Runs the next piece; True when it finished a whole step."""
        from oracle import decoder, sampler
        wl = self.wl
        if self.dp is None:
            self.dp = decoder.DecoderPass(self.W, self.tok, self.cache)
            self.next_piece = 0
        self.dp.run_piece(self.next_piece)
        self.next_piece += 1
        if self.next_piece < self.dp.n_pieces:
            return False
        tau = sampler.tau_of_step(self.s, wl.steps, wl.tau_max, wl.tau_min)
        self.tok, self.committed, _ = sampler.sample_commit(self.dp.logits, self.tok, self.committed, self.s,
                                                            wl.steps, wl.seed, tau, wl.commit_per_step)
        self.s = (self.s + 1) % wl.steps
        if self.s == 0:
            import numpy as np
            self.committed = np.zeros_like(self.committed)
        self.dp = None
        return True


def cpu_estimate(wl, n_seq=None):
    """Bounded sample for the native arm's cpu_baseline (10-30 s of host work at
    the full-scale workload): the oracle step's pieces for layer 0 (attention
    block, MoE block) and its last piece (final norm, LM head, sampler) are
    timed, and one step is estimated as L x (layer 0) + last piece.  Returns
    (seconds per step of the whole batch, description)."""
    st = OracleStep(wl, n_seq)
    t = []
    for _ in range(2):
        t0 = time.perf_counter()
        st.run_piece()
        t.append(time.perf_counter() - t0)
    st.next_piece = st.dp.n_pieces - 1       # skip to the last piece (same shapes as in a whole step)
    t0 = time.perf_counter()
    st.run_piece()
    t.append(time.perf_counter() - t0)
    per_step = (wl.n_layers * (t[0] + t[1]) + t[2]) * wl.batch / st.n_seq
    desc = (f"estimate from a bounded sample of the oracle's {wl.name} step (C={wl.canvas}, P={wl.prompt_len}, "
            f"{st.n_seq} of {wl.batch} sequences): layer 0's attention block {t[0]:.2f} s and MoE block {t[1]:.2f} s "
            f"(x {wl.n_layers} layers) + final norm, LM head and sampler {t[2]:.2f} s; the reference arm "
            f"(--impl reference) times whole steps")
    return per_step, desc


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def reference_arm(args, wl, rank):
    """The reference arm: the fp64 oracle as it stands, on this host's cores.
    Its K bench steps are K consecutive, contiguous shares of whole oracle steps
    (ceil(K / pieces) of them, pieces = 2 L + 1, see OracleStep), so the timed
    region is whole steps of the real oracle and steps / warmup are the ones
    asked for; W warm-up pieces of a throwaway step run first, untimed.  Batched
    workloads keep one of their independent sequences (the step of one sequence
    is 1/B of the batch's work), scaled to the whole batch."""
    if rank != 0:
        return
    n_seq = 1 if wl.batch > 1 else None
    K, W = args.steps, args.warmup
    warm = OracleStep(wl, n_seq)
    for _ in range(min(W, warm.pieces_per_step)):
        warm.run_piece()
    del warm
    st = OracleStep(wl, n_seq)
    n_pieces = st.pieces_per_step
    n_steps = -(-K // n_pieces)
    total = n_steps * n_pieces
    bounds = [round(i * total / K) for i in range(K + 1)]
    times, done_steps = [], 0
    for i in range(K):
        t0 = time.perf_counter()
        for _ in range(bounds[i + 1] - bounds[i]):
            done_steps += st.run_piece()
        times.append(time.perf_counter() - t0)
    elapsed = sum(times)
    value = done_steps * wl.batch * wl.canvas / (wl.steps * elapsed)
    nproc, model = host_cpu()
    sample = (f"{done_steps} whole oracle step(s) of the {wl.name} workload"
              + (f" for {st.n_seq} of its {wl.batch} independent sequences, scaled to the batch" if n_seq else "")
              + f", timed as {K} consecutive shares of its {n_pieces} pieces (per layer: attention block, MoE "
                f"block; then LM head + sampler); {min(W, n_pieces)} untimed warm-up pieces first")
    line = {"impl": "reference", "metric": metric_for(wl), "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": K, "warmup": W, "ms_per_step": elapsed / K * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": wl.name, "batch": wl.batch, "canvas": wl.canvas, "prompt": wl.prompt_len,
                       "T": wl.steps, "layers": wl.n_layers},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                             "sample": sample, "seconds_per_oracle_step": elapsed / max(done_steps, 1) *
                             (st.n_seq / wl.batch), "nproc": nproc, "cpu_model": model},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- native arm

def native_arm(args, wl, rank, world, local_rank):
    import numpy as np
    import torch
    import torch.distributed as dist
    import block_denoising_step_b200 as dg
    import synth
    from synth.device import device_weights, device_self_cond_weights, config_fields, device_prompt, device_prompt_kv

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(device=dev)
    embed, final_norm, layers = device_weights(wl, dev)
    torch.cuda.synchronize(dev)
    cfg = dg.ModelConfig(**config_fields(wl))
    sc_w = device_self_cond_weights(wl, dev) if wl.self_cond_width else None
    den = dg.Denoiser(cfg, embed, final_norm, layers, stream=stream.cuda_stream, self_cond=sc_w)
    den.set_flags(args.flags)
    if args.static_items:
        den.set_tuning(dg.Denoiser.TUNE_STATIC_ITEMS, 1)
    if args.pairs != "auto":
        den.set_tuning(dg.Denoiser.TUNE_PAIRS, {"none": 1, "all": 2}[args.pairs])
    if args.chunk_order != "auto":
        den.set_tuning(dg.Denoiser.TUNE_CHUNK_ORDER, {"id": 1, "size": 2}[args.chunk_order])
    seed = replica_seed(wl, rank)
    T = wl.steps

    def ev():
        return torch.cuda.Event(enable_timing=True)

    prefill_ms = None
    with torch.cuda.stream(stream):
        if wl.prompt_kv_given:
            for l in range(wl.n_layers):
                k, v = device_prompt_kv(wl, l, dev)
                den.set_prompt_kv(l, k, v, wl.prompt_len)
                den.synchronize()
        else:
            prompt = device_prompt(wl, dev)
            den.prefill_prompt(prompt)                       # warm (kernel attributes, first touch)
            den.synchronize()
            p0, p1 = ev(), ev()
            p0.record(stream)
            den.prefill_prompt(prompt)
            p1.record(stream)
            den.synchronize()
            prefill_ms = p0.elapsed_time(p1)
    den.synchronize()
    forced = None
    if args.routing == "uniform":
        forced = torch.from_numpy(uniform_routing(wl).reshape(-1)).to(dev)
        den.force_routing(None, forced)

    def run_steps(n, s0):
        s = s0
        for _ in range(n):
            if s == 0:
                den.init_canvas(seed)
            den.denoise_step(s, T, None)
            den.sample_commit(s, T, seed)
            s = (s + 1) % T
        return s

    s = run_steps(max(args.warmup, 3), 0)
    den.synchronize()
    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.5)                                          # let the sampler start
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    clocks.mark_start()
    launches0 = den.launch_count()
    ev0, ev1 = ev(), ev()
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
    elapsed = max_over_ranks(elapsed, world, dev)

    # experts touched per layer (the step's byte count depends on its routing):
    # averaged over one block of untimed steps after the timed region
    block_usage = []
    for _ in range(T):
        s = run_steps(1, s)
        block_usage.append(den.expert_usage())
    touched = float(np.mean(block_usage))
    usage = [u for step in block_usage for u in step]

    # per-kernel-class times: a second pass over one block with CUDA events around
    # every launch class (captured into the step graph), after the headline was
    # timed without them; graph classes report the last step's launches
    every = list(range(len(dg.KERNEL_CLASSES)))
    den.set_timing(every)
    s = run_steps(2, s)
    den.synchronize()
    for c in every:
        den.get_timing(c)
    s = run_steps(1, s)
    den.synchronize()
    den.set_timing([])
    cls_usage = den.expert_usage()                          # the step whose launches were timed
    touched_cls = sum(cls_usage) / len(cls_usage)
    classes = {}
    for c in every:
        ms, n = den.get_timing(c)
        classes[dg.KERNEL_CLASSES[c]] = {"ms": ms, "launches": n}

    # end to end through the host-buffer entry point: prompt H2D, prompt pass,
    # T steps, canvas D2H, per block
    e2e = None
    if args.e2e_blocks > 0 and not wl.prompt_kv_given and forced is None:
        prompt_h = torch.from_numpy(synth.prompt_tokens(wl)).contiguous().pin_memory()
        out_h = torch.empty(wl.batch, wl.canvas, dtype=torch.int32).pin_memory()
        den.generate_block_host(prompt_h, T, seed, out_h)                 # warm
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        e0, e1 = ev(), ev()
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

    # the pages' own sampler: whole blocks with entropy-bounded acceptance and the
    # adaptive stop (device done flags read by the host loop), from the cache as it is
    eb = None
    if args.eb_blocks > 0 and forced is None:
        out = torch.empty(wl.batch * wl.canvas, dtype=torch.int32, device=dev)
        with torch.cuda.stream(stream):
            den.generate_block_eb(None, args.eb_tmax, seed, args.eb_gamma, args.eb_stop, out)
            torch.cuda.synchronize(dev)
            e0, e1 = ev(), ev()
            e0.record(stream)
            steps = []
            for b in range(args.eb_blocks):
                steps += den.generate_block_eb(None, args.eb_tmax, seed + 1 + b, args.eb_gamma, args.eb_stop, out)
            e1.record(stream)
            torch.cuda.synchronize(dev)
        t_eb = e0.elapsed_time(e1) / 1e3
        eb = {"value": wl.batch * wl.canvas * args.eb_blocks / t_eb, "unit": UNIT,
              "mean_steps_per_block": float(np.mean(steps)), "max_steps": args.eb_tmax, "gamma": args.eb_gamma,
              "stop_threshold": args.eb_stop, "tokens_per_forward": wl.canvas / float(np.mean(steps)),
              "ms_per_block": t_eb / args.eb_blocks * 1e3,
              "note": "whole blocks through dgen_generate_block_eb from the prompt cache; gamma is chosen so that "
                      "the synthetic random-init model takes about the pages' 12 steps per 256-token block"}

    hbm, bf16, peak_kind = peaks()
    gu, dn = classes["expert_gate_up"], classes["expert_down"]
    fused = gu["launches"] > 0 and dn["launches"] == 0   # both expert GEMMs in one launch
    roof = None
    if gu["launches"]:
        per_launch_s = gu["ms"] / gu["launches"] / 1e3
        nbytes = expert_gate_up_bytes(wl, touched_cls) + (expert_down_bytes(wl, touched_cls) if fused else 0.0)
        achieved = nbytes / per_launch_s / 1e9
        roof = {"kernel": ("fused expert GEMMs (gate-up + GELU*up, then down * gate, in one persistent tcgen05 "
                           "launch; routed experts and the shared FFN)") if fused else
                          "expert_gate_up (grouped tcgen05 GEMM + GELU*up epilogue; routed experts and the "
                          "shared FFN in one launch)", "bound": "hbm",
                "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                "frac_nominal": achieved / NOMINAL_HBM_GBS, "peak_kind": peak_kind,
                "traffic": (FUSED_TRAFFIC_RATIO * nbytes
                            if FUSED_TRAFFIC_RATIO and fused and wl.name.startswith("full") else None),
                "traffic_source": "ncu dram__bytes_read.sum + dram__bytes_write.sum of the one-launch expert "
                                  "GEMMs at the full-scale shapes cut to 2 layers (ratio 0.986), scaled to this "
                                  "launch's algorithmic bytes; null for the two-launch form",
                "launches_timed": gu["launches"], "us_per_launch": per_launch_s * 1e6,
                "bytes_per_launch": nbytes,
                "experts_touched_per_layer": touched_cls,
                "timing": "CUDA events around each launch of the class in a second pass after the timed region"}
    down = None
    if dn["launches"]:
        per = dn["ms"] / dn["launches"] / 1e3
        a = expert_down_bytes(wl, touched_cls) / per / 1e9
        down = {"achieved": a, "unit": "GB/s", "frac": a / hbm, "frac_nominal": a / NOMINAL_HBM_GBS,
                "us_per_launch": per * 1e6, "bytes_per_launch": expert_down_bytes(wl, touched_cls)}
    ms_step = elapsed / args.steps * 1e3
    sb = step_bytes(wl, touched)
    value = job_tokens_per_s(world, wl, args.steps, elapsed)
    line = {"metric": metric_for(wl), "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16, experts e4m3" if wl.expert_fp8 else "bf16",
            "data": "synthetic",
            "config": {"workload": wl.name, "batch": wl.batch, "canvas": wl.canvas, "prompt": wl.prompt_len,
                       "T": wl.steps, "layers": wl.n_layers, "d_model": wl.d_model, "experts": wl.n_experts,
                       "expert_fp8": wl.expert_fp8, "self_cond_width": wl.self_cond_width,
                       "top_k": wl.top_k, "vocab": wl.vocab, "parallelism": f"replicas x{world}", "flags": args.flags,
                       "routing": args.routing, "static_items": args.static_items, "pairs": args.pairs,
                       "chunk_order": args.chunk_order,
                       "l2": f"inputs larger than L2: {sb / 1e9:.2f} GB of weights+KV streamed per step"},
            "roofline": roof,
            "expert_down": down,
            "lm_head_tensor": lm_head_tensor(wl, classes["lm_head"]["ms"], classes["lm_head"]["launches"], bf16),
            "step_hbm": {"bytes": sb, "achieved_gbs": sb / (elapsed / args.steps) / 1e9,
                         "frac": sb / (elapsed / args.steps) / 1e9 / hbm,
                         "floor_ms": sb / hbm / 1e6,
                         "tensor_floor_ms": step_flops(wl) / (bf16 * 1e12) * 1e3},
            "kernel_classes_ms_per_step": {k: v["ms"] for k, v in classes.items() if v["launches"]},
            "kernel_classes_launches": {k: v["launches"] for k, v in classes.items() if v["launches"]},
            "prefill_ms": prefill_ms,
            "self_cond": self_cond_line(wl, classes["self_cond"], hbm, bf16, ms_step),
            "experts_touched": {"mean_per_layer": touched, "of": wl.n_experts, "min": min(usage), "max": max(usage),
                                "over": f"the layers of {T} untimed steps after the timed region",
                                "class_pass_step": touched_cls},
            "e2e": e2e, "eb_sampler": eb, "gpu_launches": launches, "clocks": clk}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        per, sample = cpu_estimate(wl, 1 if wl.batch > 1 else None)
        nproc, model = host_cpu()
        line["cpu_baseline"] = {"value": wl.batch * wl.canvas / (wl.steps * per), "unit": UNIT,
                                "cores": blas_threads(), "kind": "oracle", "seconds_per_step": per,
                                "sample": sample, "nproc": nproc, "cpu_model": model}
    if rank == 0:
        print(json.dumps(line), flush=True)
    den.force_routing(None, None)
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
        call = lambda: dg._check("dgen_gemm_rowsum_variant", dg.probe_lib().dgen_gemm_rowsum_variant(
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
            call = lambda: dg._check("dgen_gemm_rowsum_variant", dg.probe_lib().dgen_gemm_rowsum_variant(
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


def attn_splits_sweep(wl):
    """CUDA-event time per attention launch (the split combine included) of the
    workload's step at forced key split counts (DGEN_TUNE_ATTN_SPLITS)."""
    import torch
    import block_denoising_step_b200 as dg
    from synth.device import device_weights, config_fields, device_prompt
    dev = torch.device("cuda", 0)
    stream = torch.cuda.Stream(device=dev)
    embed, fn, layers = device_weights(wl, dev)
    den = dg.Denoiser(dg.ModelConfig(**config_fields(wl)), embed, fn, layers, stream=stream.cuda_stream)
    res = {}
    with torch.cuda.stream(stream):
        den.prefill_prompt(device_prompt(wl, dev))
        den.synchronize()
        for splits in (1, 2, 3, 4, 6, 8):
            den.set_tuning(dg.Denoiser.TUNE_ATTN_SPLITS, splits)
            den.init_canvas(1)
            for _ in range(3):
                den.denoise_step(0, wl.steps, None)
            den.synchronize()
            den.set_timing([dg.K_ATTENTION])
            den.get_timing(dg.K_ATTENTION)
            for _ in range(20):
                den.denoise_step(0, wl.steps, None)
            den.synchronize()
            ms, n = den.get_timing(dg.K_ATTENTION)
            den.set_timing([])
            res[splits] = ms / n * 1e3
    den.close()
    print(json.dumps({"workload": wl.name, "layers": wl.n_layers,
                      "attention_us_per_launch_incl_combine_by_splits": res}), flush=True)


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
    if args.T > 0:
        wl = wl.replace(steps=args.T)
    if args.expert_fp8:
        wl = wl.replace(expert_fp8=True)
    if args.attn_splits_sweep:
        attn_splits_sweep(wl)
        return
    if args.self_cond:
        wl = wl.replace(self_cond_width=args.self_cond)
    if args.steps is None:
        args.steps = 2 * wl.n_layers + 1 if args.impl == "reference" else 600
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
