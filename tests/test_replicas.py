"""The N > 1 path of bench.py on CPU: two ranks over gloo (127.0.0.1).

The step does not shard (independent canvases per GPU: replicas only), so the
multi-GPU path is host logic: per-rank seeds, the max over ranks of the timed
region, and the whole-job throughput from the slowest rank.  The reference
arm runs on rank 0 only.
"""
import os
import socket

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import bench
    import synth
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        wl = synth.WORKLOADS["full"]
        elapsed = 1.0 + 0.5 * rank                       # rank 1 is the slowest
        t_max = bench.max_over_ranks(elapsed, world)
        seeds = [None] * world
        dist.all_gather_object(seeds, bench.replica_seed(wl, rank))
        value = bench.job_tokens_per_s(world, wl, 120, t_max)
        out[rank] = (t_max, tuple(seeds), value)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_time_and_distinct_seeds():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    import synth
    wl = synth.WORKLOADS["full"]
    for r in range(world):
        t_max, seeds, value = out[r]
        assert t_max == 1.5                              # max over ranks, the same on every rank
        assert len(set(seeds)) == world                  # independent canvases
        # 2 replicas x 256 tokens x 120 steps / 12 steps per block / 1.5 s
        assert abs(value - 2 * 256 * 120 / 12 / 1.5) < 1e-9


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(3.25, 1) == 3.25


def test_reference_arm_runs_on_rank_zero_only(capsys):
    import bench
    import synth

    class Args:
        steps = 1
        gpus = 2

    bench.reference_arm(Args(), synth.WORKLOADS["tiny"], rank=1)   # returns at once, prints nothing
    assert capsys.readouterr().out == ""
