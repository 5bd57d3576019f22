"""The allocation-free sampler entry point against the handle-based one.

dgen_sample_from_logits_noalloc serves callers that must not allocate device
memory (latency-critical serving code that cannot afford cudaMalloc's
device-wide synchronisation, hosts that own all device memory through their
own allocator, fixed memory budgets).  It keeps its scratch in one fixed
device array instead of handle-owned buffers.  Here it must reproduce
dgen_set_logits + dgen_sample_commit exactly (same kernels, same order, so the
integer outputs and the confidences are bit-identical) on two calls in a row,
the second continuing from the state the first left.  This file is collected
last so that a run stopping at the first failure has run everything else.
"""
import numpy as np
import pytest

import synth

B, C, V = 2, 256, 4096


def test_noalloc_rejects_sizes_beyond_its_scratch():
    import block_denoising_step_b200 as dg
    L = dg._lib
    # 8192 rows * 1024 tiles > 262144: rejected before any CUDA call
    assert L.dgen_sample_from_logits_noalloc(0x1000, 0x1000, 0x1000, 32, 256, 262144, 0, 12, 1, 0.8, 0.4, 0,
                                             None, None) == dg.DGEN_ESCRATCH
    assert L.dgen_sample_from_logits_noalloc(0x1000, 0x1000, 0x1000, 40, 256, 256, 0, 12, 1, 0.8, 0.4, 0,
                                             None, None) == dg.DGEN_ESCRATCH
    assert L.dgen_sample_from_logits_noalloc(None, 0x1000, 0x1000, 1, 256, 4096, 0, 12, 1, 0.8, 0.4, 0,
                                             None, None) == dg.DGEN_EINVAL


@pytest.mark.gpu
def test_noalloc_matches_handle_path_on_two_calls_in_a_row():
    torch = pytest.importorskip("torch")
    import block_denoising_step_b200 as dg
    from tests.helpers import make_denoiser

    wl = synth.WORKLOADS["tiny"].replace(batch=B, canvas=C)
    den = make_denoiser(wl)
    stream = torch.cuda.current_stream().cuda_stream
    T, seed = 12, 31337
    tok0 = synth.uniform_i32(seed, 7, 0, B * C, V)
    com0 = np.zeros(B * C, dtype=np.uint8)
    com0[::5] = 1
    tok_h = torch.from_numpy(tok0).cuda()
    com_h = torch.from_numpy(com0).cuda()
    tok_n, com_n = tok_h.clone(), com_h.clone()
    den.set_canvas(tok_h, com_h)
    for s in (3, 4):
        logits = torch.from_numpy(synth.logits_f32(seed, s, B * C, V, std=2.0).reshape(-1)).cuda()
        conf_h = torch.empty(B * C, dtype=torch.float32, device="cuda")
        conf_n = torch.full((B * C,), float("nan"), dtype=torch.float32, device="cuda")
        den.set_logits(logits, s, T)
        den.sample_commit(s, T, seed, conf_h)
        den.get_canvas(tok_h, com_h)
        den.synchronize()
        dg.sample_from_logits_noalloc(logits, tok_n, com_n, B, C, V, s, T, seed, wl.tau_max, wl.tau_min,
                                      wl.commit_per_step, conf_n, stream)
        torch.cuda.synchronize()
        assert torch.equal(tok_n, tok_h), f"step {s}: tokens differ"
        assert torch.equal(com_n, com_h), f"step {s}: committed flags differ"
        assert torch.equal(conf_n, conf_h), f"step {s}: confidences differ"
        assert int(com_n.sum()) == int(com0.sum()) + (s - 2) * -(-C // T) * B
    den.close()
