"""Block-autoregressive continuation (hyper.ai digest, Method: one 256-token
canvas at a time; stage 3 of the three-stage pipeline re-encodes the finished
canvas causally and appends it to the KV cache) through the C ABI, against the
oracle (oracle.decoder.prefill with a prefix, oracle.pipeline.generate)."""
import numpy as np
import pytest

import synth
from oracle import decoder, sampler as osamp
from tests.helpers import make_denoiser, rel_l2, gpu_step_forced, oracle_prompt_routing

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

WL = synth.WORKLOADS["tiny"].replace(batch=2, canvas=200, prompt_len=50)


def _bf16_to_f64(t):
    return t.view(torch.int16).cpu().numpy().astype(np.uint16).astype(np.uint32).__lshift__(16).view(np.float32) \
        .astype(np.float64)


def test_appended_canvas_cache_and_next_step_match_the_oracle():
    """Prompt pass, then the append pass over a canvas, with the oracle's routing
    forced in both: every layer's K and V at positions 0..P+C-1 agree with the
    oracle's (relative L2 <= 1e-2, values bf16 on both sides); the next block's
    initial canvas is the Philox stream at positions offset by C (bit-exact);
    a step on the extended cache (routing forced) matches the oracle's logits
    (relative L2 <= 1e-2 over all rows)."""
    wl = WL
    B, C, P, V, L = wl.batch, wl.canvas, wl.prompt_len, wl.vocab, wl.n_layers
    W = decoder.Weights(wl)
    prompt = synth.prompt_tokens(wl)
    cache0, p_ids = oracle_prompt_routing(W, prompt)
    canvas = synth.target_canvas(wl, stream=3)
    a_routing = []
    cache1 = decoder.prefill(W, canvas, routing=a_routing, prefix=cache0)
    a_ids = np.zeros((L, B * C, wl.top_k), dtype=np.int32)
    for l, r in enumerate(a_routing):
        a_ids[l] = r

    den = make_denoiser(wl, prompt_max=P + C)
    from synth.device import device_prompt
    den.force_routing(torch.from_numpy(p_ids.reshape(-1)).cuda(), None)
    den.prefill_prompt(device_prompt(wl))
    den.set_canvas(torch.from_numpy(canvas.reshape(-1).astype(np.int32)).cuda(), None)
    den.force_routing(torch.from_numpy(a_ids.reshape(-1)).cuda(), None)
    den.append_canvas()
    den.force_routing(None, None)
    S_max = P + 2 * C
    kc = torch.empty(B * wl.n_kv_heads * S_max * wl.head_dim, dtype=torch.bfloat16, device="cuda")
    vc = torch.empty_like(kc)
    for l in range(L):
        den.debug_read(4, l, kc)
        den.debug_read(5, l, vc)
        den.synchronize()
        k = _bf16_to_f64(kc).reshape(B, wl.n_kv_heads, S_max, wl.head_dim)[:, :, :P + C]
        v = _bf16_to_f64(vc).reshape(B, wl.n_kv_heads, S_max, wl.head_dim)[:, :, :P + C]
        ek, ev = rel_l2(k[:, :, P:], cache1[l][0][:, :, P:]), rel_l2(v[:, :, P:], cache1[l][1][:, :, P:])
        print(f"layer {l}: appended K rel-L2 {ek:.2e}, V {ev:.2e}; prompt part K {rel_l2(k[:, :, :P], cache1[l][0][:, :, :P]):.2e}")
        assert ek <= 1e-2 and ev <= 1e-2
        assert rel_l2(k[:, :, :P], cache1[l][0][:, :, :P]) <= 1e-2
    # the next block: Philox at positions C.., then one forced step on the extended cache
    den.init_canvas(wl.seed)
    t = torch.empty(B * C, dtype=torch.int32, device="cuda")
    den.get_canvas(t, None)
    den.synchronize()
    tok2 = t.cpu().numpy().reshape(B, C)
    assert np.array_equal(tok2, osamp.init_canvas(wl.seed, B, C, V, pos_offset=C))
    assert not np.array_equal(tok2, osamp.init_canvas(wl.seed, B, C, V))
    ref, diag = decoder.decoder_logits(W, tok2, cache1)
    got, _, _ = gpu_step_forced(den, wl, tok2, 0, np.stack(diag["ids"]))
    err = rel_l2(got, ref.reshape(B * C, V))
    print(f"step on the extended cache (P + C = {P + C} keys before the canvas): logits rel-L2 {err:.2e}")
    assert err <= 1e-2
    # the cache is full: one more append does not fit
    import block_denoising_step_b200 as dg
    with pytest.raises(dg.DgenError) as e:
        den.append_canvas()
    assert e.value.status == dg.DGEN_ECAP
    den.close()


def test_generate_equals_the_block_by_block_calls():
    """dgen_generate over three blocks equals driving prefill, T x (step +
    sampler), append from the host, bit for bit; the blocks' canvases differ."""
    wl = WL
    B, C, P, T, n = wl.batch, wl.canvas, wl.prompt_len, 6, 3
    den = make_denoiser(wl, prompt_max=P + (n - 1) * C)
    from synth.device import device_prompt
    prompt = device_prompt(wl)
    out = torch.empty(B * n * C, dtype=torch.int32, device="cuda")
    den.generate(prompt, n, T, wl.seed, out)
    den.synchronize()
    got = out.cpu().numpy().reshape(B, n, C)
    den.prefill_prompt(prompt)
    t = torch.empty(B * C, dtype=torch.int32, device="cuda")
    for j in range(n):
        den.init_canvas(wl.seed)
        for s in range(T):
            den.denoise_step(s, T, None)
            den.sample_commit(s, T, wl.seed)
        den.get_canvas(t, None)
        den.synchronize()
        assert np.array_equal(got[:, j], t.cpu().numpy().reshape(B, C)), j
        if j + 1 < n:
            den.append_canvas()
    assert not np.array_equal(got[:, 0], got[:, 1])
    den.close()
