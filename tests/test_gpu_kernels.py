"""GPU parity of the building blocks, through the C ABI, against the fp64 oracle.

* the tcgen05 GEMM core (dgen_gemm_bf16), on CTA pairs (dgen_gemm_bf16_pair)
  and with E4M3 operands (dgen_gemm_e4m3), against fp64 matrix products;
* Philox draws: the initial canvas and the forward process, bit-exact;
* the sampler on GIVEN fp32 logits (dgen_set_logits + dgen_sample_commit):
  integer outputs bit-exact, except a commit-set difference at a confidence
  near-tie (margin < 1e-3), which is counted; conf within 1e-5.
"""
import math

import numpy as np
import pytest

import synth
from oracle import sampler as osamp
from tests.helpers import make_denoiser, rel_l2, ceil_div

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _bf16_dev(bits, shape):
    return torch.from_numpy(bits.view(np.int16).reshape(shape)).view(torch.bfloat16).cuda()


@pytest.mark.parametrize("M,N,K", [(128, 128, 64), (128, 256, 128), (256, 128, 1024), (300, 200, 136),
                                   (1000, 520, 2816), (7, 9, 8), (129, 383, 704)])
def test_gemm_core_matches_fp64_product(M, N, K):
    import block_denoising_step_b200 as dg
    a_bits = synth.normal_bf16(1, 100, 0, M * K, 1.0)
    b_bits = synth.normal_bf16(1, 101, 0, N * K, 1.0)
    a, b = _bf16_dev(a_bits, (M, K)), _bf16_dev(b_bits, (N, K))
    d = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    dg.gemm_bf16(a, b, d, torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    ref = synth.bf16_bits_to_f64(a_bits).reshape(M, K) @ synth.bf16_bits_to_f64(b_bits).reshape(N, K).T
    got = d.cpu().numpy().astype(np.float64)
    assert np.isfinite(got).all()
    # fp32 accumulation of exact bf16 products: error ~ sqrt(K) * 2^-24 relative
    assert np.max(np.abs(got - ref)) <= 1e-5 * math.sqrt(K) * np.max(np.abs(ref)) + 1e-6


@pytest.mark.parametrize("M,N,K", [(256, 256, 64), (256, 512, 2816), (300, 200, 136), (7, 9, 8), (513, 383, 704),
                                   (2048, 768, 256)])
def test_pair_gemm_core_matches_fp64_product(M, N, K):
    """The GEMM core on CTA pairs (tcgen05.mma.cta_group::2, 256 x 256 tiles, each
    CTA holding half of the A rows and half of the B rows): several pair tiles,
    ragged M and N (the rows past M or N of a pair's halves are zero-filled by
    the copies and never stored), against the fp64 product."""
    import block_denoising_step_b200 as dg
    a_bits = synth.normal_bf16(1, 102, 0, M * K, 1.0)
    b_bits = synth.normal_bf16(1, 103, 0, N * K, 1.0)
    a, b = _bf16_dev(a_bits, (M, K)), _bf16_dev(b_bits, (N, K))
    d = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    dg.gemm_bf16_pair(a, b, d, torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    ref = synth.bf16_bits_to_f64(a_bits).reshape(M, K) @ synth.bf16_bits_to_f64(b_bits).reshape(N, K).T
    got = d.cpu().numpy().astype(np.float64)
    assert np.isfinite(got).all()
    assert np.max(np.abs(got - ref)) <= 1e-5 * math.sqrt(K) * np.max(np.abs(ref)) + 1e-6


@pytest.mark.parametrize("M,N,K", [(128, 128, 128), (256, 128, 2816), (300, 200, 144), (7, 9, 16), (129, 383, 704)])
def test_e4m3_gemm_core_matches_fp64_product(M, N, K):
    """The kind::f8f6f4 path of the GEMM core: E4M3 operands (every finite
    encoding drawn uniformly), products exact, fp32 sums."""
    import block_denoising_step_b200 as dg
    rng = np.random.default_rng(M * 7 + N * 3 + K)
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    a8 = rng.choice(codes, size=(M, K)).astype(np.uint8)
    b8 = rng.choice(codes, size=(N, K)).astype(np.uint8)
    dec = lambda x: torch.from_numpy(x).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ref = dec(a8) @ dec(b8).T
    d = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    dg.gemm_e4m3(torch.from_numpy(a8).cuda(), torch.from_numpy(b8).cuda(), d, torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    got = d.cpu().numpy().astype(np.float64)
    assert np.isfinite(got).all()
    assert np.max(np.abs(got - ref)) <= 1e-5 * math.sqrt(K) * np.max(np.abs(ref)) + 1e-6


def _tiny(**kw):
    return synth.WORKLOADS["tiny"].replace(**kw)


@pytest.fixture(scope="module")
def tiny_den():
    wl = _tiny(batch=3, canvas=200)
    den = make_denoiser(wl)
    yield wl, den
    den.close()


def test_initial_canvas_is_the_philox_stream(tiny_den):
    wl, den = tiny_den
    tok = torch.empty(wl.batch * wl.canvas, dtype=torch.int32, device="cuda")
    com = torch.ones(wl.batch * wl.canvas, dtype=torch.uint8, device="cuda")
    for seed in (0, 1, 0xDEADBEEF12345678):
        den.init_canvas(seed)
        den.get_canvas(tok, com)
        den.synchronize()
        ref = osamp.init_canvas(seed, wl.batch, wl.canvas, wl.vocab)
        assert np.array_equal(tok.cpu().numpy().reshape(wl.batch, wl.canvas), ref)
        assert int(com.sum()) == 0


@pytest.mark.parametrize("kappa", [0.0, 0.5, 0.9, 1.0])
def test_forward_process_matches_oracle(tiny_den, kappa):
    wl, den = tiny_den
    x0 = synth.uniform_i32(5, 77, 0, wl.batch * wl.canvas, wl.vocab).reshape(wl.batch, wl.canvas)
    xt = torch.empty(wl.batch * wl.canvas, dtype=torch.int32, device="cuda")
    den.forward_noise(torch.from_numpy(x0.reshape(-1)).cuda(), kappa, 1234, 3, xt)
    den.synchronize()
    k32 = float(np.float32(kappa))
    ref = osamp.forward_noise_tokens(x0, k32, 1234, wl.vocab, step=3)
    assert np.array_equal(xt.cpu().numpy().reshape(wl.batch, wl.canvas), ref)


def _structured_logits(B, C, V, seed):
    """Gaussian logits with planted structure: exact ties at the maximum, one-hot
    rows, rows with equal confidence."""
    L = synth.logits_f32(seed, 0, B * C, V, std=2.0).reshape(B, C, V).copy()
    rng = np.random.default_rng(seed)
    for b in range(B):
        for i in rng.choice(C, size=C // 8, replace=False):       # tie at the max, lower index must win
            j = int(np.argmax(L[b, i]))
            j2 = int(rng.integers(0, V))
            L[b, i, j2] = L[b, i, j]
        for i in rng.choice(C, size=4, replace=False):            # one-hot rows
            L[b, i] = 0.0
            L[b, i, int(rng.integers(0, V))] = 30.0
        src = int(rng.integers(0, C))                              # identical rows -> identical confidence
        for i in rng.choice(C, size=3, replace=False):
            L[b, i] = L[b, src]
    return L


@pytest.mark.parametrize("s,T", [(0, 12), (5, 12), (11, 12), (0, 4), (3, 4), (17, 32)])
def test_sampler_on_given_logits_matches_oracle(tiny_den, s, T):
    wl, den = tiny_den
    B, C, V = wl.batch, wl.canvas, wl.vocab
    seed = 99 + s
    L = _structured_logits(B, C, V, seed=s * 7 + T)
    tok0 = synth.uniform_i32(seed, 3, 0, B * C, V).reshape(B, C)
    m = ceil_div(C, T)
    com0 = np.zeros((B, C), dtype=bool)
    rng = np.random.default_rng(T * 100 + s)
    for b in range(B):
        com0[b, rng.choice(C, size=min(C, s * m), replace=False)] = True
    den.set_canvas(torch.from_numpy(tok0.reshape(-1).astype(np.int32)).cuda(),
                   torch.from_numpy(com0.reshape(-1).astype(np.uint8)).cuda())
    den.set_logits(torch.from_numpy(L.reshape(-1)).cuda(), s, T)
    conf = torch.empty(B * C, dtype=torch.float32, device="cuda")
    den.sample_commit(s, T, seed, conf)
    tok = torch.empty(B * C, dtype=torch.int32, device="cuda")
    com = torch.empty(B * C, dtype=torch.uint8, device="cuda")
    den.get_canvas(tok, com)
    den.synchronize()
    tok = tok.cpu().numpy().reshape(B, C)
    com = com.cpu().numpy().reshape(B, C).astype(bool)
    tau = osamp.tau_of_step(s, T, wl.tau_max, wl.tau_min)
    rtok, rcom, info = osamp.sample_commit(L.astype(np.float64), tok0, com0, s, T, seed, tau)
    assert np.max(np.abs(conf.cpu().numpy().reshape(B, C) - info["conf"])) < 1e-5
    assert np.array_equal(tok[com0], tok0[com0]) and com[com0].all()         # frozen
    near_ties = 0
    for b in range(B):
        if not np.array_equal(com[b], rcom[b]):
            assert info["margin"][b] < 1e-3, (b, info["margin"][b])
            near_ties += 1
            same = com[b] == rcom[b]
            assert np.array_equal(tok[b][same & com[b]], rtok[b][same & com[b]])
        else:
            assert np.array_equal(tok[b], rtok[b])
    print(f"sampler s={s} T={T}: near-tie commit differences in {near_ties}/{B} canvases")


@pytest.mark.parametrize("T", [4, 12, 32])
def test_one_hot_logits_recover_the_target_on_gpu(tiny_den, T):
    wl, den = tiny_den
    B, C, V = wl.batch, wl.canvas, wl.vocab
    target = synth.target_canvas(wl.replace(batch=B, canvas=C), stream=T)
    seed = 4242
    den.init_canvas(seed)
    tok = torch.empty(B * C, dtype=torch.int32, device="cuda")
    com = torch.empty(B * C, dtype=torch.uint8, device="cuda")
    prev_tok, prev_com = None, None
    rng = np.random.default_rng(T)
    for s in range(T):
        L = np.zeros((B, C, V), dtype=np.float32)
        np.put_along_axis(L, target[..., None], rng.uniform(1, 20, size=(B, C, 1)).astype(np.float32), axis=2)
        den.set_logits(torch.from_numpy(L.reshape(-1)).cuda(), s, T)
        den.sample_commit(s, T, seed)
        den.get_canvas(tok, com)
        den.synchronize()
        t, c = tok.cpu().numpy().reshape(B, C), com.cpu().numpy().reshape(B, C).astype(bool)
        if prev_com is not None:
            assert np.array_equal(t[prev_com], prev_tok[prev_com]) and c[prev_com].all()
            newly = c.sum(axis=1) - prev_com.sum(axis=1)
            expect = np.minimum(ceil_div(C, T), C - prev_com.sum(axis=1)) if s < T - 1 else C - prev_com.sum(axis=1)
            assert np.array_equal(newly, expect)
        prev_tok, prev_com = t, c
    assert prev_com.all()
    assert np.array_equal(prev_tok, target)
