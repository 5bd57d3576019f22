"""The C-ABI library loads and exports every entry point include/dgen.h declares;
host-side argument checks (no GPU needed: they return before any CUDA call)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared(header="dgen.h"):
    src = open(os.path.join(ROOT, "include", header)).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(dgen_[a-z_0-9]+)\s*\(", src)))


def test_header_declares_the_boundary_calls():
    names = _declared()
    for must in ("dgen_create", "dgen_prefill_prompt", "dgen_denoise_step", "dgen_sample_commit",
                 "dgen_generate_block", "dgen_destroy"):
        assert must in names


def test_library_exports_every_declared_symbol():
    import block_denoising_step_b200 as dg
    lib = ctypes.CDLL(dg.LIB_PATH)
    missing = [n for n in _declared() if not hasattr(lib, n)]
    assert not missing, missing
    assert set(dg.EXPORTED) == set(_declared())


def test_probe_library_exports_its_header_and_the_product_library_does_not():
    import block_denoising_step_b200 as dg
    probes = _declared("dgen_probe.h")
    assert set(probes) == set(dg.PROBE_EXPORTED)
    lib = dg.probe_lib()
    assert all(hasattr(lib, n) for n in probes)
    product = ctypes.CDLL(dg.LIB_PATH)
    assert not any(hasattr(product, n) for n in probes)


def test_every_header_is_covered_by_a_library():
    headers = sorted(f for f in os.listdir(os.path.join(ROOT, "include")) if f.endswith(".h"))
    assert headers == ["dgen.h", "dgen_probe.h"]


def test_status_strings():
    import block_denoising_step_b200 as dg
    assert dg._lib.dgen_status_str(0) == b"ok"
    assert b"invalid" in dg._lib.dgen_status_str(-1)
    assert dg._lib.dgen_status_str(12345) == b"unknown status"


def _cfg(**kw):
    import block_denoising_step_b200 as dg
    base = dict(n_layers=2, d_model=256, n_q_heads=4, n_kv_heads=4, head_dim=64, n_experts=8, top_k=2,
                expert_width=512, shared_width=0, vocab=4096, batch=1, prompt_max=64, canvas=256)
    base.update(kw)
    return dg.ModelConfig(**base)


@pytest.mark.parametrize("bad", [dict(head_dim=96), dict(d_model=200), dict(n_q_heads=6, n_kv_heads=4),
                                 dict(top_k=9), dict(expert_width=100), dict(vocab=1000), dict(canvas=2048),
                                 dict(n_experts=300, top_k=2), dict(tau_max=0.0), dict(batch=0),
                                 dict(shared_width=9 * 512)])
def test_create_rejects_bad_config_without_touching_the_gpu(bad):
    import block_denoising_step_b200 as dg
    with pytest.raises(dg.DgenError) as e:
        dg.Denoiser(_cfg(**bad), 0x1000, 0x1000, [{k: 0x1000 for k in dg.LAYER_FIELDS}] * 2)
    assert e.value.status == dg.DGEN_EINVAL


def test_create_rejects_null_or_misaligned_weights():
    import block_denoising_step_b200 as dg
    good = {k: 0x1000 for k in dg.LAYER_FIELDS}
    with pytest.raises(dg.DgenError) as e:
        dg.Denoiser(_cfg(), 0x1000, 0x1000, [good, dict(good, w_o=None)])
    assert e.value.status == dg.DGEN_EINVAL
    with pytest.raises(dg.DgenError) as e:
        dg.Denoiser(_cfg(), 0x1008, 0x1000, [good, good])
    assert e.value.status == dg.DGEN_EINVAL


def test_calls_on_null_handle_are_einval():
    import block_denoising_step_b200 as dg
    L = dg._lib
    assert L.dgen_denoise_step(None, 0, 12, None) == dg.DGEN_EINVAL
    assert L.dgen_sample_commit(None, 0, 12, 0, None) == dg.DGEN_EINVAL
    assert L.dgen_prefill_prompt(None, None, 4) == dg.DGEN_EINVAL
    assert L.dgen_destroy(None) == dg.DGEN_OK
    assert L.dgen_launch_count(None) == -1
    assert L.dgen_gemm_bf16(None, None, None, 128, 128, 7, None) == dg.DGEN_EINVAL
