"""Plain fp64 CPU oracle of the block denoising step -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its cpu_baseline
leg and its reference arm) may import anything from this package.  The product
path (the CUDA library and its Python binding) never imports, calls or links it,
and this package imports nothing from the product path: the two share no code.
The only common dependency is ``synth`` (seeded input generation, no method
arithmetic).

What it computes, and the passages it follows (DiffusionGemma; pages cited by
title and section):

* ``philox``   -- Philox4x32-10 counter-based generator (Salmon, Moraes, Dror &
  Shaw, "Parallel random numbers: as easy as 1, 2, 3", SC'11), the source of the
  method's random draws (initial canvas, uniform re-noise, forward noising).
* ``sampler``  -- the uniform-state forward process (hyper.ai digest, Method,
  eq. 1), the tempered softmax (Method, eq. 4 first line), the linear temperature
  schedule 0.8 -> 0.4 (Method, sampler paragraph; Experiment, sampler settings),
  and the confidence-ranked commit with uniform re-noise of the rest
  (alphasignal.ai article, "How text diffusion actually works", step 2).
* ``decoder``  -- the decoder logits L_t = Decoder(x_t, z_t, H) (Method, eq. 3)
  of a pre-norm MoE transformer: non-causal attention of the canvas over
  [prompt cache ; canvas] (Method, three-stage pipeline), top-k routed gated-GELU
  experts, tied LM head; and the causal prompt pass that builds the cache.

Rounding: everything is fp64, except that the tensors entering each GEMM or
attention on the GPU path (normed activations, rotated q/k and v, attention
output, expert activations, final normed state) are rounded to bf16 at the same
points, so that both sides see identical bf16-rounded inputs.
"""
from . import philox, numerics, sampler, decoder  # noqa: F401
