"""CPU oracle for the recurring decoder update (TEST INFRASTRUCTURE ONLY).

This package is the plain, slow, obviously-correct definition of what the CUDA
path computes: a Llama-style decoder's prompt prefill (which yields the first
token) and its recurring one-token decode step, plus the two-stage streaming
model built from the same primitives.  It runs in float64 with NumPy; the pages
fix no arithmetic precision, so the widest plain type is used and the GPU's
bf16/fp32 rounding sits inside the comparison tolerance.

Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import it.  The product path (``streaming_persistent_sm_b200``) never
does, and this package imports nothing from it.

Parity status per function (what pins each one, besides the code itself):
  round_bf16        - torch's fp32->bf16 conversion on every bf16 tie class
  rmsnorm           - closed form of the output RMS; scale invariance
  rope_*            - 2-D rotation by a known angle; norm preservation;
                      relative-position property; identity at position 0
  softmax           - rows sum to 1; uniform scores give the mean
  silu              - silu(0) = 0; silu(z) - silu(-z) = z
  attention         - one cached token returns v; GQA == MHA with repeated KV
  Decoder           - transformers' LlamaForCausalLM (float64) on the tiny
                      shape; prefill == incremental decode; batch rows
                      independent; paged cache == contiguous cache
  TwoStage          - the composition is this repository's own definition;
                      its implementation is pinned against an independent
                      build of that definition from transformers' float64
                      Llama driven by input vectors (three planted slips in
                      the composition are shown to break the pin)
"""
from .llama import (  # noqa: F401
    KVCache,
    Decoder,
    TwoStage,
    argmax_lowest,
    attention,
    bf16_to_f64,
    rmsnorm,
    rope_apply,
    rope_inv_freq,
    round_bf16,
    silu,
    softmax,
)
