"""CPU oracle for MLA prefill attention -- TEST INFRASTRUCTURE ONLY.

A plain, slow, fp64 restatement of what the CUDA path computes.  Only the
test suite, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
may import it; the product library never does, and there is no CPU
fallback to it.  It shares no code with the CUDA path: both take their
inputs from ``mla_synth`` and nothing else.

Functions (all pinned by tests in ``tests/test_oracle_pins.py``):

* ``dense_prefill``   -- varlen (causal or not) attention with an LSE.
* ``attn_merge``      -- log-sum-exp merge of two partial results.
* ``sparse_prefill``  -- absorbed top-k sparse attention over a shared
  latent cache.
* ``dense_prefill_sinks`` -- ``dense_prefill`` with one attention-sink logit
  per head.
* ``e4m3_quantize`` / ``e4m3_decode`` -- the FP8 (e4m3) output encoding
  with a static scale.
"""
from .attention import (  # noqa: F401
    bf16_bits_to_f64,
    visible_key_count,
    dense_prefill,
    dense_prefill_sinks,
    e4m3_decode,
    e4m3_quantize,
    attn_merge,
    sparse_prefill,
    dense_flops,
    sparse_flops,
)
