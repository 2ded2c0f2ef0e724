"""Reference oracle for the AWQ int4 weight-only decode step.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import anything
from this package.  The product path (the CUDA library and its Python binding)
never imports, links or executes it, and this package imports nothing from the
product package: the two share no code, tables, constants or helpers.  Inputs
reach both sides from the seeded generators only.

Everything here is plain, slow and written to be checked by eye against the
pages that define the method:

* ``quant``  -- RTN min/max asymmetric int4 quantizer, canonical packing,
  unpacking and exact dequantization
  (ATLAS-OLMo-3-32B-Think-v4 model card, "Quantization recipe").
* ``model``  -- the decoder definition in float64: RMSNorm, QK-norm over the
  full projections, RoPE with YaRN on the full-attention layers, GQA with a
  [SWA, SWA, SWA, full] layer pattern, SwiGLU, post-norm residuals, lm_head,
  greedy argmax (ATLAS model card "Architecture deep-dive"; Olmo 3 32B,
  "Every architecture field"; LLM Architecture KB "OLMo 3 32B", "Techniques
  used"; archdb "Olmo-3-1125-32B" field list).
* ``counts`` -- KV-cache bytes, decode/prefill FLOPs and parameter counts
  (Olmo 3 32B, "Modelled costs"; archdb KV fields; ATLAS model card "Why the
  3:1 SWA layout matters for serving").
* ``brute``  -- a second, loop-by-loop float64 implementation of one layer on
  tiny shapes, used to pin ``model`` against transposed operands, dropped
  terms and wrong indices.
* ``sampling`` -- temperature / top-p (nucleus) sampling of one token with the
  draw passed in (ATLAS model card, "Benchmarks" and "Prompting guide for
  Think models": temperature 0.6, top-p 0.95).

Parity status per function is stated in each module header.  Every function is
pinned by a ``-m "not gpu"`` test.  The decoder's conventions that the pages
state only in prose (rotation pairing, YaRN ramp, where RMSNorm adds eps, the
final norm, the window counting the current token) are pinned, besides the
invariants listed in ``model``, against the independent OLMo 3 implementation
of the ``transformers`` package run in float64 on the same weights.
"""
