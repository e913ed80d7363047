"""CPU oracle for the NVFP4 MoE train/rollout alignment path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call,
link or execute this package: it is used by ``tests/``, by
``__graft_entry__.smoke()`` (to check one small CUDA run) and by the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py``.  It shares no
code with the CUDA library and never imports it.

What it is: a plain, slow, obviously-correct restatement of what the method
computes, in float64 numpy.  Every step that the method performs in float32
is emulated by computing it in float64 and rounding to float32 once; for a
single +, -, *, / on float32 operands that double rounding gives the
correctly-rounded float32 result, because 53 >= 2*24 + 2 (S. A. Figueroa,
"When is double rounding innocuous?", SIGNUM Newsletter 30(3), 1995).

Sources (cited by short tag in each docstring):

* [QUADS-fr] "QUADS: Stabilizing NVFP4 Reinforcement Learning for MoE via
  QUantization-error Alignment across Dual Sides", gist.science French
  summary, "Résumé Technique" sections 1-5.
* [QUADS-es] the same paper, gist.science Spanish summary, sections 1-5.
* [TRACE] "TRACE : un entraînement conscient de la quantification guidé par
  le rollout pour le RL en FP4 des modèles MoE", sns.style article, sections
  "L'idée centrale de TRACE" and "Fonctionnement, côté ingénierie".
* [format] the public definition of the NVFP4 format: E2M1 elements, one
  E4M3 scale per 16 consecutive elements, one FP32 per-tensor scale.

Modules:
  formats  -- E2M1 / E4M3 / BF16 / FP32 rounding, nibble packing, scale tiling
  nvfp4    -- quantize, dequantize, residual channels, calibration, fake-quant
  moe      -- router top-k, permutation, grouped GEMM + compensation,
              SwiGLU, combine, one MoE layer
  trace    -- rollout record export and trainer replay
  layer    -- one MoE layer on both sides, composed from the steps above
  stack    -- router projection and residual connection between layers

Pins: every function here is checked in ``tests/test_oracle_*.py`` against
brute force, closed forms, library routines or invariants.  Functions with
no such pin are listed as "parity unpinned" below.

Parity unpinned: none.  ``moe.per_token_gap`` is a reported diagnostic: its
formula is pinned by closed forms, and no page fixes the value it measures.
"""
