"""Plain CPU oracle for the TurboQuant hot path (test infrastructure only).

This package is test infrastructure, not product code. Only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
it; the library and its Python binding never do, and the oracle imports
nothing from them. It shares no code, tables or constants with the CUDA path:
the only common dependency is the seeded input generator module ``workloads``.

Everything is numpy / scipy in fp64. It follows the method as the pages state
it, step by step, with no blocking, fusion or reordering:

* ``codebook``  -- Lloyd-Max scalar quantiser for the density of one coordinate
  of a randomly rotated unit vector, f_d(x) ~ (1 - x^2)^((d-3)/2) on [-1, 1]
  (aiboss88 page, "technical principles": rotated coordinates follow a Beta
  distribution and a Lloyd-Max / continuous 1-D k-means codebook is
  precomputed per coordinate; techblog-plum page, step 1: computed once, no
  inference overhead).
* ``quant``     -- Algorithm 1 (rotate, per-coordinate nearest centroid, pack,
  fp16 norm) and Algorithm 2 (Algorithm 1 at b-1 bits plus the 1-bit QJL sign
  of S times the residual, with the residual norm) and their dequantisation
  (ai-navigate-news page, "how it works"; aiboss88 page, "two-stage residual
  correction").
* ``attention`` -- inner-product scores from dequantised vectors, softmax
  decode attention over the dequantised cache, top-k.

Parity status of each function is stated in its module docstring.
"""
