"""Plain, slow fp64 CPU oracle for the DSA token indexer and ADIndex's group bank / refine.

TEST INFRASTRUCTURE ONLY. Nothing on the product path imports, calls or executes this
package: only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may use it. It shares no code with the CUDA
path (no kernels, headers, helpers or constant tables); the two meet only in the seeded
input generators, which hold none of the method's arithmetic.

Source of every definition: "ADIndex: Layer-Adaptive Sparse Attention Indexing via
Group-Level Distillation" (arXiv 2611.12956v1), cited below as "ADIndex" with its section,
equation or table.

Modules
  fp_formats  exact decoding of bf16 and FP8-e4m3 codes to float64
  indexer     Eq. (1) scores, Eq. (2) Top-K, Eq. (13) token bank, Eq. (14) refinement,
              flat and bank-reuse decode
  cost_model  score-evaluation counts of the same group plan (Appendix A, Table 5)

Parity status: every function is pinned by a ``-m "not gpu"`` test (hand values, closed
forms, brute force, invariants, Table 5) except where its docstring says "parity unpinned".
"""

from . import fp_formats, indexer, cost_model  # noqa: F401
