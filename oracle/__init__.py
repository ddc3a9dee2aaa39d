"""Plain CPU oracle for the quantised-base + LoRA linear (test infrastructure).

This package is TEST INFRASTRUCTURE.  It restates, slowly and in the order the
pages give them, the steps the CUDA library computes, so the tests can compare
the two element by element.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it; the
product path (the C-ABI library and its Python binding) never does, and there is
no CPU fallback anywhere in the product.

It shares no code, table or constant generator with the CUDA path: the NF-k
codebook here comes from ``scipy.stats.norm.ppf``; the library derives its own
table with its own inverse-normal routine.  numpy / scipy are used for
elementwise fp32 arithmetic (IEEE round-to-nearest), fp64 matrix products and
the normal quantile function; nothing is blocked, fused or reordered beyond the
definitions.

Modules
  numerics  bf16 / fp16 rounding, OCP FP8 E4M3 encode/decode
  codebook  NF-k levels (quantile construction)
  quantize  NF-k blockwise quantiser + double quantisation, bit packing, dequant;
            INT4 group-wise quantiser (QA-LoRA) and the adapter merge
  layer     forward / backward of the quantised-base + LoRA linear, group pooling, SwiGLU
  storage   bits-per-parameter and byte accounting of the formats

Parity-pinned: every function is checked in ``tests/test_oracle_*.py`` against
closed forms, invariants, brute force on tiny inputs, library routines or the
pages' printed figures.  Parity unpinned: the LQ-LoRA per-matrix choice of
(bits, block) beyond its storage arithmetic (the pages give no worked example).
"""

from . import numerics, codebook, quantize, layer, storage  # noqa: F401
