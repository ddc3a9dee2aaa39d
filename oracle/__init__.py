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
  lqlora    LQ-LoRA initialisation: alternating truncated SVD and NF-k quantisation
  allocation LQ-LoRA's budgeted (bits, block) choice per matrix (multiple-choice knapsack)
  loqa      LoQA: gradients of the loss with respect to the INT4 scale and zero point

Parity-pinned: every function is checked in ``tests/test_oracle_*.py`` against
closed forms, invariants, brute force on tiny inputs, library routines or the
pages' printed figures (the allocation against exhaustive search and the two
closed-form ends of the budget; the initialisation against constructed SVDs, an
exactly low-rank matrix and its zero-iteration case; the LoQA gradients against
finite differences of the loss, brute force and the pooled-adapter identity of a
zero-point shift).  The pages print no worked example for the two LQ-LoRA parts
or for LoQA, so what they pin is the reading of the abstract that these modules
state, not numbers from the pages.
"""

from . import numerics, codebook, quantize, layer, storage, lqlora, allocation, loqa  # noqa: F401
