"""CPU oracle for the scaled quantized linear-layer GEMM — TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The
product path (the C-ABI library and its Python binding) never calls it, and
it shares no code, table or constant generator with the CUDA sources.

What it computes (numpy, fp64 unless a quantisation decision is taken, where
it uses fp32 exactly as the method's dynamic quantiser does):

* y = dequant(A_q) . dequant(W_q)^T rounded to bf16, for the four formats of
  the linear backend in "Helion in the vLLM backend" (ai-radar.it, first
  paragraph: FP8_Dynamic, W8A8_INT8, Block_FP8) and the NVFP4 ``mm_fp4`` GEMM
  of FlashInfer PR 3948 ("perf(gemm): update mm_fp4 cute-dsl tactic
  heuristic ...", benchmark command with ``--use_nvfp4``);
* the dynamic quantisers that produce A_q and W_q (amax -> scale -> codes);
* the Split-K and Swap-AB rewrites of the same contraction ("Helion in the
  vLLM backend", second paragraph), which must leave the exact sums unchanged.

Modules: ``formats`` (bit-level decode tables, nearest-even encoders, bf16
rounding), ``quant`` (the four quantisers), ``gemm`` (the contraction and its
epilogues).  Every function that has no independent pin says "parity
unpinned" in its docstring; the pins live in ``tests/test_oracle_*.py``.
"""
from . import formats, quant, gemm  # noqa: F401

__all__ = ["formats", "quant", "gemm"]
