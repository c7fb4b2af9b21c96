"""CPU oracle for the low-bit routed-expert MoE FFN layer.

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the test suite, the smoke check of
the package entry point and the benchmark's CPU-baseline leg may import or run
anything under ``oracle/``.  The product path (the CUDA library and its Python
binding) never does, and shares no code, table or constant generator with it.

The oracle is plain, slow and written to be checked by eye: numpy, float64 for
every floating-point accumulation, with the exact IEEE fp32 / bf16 steps spelled
out wherever a float decides an integer (a quantised code, a routing choice).
Each function names the passage it follows on the source pages:

* "Every Expert Counts: ExactMoE for Memory-Efficient W4A16 Inference", abstract
  -- symmetric group-128 four-bit routed experts, BF16 router, unchanged top-k.
* "PagedMoE: Cross-Precision Expert Caching for Token-Level Dynamic Precision in
  SSD-Resident MoE Inference", abstract -- bitplane layout, lower precisions are
  prefixes of higher ones, prefix length from the routing weights.
* "MatMoE: Matryoshka Mixture-of-Experts with Dynamic Mixed-Precision
  Quantization for Efficient Inference", abstract -- floor-and-compensation
  quantisation, per-expert bit-width from routing scores.
* "MoET in FP4 MoE Inference" (Q&A page) -- NVFP4 named, router kept at high
  precision, FP4/INT4 expert weights.

Where the pages leave a step open, the docstring says which reading is taken
("reading R<n>"); the readings are listed together in the design notes.

Parity status: every function here is pinned by ``tests/test_oracle_*.py``
against closed forms, brute force, library routines or hand-derived worked
examples.  Nothing is "parity unpinned".
"""
