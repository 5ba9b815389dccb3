"""Plain, slow, fp64 CPU oracle for Reduced Matrix Multiplication (RMM).

TEST INFRASTRUCTURE.  Only the test suite, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference leg may import anything in this package.
It shares no code with the CUDA library (no headers, kernels, helpers or
tables); the only thing the two sides share is the seeded input generator in
``workloads``, which holds none of the method's arithmetic.

Modules:
  rmm           scores, top-k selection and the reduced product
  attention     reduced attention (head_dim reduction in QK^T, token
                reduction in PV)
  decode_attention  the same for one new query token over a KV cache
  block         products sharing one selection; a gated MLP block with every
                product reduced
  conditioning  deterministic score-gap widening of generated inputs, so the
                fp32 GPU ranking and the fp64 oracle ranking must agree

Parity status: every function is pinned by the ``-m "not gpu"`` tests in
``tests/test_oracle_*.py`` (closed forms, brute force, special cases that
reduce to library routines, error bounds).  The attention READINGS R1-R6
(see ``oracle.attention``) are choices where the page is silent; the
functions are pinned to those readings, and the readings themselves are
"parity unpinned" against the page.
"""
from . import rmm, attention, decode_attention, block, conditioning  # noqa: F401
from .rmm import (k_from_rho, column_sq_norms, column_norms, topk_indices,  # noqa: F401
                  reduced_matmul, dense_matmul, rmm as rmm_path, decode,
                  dequantize_w8, reduced_matmul_w8, rmm_w8)
from .attention import reduced_attention, attention_head, kv_head_of  # noqa: F401
from .decode_attention import decode_attention_head  # noqa: F401
