"""fp64 CPU oracle for the joint text+image attention hot path.

TEST INFRASTRUCTURE ONLY.  This package is the plain, slow, obviously correct
statement of what the CUDA library computes, used to check it.  Only the
tests, the smoke check and the benchmark's CPU-baseline leg may import it;
the product path (the C-ABI library and its Python binding) never calls it
and shares no code, table or helper with it.

Modules:
  formats    round-to-nearest-even into bf16 / fp16 and OCP FP8 E4M3
  rope       three-axis (t, h, w) rotary embedding
  attention  softmax(q~ k~^T / sqrt(D)) v and its log-sum-exp, per (b, h)
  fp8        per-64-token block quantisation to E4M3 with fp32 scales
  merge      combination of partial (O, LSE) results over disjoint key sets

Every function is pinned by tests/test_oracle_*.py against brute force at 50
digits, library routines, closed forms and invariants (see those files).
"""
from . import formats, rope, attention, fp8, merge  # noqa: F401
