"""CPU oracle for the HEAL hot path -- TEST INFRASTRUCTURE, not product code.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its ``cpu_baseline``
leg and ``--impl reference`` arm) may import or run anything in this package.  The
product path (``error_compensated_gemm_b200``) never imports it and shares no code,
table or constant generator with it; both sides only receive the same seeded
inputs from ``synthetic/``.

Everything here is plain numpy (float64 / int64) and, for the 16-bit roundings,
the numpy / PyTorch CPU dtype conversions.  It is deliberately slow and unblocked:
each function is the definition of what the method computes, or the method's steps
in the order the pages give them.

Sources (all five pages describe the same paper, "Demystifying Numerical
Instability in LLM Inference: Achieving Reproducible Inference for Mission-Critical
Tasks with HEAL", arXiv 2606.21023):
  * the authors' v2 abstract (paperdot tracker page);
  * the gist.science technical summary, sections "1. Root Cause Analysis",
    "2.A Mitigating Attention Truncation via INT16 Quantization" and
    "2.B Mitigating GEMM Truncation via Algebraic Error Compensation".

Parity status per function is listed in each module header.  Every function is
pinned by ``tests/test_oracle_*.py`` to something other than itself (closed forms,
exact rational brute force, special cases, printed constants of the pages).
"""
