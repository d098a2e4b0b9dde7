"""Float64 CPU oracle for the batched block-Shampoo (DASH) step.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this package:
only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
arm of ``bench.py`` may call it.  It shares no code, tables or constants with
the CUDA library; the only thing both sides consume is the seeded input
generator module ``matrix_inverse_roots_stack_b200.workloads``, which holds no
arithmetic of the method.

Source of the method: "DASH: Faster Shampoo via Batched Block Preconditioning
and Efficient Inverse-Root Solvers" (howistudyai.com explainer of
arXiv 2602.02016), sections "Building blocks", "High-level flow" and
"Step-by-step".  Where that page is silent the plainest reading is taken and
named in each docstring.

Modules
-------
roots      inverse fourth roots: exact (eigendecomposition, "level 1"),
           truncated-method spectral evaluation ("level 2"), and the
           step-by-step matrix recurrences ("level 3"); power iteration;
           Chebyshev fit.
jacobi     a cyclic Jacobi eigensolver written out by hand (independent of
           LAPACK) for brute-force pins on tiny matrices.
step       blocking, factor EMA, preconditioning, Adam grafting, the full step.

Parity status: every function here is pinned by a ``-m "not gpu"`` test
against closed forms, invariants, a library routine or brute force (see
tests/test_oracle_*.py).  No function is "parity unpinned".
"""

from . import roots, jacobi, step  # noqa: F401
