"""Float64 CPU oracle for the blocked Shampoo step.

TEST INFRASTRUCTURE ONLY.  This package is a plain, slow restatement of what
the method computes, written to check the CUDA path.  Only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline / reference arm may
import it.  The product path (the C-ABI library and its Python binding) never
imports, links or calls anything here, and this package imports nothing from
the product path.

Sources (web pages; cited by title and section/cue):

* "Shampoo optimizer" notes — section "Key Components" (one preconditioner per
  dimension, L in R^{m x m}, R in R^{n x n}) and the simplified matrix-case
  listing (L += G G^T, R += G^T G, W -= eta L^{-1/4} G R^{-1/4}, preconditioners
  updated before the parameters).
* Podcast transcript "Preconditioned optimization without the full matrix
  cost" (Gupta, Koren, Singer 2018) — cue 20 (update rule), cue 22 (the
  two-sided quarter powers equal the Kronecker product form), cue 24 (memory
  and cost), cue 26 (order-k tensors), cue 28 (roots recomputed only every
  20-100 steps; momentum ahead of the preconditioner).
* "DASH: Faster Shampoo via Batched Block Preconditioning and Efficient
  Inverse-Root Solvers" — abstract (blocks stacked into 3D tensors; Newton-DB
  and Chebyshev inverse-root solvers; matrix scaling).
* "SOAP: Improving and Stabilizing Shampoo using Adam" — abstract excerpt
  (Shampoo with the 1/2 power, i.e. p = 2).

Modules:

* ``shampoo``     block partition, statistics, exact inverse p-th root by
                  symmetric eigendecomposition, preconditioned update, and the
                  stepping loop.  Pinned by closed forms (tests/test_oracle_pins.py).
* ``chebyshev``   Chebyshev interpolation of x^{-1/p} and its Clenshaw
                  evaluation on a matrix (the polynomial the Chebyshev solver
                  evaluates).  Pinned against numpy's Chebyshev routines and
                  polynomial exactness.
* ``iter_mirror`` float64 restatements of the coupled-Newton (both correction
                  degrees) and Newton-DB iterations, used only as a diagnostic
                  (never as a parity gate).  Pinned by convergence to the
                  exact root and by the correction's Taylor order.
* ``tensor``      order-k tensor Shampoo (podcast cue 26): per-mode statistics,
                  -1/(2k) roots, mode-wise contractions.  Pinned by the matrix
                  case, a Kronecker brute force and a rank-one closed form
                  (tests/test_oracle_tensor.py).
* ``soap``        SOAP (pith.science SOAP record: Adam run in the eigenbasis of
                  Shampoo's preconditioner, basis recomputed at a fixed
                  frequency).  Pinned by the constant-gradient and first-step
                  closed forms (the latter from the SVD), the reduction to
                  Adam on diagonal statistics, rotation equivariance and
                  eigenvector-sign invariance (tests/test_oracle_soap.py).
"""
from .shampoo import (Block, block_table, inverse_root, accumulate,
                      precondition, ShampooOracle, rel_fro)
from .chebyshev import (chebyshev_nodes, interpolation_coefficients,
                        inverse_root_coefficients, clenshaw_matrix,
                        chebyshev_inverse_root, scaled_interval_lo)
from . import iter_mirror

__all__ = [
    "Block", "block_table", "inverse_root", "accumulate", "precondition",
    "ShampooOracle", "rel_fro", "chebyshev_nodes", "interpolation_coefficients",
    "inverse_root_coefficients", "clenshaw_matrix", "chebyshev_inverse_root",
    "scaled_interval_lo", "iter_mirror",
]
