"""Float64 oracle: blocked Shampoo statistics, exact inverse roots, update.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Everything here is float64 on the CPU.  Inputs are exact float64 casts of the
fp32 / bf16 buffers the GPU receives.  Roots are exact (symmetric
eigendecomposition), not iterative: the iterative solvers of the CUDA path are
ways of reaching this same result faster.

Readings of the pages that this file fixes:

* Blocking: each m x n weight is cut into a ceil(m/B) x ceil(n/B) grid of
  blocks aligned at multiples of B; the last block row / column is ragged.
  Block (i, j) owns its own left and right statistics (DASH abstract: blocks
  stacked into 3D tensors).  The oracle keeps ragged blocks at their real
  r x c extent (no padding).
* Statistics: L <- beta L + G G^T, R <- beta R + G^T G with no (1 - beta)
  factor; beta = 1 is the plain running sum of the "Shampoo optimizer" notes'
  matrix-case listing.
* Damping: statistics start at zero and the root is taken of (L + eps I).
  With beta = 1 this is identical to the notes' initialisation L = eps I.
* Order within a step: accumulate statistics, then (every ``refresh_every``
  steps, counting from step 0) recompute the roots, then apply the update
  with the current roots (podcast cue 28: roots refreshed only every so many
  steps; the notes' listing: preconditioners before parameters).
* No grafting.  Momentum is off by default (the update uses the raw
  gradient); ``momentum = alpha > 0`` folds ordinary momentum in before
  preconditioning (podcast cue 28: momentum 0.9 ahead of the
  preconditioner): per block M <- alpha M + G from M = 0, the statistics still
  take the raw G, and the update is XL M XR.
* The diagonal variant for dimensions above about 1200 (podcast cue 28) never
  applies to blocks, whose sides are at most the block size (<= 1024).
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Sequence, Tuple

import numpy as np


@dataclass(frozen=True)
class Block:
    """One B x B tile of one weight: rows [row0, row0+r), cols [col0, col0+c)."""

    param: int
    row0: int
    col0: int
    r: int
    c: int


def block_table(shapes: Sequence[Tuple[int, int]], block: int) -> List[Block]:
    """Partition every weight into B x B blocks, in (param, block row, block
    column) order.  DASH abstract: preconditioner blocks stacked into 3D
    tensors; the last row / column of blocks keeps its real (ragged) size."""
    out = []
    for pi, (m, n) in enumerate(shapes):
        for i0 in range(0, m, block):
            for j0 in range(0, n, block):
                out.append(Block(pi, i0, j0, min(block, m - i0), min(block, n - j0)))
    return out


def accumulate(L: np.ndarray, R: np.ndarray, G: np.ndarray, beta: float):
    """Left and right statistics of one block ("Shampoo optimizer" notes,
    matrix-case listing; podcast cue 20): L' = beta L + G G^T and
    R' = beta R + G^T G."""
    G = np.asarray(G, dtype=np.float64)
    return beta * L + G @ G.T, beta * R + G.T @ G


def inverse_root(A: np.ndarray, p: int, eps: float) -> np.ndarray:
    """Principal inverse p-th root of the damped statistic, (A + eps I)^{-1/p}.

    "Shampoo optimizer" notes (the listing raises L and R to the -1/4 power;
    p = 4), SOAP abstract (the 1/2-power variant; p = 2).  Computed exactly by
    the symmetric eigendecomposition A = Q diag(lam) Q^T.  A is symmetrised and
    eigenvalues are clamped at 0 before eps is added: both are no-ops for an
    exact Gram matrix and only absorb rounding in fp32 statistics.
    """
    A = np.asarray(A, dtype=np.float64)
    S = 0.5 * (A + A.T)
    lam, Q = np.linalg.eigh(S)
    lam = np.maximum(lam, 0.0) + eps
    return (Q * (lam ** (-1.0 / p))[None, :]) @ Q.T


def precondition(XL: np.ndarray, G: np.ndarray, XR: np.ndarray) -> np.ndarray:
    """Preconditioned gradient P = L^{-1/p} G R^{-1/p} (notes' listing;
    podcast cue 20: the gradient sandwiched between the two roots)."""
    return XL @ np.asarray(G, dtype=np.float64) @ XR


def rel_fro(x: np.ndarray, ref: np.ndarray) -> float:
    """Relative Frobenius error ||x - ref||_F / ||ref||_F (0 if both are 0)."""
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref)
    num = np.linalg.norm(x - ref)
    if den == 0.0:
        return 0.0 if num == 0.0 else float("inf")
    return float(num / den)


class ShampooOracle:
    """Blocked Shampoo in float64, one step at a time.

    ``step(grads)`` follows the notes' loop body for every block: update the
    statistics, refresh the roots when ``t % refresh_every == 0`` (t counted
    from 0), then W_b <- W_b - lr * XL_b G_b XR_b.  It returns the list of
    per-block preconditioned gradients P_b of this step, which is what the
    update subtracts (scaled by lr).

    ``blocks`` may restrict the oracle to a subset of block indices (blocks are
    independent), which is how large workloads are sampled.
    """

    def __init__(self, shapes, block, beta, eps, lr, root_p=4, refresh_every=1,
                 weights=None, blocks: Sequence[int] | None = None, momentum: float = 0.0):
        self.shapes = [tuple(s) for s in shapes]
        self.B = int(block)
        self.beta = float(beta)
        self.eps = float(eps)
        self.lr = float(lr)
        self.p = int(root_p)
        self.refresh_every = int(refresh_every)
        self.table = block_table(self.shapes, self.B)
        self.active = list(range(len(self.table))) if blocks is None else list(blocks)
        if weights is None:
            # "Shampoo optimizer" notes' listing: W starts at zeros(m, n).
            self.W = [np.zeros(s) for s in self.shapes]
        else:
            self.W = [np.array(w, dtype=np.float64) for w in weights]
        self.L = {b: np.zeros((self.table[b].r,) * 2) for b in self.active}
        self.R = {b: np.zeros((self.table[b].c,) * 2) for b in self.active}
        self.XL = {b: None for b in self.active}
        self.XR = {b: None for b in self.active}
        self.momentum = float(momentum)
        self.M = {b: np.zeros((self.table[b].r, self.table[b].c)) for b in self.active}
        self.t = 0

    def block_of(self, grads, b):
        blk = self.table[b]
        g = grads[blk.param]
        return np.asarray(g[blk.row0:blk.row0 + blk.r, blk.col0:blk.col0 + blk.c],
                          dtype=np.float64)

    def step(self, grads) -> dict:
        refresh = (self.t % self.refresh_every) == 0
        P = {}
        for b in self.active:
            G = self.block_of(grads, b)
            self.L[b], self.R[b] = accumulate(self.L[b], self.R[b], G, self.beta)
            if refresh:
                self.XL[b] = inverse_root(self.L[b], self.p, self.eps)
                self.XR[b] = inverse_root(self.R[b], self.p, self.eps)
            if self.momentum > 0.0:
                self.M[b] = self.momentum * self.M[b] + G
                P[b] = precondition(self.XL[b], self.M[b], self.XR[b])
            else:
                P[b] = precondition(self.XL[b], G, self.XR[b])
            blk = self.table[b]
            self.W[blk.param][blk.row0:blk.row0 + blk.r,
                              blk.col0:blk.col0 + blk.c] -= self.lr * P[b]
        self.t += 1
        return P
