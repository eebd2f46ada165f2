"""Float64 oracle for order-k tensor Shampoo (the next row after the matrix case).

TEST INFRASTRUCTURE ONLY (see the package docstring).

Podcast transcript "Preconditioned optimization without the full matrix
cost", cue 26 (the paper's general-order algorithm):
  * one preconditioning matrix per dimension of the gradient tensor, each
    accumulating the contraction of the gradient with itself along every other
    dimension (for a matrix: G G^T and G^T G);
  * each is applied to the gradient by a tensor-matrix contraction along its
    own mode, with the power -1/(2k) for an order-k tensor (-1/4 for k = 2);
  * the modes may be applied in any order.

Readings (as in the matrix oracle): statistics start at zero and decay by
beta with no (1 - beta) factor; roots are of (H + eps I), by symmetric
eigendecomposition; roots are refreshed every ``refresh_every`` steps from
step 0; the update is W <- W - lr P.

Diagonal variant (cue 28: past a size threshold, about 1200 in the paper's
experiments, a dimension keeps only the diagonal of its statistic, decided
independently per dimension): a mode with n_i > ``diag_threshold`` keeps
h_i = diag(H_i), updated as h_i <- beta h_i + (sum over the other modes of
G^2), and is preconditioned by the scaling d_i = (h_i + eps)^{-1/(2k)} along
its dimension (d_i = 0 where h_i + eps = 0, which only happens with eps = 0
on an index the gradient has never touched).
"""
from __future__ import annotations

from typing import List, Sequence

import numpy as np

from .shampoo import inverse_root


def mode_statistic(G: np.ndarray, i: int) -> np.ndarray:
    """Contraction of G with itself over every mode but i: an n_i x n_i matrix
    (the mode-i unfolding times its transpose)."""
    others = [j for j in range(G.ndim) if j != i]
    return np.tensordot(G, G, axes=(others, others))


def mode_product(G: np.ndarray, M: np.ndarray, i: int) -> np.ndarray:
    """G x_i M: out[..., a, ...] = sum_b M[a, b] G[..., b, ...] along mode i."""
    out = np.tensordot(M, G, axes=([1], [i]))  # the new mode comes first
    return np.moveaxis(out, 0, i)


def precondition_tensor(G: np.ndarray, roots: Sequence[np.ndarray], order: Sequence[int] | None = None) -> np.ndarray:
    """G x_1 X_1 x_2 X_2 ... x_k X_k (the modes in the given order)."""
    P = np.asarray(G, dtype=np.float64)
    for i in (range(G.ndim) if order is None else order):
        P = mode_product(P, roots[i], i)
    return P


def mode_diagonal_statistic(G: np.ndarray, i: int) -> np.ndarray:
    """diag(mode_statistic(G, i)): the sum of G^2 over every mode but i."""
    others = tuple(j for j in range(G.ndim) if j != i)
    return np.sum(np.asarray(G, dtype=np.float64) ** 2, axis=others)


def diagonal_root(h: np.ndarray, p: int, eps: float) -> np.ndarray:
    """(h + eps)^{-1/p} elementwise, 0 where h + eps = 0."""
    x = np.asarray(h, dtype=np.float64) + eps
    out = np.zeros_like(x)
    pos = x > 0
    out[pos] = x[pos] ** (-1.0 / p)
    return out


class TensorShampooOracle:
    """Order-k Shampoo on one tensor parameter, one step at a time.  Modes
    longer than ``diag_threshold`` (None: none) use the diagonal variant."""

    def __init__(self, shape, beta: float, eps: float, lr: float, refresh_every: int = 1, weight=None,
                 diag_threshold: int | None = None):
        self.shape = tuple(int(x) for x in shape)
        self.k = len(self.shape)
        self.beta = float(beta)
        self.eps = float(eps)
        self.lr = float(lr)
        self.refresh_every = int(refresh_every)
        self.diag = [diag_threshold is not None and n > diag_threshold for n in self.shape]
        self.H: List[np.ndarray] = [np.zeros(n) if d else np.zeros((n, n)) for n, d in zip(self.shape, self.diag)]
        self.X: List[np.ndarray] = [None] * self.k
        self.W = np.zeros(self.shape) if weight is None else np.array(weight, dtype=np.float64)
        self.t = 0

    def step(self, grad) -> np.ndarray:
        """Accumulate, refresh the roots (power -1/(2k)) when due, precondition,
        update; returns the preconditioned gradient P."""
        G = np.asarray(grad, dtype=np.float64)
        for i in range(self.k):
            stat = mode_diagonal_statistic(G, i) if self.diag[i] else mode_statistic(G, i)
            self.H[i] = self.beta * self.H[i] + stat
        if self.t % self.refresh_every == 0:
            self.X = [diagonal_root(H, 2 * self.k, self.eps) if d else inverse_root(H, 2 * self.k, self.eps)
                      for H, d in zip(self.H, self.diag)]
        P = G
        for i in range(self.k):
            if self.diag[i]:
                shape = [1] * self.k
                shape[i] = self.shape[i]
                P = P * self.X[i].reshape(shape)
            else:
                P = mode_product(P, self.X[i], i)
        self.W -= self.lr * P
        self.t += 1
        return P
