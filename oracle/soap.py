"""Float64 oracle for the SOAP step: Adam in the eigenbasis of Shampoo's
preconditioner.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Pages: the pith.science record of "SOAP: Improving and Stabilizing Shampoo
using Adam" (abstract and claims: Shampoo with the 1/2 power equals Adafactor
run in the eigenbasis of Shampoo's preconditioner; SOAP runs Adam in that
eigenbasis, with one extra hyper-parameter, the frequency at which the basis
is recomputed, which is kept fixed in between) and the Substack survey "SOAP:
Optimizing Shampoo for Efficient Large Language Model Training"
(introduction: Shampoo's eigendecompositions are its bottleneck).

Readings (the pages give the idea, not the algorithm):

* Blocks and statistics as in the Shampoo oracle: per block,
  L <- beta L + G G^T and R <- beta R + G^T G, from zero.
* Order within step t (t from 0): Adam in the current basis, then the
  statistics take G_t, then, if t % refresh_every == 0, the basis is
  recomputed from them: Q_L and Q_R, the eigenvectors of L and R (symmetric
  eigendecomposition).  Before the first refresh the basis is the identity,
  so step 0 is plain Adam.  The current gradient thus never enters its own
  projection: with a basis built from statistics that include G_t, the
  rotated gradient Q_L^T G_t Q_R has exact zeros (at step 0 it is diagonal,
  G's singular values), which any fp32 evaluation turns into rounding noise
  and Adam's normalisation below then scales to +-1.
* Adam with the defaults of its paper (beta1 0.9, beta2 0.999, eps 1e-8) on
  the rotated gradient G' = Q_L^T G Q_R:
    m <- beta1 m + (1 - beta1) G                    (first moment, kept in the
                                                     original coordinates, so
                                                     a new basis rotates it)
    v <- beta2 v + (1 - beta2) (G')^2               (second moment, elementwise,
                                                     in the eigenbasis)
    N' = (Q_L^T m Q_R / (1 - beta1^t)) / (sqrt(v / (1 - beta2^t)) + eps)
    W <- W - lr Q_L N' Q_R^T                        (t = steps taken, from 1)
  With a fixed basis this is exactly Adam run on the rotated gradients.
* On a refresh, the second moment is carried over to the new basis as the
  diagonal of the same (diagonal) covariance:
  v <- (P_L o P_L) v (P_R o P_R)^T with P = Q_new^T Q_old (o: elementwise
  product).  This is exact when the new basis only reorders or flips the old
  vectors (an eigendecomposition returns its vectors in eigenvalue order, which
  changes as eigenvalues cross), so the step does not depend on that order.
"""
from __future__ import annotations

from typing import Sequence

import numpy as np

from .shampoo import accumulate, block_table


def eigenbasis(S: np.ndarray) -> np.ndarray:
    """Eigenvectors of the symmetric statistic S (columns, ascending
    eigenvalues)."""
    S = np.asarray(S, dtype=np.float64)
    _, Q = np.linalg.eigh(0.5 * (S + S.T))
    return Q


def adam_direction(m_rot: np.ndarray, v: np.ndarray, t: int, beta1: float, beta2: float,
                   eps: float) -> np.ndarray:
    """Bias-corrected Adam direction from the rotated first moment and the
    second moment (elementwise)."""
    mhat = m_rot / (1.0 - beta1 ** t)
    vhat = v / (1.0 - beta2 ** t)
    return mhat / (np.sqrt(vhat) + eps)


class SoapOracle:
    """SOAP over blocked 2-D weights in float64, one step at a time."""

    def __init__(self, shapes, block, beta, lr, refresh_every=10, beta1=0.9, beta2=0.999, eps=1e-8,
                 weights=None, blocks: Sequence[int] | None = None):
        self.shapes = [tuple(s) for s in shapes]
        self.B = int(block)
        self.beta, self.lr = float(beta), float(lr)
        self.refresh_every = int(refresh_every)
        self.beta1, self.beta2, self.eps = float(beta1), float(beta2), float(eps)
        self.table = block_table(self.shapes, self.B)
        self.active = list(range(len(self.table))) if blocks is None else list(blocks)
        self.W = ([np.zeros(s) for s in self.shapes] if weights is None
                  else [np.array(w, dtype=np.float64) for w in weights])
        z = lambda r, c: np.zeros((r, c))
        self.L = {b: z(self.table[b].r, self.table[b].r) for b in self.active}
        self.R = {b: z(self.table[b].c, self.table[b].c) for b in self.active}
        self.QL = {b: None for b in self.active}
        self.QR = {b: None for b in self.active}
        self.m = {b: z(self.table[b].r, self.table[b].c) for b in self.active}
        self.v = {b: z(self.table[b].r, self.table[b].c) for b in self.active}
        self.t = 0

    def step(self, grads) -> dict:
        """Returns the per-block update directions N_b (W_b -= lr N_b)."""
        refresh = self.t % self.refresh_every == 0
        self.t += 1
        out = {}
        for b in self.active:
            blk = self.table[b]
            G = np.asarray(grads[blk.param][blk.row0:blk.row0 + blk.r, blk.col0:blk.col0 + blk.c],
                           dtype=np.float64)
            if self.QL[b] is None:
                self.QL[b], self.QR[b] = np.eye(blk.r), np.eye(blk.c)
            QL, QR = self.QL[b], self.QR[b]
            Gr = QL.T @ G @ QR
            self.m[b] = self.beta1 * self.m[b] + (1.0 - self.beta1) * G
            self.v[b] = self.beta2 * self.v[b] + (1.0 - self.beta2) * Gr * Gr
            Nr = adam_direction(QL.T @ self.m[b] @ QR, self.v[b], self.t, self.beta1, self.beta2, self.eps)
            N = QL @ Nr @ QR.T
            out[b] = N
            self.W[blk.param][blk.row0:blk.row0 + blk.r, blk.col0:blk.col0 + blk.c] -= self.lr * N
            self.L[b], self.R[b] = accumulate(self.L[b], self.R[b], G, self.beta)
            if refresh:
                QL_new, QR_new = eigenbasis(self.L[b]), eigenbasis(self.R[b])
                PL = (QL_new.T @ QL) ** 2
                PR = (QR_new.T @ QR) ** 2
                self.v[b] = PL @ self.v[b] @ PR.T
                self.QL[b], self.QR[b] = QL_new, QR_new
        return out
