"""Pins of the SOAP oracle (oracle/soap.py) against what the mathematics fixes.

Adam's eps amplifies rounding noise in directions where the rotated gradient
is zero by 1/eps, so the pins take eps = 1e-3, far above that noise.

* Step 0 runs in the identity basis: with bias correction the direction is
  g / (|g| + eps) elementwise (a dropped bias correction fails it).
* Diagonal statistics: every basis is a signed permutation and SOAP is
  elementwise Adam on the gradient itself at every step (off-diagonal
  directions stay 0), also when the eigenvalue order changes between
  refreshes (the second moment's carry-over to the new basis).
* After a refresh, with the basis kept fixed, SOAP is Adam run on the rotated
  gradients from the carried-over state, both moments in rotated coordinates.
* The basis of a refresh is the eigenbasis of the statistics through that
  step (it diagonalises them), and it is first used one step later.
* Eigenvector signs do not matter.
* Blocks are independent and the weights move by lr times the direction.
"""
import numpy as np
import pytest

from oracle import soap
from oracle.shampoo import accumulate


def run(shapes, grads_seq, block, **kw):
    o = soap.SoapOracle(shapes, block, kw.pop("beta", 0.9), kw.pop("lr", 1e-2), **kw)
    outs = [o.step(g) for g in grads_seq]
    return o, outs


def test_step0_is_elementwise_adam():
    rng = np.random.default_rng(0)
    G = rng.standard_normal((24, 16))
    _, outs = run([(24, 16)], [[G]], 32, eps=1e-3)
    np.testing.assert_allclose(outs[0][0], G / (np.abs(G) + 1e-3), atol=1e-12)


def test_diagonal_statistics_reduce_to_adam_on_the_gradient():
    rng = np.random.default_rng(2)
    n, steps = 16, 7
    scales = rng.uniform(0.5, 2.0, size=n)          # distinct diagonal statistics whose order changes
    seq = [[np.diag(scales * rng.standard_normal(n))] for _ in range(steps)]
    _, outs = run([(n, n)], seq, 32, refresh_every=1, beta1=0.8, beta2=0.95, eps=1e-3)
    for i in range(n):
        g = np.array([s[0][i, i] for s in seq])
        for t in range(1, steps + 1):
            w1 = 0.8 ** np.arange(t - 1, -1, -1) * 0.2      # weights of g_1..g_t in m_t
            w2 = 0.95 ** np.arange(t - 1, -1, -1) * 0.05
            mhat = (w1 @ g[:t]) / (1 - 0.8 ** t)
            vhat = (w2 @ g[:t] ** 2) / (1 - 0.95 ** t)
            assert abs(outs[t - 1][0][i, i] - mhat / (np.sqrt(vhat) + 1e-3)) < 1e-10
    for N in outs:
        assert np.abs(N[0] - np.diag(np.diag(N[0]))).max() < 1e-12


def test_fixed_basis_after_a_refresh_is_adam_on_rotated_gradients():
    rng = np.random.default_rng(5)
    r, c, steps = 8, 11, 6
    seq = [[rng.standard_normal((r, c))] for _ in range(steps)]
    o = soap.SoapOracle([(r, c)], 16, 0.9, 1e-2, refresh_every=100, beta1=0.9, beta2=0.99, eps=1e-3)
    o.step(seq[0])                       # step 0 refreshes: the basis of steps 1.. is now fixed
    QL, QR = o.QL[0], o.QR[0]
    m = QL.T @ o.m[0] @ QR               # the state carried into the new basis
    v = o.v[0].copy()
    for t, g in enumerate(seq[1:], start=2):
        N = o.step(g)[0]
        gr = QL.T @ g[0] @ QR
        m = 0.9 * m + 0.1 * gr
        v = 0.99 * v + 0.01 * gr * gr
        want = QL @ ((m / (1 - 0.9 ** t)) / (np.sqrt(v / (1 - 0.99 ** t)) + 1e-3)) @ QR.T
        np.testing.assert_allclose(N, want, atol=1e-9)


def test_refresh_basis_diagonalises_the_statistics_and_is_used_next_step():
    rng = np.random.default_rng(7)
    seq = [[rng.standard_normal((12, 12))] for _ in range(3)]
    o = soap.SoapOracle([(12, 12)], 16, 0.9, 1e-2, refresh_every=2)
    L = np.zeros((12, 12))
    R = np.zeros((12, 12))
    for t, g in enumerate(seq):
        basis_before = (o.QL[0], o.QR[0])
        o.step(g)
        L, R = accumulate(L, R, g[0], 0.9)
        if t % 2 == 0:
            for Q, S in ((o.QL[0], L), (o.QR[0], R)):
                D = Q.T @ S @ Q
                assert np.abs(D - np.diag(np.diag(D))).max() < 1e-10 * np.abs(S).max()
                np.testing.assert_allclose(Q.T @ Q, np.eye(12), atol=1e-12)
        else:
            assert basis_before[0] is o.QL[0] and basis_before[1] is o.QR[0]


def test_eigenvector_signs_do_not_matter(monkeypatch):
    rng = np.random.default_rng(4)
    seq = [[rng.standard_normal((12, 9))] for _ in range(5)]
    _, a = run([(12, 9)], seq, 16, refresh_every=1)
    base = soap.eigenbasis
    flip = lambda S: base(S) * np.where(np.arange(S.shape[0]) % 2, -1.0, 1.0)[None, :]
    monkeypatch.setattr(soap, "eigenbasis", flip)
    _, b = run([(12, 9)], seq, 16, refresh_every=1)
    for x, y in zip(a, b):
        np.testing.assert_allclose(x[0], y[0], atol=1e-10)


def test_blocks_are_independent_and_weights_move_by_lr():
    rng = np.random.default_rng(6)
    shapes = [(40, 24)]
    seq = [[rng.standard_normal(shapes[0])] for _ in range(3)]
    o, outs = run(shapes, seq, 16, lr=0.5)
    W = np.zeros(shapes[0])
    for N in outs:
        for b, blk in enumerate(o.table):
            W[blk.row0:blk.row0 + blk.r, blk.col0:blk.col0 + blk.c] -= 0.5 * N[b]
    np.testing.assert_allclose(o.W[0], W, atol=1e-12)
    o1, outs1 = run([(16, 16)], [[g[0][:16, :16]] for g in seq], 16, lr=0.5)
    for x, y in zip(outs, outs1):
        np.testing.assert_allclose(x[0], y[0], atol=1e-10)
