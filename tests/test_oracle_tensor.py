"""Pins of the order-k tensor Shampoo oracle (oracle/tensor.py).

Each compares the oracle with something it does not compute itself: the
matrix oracle (k = 2), an explicit Kronecker product, explicit index loops, a
closed form, or a property the pages state (mode order does not matter).
"""
import numpy as np
import pytest

import oracle
from oracle import shampoo as osh
from oracle import tensor as ot


def test_order_two_is_the_matrix_step():
    """For a matrix the per-mode statistics are G G^T and G^T G and the power
    is -1/(2k) = -1/4: three steps of the tensor oracle equal the matrix
    oracle on one block, updates and weights alike."""
    rng = np.random.default_rng(50)
    shape = (24, 18)
    t = ot.TensorShampooOracle(shape, beta=0.9, eps=1e-3, lr=1e-2, refresh_every=2)
    m = osh.ShampooOracle([shape], block=32, beta=0.9, eps=1e-3, lr=1e-2, root_p=4, refresh_every=2)
    for _ in range(3):
        G = rng.standard_normal(shape)
        Pt = t.step(G)
        Pm = m.step([G])[0]
        assert osh.rel_fro(Pt, Pm) < 1e-12
    assert osh.rel_fro(t.W, m.W[0]) < 1e-12


def test_mode_statistic_matches_index_loops():
    rng = np.random.default_rng(51)
    G = rng.standard_normal((2, 3, 4))
    H1 = np.zeros((3, 3))
    for a in range(3):
        for b in range(3):
            H1[a, b] = sum(G[i, a, k] * G[i, b, k] for i in range(2) for k in range(4))
    assert np.allclose(ot.mode_statistic(G, 1), H1, rtol=1e-13, atol=1e-13)


def test_preconditioner_is_the_kronecker_product():
    """For an order-3 tensor, the mode-wise contraction equals the Kronecker
    product of the three factors acting on the row-major vectorisation.  The
    factors are not symmetric, so a transposed contraction fails."""
    rng = np.random.default_rng(52)
    G = rng.standard_normal((3, 4, 5))
    X = [rng.standard_normal((n, n)) for n in G.shape]
    brute = (np.kron(np.kron(X[0], X[1]), X[2]) @ G.reshape(-1)).reshape(G.shape)
    assert np.allclose(ot.precondition_tensor(G, X), brute, rtol=1e-12, atol=1e-12)


def test_mode_order_does_not_matter():
    rng = np.random.default_rng(53)
    G = rng.standard_normal((3, 4, 5, 2))
    X = [rng.standard_normal((n, n)) for n in G.shape]
    a = ot.precondition_tensor(G, X, order=[0, 1, 2, 3])
    b = ot.precondition_tensor(G, X, order=[3, 1, 0, 2])
    assert np.allclose(a, b, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("shape", [(4, 5, 6), (3, 3, 8, 16)])
def test_rank_one_first_step_closed_form(shape):
    """G = a (x) b (x) ... rank one, from zero statistics: every mode statistic
    is ||G||^2 times the projector on its factor, each root scales the factor
    direction by (||G||^2 + eps)^{-1/(2k)}, and the k modes together give
    P = (||G||^2 + eps)^{-1/2} G."""
    rng = np.random.default_rng(54)
    factors = [rng.standard_normal(n) for n in shape]
    G = factors[0]
    for f in factors[1:]:
        G = np.multiply.outer(G, f)
    eps = 1e-3
    t = ot.TensorShampooOracle(shape, beta=1.0, eps=eps, lr=1.0)
    P = t.step(G)
    expect = G / np.sqrt(np.sum(G * G) + eps)
    assert osh.rel_fro(P, expect) < 1e-10


def test_roots_use_the_order_dependent_power():
    """The root of each mode statistic is its -1/(2k) power: X^(2k) (H + eps I) = I."""
    rng = np.random.default_rng(55)
    shape = (5, 6, 7)
    t = ot.TensorShampooOracle(shape, beta=1.0, eps=1e-2, lr=1e-2)
    t.step(rng.standard_normal(shape))
    for H, X in zip(t.H, t.X):
        n = H.shape[0]
        assert np.allclose(np.linalg.matrix_power(X, 6) @ (H + 1e-2 * np.eye(n)), np.eye(n), atol=1e-9)


def test_diagonal_variant_equals_full_when_the_statistic_is_diagonal():
    """A gradient whose mode-0 fibres are mutually orthogonal has a diagonal
    mode-0 statistic, so the diagonal variant of that mode (a threshold below
    its length) must give the full variant's update exactly."""
    from oracle.tensor import TensorShampooOracle
    rng = np.random.default_rng(11)
    n0, n1, n2 = 6, 4, 5
    seq = []
    for _ in range(3):
        Q = np.linalg.qr(rng.standard_normal((n1 * n2, n0)))[0]     # orthonormal columns
        seq.append((Q * rng.uniform(0.5, 2.0, size=n0)).T.reshape(n0, n1, n2))
    full = TensorShampooOracle((n0, n1, n2), 0.9, 1e-3, 1e-2)
    diag = TensorShampooOracle((n0, n1, n2), 0.9, 1e-3, 1e-2, diag_threshold=5)   # only mode 0 (6 > 5)
    assert diag.diag == [True, False, False]
    for G in seq:
        np.testing.assert_allclose(diag.step(G), full.step(G), atol=1e-12)


def test_diagonal_variant_rank_one_closed_form():
    """G = a (x) b (x) c: the diagonal statistics are a^2 |b|^2 |c|^2 etc., so
    with every mode diagonal the first step is
    G_ijk * prod over modes of (stat + eps)^{-1/6}."""
    from oracle.tensor import TensorShampooOracle
    rng = np.random.default_rng(12)
    a, b, c = rng.standard_normal(5), rng.standard_normal(7), rng.standard_normal(3)
    G = np.einsum("i,j,k->ijk", a, b, c)
    eps = 1e-2
    o = TensorShampooOracle(G.shape, 1.0, eps, 1.0, diag_threshold=0)
    P = o.step(G)
    na, nb, nc = a @ a, b @ b, c @ c
    da = (a ** 2 * nb * nc + eps) ** (-1 / 6)
    db = (b ** 2 * na * nc + eps) ** (-1 / 6)
    dc = (c ** 2 * na * nb + eps) ** (-1 / 6)
    np.testing.assert_allclose(P, G * np.einsum("i,j,k->ijk", da, db, dc), rtol=1e-12)


def test_diagonal_root_of_an_untouched_index_is_zero():
    from oracle.tensor import diagonal_root
    np.testing.assert_array_equal(diagonal_root(np.array([0.0, 16.0]), 4, 0.0), np.array([0.0, 0.5]))
