"""Pins of the float64 oracle to facts fixed by the pages and by mathematics.

None of these re-types the oracle's own formula: each compares it with a
closed form, a different library routine, a brute-force construction, or an
invariant, chosen so that a dropped term, a wrong sign / index / exponent or a
transposed operand in the oracle fails at least one of them.
"""
import json
import os

import numpy as np
import pytest
import scipy.linalg

import oracle
from oracle import shampoo as osh
from oracle import chebyshev as och
from oracle import iter_mirror as oim
import workloads


def rand_spd(n, rng, kappa=1e2):
    q = workloads.haar_orthogonal(n, rng)
    lam = workloads.spd_spectrum(n, kappa, rng)
    return (q * lam) @ q.T, q, lam


# ---------------------------------------------------------------- golden files

def test_golden_root_2x2(golden_dir):
    """Hand-derived root of [[2,1],[1,2]] (tests/golden/inverse_root_2x2.json)."""
    fx = json.load(open(os.path.join(golden_dir, "inverse_root_2x2.json")))
    A = np.array(fx["A"])
    for case in fx["cases"]:
        X = oracle.inverse_root(A, case["p"], fx["eps"])
        np.testing.assert_allclose(X, np.array(case["X"]), rtol=0, atol=1e-14)


@pytest.mark.parametrize("beta_idx", [0, 1, 2])
def test_golden_first_step_rank1(golden_dir, beta_idx):
    """Hand-derived first step for G = u v^T (tests/golden/first_step_rank1.json)."""
    fx = json.load(open(os.path.join(golden_dir, "first_step_rank1.json")))
    G = np.array(fx["G"])
    o = oracle.ShampooOracle([G.shape], block=2, beta=fx["beta_values"][beta_idx],
                             eps=fx["eps"], lr=fx["lr"], root_p=fx["p"])
    P = o.step([G])
    np.testing.assert_allclose(P[0], np.array(fx["P"]), atol=1e-14)
    np.testing.assert_allclose(o.W[0], np.array(fx["W1_from_zero"]), atol=1e-14)


# ---------------------------------------------------------------- p1 diagonal

@pytest.mark.parametrize("p", [2, 4])
def test_root_diagonal_closed_form(p):
    d = np.array([4.0, 1e-3, 7.5, 0.0, 123.0])
    eps = 1e-2
    X = oracle.inverse_root(np.diag(d), p, eps)
    np.testing.assert_allclose(X, np.diag((d + eps) ** (-1.0 / p)), rtol=1e-13, atol=0)


# ---------------------------------------------------------------- p2 2x2 closed form

def _sqrt_2x2(A):
    """Classical closed form sqrt(A) = (A + delta I) / sqrt(tr A + 2 delta),
    delta = sqrt(det A), for a 2x2 SPD matrix."""
    delta = np.sqrt(np.linalg.det(A))
    return (A + delta * np.eye(2)) / np.sqrt(np.trace(A) + 2 * delta)


@pytest.mark.parametrize("seed", range(5))
def test_root_2x2_closed_form(seed):
    rng = np.random.default_rng(seed)
    B = rng.standard_normal((2, 2))
    A = B @ B.T
    eps = 0.3
    Ad = A + eps * np.eye(2)
    s = _sqrt_2x2(Ad)
    q = _sqrt_2x2(s)                      # A^{1/4}
    inv4 = np.array([[q[1, 1], -q[0, 1]], [-q[1, 0], q[0, 0]]]) / (q[0, 0] * q[1, 1] - q[0, 1] * q[1, 0])
    inv2 = np.array([[s[1, 1], -s[0, 1]], [-s[1, 0], s[0, 0]]]) / (s[0, 0] * s[1, 1] - s[0, 1] * s[1, 0])
    np.testing.assert_allclose(oracle.inverse_root(A, 4, eps), inv4, rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(oracle.inverse_root(A, 2, eps), inv2, rtol=1e-11, atol=1e-13)


# ---------------------------------------------------------------- p3 first step = polar-like factor

@pytest.mark.parametrize("shape", [(7, 4), (4, 7), (6, 6)])
@pytest.mark.parametrize("p", [2, 4])
def test_first_step_svd_closed_form(shape, p):
    """From zero statistics, P_1 = U diag(sigma / (sigma^2 + eps)^{2/p}) V^T
    (G = U Sigma V^T): the two quarter powers compose into a half power
    (podcast cue 22).  Uses numpy's SVD, a different routine from eigh."""
    rng = np.random.default_rng(1)
    G = rng.standard_normal(shape)
    eps = 0.05
    o = oracle.ShampooOracle([shape], block=max(shape), beta=0.7, eps=eps, lr=1.0, root_p=p)
    P = o.step([G])[0]
    U, sig, Vt = np.linalg.svd(G, full_matrices=False)
    expect = (U * (sig / (sig ** 2 + eps) ** (2.0 / p))) @ Vt
    np.testing.assert_allclose(P, expect, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(o.W[0], -expect, rtol=1e-11, atol=1e-12)


# ---------------------------------------------------------------- p4 invariants

@pytest.mark.parametrize("p", [2, 4])
def test_root_invariants(p):
    rng = np.random.default_rng(3)
    A, _, _ = rand_spd(24, rng, kappa=1e4)
    eps = 1e-3
    X = oracle.inverse_root(A, p, eps)
    n = A.shape[0]
    resid = np.linalg.norm(np.linalg.matrix_power(X, p) @ (A + eps * np.eye(n)) - np.eye(n)) / np.sqrt(n)
    assert resid < 1e-10
    assert np.linalg.norm(X - X.T) < 1e-12 * np.linalg.norm(X)
    assert np.linalg.norm(X @ A - A @ X) < 1e-10 * np.linalg.norm(X) * np.linalg.norm(A)
    assert np.all(np.linalg.eigvalsh(X) > 0)


# ---------------------------------------------------------------- p5 Kronecker brute force

def test_kronecker_equivalence_tiny():
    """Podcast cue 22: with W and G flattened, the sandwich equals the
    Kronecker product of L^{1/4} and R^{1/4}, inverted, applied to vec(G).
    Brute force at the Tiny block size (B = 32: a 1024 x 1024 system), with the
    fractional powers from scipy's Schur-based routine, not from eigh."""
    rng = np.random.default_rng(5)
    r, c = 32, 32
    Gs = [rng.standard_normal((r, c)) for _ in range(3)]
    eps = 1e-6
    o = oracle.ShampooOracle([(r, c)], block=32, beta=1.0, eps=eps, lr=1.0, root_p=4)
    for G in Gs:
        P = o.step([G])[0]
    G = Gs[-1]
    L = sum(g @ g.T for g in Gs) + eps * np.eye(r)
    R = sum(g.T @ g for g in Gs) + eps * np.eye(c)
    Lq = np.real(scipy.linalg.fractional_matrix_power(L, 0.25))
    Rq = np.real(scipy.linalg.fractional_matrix_power(R, 0.25))
    K = np.kron(Lq, Rq)                    # row-major vec: vec(A X B) = (A kron B^T) vec X
    vecP = np.linalg.solve(K, G.reshape(-1))
    np.testing.assert_allclose(P.reshape(-1), vecP, rtol=1e-7, atol=1e-9)


def test_kronecker_nonsymmetric_orientation():
    """Same brute force on a non-square block, which catches a swapped L / R
    or a transposed gradient (the shapes would not even conform)."""
    rng = np.random.default_rng(6)
    r, c = 12, 5
    G = rng.standard_normal((r, c))
    eps = 1e-2
    o = oracle.ShampooOracle([(r, c)], block=12, beta=1.0, eps=eps, lr=1.0, root_p=4)
    P = o.step([G])[0]
    Lq = np.real(scipy.linalg.fractional_matrix_power(G @ G.T + eps * np.eye(r), 0.25))
    Rq = np.real(scipy.linalg.fractional_matrix_power(G.T @ G + eps * np.eye(c), 0.25))
    vecP = np.linalg.solve(np.kron(Lq, Rq), G.reshape(-1))
    np.testing.assert_allclose(P.reshape(-1), vecP, rtol=1e-9, atol=1e-11)


# ---------------------------------------------------------------- p6 spectral closed form

@pytest.mark.parametrize("kappa", [1e2, 1e4])
@pytest.mark.parametrize("p", [2, 4])
def test_root_spectral_closed_form(kappa, p):
    A, Q, lam = workloads.spd_batch(2, 40, kappa, seed=11, return_parts=True)
    eps = 1e-9
    for b in range(2):
        expect = (Q[b] * (lam[b] + eps) ** (-1.0 / p)) @ Q[b].T
        got = oracle.inverse_root(A[b], p, eps)
        assert osh.rel_fro(got, expect) < 1e-11


# ---------------------------------------------------------------- p7 scaling / orthogonal invariance

def test_root_scaling_and_orthogonal_invariance():
    rng = np.random.default_rng(7)
    A, _, _ = rand_spd(16, rng)
    eps, c, p = 1e-3, 37.5, 4
    X = oracle.inverse_root(A, p, eps)
    np.testing.assert_allclose(oracle.inverse_root(c * A, p, c * eps), c ** (-1.0 / p) * X, rtol=1e-11)
    Q = workloads.haar_orthogonal(16, rng)
    np.testing.assert_allclose(oracle.inverse_root(Q @ A @ Q.T, p, eps), Q @ X @ Q.T, rtol=1e-10, atol=1e-12)


# ---------------------------------------------------------------- p8 padding invariance

def test_padding_invariance():
    """A zero-padded block with a positive pad diagonal has a root whose valid
    part equals the unpadded root (the padded matrix is block diagonal)."""
    rng = np.random.default_rng(8)
    A, _, _ = rand_spd(20, rng)
    eps = 1e-4
    Ap = np.zeros((32, 32))
    Ap[:20, :20] = A
    Ap[20:, 20:] = np.eye(12) * 5.0
    Xp = oracle.inverse_root(Ap, 4, eps)
    np.testing.assert_allclose(Xp[:20, :20], oracle.inverse_root(A, 4, eps), rtol=1e-11, atol=1e-13)
    assert np.abs(Xp[:20, 20:]).max() < 1e-13


def test_ragged_blocks_match_unblocked_region():
    """The oracle keeps ragged blocks at their real size: the block at the
    ragged corner sees exactly the corner sub-gradient."""
    rng = np.random.default_rng(9)
    G = rng.standard_normal((45, 70))
    o = oracle.ShampooOracle([(45, 70)], block=32, beta=1.0, eps=1e-3, lr=1.0)
    P = o.step([G])
    corner = [b for b, blk in enumerate(o.table) if blk.row0 == 32 and blk.col0 == 64][0]
    Gc = G[32:, 64:]
    U, s, Vt = np.linalg.svd(Gc, full_matrices=False)
    np.testing.assert_allclose(P[corner], (U * (s / np.sqrt(s ** 2 + 1e-3))) @ Vt, rtol=1e-10, atol=1e-12)


# ---------------------------------------------------------------- p9 beta = 1 equivalence

def test_beta_one_equals_eps_identity_initialisation():
    """With beta = 1, taking the root of (L + eps I) from zero statistics is the
    notes' listing literally: L starts at eps I and the root is L^{-1/4}."""
    rng = np.random.default_rng(10)
    Gs = [rng.standard_normal((8, 6)) for _ in range(4)]
    eps = 1e-3
    o = oracle.ShampooOracle([(8, 6)], block=8, beta=1.0, eps=eps, lr=1e-2)
    Lit, Rit, W = eps * np.eye(8), eps * np.eye(6), np.zeros((8, 6))
    for G in Gs:
        o.step([G])
        Lit = Lit + G @ G.T
        Rit = Rit + G.T @ G
        lamL, QL = np.linalg.eigh(Lit)
        lamR, QR = np.linalg.eigh(Rit)
        W = W - 1e-2 * ((QL * lamL ** -0.25) @ QL.T) @ G @ ((QR * lamR ** -0.25) @ QR.T)
    np.testing.assert_allclose(o.W[0], W, rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------- p10 statistics closed form

@pytest.mark.parametrize("beta", [1.0, 0.95, 0.5])
def test_statistics_constant_gradient_geometric_sum(beta):
    """Constant G: L_t = (sum_{k<=t} beta^k) G G^T = (1 - beta^{t+1}) / (1 - beta) G G^T."""
    rng = np.random.default_rng(12)
    G = rng.standard_normal((5, 3))
    o = oracle.ShampooOracle([(5, 3)], block=5, beta=beta, eps=1e-3, lr=1.0)
    for t in range(6):
        o.step([G])
        a = (t + 1) if beta == 1.0 else (1 - beta ** (t + 1)) / (1 - beta)
        np.testing.assert_allclose(o.L[0], a * (G @ G.T), rtol=1e-13)
        np.testing.assert_allclose(o.R[0], a * (G.T @ G), rtol=1e-13)


def test_statistics_unit_gradients_count():
    """G = e_i e_j^T adds 1 to L[i, i] and R[j, j] only (beta = 1)."""
    o = oracle.ShampooOracle([(4, 3)], block=4, beta=1.0, eps=1.0, lr=0.0)
    hits = [(0, 1), (2, 2), (0, 0), (3, 1)]
    for i, j in hits:
        G = np.zeros((4, 3))
        G[i, j] = 1.0
        o.step([G])
    np.testing.assert_array_equal(o.L[0], np.diag([2.0, 0, 1, 1]))
    np.testing.assert_array_equal(o.R[0], np.diag([1.0, 2, 1]))


# ---------------------------------------------------------------- stale roots between refreshes

@pytest.mark.parametrize("refresh", [1, 3])
def test_refresh_schedule_closed_form(refresh):
    """G_t = c_t G0.  Then L_t = a_t G0 G0^T with a_t = sum_k beta^{t-k} c_k^2,
    and the step-t update uses the roots of the last refresh step r(t):
    P_t = c_t U diag(sigma / (a_{r(t)} sigma^2 + eps)^{1/2}) V^T.
    Pins accumulate -> refresh (t % k == 0, from t = 0) -> apply, and the
    staleness of roots between refreshes (podcast cue 28)."""
    rng = np.random.default_rng(13)
    G0 = rng.standard_normal((6, 4))
    U, sig, Vt = np.linalg.svd(G0, full_matrices=False)
    cs = [1.0, 2.0, 0.5, 3.0, 1.5, 0.25, 2.5, 1.0]
    beta, eps = 0.9, 1e-2
    o = oracle.ShampooOracle([(6, 4)], block=6, beta=beta, eps=eps, lr=1.0, refresh_every=refresh)
    a = 0.0
    a_ref = None
    for t, c in enumerate(cs):
        P = o.step([c * G0])[0]
        a = beta * a + c * c
        if t % refresh == 0:
            a_ref = a
        expect = c * (U * (sig / np.sqrt(a_ref * sig ** 2 + eps))) @ Vt
        np.testing.assert_allclose(P, expect, rtol=1e-10, atol=1e-12)


# ---------------------------------------------------------------- partition

def test_block_table_counts():
    assert len(oracle.block_table(workloads.WORKLOADS["tiny"].shapes, 32)) == 2
    assert len(oracle.block_table(workloads.WORKLOADS["lowrank"].shapes, 256)) == 64
    gpt2 = oracle.block_table(workloads.WORKLOADS["gpt2"].shapes, 512)
    assert len(gpt2) == 456
    assert len(oracle.block_table(workloads.WORKLOADS["llama"].shapes, 1024)) == 1024
    # 768 = 512 + 256 rows; 2304 = 4 x 512 + 256 columns
    first = [b for b in gpt2 if b.param == 0]
    assert sorted({b.r for b in first}) == [256, 512]
    assert sorted({b.c for b in first}) == [256, 512]
    assert sum(b.r * b.c for b in gpt2) == workloads.WORKLOADS["gpt2"].n_params
    ragged = sum(1 for b in gpt2 if b.r < 512 or b.c < 512)
    assert ragged == 252


def test_block_table_order_and_cover():
    t = oracle.block_table([(70, 40), (10, 10)], 32)
    assert [(b.param, b.row0, b.col0, b.r, b.c) for b in t] == [
        (0, 0, 0, 32, 32), (0, 0, 32, 32, 8), (0, 32, 0, 32, 32), (0, 32, 32, 32, 8),
        (0, 64, 0, 6, 32), (0, 64, 32, 6, 8), (1, 0, 0, 10, 10)]


# ---------------------------------------------------------------- Chebyshev

def test_chebyshev_coefficients_match_numpy():
    """Interpolation at first-kind points equals numpy's chebinterpolate."""
    for p, a, d in [(4, 1e-2, 16), (2, 0.1, 32), (4, 1e-4, 32)]:
        c = och.inverse_root_coefficients(p, a, d)
        ref = np.polynomial.chebyshev.chebinterpolate(
            lambda t: (0.5 * (1 - a) * t + 0.5 * (1 + a)) ** (-1.0 / p), d)
        np.testing.assert_allclose(c, ref, rtol=1e-12, atol=1e-13)


def test_chebyshev_interpolation_exact_for_polynomials():
    d = 7
    poly = np.polynomial.Polynomial([0.3, -1.0, 2.0, 0.0, 0.5, -0.25])
    c = och.interpolation_coefficients(poly, 0.2, 1.0, d)
    t = np.linspace(-1, 1, 33)
    x = 0.4 * t + 0.6
    np.testing.assert_allclose(np.polynomial.chebyshev.chebval(t, c), poly(x), rtol=1e-12, atol=1e-12)
    assert np.all(np.abs(c[6:]) < 1e-13)


def test_clenshaw_matrix_matches_eigen_evaluation():
    """Clenshaw on a symmetric matrix equals Q diag(chebval(lambda)) Q^T."""
    rng = np.random.default_rng(14)
    A, Q, lam = workloads.spd_batch(1, 20, 1e2, seed=15, return_parts=True)
    t = 2 * lam[0] - 1.0           # spectrum mapped into [-1, 1]
    Xt = (Q[0] * t) @ Q[0].T
    c = rng.standard_normal(12)
    got = och.clenshaw_matrix(Xt, c)
    expect = (Q[0] * np.polynomial.chebyshev.chebval(t, c)) @ Q[0].T
    np.testing.assert_allclose(got, expect, rtol=1e-11, atol=1e-11)


@pytest.mark.parametrize("p", [2, 4])
def test_chebyshev_root_converges_to_exact_root(p):
    """With the spectrum inside [a, 1] the polynomial approaches the exact root
    as the degree grows (scaled kappa = 1e2)."""
    A = workloads.spd_batch(1, 24, 1e2, seed=16)[0]
    eps = 0.0
    s = np.linalg.norm(A)
    lo = 1e-2 * 0.999                       # spectrum lower bound of A (lam_min = 1e-2)
    exact = oracle.inverse_root(A, p, eps)
    errs = [osh.rel_fro(och.chebyshev_inverse_root(A, p, eps, d, lo=lo), exact) for d in (8, 16, 32, 64)]
    assert errs[0] > errs[1] > errs[2] > errs[3]
    assert errs[3] < 1e-4


def test_chebyshev_interval_reading():
    assert och.scaled_interval_lo(10.0, 1e-3, 0.0) == pytest.approx(1e-4)
    assert och.scaled_interval_lo(10.0, 1e-3, 2.0) == pytest.approx(0.2)
    assert och.scaled_interval_lo(1.0, 5.0, 0.0) == 0.5
    with pytest.raises(ValueError):
        och.scaled_interval_lo(1.0, 0.0, 0.0)


# ---------------------------------------------------------------- iteration mirrors

@pytest.mark.parametrize("p", [2, 4])
def test_coupled_newton_mirror_converges(p):
    A = workloads.spd_batch(1, 32, 1e3, seed=17)[0]
    X, k, res = oim.coupled_newton(A, p, 1e-6, iters=60, tol=1e-13)
    assert res < 1e-12 and k < 60
    assert osh.rel_fro(X, oracle.inverse_root(A, p, 1e-6)) < 1e-10


@pytest.mark.parametrize("p", [2, 4])
def test_newton_db_mirror_converges(p):
    A = workloads.spd_batch(1, 32, 1e3, seed=18)[0]
    X, k, res = oim.newton_db(A, p, 1e-6, iters=60, tol=1e-13)
    assert res < 1e-12
    assert osh.rel_fro(X, oracle.inverse_root(A, p, 1e-6)) < 1e-10


def test_mirror_fixed_iterations_not_converged_is_visible():
    """With too few iterations the mirrors report a large residual: the
    residual is a faithful convergence signal."""
    A = workloads.spd_batch(1, 32, 1e6, seed=19)[0]
    _, k, res = oim.coupled_newton(A, 4, 0.0, iters=5)
    assert k == 5 and res > 0.1


def test_rel_fro():
    assert osh.rel_fro(np.ones(4), np.ones(4)) == 0.0
    assert osh.rel_fro(np.array([1.0, 0]), np.array([2.0, 0])) == pytest.approx(0.5)
    assert osh.rel_fro(np.zeros(2), np.zeros(2)) == 0.0


def test_spectral_scale_keeps_the_root_and_saves_iterations():
    """The coupled-Newton scale min(||A+eps I||_F, 1.25 lam_est): the root is
    scale-invariant ((cA)^{-1/p} = c^{-1/p} A^{-1/p}), so both scalings reach the
    exact root; the spectral one starts the largest eigenvalue near 0.8 instead
    of lam_max / ||A||_F and needs fewer iterations on Wishart statistics."""
    from oracle import iter_mirror as im
    rng = np.random.default_rng(8)
    G = rng.standard_normal((256, 256))
    A = G @ G.T
    eps = 1e-3
    ref = oracle.inverse_root(A, 4, eps)
    Xf, kf, _ = im.coupled_newton(A, 4, eps, 80, tol=1e-10, trace_tol=True)
    Xs, ks, _ = im.coupled_newton(A, 4, eps, 80, tol=1e-10, scale="spectral", trace_tol=True)
    assert oracle.rel_fro(Xf, ref) < 1e-8 and oracle.rel_fro(Xs, ref) < 1e-8
    assert ks <= kf - 2, (ks, kf)
    lam = np.linalg.eigvalsh(A + eps * np.eye(256))[-1]
    est = im.power_estimate(A + eps * np.eye(256))
    assert 0.9 * lam <= est <= lam * (1 + 1e-12)


@pytest.mark.parametrize("p", [2, 4])
def test_correction_polynomial_is_third_order_in_the_scalar_root(p):
    """The degree-2 correction T(mu) = c0 + c1 x + c2 x^2 (x = 1 - mu) must be
    the Taylor polynomial of mu^{-1/p} about 1: its error against the power
    function shrinks like x^3, with leading coefficient (1/p)(1/p + 1)(1/p + 2)/6.
    A wrong c1 leaves an O(x) error, a wrong c2 an O(x^2) one."""
    lead = (1 / p) * (1 / p + 1) * (1 / p + 2) / 6
    for x in (1e-2, 2e-3):
        mu = 1.0 - x
        T = oim.correction(np.array([[mu]]), p, 2)[0, 0]
        assert (mu ** (-1.0 / p) - T) / x ** 3 == pytest.approx(lead, rel=0.05)
    # degree 1 is the coupled-Newton T = ((p + 1) - mu) / p
    assert oim.correction(np.array([[0.3]]), p, 1)[0, 0] == pytest.approx((p + 1 - 0.3) / p)


@pytest.mark.parametrize("p", [2, 4])
def test_correction_keeps_eigenvalues_increasing_below_one(p):
    """Truncating a series of positive terms underestimates mu^{-1/p}, so the
    eigenvalue map mu -> mu T(mu)^p sends (0, 1] into (mu, 1]: the iterates
    grow monotonically to 1 and the trace residual stays a bound.  Near 0 the
    growth factor is (c0 + c1 + c2)^p."""
    mu = np.concatenate([np.logspace(-24, -1, 200), np.linspace(0.1, 1.0, 400)])
    f = np.array([m * oim.correction(np.array([[m]]), p, 2)[0, 0] ** p for m in mu])
    assert np.all(f <= 1.0 + 1e-15) and np.all(f[:-1] > mu[:-1])
    growth = f[0] / mu[0]
    assert growth == pytest.approx(sum(oim.binomial_coefficients(p, 2)) ** p, rel=1e-6)
    assert growth > ((p + 1) / p) ** p * 1.4


@pytest.mark.parametrize("p", [2, 4])
def test_cubic_newton_mirror_reaches_the_exact_root_in_fewer_iterations(p):
    """Both correction degrees converge to the eigendecomposition root; the
    degree-2 one in at most three quarters of the iterations on a spectrum
    spanning 1e6, and a diagonal input gives the scalar closed form."""
    A = workloads.spd_batch(1, 48, 1e6, seed=23)[0]
    ref = oracle.inverse_root(A, p, 0.0)
    X1, k1, _ = oim.coupled_newton(A, p, 0.0, 80, tol=1e-12, trace_tol=True)
    X2, k2, _ = oim.coupled_newton(A, p, 0.0, 80, tol=1e-12, trace_tol=True, degree=2)
    assert osh.rel_fro(X1, ref) < 1e-8 and osh.rel_fro(X2, ref) < 1e-8
    assert k2 <= 0.75 * k1, (k1, k2)
    d = np.array([1.0, 0.5, 1e-3, 1e-5])
    Xd, _, _ = oim.coupled_newton(np.diag(d), p, 0.0, 80, tol=1e-14, trace_tol=True, degree=2)
    assert np.allclose(np.diag(Xd), d ** (-1.0 / p), rtol=1e-10)
    assert np.abs(Xd - np.diag(np.diag(Xd))).max() == 0.0


# ---------------------------------------------------------------- momentum (podcast cue 28)

@pytest.mark.parametrize("alpha", [0.5, 0.9])
def test_momentum_constant_gradient_geometric_sum(alpha):
    """A constant gradient G every step: the momentum buffer after t + 1 steps
    is (1 + alpha + ... + alpha^t) G, so the preconditioned direction is the
    momentum-free one scaled by (1 - alpha^(t+1)) / (1 - alpha), while the
    statistics (and therefore the roots) are those of the raw gradient."""
    rng = np.random.default_rng(41)
    G = rng.standard_normal((24, 16))
    kw = dict(shapes=[(24, 16)], block=32, beta=1.0, eps=1e-3, lr=1e-2, root_p=4, refresh_every=1)
    plain = osh.ShampooOracle(**kw)
    mom = osh.ShampooOracle(**kw, momentum=alpha)
    for t in range(5):
        Pp = plain.step([G])[0]
        Pm = mom.step([G])[0]
        factor = (1.0 - alpha ** (t + 1)) / (1.0 - alpha)
        assert osh.rel_fro(Pm, factor * Pp) < 1e-12
        assert np.array_equal(mom.L[0], plain.L[0]) and np.array_equal(mom.R[0], plain.R[0])


def test_momentum_zero_is_the_plain_step():
    rng = np.random.default_rng(42)
    kw = dict(shapes=[(40, 70)], block=32, beta=0.9, eps=1e-4, lr=1e-2, root_p=4, refresh_every=2)
    a, b = osh.ShampooOracle(**kw), osh.ShampooOracle(**kw, momentum=0.0)
    for _ in range(3):
        g = [rng.standard_normal((40, 70))]
        Pa, Pb = a.step(g), b.step(g)
        assert all(np.array_equal(Pa[k], Pb[k]) for k in Pa)
    assert all(np.array_equal(x, y) for x, y in zip(a.W, b.W))


def test_momentum_alternating_gradient_closed_form():
    """Gradients G, -G, G, ...: the buffer is G (1 - alpha + alpha^2 - ...),
    i.e. M_t = G (1 - (-alpha)^(t+1)) / (1 + alpha) times the sign of step t;
    with fixed roots (refreshed at step 0 only, beta = 1 keeps G G^T growing
    but roots stay those of step 0) the directions follow that closed form."""
    alpha = 0.9
    rng = np.random.default_rng(43)
    G = rng.standard_normal((16, 24))
    kw = dict(shapes=[(16, 24)], block=32, beta=1.0, eps=1e-3, lr=1e-2, root_p=4, refresh_every=1000)
    mom = osh.ShampooOracle(**kw, momentum=alpha)
    P0 = mom.step([G])[0]  # step 0: M = G, roots of G G^T
    for t in range(1, 6):
        sign = -1.0 if t % 2 else 1.0
        P = mom.step([sign * G])[0]
        expect = sign * (1.0 - (-alpha) ** (t + 1)) / (1.0 + alpha)
        assert osh.rel_fro(P, expect * P0) < 1e-12
