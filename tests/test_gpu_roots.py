"""Batched inverse p-th roots on the GPU vs the float64 oracle.

Inputs: SPD stacks Q diag(lam) Q^T with an exact condition number (the solver
sweep's recipe), cast to fp32; the oracle takes the same fp32 values.
Gates: relative Frobenius error per root <= 2e-3 against the exact root for
coupled Newton and Newton-DB where the fp32 conditioning floor allows it
(kappa <= 1e4); Chebyshev against the float64 Clenshaw evaluation of the same
polynomial (its distance to the exact root is a property of the degree).
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import oracle
from oracle import chebyshev as och
import workloads
from parity import root_gate

TOL = 2e-3


@pytest.fixture(scope="module")
def sb():
    import shampoo_family_second_b200 as sb
    return sb


def run(sb, A32, **kw):
    X, it, st = sb.inv_root_batched(torch.from_numpy(A32).cuda(), **kw)
    torch.cuda.synchronize()
    return X.cpu().numpy().astype(np.float64), it.cpu().numpy(), int(st.item())


@pytest.mark.parametrize("n,batch", [(64, 4), (256, 3), (384, 2)])
@pytest.mark.parametrize("p", [2, 4])
@pytest.mark.parametrize("kappa", [1e2, 1e4])
@pytest.mark.parametrize("solver", [0, 3])
def test_newton_fixed(sb, n, batch, p, kappa, solver):
    A32 = workloads.spd_batch(batch, n, kappa, seed=n + p).astype(np.float32)
    X, it, st = run(sb, A32, p=p, eps=0.0, solver=solver, iters=30, tol=0.0)
    assert st == 0
    assert np.all(it == 30)
    for b in range(batch):
        A = A32[b].astype(np.float64)
        ref = oracle.inverse_root(A, p, 0.0)
        assert oracle.rel_fro(X[b], ref) < root_gate(A, p, 0.0), (b, oracle.rel_fro(X[b], ref))


@pytest.mark.parametrize("p", [2, 4])
@pytest.mark.parametrize("solver", [0, 3])
def test_newton_residual_mode(sb, p, solver):
    A32 = workloads.spd_batch(4, 128, 1e3, seed=5).astype(np.float32)
    X, it, st = run(sb, A32, p=p, eps=1e-6, solver=solver, iters=40, tol=1e-5)
    assert st == 0
    assert np.all(it > 0) and np.all(it < 40)
    for b in range(4):
        ref = oracle.inverse_root(A32[b].astype(np.float64), p, 1e-6)
        assert oracle.rel_fro(X[b], ref) < TOL


@pytest.mark.parametrize("p", [2, 4])
@pytest.mark.parametrize("kappa", [1e2, 1e4, 1e6])
def test_cubic_newton_iterations_follow_the_float64_mirror(sb, p, kappa):
    """The second-degree correction stops where its float64 restatement (same
    spectral scale, same trace test) stops, give or take one iteration of fp32
    rounding, and in fewer iterations than plain coupled Newton on the GPU."""
    from oracle import iter_mirror as im
    A32 = workloads.spd_batch(4, 256, kappa, seed=int(np.log10(kappa)) + 10 * p).astype(np.float32)
    tol = 1e-5
    X3, it3, st3 = run(sb, A32, p=p, eps=0.0, solver=sb.SOLVER_NEWTON_CUBIC, iters=40, tol=tol)
    X0, it0, st0 = run(sb, A32, p=p, eps=0.0, solver=sb.SOLVER_NEWTON, iters=40, tol=tol)
    assert st3 & ~sb.DEVFLAG_STAGNATED == 0 and st0 & ~sb.DEVFLAG_STAGNATED == 0
    for b in range(4):
        A = A32[b].astype(np.float64)
        _, k, _ = im.coupled_newton(A, p, 0.0, 40, tol=tol, scale="spectral", trace_tol=True, degree=2)
        assert abs(abs(int(it3[b])) - k) <= 1, (b, it3[b], k)
        assert abs(int(it3[b])) < abs(int(it0[b])), (b, it3[b], it0[b])
        ref = oracle.inverse_root(A, p, 0.0)
        e3, e0 = oracle.rel_fro(X3[b], ref), oracle.rel_fro(X0[b], ref)
        assert e3 < max(root_gate(A, p, 0.0), 1.5 * e0), (b, e3, e0)


@pytest.mark.parametrize("p", [2, 4])
@pytest.mark.parametrize("tol", [0.0, 1e-5])
def test_newton_db(sb, p, tol):
    A32 = workloads.spd_batch(3, 256, 1e3, seed=9).astype(np.float32)
    X, it, st = run(sb, A32, p=p, eps=0.0, solver=sb.SOLVER_NEWTON_DB, iters=30, tol=tol)
    assert st == 0
    for b in range(3):
        ref = oracle.inverse_root(A32[b].astype(np.float64), p, 0.0)
        assert oracle.rel_fro(X[b], ref) < TOL, oracle.rel_fro(X[b], ref)


@pytest.mark.parametrize("p", [2, 4])
@pytest.mark.parametrize("degree", [16, 32])
def test_chebyshev_polynomial_parity(sb, p, degree):
    kappa = 1e2
    A32 = workloads.spd_batch(3, 256, kappa, seed=11).astype(np.float32)
    lo = 0.999 / kappa                       # lower spectral bound of A (lam_min = 1/kappa)
    X, it, st = run(sb, A32, p=p, eps=0.0, solver=sb.SOLVER_CHEBYSHEV, cheb_degree=degree, cheb_lo=lo)
    assert st == 0
    assert np.all(it == degree)
    for b in range(3):
        ref = och.chebyshev_inverse_root(A32[b].astype(np.float64), p, 0.0, degree, lo=lo)
        assert oracle.rel_fro(X[b], ref) < TOL, oracle.rel_fro(X[b], ref)


def test_not_converged_flag(sb):
    A32 = workloads.spd_batch(2, 64, 1e6, seed=13).astype(np.float32)
    X, it, st = run(sb, A32, p=4, eps=0.0, solver=sb.SOLVER_NEWTON, iters=2, tol=1e-6)
    assert st & sb.DEVFLAG_NOT_CONVERGED
    assert np.all(it == -2)


@pytest.mark.parametrize("solver", [0, 1, 3])
def test_rank_deficient_input_finishes_before_the_cap(sb, solver):
    """Rank-deficient input with eps = 0 (a 128 x 128 G^T G of rank 64, like
    the ragged blocks of the GPT-2 shapes): the null space sits at the damping
    floor 2^-24 s.  The solver must end without NOT_CONVERGED (converged, or
    stopped at a stagnated residual) well below the cap.  The root is checked
    against the exact root on the range space, and on the null space only for
    being finite (there it is set by the damping floor alone; the exact root
    is infinite at eps = 0)."""
    rng = np.random.default_rng(31)
    G = rng.standard_normal((3, 64, 128)).astype(np.float32)
    A32 = np.einsum("bki,bkj->bij", G, G).astype(np.float32)
    cap = 80
    X, it, st = run(sb, A32, p=4, eps=0.0, solver=solver, iters=cap, tol=1e-5)
    assert st & ~sb.DEVFLAG_STAGNATED == 0, st
    stages = 2 if solver == 1 else 1
    assert np.all(np.abs(it) < stages * cap // 2), it
    for b in range(3):
        lam, Q = np.linalg.eigh(A32[b].astype(np.float64))
        rng_ = lam > 1e-3 * lam[-1]
        assert rng_.sum() == 64
        Qr = Q[:, rng_]
        got = Qr.T @ X[b] @ Qr
        ref = np.diag(lam[rng_] ** -0.25)
        assert oracle.rel_fro(got, ref) < TOL, (b, oracle.rel_fro(got, ref))
        assert np.all(np.isfinite(X[b]))


@pytest.mark.parametrize("solver,kmin", [(0, 24), (1, 26), (3, 17)])
def test_stagnation_stops_before_the_cap(sb, solver, kmin):
    """A tolerance below the fp32 resolution of the trace residual (1e-12;
    the residual settles near 1e-8, where the fp32 iterate stops changing):
    the solver must stop once the residual no longer improves, from iteration
    kmin on, flag STAGNATED rather than NOT_CONVERGED, stay well below the
    cap, and return the converged root.  The signed trace can land within
    1e-12 of zero by chance on the way down, so a matrix may also end as
    converged; most must stagnate."""
    A32 = workloads.spd_batch(4, 128, 1e2, seed=33).astype(np.float32)
    cap = 80
    X, it, st = run(sb, A32, p=4, eps=0.0, solver=solver, iters=cap, tol=1e-12)
    assert st & sb.DEVFLAG_STAGNATED and not st & sb.DEVFLAG_NOT_CONVERGED, st
    stages = 2 if solver == 1 else 1
    stag = it < 0
    assert stag.sum() >= 2, it
    assert np.all(-it[stag] >= kmin) and np.all(np.abs(it) < stages * cap), it
    for b in range(4):
        ref = oracle.inverse_root(A32[b].astype(np.float64), 4, 0.0)
        assert oracle.rel_fro(X[b], ref) < TOL, (b, oracle.rel_fro(X[b], ref))


def test_nonfinite_flag(sb):
    A32 = workloads.spd_batch(2, 64, 1e2, seed=14).astype(np.float32)
    A32[1, 3, 5] = np.nan
    X, it, st = run(sb, A32, p=4, eps=0.0, solver=sb.SOLVER_NEWTON, iters=5, tol=0.0)
    assert st & sb.DEVFLAG_NONFINITE
    assert np.all(np.isfinite(X[0]))


@pytest.mark.parametrize("solver,per_iter", [(0, 4), (1, 3), (3, 5)])
def test_graph_loop_matches_plain_launches(sb, solver, per_iter):
    """Residual-checked iterations after the first run as a CUDA graph loop
    that the device ends once every matrix is finished.  With profiling on
    (per-launch events) the host issues the iterations one by one up to the
    cap instead.  Both must give bit-identical roots and iteration counts, and
    the graph loop must run about the iterations needed, not the cap's worth."""
    A32 = workloads.spd_batch(6, 256, 1e3, seed=41).astype(np.float32)
    kw = dict(p=4, eps=1e-6, solver=solver, iters=60, tol=1e-5)
    sb.profile_enable(True)
    try:
        X1, it1, st1 = run(sb, A32, **kw)
    finally:
        sb.profile_enable(False)
    n0 = sb.launch_count()
    X2, it2, st2 = run(sb, A32, **kw)
    n1 = sb.launch_count()
    assert st1 == st2 == 0
    assert np.array_equal(it1, it2)
    assert np.array_equal(X1, X2)
    stages = 2 if solver == 1 else 1
    needed = int(np.max(it2))  # both stages for Newton-DB p = 4
    # prologue, norm, finalize, report and per stage one extra loop pass at most
    assert n1 - n0 <= 8 + per_iter * (needed + 2 * stages), (n1 - n0, needed)
    assert n1 - n0 < per_iter * 60 * stages


def test_newton_uses_the_spectral_scale(sb):
    """Coupled Newton scales by min(||A+eps I||_F, 1.25 x a power-iteration
    estimate of the largest eigenvalue): on Wishart statistics G G^T of a
    256 x 512 gradient (condition about 31, largest eigenvalue 0.15 of the
    Frobenius norm) it stops in fewer iterations than the same iteration needs
    under Frobenius scaling (float64: 7 against 9), with the same root."""
    from oracle import iter_mirror as im
    rng = np.random.default_rng(12)
    G = rng.standard_normal((4, 256, 512)).astype(np.float32)
    A32 = np.einsum("bij,bkj->bik", G, G).astype(np.float32)
    X, it, st = run(sb, A32, p=4, eps=1e-3, solver=sb.SOLVER_NEWTON, iters=60, tol=1e-5)
    assert st == 0
    for b in range(4):
        A = A32[b].astype(np.float64)
        _, k_frob, _ = im.coupled_newton(A, 4, 1e-3, 60, tol=1e-5, trace_tol=True)
        assert it[b] < k_frob, (it[b], k_frob)
        ref = oracle.inverse_root(A, 4, 1e-3)
        assert oracle.rel_fro(X[b], ref) < root_gate(A, 4, 1e-3)


@pytest.mark.parametrize("p", [6, 8])
@pytest.mark.parametrize("solver,tol", [(0, 0.0), (0, 1e-5), (3, 1e-5)])
def test_newton_higher_orders(sb, p, solver, tol):
    """Coupled Newton for the -1/6 and -1/8 powers of order-3 and order-4
    tensor Shampoo (T^6 = T^4 T^2, T^8 = T^4 T^4 in one more stack): the exact
    root within 2e-3 at kappa 1e3, residual-checked runs well below the cap."""
    A32 = workloads.spd_batch(4, 192, 1e3, seed=60 + p).astype(np.float32)
    X, it, st = run(sb, A32, p=p, eps=0.0, solver=solver, iters=40, tol=tol)
    assert st == 0
    if tol > 0:
        assert np.all(it > 0) and np.all(it < 30), it
    for b in range(4):
        ref = oracle.inverse_root(A32[b].astype(np.float64), p, 0.0)
        assert oracle.rel_fro(X[b], ref) < TOL, (b, oracle.rel_fro(X[b], ref))


@pytest.mark.parametrize("p", [6, 8])
def test_chebyshev_higher_orders(sb, p):
    A32 = workloads.spd_batch(3, 128, 1e2, seed=61).astype(np.float32)
    lo = 0.999e-2
    X, it, st = run(sb, A32, p=p, eps=0.0, solver=sb.SOLVER_CHEBYSHEV, cheb_degree=24, cheb_lo=lo)
    assert st == 0
    for b in range(3):
        ref = och.chebyshev_inverse_root(A32[b].astype(np.float64), p, 0.0, 24, lo=lo)
        assert oracle.rel_fro(X[b], ref) < TOL


def test_newton_db_refuses_higher_orders(sb):
    A = torch.zeros((1, 64, 64), device="cuda")
    with pytest.raises(sb.ShampooError):
        sb.inv_root_batched(A, p=6, solver=sb.SOLVER_NEWTON_DB)

