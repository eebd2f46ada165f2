"""The inverse-root solver sweep at its own batch shapes, gated.

Inputs: the sweep's stacks 512 x 256^2, 128 x 512^2 and 64 x 1024^2 of SPD
matrices Q diag(lam) Q^T (Haar Q, lam log-uniform with condition number kappa
forced exactly), kappa in {1e2, 1e4, 1e6, 1e8}, cast to fp32; eps = 0.  Every
case runs the whole stack on the GPU through the C ABI; the oracle checks two
matrices of each (the first and the last), one by one.

Solvers and gates (DASH abstract: Newton-DB and Chebyshev solvers; the
coupled-Newton family is the reading of the Newton iterations):

* coupled Newton (both correction degrees) and Newton-DB, residual-checked
  (tol 1e-5, cap 40): against the exact root of the same fp32 matrix at the
  gate max(2e-3, 2 F) (tests/parity.py: no fp32-input method can do better
  than the root's own sensitivity to rounding its input, or than
  single-precision LAPACK with the same damping; the gate is the plain 2e-3
  wherever that floor is below 1e-3, which holds at kappa <= 1e4 except for
  p = 2 at n = 1024, where the solvers' damping 2^-24 ||A||_F moves the
  smallest eigenvalue 1e-4 by 0.45%).  At kappa = 1e8 the fp32 matrix itself
  is not positive definite beyond its own rounding (its smallest eigenvalues
  1e-8 sit below 4 u ||A||_F), so its undamped root is undefined or set by
  rounding alone; the reference there is the exact root of the matrix with
  the damping the solvers apply, eps_eff = 2^-24 ||A||_F, gated at its own
  floor;
* Chebyshev, degree 16 and 32, interval [0.999/kappa, 1] in A's units:
  polynomial parity, against the float64 Clenshaw evaluation of the same
  interpolant on the same damped matrix (the GPU damps with
  eps_eff = max(eps, 2^-24 ||A + eps I||_F)), 2e-3; its distance to the exact
  root is a property of the degree.

* coupled Newton with fp64 iterates (tol 1e-12): against the exact root of
  the damped input sym(A) + eps_eff I it computes, at 1e-6 for every kappa
  (its error against the undamped root is reported beside it).

p in {2, 4} throughout.  The device status may only carry STAGNATED (a
residual held up by fp32 rounding above tol), never NOT_CONVERGED.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import oracle
from oracle import chebyshev as och
import workloads
from parity import BASE_TOL, effective_eps, root_gate

SOLVERS = (("newton", 0, 0), ("newton_cubic", 3, 0), ("newton_db", 1, 0), ("chebyshev16", 2, 16),
           ("chebyshev32", 2, 32), ("newton_cubic_f64", 4, 0))
TOL_F64 = 1e-6
CAP, TOL_RES = 40, 1e-5


@pytest.fixture(scope="module")
def sb():
    import shampoo_family_second_b200 as sb
    return sb


CASES = [(batch, n, kappa) for batch, n in workloads.SWEEP_SHAPES for kappa in workloads.SWEEP_KAPPAS]


@pytest.mark.parametrize("batch,n,kappa", CASES, ids=[f"{b}x{n}sq-kappa{k:.0e}" for b, n, k in CASES])
def test_sweep_case(sb, batch, n, kappa):
    A32 = workloads.spd_batch(batch, n, kappa, seed=4321 + n).astype(np.float32)
    A = torch.from_numpy(A32).cuda()
    samples = (0, batch - 1)
    exact, gates = {}, {}
    report = []
    for p in (2, 4):
        for s in samples:
            A64 = A32[s].astype(np.float64)
            # the undamped root where the fp32 matrix is positive definite beyond its own
            # rounding (smallest eigenvalue above 4 u ||A||_F), else the damped one (R21)
            lam_min = np.linalg.eigvalsh(A64)[0]
            e_ref = 0.0 if lam_min > 4 * 2.0 ** -24 * np.linalg.norm(A64) else effective_eps(A64, 0.0)
            exact[p, s] = oracle.inverse_root(A64, p, e_ref)
            gates[p, s] = root_gate(A64, p, e_ref)
            assert np.isfinite(gates[p, s]) and np.all(np.isfinite(exact[p, s]))
        for name, solver, degree in SOLVERS:
            if solver == 2:
                lo = 0.999 / kappa
                X, it, st = sb.inv_root_batched(A, p=p, eps=0.0, solver=2, cheb_degree=degree, cheb_lo=lo)
            else:
                X, it, st = sb.inv_root_batched(A, p=p, eps=0.0, solver=solver, iters=CAP,
                                                tol=1e-12 if solver == 4 else TOL_RES)
            torch.cuda.synchronize()
            st = int(st.item())
            it = it.cpu().numpy()
            assert st & ~sb.DEVFLAG_STAGNATED == 0, (name, p, st)
            if solver == 2:
                assert np.all(it == degree)
            else:
                stages = 2 if (solver == 1 and p == 4) else 1
                assert np.all(np.abs(it) >= 1) and np.all(np.abs(it) <= stages * CAP), (name, p, it.min(), it.max())
            for s in samples:
                Xs = X[s].cpu().numpy().astype(np.float64)
                assert np.all(np.isfinite(Xs))
                A64 = A32[s].astype(np.float64)
                if solver == 2:
                    ref = och.chebyshev_inverse_root(A64, p, effective_eps(A64, 0.0), degree, lo=lo)
                    e, gate = oracle.rel_fro(Xs, ref), BASE_TOL
                    e_exact = oracle.rel_fro(Xs, exact[p, s])
                elif solver == 4:
                    # fp64 iterates: the exact root of the damped input itself
                    damped = 0.5 * (A64 + A64.T) + effective_eps(A64, 0.0) * np.eye(n)
                    e, gate = oracle.rel_fro(Xs, oracle.inverse_root(damped, p, 0.0)), TOL_F64
                    e_exact = oracle.rel_fro(Xs, exact[p, s])
                else:
                    e, gate = oracle.rel_fro(Xs, exact[p, s]), gates[p, s]
                    e_exact = e
                report.append((name, p, s, e, gate, e_exact, int(np.abs(it).max())))
                assert e < gate, (name, p, s, e, gate)
        del X
    print(f"\nsweep {batch}x{n}^2 kappa {kappa:.0e}: " + "; ".join(
        f"{nm} p{p} #{s}: {e:.1e}/{g:.1e}" + (f" (exact-root {ex:.1e})" if nm.startswith("cheb") or nm.endswith("f64")
                                              else "") + ("" if nm.startswith("cheb") else f" it {k}")
        for nm, p, s, e, g, ex, k in report))
