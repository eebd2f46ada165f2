"""Batched symmetric eigendecomposition on the GPU (eigh_batched).

Eigenvectors are unique only up to sign (and within clusters of equal
eigenvalues), so the checks are on what is unique: the eigenvalues (against
numpy's float64 eigh of the same fp32 matrix), and that Q is orthogonal and
diagonalises A.  Cold start: cyclic Jacobi, then Newton-Schulz
orthogonalisation steps.  Warm start from a perturbed exact basis: Jacobi on
the nearly diagonal Q^T A Q, the rotated basis, then orthogonalisation;
repeated calls stay at the fp32 floor.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import workloads

TOL = 2e-5


@pytest.fixture(scope="module")
def sb():
    import shampoo_family_second_b200 as sb
    return sb


def checks(A, Q, lam):
    A = A.astype(np.float64)
    Q = Q.astype(np.float64)
    n = A.shape[0]
    norm = np.linalg.norm(A)
    orth = np.linalg.norm(Q.T @ Q - np.eye(n)) / np.sqrt(n)
    D = Q.T @ A @ Q
    off = np.linalg.norm(D - np.diag(np.diag(D))) / norm
    ref = np.linalg.eigvalsh(A)
    lam_err = np.abs(np.sort(lam.astype(np.float64)) - ref).max() / np.abs(ref).max()
    return orth, off, lam_err


@pytest.mark.parametrize("n", [64, 256, 512])
@pytest.mark.parametrize("kappa", [1e2, 1e5])
def test_cold_start(sb, n, kappa):
    A32 = workloads.spd_batch(3, n, kappa, seed=n + 3).astype(np.float32)
    Q, lam, st = sb.eigh_batched(torch.from_numpy(A32).cuda(), jacobi_sweeps=20, refine_iters=2)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    Q, lam = Q.cpu().numpy(), lam.cpu().numpy()
    for b in range(3):
        orth, off, lam_err = checks(A32[b], Q[b], lam[b])
        assert orth < TOL and off < TOL and lam_err < TOL, (b, orth, off, lam_err)


def test_rank_deficient_statistics(sb):
    """G G^T of a 128 x 40 gradient: a 88-dimensional zero eigenspace."""
    rng = np.random.default_rng(8)
    G = rng.standard_normal((2, 128, 40)).astype(np.float32)
    A32 = np.einsum("bik,bjk->bij", G, G).astype(np.float32)
    Q, lam, st = sb.eigh_batched(torch.from_numpy(A32).cuda(), jacobi_sweeps=20, refine_iters=2)
    torch.cuda.synchronize()
    Q, lam = Q.cpu().numpy(), lam.cpu().numpy()
    for b in range(2):
        orth, off, lam_err = checks(A32[b], Q[b], lam[b])
        assert orth < TOL and off < TOL and lam_err < TOL, (b, orth, off, lam_err)


def test_warm_start_from_a_nearby_basis(sb):
    n = 256
    A64, Q64, lam64 = workloads.spd_batch(2, n, 1e3, seed=21, return_parts=True)
    A32 = A64.astype(np.float32)
    rng = np.random.default_rng(4)
    Q0 = np.empty_like(Q64)
    for b in range(2):
        K = rng.standard_normal((n, n)) * 1e-5
        K = K - K.T
        Q0[b] = Q64[b] @ (np.eye(n) + K + 0.5 * K @ K)   # a rotation close to exp(K)
    A = torch.from_numpy(A32).cuda()
    errs = []
    Q = torch.from_numpy(Q0.astype(np.float32)).cuda()
    for it in range(3):
        Q, lam, st = sb.eigh_batched(A, Q=Q, warm_start=True, refine_iters=1)
        torch.cuda.synchronize()
        Qh = Q.cpu().numpy()
        errs.append(max(checks(A32[b], Qh[b], lam.cpu().numpy()[b])[1] for b in range(2)))
    assert errs[1] < 0.1 * errs[0] or errs[1] < TOL, errs
    assert errs[-1] < TOL, errs


def test_orthogonalisation_steps_do_not_degrade_the_basis(sb):
    """Newton-Schulz orthogonalisation keeps an fp32-accurate Jacobi basis at
    the fp32 floor (no step may make it worse than 2x the Jacobi result or
    5e-6)."""
    A32 = workloads.spd_batch(2, 256, 1e4, seed=40).astype(np.float32)
    A = torch.from_numpy(A32).cuda()
    res = []
    for k in (0, 1, 2):
        Q, lam, st = sb.eigh_batched(A, jacobi_sweeps=20, refine_iters=k)
        torch.cuda.synchronize()
        Qh, lh = Q.cpu().numpy(), lam.cpu().numpy()
        res.append(max(checks(A32[b], Qh[b], lh[b])[0] for b in range(2)))
    assert res[1] <= max(2 * res[0], 5e-6) and res[2] <= max(2 * res[0], 5e-6), res
