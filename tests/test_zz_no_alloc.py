"""inv_root_batched_noalloc: the inverse-root solver for callers that cannot
allocate device memory (its scratch is a fixed array inside the library).

Called through the C ABI and compared with inv_root_batched (caller-owned
scratch) on the same inputs, on two calls in a row: the second call reuses the
fixed scratch the first one left behind.  This file is collected last so that
a failing run that stops at the first failure has run every other test.
"""
import ctypes

import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import oracle
import workloads

TOL = 1e-6  # both paths run the same kernels on the same data


@pytest.fixture(scope="module")
def sb():
    import shampoo_family_second_b200 as sb
    return sb


def call_noalloc(sb, A, p, eps, solver, iters, tol, degree=32, lo=0.0):
    X = torch.empty_like(A)
    it = torch.zeros(A.shape[0], dtype=torch.int32, device=A.device)
    st = torch.zeros(1, dtype=torch.int32, device=A.device)
    rc = sb.lib.inv_root_batched_noalloc(A.data_ptr(), X.data_ptr(), A.shape[0], A.shape[1], p, eps, solver,
                                         iters, tol, degree, lo, it.data_ptr(), st.data_ptr(),
                                         torch.cuda.current_stream().cuda_stream)
    assert rc == 0, sb.last_error()
    return X, it, st


@pytest.mark.parametrize("solver,n,batch,tol", [(0, 256, 12, 1e-5), (1, 128, 6, 0.0), (2, 384, 5, 0.0)])
def test_noalloc_matches_inv_root_batched_on_two_calls(sb, solver, n, batch, tol):
    for call in range(2):
        A64 = workloads.spd_batch(batch, n, 1e3, seed=100 * solver + call)
        A = torch.from_numpy(A64.astype(np.float32)).cuda()
        lo = 0.999e-3 if solver == 2 else 0.0
        X_ref, it_ref, st_ref = sb.inv_root_batched(A, p=4, eps=1e-6, solver=solver, iters=30, tol=tol,
                                                    cheb_degree=32, cheb_lo=lo)
        X, it, st = call_noalloc(sb, A, 4, 1e-6, solver, 30, tol, 32, lo)
        torch.cuda.synchronize()
        assert int(st.item()) == int(st_ref.item()) == 0
        assert torch.equal(it, it_ref)
        Xr, Xn = X_ref.cpu().numpy().astype(np.float64), X.cpu().numpy().astype(np.float64)
        for b in range(batch):
            assert oracle.rel_fro(Xn[b], Xr[b]) <= TOL


def test_noalloc_largest_block_in_chunks(sb):
    """n = 1024 with coupled Newton needs 28 MiB of scratch per matrix: the
    fixed 32 MiB array takes one matrix at a time."""
    A64 = workloads.spd_batch(2, 1024, 1e3, seed=7)
    A = torch.from_numpy(A64.astype(np.float32)).cuda()
    X_ref, it_ref, st_ref = sb.inv_root_batched(A, p=4, eps=1e-6, solver=0, iters=20, tol=0.0)
    X, it, st = call_noalloc(sb, A, 4, 1e-6, 0, 20, 0.0)
    torch.cuda.synchronize()
    assert int(st.item()) == int(st_ref.item()) == 0
    assert torch.equal(it, it_ref)
    Xr, Xn = X_ref.cpu().numpy().astype(np.float64), X.cpu().numpy().astype(np.float64)
    for b in range(2):
        assert oracle.rel_fro(Xn[b], Xr[b]) <= TOL


def test_noalloc_residual_checked_chunks(sb):
    """n = 1024, second-degree coupled Newton, tol 1e-5, batch 3: one matrix
    per chunk of the fixed array, so the residual accumulators and the
    iteration counter are reset for each chunk, and the iterations run as
    plain launches.  Roots and iteration counts equal inv_root_batched's
    (caller-owned scratch, one chunk, graph loop) on two calls in a row."""
    for call in range(2):
        A64 = workloads.spd_batch(3, 1024, 1e3, seed=70 + call)
        A = torch.from_numpy(A64.astype(np.float32)).cuda()
        X_ref, it_ref, st_ref = sb.inv_root_batched(A, p=4, eps=1e-6, solver=3, iters=40, tol=1e-5)
        X, it, st = call_noalloc(sb, A, 4, 1e-6, 3, 40, 1e-5)
        torch.cuda.synchronize()
        assert int(st.item()) == int(st_ref.item()) == 0
        assert torch.equal(it, it_ref)
        assert int(it.min().item()) > 0
        Xr, Xn = X_ref.cpu().numpy().astype(np.float64), X.cpu().numpy().astype(np.float64)
        for b in range(3):
            assert oracle.rel_fro(Xn[b], Xr[b]) <= TOL
