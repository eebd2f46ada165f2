"""Order-k tensor Shampoo on the GPU vs the float64 oracle (oracle/tensor.py).

Podcast transcript "Preconditioned optimization without the full matrix
cost", cue 26: one statistic per dimension of the gradient tensor (the
gradient contracted with itself over every other dimension), roots with the
power -1/(2k), applied by contractions along each dimension.

Shapes: 3 x 3 convolution kernels (order 4: two tiny modes, padded to 32; in
the larger one their statistics take the split-K Gram path), an order-3
tensor with ragged dimensions, an order-2 tensor (the unblocked matrix case,
p = 4), and bf16 gradients; all in one handle, so the unfolding area is
reused across parameters.  Checked per step, parameter and mode:
statistics (1e-5 against the oracle's H_i), roots on refresh steps
(root_checks on the GPU's own statistics with p = 2k), the apply stage (the
float64 mode products of the GPU's own roots and the gradient, 2e-5 times the
cancellation factor) and the update end to end (max(2e-3, 2 F_update) with
the fp32 LAPACK tensor pipeline as the floor's reference).
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import oracle
from oracle.tensor import TensorShampooOracle
import workloads
from parity import Fp32ReferenceTensorShampoo, root_checks, tensor_apply_check, update_gate

TOL_STATS = 1e-5
NULL_SPREAD = 0.10
# (3, 3, 96, 400): its 3-long modes unfold to 115200 columns, which the split-K
# Gram kernel reduces instead of a single GEMM tile
SHAPES = ((3, 3, 16, 40), (24, 40, 56), (64, 48), (5, 7, 9, 11), (3, 3, 96, 400))


@pytest.fixture(scope="module")
def sb():
    import shampoo_family_second_b200 as sb
    return sb


def dev(g, bf16):
    if bf16:
        return torch.from_numpy(workloads.bf16_bits(g).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(g).cuda()


@pytest.mark.parametrize("solver,bf16", [(3, False), (0, False), (3, True), (2, False)])
def test_tensor_shampoo_parity(sb, solver, bf16):
    # eps 1e-2 keeps the order-2 parameter's first statistic (rank 48 of 64)
    # off the fp32 plateau of coupled Newton on rank-deficient statistics
    # (its null-space eigenvalues, scaled, would sit near 5e-7 at eps 1e-4,
    # at the 3xTF32 rounding level of M); that regime is gated elsewhere.
    beta, eps, lr, every, steps = 0.9, 1e-2, 1e-3, 2, 4
    if solver == 2:   # Chebyshev: a spectral lower bound large enough for the degree-32 interpolant
        eps = 1.0
    cfg = sb.make_config(32, beta, eps, lr, solver=solver, iters=40, tol=0.0 if solver == 2 else 1e-5,
                         refresh_every=every, cheb_degree=32, grad_dtype=sb.BF16 if bf16 else sb.F32)
    opt = sb.TensorShampoo(SHAPES, cfg)
    refs = [TensorShampooOracle(s, beta, eps, lr, every) for s in SHAPES]
    refs32 = [Fp32ReferenceTensorShampoo(s, beta, eps, every) for s in SHAPES]
    W = [torch.zeros(s, dtype=torch.float32, device="cuda") for s in SHAPES]
    rng = np.random.default_rng(77 + solver)
    worst = {"update": 0.0, "apply": 0.0, "stats": 0.0, "root": 0.0}
    from oracle import chebyshev as och
    for t in range(steps):
        grads = [rng.standard_normal(s).astype(np.float32) for s in SHAPES]
        if bf16:
            grads = [workloads.round_to_bf16(g) for g in grads]
        before = [w.double() for w in W]
        opt.step(W, [dev(g, bf16) for g in grads])
        P_ref = [r.step(g) for r, g in zip(refs, grads)]
        P_32 = [r.step(g) for r, g in zip(refs32, grads)]
        torch.cuda.synchronize()
        for j, shape in enumerate(SHAPES):
            k = len(shape)
            Pg = ((before[j] - W[j].double()) / lr).cpu().numpy()
            roots = []
            for i, n in enumerate(shape):
                H, X = opt.mode_views(j, i)
                H = H[:n, :n].cpu().numpy().astype(np.float64)
                X = X[:n, :n].cpu().numpy().astype(np.float64)
                roots.append(X)
                es = oracle.rel_fro(H, refs[j].H[i])
                worst["stats"] = max(worst["stats"], es)
                assert es < TOL_STATS, (t, j, i, "stats", es)
                if t % every == 0:
                    if solver == 2:
                        ref = och.chebyshev_inverse_root(H, 2 * k, eps, 32, lo=0.0)
                        er, gate = oracle.rel_fro(X, ref), 2e-3
                    else:
                        er, gate, spread = root_checks(X, H, 2 * k, eps)
                        if spread is not None:
                            assert spread < NULL_SPREAD, (t, j, i, "null-space root", spread)
                    worst["root"] = max(worst["root"], er)
                    assert er < gate, (t, j, i, "root", er, gate)
            ea, ga = tensor_apply_check(Pg, grads[j], roots)
            worst["apply"] = max(worst["apply"], ea)
            assert ea < ga, (t, j, "apply", ea, ga)
            if solver != 2:
                e = oracle.rel_fro(Pg, P_ref[j])
                worst["update"] = max(worst["update"], e)
                assert e < update_gate(P_32[j], P_ref[j]), (t, j, "update", e)
    assert opt.status() & ~sb.DEVFLAG_STAGNATED == 0
    print(f"\ntensor solver {solver} bf16 {bf16}: worst update {worst['update']:.2e}, apply {worst['apply']:.2e}, "
          f"root {worst['root']:.2e}, statistics {worst['stats']:.2e}")


def test_order2_tensor_equals_unblocked_matrix_step(sb):
    """An order-2 tensor is the matrix case without blocking: the same
    statistics and update as the blocked matrix step with one block covering
    the whole weight (block = 64 for a 64 x 48 weight), to fp32 rounding."""
    shape = (64, 48)
    cfg = sb.make_config(64, 0.9, 1e-4, 1e-3, solver=3, iters=40, tol=1e-5, refresh_every=1)
    ten = sb.TensorShampoo([shape], cfg)
    mat = sb.Shampoo([shape], cfg)
    W1 = [torch.zeros(shape, device="cuda")]
    W2 = [torch.zeros(shape, device="cuda")]
    rng = np.random.default_rng(5)
    for _ in range(3):
        g = torch.from_numpy(rng.standard_normal(shape).astype(np.float32)).cuda()
        ten.step(W1, [g])
        mat.step(W2, [g])
    torch.cuda.synchronize()
    a, b = W1[0].double().cpu().numpy(), W2[0].double().cpu().numpy()
    assert oracle.rel_fro(a, b) < 1e-5


@pytest.mark.parametrize("shapes,threshold", [(((2048, 40), (3, 3, 16, 1100)), 0), (((64, 48), (20, 30, 40)), 32)])
def test_diagonal_variant_parity(sb, shapes, threshold):
    """Podcast cue 28's diagonal variant: dimensions longer than the threshold
    (default 1024, the largest root the solvers compute) keep only the
    diagonal of their statistic.  Diagonal modes: h against the oracle's
    (1e-5) and d against (h_gpu + eps)^{-1/(2k)} (1e-5); matrix modes as in
    the parity test above; the update against the float64 oracle with the
    same threshold, and the apply stage against the float64 mode products and
    scalings of the GPU's own roots."""
    from oracle.tensor import diagonal_root, mode_product
    beta, eps, lr, every, steps = 0.9, 1e-2, 1e-3, 2, 3
    cfg = sb.make_config(32, beta, eps, lr, solver=3, iters=40, tol=1e-5, refresh_every=every,
                         diag_threshold=threshold)
    opt = sb.TensorShampoo(shapes, cfg)
    thr = threshold if threshold > 0 else 1024
    refs = [TensorShampooOracle(s, beta, eps, lr, every, diag_threshold=thr) for s in shapes]
    W = [torch.zeros(s, dtype=torch.float32, device="cuda") for s in shapes]
    rng = np.random.default_rng(31)
    for t in range(steps):
        grads = [rng.standard_normal(s).astype(np.float32) for s in shapes]
        before = [w.double() for w in W]
        opt.step(W, [torch.from_numpy(g).cuda() for g in grads])
        P_ref = [r.step(g) for r, g in zip(refs, grads)]
        torch.cuda.synchronize()
        for j, shape in enumerate(shapes):
            k = len(shape)
            Pg = ((before[j] - W[j].double()) / lr).cpu().numpy()
            P64 = grads[j].astype(np.float64)
            Pabs = np.abs(P64)
            for i, n in enumerate(shape):
                a, b = opt.mode_views(j, i)
                if refs[j].diag[i]:
                    h, d = a.cpu().numpy().astype(np.float64), b.cpu().numpy().astype(np.float64)
                    assert h.shape == (n,)
                    assert oracle.rel_fro(h, refs[j].H[i]) < TOL_STATS
                    if t % every == 0:
                        assert oracle.rel_fro(d, diagonal_root(h, 2 * k, eps)) < 1e-5
                    shp = [1] * k
                    shp[i] = n
                    P64, Pabs = P64 * d.reshape(shp), Pabs * np.abs(d).reshape(shp)
                else:
                    H = a[:n, :n].cpu().numpy().astype(np.float64)
                    X = b[:n, :n].cpu().numpy().astype(np.float64)
                    assert oracle.rel_fro(H, refs[j].H[i]) < TOL_STATS
                    if t % every == 0:
                        er, gate, _ = root_checks(X, H, 2 * k, eps)
                        assert er < gate, (t, j, i, er, gate)
                    P64, Pabs = mode_product(P64, X, i), mode_product(Pabs, np.abs(X), i)
            cancel = max(1.0, np.linalg.norm(Pabs) / np.linalg.norm(P64))
            assert oracle.rel_fro(Pg, P64) < 2e-5 * cancel, (t, j, "apply")
            e = oracle.rel_fro(Pg, P_ref[j])
            assert e < 2e-3, (t, j, "update", e)
    assert opt.status() & ~sb.DEVFLAG_STAGNATED == 0
