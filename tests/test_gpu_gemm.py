"""Tensor-core GEMM engine (3xTF32 tcgen05) vs float64 products.

The engine is what every stage's contraction runs on; here it is called
through the C-ABI utility ``shampoo_gemm_batched``: D = alpha A B^T + beta C +
gamma I.  Tolerance: 3xTF32 keeps about 21 bits per product, so the relative
Frobenius error of a product of Gaussian matrices stays near 1e-6; the bar
below is 2e-5 (fp32 reduction over n up to 1024 included).
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

TOL = 2e-5


def rel(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


@pytest.fixture(scope="module")
def sb():
    import shampoo_family_second_b200 as sb
    return sb


@pytest.mark.parametrize("n", [32, 64, 128, 256, 384, 512, 1024])
def test_gemm_matches_float64(sb, n):
    rng = np.random.default_rng(n)
    batch = 3
    A = rng.standard_normal((batch, n, n)).astype(np.float32)
    B = rng.standard_normal((batch, n, n)).astype(np.float32)
    D, status = sb.gemm_batched(torch.from_numpy(A).cuda(), torch.from_numpy(B).cuda())
    D = D.cpu().numpy().astype(np.float64)
    for i in range(batch):
        ref = A[i].astype(np.float64) @ B[i].astype(np.float64).T
        assert rel(D[i], ref) < TOL, (n, i, rel(D[i], ref))
    assert int(status.item()) == 0


def test_gemm_epilogue_alpha_beta_gamma_inplace(sb):
    rng = np.random.default_rng(7)
    n, batch = 256, 2
    A = rng.standard_normal((batch, n, n)).astype(np.float32)
    B = rng.standard_normal((batch, n, n)).astype(np.float32)
    C = rng.standard_normal((batch, n, n)).astype(np.float32)
    Ct = torch.from_numpy(C).cuda()
    D, _ = sb.gemm_batched(torch.from_numpy(A).cuda(), torch.from_numpy(B).cuda(), Ct, alpha=-0.5, beta=0.75,
                           gamma=2.0, out=Ct)
    D = D.cpu().numpy().astype(np.float64)
    for i in range(batch):
        ref = -0.5 * A[i].astype(np.float64) @ B[i].astype(np.float64).T + 0.75 * C[i] + 2.0 * np.eye(n)
        assert rel(D[i], ref) < TOL


def test_gemm_structured_exact(sb):
    """Products with small-integer entries are exact in 3xTF32: bit-exact check,
    which catches a wrong operand layout (transposed tile, swapped planes)."""
    rng = np.random.default_rng(3)
    n, batch = 256, 2
    A = rng.integers(-8, 9, size=(batch, n, n)).astype(np.float32)
    B = rng.integers(-8, 9, size=(batch, n, n)).astype(np.float32)
    D, _ = sb.gemm_batched(torch.from_numpy(A).cuda(), torch.from_numpy(B).cuda())
    ref = np.einsum("bij,bkj->bik", A.astype(np.float64), B.astype(np.float64))
    np.testing.assert_array_equal(D.cpu().numpy(), ref.astype(np.float32))


@pytest.mark.parametrize("n", [32, 96, 256, 384, 512])
def test_gemm_true_product_mn_major_b(sb, n):
    """op(B) = B: the B operand is read MN-major (K x N row-major)."""
    rng = np.random.default_rng(100 + n)
    batch = 2
    A = rng.standard_normal((batch, n, n)).astype(np.float32)
    B = rng.standard_normal((batch, n, n)).astype(np.float32)
    D, _ = sb.gemm_batched(torch.from_numpy(A).cuda(), torch.from_numpy(B).cuda(), trans_b=False)
    D = D.cpu().numpy().astype(np.float64)
    for i in range(batch):
        ref = A[i].astype(np.float64) @ B[i].astype(np.float64)
        assert rel(D[i], ref) < TOL, (n, i, rel(D[i], ref))
    Ai = rng.integers(-8, 9, size=(1, n, n)).astype(np.float32)
    Bi = rng.integers(-8, 9, size=(1, n, n)).astype(np.float32)
    Di, _ = sb.gemm_batched(torch.from_numpy(Ai).cuda(), torch.from_numpy(Bi).cuda(), trans_b=False)
    np.testing.assert_array_equal(Di.cpu().numpy()[0], (Ai[0].astype(np.float64) @ Bi[0]).astype(np.float32))


def test_gemm_accumulation_bias_bounded(sb):
    """The tensor core adds into fp32 with truncation, which biases sums of
    same-sign terms toward zero.  The engine keeps the exact hi*hi products and
    the small corrections in separate accumulators; the remaining mean
    relative bias at K = 1024 stays below 5e-6 (one accumulator over all three
    products shows about 1.1e-5)."""
    rng = np.random.default_rng(21)
    n = 1024
    A = np.abs(rng.standard_normal((1, n, n))).astype(np.float32)
    B = np.abs(rng.standard_normal((1, n, n))).astype(np.float32)
    D, _ = sb.gemm_batched(torch.from_numpy(A).cuda(), torch.from_numpy(B).cuda())
    ref = A[0].astype(np.float64) @ B[0].astype(np.float64).T
    bias = float(np.mean((D.cpu().numpy()[0].astype(np.float64) - ref) / ref))
    assert abs(bias) < 5e-6, bias


def test_gemm_lo_plane_is_used(sb):
    """Entries 1 + 2^-15 are not tf32-exact: a single-pass tf32 product would
    lose them; 3xTF32 must keep them (relative error far below 2^-11)."""
    n = 128
    A = np.full((1, n, n), 1.0 + 2.0 ** -15, dtype=np.float32)
    B = np.full((1, n, n), 1.0 - 2.0 ** -14, dtype=np.float32)
    D, _ = sb.gemm_batched(torch.from_numpy(A).cuda(), torch.from_numpy(B).cuda())
    ref = n * (1.0 + 2.0 ** -15) * (1.0 - 2.0 ** -14)
    got = D.cpu().numpy().astype(np.float64)
    assert np.max(np.abs(got - ref)) / ref < 1e-6
