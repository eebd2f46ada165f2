"""Parity gates shared by the GPU tests (float64, oracle-side arithmetic).

Root gate (conditioning floor).  A root computed from fp32 statistics in fp32
arithmetic cannot be closer to the exact float64 root than fp32 arithmetic
allows.  The floor F is the larger of two measured numbers:

* the root's sensitivity to rounding its input: the median relative change of
  (A + eps I)^{-1/p} over 5 seeded symmetric perturbations E with
  ||E||_2 = u ||A||_2, u = 2^-24;
* the error of the textbook backward-stable fp32 method on the same input:
  single-precision LAPACK (scipy's ``eigh``, ``ssyevd``), roots
  (max(lam, 0) + eps)^{-1/p} formed in fp32, against the float64 oracle.

The gate is max(2e-3, 2 F).  In well-conditioned cases F is far below 1e-3
and the gate is the plain 2e-3.

Update gate.  The same reading for the preconditioned update: F_update is the
relative error, against the float64 oracle, of an fp32 reference pipeline
(float32 statistics and products, single-precision LAPACK roots) run on the
same gradients; the gate is max(2e-3, 2 F_update).

Apply gate (stage parity of the update).  The GPU's update of a block,
Delta W / lr, is compared with the float64 product XL_gpu G XR_gpu of the
GPU's own fp32 roots and the same gradient, which isolates the two apply
products and the masked scatter into W from the roots' own error.  Each
fp32-accurate product (3xTF32 with round-to-nearest segment sums) carries an
elementwise error of order 2^-22 sum_k |a_ik| |b_kj|, so the gate is
TOL_APPLY = 2e-5 times the cancellation factor
|| |XL| |G| |XR| ||_F / ||XL G XR||_F (at least 1).

Both fp32 references damp with eps_eff = max(eps, u ||A + eps I||_F), the
damping the GPU solvers apply: statistics accumulated in fp32 can be
indefinite at the level u ||A||, and a smaller eps is below fp32 resolution.
"""
import numpy as np
import scipy.linalg

from oracle import inverse_root, rel_fro

U32 = 2.0 ** -24
BASE_TOL = 2e-3


def perturbation_floor(A, p, eps, seeds=5, u=U32, basis=None):
    """Median relative change of the root under u ||A||_2 symmetric
    perturbations; measured on Q^T X Q when a basis Q is given."""
    A = np.asarray(A, dtype=np.float64)
    proj = (lambda M: M) if basis is None else (lambda M: basis.T @ M @ basis)
    ex = proj(inverse_root(A, p, eps))
    norm2 = np.linalg.norm(A, 2)
    out = []
    for sd in range(seeds):
        rng = np.random.default_rng(1000 + sd)
        E = rng.standard_normal(A.shape)
        E = E + E.T
        E *= u * norm2 / np.linalg.norm(E, 2)
        out.append(rel_fro(proj(inverse_root(A + E, p, eps)), ex))
    return float(np.median(out))


def effective_eps(A, eps):
    n = np.asarray(A).shape[0]
    s = np.linalg.norm(np.asarray(A, dtype=np.float64) + eps * np.eye(n))
    return max(eps, U32 * s)


def lapack_fp32_root(A, p, eps):
    eps = effective_eps(A, eps)
    A32 = np.asarray(A, dtype=np.float32)
    A32 = (A32 + A32.T) * np.float32(0.5)
    lam, Q = scipy.linalg.eigh(A32, driver="evd")
    assert lam.dtype == np.float32
    lam = np.maximum(lam, np.float32(0.0)) + np.float32(eps)
    with np.errstate(divide="ignore", over="ignore"):
        d = lam ** np.float32(-1.0 / p)
    d[~np.isfinite(d)] = np.float32(0.0)
    return ((Q * d) @ Q.T).astype(np.float64)


def lapack_fp32_floor(A, p, eps):
    A = np.asarray(A, dtype=np.float64)
    return rel_fro(lapack_fp32_root(A, p, eps), inverse_root(A, p, eps))


def conditioning_floor(A, p, eps):
    return max(perturbation_floor(A, p, eps), lapack_fp32_floor(A, p, eps))


def root_gate(A, p, eps, factor=2.0):
    return max(BASE_TOL, factor * conditioning_floor(A, p, eps))


class Fp32ReferenceShampoo:
    """The blocked step in float32 with LAPACK roots: the update floor's
    reference (statistics, roots and products all in single precision)."""

    def __init__(self, shapes, block, beta, eps, root_p, refresh_every, blocks, momentum=0.0):
        from oracle import block_table
        self.table = block_table(shapes, block)
        self.blocks = list(blocks)
        self.beta, self.eps, self.p, self.k = np.float32(beta), eps, root_p, refresh_every
        self.L = {b: np.zeros((self.table[b].r,) * 2, np.float32) for b in self.blocks}
        self.R = {b: np.zeros((self.table[b].c,) * 2, np.float32) for b in self.blocks}
        self.alpha = np.float32(momentum)
        self.M = {b: np.zeros((self.table[b].r, self.table[b].c), np.float32) for b in self.blocks}
        self.XL, self.XR = {}, {}
        self.t = 0

    def step(self, grads):
        P = {}
        refresh = self.t % self.k == 0
        for b in self.blocks:
            blk = self.table[b]
            G = np.asarray(grads[blk.param][blk.row0:blk.row0 + blk.r, blk.col0:blk.col0 + blk.c], np.float32)
            self.L[b] = self.beta * self.L[b] + G @ G.T
            self.R[b] = self.beta * self.R[b] + G.T @ G
            if refresh:
                self.XL[b] = lapack_fp32_root(self.L[b], self.p, self.eps).astype(np.float32)
                self.XR[b] = lapack_fp32_root(self.R[b], self.p, self.eps).astype(np.float32)
            if self.alpha > 0:
                self.M[b] = self.alpha * self.M[b] + G
                P[b] = (self.XL[b] @ self.M[b] @ self.XR[b]).astype(np.float64)
            else:
                P[b] = (self.XL[b] @ G @ self.XR[b]).astype(np.float64)
        self.t += 1
        return P


def update_gate(P_fp32, P_oracle):
    return max(BASE_TOL, 2.0 * rel_fro(P_fp32, P_oracle))


TOL_APPLY = 2e-5


def apply_check(P_gpu, XL, G, XR):
    """(error, gate) of the GPU's update direction against the float64
    product of the GPU's own roots and the gradient (the apply stage alone)."""
    XL = np.asarray(XL, dtype=np.float64)
    G = np.asarray(G, dtype=np.float64)
    XR = np.asarray(XR, dtype=np.float64)
    P64 = XL @ G @ XR
    den = np.linalg.norm(P64)
    cancel = np.linalg.norm(np.abs(XL) @ np.abs(G) @ np.abs(XR)) / den if den > 0 else 1.0
    return rel_fro(P_gpu, P64), TOL_APPLY * max(1.0, cancel)


def split_range_null(S, eps):
    """Eigen-split of symmetric statistics S: the range space (eigenvalues
    above 10 eps and above 100 u ||S||_2, i.e. determined by the gradients)
    and the rest (determined by the damping eps and rounding)."""
    S = 0.5 * (np.asarray(S, dtype=np.float64) + np.asarray(S, dtype=np.float64).T)
    lam, Q = np.linalg.eigh(S)
    thr = max(10.0 * eps, 100.0 * U32 * max(abs(lam[-1]), 1e-300))
    keep = lam > thr
    return Q[:, keep], Q[:, ~keep], lam


def root_checks(X, S, p, eps):
    """(range error, range gate, null-space eigenvalue spread or None).

    For full-rank statistics the range space is everything and this is the
    plain root gate.  Otherwise the root is compared on the range space (the
    part the preconditioned gradient uses, since a gradient block lies in the
    range of its own statistics) and, on the null space, its eigenvalues are
    returned relative to (eps_eff + lam)^{-1/p} for a validity check."""
    X = np.asarray(X, dtype=np.float64)
    S = np.asarray(S, dtype=np.float64)
    Qr, Qn, lam = split_range_null(S, eps)
    ref = inverse_root(S, p, eps)
    if Qn.shape[1] == 0:
        return rel_fro(X, ref), root_gate(S, p, eps), None
    pr = lambda M: Qr.T @ M @ Qr
    err = rel_fro(pr(X), pr(ref))
    f32 = rel_fro(pr(lapack_fp32_root(S, p, eps)), pr(ref))
    gate = max(BASE_TOL, 2.0 * max(f32, perturbation_floor(S, p, eps, basis=Qr)))
    Xn = Qn.T @ (0.5 * (X + X.T)) @ Qn
    mu = np.linalg.eigvalsh(Xn)
    lam_n = np.maximum(lam[: Qn.shape[1]], 0.0)
    e = effective_eps(S, eps)
    lo = (lam_n.max() + e) ** (-1.0 / p)      # the band the null-space root must lie in
    hi = (lam_n.min() + e) ** (-1.0 / p)
    below = np.maximum(0.0, lo - mu) / lo
    above = np.maximum(0.0, mu - hi) / hi
    spread = float(max(below.max(), above.max()))
    return err, gate, spread


class Fp32ReferenceTensorShampoo:
    """Order-k tensor Shampoo in float32 with LAPACK roots (the update floor's
    reference for the tensor path): fp32 statistics, single-precision
    eigendecomposition roots with the power -1/(2k), fp32 mode products."""

    def __init__(self, shape, beta, eps, refresh_every):
        self.shape = tuple(shape)
        self.k = len(self.shape)
        self.beta, self.eps, self.every = np.float32(beta), eps, refresh_every
        self.H = [np.zeros((n, n), np.float32) for n in self.shape]
        self.X = [None] * self.k
        self.t = 0

    def step(self, G):
        from oracle.tensor import mode_statistic, precondition_tensor
        G = np.asarray(G, np.float32)
        for i in range(self.k):
            self.H[i] = (self.beta * self.H[i] + mode_statistic(G, i)).astype(np.float32)
        if self.t % self.every == 0:
            self.X = [lapack_fp32_root(H, 2 * self.k, self.eps).astype(np.float32) for H in self.H]
        self.t += 1
        return precondition_tensor(G, self.X).astype(np.float64)


def tensor_apply_check(P_gpu, G, roots):
    """(error, gate) of the tensor path's update direction against the float64
    mode products of the GPU's own roots and the gradient (apply stage)."""
    from oracle.tensor import precondition_tensor
    G = np.asarray(G, dtype=np.float64)
    roots = [np.asarray(X, dtype=np.float64) for X in roots]
    P64 = precondition_tensor(G, roots)
    den = np.linalg.norm(P64)
    cancel = np.linalg.norm(precondition_tensor(np.abs(G), [np.abs(X) for X in roots])) / den if den > 0 else 1.0
    return rel_fro(P_gpu, P64), TOL_APPLY * max(1.0, cancel)


class Fp32ReferenceSoap:
    """SOAP in float32 with single-precision LAPACK eigenbases: the update
    floor's reference for the SOAP path (same order of operations as
    oracle.soap.SoapOracle)."""

    def __init__(self, shapes, block, beta, refresh_every, beta1, beta2, eps, blocks):
        from oracle import block_table
        self.table = block_table(shapes, block)
        self.blocks = list(blocks)
        f = np.float32
        self.beta, self.k = f(beta), refresh_every
        self.b1, self.b2, self.eps = f(beta1), f(beta2), f(eps)
        self.L = {b: np.zeros((self.table[b].r,) * 2, f) for b in self.blocks}
        self.R = {b: np.zeros((self.table[b].c,) * 2, f) for b in self.blocks}
        self.QL = {b: np.eye(self.table[b].r, dtype=f) for b in self.blocks}
        self.QR = {b: np.eye(self.table[b].c, dtype=f) for b in self.blocks}
        self.m = {b: np.zeros((self.table[b].r, self.table[b].c), f) for b in self.blocks}
        self.v = {b: np.zeros((self.table[b].r, self.table[b].c), f) for b in self.blocks}
        self.t = 0

    def step(self, grads):
        refresh = self.t % self.k == 0
        self.t += 1
        c1 = np.float32(1.0 / (1.0 - float(self.b1) ** self.t))
        c2 = np.float32(1.0 / (1.0 - float(self.b2) ** self.t))
        out = {}
        for b in self.blocks:
            blk = self.table[b]
            G = np.asarray(grads[blk.param][blk.row0:blk.row0 + blk.r, blk.col0:blk.col0 + blk.c], np.float32)
            QL, QR = self.QL[b], self.QR[b]
            Gr = QL.T @ G @ QR
            self.m[b] = self.b1 * self.m[b] + (np.float32(1) - self.b1) * G
            self.v[b] = self.b2 * self.v[b] + (np.float32(1) - self.b2) * Gr * Gr
            Nr = (QL.T @ self.m[b] @ QR * c1) / (np.sqrt(self.v[b] * c2) + self.eps)
            out[b] = (QL @ Nr @ QR.T).astype(np.float64)
            self.L[b] = self.beta * self.L[b] + G @ G.T
            self.R[b] = self.beta * self.R[b] + G.T @ G
            if refresh:
                QLn = scipy.linalg.eigh(0.5 * (self.L[b] + self.L[b].T), driver="evd")[1].astype(np.float32)
                QRn = scipy.linalg.eigh(0.5 * (self.R[b] + self.R[b].T), driver="evd")[1].astype(np.float32)
                PL = (QLn.T @ QL) ** 2
                PR = (QRn.T @ QR) ** 2
                self.v[b] = PL @ self.v[b] @ PR.T
                self.QL[b], self.QR[b] = QLn, QRn
        return out
