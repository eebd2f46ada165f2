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
"""
import numpy as np
import scipy.linalg

from oracle import inverse_root, rel_fro

U32 = 2.0 ** -24
BASE_TOL = 2e-3


def perturbation_floor(A, p, eps, seeds=5, u=U32):
    A = np.asarray(A, dtype=np.float64)
    ex = inverse_root(A, p, eps)
    norm2 = np.linalg.norm(A, 2)
    out = []
    for sd in range(seeds):
        rng = np.random.default_rng(1000 + sd)
        E = rng.standard_normal(A.shape)
        E = E + E.T
        E *= u * norm2 / np.linalg.norm(E, 2)
        out.append(rel_fro(inverse_root(A + E, p, eps), ex))
    return float(np.median(out))


def lapack_fp32_root(A, p, eps):
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


def root_gate(A, p, eps):
    return max(BASE_TOL, 2.0 * conditioning_floor(A, p, eps))
