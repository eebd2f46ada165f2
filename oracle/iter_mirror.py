"""Float64 restatements of the iterative inverse-root solvers (diagnostic).

TEST INFRASTRUCTURE ONLY (see the package docstring).  Never used as a parity
gate: the gate is the exact root of ``oracle.shampoo.inverse_root``.  These
mirrors take the same steps as the CUDA solvers in float64, so that when a
parity check fails one can tell "not converged / method error" from "fp32
rounding".

Both start from the damped, scaled matrix A' = (A + eps I) / s and unscale by
s^{-1/p} at the end: s = ||A + eps I||_F (spec(A') in (0, 1]), or for coupled
Newton on the GPU the power-iteration scale of spectral_scale.

* Coupled Newton for A'^{-1/p} (Guo & Higham, "A Schur-Newton method for the
  matrix p-th root and its inverse", 2006): X_0 = I, M_0 = A';
  T = ((p + 1) I - M) / p;  X <- X T;  M <- T^p M.  M -> I, X -> A'^{-1/p}.
* The same coupled form with a higher-degree correction: T is the degree-m
  truncation sum_{j<=m} c_j (I - M)^j of the binomial series of
  M^{-1/p} = (I - (I - M))^{-1/p}, c_0 = 1, c_j = c_{j-1} (j - 1 + 1/p) / j.
  m = 1 gives the Newton T above; the CUDA solver's NEWTON_CUBIC takes m = 2
  from the second iteration on, after one plain Newton step.
* Newton-DB, read as the coupled Denman-Beavers-family square-root iteration
  in its multiplication-only (Newton-Schulz) form (Higham, "Functions of
  Matrices", 2008, sec. 6.3 and 6.8): Y_0 = A', Z_0 = I;
  T = (3 I - Z Y) / 2;  Y <- Y T;  Z <- T Z.  Y -> A'^{1/2}, Z -> A'^{-1/2}.
  p = 2 takes Z; p = 4 runs the iteration a second time on A'' = Y (the first
  run's square root) and takes that run's Z = A'^{-1/4}.
"""
from __future__ import annotations

import numpy as np


def frobenius_scale(A: np.ndarray, eps: float):
    n = A.shape[0]
    Ad = np.asarray(A, dtype=np.float64) + eps * np.eye(n)
    s = float(np.linalg.norm(Ad))
    return Ad / s, s


def power_estimate(Ad: np.ndarray, steps: int = 12) -> float:
    """Largest-eigenvalue estimate of a symmetric positive semi-definite
    matrix: `steps` power steps x <- Ad x / ||Ad x|| from the fixed start
    vector 1 + 0.3 ((7919 j) mod 17) / 17; returns the last norm (a lower
    estimate)."""
    n = Ad.shape[0]
    x = 1.0 + 0.3 * ((np.arange(n) * 7919) % 17) / 17.0
    x = x / np.linalg.norm(x)
    lam = 0.0
    for _ in range(steps):
        y = Ad @ x
        lam = float(np.linalg.norm(y))
        if lam <= 0.0:
            break
        x = y / lam
    return lam


def spectral_scale(A: np.ndarray, eps: float):
    """Scale of the coupled-Newton solver: s = min(||A + eps I||_F,
    1.25 power_estimate(A + eps I)).  The scaled spectrum stays inside the
    iteration's region of convergence (0, p + 1) even when the estimate is low,
    and its largest eigenvalue lands near 0.8."""
    n = A.shape[0]
    Ad = np.asarray(A, dtype=np.float64) + eps * np.eye(n)
    s = float(np.linalg.norm(Ad))
    lam = power_estimate(Ad)
    if lam > 0.0 and 1.25 * lam < s:
        s = 1.25 * lam
    return Ad / s, s


def binomial_coefficients(p: int, m: int):
    """c_0..c_m of (1 - x)^{-1/p} = sum_j c_j x^j."""
    c = [1.0]
    for j in range(1, m + 1):
        c.append(c[-1] * (j - 1 + 1.0 / p) / j)
    return c


def correction(M: np.ndarray, p: int, degree: int) -> np.ndarray:
    """T = sum_{j<=degree} c_j (I - M)^j."""
    eye = np.eye(M.shape[0])
    D = eye - M
    T = np.zeros_like(M)
    P = eye
    for cj in binomial_coefficients(p, degree):
        T = T + cj * P
        P = P @ D
    return T


def coupled_newton(A: np.ndarray, p: int, eps: float, iters: int, tol: float = 0.0, scale: str = "frobenius",
                   trace_tol: bool = False, degree: int = 1):
    """Returns (X, iterations run, final residual).  The residual is
    ||M - I||_F / sqrt(n), or tr(I - M) / n with trace_tol (the CUDA solver's
    stopping test).  degree > 1 uses that correction degree from the second
    iteration on (the first is a plain Newton step)."""
    M, s = (spectral_scale if scale == "spectral" else frobenius_scale)(A, eps)
    n = M.shape[0]
    eye = np.eye(n)
    X = eye.copy()

    def residual(M):
        return np.trace(eye - M) / n if trace_tol else np.linalg.norm(M - eye) / np.sqrt(n)

    res = residual(M)
    k = 0
    while k < iters and not (tol > 0.0 and res <= tol):
        T = ((p + 1) * eye - M) / p if (degree == 1 or k == 0) else correction(M, p, degree)
        X = X @ T
        M = np.linalg.matrix_power(T, p) @ M
        res = residual(M)
        k += 1
    return X * s ** (-1.0 / p), k, res


def newton_schulz_sqrt(A1: np.ndarray, iters: int, tol: float = 0.0):
    """One Newton-DB stage on a matrix with spectrum in (0, 1].
    Returns (Y ~ A1^{1/2}, Z ~ A1^{-1/2}, iterations, ||Z Y - I||_F / sqrt(n))."""
    n = A1.shape[0]
    eye = np.eye(n)
    Y = A1.copy()
    Z = eye.copy()
    k = 0
    res = np.linalg.norm(Z @ Y - eye) / np.sqrt(n)
    while k < iters and not (tol > 0.0 and res <= tol):
        T = 0.5 * (3.0 * eye - Z @ Y)
        Y, Z = Y @ T, T @ Z
        res = np.linalg.norm(Z @ Y - eye) / np.sqrt(n)
        k += 1
    return Y, Z, k, res


def newton_db(A: np.ndarray, p: int, eps: float, iters: int, tol: float = 0.0):
    """Returns (X, total iterations, final residual)."""
    A1, s = frobenius_scale(A, eps)
    Y, Z, k1, res = newton_schulz_sqrt(A1, iters, tol)
    if p == 2:
        return Z * s ** -0.5, k1, res
    if p != 4:
        raise ValueError("Newton-DB supports p = 2 and p = 4")
    _, Z2, k2, res2 = newton_schulz_sqrt(Y, iters, tol)
    return Z2 * s ** -0.25, k1 + k2, res2
