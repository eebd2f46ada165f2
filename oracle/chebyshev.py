"""Float64 oracle for the Chebyshev inverse-root variant.

TEST INFRASTRUCTURE ONLY (see the package docstring).

The DASH abstract names Chebyshev-polynomial approximation of inverse matrix
roots but does not define it.  Reading used here (a published method,
Trefethen, "Approximation Theory and Approximation Practice", ch. 3-4, and
Clenshaw's recurrence, 1955):

* scale: A' = (A + eps I) / s with s = ||A + eps I||_F, so spec(A') is in (0, 1]
  (the "matrix scaling" the DASH abstract refers to, read as Frobenius);
* interval [a, 1] with a = lo / s, where lo is a lower bound of the spectrum of
  A + eps I in A's own units (``lo <= 0`` means eps); a >= 1 is clamped to 1/2;
* f(x) = x^{-1/p} is interpolated at the d+1 Chebyshev points of the first
  kind, mapped to [a, 1]; the coefficients c_0..c_d are those of
  p(t) = sum_k c_k T_k(t) on t in [-1, 1] (c_0 already halved);
* evaluate p on Xt = (2 A' - (1 + a) I) / (1 - a) by Clenshaw's recurrence
  b_k = 2 Xt b_{k+1} - b_{k+2} + c_k I, result Xt b_1 - b_2 + c_0 I;
* unscale: X = s^{-1/p} p(Xt).

The polynomial is an approximation: its distance to the exact root is a
property of (d, a), not a parity failure.  The GPU's Chebyshev solver is
compared with ``chebyshev_inverse_root`` (same polynomial, float64).
"""
from __future__ import annotations

from typing import Callable

import numpy as np


def chebyshev_nodes(d: int) -> np.ndarray:
    """t_j = cos(pi (j + 1/2) / (d + 1)), j = 0..d (first kind)."""
    j = np.arange(d + 1, dtype=np.float64)
    return np.cos(np.pi * (j + 0.5) / (d + 1))


def interpolation_coefficients(f: Callable[[np.ndarray], np.ndarray], a: float,
                               b: float, d: int) -> np.ndarray:
    """Coefficients c_0..c_d of the degree-d interpolant of f on [a, b] at the
    Chebyshev points of the first kind, as p(t) = sum_k c_k T_k(t) with
    x = ((b - a) t + (b + a)) / 2 (discrete orthogonality of T_k at the nodes)."""
    j = np.arange(d + 1, dtype=np.float64)
    theta = np.pi * (j + 0.5) / (d + 1)
    x = 0.5 * (b - a) * np.cos(theta) + 0.5 * (b + a)
    fx = f(x)
    k = np.arange(d + 1, dtype=np.float64)
    c = (2.0 / (d + 1)) * (np.cos(np.outer(k, theta)) @ fx)
    c[0] *= 0.5
    return c


def inverse_root_coefficients(p: int, a: float, d: int) -> np.ndarray:
    """Interpolation coefficients of x^{-1/p} on [a, 1]."""
    return interpolation_coefficients(lambda x: x ** (-1.0 / p), a, 1.0, d)


def scaled_interval_lo(s: float, eps: float, lo: float) -> float:
    """Lower end a of the scaled interval: (lo if lo > 0 else eps) / s,
    clamped to 1/2 when it reaches 1 (a degenerate interval)."""
    base = lo if lo > 0.0 else eps
    if not base > 0.0:
        raise ValueError("Chebyshev interval needs eps > 0 or lo > 0")
    a = base / s
    return 0.5 if a >= 1.0 else a


def clenshaw_matrix(Xt: np.ndarray, c: np.ndarray) -> np.ndarray:
    """sum_k c_k T_k(Xt) by Clenshaw's recurrence, in float64."""
    n = Xt.shape[0]
    eye = np.eye(n)
    d = len(c) - 1
    b1 = np.zeros((n, n))   # b_{k+1}
    b2 = np.zeros((n, n))   # b_{k+2}
    for k in range(d, 0, -1):
        bk = 2.0 * (Xt @ b1) - b2 + c[k] * eye
        b2, b1 = b1, bk
    return Xt @ b1 - b2 + c[0] * eye


def chebyshev_inverse_root(A: np.ndarray, p: int, eps: float, degree: int,
                           lo: float = 0.0, valid: int | None = None) -> np.ndarray:
    """Chebyshev approximation of (A + eps I)^{-1/p} (see module docstring).

    ``valid`` restricts the statistic to its leading ``valid`` x ``valid``
    part (a ragged block); the result has that size.
    """
    A = np.asarray(A, dtype=np.float64)
    if valid is not None:
        A = A[:valid, :valid]
    n = A.shape[0]
    Ad = A + eps * np.eye(n)
    s = np.linalg.norm(Ad)
    a = scaled_interval_lo(s, eps, lo)
    c = inverse_root_coefficients(p, a, degree)
    Xt = (2.0 * (Ad / s) - (1.0 + a) * np.eye(n)) / (1.0 - a)
    return s ** (-1.0 / p) * clenshaw_matrix(Xt, c)
