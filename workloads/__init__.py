"""Seeded synthetic inputs for the blocked Shampoo step.

This module only draws numbers: gradients shaped like the workloads the pages
describe, and symmetric positive definite matrices with a prescribed spectrum.
It holds none of the method's arithmetic (no statistics, no roots, no update),
so both the float64 oracle and the CUDA path can be fed from it without sharing
any code.

Workloads (sizes and hyper-parameters as stated for each one):

* ``tiny``      one fp32 weight 64x32, block 32, G ~ N(0, 1), beta=1, eps=1e-6,
                lr=1e-3, p=4, coupled Newton with 20 fixed iterations.
* ``lowrank``   4 fp32 weights 1024x1024, block 256, G = low rank (r=16, unit
                entry variance) + N(0, 0.01^2) noise, beta=0.95, eps=1e-8,
                root refresh every 10 steps.
* ``gpt2``      GPT-2-small layer shapes (12 x {768x2304, 768x768, 768x3072,
                3072x768}), block 512, ragged edges, fp32 G ~ N(0, 0.02^2) with
                per-column scale log-uniform in [1e-2, 1], beta=0.999,
                eps=1e-12, root every step.
* ``llama``     Llama-1B layer shapes (16 x {4 x 2048x2048, 2 x 2048x8192,
                8192x2048}), block 1024, bf16 G ~ N(0, 0.01^2), beta=0.999,
                eps=1e-10, root refresh every 10 steps.
* ``spd_batch`` stacked SPD matrices Q diag(lam) Q^T, Q Haar, lam log-uniform
                with the condition number forced exactly.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace
from typing import Callable, List, Sequence, Tuple

import numpy as np

SOLVER_NEWTON = 0
SOLVER_NEWTON_DB = 1
SOLVER_CHEBYSHEV = 2
SOLVER_NEWTON_CUBIC = 3

DTYPE_F32 = 0
DTYPE_BF16 = 1


@dataclass(frozen=True)
class Workload:
    """Shapes and hyper-parameters of one synthetic Shampoo workload."""

    name: str
    shapes: Tuple[Tuple[int, int], ...]
    block: int
    beta: float
    eps: float
    lr: float
    root_p: int = 4
    solver: int = SOLVER_NEWTON
    iters: int = 40
    tol: float = 1e-5
    refresh_every: int = 1
    cheb_degree: int = 32
    cheb_lo: float = 0.0
    grad_dtype: int = DTYPE_F32
    momentum: float = 0.0
    diag_threshold: int = 0
    steps: int = 10
    seed: int = 1234

    @property
    def n_params(self) -> int:
        return int(sum(m * n for m, n in self.shapes))


def _gpt2_shapes() -> Tuple[Tuple[int, int], ...]:
    layer = ((768, 2304), (768, 768), (768, 3072), (3072, 768))
    return tuple(s for _ in range(12) for s in layer)


def _llama_shapes() -> Tuple[Tuple[int, int], ...]:
    layer = ((2048, 2048),) * 4 + ((2048, 8192),) * 2 + ((8192, 2048),)
    return tuple(s for _ in range(16) for s in layer)


WORKLOADS = {
    "tiny": Workload(
        name="tiny", shapes=((64, 32),), block=32, beta=1.0, eps=1e-6, lr=1e-3,
        root_p=4, solver=SOLVER_NEWTON, iters=20, tol=0.0, refresh_every=1,
        steps=10, seed=1234 + 0),
    "lowrank": Workload(
        name="lowrank", shapes=((1024, 1024),) * 4, block=256, beta=0.95,
        eps=1e-8, lr=1e-3, root_p=4, solver=SOLVER_NEWTON_CUBIC, iters=40, tol=1e-5,
        refresh_every=10, steps=100, seed=1234 + 1),
    "gpt2": Workload(
        name="gpt2", shapes=_gpt2_shapes(), block=512, beta=0.999, eps=1e-12,
        lr=1e-3, root_p=4, solver=SOLVER_NEWTON_CUBIC, iters=40, tol=1e-5,
        refresh_every=1, steps=10, seed=1234 + 2),
    "llama": Workload(
        name="llama", shapes=_llama_shapes(), block=1024, beta=0.999,
        eps=1e-10, lr=1e-3, root_p=4, solver=SOLVER_NEWTON_CUBIC, iters=40, tol=1e-5,
        refresh_every=10, grad_dtype=DTYPE_BF16, steps=20, seed=1234 + 3),
}


def workload(name: str, **overrides) -> Workload:
    return replace(WORKLOADS[name], **overrides)


# ---------------------------------------------------------------------------
# bf16 helpers (numpy has no bf16): values are carried as float32 numbers that
# are exactly representable in bf16, and as their upper 16 bits for the device.
# ---------------------------------------------------------------------------

def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); return float32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    u = (u + 0x7FFF + lsb) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32)


def bf16_bits(x_bf16_valued: np.ndarray) -> np.ndarray:
    """Upper 16 bits of float32 values that are already bf16-exact."""
    x = np.ascontiguousarray(x_bf16_valued, dtype=np.float32)
    return (x.view(np.uint32) >> 16).astype(np.uint16)


# ---------------------------------------------------------------------------
# Gradient streams
# ---------------------------------------------------------------------------

class GradientStream:
    """Deterministic per-step gradients for a workload.

    ``next()`` returns one list of float32 arrays (one per weight, row-major
    m x n).  For bf16 workloads the values are already rounded to bf16.
    Each weight draws from its own substream (``SeedSequence.spawn``) so a
    subset of weights can be regenerated without the others.
    """

    def __init__(self, wl: Workload, seed: int | None = None,
                 params: Sequence[int] | None = None):
        self.wl = wl
        root = np.random.SeedSequence(wl.seed if seed is None else seed)
        children = root.spawn(len(wl.shapes))
        self.params = list(range(len(wl.shapes))) if params is None else list(params)
        self.rngs = {i: np.random.default_rng(children[i]) for i in self.params}
        self.fixed = {}
        for i in self.params:
            m, n = wl.shapes[i]
            rng = self.rngs[i]
            if wl.name == "lowrank":
                u = rng.standard_normal((m, 16), dtype=np.float32)
                v = rng.standard_normal((n, 16), dtype=np.float32)
                self.fixed[i] = (u, v)
            elif wl.name == "gpt2":
                self.fixed[i] = (10.0 ** rng.uniform(-2.0, 0.0, size=n)).astype(np.float32)
        self.t = 0

    def _draw(self, i: int) -> np.ndarray:
        wl = self.wl
        m, n = wl.shapes[i]
        rng = self.rngs[i]
        if wl.name == "lowrank":
            u, v = self.fixed[i]
            s = rng.standard_normal((16, 16), dtype=np.float32)
            g = (u @ s @ v.T) / np.float32(16.0)
            g += np.float32(0.01) * rng.standard_normal((m, n), dtype=np.float32)
            return g.astype(np.float32)
        if wl.name == "gpt2":
            col = self.fixed[i]
            g = rng.standard_normal((m, n), dtype=np.float32) * np.float32(0.02)
            return (g * col[None, :]).astype(np.float32)
        if wl.name == "llama":
            g = rng.standard_normal((m, n), dtype=np.float32) * np.float32(0.01)
            return round_to_bf16(g)
        # tiny and any ad-hoc workload: unit Gaussian
        g = rng.standard_normal((m, n), dtype=np.float32)
        if wl.grad_dtype == DTYPE_BF16:
            g = round_to_bf16(g)
        return g

    def next(self) -> List[np.ndarray]:
        out = [self._draw(i) for i in self.params]
        self.t += 1
        return out


# ---------------------------------------------------------------------------
# SPD matrices with a prescribed condition number (inverse-root solver sweep)
# ---------------------------------------------------------------------------

def haar_orthogonal(n: int, rng: np.random.Generator) -> np.ndarray:
    """Haar-distributed orthogonal matrix: QR of a Gaussian with the signs of
    R's diagonal folded into Q (Mezzadri, 2007)."""
    z = rng.standard_normal((n, n))
    q, r = np.linalg.qr(z)
    return q * np.sign(np.diag(r))[None, :]


def spd_spectrum(n: int, kappa: float, rng: np.random.Generator) -> np.ndarray:
    """lam_i = kappa^(-u_i), u_i ~ U(0,1), with lam = 1 and lam = 1/kappa forced."""
    u = rng.uniform(0.0, 1.0, size=n)
    if n >= 1:
        u[0] = 0.0
    if n >= 2:
        u[1] = 1.0
    return kappa ** (-u)


def spd_batch(batch: int, n: int, kappa: float, seed: int = 0,
              return_parts: bool = False):
    """float64 stack (batch, n, n) of Q diag(lam) Q^T; optionally (A, Q, lam)."""
    rng = np.random.default_rng(seed)
    a = np.empty((batch, n, n))
    qs = np.empty((batch, n, n)) if return_parts else None
    lams = np.empty((batch, n)) if return_parts else None
    for b in range(batch):
        q = haar_orthogonal(n, rng)
        lam = spd_spectrum(n, kappa, rng)
        a[b] = (q * lam[None, :]) @ q.T
        if return_parts:
            qs[b] = q
            lams[b] = lam
    if return_parts:
        return a, qs, lams
    return a


SWEEP_SHAPES = ((512, 256), (128, 512), (64, 1024))  # (batch, n)
SWEEP_KAPPAS = (1e2, 1e4, 1e6, 1e8)
