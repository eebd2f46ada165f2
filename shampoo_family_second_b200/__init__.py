"""Blocked Shampoo optimizer step on one NVIDIA B200 (sm_100a).

Python binding of ``libshampoo.so`` (C ABI: ``include/shampoo.h``).  This
module only marshals arguments: every stage of the step (stacking, statistics,
inverse roots, preconditioned update) runs in the library's CUDA kernels.
PyTorch supplies device memory and streams.  There is no CPU fallback: if the
library is missing, importing this package fails.

Build the library with ``python shampoo_family_second_b200/build.py``.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import List, Optional, Sequence, Tuple

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libshampoo.so")

OK = 0
ERR_INVALID_ARG = -1
ERR_UNSUPPORTED = -2
ERR_WORKSPACE = -3
ERR_CUDA = -4
ERR_DEVICE = -5

DEVFLAG_NONFINITE = 1
DEVFLAG_NOT_CONVERGED = 2
DEVFLAG_TIMEOUT = 4
DEVFLAG_STAGNATED = 8

SOLVER_NEWTON = 0
SOLVER_NEWTON_DB = 1
SOLVER_CHEBYSHEV = 2
SOLVER_NEWTON_CUBIC = 3
SOLVER_NEWTON_CUBIC_F64 = 4

F32 = 0
BF16 = 1

KERNEL_GEMM = 0
KERNEL_STACK = 1
KERNEL_NORM = 2
KERNEL_PROLOGUE = 3
KERNEL_CHECK = 4
KERNEL_FINALIZE = 5
KERNEL_CHEB_COEF = 6
KERNEL_SCALE = 7
KERNEL_MIRROR = 8
KERNEL_EIGEN = 9
KERNEL_GEMM_F64 = 10
KERNEL_PERMUTE = 11
KERNEL_GRAM = 12
KERNEL_DIAG = 13
KERNEL_SOAP = 14
KERNEL_PLANES = 15
KERNEL_MODE_SMALL = 16
KERNEL_KINDS = 17
KERNEL_NAMES = ("gemm3x_tf32", "stack_blocks", "frob_norm", "prologue", "check", "finalize", "cheb_coef",
                "spectral_scale", "mirror_lower", "jacobi_eig", "dgemm_f64", "tensor_permute", "gram_small",
                "diag_modes", "soap_elementwise", "split_planes", "tensor_mode_small")

# Exported symbols, in header order (tests compare this with include/shampoo.h).
EXPORTS = (
    "shampoo_status_string", "shampoo_last_error", "shampoo_query_sizes", "shampoo_init", "shampoo_step",
    "shampoo_step_strided", "shampoo_get_status", "shampoo_block_table", "shampoo_state_views",
    "shampoo_sync_statistics", "shampoo_momentum_view", "shampoo_set_step", "shampoo_destroy",
    "inv_root_scratch_bytes", "inv_root_scratch_bytes_p", "inv_root_batched", "inv_root_batched_noalloc",
    "shampoo_tensor_query_sizes", "shampoo_tensor_init", "shampoo_tensor_step", "shampoo_tensor_views",
    "shampoo_tensor_get_status", "shampoo_tensor_destroy", "shampoo_soap_query_sizes", "shampoo_soap_init",
    "shampoo_soap_step", "shampoo_soap_views", "shampoo_soap_get_status", "shampoo_soap_destroy",
    "shampoo_pack_blocks", "eigh_scratch_bytes", "eigh_batched",
    "shampoo_gemm_scratch_bytes",
    "shampoo_gemm_batched",
    "shampoo_dgemm_batched",
    "shampoo_profile_enable", "shampoo_profile_reset", "shampoo_profile_read", "shampoo_launch_count",
)


class ShampooError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{_status_name(code)}: {msg}")
        self.code = code


class SoapConfig(ctypes.Structure):
    """Mirror of ``shampoo_soap_config`` (include/shampoo.h)."""

    _fields_ = [("beta1", ctypes.c_float), ("beta2", ctypes.c_float), ("eps", ctypes.c_float),
                ("jacobi_sweeps", ctypes.c_int32), ("refine_iters", ctypes.c_int32)]


class Config(ctypes.Structure):
    """Mirror of ``shampoo_config`` (include/shampoo.h)."""

    _fields_ = [
        ("block", ctypes.c_int32), ("beta", ctypes.c_float), ("eps", ctypes.c_float), ("lr", ctypes.c_float),
        ("root_p", ctypes.c_int32), ("solver", ctypes.c_int32), ("iters", ctypes.c_int32), ("tol", ctypes.c_float),
        ("refresh_every", ctypes.c_int32), ("cheb_degree", ctypes.c_int32), ("cheb_lo", ctypes.c_float),
        ("grad_dtype", ctypes.c_int32), ("momentum", ctypes.c_float), ("diag_threshold", ctypes.c_int32),
    ]


def make_config(block: int, beta: float, eps: float, lr: float, root_p: int = 4, solver: int = SOLVER_NEWTON,
                iters: int = 40, tol: float = 1e-5, refresh_every: int = 1, cheb_degree: int = 32,
                cheb_lo: float = 0.0, grad_dtype: int = F32, momentum: float = 0.0, diag_threshold: int = 0) -> Config:
    return Config(block, beta, eps, lr, root_p, solver, iters, tol, refresh_every, cheb_degree, cheb_lo, grad_dtype,
                  momentum, diag_threshold)


def config_from_workload(wl) -> Config:
    """Config of a ``workloads.Workload`` preset."""
    return make_config(wl.block, wl.beta, wl.eps, wl.lr, wl.root_p, wl.solver, wl.iters, wl.tol, wl.refresh_every,
                       wl.cheb_degree, wl.cheb_lo, wl.grad_dtype, getattr(wl, "momentum", 0.0),
                       getattr(wl, "diag_threshold", 0))


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python shampoo_family_second_b200/build.py` "
                          "(the CUDA library is required; there is no fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.c_void_p
    I32, I64, F = ctypes.c_int32, ctypes.c_int64, ctypes.c_float
    sz = ctypes.POINTER(ctypes.c_size_t)
    sig = {
        "shampoo_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "shampoo_last_error": (ctypes.c_char_p, []),
        "shampoo_query_sizes": (ctypes.c_int, [ctypes.POINTER(Config), I32, ctypes.POINTER(I64), ctypes.POINTER(I64),
                                               sz, sz]),
        "shampoo_init": (ctypes.c_int, [ctypes.POINTER(Config), I32, ctypes.POINTER(I64), ctypes.POINTER(I64), P,
                                        ctypes.c_size_t, P, ctypes.c_size_t, P, ctypes.POINTER(P)]),
        "shampoo_step": (ctypes.c_int, [P, ctypes.POINTER(P), ctypes.POINTER(P), P]),
        "shampoo_step_strided": (ctypes.c_int, [P, ctypes.POINTER(P), ctypes.POINTER(P), ctypes.POINTER(I64), P]),
        "shampoo_get_status": (ctypes.c_int, [P, ctypes.POINTER(I32), I32]),
        "shampoo_block_table": (ctypes.c_int, [P, ctypes.POINTER(I32), ctypes.POINTER(I64)]),
        "shampoo_state_views": (ctypes.c_int, [P, ctypes.POINTER(P), ctypes.POINTER(P), ctypes.POINTER(P),
                                               ctypes.POINTER(P), ctypes.POINTER(I64)]),
        "shampoo_momentum_view": (ctypes.c_int, [P, ctypes.POINTER(P)]),
        "shampoo_sync_statistics": (ctypes.c_int, [P, P]),
        "shampoo_set_step": (ctypes.c_int, [P, I64]),
        "shampoo_destroy": (None, [P]),
        "inv_root_scratch_bytes": (ctypes.c_int, [I64, I32, I32, sz]),
        "inv_root_scratch_bytes_p": (ctypes.c_int, [I64, I32, I32, I32, sz]),
        "inv_root_batched": (ctypes.c_int, [P, P, I64, I32, I32, F, I32, I32, F, I32, F, P, ctypes.c_size_t, P, P, P]),
        "inv_root_batched_noalloc": (ctypes.c_int, [P, P, I64, I32, I32, F, I32, I32, F, I32, F, P, P, P]),
        "shampoo_tensor_query_sizes": (ctypes.c_int, [ctypes.POINTER(Config), I32, ctypes.POINTER(I32),
                                                      ctypes.POINTER(I64), sz, sz]),
        "shampoo_tensor_init": (ctypes.c_int, [ctypes.POINTER(Config), I32, ctypes.POINTER(I32), ctypes.POINTER(I64),
                                               P, ctypes.c_size_t, P, ctypes.c_size_t, P, ctypes.POINTER(P)]),
        "shampoo_tensor_step": (ctypes.c_int, [P, ctypes.POINTER(P), ctypes.POINTER(P), P]),
        "shampoo_tensor_views": (ctypes.c_int, [P, I32, I32, ctypes.POINTER(P), ctypes.POINTER(P),
                                                ctypes.POINTER(I32), ctypes.POINTER(I32), ctypes.POINTER(I64)]),
        "shampoo_tensor_get_status": (ctypes.c_int, [P, ctypes.POINTER(I32), I32]),
        "shampoo_tensor_destroy": (None, [P]),
        "shampoo_soap_query_sizes": (ctypes.c_int, [ctypes.POINTER(Config), ctypes.POINTER(SoapConfig), I32,
                                                    ctypes.POINTER(I64), ctypes.POINTER(I64), sz, sz]),
        "shampoo_soap_init": (ctypes.c_int, [ctypes.POINTER(Config), ctypes.POINTER(SoapConfig), I32,
                                             ctypes.POINTER(I64), ctypes.POINTER(I64), P, ctypes.c_size_t, P,
                                             ctypes.c_size_t, P, ctypes.POINTER(P)]),
        "shampoo_soap_step": (ctypes.c_int, [P, ctypes.POINTER(P), ctypes.POINTER(P), P]),
        "shampoo_soap_views": (ctypes.c_int, [P] + [ctypes.POINTER(P)] * 6 + [ctypes.POINTER(I64)]),
        "shampoo_soap_get_status": (ctypes.c_int, [P, ctypes.POINTER(I32), I32]),
        "shampoo_soap_destroy": (None, [P]),
        "shampoo_pack_blocks": (ctypes.c_int, [P, I32, I32, ctypes.POINTER(P), ctypes.POINTER(I64), I32, P, I32, F,
                                               I32, I32, P]),
        "eigh_scratch_bytes": (ctypes.c_int, [I64, I32, sz]),
        "eigh_batched": (ctypes.c_int, [P, P, P, I64, I32, I32, I32, I32, P, ctypes.c_size_t, P, P]),
        "shampoo_gemm_scratch_bytes": (ctypes.c_int, [I64, I32, sz]),
        "shampoo_gemm_batched": (ctypes.c_int, [P, P, P, P, I64, I32, I32, F, F, F, P, ctypes.c_size_t, P, P]),
        "shampoo_dgemm_batched": (ctypes.c_int, [P, P, P, P, I64, I32, ctypes.c_double, ctypes.c_double,
                                                 ctypes.c_double, P, P]),
        "shampoo_profile_enable": (None, [I32]),
        "shampoo_profile_reset": (None, []),
        "shampoo_profile_read": (ctypes.c_int, [I32, ctypes.POINTER(I64), ctypes.POINTER(ctypes.c_double),
                                                ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_double)]),
        "shampoo_launch_count": (ctypes.c_uint64, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = _load()


def _status_name(code: int) -> str:
    return lib.shampoo_status_string(int(code)).decode()


def last_error() -> str:
    return lib.shampoo_last_error().decode()


def _check(code: int):
    if code != OK:
        raise ShampooError(code, last_error())


def _i64_array(values) -> ctypes.Array:
    return (ctypes.c_int64 * len(values))(*[int(v) for v in values])


def _stream_ptr(stream) -> Optional[int]:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


# ---------------------------------------------------------------------------
# sizes (host only)
# ---------------------------------------------------------------------------

def query_sizes(cfg: Config, shapes: Sequence[Tuple[int, int]]) -> Tuple[int, int]:
    rows = _i64_array([s[0] for s in shapes])
    cols = _i64_array([s[1] for s in shapes])
    sb, xb = ctypes.c_size_t(0), ctypes.c_size_t(0)
    _check(lib.shampoo_query_sizes(ctypes.byref(cfg), len(shapes), rows, cols, ctypes.byref(sb), ctypes.byref(xb)))
    return sb.value, xb.value


def inv_root_scratch_bytes(batch: int, n: int, solver: int, p: int = 4) -> int:
    b = ctypes.c_size_t(0)
    _check(lib.inv_root_scratch_bytes_p(batch, n, solver, p, ctypes.byref(b)))
    return b.value


def gemm_scratch_bytes(batch: int, n: int) -> int:
    b = ctypes.c_size_t(0)
    _check(lib.shampoo_gemm_scratch_bytes(batch, n, ctypes.byref(b)))
    return b.value


# ---------------------------------------------------------------------------
# the optimizer
# ---------------------------------------------------------------------------

class Shampoo:
    """Blocked Shampoo over a fixed list of 2-D weights.

    ``step(weights, grads)`` updates the fp32 weights in place on the current
    (or given) CUDA stream.  State and scratch are torch allocations owned by
    this object; the library allocates nothing.
    """

    def __init__(self, shapes: Sequence[Tuple[int, int]], cfg: Config, device=None, stream=None):
        import torch
        self.shapes = [tuple(int(x) for x in s) for s in shapes]
        self.cfg = cfg
        self.device = torch.device("cuda" if device is None else device)
        self.state_bytes, self.scratch_bytes = query_sizes(cfg, self.shapes)
        self.state = torch.empty(self.state_bytes, dtype=torch.uint8, device=self.device)
        self.scratch = torch.empty(self.scratch_bytes, dtype=torch.uint8, device=self.device)
        rows = _i64_array([s[0] for s in self.shapes])
        cols = _i64_array([s[1] for s in self.shapes])
        h = ctypes.c_void_p(None)
        with torch.cuda.device(self.device):
            _check(lib.shampoo_init(ctypes.byref(cfg), len(self.shapes), rows, cols, self.state.data_ptr(),
                                    self.state_bytes, self.scratch.data_ptr(), self.scratch_bytes,
                                    _stream_ptr(stream), ctypes.byref(h)))
        self._h = h
        self._destroy = lib.shampoo_destroy
        nb = ctypes.c_int32(0)
        _check(lib.shampoo_block_table(self._h, ctypes.byref(nb), None))
        self.nb = nb.value
        self._wbuf = (ctypes.c_void_p * len(self.shapes))()
        self._gbuf = (ctypes.c_void_p * len(self.shapes))()
        self._ldbuf = (ctypes.c_int64 * len(self.shapes))()

    def __del__(self):
        # The library handle is held by the instance: at interpreter shutdown
        # the module's globals may already be cleared.
        h = getattr(self, "_h", None)
        destroy = getattr(self, "_destroy", None)
        if h is not None and h.value and destroy is not None:
            destroy(h)
            self._h = None

    def step(self, weights, grads, stream=None):
        """Weights and gradients may be row-strided views (for instance blocks
        of larger tensors): unit column stride, and the same row stride for a
        weight and its gradient."""
        import torch
        want = torch.bfloat16 if self.cfg.grad_dtype == BF16 else torch.float32
        if len(weights) != len(self.shapes) or len(grads) != len(self.shapes):
            raise ValueError("one weight and one gradient per shape")
        strided = False
        for i, (w, g) in enumerate(zip(weights, grads)):
            if w.dtype != torch.float32 or g.dtype != want:
                raise TypeError(f"param {i}: weights must be float32 and grads {want}")
            if tuple(w.shape) != self.shapes[i] or tuple(g.shape) != self.shapes[i]:
                raise ValueError(f"param {i}: shape mismatch")
            rows, cols = self.shapes[i]
            ldw = w.stride(0) if rows > 1 else cols
            ldg = g.stride(0) if rows > 1 else cols
            if (cols > 1 and (w.stride(1) != 1 or g.stride(1) != 1)) or ldw != ldg or ldw < cols:
                raise ValueError(f"param {i}: weight and gradient need unit column stride and one row stride")
            self._ldbuf[i] = ldw
            strided |= ldw != cols
            self._wbuf[i] = w.data_ptr()
            self._gbuf[i] = g.data_ptr()
        if strided:
            _check(lib.shampoo_step_strided(self._h, self._wbuf, self._gbuf, self._ldbuf, _stream_ptr(stream)))
        else:
            _check(lib.shampoo_step(self._h, self._wbuf, self._gbuf, _stream_ptr(stream)))

    def status(self, reset: bool = False) -> int:
        s = ctypes.c_int32(0)
        _check(lib.shampoo_get_status(self._h, ctypes.byref(s), 1 if reset else 0))
        return s.value

    def block_table(self) -> List[Tuple[int, int, int, int, int]]:
        nb = ctypes.c_int32(0)
        buf = (ctypes.c_int64 * (5 * self.nb))()
        _check(lib.shampoo_block_table(self._h, ctypes.byref(nb), buf))
        return [tuple(buf[5 * b:5 * b + 5]) for b in range(nb.value)]

    def _views(self):
        ptrs = [ctypes.c_void_p() for _ in range(4)]
        step = ctypes.c_int64(0)
        _check(lib.shampoo_state_views(self._h, *[ctypes.byref(p) for p in ptrs], ctypes.byref(step)))
        return [p.value for p in ptrs], step.value

    @property
    def step_count(self) -> int:
        return self._views()[1]

    def statistics(self, stream=None):
        """(L, R) as views (nb, B, B) into the state buffer: float32, or float64
        with the fp64-iterate solver (which keeps the statistics in fp64).
        The part of fp32 statistics below the diagonal tiles is first filled in
        on ``stream`` (default: the current stream), as steps without a root
        refresh leave it stale."""
        import torch
        _check(lib.shampoo_sync_statistics(self._h, _stream_ptr(stream)))
        (pl, pr, _, _), _ = self._views()
        B, nb = self.cfg.block, self.nb
        base = self.state.data_ptr()
        if self.cfg.solver == SOLVER_NEWTON_CUBIC_F64:
            dt, es = torch.float64, 8
        else:
            dt, es = torch.float32, 4
        fl = self.state[:self.state_bytes - self.state_bytes % es].view(dt)
        L = fl[(pl - base) // es:(pl - base) // es + nb * B * B].view(nb, B, B)
        R = fl[(pr - base) // es:(pr - base) // es + nb * B * B].view(nb, B, B)
        return L, R

    def roots(self):
        """(XL, XR) as float32 views (nb, B, B) into the state buffer."""
        import torch
        (_, _, pxl, pxr), _ = self._views()
        B, nb = self.cfg.block, self.nb
        base = self.state.data_ptr()
        fl = self.state.view(torch.float32)
        XL = fl[(pxl - base) // 4:(pxl - base) // 4 + nb * B * B].view(nb, B, B)
        XR = fl[(pxr - base) // 4:(pxr - base) // 4 + nb * B * B].view(nb, B, B)
        return XL, XR

    def momentum(self):
        """The momentum stack (nb, B, B) as a float32 view into the state
        buffer, or None when momentum is off."""
        import torch
        ptr = ctypes.c_void_p()
        _check(lib.shampoo_momentum_view(self._h, ctypes.byref(ptr)))
        if not ptr.value:
            return None
        B, nb = self.cfg.block, self.nb
        off = (ptr.value - self.state.data_ptr()) // 4
        return self.state.view(torch.float32)[off:off + nb * B * B].view(nb, B, B)

    def set_step_count(self, step: int):
        """Sets the step counter (the refresh schedule counts from it)."""
        _check(lib.shampoo_set_step(self._h, int(step)))

    def state_dict(self):
        """Checkpoint: a copy of the state bytes and the step counter."""
        return {"state": self.state.clone(), "step": self.step_count}

    def load_state_dict(self, sd):
        self.state.copy_(sd["state"])
        _check(lib.shampoo_set_step(self._h, int(sd["step"])))


def tensor_query_sizes(cfg: Config, shapes: Sequence[Sequence[int]]) -> Tuple[int, int]:
    orders = (ctypes.c_int32 * len(shapes))(*[len(s) for s in shapes])
    dims = _i64_array([d for s in shapes for d in s])
    sb, xb = ctypes.c_size_t(0), ctypes.c_size_t(0)
    _check(lib.shampoo_tensor_query_sizes(ctypes.byref(cfg), len(shapes), orders, dims, ctypes.byref(sb),
                                          ctypes.byref(xb)))
    return sb.value, xb.value


class TensorShampoo:
    """Order-k tensor Shampoo over a fixed list of tensor weights (order 2 to
    4, every dimension at most 1024): one statistic and one -1/(2k) root per
    dimension, applied by contractions along each dimension.

    ``step(weights, grads)`` updates the fp32 weights in place; gradients are
    fp32 or bf16 (cfg.grad_dtype), natural row-major layout.  State and
    scratch are torch allocations owned by this object."""

    def __init__(self, shapes: Sequence[Sequence[int]], cfg: Config, device=None, stream=None):
        import torch
        self.shapes = [tuple(int(x) for x in s) for s in shapes]
        self.cfg = cfg
        self.device = torch.device("cuda" if device is None else device)
        self.state_bytes, self.scratch_bytes = tensor_query_sizes(cfg, self.shapes)
        self.state = torch.empty(self.state_bytes, dtype=torch.uint8, device=self.device)
        self.scratch = torch.empty(self.scratch_bytes, dtype=torch.uint8, device=self.device)
        orders = (ctypes.c_int32 * len(self.shapes))(*[len(s) for s in self.shapes])
        dims = _i64_array([d for s in self.shapes for d in s])
        h = ctypes.c_void_p(None)
        with torch.cuda.device(self.device):
            _check(lib.shampoo_tensor_init(ctypes.byref(cfg), len(self.shapes), orders, dims, self.state.data_ptr(),
                                           self.state_bytes, self.scratch.data_ptr(), self.scratch_bytes,
                                           _stream_ptr(stream), ctypes.byref(h)))
        self._h = h
        self._destroy = lib.shampoo_tensor_destroy
        self._wbuf = (ctypes.c_void_p * len(self.shapes))()
        self._gbuf = (ctypes.c_void_p * len(self.shapes))()

    def __del__(self):
        h = getattr(self, "_h", None)
        destroy = getattr(self, "_destroy", None)
        if h is not None and h.value and destroy is not None:
            destroy(h)
            self._h = None

    def step(self, weights, grads, stream=None):
        import torch
        want = torch.bfloat16 if self.cfg.grad_dtype == BF16 else torch.float32
        if len(weights) != len(self.shapes) or len(grads) != len(self.shapes):
            raise ValueError("one weight and one gradient per shape")
        for i, (w, g) in enumerate(zip(weights, grads)):
            if w.dtype != torch.float32 or g.dtype != want:
                raise TypeError(f"param {i}: weights must be float32 and grads {want}")
            if tuple(w.shape) != self.shapes[i] or tuple(g.shape) != self.shapes[i]:
                raise ValueError(f"param {i}: shape mismatch")
            if not (w.is_contiguous() and g.is_contiguous()):
                raise ValueError(f"param {i}: weight and gradient must be contiguous")
            self._wbuf[i] = w.data_ptr()
            self._gbuf[i] = g.data_ptr()
        _check(lib.shampoo_tensor_step(self._h, self._wbuf, self._gbuf, _stream_ptr(stream)))

    def status(self, reset: bool = False) -> int:
        s = ctypes.c_int32(0)
        _check(lib.shampoo_tensor_get_status(self._h, ctypes.byref(s), 1 if reset else 0))
        return s.value

    def mode_views(self, param: int, mode: int):
        """(H, X) of one mode as float32 (npad, npad) views into the state (the
        statistic's dimension d occupies the leading d x d block), or, for a
        mode that keeps only its diagonal, the d-vectors (h, d)."""
        import torch
        ph, px = ctypes.c_void_p(), ctypes.c_void_p()
        npad, diag, step = ctypes.c_int32(0), ctypes.c_int32(0), ctypes.c_int64(0)
        _check(lib.shampoo_tensor_views(self._h, param, mode, ctypes.byref(ph), ctypes.byref(px),
                                        ctypes.byref(npad), ctypes.byref(diag), ctypes.byref(step)))
        fl = self.state.view(torch.float32)
        base = self.state.data_ptr()
        n = npad.value
        if diag.value:
            return (fl[(ph.value - base) // 4:(ph.value - base) // 4 + n],
                    fl[(px.value - base) // 4:(px.value - base) // 4 + n])
        H = fl[(ph.value - base) // 4:(ph.value - base) // 4 + n * n].view(n, n)
        X = fl[(px.value - base) // 4:(px.value - base) // 4 + n * n].view(n, n)
        return H, X


# ---------------------------------------------------------------------------
# stateless entry points
# ---------------------------------------------------------------------------

def inv_root_batched(A, p: int = 4, eps: float = 0.0, solver: int = SOLVER_NEWTON, iters: int = 40,
                     tol: float = 0.0, cheb_degree: int = 32, cheb_lo: float = 0.0, out=None, scratch=None,
                     stream=None):
    """X_i ~ (A_i + eps I)^{-1/p} for a float32 CUDA stack A (batch, n, n).

    Returns (X, iters_used (int32, batch), status (int32, 1)); both stay on the
    device (no host sync)."""
    import torch
    if A.dtype != torch.float32 or A.dim() != 3 or A.shape[1] != A.shape[2] or not A.is_cuda:
        raise ValueError("A must be a float32 CUDA tensor (batch, n, n)")
    A = A.contiguous()
    batch, n = A.shape[0], A.shape[1]
    X = torch.empty_like(A) if out is None else out
    if scratch is None:
        scratch = torch.empty(inv_root_scratch_bytes(batch, n, solver, p), dtype=torch.uint8, device=A.device)
    iters_used = torch.zeros(batch, dtype=torch.int32, device=A.device)
    status = torch.zeros(1, dtype=torch.int32, device=A.device)
    with torch.cuda.device(A.device):
        _check(lib.inv_root_batched(A.data_ptr(), X.data_ptr(), batch, n, p, eps, solver, iters, tol, cheb_degree,
                                    cheb_lo, scratch.data_ptr(), scratch.numel(), iters_used.data_ptr(),
                                    status.data_ptr(), _stream_ptr(stream)))
    return X, iters_used, status


def eigh_batched(A, Q=None, warm_start: bool = False, jacobi_sweeps: int = 15, refine_iters: int = 2,
                 stream=None):
    """Q_i (eigenvectors as columns) and lam_i of a float32 CUDA stack of
    symmetric matrices A (batch, n, n); with warm_start, Q holds an
    approximate basis on entry and is refined in place.  Returns
    (Q, lam, status), all on the device."""
    import torch
    if A.dtype != torch.float32 or A.dim() != 3 or A.shape[1] != A.shape[2] or not A.is_cuda:
        raise ValueError("A must be a float32 CUDA tensor (batch, n, n)")
    A = A.contiguous()
    batch, n = A.shape[0], A.shape[1]
    if Q is None:
        if warm_start:
            raise ValueError("warm_start needs Q")
        Q = torch.empty_like(A)
    lam = torch.empty((batch, n), dtype=torch.float32, device=A.device)
    b = ctypes.c_size_t(0)
    _check(lib.eigh_scratch_bytes(batch, n, ctypes.byref(b)))
    scratch = torch.empty(b.value, dtype=torch.uint8, device=A.device)
    status = torch.zeros(1, dtype=torch.int32, device=A.device)
    with torch.cuda.device(A.device):
        _check(lib.eigh_batched(A.data_ptr(), Q.data_ptr(), lam.data_ptr(), batch, n, 1 if warm_start else 0,
                                jacobi_sweeps, refine_iters, scratch.data_ptr(), scratch.numel(), status.data_ptr(),
                                _stream_ptr(stream)))
    return Q, lam, status


def gemm_batched(A, B, C=None, alpha: float = 1.0, beta: float = 0.0, gamma: float = 0.0, trans_b: bool = True,
                 out=None, scratch=None, stream=None):
    """D_i = alpha A_i op(B_i) + beta C_i + gamma I on the tensor cores (3xTF32),
    op(B) = B^T if trans_b else B."""
    import torch
    for t in (A, B) + ((C,) if C is not None else ()):
        if t.dtype != torch.float32 or t.dim() != 3 or not t.is_cuda:
            raise ValueError("operands must be float32 CUDA tensors (batch, n, n)")
    A, B = A.contiguous(), B.contiguous()
    C = None if C is None else C.contiguous()
    batch, n = A.shape[0], A.shape[1]
    D = torch.empty_like(A) if out is None else out
    if scratch is None:
        scratch = torch.empty(gemm_scratch_bytes(batch, n), dtype=torch.uint8, device=A.device)
    status = torch.zeros(1, dtype=torch.int32, device=A.device)
    with torch.cuda.device(A.device):
        _check(lib.shampoo_gemm_batched(A.data_ptr(), B.data_ptr(), _ptr(C), D.data_ptr(), batch, n,
                                        0 if trans_b else 1, alpha, beta, gamma, scratch.data_ptr(), scratch.numel(),
                                        status.data_ptr(),
                                        _stream_ptr(stream)))
    return D, status


def dgemm_batched(A, B, C=None, alpha: float = 1.0, beta: float = 0.0, gamma: float = 0.0, out=None,
                  stream=None):
    """D_i = alpha A_i B_i + beta C_i + gamma I in fp64 on the fp64 tensor-core
    instruction (the products of SOLVER_NEWTON_CUBIC_F64)."""
    import torch
    for t in (A, B) + ((C,) if C is not None else ()):
        if t.dtype != torch.float64 or t.dim() != 3 or not t.is_cuda:
            raise ValueError("operands must be float64 CUDA tensors (batch, n, n)")
    A, B = A.contiguous(), B.contiguous()
    C = None if C is None else C.contiguous()
    batch, n = A.shape[0], A.shape[1]
    D = torch.empty_like(A) if out is None else out
    status = torch.zeros(1, dtype=torch.int32, device=A.device)
    with torch.cuda.device(A.device):
        _check(lib.shampoo_dgemm_batched(A.data_ptr(), B.data_ptr(), _ptr(C), D.data_ptr(), batch, n, alpha, beta,
                                         gamma, status.data_ptr(), _stream_ptr(stream)))
    return D, status


def make_soap_config(beta1: float = 0.9, beta2: float = 0.999, eps: float = 1e-8, jacobi_sweeps: int = 15,
                     refine_iters: int = 1) -> SoapConfig:
    return SoapConfig(beta1, beta2, eps, jacobi_sweeps, refine_iters)


class Soap:
    """SOAP (Adam in the eigenbasis of Shampoo's preconditioner) over a fixed
    list of 2-D weights, blocked like ``Shampoo``.  ``cfg`` gives block, beta,
    lr, refresh_every and grad_dtype; ``sc`` the Adam and eigensolver
    settings.  State and scratch are torch allocations owned by this object."""

    def __init__(self, shapes: Sequence[Tuple[int, int]], cfg: Config, sc: SoapConfig, device=None, stream=None):
        import torch
        self.shapes = [tuple(int(x) for x in s) for s in shapes]
        self.cfg, self.sc = cfg, sc
        self.device = torch.device("cuda" if device is None else device)
        rows = _i64_array([s[0] for s in self.shapes])
        cols = _i64_array([s[1] for s in self.shapes])
        sb_, xb = ctypes.c_size_t(0), ctypes.c_size_t(0)
        _check(lib.shampoo_soap_query_sizes(ctypes.byref(cfg), ctypes.byref(sc), len(self.shapes), rows, cols,
                                            ctypes.byref(sb_), ctypes.byref(xb)))
        self.state_bytes, self.scratch_bytes = sb_.value, xb.value
        self.state = torch.empty(self.state_bytes, dtype=torch.uint8, device=self.device)
        self.scratch = torch.empty(self.scratch_bytes, dtype=torch.uint8, device=self.device)
        h = ctypes.c_void_p(None)
        with torch.cuda.device(self.device):
            _check(lib.shampoo_soap_init(ctypes.byref(cfg), ctypes.byref(sc), len(self.shapes), rows, cols,
                                         self.state.data_ptr(), self.state_bytes, self.scratch.data_ptr(),
                                         self.scratch_bytes, _stream_ptr(stream), ctypes.byref(h)))
        self._h = h
        self._destroy = lib.shampoo_soap_destroy
        self.nb = sum(-(-m // cfg.block) * -(-n // cfg.block) for m, n in self.shapes)
        self._wbuf = (ctypes.c_void_p * len(self.shapes))()
        self._gbuf = (ctypes.c_void_p * len(self.shapes))()

    def __del__(self):
        h = getattr(self, "_h", None)
        destroy = getattr(self, "_destroy", None)
        if h is not None and h.value and destroy is not None:
            destroy(h)
            self._h = None

    def step(self, weights, grads, stream=None):
        import torch
        want = torch.bfloat16 if self.cfg.grad_dtype == BF16 else torch.float32
        if len(weights) != len(self.shapes) or len(grads) != len(self.shapes):
            raise ValueError("one weight and one gradient per shape")
        for i, (w, g) in enumerate(zip(weights, grads)):
            if w.dtype != torch.float32 or g.dtype != want:
                raise TypeError(f"param {i}: weights must be float32 and grads {want}")
            if tuple(w.shape) != self.shapes[i] or tuple(g.shape) != self.shapes[i]:
                raise ValueError(f"param {i}: shape mismatch")
            if not (w.is_contiguous() and g.is_contiguous()):
                raise ValueError(f"param {i}: weight and gradient must be contiguous")
            self._wbuf[i] = w.data_ptr()
            self._gbuf[i] = g.data_ptr()
        _check(lib.shampoo_soap_step(self._h, self._wbuf, self._gbuf, _stream_ptr(stream)))

    def status(self, reset: bool = False) -> int:
        s = ctypes.c_int32(0)
        _check(lib.shampoo_soap_get_status(self._h, ctypes.byref(s), 1 if reset else 0))
        return s.value

    def views(self):
        """dict of float32 (nb, B, B) views: L, R, QL, QR, m, v."""
        import torch
        ptrs = [ctypes.c_void_p() for _ in range(6)]
        step = ctypes.c_int64(0)
        _check(lib.shampoo_soap_views(self._h, *[ctypes.byref(p) for p in ptrs], ctypes.byref(step)))
        fl = self.state.view(torch.float32)
        base = self.state.data_ptr()
        B, nb = self.cfg.block, self.nb
        out = {}
        for name, p in zip(("L", "R", "QL", "QR", "m", "v"), ptrs):
            o = (p.value - base) // 4
            out[name] = fl[o:o + nb * B * B].view(nb, B, B)
        out["step"] = step.value
        return out


class BlockPacker:
    """Moves a fixed list of blocks between matrices and a packed fp32 buffer
    in one kernel launch per call (shampoo_pack_blocks).

    ``blocks``: (param, row0, col0, r, c, offset) tuples, offset in floats of
    the packed buffer.  The device table is built once."""

    def __init__(self, blocks, device):
        import torch
        self.blocks = [tuple(int(x) for x in b) for b in blocks]
        self.n = len(self.blocks)
        self.table = torch.tensor(self.blocks if self.blocks else [[0] * 6], dtype=torch.int64, device=device)
        self.max_rows = max([b[3] for b in self.blocks], default=1)
        self.max_cols = max([b[4] for b in self.blocks], default=1)

    def _call(self, mats, packed, direction, scale, stream):
        import torch
        if self.n == 0:
            return
        ptrs = (ctypes.c_void_p * len(mats))(*[m.data_ptr() for m in mats])
        ld = _i64_array([m.stride(0) if m.dim() == 2 else m.shape[-1] for m in mats])
        for m in mats:
            if m.dim() != 2 or (m.shape[1] > 1 and m.stride(1) != 1):
                raise ValueError("matrices must be 2-D with unit column stride")
        dt = BF16 if mats[0].dtype == torch.bfloat16 else F32
        if packed.dtype != torch.float32 or not packed.is_contiguous():
            raise ValueError("the packed buffer must be contiguous float32")
        _check(lib.shampoo_pack_blocks(self.table.data_ptr(), self.n, len(mats), ptrs, ld, dt, packed.data_ptr(),
                                       direction, scale, self.max_rows, self.max_cols, _stream_ptr(stream)))

    def gather(self, mats, packed, scale: float = 1.0, stream=None):
        self._call(mats, packed, 0, scale, stream)

    def scatter(self, packed, mats, stream=None):
        self._call(mats, packed, 1, 1.0, stream)


# ---------------------------------------------------------------------------
# profiling
# ---------------------------------------------------------------------------

@dataclass
class KernelTally:
    launches: int
    total_ms: float
    alg_flops: float
    alg_bytes: float


def profile_enable(on: bool = True):
    lib.shampoo_profile_enable(1 if on else 0)


def profile_reset():
    lib.shampoo_profile_reset()


def profile_read(kind: int) -> KernelTally:
    n = ctypes.c_int64(0)
    ms, fl, by = ctypes.c_double(0), ctypes.c_double(0), ctypes.c_double(0)
    _check(lib.shampoo_profile_read(kind, ctypes.byref(n), ctypes.byref(ms), ctypes.byref(fl), ctypes.byref(by)))
    return KernelTally(n.value, ms.value, fl.value, by.value)


def launch_count() -> int:
    return int(lib.shampoo_launch_count())
