"""C-ABI boundary without a GPU: the library loads, exports every symbol that
include/shampoo.h declares, and its host-only entry points validate
arguments and compute sizes (no CUDA call is made by these)."""
import ctypes
import os
import re

import pytest

import oracle
import workloads

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def sb():
    import shampoo_family_second_b200 as sb
    return sb


def header_functions():
    text = open(os.path.join(ROOT, "include", "shampoo.h")).read()
    return re.findall(r"^SHAMPOO_API [^(]*?\b(\w+)\(", text, flags=re.M)


def test_library_exports_every_declared_symbol(sb):
    declared = header_functions()
    assert len(declared) >= 15
    lib = ctypes.CDLL(sb.LIB_PATH)
    for name in declared:
        assert hasattr(lib, name), name
    assert tuple(declared) == sb.EXPORTS


def test_status_strings(sb):
    assert sb.lib.shampoo_status_string(0) == b"SHAMPOO_OK"
    assert sb.lib.shampoo_status_string(-3) == b"SHAMPOO_ERR_WORKSPACE"
    assert sb.lib.shampoo_status_string(12345) == b"SHAMPOO_UNKNOWN_STATUS"


def test_query_sizes_memory_is_quadratic_per_block(sb):
    """One B x B statistic per side per block (notes' "Key Components":
    O(m^2 + n^2) memory): state = stats (2 nb B^2 fp32) + roots (2 nb B^2
    fp32) + one B-vector per root (the power iterate of the scale) + a small
    table."""
    for name in ("tiny", "lowrank", "gpt2", "llama"):
        wl = workloads.workload(name)
        cfg = sb.config_from_workload(wl)
        state, scratch = sb.query_sizes(cfg, wl.shapes)
        nb = len(oracle.block_table(wl.shapes, wl.block))
        core = 2 * nb * wl.block ** 2 * 4 * 2
        vecs = 2 * nb * wl.block * 4
        assert core + vecs <= state <= core + vecs + 64 * 1024 + 64 * nb
        assert scratch > 3 * nb * wl.block ** 2 * 4


def test_scratch_holds_the_split_roots_where_they_pay(sb):
    """Scratch per (B x B) block element, beside the solver's: G and G^T
    (fp32 both, or bf16 both), T (fp32), the XL planes (three bf16, bf16
    gradients without momentum only) and the stored tf32 split of XR (hi and
    lo, fp32, only when roots are kept for several steps).  Checked as exact
    differences between configurations, so the solver's share cancels."""
    shapes = [(1024, 1024)]
    nb, B = 4, 512
    elems = nb * B * B

    def scratch(**kw):
        base = dict(block=B, beta=0.95, eps=1e-8, lr=1e-3, solver=sb.SOLVER_NEWTON_CUBIC)
        base.update(kw)
        return sb.query_sizes(sb.make_config(**base), shapes)[1]

    f32_every = scratch(refresh_every=1)
    f32_ten = scratch(refresh_every=10)
    bf16_ten = scratch(refresh_every=10, grad_dtype=sb.BF16)
    bf16_mom = scratch(refresh_every=10, grad_dtype=sb.BF16, momentum=0.9)
    assert f32_ten - f32_every == 2 * elems * 4            # XR hi and lo
    assert bf16_ten - f32_ten == 3 * elems * 2 - elems * 4  # XL planes in, the fp32 G^T stack out
    assert bf16_mom == f32_ten                              # momentum: fp32 G^T kept, no planes


@pytest.mark.parametrize("field,value", [("block", 48), ("block", 2048), ("root_p", 3), ("solver", 7),
                                         ("iters", 0), ("refresh_every", 0), ("beta", 1.5), ("eps", -1.0),
                                         ("grad_dtype", 5)])
def test_config_validation(sb, field, value):
    cfg = sb.make_config(32, 1.0, 1e-6, 1e-3)
    setattr(cfg, field, value)
    with pytest.raises(sb.ShampooError) as e:
        sb.query_sizes(cfg, [(64, 32)])
    assert e.value.code == sb.ERR_INVALID_ARG
    assert sb.last_error()


def test_chebyshev_needs_interval(sb):
    cfg = sb.make_config(32, 1.0, 0.0, 1e-3, solver=sb.SOLVER_CHEBYSHEV, cheb_degree=16, cheb_lo=0.0)
    with pytest.raises(sb.ShampooError):
        sb.query_sizes(cfg, [(64, 32)])
    cfg.cheb_degree = 1
    cfg.eps = 1e-3
    with pytest.raises(sb.ShampooError):
        sb.query_sizes(cfg, [(64, 32)])


def test_bad_shapes(sb):
    cfg = sb.make_config(32, 1.0, 1e-6, 1e-3)
    with pytest.raises(sb.ShampooError):
        sb.query_sizes(cfg, [(0, 32)])
    with pytest.raises(sb.ShampooError):
        sb.query_sizes(cfg, [])


def test_inv_root_argument_errors_before_any_launch(sb):
    L = sb.lib
    n0 = sb.launch_count()
    # NULL pointers, bad n, bad p: all rejected on the host.
    assert L.inv_root_batched(None, None, 4, 64, 4, 0.0, 0, 10, 0.0, 16, 0.0, None, 0, None, None, None) == -1
    assert L.inv_root_batched(1024, 1024, 4, 65, 4, 0.0, 0, 10, 0.0, 16, 0.0, 4096, 1 << 20, None, None, None) == -1
    assert L.inv_root_batched(1024, 1024, 4, 64, 3, 0.0, 0, 10, 0.0, 16, 0.0, 4096, 1 << 20, None, None, None) == -1
    assert L.inv_root_batched(1024, 1024, 4, 64, 4, 0.0, 0, 0, 0.0, 16, 0.0, 4096, 1 << 20, None, None, None) == -1
    assert L.inv_root_batched(1024, 1024, 0, 64, 4, 0.0, 0, 10, 0.0, 16, 0.0, 4096, 1 << 20, None, None, None) == 0
    assert sb.launch_count() == n0


def test_scratch_sizes(sb):
    a = sb.inv_root_scratch_bytes(64, 1024, sb.SOLVER_NEWTON)
    b = sb.inv_root_scratch_bytes(128, 1024, sb.SOLVER_NEWTON)
    per = b - a
    assert per == 64 * (7 * 1024 * 1024 * 4 + 4 * (8 + 64 + 2))   # Newton: 7 stacks per matrix
    assert sb.inv_root_scratch_bytes(64, 1024, sb.SOLVER_NEWTON_DB) < a
    # the second-degree correction reuses the Newton stacks (T, T^2, T^4 also hold D = I - M)
    assert sb.inv_root_scratch_bytes(64, 1024, sb.SOLVER_NEWTON_CUBIC) == a
    assert sb.gemm_scratch_bytes(3, 256) == 0   # operands are split on chip
    # the no-alloc entry point's fixed 32 MiB covers one matrix of every fp32 solver at every size
    for solver in (sb.SOLVER_NEWTON, sb.SOLVER_NEWTON_DB, sb.SOLVER_CHEBYSHEV, sb.SOLVER_NEWTON_CUBIC):
        assert sb.inv_root_scratch_bytes(1, 1024, solver) <= 32 << 20
    with pytest.raises(sb.ShampooError):
        sb.inv_root_scratch_bytes(4, 100, 0)
    # fp64 iterates: the same 7 stacks at 8 bytes per element; beyond the
    # no-alloc array at n = 1024
    f64 = sb.inv_root_scratch_bytes(128, 1024, sb.SOLVER_NEWTON_CUBIC_F64) - \
        sb.inv_root_scratch_bytes(64, 1024, sb.SOLVER_NEWTON_CUBIC_F64)
    assert f64 == 64 * (7 * 1024 * 1024 * 8 + 4 * (8 + 64 + 2))
    assert sb.inv_root_scratch_bytes(1, 1024, sb.SOLVER_NEWTON_CUBIC_F64) > 32 << 20
    with pytest.raises(sb.ShampooError):   # no solver 5
        sb.inv_root_scratch_bytes(4, 256, 5)


def test_every_solver_is_accepted_by_the_step_config(sb):
    """Each solver id of the header passes the step's argument checks (sizes
    are queried without a GPU); an unknown id is refused."""
    for solver in (sb.SOLVER_NEWTON, sb.SOLVER_NEWTON_DB, sb.SOLVER_NEWTON_CUBIC, sb.SOLVER_NEWTON_CUBIC_F64):
        state, scratch = sb.query_sizes(sb.make_config(256, 0.95, 1e-8, 1e-3, solver=solver), [(1024, 1024)])
        assert state > 0 and scratch > 0
    with pytest.raises(sb.ShampooError):
        sb.query_sizes(sb.make_config(256, 0.95, 1e-8, 1e-3, solver=5), [(1024, 1024)])


def test_init_rejects_missing_buffers_without_cuda(sb):
    cfg = sb.make_config(32, 1.0, 1e-6, 1e-3)
    rows = (ctypes.c_int64 * 1)(64)
    cols = (ctypes.c_int64 * 1)(32)
    h = ctypes.c_void_p()
    assert sb.lib.shampoo_init(ctypes.byref(cfg), 1, rows, cols, None, 0, None, 0, None, ctypes.byref(h)) == -1
    assert sb.lib.shampoo_init(ctypes.byref(cfg), 1, rows, cols, 256, 0, 512, 0, None, ctypes.byref(h)) == -3
    assert sb.lib.shampoo_init(ctypes.byref(cfg), 1, rows, cols, 255, 1 << 30, 512, 1 << 30, None,
                               ctypes.byref(h)) == -2


def test_strided_step_refuses_a_null_handle():
    """The strided step checks its arguments before any launch: a null handle
    is refused with ERR_INVALID_ARG without touching the device."""
    import ctypes
    sb = pytest.importorskip("shampoo_family_second_b200")
    ld = (ctypes.c_int64 * 1)(4)
    w = (ctypes.c_void_p * 1)(None)
    assert sb.lib.shampoo_step_strided(None, w, w, ld, None) == sb.ERR_INVALID_ARG
    assert "handle" in sb.last_error()
    assert sb.lib.shampoo_sync_statistics(None, None) == sb.ERR_INVALID_ARG
    assert "handle" in sb.last_error()


def test_momentum_state_is_one_more_block_stack(sb):
    """Momentum adds one (nb, B, B) fp32 stack to the state and nothing to the
    scratch; alpha must lie in [0, 1)."""
    shapes = [(1024, 768), (300, 512)]
    off = sb.make_config(256, 0.95, 1e-8, 1e-3)
    on = sb.make_config(256, 0.95, 1e-8, 1e-3, momentum=0.9)
    s0, x0 = sb.query_sizes(off, shapes)
    s1, x1 = sb.query_sizes(on, shapes)
    nb = len(oracle.block_table(shapes, 256))
    assert x1 == x0
    assert s1 - s0 == nb * 256 * 256 * 4
    for bad in (1.0, -0.1, float("nan")):
        with pytest.raises(sb.ShampooError):
            sb.query_sizes(sb.make_config(256, 0.95, 1e-8, 1e-3, momentum=bad), shapes)


def test_tensor_sizes_and_validation(sb):
    """Tensor Shampoo: orders 2..4; state holds one statistic and one root per
    mode (padded to multiples of 32), or two vectors for a mode past the
    diagonal threshold."""
    cfg = sb.make_config(32, 0.9, 1e-4, 1e-3, solver=3)
    state, scratch = sb.tensor_query_sizes(cfg, [(3, 3, 64, 128)])
    per_mode = [32, 32, 64, 128]
    assert state >= sum(2 * n * n * 4 for n in per_mode)
    assert scratch > 0
    for bad in ([(5,)], [(2, 2, 2, 2, 2)], [(0, 4)]):
        with pytest.raises(sb.ShampooError) as e:
            sb.tensor_query_sizes(cfg, bad)
        assert e.value.code == sb.ERR_INVALID_ARG
    # a dimension above the diagonal threshold keeps a vector: 2048 + 2048 floats, not 2048^2
    state_d, _ = sb.tensor_query_sizes(cfg, [(2048, 8)])
    assert state_d < 2 * 2048 * 2048 * 4
    with pytest.raises(sb.ShampooError) as e:
        sb.tensor_query_sizes(cfg, [((1 << 20) + 1, 2)])
    assert e.value.code == sb.ERR_UNSUPPORTED
    with pytest.raises(sb.ShampooError) as e:
        sb.tensor_query_sizes(sb.make_config(32, 0.9, 1e-4, 1e-3, solver=3, diag_threshold=2000), [(8, 8)])
    assert e.value.code == sb.ERR_INVALID_ARG
    db = sb.make_config(32, 0.9, 1e-4, 1e-3, solver=1)
    sb.tensor_query_sizes(db, [(40, 50)])
    with pytest.raises(sb.ShampooError):
        sb.tensor_query_sizes(db, [(4, 5, 6)])


def test_eigh_argument_errors(sb):
    b = ctypes.c_size_t(0)
    assert sb.lib.eigh_scratch_bytes(4, 64, ctypes.byref(b)) == 0 and b.value >= 4 * 5 * 64 * 64 * 4
    assert sb.lib.eigh_scratch_bytes(4, 48, ctypes.byref(b)) == sb.ERR_INVALID_ARG
    assert sb.lib.eigh_batched(None, None, None, 0, 64, 0, 10, 2, None, 0, None, None) == 0
    assert sb.lib.eigh_batched(None, None, None, 2, 64, 0, 10, 2, None, 0, None, None) == sb.ERR_INVALID_ARG


def test_soap_sizes_and_validation(sb):
    """SOAP keeps statistics, bases and their transposes (2 nb stacks each) and
    the two moments (nb each): 8 nb block matrices of state."""
    cfg = sb.make_config(128, 0.95, 0.0, 1e-3, refresh_every=10)
    sc = sb.make_soap_config()
    rows = (ctypes.c_int64 * 2)(256, 128)
    cols = (ctypes.c_int64 * 2)(256, 384)
    st, xs = ctypes.c_size_t(0), ctypes.c_size_t(0)
    assert sb.lib.shampoo_soap_query_sizes(ctypes.byref(cfg), ctypes.byref(sc), 2, rows, cols, ctypes.byref(st),
                                           ctypes.byref(xs)) == 0
    nb = 4 + 3
    assert st.value >= 8 * nb * 128 * 128 * 4
    for bad in (sb.make_soap_config(beta1=1.0), sb.make_soap_config(eps=0.0), sb.make_soap_config(jacobi_sweeps=0)):
        assert sb.lib.shampoo_soap_query_sizes(ctypes.byref(cfg), ctypes.byref(bad), 2, rows, cols,
                                               ctypes.byref(st), ctypes.byref(xs)) == sb.ERR_INVALID_ARG
