"""The full blocked Shampoo step on the GPU vs the float64 oracle.

Per step and per block: statistics (GPU fp32 L, R vs the float64 oracle's,
1e-5 relative Frobenius), roots (the GPU roots vs the oracle's exact root of
the GPU's own fp32 statistics: isolates the solver from fp32 statistics
rounding), the update P_b = -(W_t - W_{t-1}) / lr against the float64
product of the GPU's own roots and the gradient (the apply stage alone:
2e-5 times the cancellation factor, parity.apply_check), and the same update
against the fully float64 pipeline, <= max(2e-3, 2 F_update) relative
Frobenius per block.

Small ragged blocks have rank-deficient statistics (a 32 x 15 gradient
block gives a 32 x 32 L of rank 15).  On the null space the root is set by
eps and by rounding noise alone, and an iterative fp32 solver's error there
is larger than single-precision LAPACK's; the gradient has no component
there, so the update does not see it.  Roots are therefore compared on the
range space of the statistics at max(2e-3, 2 F) (F measured on the same
projection), and on the null space the root's eigenvalues must lie within
10% of the band [(lam_max + eps)^{-1/p}, (lam_min + eps)^{-1/p}] spanned by
the null-space eigenvalues lam (tests/parity.py, root_checks).
Full-rank statistics get the plain 2 F gate.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import oracle
import workloads
from parity import Fp32ReferenceShampoo, apply_check, root_checks, root_gate, update_gate

TOL_UPDATE = 2e-3
TOL_ROOT = 2e-3
NULL_SPREAD = 0.10
TOL_STATS = 1e-5


@pytest.fixture(scope="module")
def sb():
    import shampoo_family_second_b200 as sb
    return sb


def bf16_tensor(x32):
    return torch.from_numpy(workloads.bf16_bits(x32).view(np.int16)).view(torch.bfloat16)


def run_parity(sb, wl, steps, check_roots=True, blocks=None):
    cfg = sb.config_from_workload(wl)
    opt = sb.Shampoo(wl.shapes, cfg)
    W = [torch.zeros(s, dtype=torch.float32, device="cuda") for s in wl.shapes]
    ref = oracle.ShampooOracle(wl.shapes, wl.block, wl.beta, wl.eps, wl.lr, wl.root_p, wl.refresh_every,
                               blocks=blocks)
    table = opt.block_table()
    assert [tuple(t) for t in table] == [(b.param, b.row0, b.col0, b.r, b.c) for b in ref.table]
    ref32 = Fp32ReferenceShampoo(wl.shapes, wl.block, wl.beta, wl.eps, wl.root_p, wl.refresh_every, ref.active)
    stream = workloads.GradientStream(wl)
    worst = {"update": 0.0, "root": 0.0, "stats": 0.0, "apply": 0.0}
    for t in range(steps):
        grads = stream.next()
        if wl.grad_dtype == workloads.DTYPE_BF16:
            G = [bf16_tensor(g).cuda() for g in grads]
        else:
            G = [torch.from_numpy(g).cuda() for g in grads]
        before = [w.clone() for w in W]
        opt.step(W, G)
        P_ref = ref.step(grads)
        P_32 = ref32.step(grads)
        torch.cuda.synchronize()
        dW = [((b.double() - a.double()) / wl.lr).cpu().numpy() for a, b in zip(W, before)]
        L, R = opt.statistics()
        L, R = L.cpu().numpy().astype(np.float64), R.cpu().numpy().astype(np.float64)
        XL, XR = opt.roots()
        XL, XR = XL.cpu().numpy().astype(np.float64), XR.cpu().numpy().astype(np.float64)
        for b in ref.active:
            blk = ref.table[b]
            Pg = dW[blk.param][blk.row0:blk.row0 + blk.r, blk.col0:blk.col0 + blk.c]
            ea, ga = apply_check(Pg, XL[b, :blk.r, :blk.r], ref.block_of(grads, b), XR[b, :blk.c, :blk.c])
            worst["apply"] = max(worst["apply"], ea)
            assert ea < ga, (t, b, "apply", ea, ga)
            e = oracle.rel_fro(Pg, P_ref[b])
            worst["update"] = max(worst["update"], e)
            assert e < update_gate(P_32[b], P_ref[b]), (t, b, "update", e)
            es = max(oracle.rel_fro(L[b, :blk.r, :blk.r], ref.L[b]), oracle.rel_fro(R[b, :blk.c, :blk.c], ref.R[b]))
            worst["stats"] = max(worst["stats"], es)
            assert es < TOL_STATS, (t, b, "stats", es)
            if check_roots and t % wl.refresh_every == 0:
                for X, S, v in ((XL, L, blk.r), (XR, R, blk.c)):
                    er, gate, spread = root_checks(X[b, :v, :v], S[b, :v, :v], wl.root_p, wl.eps)
                    worst["root"] = max(worst["root"], er)
                    assert er < gate, (t, b, "root", er, gate)
                    if spread is not None:
                        assert spread < NULL_SPREAD, (t, b, "null-space root", spread)
    assert opt.status() == 0
    print(f"\n{wl.name} {wl.shapes}: worst update {worst['update']:.2e}, root {worst['root']:.2e}, "
          f"apply {worst['apply']:.2e}, statistics {worst['stats']:.2e}")
    return worst


def test_tiny_workload(sb):
    """Tiny: one 64x32 weight, block 32, 10 steps, beta = 1, Newton 20 iterations."""
    wl = workloads.workload("tiny")
    run_parity(sb, wl, wl.steps)


@pytest.mark.parametrize("shapes", [((33, 47),), ((64, 45), (20, 96)), ((100, 33),)])
def test_ragged_blocks(sb, shapes):
    wl = workloads.workload("tiny", shapes=shapes, steps=4, iters=40, tol=1e-5, beta=0.9, eps=1e-4)
    run_parity(sb, wl, wl.steps)


@pytest.mark.parametrize("solver", [1, 2, 3])
def test_other_solvers_in_step(sb, solver):
    # Chebyshev needs a spectral lower bound: eps large enough that a = eps / s
    # keeps the degree-32 interpolant within tolerance.
    over = dict(solver=solver, iters=30, tol=0.0)
    if solver == 2:
        over.update(eps=1.0, cheb_degree=32, cheb_lo=0.0)
    wl = workloads.workload("tiny", steps=3, **over)
    cfg = sb.config_from_workload(wl)
    opt = sb.Shampoo(wl.shapes, cfg)
    W = [torch.zeros(s, dtype=torch.float32, device="cuda") for s in wl.shapes]
    stream = workloads.GradientStream(wl)
    from oracle import chebyshev as och
    for t in range(wl.steps):
        G = stream.next()
        opt.step(W, [torch.from_numpy(g).cuda() for g in G])
        torch.cuda.synchronize()
        L, R = opt.statistics()
        XL, XR = opt.roots()
        L, R, XL, XR = [x.cpu().numpy().astype(np.float64) for x in (L, R, XL, XR)]
        for b in range(opt.nb):
            for X, S in ((XL, L), (XR, R)):
                if solver == 2:
                    ref = och.chebyshev_inverse_root(S[b], wl.root_p, wl.eps, wl.cheb_degree, lo=0.0)
                else:
                    ref = oracle.inverse_root(S[b], wl.root_p, wl.eps)
                assert oracle.rel_fro(X[b], ref) < TOL_ROOT
    assert opt.status() == 0


def test_p2_step(sb):
    wl = workloads.workload("tiny", root_p=2, steps=3, iters=30)
    run_parity(sb, wl, wl.steps)


def test_bf16_gradients(sb):
    wl = workloads.workload("tiny", shapes=((64, 96),), grad_dtype=workloads.DTYPE_BF16, steps=3, iters=30)
    run_parity(sb, wl, wl.steps)


def test_refresh_schedule(sb):
    wl = workloads.workload("tiny", steps=7, refresh_every=3, iters=30, beta=0.9)
    run_parity(sb, wl, wl.steps)


def test_checkpoint_resume_bit_identical(sb):
    wl = workloads.workload("tiny", shapes=((64, 96),), steps=6, iters=25)
    cfg = sb.config_from_workload(wl)
    grads = [[torch.from_numpy(g).cuda() for g in gs]
             for gs in (workloads.GradientStream(wl).next() for _ in range(1))]
    stream = workloads.GradientStream(wl)
    grads = [[torch.from_numpy(g).cuda() for g in stream.next()] for _ in range(wl.steps)]
    a = sb.Shampoo(wl.shapes, cfg)
    Wa = [torch.zeros(s, device="cuda") for s in wl.shapes]
    for t in range(wl.steps):
        a.step(Wa, grads[t])
        if t == 2:
            ckpt = a.state_dict()
            Wckpt = [w.clone() for w in Wa]
    b = sb.Shampoo(wl.shapes, cfg)
    b.load_state_dict(ckpt)
    Wb = Wckpt
    for t in range(3, wl.steps):
        b.step(Wb, grads[t])
    torch.cuda.synchronize()
    for x, y in zip(Wa, Wb):
        assert torch.equal(x, y)
    assert b.step_count == a.step_count == wl.steps


def test_sharded_collectives_on_a_single_rank_nccl_group(sb, tmp_path):
    """The sharded optimizer's collective path on NCCL, with one rank (every
    GPU call here has one GPU, and ranks that wait on each other cannot share
    one): the packed reduce-scatter of local gradients and the all-gather of
    updated blocks run as NCCL calls on the real packed buffers, where with a
    single rank each is a copy.  Both gradient modes end with weights
    bit-identical to the unsharded step."""
    from datetime import timedelta

    import torch.distributed as dist
    from shampoo_family_second_b200 import sharded
    if dist.is_initialized():
        pytest.skip("a process group is already initialised in this process")
    store = dist.FileStore(str(tmp_path / "store"), 1)
    dist.init_process_group("nccl", store=store, rank=0, world_size=1, timeout=timedelta(seconds=60))
    try:
        shapes = ((96, 80), (40, 70))
        wl = workloads.workload("tiny", shapes=shapes, block=32, steps=3, iters=30, tol=1e-5, beta=0.9, eps=1e-4,
                                solver=workloads.SOLVER_NEWTON_CUBIC)
        cfg = sb.config_from_workload(wl)
        full = sb.Shampoo(shapes, cfg)
        reduced = sharded.ShardedShampoo(shapes, cfg)
        packed = sharded.ShardedShampoo(shapes, cfg, grads_reduced=False)
        assert reduced.collective and packed.collective and dist.get_backend() == "nccl"
        W1, W2, W3 = ([torch.zeros(s, dtype=torch.float32, device="cuda") for s in shapes] for _ in range(3))
        stream = workloads.GradientStream(wl)
        for _ in range(wl.steps):
            G = [torch.from_numpy(g).cuda() for g in stream.next()]
            full.step(W1, G)
            reduced.step(W2, G)
            packed.step(W3, G)
        torch.cuda.synchronize()
        for a, b, c in zip(W1, W2, W3):
            assert torch.equal(a, b) and torch.equal(a, c)
    finally:
        dist.destroy_process_group()


def test_bf16_checkpoint_resume_between_refreshes(sb):
    """bf16 gradients, blocks of 256 with ragged edges, refresh every 3 steps.
    The first apply product reads the roots as three bf16 planes, split after
    each refresh; a handle restored from a checkpoint taken after step 3
    resumes at step 4, which does not refresh, so it must split the restored
    roots first.  Both runs end with bit-identical weights, and every update
    of the resumed run matches XL_gpu G XR_gpu in float64 (the apply stage)."""
    shapes = ((300, 520), (256, 200))
    wl = workloads.workload("tiny", shapes=shapes, block=256, grad_dtype=workloads.DTYPE_BF16, steps=8,
                            iters=30, tol=1e-5, beta=0.9, eps=1e-4, refresh_every=3,
                            solver=workloads.SOLVER_NEWTON_CUBIC)
    cfg = sb.config_from_workload(wl)
    stream = workloads.GradientStream(wl)
    host = [stream.next() for _ in range(wl.steps)]
    grads = [[bf16_tensor(g).cuda() for g in gs] for gs in host]
    a = sb.Shampoo(wl.shapes, cfg)
    Wa = [torch.zeros(s, device="cuda") for s in wl.shapes]
    for t in range(wl.steps):
        a.step(Wa, grads[t])
        if t == 3:
            ckpt = {k: (v.clone() if torch.is_tensor(v) else v) for k, v in a.state_dict().items()}
            Wckpt = [w.clone() for w in Wa]
    b = sb.Shampoo(wl.shapes, cfg)
    b.load_state_dict(ckpt)
    Wb = Wckpt
    table = [tuple(x) for x in b.block_table()]
    for t in range(4, wl.steps):
        before = [w.double() for w in Wb]
        b.step(Wb, grads[t])
        torch.cuda.synchronize()
        XL, XR = [x.cpu().numpy().astype(np.float64) for x in b.roots()]
        for k, (param, r0, c0, r, c) in enumerate(table):
            Pg = ((before[param] - Wb[param].double()) / wl.lr).cpu().numpy()[r0:r0 + r, c0:c0 + c]
            G = host[t][param][r0:r0 + r, c0:c0 + c]
            ea, ga = apply_check(Pg, XL[k, :r, :r], G, XR[k, :c, :c])
            assert ea < ga, (t, k, ea, ga)
    for x, y in zip(Wa, Wb):
        assert torch.equal(x, y)
    assert b.status() & ~sb.DEVFLAG_STAGNATED == 0


def test_nonfinite_gradient_sets_status(sb):
    wl = workloads.workload("tiny", steps=1)
    opt = sb.Shampoo(wl.shapes, sb.config_from_workload(wl))
    W = [torch.zeros(s, device="cuda") for s in wl.shapes]
    g = torch.randn(wl.shapes[0], device="cuda")
    g[5, 7] = float("inf")
    opt.step(W, [g])
    st = opt.status(reset=True)
    assert st & sb.DEVFLAG_NONFINITE
    assert opt.status() == 0


def test_launch_count_increases(sb):
    wl = workloads.workload("tiny", steps=1)
    opt = sb.Shampoo(wl.shapes, sb.config_from_workload(wl))
    W = [torch.zeros(s, device="cuda") for s in wl.shapes]
    n0 = sb.launch_count()
    opt.step(W, [torch.randn(wl.shapes[0], device="cuda")])
    torch.cuda.synchronize()
    # stack + stats + norm + prologue + 20 + 19 * 2 Newton launches + finalize + 2 apply (a root
    # refresh every step: the second apply splits XR on chip, with no split pass)
    assert sb.launch_count() - n0 == 1 + 1 + 1 + 1 + 20 + 19 * 2 + 1 + 2


@pytest.mark.parametrize("block,shape", [(512, (700, 1024)), (1024, (1024, 2048))])
def test_large_blocks_parity(sb, block, shape):
    """Blocks of 512 (with a ragged block row of 188) and 1024 with the
    workloads' solver, over two steps with beta 0.9: every statistic matches
    the float64 oracle, every root passes its gate, every block's update
    matches the float64 product of the GPU's own roots and gradient (the
    apply stage) and the fully float64 pipeline (end to end)."""
    wl = workloads.workload("tiny", shapes=(shape,), block=block, steps=2, iters=30, tol=1e-5, beta=0.9, eps=1e-4,
                            solver=workloads.SOLVER_NEWTON_CUBIC)
    opt = sb.Shampoo(wl.shapes, sb.config_from_workload(wl))
    W = [torch.zeros(s, dtype=torch.float32, device="cuda") for s in wl.shapes]
    ref = oracle.ShampooOracle(wl.shapes, wl.block, wl.beta, wl.eps, wl.lr, wl.root_p, wl.refresh_every)
    ref32 = Fp32ReferenceShampoo(wl.shapes, wl.block, wl.beta, wl.eps, wl.root_p, wl.refresh_every, ref.active)
    stream = workloads.GradientStream(wl)
    for t in range(wl.steps):
        G = stream.next()
        before = [w.double() for w in W]
        opt.step(W, [torch.from_numpy(g).cuda() for g in G])
        P_ref = ref.step(G)
        P_32 = ref32.step(G)
        torch.cuda.synchronize()
        dW = [((a - w.double()) / wl.lr).cpu().numpy() for a, w in zip(before, W)]
        XL, XR = opt.roots()
        XL, XR = XL.cpu().numpy().astype(np.float64), XR.cpu().numpy().astype(np.float64)
        for b, blk in enumerate(ref.table):
            Pg = dW[blk.param][blk.row0:blk.row0 + blk.r, blk.col0:blk.col0 + blk.c]
            ea, ga = apply_check(Pg, XL[b, :blk.r, :blk.r], ref.block_of(G, b), XR[b, :blk.c, :blk.c])
            assert ea < ga, (t, b, "apply", ea, ga)
            e = oracle.rel_fro(Pg, P_ref[b])
            assert e < update_gate(P_32[b], P_ref[b]), (t, b, "update", e)
    L, R = opt.statistics()
    L, R = L.cpu().numpy(), R.cpu().numpy()
    for b, blk in enumerate(ref.table):
        assert oracle.rel_fro(L[b, :blk.r, :blk.r].astype(np.float64), ref.L[b]) < TOL_STATS
        assert oracle.rel_fro(R[b, :blk.c, :blk.c].astype(np.float64), ref.R[b]) < TOL_STATS
    for b, blk in enumerate(ref.table):
        for X, S, v in ((XL, L, blk.r), (XR, R, blk.c)):
            er, gate, _ = root_checks(X[b, :v, :v], S[b, :v, :v].astype(np.float64), wl.root_p, wl.eps)
            assert er < gate, (b, er, gate)
    assert opt.status() & ~sb.DEVFLAG_STAGNATED == 0


def test_statistics_between_refreshes(sb):
    """Steps without a refresh update only the statistics tiles on or above the
    diagonal; the rest is filled from the transpose on refresh steps (before
    the roots) and by statistics() for readers.  Blocks of 512 (two tile
    columns, a ragged block row of 188), refresh every 3 steps, 7 steps: the
    statistics read after every step equal the float64 oracle's; the roots of
    the refreshes at steps 3 and 6, taken after two steps that left the lower
    tiles stale, pass their gate against the GPU's own statistics; every
    update matches XL_gpu G XR_gpu in float64."""
    wl = workloads.workload("tiny", shapes=((700, 1024),), block=512, steps=7, iters=30, tol=1e-5, beta=0.9,
                            eps=1e-4, refresh_every=3, solver=workloads.SOLVER_NEWTON_CUBIC)
    opt = sb.Shampoo(wl.shapes, sb.config_from_workload(wl))
    W = [torch.zeros(s, dtype=torch.float32, device="cuda") for s in wl.shapes]
    ref = oracle.ShampooOracle(wl.shapes, wl.block, wl.beta, wl.eps, wl.lr, wl.root_p, wl.refresh_every)
    stream = workloads.GradientStream(wl)
    for t in range(wl.steps):
        G = stream.next()
        before = [w.double() for w in W]
        opt.step(W, [torch.from_numpy(g).cuda() for g in G])
        ref.step(G)
        torch.cuda.synchronize()
        dW = [((a - w.double()) / wl.lr).cpu().numpy() for a, w in zip(before, W)]
        XL, XR = [x.cpu().numpy().astype(np.float64) for x in opt.roots()]
        L, R = [x.cpu().numpy().astype(np.float64) for x in opt.statistics()]
        for b, blk in enumerate(ref.table):
            assert oracle.rel_fro(L[b, :blk.r, :blk.r], ref.L[b]) < TOL_STATS, (t, b)
            assert oracle.rel_fro(R[b, :blk.c, :blk.c], ref.R[b]) < TOL_STATS, (t, b)
            if t % wl.refresh_every == 0:
                for X, S, v in ((XL, L, blk.r), (XR, R, blk.c)):
                    er, gate, _ = root_checks(X[b, :v, :v], S[b, :v, :v], wl.root_p, wl.eps)
                    assert er < gate, (t, b, er, gate)
            Pg = dW[blk.param][blk.row0:blk.row0 + blk.r, blk.col0:blk.col0 + blk.c]
            ea, ga = apply_check(Pg, XL[b, :blk.r, :blk.r], ref.block_of(G, b), XR[b, :blk.c, :blk.c])
            assert ea < ga, (t, b, "apply", ea, ga)
    assert opt.status() & ~sb.DEVFLAG_STAGNATED == 0


def test_strided_block_views_match_the_full_step(sb):
    """Blocks are independent: the weights' blocks, given to the optimizer as
    strided views (each block a parameter of its own, via the strided step),
    end with exactly the weights of the optimizer over the full weights, and
    so does the sharded optimizer on a single rank (one process, which owns
    every block), in place and with its blocks packed into contiguous
    buffers.  One weight has rows of 70 floats (no vector loads)."""
    from shampoo_family_second_b200 import sharded
    shapes = ((96, 80), (40, 70))
    wl = workloads.workload("tiny", shapes=shapes, block=32, steps=3, iters=30, tol=1e-5, beta=0.9, eps=1e-4,
                            solver=workloads.SOLVER_NEWTON_CUBIC)
    cfg = sb.config_from_workload(wl)
    blocks = sharded.block_list(shapes, 32)
    full = sb.Shampoo(shapes, cfg)
    per_block = sb.Shampoo([(b[3], b[4]) for b in blocks], cfg)
    shard = sharded.ShardedShampoo(shapes, cfg)
    packed = sharded.ShardedShampoo(shapes, cfg, grads_reduced=False)  # blocks packed into contiguous buffers
    W1, W2, W3, W4 = ([torch.zeros(s, dtype=torch.float32, device="cuda") for s in shapes] for _ in range(4))
    stream = workloads.GradientStream(wl)

    def views(T):
        return [T[p][r0:r0 + r, c0:c0 + c] for p, r0, c0, r, c in blocks]

    for t in range(wl.steps):
        G = [torch.from_numpy(g).cuda() for g in stream.next()]
        full.step(W1, G)
        per_block.step(views(W2), views(G))
        shard.step(W3, G)
        packed.step(W4, G)
    torch.cuda.synchronize()
    for a, b, c, d in zip(W1, W2, W3, W4):
        assert torch.equal(a, b) and torch.equal(a, c) and torch.equal(a, d)
    assert full.status() & ~sb.DEVFLAG_STAGNATED == 0 and per_block.status() & ~sb.DEVFLAG_STAGNATED == 0
