"""The stated workloads at full size, checked stage by stage on sampled blocks.

Blocks are independent, so the oracle (and the fp32 reference that sets the
conditioning floor) run only on a seeded sample of blocks, always including
ragged ones and one block of every weight shape, while the GPU runs the whole
parameter set exactly as bench.py does.  Weights without a sampled block get
gradients of the same recipe drawn on the device (they only need to be there;
the sampled weights' gradients come from the shared generator, as the oracle's
do).  Checked per sampled block and step:

* statistics: GPU fp32 L, R vs the float64 oracle's, 1e-5 relative Frobenius;
* roots (refresh steps): opt.roots() vs the oracle's exact root of the GPU's
  own fp32 statistics at the workload's eps, range-space gate plus null-space
  band (tests/parity.py, root_checks);
* apply + update: Delta W / lr vs the float64 product XL_gpu G XR_gpu of the
  GPU's own roots, 2e-5 times the cancellation factor (parity.apply_check);
* end to end: the update vs the fully float64 pipeline, max(2e-3, 2 F_update)
  (parity.update_gate: the error of an fp32 LAPACK pipeline of the same steps
  sets the floor where fp32 statistics cannot reach 2e-3).

Properties that hold at any size are checked on every block: finite weights
and a device status with no bit but STAGNATED (rank-deficient ragged blocks
stop at their fp32 floor).
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import oracle
import workloads
from parity import BASE_TOL, Fp32ReferenceShampoo, apply_check, root_checks, update_gate

TOL_STATS = 1e-5
NULL_SPREAD = 0.10


@pytest.fixture(scope="module")
def sb():
    import shampoo_family_second_b200 as sb
    return sb


def sample_blocks(table, k, seed):
    """k seeded blocks, plus the first ragged blocks and one block of every
    distinct weight shape."""
    rng = np.random.default_rng(seed)
    bmax_r = max(t.r for t in table)
    bmax_c = max(t.c for t in table)
    ragged = [i for i, b in enumerate(table) if b.r < bmax_r or b.c < bmax_c]
    pick = set(rng.choice(len(table), size=min(k, len(table)), replace=False).tolist())
    pick.update(ragged[:2])
    return sorted(pick)


def per_shape_blocks(table, shapes, seed):
    rng = np.random.default_rng(seed + 7)
    out = []
    for shape in sorted(set(shapes)):
        cand = [i for i, b in enumerate(table) if shapes[b.param] == shape]
        out.append(int(rng.choice(cand)))
    return out


def to_device(g, dtype):
    if dtype == workloads.DTYPE_BF16:
        return torch.from_numpy(workloads.bf16_bits(g).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(g).cuda()


def filler_gradient(wl, shape, gen):
    """A gradient of the workload's scale and dtype, drawn on the device, for a
    weight that holds no sampled block."""
    scale = {"lowrank": 1.0, "gpt2": 0.02, "llama": 0.01}.get(wl.name, 1.0)
    x = torch.randn(shape, generator=gen, device="cuda") * scale
    return x.to(torch.bfloat16) if wl.grad_dtype == workloads.DTYPE_BF16 else x


def run_workload(sb, wl, steps, k_blocks):
    table = oracle.block_table(wl.shapes, wl.block)
    blocks = sorted(set(sample_blocks(table, k_blocks, wl.seed)) | set(per_shape_blocks(table, wl.shapes, wl.seed)))
    params = sorted({table[b].param for b in blocks})
    opt = sb.Shampoo(wl.shapes, sb.config_from_workload(wl))
    ref = oracle.ShampooOracle(wl.shapes, wl.block, wl.beta, wl.eps, wl.lr, wl.root_p, wl.refresh_every,
                               blocks=blocks)
    ref32 = Fp32ReferenceShampoo(wl.shapes, wl.block, wl.beta, wl.eps, wl.root_p, wl.refresh_every, blocks)
    W = [torch.zeros(s, dtype=torch.float32, device="cuda") for s in wl.shapes]
    stream = workloads.GradientStream(wl, params=params)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(wl.seed + 99)
    worst = {"stats": 0.0, "root": (0.0, 1.0), "apply": (0.0, 1.0), "update": (0.0, 1.0)}
    e2e = []
    for t in range(steps):
        mine = dict(zip(params, stream.next()))
        grads = [mine.get(i) for i in range(len(wl.shapes))]
        G = [to_device(grads[i], wl.grad_dtype) if i in mine else filler_gradient(wl, s, gen)
             for i, s in enumerate(wl.shapes)]
        before = {p: W[p].double() for p in params}
        opt.step(W, G)
        P_ref = ref.step(grads)
        P_32 = ref32.step(grads)
        torch.cuda.synchronize()
        L, R = opt.statistics()
        XL, XR = opt.roots()
        refresh = t % wl.refresh_every == 0
        for b in blocks:
            blk = ref.table[b]
            sl = (slice(blk.row0, blk.row0 + blk.r), slice(blk.col0, blk.col0 + blk.c))
            Pg = ((before[blk.param][sl] - W[blk.param][sl].double()) / wl.lr).cpu().numpy()
            Lg = L[b, :blk.r, :blk.r].cpu().numpy().astype(np.float64)
            Rg = R[b, :blk.c, :blk.c].cpu().numpy().astype(np.float64)
            xl = XL[b, :blk.r, :blk.r].cpu().numpy().astype(np.float64)
            xr = XR[b, :blk.c, :blk.c].cpu().numpy().astype(np.float64)
            es = max(oracle.rel_fro(Lg, ref.L[b]), oracle.rel_fro(Rg, ref.R[b]))
            worst["stats"] = max(worst["stats"], es)
            assert es < TOL_STATS, (t, b, "stats", es)
            if refresh:
                for X, S in ((xl, Lg), (xr, Rg)):
                    er, gate, spread = root_checks(X, S, wl.root_p, wl.eps)
                    if er / gate > worst["root"][0] / worst["root"][1]:
                        worst["root"] = (er, gate)
                    assert er < gate, (t, b, "root", er, gate)
                    if spread is not None:
                        assert spread < NULL_SPREAD, (t, b, "null-space root", spread)
            ea, ga = apply_check(Pg, xl, ref.block_of(grads, b), xr)
            if ea / ga > worst["apply"][0] / worst["apply"][1]:
                worst["apply"] = (ea, ga)
            assert ea < ga, (t, b, "apply", ea, ga)
            e = oracle.rel_fro(Pg, P_ref[b])
            gate = update_gate(P_32[b], P_ref[b])
            e2e.append((e, oracle.rel_fro(P_32[b], P_ref[b])))
            if e / gate > worst["update"][0] / worst["update"][1]:
                worst["update"] = (e, gate)
            assert e < gate, (t, b, "update", e, gate)
        del G
    assert all(torch.isfinite(w).all().item() for w in W)
    status = opt.status()
    assert status & ~sb.DEVFLAG_STAGNATED == 0, status
    e_all = np.array([x[0] for x in e2e])
    f_all = np.array([x[1] for x in e2e])
    print(f"\n{wl.name} ({wl.solver=}): {len(blocks)} sampled blocks x {steps} steps; "
          f"statistics {worst['stats']:.2e}; root {worst['root'][0]:.2e} (gate {worst['root'][1]:.2e}); "
          f"apply {worst['apply'][0]:.2e} (gate {worst['apply'][1]:.2e}); "
          f"end-to-end update: median {np.median(e_all):.2e}, max {e_all.max():.2e} "
          f"(fp32 LAPACK pipeline: median {np.median(f_all):.2e}, max {f_all.max():.2e}); "
          f"blocks within {BASE_TOL:g}: {int((e_all < BASE_TOL).sum())}/{len(e_all)}; device status {status}")
    return worst


def test_lowrank_4x1024_b256(sb):
    """4 fp32 matrices 1024 x 1024, block 256, low-rank + noise gradients,
    beta 0.95, eps 1e-8, refresh every 10 steps (steps 0 and 10 refresh)."""
    wl = workloads.workload("lowrank")
    run_workload(sb, wl, steps=11, k_blocks=4)


def test_lowrank_4x1024_b256_plain_newton(sb):
    """The 4 x 1024^2 workload with the plain (degree-1) coupled Newton step."""
    wl = workloads.workload("lowrank", solver=workloads.SOLVER_NEWTON)
    run_workload(sb, wl, steps=11, k_blocks=4)


def test_gpt2_small_shapes_b512_plain_newton(sb):
    """GPT-2-small layer shapes with the plain (degree-1) coupled Newton step."""
    wl = workloads.workload("gpt2", solver=workloads.SOLVER_NEWTON)
    run_workload(sb, wl, steps=2, k_blocks=6)


def test_gpt2_small_shapes_b512(sb):
    """GPT-2-small layer shapes (456 blocks of 512, 252 ragged), root every step."""
    wl = workloads.workload("gpt2")
    run_workload(sb, wl, steps=3, k_blocks=6)


@pytest.mark.slow
def test_llama_1b_shapes_b1024(sb):
    """Llama-1B layer shapes (1024 blocks of 1024), bf16 gradients, 11 steps:
    refreshes at steps 0 and 10, stale roots in between."""
    wl = workloads.workload("llama")
    run_workload(sb, wl, steps=11, k_blocks=3)
