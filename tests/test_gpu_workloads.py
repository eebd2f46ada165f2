"""The stated workloads at full size, checked on sampled blocks.

Blocks are independent, so the oracle (and the fp32 reference that sets the
conditioning floor) run only on a seeded sample of blocks, always including
ragged ones, while the GPU runs the whole parameter set exactly as bench.py
does.  Checked per sampled block and step: statistics (1e-5 relative
Frobenius) and the update (max(2e-3, 2 F_update), see tests/parity.py).
Properties that hold at any size are checked on every block: finite weights
and a clean device status.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import oracle
import workloads
from parity import Fp32ReferenceShampoo, update_gate

TOL_STATS = 1e-5


@pytest.fixture(scope="module")
def sb():
    import shampoo_family_second_b200 as sb
    return sb


def sample_blocks(table, k, seed):
    rng = np.random.default_rng(seed)
    ragged = [i for i, b in enumerate(table) if b.r < max(t.r for t in table) or b.c < max(t.c for t in table)]
    pick = set(rng.choice(len(table), size=min(k, len(table)), replace=False).tolist())
    pick.update(ragged[:2])
    return sorted(pick)


def to_device(g, dtype):
    if dtype == workloads.DTYPE_BF16:
        return torch.from_numpy(workloads.bf16_bits(g).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(g).cuda()


def run_workload(sb, wl, steps, k_blocks):
    opt = sb.Shampoo(wl.shapes, sb.config_from_workload(wl))
    ref = oracle.ShampooOracle(wl.shapes, wl.block, wl.beta, wl.eps, wl.lr, wl.root_p, wl.refresh_every)
    blocks = sample_blocks(ref.table, k_blocks, wl.seed)
    ref = oracle.ShampooOracle(wl.shapes, wl.block, wl.beta, wl.eps, wl.lr, wl.root_p, wl.refresh_every,
                               blocks=blocks)
    ref32 = Fp32ReferenceShampoo(wl.shapes, wl.block, wl.beta, wl.eps, wl.root_p, wl.refresh_every, blocks)
    W = [torch.zeros(s, dtype=torch.float32, device="cuda") for s in wl.shapes]
    stream = workloads.GradientStream(wl)
    report = []
    for t in range(steps):
        grads = stream.next()
        G = [to_device(g, wl.grad_dtype) for g in grads]
        before = {blk.param: W[blk.param].clone() for blk in (ref.table[b] for b in blocks)}
        opt.step(W, G)
        P_ref = ref.step(grads)
        P_32 = ref32.step(grads)
        torch.cuda.synchronize()
        L, R = opt.statistics()
        for b in blocks:
            blk = ref.table[b]
            sl = (slice(blk.row0, blk.row0 + blk.r), slice(blk.col0, blk.col0 + blk.c))
            Pg = ((before[blk.param][sl] - W[blk.param][sl]) / wl.lr).cpu().numpy().astype(np.float64)
            e = oracle.rel_fro(Pg, P_ref[b])
            gate = update_gate(P_32[b], P_ref[b])
            Lg = L[b, :blk.r, :blk.r].cpu().numpy().astype(np.float64)
            Rg = R[b, :blk.c, :blk.c].cpu().numpy().astype(np.float64)
            es = max(oracle.rel_fro(Lg, ref.L[b]), oracle.rel_fro(Rg, ref.R[b]))
            report.append((t, b, e, gate, es))
            assert es < TOL_STATS, (t, b, "stats", es)
            assert e < gate, (t, b, "update", e, gate)
        del G
    assert all(torch.isfinite(w).all().item() for w in W)
    status = opt.status()
    # rank-deficient ragged blocks stall at the fp32 floor (STAGNATED)
    assert status & ~(sb.DEVFLAG_NOT_CONVERGED | sb.DEVFLAG_STAGNATED) == 0, status
    print(f"\n{wl.name}: {len(blocks)} sampled blocks x {steps} steps; worst update error "
          f"{max(r[2] for r in report):.2e} (tightest gate {min(r[3] for r in report):.2e}), "
          f"worst statistics error {max(r[4] for r in report):.2e}, device status {status}")
    return report


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
    run_workload(sb, wl, steps=2, k_blocks=6)


@pytest.mark.slow
def test_llama_1b_shapes_b1024(sb):
    """Llama-1B layer shapes (1024 blocks of 1024), bf16 gradients."""
    wl = workloads.workload("llama")
    run_workload(sb, wl, steps=1, k_blocks=3)
