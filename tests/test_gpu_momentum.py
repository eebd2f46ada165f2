"""Momentum ahead of the preconditioner, on the GPU vs the float64 oracle.

Podcast transcript "Preconditioned optimization without the full matrix
cost", cue 28: momentum (0.9) is applied before the preconditioner.  Reading:
per block M <- alpha M + G from M = 0, the statistics keep the raw G, and the
update is W <- W - lr XL M XR (the oracle's ``momentum`` option, pinned in
tests/test_oracle_pins.py).  The GPU folds the momentum update into the
stacking pass and reads M as the right operand of the first apply product.

Checked per step and block: statistics (1e-5), the momentum stack against the
oracle's M (fp32 accumulation over a few steps: 1e-6), roots on refresh steps
(root_checks on the GPU's own statistics), the apply stage against the
float64 product XL_gpu M_gpu XR_gpu (parity.apply_check), and the update end
to end against the float64 pipeline (max(2e-3, 2 F_update)).
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import oracle
import workloads
from parity import Fp32ReferenceShampoo, apply_check, root_checks, update_gate

ALPHA = 0.9
TOL_STATS = 1e-5
TOL_MOM = 1e-6
NULL_SPREAD = 0.10


@pytest.fixture(scope="module")
def sb():
    import shampoo_family_second_b200 as sb
    return sb


def dev(g, dtype):
    if dtype == workloads.DTYPE_BF16:
        return torch.from_numpy(workloads.bf16_bits(g).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(g).cuda()


CASES = {
    "tiny": dict(shapes=((64, 32),), block=32, steps=6, refresh_every=2),
    "ragged": dict(shapes=((64, 45), (20, 96)), block=32, steps=5, refresh_every=2),
    "bf16": dict(shapes=((64, 96),), block=32, steps=4, refresh_every=1, grad_dtype=workloads.DTYPE_BF16),
    "b256": dict(shapes=((512, 700),), block=256, steps=4, refresh_every=3),
}


@pytest.mark.parametrize("case", sorted(CASES))
def test_momentum_step_parity(sb, case):
    wl = workloads.workload("tiny", iters=40, tol=1e-5, beta=0.95, eps=1e-4, momentum=ALPHA,
                            solver=workloads.SOLVER_NEWTON_CUBIC, **CASES[case])
    opt = sb.Shampoo(wl.shapes, sb.config_from_workload(wl))
    ref = oracle.ShampooOracle(wl.shapes, wl.block, wl.beta, wl.eps, wl.lr, wl.root_p, wl.refresh_every,
                               momentum=ALPHA)
    ref32 = Fp32ReferenceShampoo(wl.shapes, wl.block, wl.beta, wl.eps, wl.root_p, wl.refresh_every, ref.active,
                                 momentum=ALPHA)
    W = [torch.zeros(s, dtype=torch.float32, device="cuda") for s in wl.shapes]
    stream = workloads.GradientStream(wl)
    worst = {"apply": 0.0, "update": 0.0, "mom": 0.0}
    for t in range(wl.steps):
        grads = stream.next()
        before = [w.double() for w in W]
        opt.step(W, [dev(g, wl.grad_dtype) for g in grads])
        P_ref = ref.step(grads)
        P_32 = ref32.step(grads)
        torch.cuda.synchronize()
        dW = [((a - w.double()) / wl.lr).cpu().numpy() for a, w in zip(before, W)]
        L, R = opt.statistics()
        XL, XR = opt.roots()
        M = opt.momentum()
        L, R, XL, XR, M = (x.cpu().numpy().astype(np.float64) for x in (L, R, XL, XR, M))
        for b in ref.active:
            blk = ref.table[b]
            r, c = blk.r, blk.c
            assert max(oracle.rel_fro(L[b, :r, :r], ref.L[b]), oracle.rel_fro(R[b, :c, :c], ref.R[b])) < TOL_STATS
            em = oracle.rel_fro(M[b, :r, :c], ref.M[b])
            worst["mom"] = max(worst["mom"], em)
            assert em < TOL_MOM, (t, b, "momentum", em)
            assert not np.any(M[b, r:, :]) and not np.any(M[b, :, c:]), "momentum padding must stay zero"
            if t % wl.refresh_every == 0:
                for X, S, v in ((XL, L, r), (XR, R, c)):
                    er, gate, spread = root_checks(X[b, :v, :v], S[b, :v, :v], wl.root_p, wl.eps)
                    assert er < gate, (t, b, "root", er, gate)
                    if spread is not None:
                        assert spread < NULL_SPREAD
            Pg = dW[blk.param][blk.row0:blk.row0 + r, blk.col0:blk.col0 + c]
            ea, ga = apply_check(Pg, XL[b, :r, :r], M[b, :r, :c], XR[b, :c, :c])
            worst["apply"] = max(worst["apply"], ea)
            assert ea < ga, (t, b, "apply", ea, ga)
            e = oracle.rel_fro(Pg, P_ref[b])
            worst["update"] = max(worst["update"], e)
            assert e < update_gate(P_32[b], P_ref[b]), (t, b, "update", e)
    assert opt.status() & ~sb.DEVFLAG_STAGNATED == 0
    print(f"\nmomentum {case}: worst update {worst['update']:.2e}, apply {worst['apply']:.2e}, "
          f"momentum {worst['mom']:.2e}")


def test_momentum_off_has_no_stack(sb):
    wl = workloads.workload("tiny")
    opt = sb.Shampoo(wl.shapes, sb.config_from_workload(wl))
    assert opt.momentum() is None
