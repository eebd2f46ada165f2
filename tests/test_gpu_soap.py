"""SOAP on the GPU vs the float64 oracle (oracle/soap.py).

pith.science SOAP record: Adam run in the eigenbasis of Shampoo's
preconditioner, the basis recomputed every refresh_every steps.  Checked per
step and block:

* statistics against the oracle's (1e-5) and the first moment m (1e-6);
* on refresh steps, the basis: orthogonal and diagonalising the GPU's own
  statistics (eigenvectors are unique only up to sign and order, so these are
  the checks of what is unique), 2e-5;
* the step itself: Delta W / lr against the float64 SOAP direction computed
  from the GPU's own basis and moments as they were before the step, 1e-4;
* end to end (square blocks, whose statistics have no null space): the
  update against the fully float64 pipeline within max(2e-3, 2 F), F the
  error of an fp32 pipeline with single-precision LAPACK eigenbases (the
  eigenvectors of nearly equal eigenvalues turn with any fp32 rounding of the
  statistics, and Adam's elementwise step follows the basis).

Ragged blocks (whose statistics have null spaces at the first refresh, where
the basis is arbitrary) get every check but the end-to-end one.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import oracle
from oracle.soap import SoapOracle
import workloads
from parity import BASE_TOL, Fp32ReferenceSoap

HP = dict(beta=0.95, lr=1e-2, refresh_every=2, beta1=0.9, beta2=0.99, eps=1e-6)
TOL_STATS, TOL_M, TOL_BASIS, TOL_STEP = 1e-5, 1e-6, 2e-5, 1e-4


@pytest.fixture(scope="module")
def sb():
    import shampoo_family_second_b200 as sb
    return sb


def soap_direction(QL, QR, m_before, v_before, G, t, hp):
    Gr = QL.T @ G @ QR
    m = hp["beta1"] * m_before + (1 - hp["beta1"]) * G
    v = hp["beta2"] * v_before + (1 - hp["beta2"]) * Gr * Gr
    Nr = (QL.T @ m @ QR / (1 - hp["beta1"] ** t)) / (np.sqrt(v / (1 - hp["beta2"] ** t)) + hp["eps"])
    return QL @ Nr @ QR.T


@pytest.mark.parametrize("case", ["square", "ragged", "bf16"])
def test_soap_step_parity(sb, case):
    B = 64
    shapes = {"square": ((128, 128), (64, 64)), "ragged": ((100, 70), (40, 96)), "bf16": ((128, 64),)}[case]
    dtype = workloads.DTYPE_BF16 if case == "bf16" else workloads.DTYPE_F32
    steps = 5
    cfg = sb.make_config(B, HP["beta"], 0.0, HP["lr"], refresh_every=HP["refresh_every"], grad_dtype=dtype)
    sc = sb.make_soap_config(HP["beta1"], HP["beta2"], HP["eps"], jacobi_sweeps=20, refine_iters=1)
    opt = sb.Soap(shapes, cfg, sc)
    ref = SoapOracle(shapes, B, HP["beta"], HP["lr"], HP["refresh_every"], HP["beta1"], HP["beta2"], HP["eps"])
    ref32 = Fp32ReferenceSoap(shapes, B, HP["beta"], HP["refresh_every"], HP["beta1"], HP["beta2"], HP["eps"],
                              ref.active)
    W = [torch.zeros(s, dtype=torch.float32, device="cuda") for s in shapes]
    rng = np.random.default_rng(90)
    worst = {"step": 0.0, "e2e": 0.0}
    for t in range(steps):
        grads = [rng.standard_normal(s).astype(np.float32) for s in shapes]
        if dtype == workloads.DTYPE_BF16:
            grads = [workloads.round_to_bf16(g) for g in grads]
            G = [torch.from_numpy(workloads.bf16_bits(g).view(np.int16)).view(torch.bfloat16).cuda() for g in grads]
        else:
            G = [torch.from_numpy(g).cuda() for g in grads]
        st0 = {k: v.double().cpu().numpy() for k, v in opt.views().items() if k != "step"}
        before = [w.double() for w in W]
        opt.step(W, G)
        N_ref = ref.step(grads)
        N_32 = ref32.step(grads)
        torch.cuda.synchronize()
        st1 = {k: v.double().cpu().numpy() for k, v in opt.views().items() if k != "step"}
        for b in ref.active:
            blk = ref.table[b]
            r, c = blk.r, blk.c
            g = np.asarray(grads[blk.param][blk.row0:blk.row0 + r, blk.col0:blk.col0 + c], np.float64)
            assert oracle.rel_fro(st1["L"][b, :r, :r], ref.L[b]) < TOL_STATS
            assert oracle.rel_fro(st1["R"][b, :c, :c], ref.R[b]) < TOL_STATS
            assert oracle.rel_fro(st1["m"][b, :r, :c], ref.m[b]) < TOL_M
            Ng = ((before[blk.param] - W[blk.param].double()) / HP["lr"]).cpu().numpy()[
                blk.row0:blk.row0 + r, blk.col0:blk.col0 + c]
            N64 = soap_direction(st0["QL"][b, :r, :r], st0["QR"][b, :c, :c], st0["m"][b, :r, :c],
                                 st0["v"][b, :r, :c], g.astype(np.float64), t + 1, HP)
            es = oracle.rel_fro(Ng, N64)
            worst["step"] = max(worst["step"], es)
            assert es < TOL_STEP, (t, b, "step", es)
            if t % HP["refresh_every"] == 0:
                for Q, S, n in ((st1["QL"][b], st1["L"][b], r), (st1["QR"][b], st1["R"][b], c)):
                    Qv, Sv = Q[:n, :n], S[:n, :n]
                    orth = np.linalg.norm(Qv.T @ Qv - np.eye(n)) / np.sqrt(n)
                    D = Qv.T @ Sv @ Qv
                    off = np.linalg.norm(D - np.diag(np.diag(D))) / np.linalg.norm(Sv)
                    assert orth < TOL_BASIS and off < TOL_BASIS, (t, b, orth, off)
            if case != "ragged":
                e = oracle.rel_fro(Ng, N_ref[b])
                gate = max(BASE_TOL, 2.0 * oracle.rel_fro(N_32[b], N_ref[b]))
                worst["e2e"] = max(worst["e2e"], e)
                assert e < gate, (t, b, "end to end", e, gate)
    assert opt.status() == 0
    print(f"\nsoap {case}: worst step {worst['step']:.2e}, end to end {worst['e2e']:.2e}")
