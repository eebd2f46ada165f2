"""The root gate's conditioning floor behaves as the arithmetic says: small
for well-conditioned inputs (gate = 2e-3), growing with kappa, and the fp32
LAPACK reference really runs in single precision."""
import numpy as np

import workloads
from parity import lapack_fp32_floor, perturbation_floor, root_gate


def test_floor_small_when_well_conditioned():
    A = workloads.spd_batch(1, 64, 1e2, seed=1)[0].astype(np.float32).astype(np.float64)
    assert perturbation_floor(A, 4, 0.0) < 1e-5
    assert lapack_fp32_floor(A, 4, 0.0) < 1e-4
    assert root_gate(A, 4, 0.0) == 2e-3


def test_floor_grows_with_condition_number():
    f = []
    for kappa in (1e2, 1e4, 1e6):
        A = workloads.spd_batch(1, 64, kappa, seed=2)[0].astype(np.float32).astype(np.float64)
        f.append(perturbation_floor(A, 2, 0.0))
    assert f[0] < f[1] < f[2]
    assert 30 < f[1] / f[0] < 300 and 30 < f[2] / f[1] < 300   # ~ linear in kappa


def test_lapack_reference_is_single_precision():
    # kappa = 1e6 in fp32: a double-precision solver would be ~1e-7 accurate here.
    A = workloads.spd_batch(1, 128, 1e6, seed=3)[0].astype(np.float32).astype(np.float64)
    assert lapack_fp32_floor(A, 2, 0.0) > 1e-4
