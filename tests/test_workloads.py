"""Seeded input generators: determinism, shapes, spectra, bf16 rounding."""
import numpy as np
import pytest

import workloads


def test_gradient_stream_deterministic_and_subsettable():
    wl = workloads.workload("gpt2")
    a = workloads.GradientStream(wl).next()
    b = workloads.GradientStream(wl).next()
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)
    sub = workloads.GradientStream(wl, params=[3, 7]).next()
    np.testing.assert_array_equal(sub[0], a[3])
    np.testing.assert_array_equal(sub[1], a[7])
    assert [g.shape for g in a] == list(wl.shapes)
    assert all(g.dtype == np.float32 for g in a)


def test_lowrank_stream_statistics():
    wl = workloads.workload("lowrank")
    g = workloads.GradientStream(wl, params=[0]).next()[0]
    assert g.shape == (1024, 1024)
    assert 0.8 < g.var() < 1.2             # "scale 1"
    s = np.linalg.svd(g[:256, :256], compute_uv=False)
    assert s[15] / s[16] > 3               # rank-16 signal above the 0.01 noise edge (~0.32)


def test_gpt2_column_scales():
    wl = workloads.workload("gpt2")
    st = workloads.GradientStream(wl, params=[1])
    col = st.fixed[1]
    assert col.min() >= 1e-2 and col.max() <= 1.0
    g = st.next()[0]
    ratio = g.std(axis=0) / (0.02 * col)
    assert 0.85 < np.median(ratio) < 1.15


def test_bf16_rounding():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 2 ** -9, 1.0 + 3 * 2 ** -9, -3.14159, 0.0], dtype=np.float32)
    r = workloads.round_to_bf16(x)
    assert r[0] == 1.0
    assert r[1] == 1.0 + 2 ** -7 or r[1] == 1.0     # exact tie -> even
    assert r[2] == 1.0                               # below half ulp
    assert r[3] == 1.0 + 2 ** -7                     # above half ulp
    bits = r.view(np.uint32)
    assert np.all(bits & 0xFFFF == 0)
    np.testing.assert_array_equal(workloads.bf16_bits(r), (bits >> 16).astype(np.uint16))
    wl = workloads.workload("llama")
    g = workloads.GradientStream(wl, params=[0]).next()[0]
    assert np.all(g.view(np.uint32) & 0xFFFF == 0)


@pytest.mark.parametrize("kappa", workloads.SWEEP_KAPPAS)
def test_spd_batch_condition_number(kappa):
    A, Q, lam = workloads.spd_batch(2, 24, kappa, seed=3, return_parts=True)
    for b in range(2):
        assert lam[b].max() == 1.0
        assert lam[b].min() == pytest.approx(1.0 / kappa, rel=1e-15)
        np.testing.assert_allclose(Q[b].T @ Q[b], np.eye(24), atol=1e-12)
        np.testing.assert_allclose(A[b], A[b].T, atol=0)
    if kappa <= 1e4:
        ev = np.linalg.eigvalsh(A[0])
        assert ev.max() / ev.min() == pytest.approx(kappa, rel=1e-6)
