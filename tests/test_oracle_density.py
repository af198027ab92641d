"""Pins of the oracle's Soft-Riesz density (DensityKV §3 "Soft-Riesz Density", App. B.1).

Each check uses something other than the oracle's own formula: hand-computed
constants, pure-Python loops, the norm expansion of the distance, or exact
algebraic consequences (duplicates, scaling, permutation)."""
import math

import numpy as np
import pytest

from oracle.density import density, soft_riesz, sq_dists


def test_two_point_closed_form_constants():
    # a=(1,2), b=(4,6): ||a-b||^2 = 9+16 = 25; h=2 -> x = 12.5; eps=0.5 -> 13.
    a = np.array([[1.0, 2.0]])
    b = np.array([[4.0, 6.0]])
    assert density(a, b, h=2.0, eps=0.5, s=2.0)[0] == pytest.approx(1.0 / 13.0, rel=1e-15)
    assert density(a, b, h=2.0, eps=0.5, s=4.0)[0] == pytest.approx(1.0 / 169.0, rel=1e-15)
    assert density(a, b, h=2.0, eps=0.5, s=1.0)[0] == pytest.approx(13.0 ** -0.5, rel=1e-15)
    # a decay exponent of 0 counts neighbours
    assert density(a, np.vstack([b, b, a + 7]), h=2.0, eps=0.5, s=0.0)[0] == pytest.approx(3.0)


def test_sq_dists_matches_python_loop():
    rng = np.random.default_rng(0)
    A = rng.standard_normal((5, 7))
    B = rng.standard_normal((9, 7))
    D = sq_dists(A, B)
    for i in range(5):
        for j in range(9):
            acc = 0.0
            for k in range(7):
                acc += (A[i, k] - B[j, k]) ** 2
            assert D[i, j] == pytest.approx(acc, rel=1e-13, abs=1e-13)


def test_density_matches_norm_expansion():
    # independent route: ||a||^2 + ||b||^2 - 2 a.b through a matrix product
    rng = np.random.default_rng(1)
    A = rng.standard_normal((40, 64))
    B = rng.standard_normal((70, 64))
    G = A @ B.T
    x = ((A * A).sum(1)[:, None] + (B * B).sum(1)[None, :] - 2 * G) / 64.0
    ref = (1.0 / (x + 1e-3)).sum(1)
    np.testing.assert_allclose(density(A, B, h=64.0, eps=1e-3, s=2.0), ref, rtol=1e-11)


def test_self_exclusion_by_id_matches_pair_loop():
    rng = np.random.default_rng(2)
    K = rng.standard_normal((6, 3))
    ids = np.array([5, 9, 2, 7, 11, 3])
    rho = density(K, K, h=3.0, eps=1e-3, s=2.0, row_ids=ids, col_ids=ids)
    for i in range(6):
        acc = 0.0
        for j in range(6):
            if i == j:
                continue
            x = sum((K[i, k] - K[j, k]) ** 2 for k in range(3)) / 3.0
            acc += 1.0 / (x + 1e-3)
        assert rho[i] == pytest.approx(acc, rel=1e-12)


def test_exclusion_follows_ids_not_positions():
    # rows that are a reordered subset of the columns exclude the column with
    # their own id; rows whose ids the columns do not hold exclude nothing
    rng = np.random.default_rng(5)
    K = rng.standard_normal((5, 4))
    ids = np.array([10, 11, 12, 13, 14])
    rows, rid = K[[3, 0]], ids[[3, 0]]
    got = density(rows, K, h=4.0, eps=0.5, s=2.0, row_ids=rid, col_ids=ids)
    for r in range(2):
        acc = 0.0
        for j in range(5):
            if ids[j] == rid[r]:
                continue
            acc += 1.0 / (sum((rows[r, k] - K[j, k]) ** 2 for k in range(4)) / 4.0 + 0.5)
        assert got[r] == pytest.approx(acc, rel=1e-12)
    fresh = density(K, K, h=4.0, eps=0.5, s=2.0, row_ids=ids + 100, col_ids=ids)
    np.testing.assert_allclose(fresh, density(K, K, h=4.0, eps=0.5, s=2.0), rtol=1e-15)


def test_duplicate_raises_density_by_inverse_eps_power():
    # an exact duplicate with a new id adds eps^(-s/2) to its twin (1000 at eps=1e-3, s=2)
    rng = np.random.default_rng(3)
    K = rng.standard_normal((8, 16))
    ids = np.arange(8)
    before = density(K, K, h=16.0, eps=1e-3, s=2.0, row_ids=ids, col_ids=ids)
    K2 = np.vstack([K, K[3:4]])
    ids2 = np.append(ids, 100)
    after = density(K2, K2, h=16.0, eps=1e-3, s=2.0, row_ids=ids2, col_ids=ids2)
    assert after[3] - before[3] == pytest.approx(1000.0, rel=1e-9)
    assert after[8] == pytest.approx(after[3], rel=1e-12)
    for s in (1.0, 3.0):
        b = density(K, K, h=16.0, eps=1e-3, s=s, row_ids=ids, col_ids=ids)
        a = density(K2, K2, h=16.0, eps=1e-3, s=s, row_ids=ids2, col_ids=ids2)
        assert a[3] - b[3] == pytest.approx(1e-3 ** (-s / 2), rel=1e-9)


def test_permutation_and_scale_invariance():
    rng = np.random.default_rng(4)
    A = rng.standard_normal((10, 8))
    B = rng.standard_normal((20, 8))
    r = density(A, B, h=8.0, eps=0.1, s=2.0)
    perm = rng.permutation(20)
    np.testing.assert_allclose(density(A, B[perm], h=8.0, eps=0.1, s=2.0), r, rtol=1e-13)
    # scaling keys by c and h by c^2 leaves every x unchanged
    np.testing.assert_allclose(density(3 * A, 3 * B, h=72.0, eps=0.1, s=2.0), r, rtol=1e-12)


def test_phi_monotone_and_bounded():
    x = np.linspace(0, 50, 101)
    f = soft_riesz(x, 1e-3, 2.0)
    assert np.all(np.diff(f) < 0)
    assert f[0] == pytest.approx(1000.0)
    assert math.isclose(soft_riesz(0.0, 1.0, 2.0), 1.0)
