"""Pins of the oracle's attention and of the generator's RoPE geometry.

DensityKV Fig. 2 / §5 (native attention over retained states); App. A.1 (post-RoPE
key distance equals the worst-case normalised logit discrepancy; RoPE rotations
are orthogonal)."""
import numpy as np
import pytest

import kvgen
from oracle.attention import attention


def test_single_key_returns_its_value():
    rng = np.random.default_rng(0)
    Q = rng.standard_normal((5, 16))
    K = rng.standard_normal((1, 16))
    V = rng.standard_normal((1, 16))
    O, lse = attention(Q, K, V)
    np.testing.assert_allclose(O, np.repeat(V, 5, 0), rtol=1e-14)
    np.testing.assert_allclose(lse, (Q @ K[0]) / 4.0, rtol=1e-13)


def test_equal_keys_average_values():
    rng = np.random.default_rng(1)
    Q = rng.standard_normal((3, 8))
    K = np.repeat(rng.standard_normal((1, 8)), 6, 0)
    V = rng.standard_normal((6, 8))
    O, lse = attention(Q, K, V)
    np.testing.assert_allclose(O, np.repeat(V.mean(0, keepdims=True), 3, 0), rtol=1e-13)
    np.testing.assert_allclose(lse, Q @ K[0] / np.sqrt(8) + np.log(6), rtol=1e-13)


def test_two_keys_logistic_weights():
    q = np.array([[1.0, 2.0, 0.0, -1.0]])
    K = np.array([[0.5, 0.0, 1.0, 0.0], [0.0, 1.0, 0.0, 2.0]])
    V = np.array([[1.0, 0.0, 0.0, 0.0], [0.0, 1.0, 0.0, 0.0]])
    # logits: (0.5)/2 = 0.25 and (2 - 2)/2 = 0 -> weight of key 0 = 1/(1+e^-0.25)
    w0 = 1.0 / (1.0 + np.exp(-0.25))
    O, lse = attention(q, K, V)
    assert O[0, 0] == pytest.approx(w0, rel=1e-14)
    assert O[0, 1] == pytest.approx(1 - w0, rel=1e-14)
    assert lse[0] == pytest.approx(np.log(np.exp(0.25) + 1.0), rel=1e-14)


def test_key_permutation_and_logit_shift():
    rng = np.random.default_rng(2)
    Q = rng.standard_normal((4, 32))
    K = rng.standard_normal((50, 32))
    V = rng.standard_normal((50, 32))
    O, lse = attention(Q, K, V)
    p = rng.permutation(50)
    O2, lse2 = attention(Q, K[p], V[p])
    np.testing.assert_allclose(O2, O, rtol=1e-12)
    np.testing.assert_allclose(lse2, lse, rtol=1e-12)
    # a huge common logit offset (q along an extra axis all keys share) changes nothing but lse
    Qx = np.hstack([Q, np.full((4, 1), 800.0)])
    Kx = np.hstack([K, np.ones((50, 1))])
    Ox, lsex = attention(Qx, Kx, V, scale=1 / np.sqrt(32))
    np.testing.assert_allclose(Ox, O, rtol=1e-10)
    np.testing.assert_allclose(lsex - 800 / np.sqrt(32), lse, rtol=1e-10)


def test_rope_is_orthogonal_and_distance_equals_worst_logit_gap():
    d = 128
    rng = np.random.default_rng(3)
    x = rng.standard_normal((2, d)).astype(np.float32)
    ang = kvgen.rope_angles(d, np.array([5.0, 5.0]), np.array([3.0, 3.0]), np.array([7.0, 7.0]))
    y = kvgen.apply_rope(x, ang)
    # rotation by the same position preserves norms and distances
    np.testing.assert_allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-5)
    assert np.linalg.norm(y[0] - y[1]) == pytest.approx(np.linalg.norm(x[0] - x[1]), rel=1e-5)
    # App. A.1: ||k1-k2|| = max_q |q.(k1-k2)|/||q||, attained at q parallel to k1-k2
    dk = (y[0] - y[1]).astype(np.float64)
    assert abs(dk @ dk) / np.linalg.norm(dk) == pytest.approx(np.linalg.norm(dk), rel=1e-12)
    qs = rng.standard_normal((1000, d))
    gaps = np.abs(qs @ dk) / np.linalg.norm(qs, axis=1)
    assert gaps.max() <= np.linalg.norm(dk) * (1 + 1e-12)


def test_rope_pair_split():
    assert kvgen.rope_pairs(128) == (22, 21, 21)
    assert kvgen.rope_pairs(64) == (12, 10, 10)
