"""Pins for the oracle's rotary position embedding (no GPU).

* brute force: each lane pair as a complex number a + ib multiplied by
  e^{i theta} with Python's complex arithmetic (an independent formulation);
* closed forms: identity tables leave x unchanged; a quarter turn maps
  (a, b) to (-b, a); every pair keeps its Euclidean norm; two rotations compose
  into one by the sum of the angles;
* the property RoPE exists for: with angles s * w_j, the dot product of a rotated
  query at position s1 and a rotated key at s2 depends only on s1 - s2;
* the two pairings are the same rotation up to a fixed permutation of lanes;
* a planted mistake (pairing the wrong lanes) is caught by the brute force.
"""

import cmath
import math

import numpy as np
import pytest

import oracle
from oracle import rope as orope


def _tables_from_angles(theta):
    return np.cos(theta), np.sin(theta)


def _brute(x, theta, mode):
    S, D = x.shape[-2], x.shape[-1]
    out = np.array(x, dtype=np.float64, copy=True)
    flat, fo = x.reshape(-1, S, D), out.reshape(-1, S, D)
    for r in range(flat.shape[0]):
        for s in range(S):
            for j in range(D // 2):
                ia, ib = (j, j + D // 2) if mode == "half" else (2 * j, 2 * j + 1)
                z = complex(float(flat[r, s, ia]), float(flat[r, s, ib])) * cmath.exp(1j * float(theta[s, j]))
                fo[r, s, ia], fo[r, s, ib] = z.real, z.imag
    return out


@pytest.mark.parametrize("mode", ["half", "interleaved"])
@pytest.mark.parametrize("D", [4, 8, 16])
def test_brute_force_complex_rotation(mode, D):
    g = np.random.default_rng(D)
    x = g.standard_normal((2, 3, 5, D))
    theta = g.uniform(-7, 7, (5, D // 2))
    c, s = _tables_from_angles(theta)
    np.testing.assert_allclose(oracle.rope_apply(x, c, s, mode), _brute(x, theta, mode),
                               rtol=0, atol=1e-13)


@pytest.mark.parametrize("mode", ["half", "interleaved"])
def test_identity_and_quarter_turn(mode):
    g = np.random.default_rng(1)
    x = g.standard_normal((4, 6, 8))
    ones, zeros = np.ones((6, 4)), np.zeros((6, 4))
    assert np.array_equal(oracle.rope_apply(x, ones, zeros, mode), x)
    y = oracle.rope_apply(x, zeros, ones, mode)
    ia, ib = orope.pair_lanes(8, mode)
    assert np.array_equal(y[..., ia], -x[..., ib]) and np.array_equal(y[..., ib], x[..., ia])


@pytest.mark.parametrize("mode", ["half", "interleaved"])
def test_pair_norms_kept_and_rotations_compose(mode):
    g = np.random.default_rng(2)
    x = g.standard_normal((3, 7, 12))
    t1, t2 = g.uniform(-4, 4, (7, 6)), g.uniform(-4, 4, (7, 6))
    y = oracle.rope_apply(x, *_tables_from_angles(t1), mode)
    ia, ib = orope.pair_lanes(12, mode)
    np.testing.assert_allclose(y[..., ia] ** 2 + y[..., ib] ** 2, x[..., ia] ** 2 + x[..., ib] ** 2,
                               rtol=1e-13)
    z = oracle.rope_apply(y, *_tables_from_angles(t2), mode)
    np.testing.assert_allclose(z, oracle.rope_apply(x, *_tables_from_angles(t1 + t2), mode),
                               atol=1e-12)


@pytest.mark.parametrize("mode", ["half", "interleaved"])
def test_scores_depend_only_on_relative_position(mode):
    D, S = 16, 40
    w = 10000.0 ** (-np.arange(D // 2) * 2.0 / D)
    theta = np.arange(S)[:, None] * w[None, :]
    c, s = _tables_from_angles(theta)
    g = np.random.default_rng(3)
    qv, kv = g.standard_normal(D), g.standard_normal(D)
    q = oracle.rope_apply(np.tile(qv, (S, 1)), c, s, mode)   # the same query at every position
    k = oracle.rope_apply(np.tile(kv, (S, 1)), c, s, mode)
    for s1, s2, shift in ((5, 2, 17), (0, 9, 30), (12, 12, 20)):
        assert math.isclose(q[s1] @ k[s2], q[s1 + shift] @ k[s2 + shift], rel_tol=1e-11, abs_tol=1e-11)


def test_pairings_agree_up_to_a_lane_permutation():
    D = 16
    g = np.random.default_rng(4)
    x = g.standard_normal((2, 5, D))
    c, s = _tables_from_angles(g.uniform(-3, 3, (5, D // 2)))
    perm = np.empty(D, dtype=int)            # interleaved lane -> half lane
    perm[0::2], perm[1::2] = np.arange(D // 2), np.arange(D // 2) + D // 2
    xh = np.empty_like(x)
    xh[..., perm] = x
    yh = oracle.rope_apply(xh, c, s, "half")
    np.testing.assert_array_equal(yh[..., perm], oracle.rope_apply(x, c, s, "interleaved"))


def test_planted_wrong_pairing_is_caught(monkeypatch):
    g = np.random.default_rng(5)
    x = g.standard_normal((1, 3, 8))
    theta = g.uniform(-2, 2, (3, 4))
    good = oracle.rope_apply(x, *_tables_from_angles(theta), "half")
    monkeypatch.setattr(orope, "pair_lanes", lambda D, mode: (np.arange(D // 2) * 2, np.arange(D // 2) * 2 + 1))
    bad = orope.rope_apply(x, *_tables_from_angles(theta), "half")
    ref = _brute(x, theta, "half")
    assert np.allclose(good, ref, atol=1e-13) and not np.allclose(bad, ref, atol=1e-3)
