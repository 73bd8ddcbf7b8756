"""Pins for the projection oracle (oracle/projection.py), against things other than itself.

* brute force: scalar loops over tiny shapes, summed with math.fsum, written from
  y[n] = sum_c x[c] W[n, c] + b[n] and the head layout (column h D + d of the Q, K or V
  block is head h, lane d);
* routing: a weight with a single 1 sends one input channel to exactly one (q/k/v,
  head, lane) output, and nowhere else;
* the output projection with the identity weight lays the heads side by side;
* linearity, and RoPE with identity tables changes nothing;
* planted mistakes (an untransposed weight, heads and lanes swapped) are caught.
No GPU is used here.
"""

import math

import numpy as np
import pytest

import oracle
from oracle import projection as P


def _rng(s):
    return np.random.default_rng(s)


def brute_qkv(x, w, b, H, D):
    B, S, C = x.shape
    out = np.zeros((3, B, H, S, D))
    for which in range(3):
        for bb in range(B):
            for h in range(H):
                for s in range(S):
                    for d in range(D):
                        n = which * H * D + h * D + d
                        acc = math.fsum(float(x[bb, s, c]) * float(w[n, c]) for c in range(C))
                        out[which, bb, h, s, d] = acc + (0.0 if b is None else float(b[n]))
    return out


def brute_out(o, w, b):
    B, H, S, D = o.shape
    Cout = w.shape[0]
    y = np.zeros((B, S, Cout))
    for bb in range(B):
        for s in range(S):
            for n in range(Cout):
                acc = math.fsum(float(o[bb, h, s, d]) * float(w[n, h * D + d])
                                for h in range(H) for d in range(D))
                y[bb, s, n] = acc + (0.0 if b is None else float(b[n]))
    return y


@pytest.mark.parametrize("B,S,C,H,D,bias", [(1, 3, 5, 2, 4, True), (2, 4, 6, 3, 2, False),
                                            (2, 2, 8, 1, 6, True)])
def test_qkv_brute_force(B, S, C, H, D, bias):
    r = _rng(B * 100 + S * 10 + C)
    x = r.standard_normal((B, S, C))
    w = r.standard_normal((3 * H * D, C))
    b = r.standard_normal(3 * H * D) if bias else None
    got = P.qkv_projection(x, w, b, H, D)
    ref = brute_qkv(x, w, b, H, D)
    for i in range(3):
        assert got[i].shape == (B, H, S, D)
        assert np.max(np.abs(got[i] - ref[i])) <= 1e-12


@pytest.mark.parametrize("bias", [True, False])
def test_out_projection_brute_force(bias):
    r = _rng(3)
    o = r.standard_normal((2, 3, 4, 5))
    w = r.standard_normal((7, 15))
    b = r.standard_normal(7) if bias else None
    assert np.max(np.abs(P.out_projection(o, w, b) - brute_out(o, w, b))) <= 1e-12


def test_one_hot_weight_routes_one_channel_to_one_lane():
    B, S, C, H, D = 2, 3, 6, 4, 8
    x = _rng(4).standard_normal((B, S, C))
    for which, h, d, c in [(0, 0, 0, 0), (1, 3, 7, 5), (2, 2, 3, 1)]:
        w = np.zeros((3 * H * D, C))
        w[which * H * D + h * D + d, c] = 1.0
        outs = P.qkv_projection(x, w, None, H, D)
        for i, t in enumerate(outs):
            want = np.zeros((B, H, S, D))
            if i == which:
                want[:, h, :, d] = x[:, :, c]
            assert np.array_equal(t, want)


def test_identity_out_projection_puts_heads_side_by_side():
    o = _rng(5).standard_normal((2, 3, 4, 5))
    y = P.out_projection(o, np.eye(15), None)
    for h in range(3):
        assert np.array_equal(y[:, :, h * 5:(h + 1) * 5], o[:, h])


def test_linearity_and_bias():
    r = _rng(6)
    x1, x2 = r.standard_normal((2, 1, 3, 16))
    w = r.standard_normal((3 * 2 * 4, 16))
    b = r.standard_normal(24)
    a = P.qkv_projection(x1 + 2 * x2, w, b, 2, 4)
    p1 = P.qkv_projection(x1, w, b, 2, 4)
    p2 = P.qkv_projection(x2, w, None, 2, 4)
    for i in range(3):
        assert np.max(np.abs(a[i] - (p1[i] + 2 * p2[i]))) <= 1e-12


@pytest.mark.parametrize("mode", ["half", "interleaved"])
def test_rope_with_identity_tables_is_the_plain_projection(mode):
    r = _rng(7)
    x = r.standard_normal((1, 5, 8))
    w = r.standard_normal((3 * 2 * 4, 8))
    cos, sin = np.ones((5, 2)), np.zeros((5, 2))
    plain = P.qkv_projection(x, w, None, 2, 4)
    rot = P.qkv_rope_projection(x, w, None, 2, 4, cos, sin, mode)
    for i in range(3):
        assert np.array_equal(plain[i], rot[i])
    # a quarter turn moves Q and K but never V
    cos, sin = np.zeros((5, 2)), np.ones((5, 2))
    rot = P.qkv_rope_projection(x, w, None, 2, 4, cos, sin, mode)
    assert not np.allclose(rot[0], plain[0]) and not np.allclose(rot[1], plain[1])
    assert np.array_equal(rot[2], plain[2])


def test_planted_mistakes_are_caught():
    r = _rng(8)
    B, S, C, H, D = 1, 3, 12, 2, 6          # 3 H D = 36, C = 12: W is not square
    x = r.standard_normal((B, S, C))
    w = r.standard_normal((3 * H * D, C))
    ref = brute_qkv(x, w, None, H, D)
    # heads and lanes swapped in the column layout
    t = (x.reshape(B * S, C) @ w.T).reshape(B, S, 3, D, H)
    wrong = t[:, :, 0].transpose(0, 3, 1, 2)
    assert np.max(np.abs(wrong - ref[0])) > 1e-3
    # Q, K, V blocks taken in the wrong order (K where Q belongs)
    t = (x.reshape(B * S, C) @ w.T).reshape(B, S, 3, H, D)
    assert np.max(np.abs(t[:, :, 1].transpose(0, 2, 1, 3) - ref[0])) > 1e-3
