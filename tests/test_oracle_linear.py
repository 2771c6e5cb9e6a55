"""Pins of the oracle's dense layer and query head (CPU only).

The module around the operator has four linear layers: the value and output
projections (discosf.com/news/5175395 §2.2, §3.1) and the query head that
predicts offsets and logits (cf-1.com/news/4799680 §3.2).  Pins: a
hand-worked example (tests/golden/worked_linear_2x3.json), identity and zero
weights, the adjoint identities of a bilinear map, the column order of the
query head checked through closed forms, and central differences of the
head's chain rule.
"""
import json
import os

import numpy as np
import pytest

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def test_golden_worked_linear(oracle_mod):
    o = oracle_mod
    g = _load("worked_linear_2x3.json")
    x, w, b = (np.array(g[k], np.float64) for k in ("x", "weight", "bias"))
    assert np.array_equal(o.linear(x, w, b), np.array(g["expected_y"]))
    gx, gw, gb = o.linear_backward(x, w, np.array(g["grad_y"], np.float64))
    assert np.array_equal(gx, np.array(g["expected_grad_x"]))
    assert np.array_equal(gw, np.array(g["expected_grad_weight"]))
    assert np.array_equal(gb, np.array(g["expected_grad_bias"]))


def test_identity_and_zero_weights(oracle_mod):
    o = oracle_mod
    rng = np.random.default_rng(5)
    x = rng.standard_normal((3, 4, 8))
    b = rng.standard_normal(8)
    assert np.array_equal(o.linear(x, np.eye(8)), x)
    assert np.array_equal(o.linear(x, np.eye(8), b), x + b)
    assert np.array_equal(o.linear(x, np.zeros((5, 8)), b[:5]), np.broadcast_to(b[:5], (3, 4, 5)))
    # a permutation matrix permutes the features
    perm = rng.permutation(8)
    assert np.array_equal(o.linear(x, np.eye(8)[perm]), x[..., perm])


def test_adjoint_identities(oracle_mod):
    """y = x W^T is bilinear: <g, y> = <grad_x, x> = <grad_W, W>, and
    grad_b = the column sums of g."""
    o = oracle_mod
    rng = np.random.default_rng(6)
    x, w, g = rng.standard_normal((37, 24)), rng.standard_normal((19, 24)), rng.standard_normal((37, 19))
    y = o.linear(x, w)
    gx, gw, gb = o.linear_backward(x, w, g)
    s = np.abs(g).sum() * np.abs(y).max()
    assert abs((g * y).sum() - (gx * x).sum()) <= 1e-12 * s
    assert abs((g * y).sum() - (gw * w).sum()) <= 1e-12 * s
    assert np.allclose(gb, g.sum(0), rtol=0, atol=1e-12 * np.abs(g).sum())


def _levels():
    return np.array([[3, 5], [2, 7]], np.int64)  # (H, W), W != H on each level


def test_query_head_column_order(oracle_mod):
    """Zero weights make the head's outputs its bias: offset (m, l, k, c) sits
    at column ((m*L + l)*K + k)*2 + c and logit (m, l*K + k) at column
    2P + m*L*K + l*K + k.  Locations then equal ref + bias / (W_l, H_l), and
    a run of logits with one entry 60 above the others gives that entry
    weight 1 (exp(-60) is below float64 rounding of 1)."""
    o = oracle_mod
    M, L, K, C = 2, 2, 3, 8
    P = M * L * K
    sh = _levels()
    b = np.zeros(3 * P)
    b[:2 * P] = np.arange(2 * P) + 1.0          # distinct offsets
    hot = [(0, 4), (1, 0)]                       # (m, position in the run)
    for m, j in hot:
        b[2 * P + m * L * K + j] = 60.0
    q = np.zeros((1, 1, C))
    ref = np.array([[[0.25, 0.75]]])
    loc, a = o.query_head(q, np.zeros((3 * P, C)), b, ref, sh, M, L, K)
    for m in range(M):
        for l in range(L):
            H, W = sh[l]
            for k in range(K):
                col = ((m * L + l) * K + k) * 2
                assert loc[0, 0, m, l, k, 0] == 0.25 + b[col] / W
                assert loc[0, 0, m, l, k, 1] == 0.75 + b[col + 1] / H
    for m, j in hot:
        assert abs(a[0, 0, m].reshape(-1)[j] - 1.0) <= 1e-15
        assert a[0, 0, m].reshape(-1).sum() == pytest.approx(1.0, abs=1e-15)


def test_query_head_backward_central_differences(oracle_mod):
    """The gradient of J = <G_loc, loc> + <G_A, A> with respect to the head's
    linear outputs (here the bias, with zero weights) equals
    query_head_backward's grad_head; with respect to the reference point it
    equals grad_reference_points."""
    o = oracle_mod
    rng = np.random.default_rng(7)
    M, L, K, C = 2, 2, 2, 8
    P = M * L * K
    sh = _levels()
    b = rng.standard_normal(3 * P)
    w = np.zeros((3 * P, C))
    q = rng.standard_normal((1, 1, C))
    ref = rng.uniform(0, 1, (1, 1, 2))
    G_loc = rng.standard_normal((1, 1, M, L, K, 2))
    G_A = rng.standard_normal((1, 1, M, L, K))

    def J(bb, rr):
        loc, a = o.query_head(q, w, bb, rr, sh, M, L, K)
        return (G_loc * loc).sum() + (G_A * a).sum()

    _, a = o.query_head(q, w, b, ref, sh, M, L, K)
    gh, gref = o.query_head_backward(sh, a, G_loc, G_A)
    h = 1e-6
    for j in range(3 * P):
        e = np.zeros(3 * P)
        e[j] = h
        fd = (J(b + e, ref) - J(b - e, ref)) / (2 * h)
        assert abs(fd - gh[0, 0, j]) <= 1e-7 * (1 + abs(fd)), j
    for c in range(2):
        e = np.zeros((1, 1, 2))
        e[..., c] = h
        fd = (J(b, ref + e) - J(b, ref - e)) / (2 * h)
        assert abs(fd - gref[0, 0, c]) <= 1e-7 * (1 + abs(fd)), c
