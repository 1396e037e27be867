"""Pins of the router oracle against closed forms, brute force and finite differences."""
import itertools

import numpy as np
import pytest

from oracle import router as orouter


def test_softmax_closed_forms():
    # equal logits -> uniform; a shift of all logits changes nothing; two experts -> logistic
    np.testing.assert_allclose(orouter.softmax(np.zeros((1, 5))), np.full((1, 5), 0.2))
    l = np.random.default_rng(0).standard_normal((4, 7))
    np.testing.assert_allclose(orouter.softmax(l), orouter.softmax(l + 3.5), rtol=1e-14)
    a = 0.7
    np.testing.assert_allclose(orouter.softmax(np.array([[a, 0.0]]))[0, 0], 1 / (1 + np.exp(-a)), rtol=1e-15)
    np.testing.assert_allclose(orouter.softmax(l).sum(axis=1), 1.0, rtol=1e-14)


def test_minus_inf_expert_gets_zero_and_is_last():
    l = np.array([[0.5, -np.inf, 0.1, -np.inf]], dtype=np.float32)
    p = orouter.softmax(l)
    assert p[0, 1] == 0.0 and p[0, 3] == 0.0
    idx, pr = orouter.topk(l, 3)
    assert idx.tolist() == [[0, 2, 1]]        # the -inf experts come last, lower index first
    assert pr[0, 2] == 0.0
    with pytest.raises(ValueError):
        orouter.softmax(np.full((1, 3), -np.inf))


def test_topk_brute_force_and_ties():
    rng = np.random.default_rng(1)
    # integer logits in a small range: many ties
    l = rng.integers(-2, 3, size=(64, 6)).astype(np.float32)
    for k in (1, 2, 4, 6):
        idx, pr = orouter.topk(l, k)
        for t in range(64):
            # brute force: the chosen set maximises the sum of logits, and among sets with
            # the same sorted values the lexicographically smallest indices win
            best = max(itertools.combinations(range(6), k),
                       key=lambda c: (sorted((float(l[t, e]) for e in c), reverse=True), [-e for e in c]))
            assert sorted(idx[t].tolist()) == sorted(best)
            vals = [float(l[t, e]) for e in idx[t]]
            assert vals == sorted(vals, reverse=True)
            for j in range(k - 1):      # equal logits: lower index first
                if vals[j] == vals[j + 1]:
                    assert idx[t, j] < idx[t, j + 1]
        np.testing.assert_allclose(pr, np.take_along_axis(orouter.softmax(l), idx, axis=1))


def test_backward_finite_differences():
    rng = np.random.default_rng(2)
    T, E, k = 5, 8, 3
    l = rng.standard_normal((T, E))
    idx, _ = orouter.topk(l.astype(np.float32), k)
    w = rng.standard_normal((T, k))           # L = sum_t,j w[t, j] * P[t, idx[t, j]]

    def loss(x):
        return float(np.sum(w * np.take_along_axis(orouter.softmax(x), idx, axis=1)))

    g = orouter.topk_backward(l, idx, w)
    h = 1e-6
    fd = np.zeros_like(l)
    for t in range(T):
        for e in range(E):
            a, b = l.copy(), l.copy()
            a[t, e] += h
            b[t, e] -= h
            fd[t, e] = (loss(a) - loss(b)) / (2 * h)
    np.testing.assert_allclose(g, fd, rtol=1e-6, atol=1e-9)
    # the gradient of a softmax-only loss sums to zero over the experts of a token
    np.testing.assert_allclose(g.sum(axis=1), 0.0, atol=1e-14)
