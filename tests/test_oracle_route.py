"""Pins of the oracle's sigmoid-affinity top-K routing.

Checked against properties that fix it: with no bias the sigmoid is monotone,
so the choice is numpy's stable descending sort of the logits; with equal
logits the choice is the bias order; a large bias on k experts forces them in
(ordered by their logits), so the bias is added to the score; the affinities
are scipy's logistic function of the chosen logits; equal scores go to the
lower expert index.
"""

import numpy as np
from scipy.special import expit


def test_no_bias_is_a_sort_of_the_logits(oracle):
    rng = np.random.default_rng(7401)
    T, E, k = 50, 64, 6
    u = rng.standard_normal((T, E)).astype(np.float32)
    ids, aff, _ = oracle.route_topk(u, np.zeros(E, np.float32), k)
    want = np.argsort(-u.astype(np.float64), axis=1, kind="stable")[:, :k]
    np.testing.assert_array_equal(ids, want)
    np.testing.assert_allclose(aff, expit(np.take_along_axis(u, want, 1).astype(np.float64)),
                               rtol=1e-15)


def test_equal_logits_follow_the_bias(oracle):
    rng = np.random.default_rng(7402)
    T, E, k = 4, 40, 8
    b = rng.permutation(E).astype(np.float32) * 0.01
    ids, aff, score = oracle.route_topk(np.zeros((T, E), np.float32), b, k)
    want = np.argsort(-b, kind="stable")[:k]
    for t in range(T):
        np.testing.assert_array_equal(ids[t], want)
    assert np.all(aff == 0.5)
    np.testing.assert_allclose(score[0], 0.5 + b.astype(np.float64), rtol=0, atol=1e-16)


def test_large_bias_forces_experts_in(oracle):
    rng = np.random.default_rng(7403)
    T, E, k = 30, 100, 5
    u = rng.standard_normal((T, E)).astype(np.float32)
    forced = rng.choice(E, size=k, replace=False)
    b = np.zeros(E, np.float32)
    b[forced] = 10.0
    ids, aff, _ = oracle.route_topk(u, b, k)
    for t in range(T):
        assert set(ids[t]) == set(forced)
        # among the forced experts the order is by logit (the bias is equal)
        assert np.all(np.diff(u[t, ids[t]]) <= 0)
    # the affinities are the sigmoid alone, without the bias
    np.testing.assert_allclose(aff, expit(np.take_along_axis(u, ids, 1).astype(np.float64)),
                               rtol=1e-15)


def test_ties_go_to_the_lower_index(oracle):
    E, k = 12, 4
    u = np.zeros((1, E), np.float32)
    u[0, [3, 7, 9]] = 1.0
    ids, _, _ = oracle.route_topk(u, np.zeros(E, np.float32), k)
    np.testing.assert_array_equal(ids[0], [3, 7, 9, 0])
