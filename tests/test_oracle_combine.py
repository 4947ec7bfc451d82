"""Pins of the oracle's unpermute + combine.

Checked against what the definition fixes by itself: one slot with normalized
weights copies its row exactly; k copies of one row reproduce it (weights sum
to 1); the order of a token's slots does not matter; a dropped slot equals
leaving it out; unnormalized small-integer data gives exact integer sums
(brute force with Python integers); the routing maps of the permuting
quantizer undo the permutation (combine of the permuted input with unit
weights and k = 1 is the input).
"""

import numpy as np
import torch

from fp8_fine_grained_permute_b200 import workloads as W


def bf16(a):
    return torch.as_tensor(np.asarray(a, np.float32)).to(torch.bfloat16)


def f64(t):
    return t.to(torch.float64).numpy()


def test_single_slot_normalized_is_a_copy(oracle):
    rng = np.random.default_rng(7301)
    R, C, T = 9, 64, 9
    y = bf16(rng.standard_normal((R, C)))
    rows = rng.permutation(R).astype(np.int32)
    aff = rng.uniform(0.1, 0.9, (T, 1)).astype(np.float32)
    out, bound = oracle.unpermute_combine(y, rows, aff, normalize=True)
    np.testing.assert_array_equal(out, f64(y)[rows])
    np.testing.assert_array_equal(bound, np.abs(f64(y)[rows]))


def test_repeated_row_reproduces_it(oracle):
    rng = np.random.default_rng(7302)
    R, C, T, k = 5, 32, 5, 6
    y = bf16(rng.standard_normal((R, C)))
    rows = np.repeat(np.arange(T, dtype=np.int32), k)
    aff = rng.uniform(0.01, 1.0, (T, k)).astype(np.float32)
    out, _ = oracle.unpermute_combine(y, rows, aff, normalize=True)
    np.testing.assert_allclose(out, f64(y)[:T], rtol=1e-14, atol=0)


def test_slot_order_does_not_matter(oracle):
    rng = np.random.default_rng(7303)
    R, C, T, k = 40, 48, 10, 4
    y = bf16(rng.standard_normal((R, C)))
    rows = rng.integers(0, R, (T, k)).astype(np.int32)
    aff = rng.uniform(0.01, 1.0, (T, k)).astype(np.float32)
    perm = np.array([rng.permutation(k) for _ in range(T)])
    rows_p = np.take_along_axis(rows, perm, 1)
    aff_p = np.take_along_axis(aff, perm, 1)
    for norm in (True, False):
        a, _ = oracle.unpermute_combine(y, rows.ravel(), aff, normalize=norm)
        b, _ = oracle.unpermute_combine(y, rows_p.ravel(), aff_p, normalize=norm)
        np.testing.assert_allclose(a, b, rtol=1e-13, atol=1e-13)


def test_dropped_slot_equals_leaving_it_out(oracle):
    rng = np.random.default_rng(7304)
    R, C, T, k = 30, 16, 8, 3
    y = bf16(rng.standard_normal((R, C)))
    rows = rng.integers(0, R, (T, k)).astype(np.int32)
    aff = rng.uniform(0.01, 1.0, (T, k)).astype(np.float32)
    rows_d = rows.copy()
    rows_d[:, 1] = -1           # no row
    rows_d[3, 2] = R            # out of range: dropped as well
    others = [t for t in range(T) if t != 3]
    for norm in (True, False):
        got, _ = oracle.unpermute_combine(y, rows_d.ravel(), aff, normalize=norm)
        two, _ = oracle.unpermute_combine(y, rows[:, [0, 2]].copy().ravel(),
                                          aff[:, [0, 2]].copy(), normalize=norm)
        one, _ = oracle.unpermute_combine(y, rows[3:4, :1].copy().ravel(), aff[3:4, :1].copy(),
                                          normalize=norm)
        np.testing.assert_array_equal(got[others], two[others])
        np.testing.assert_array_equal(got[3], one[0])


def test_all_dropped_token_is_zero(oracle):
    y = bf16(np.ones((4, 8)))
    rows = np.array([-1, -1, 0, 1], np.int32)
    aff = np.array([[0.5, 0.5], [0.25, 0.75]], np.float32)
    out, _ = oracle.unpermute_combine(y, rows, aff, normalize=True)
    assert not out[0].any()
    np.testing.assert_array_equal(out[1], np.ones(8))


def test_unnormalized_small_integers_exact(oracle):
    rng = np.random.default_rng(7305)
    R, C, T, k = 50, 24, 20, 5
    iy = rng.integers(-100, 101, (R, C))
    ia = rng.integers(-8, 9, (T, k))
    rows = rng.integers(-1, R, (T, k)).astype(np.int32)
    out, _ = oracle.unpermute_combine(bf16(iy), rows.ravel(), ia.astype(np.float32),
                                      normalize=False)
    for t in range(T):
        for c in range(C):
            want = sum(int(ia[t, j]) * int(iy[rows[t, j], c]) for j in range(k) if rows[t, j] >= 0)
            assert out[t, c] == want


def test_unit_weights_undo_the_permutation(oracle):
    # the permuting quantizer's token_row maps each (token, slot) to its row in
    # expert order; with k = 1 the combine of the permuted rows is the input
    cfg = W.CONFIGS["tiny"]
    T, E = cfg.T, cfg.E
    rng = np.random.default_rng(7306)
    ids = rng.integers(0, E, (T, 1)).astype(np.int32)
    r = oracle.route(ids, E)
    x = bf16(rng.standard_normal((T, 40)))
    permuted = x[torch.from_numpy(r["row_token"]).long()]
    out, _ = oracle.unpermute_combine(permuted, r["token_row"], np.ones((T, 1), np.float32),
                                      normalize=False)
    np.testing.assert_array_equal(out, f64(x))
