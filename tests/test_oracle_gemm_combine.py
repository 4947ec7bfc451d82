"""Pins of the oracle's fused down-projection + combine (gemm_combine_entries)
against values the mathematics fixes, computed without the oracle's GEMM:

* unit scales and small integer codes make every product exact, so with the
  raw affinities as weights (normalize = 0) and all of them 1, a token's output
  is the plain integer sum of its rows' dot products, done here by integer
  matmuls per expert;
* normalized equal affinities make the output the mean of those rows;
* a slot whose row lies outside [0, offsets[E]) adds nothing, and a token
  whose kept affinities sum to 0 gets zeros.
"""

import numpy as np
import pytest

import oracle



# E4M3 codes of small integers: 0x38 = 1.0, 0x40 = 2.0, sign bit 0x80
CODE = {0: 0x00, 1: 0x38, 2: 0x40, -1: 0xB8, -2: 0xC0}


def _case(seed, E=3, T=20, k=3, N=256, K=256):
    rng = np.random.default_rng(seed)
    ids = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    r = oracle.route(ids, E)
    R = int(r["offsets"][-1])
    ia = rng.integers(-2, 3, (R, K))
    ib = rng.integers(-2, 3, (E, N, K))
    a = np.vectorize(CODE.get)(ia).astype(np.uint8)
    b = np.vectorize(CODE.get)(ib).astype(np.uint8)
    sa = np.ones((K // 128, R), np.float32)
    sb = np.ones((E, N // 128, K // 128), np.float32)
    # integer reference of every row: Y[r] = ia[r] @ ib[e(r)].T
    expert_of_row = np.repeat(np.arange(E), np.diff(r["offsets"]))
    Y = np.stack([ia[i] @ ib[expert_of_row[i]].T for i in range(R)]).astype(np.int64)
    return ids, r, a, sa, b, sb, Y, T, k, N


def _all_entries(T, N):
    t, c = np.meshgrid(np.arange(T), np.arange(N), indexing="ij")
    return t.ravel(), c.ravel()


def test_unit_affinities_sum_integer_rows():
    ids, r, a, sa, b, sb, Y, T, k, N = _case(1)
    aff = np.ones((T, k), np.float32)
    t, c = _all_entries(T, N)
    out, bound, mag = oracle.gemm_combine_entries(a, sa, b, sb, r["offsets"], r["token_row"], aff,
                                                  t, c, normalize=False)
    tr = r["token_row"].reshape(T, k)
    want = np.stack([Y[tr[i]].sum(axis=0) for i in range(T)]).ravel().astype(np.float64)
    assert np.array_equal(out, want)
    assert np.all(mag <= bound + 1e-9)


def test_equal_normalized_affinities_average_rows():
    ids, r, a, sa, b, sb, Y, T, k, N = _case(2)
    aff = np.full((T, k), 0.25, np.float32)
    t, c = _all_entries(T, N)
    out, _, _ = oracle.gemm_combine_entries(a, sa, b, sb, r["offsets"], r["token_row"], aff, t, c)
    tr = r["token_row"].reshape(T, k)
    want = np.stack([Y[tr[i]].sum(axis=0) / k for i in range(T)]).ravel()
    assert np.allclose(out, want, rtol=1e-15, atol=1e-12)


def test_dropped_slots_and_zero_sum_tokens():
    ids, r, a, sa, b, sb, Y, T, k, N = _case(3)
    tr = r["token_row"].copy().reshape(T, k)
    tr[0, 1] = -1                      # dropped slot
    tr[1, :] = -1                      # token without rows
    aff = np.ones((T, k), np.float32)
    aff[2, :] = 0.0                    # kept affinities sum to 0
    t, c = _all_entries(T, N)
    out, _, _ = oracle.gemm_combine_entries(a, sa, b, sb, r["offsets"], tr.ravel(), aff, t, c)
    out = out.reshape(T, N)
    assert np.array_equal(out[0], (Y[tr[0, 0]] + Y[tr[0, 2]]) / 2.0)
    assert np.all(out[1] == 0) and np.all(out[2] == 0)
