"""The oracle's expert-parallel exchange (CPU): a hand-worked example, the
one-rank case (nothing moves), conservation of rows, and the combine as the
dispatch's inverse."""

import numpy as np


def _source(expert_of_row, K, E, seed):
    """Rows already grouped by expert: row i has expert expert_of_row[i]."""
    rng = np.random.default_rng(seed)
    n = len(expert_of_row)
    xq = rng.integers(0, 256, (n, K), dtype=np.uint8)
    sa = rng.random((K // 128, n), dtype=np.float32)
    counts = np.bincount(np.asarray(expert_of_row, int), minlength=E)
    return xq, sa, np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)


def test_hand_worked_two_ranks(oracle):
    # E = 4 over W = 2: rank 0 owns experts 0, 1; rank 1 owns 2, 3.
    s0 = _source([0, 0, 1, 2, 3], 128, 4, 1)     # rows 0..4
    s1 = _source([1, 2, 2, 3], 128, 4, 2)        # rows 0..3
    d = oracle.ep_dispatch([s0, s1], 2)
    # rank 0: expert 0 <- s0 rows 0, 1; expert 1 <- s0 row 2, then s1 row 0
    assert d[0]["origin"].tolist() == [[0, 0], [0, 1], [0, 2], [1, 0]]
    assert d[0]["offsets"].tolist() == [0, 2, 4]
    # rank 1: expert 2 <- s0 row 3, s1 rows 1, 2; expert 3 <- s0 row 4, s1 row 3
    assert d[1]["origin"].tolist() == [[0, 3], [1, 1], [1, 2], [0, 4], [1, 3]]
    assert d[1]["offsets"].tolist() == [0, 3, 5]
    assert np.array_equal(d[1]["xq"][1], s1[0][1]) and np.array_equal(d[1]["sa"][:, 1], s1[1][:, 1])


def test_one_rank_moves_nothing(oracle):
    s = _source([0, 0, 1, 3, 3, 3], 256, 4, 3)
    d = oracle.ep_dispatch([s], 1)[0]
    assert np.array_equal(d["xq"], s[0]) and np.array_equal(d["sa"], s[1])
    assert np.array_equal(d["offsets"], s[2])


def test_rows_conserved_and_combine_inverts(oracle):
    rng = np.random.default_rng(4)
    W, E, K = 4, 16, 256
    srcs = [_source(np.sort(rng.integers(0, E, int(rng.integers(0, 40)))), K, E, 10 + s)
            for s in range(W)]
    d = oracle.ep_dispatch(srcs, W)
    assert sum(len(x["origin"]) for x in d) == sum(len(s[0]) for s in srcs)
    for r, x in enumerate(d):
        counts = np.diff(x["offsets"])
        want = sum(np.diff(s[2])[r * E // W:(r + 1) * E // W] for s in srcs)
        assert np.array_equal(counts, want)
    # outputs that depend only on the row: the combine returns each source's rows
    y = [x["xq"][:, :16].astype(np.float32) * 2.0 for x in d]
    back = oracle.ep_combine(y, d, [len(s[0]) for s in srcs])
    for s, b in zip(srcs, back):
        assert np.array_equal(b, s[0][:, :16].astype(np.float32) * 2.0)
