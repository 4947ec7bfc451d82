"""The oracle's threaded drivers and its dense fp64 GEMM (CPU only).

The threaded drivers must return exactly what one call of the plain function
returns (they only cut the input into independent experts, rows or column
groups).  The dense GEMM reference, a library matmul of the dequantized
operands, is pinned by a closed form (unit scales and small integer codes give
an exact integer product) and against the scalar per-entry oracle."""

import numpy as np
import pytest

from fp8_fine_grained_permute_b200 import workloads as W


@pytest.mark.parametrize("nthreads", [1, 3, 8])
def test_threaded_weight_quantize_and_transpose_equal_single_call(oracle, nthreads):
    for shape in [(3, 256, 384), (1, 640, 256), (9, 128, 128)]:
        w = W.gen_normal_bf16(shape, 0.02, 5, shape[0])
        ref = oracle.quantize_weight(w)
        got = oracle.quantize_weight_threaded(w, nthreads)
        assert all(np.array_equal(x, y) for x, y in zip(ref, got))
        tr = oracle.transpose_blockq(*ref)
        tg = oracle.transpose_blockq_threaded(*ref, nthreads=nthreads)
        assert all(np.array_equal(x, y) for x, y in zip(tr, tg))


@pytest.mark.parametrize("nthreads", [1, 4])
def test_threaded_rows_and_colwise_equal_single_call(oracle, nthreads):
    x = W.gen_grad_bf16((301, 384), 5, 3)
    r = oracle.quantize_act(x, None, 1)
    xq, sa = oracle.quantize_rows_threaded(x, nthreads)
    assert np.array_equal(r["xq"], xq) and np.array_equal(r["sa"], sa)
    off = np.array([0, 5, 5, 200, 301], np.int32)
    rm = np.random.default_rng(1).integers(0, 301, 301).astype(np.int32)
    for row_map in (None, rm):
        r = oracle.quantize_act_colwise(x, off, row_map=row_map)
        q = oracle.quantize_act_colwise_threaded(x, off, row_map=row_map, nthreads=nthreads)
        assert all(np.array_equal(r[k], q[k]) for k in r)


def test_threaded_gemm_entries_equal_single_call(oracle):
    a = W.gen_e4m3_codes((70, 256), 3, 1).numpy()
    sa = W.gen_scales((2, 70), 3, 2).numpy()
    b = W.gen_e4m3_codes((2, 128, 256), 3, 3).numpy()
    sb = W.gen_scales((2, 1, 2), 3, 4).numpy()
    off = np.array([0, 30, 70], np.int32)
    rng = np.random.default_rng(2)
    rows, cols = rng.integers(0, 70, 500), rng.integers(0, 128, 500)
    r1 = oracle.gemm_mgrouped_entries(a, sa, b, sb, off, rows, cols)
    r2 = oracle.gemm_mgrouped_entries_threaded(a, sa, b, sb, off, rows, cols, nthreads=5)
    assert np.array_equal(r1[0], r2[0]) and np.array_equal(r1[1], r2[1])


def test_dense_gemm_exact_on_small_integers(oracle):
    """Unit scales and codes of the integers 0..7 (E4M3 codes 0x00..0x48 hold
    them exactly): the product is an integer matrix product, known exactly."""
    dq = oracle.e4m3_decode_table()
    ints = {int(v): c for c, v in enumerate(dq) if np.isfinite(v) and c < 0x80 and v == int(v) and v <= 7}
    rng = np.random.default_rng(7)
    av = rng.integers(0, 8, (64, 384))
    bv = rng.integers(0, 8, (256, 384))
    lut = np.array([ints[i] for i in range(8)], np.uint8)
    ref, bound = oracle.gemm_dense_fp64(lut[av], np.ones((3, 64), np.float32), lut[bv],
                                        np.ones((2, 3), np.float32))
    exact = av.astype(np.int64) @ bv.astype(np.int64).T
    assert np.array_equal(ref, exact.astype(np.float64))
    assert np.array_equal(bound, exact.astype(np.float64))


def test_dense_gemm_matches_scalar_entries(oracle):
    """Random codes and scales: the matmul reference equals the scalar oracle's
    per-entry fp64 sum to within fp64 rounding (2^-40 of the |term| sum)."""
    M, N, K = 96, 256, 512
    a = W.gen_e4m3_codes((M, K), 9, 1).numpy()
    sa = W.gen_scales((K // 128, M), 9, 2).numpy()
    b = W.gen_e4m3_codes((1, N, K), 9, 3).numpy()
    sb = W.gen_scales((1, N // 128, K // 128), 9, 4).numpy()
    ref, bound = oracle.gemm_dense_fp64(a, sa, b, sb)
    r, c = np.meshgrid(np.arange(M), np.arange(N), indexing="ij")
    sref, sbound = oracle.gemm_mgrouped_entries(a, sa, b, sb, np.array([0, M], np.int32),
                                                r.ravel(), c.ravel())
    assert np.all(np.abs(ref.ravel() - sref) <= 2.0 ** -40 * sbound)
    assert np.all(np.abs(bound.ravel() - sbound) <= 2.0 ** -40 * sbound)
