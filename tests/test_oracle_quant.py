"""Pins of the oracle's quantize, permute, transpose and GEMM references.

Each test checks the oracle against something other than itself: an invariant
fixed by the format or the method (max element -> +-448, dequantisation error
bound, square-block transpose commutes with dequantisation, every (token, slot)
dispatched exactly once), a special case that reduces to a library routine
(power-of-two scales -> torch's float8 cast; unit scales with small integers ->
exact int64 matmul; one expert -> numpy fp64 matmul), or brute force.
"""

import math
from fractions import Fraction

import numpy as np
import pytest
import torch

from fp8_fine_grained_permute_b200 import workloads as W


def bf16_bits(a) -> np.ndarray:
    t = torch.as_tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def bf16_to_f32(u: np.ndarray) -> np.ndarray:
    return (u.astype(np.uint32) << 16).view(np.float32)


def rand_bf16(shape, seed, scale=1.0):
    rng = np.random.default_rng(seed)
    return bf16_bits(rng.standard_normal(shape) * scale)


DQ = None


def dq(oracle, codes):
    global DQ
    if DQ is None:
        DQ = oracle.e4m3_decode_table()
    return DQ[codes]


# --------------------------------------------------------------------------
# tile quantisation
# --------------------------------------------------------------------------

def test_max_element_maps_to_448_for_every_bf16_amax(oracle):
    """For every positive finite bf16 value a, a tile whose largest magnitude
    is a encodes that element as +-448 (0x7E / 0xFE)."""
    pos = np.arange(1, 0x7F80, dtype=np.uint16)          # all positive finite bf16
    T = pos.size
    x = np.zeros((T, 128), np.uint16)
    col = np.arange(T) % 128
    x[np.arange(T), col] = pos
    x[np.arange(T) % 7 == 3, (col[np.arange(T) % 7 == 3] + 1) % 128] = 0x8000  # some -0
    out = oracle.quantize_act(x, None, 1)
    assert np.all(out["xq"][np.arange(T), col] == 0x7E)
    neg = pos | 0x8000
    x2 = np.zeros((T, 128), np.uint16)
    x2[np.arange(T), col] = neg
    out2 = oracle.quantize_act(x2, None, 1)
    assert np.all(out2["xq"][np.arange(T), col] == 0xFE)
    assert np.all(out["sa"] > 0)


def test_random_tiles_max_maps_to_448_and_error_bound(oracle):
    x = rand_bf16((512, 1024), 1)
    x[3, :128] = bf16_bits(np.random.default_rng(2).standard_normal(128) * 1e-30)
    x[5, 128:256] = bf16_bits(np.random.default_rng(3).standard_normal(128) * 1e30)
    out = oracle.quantize_act(x, None, 1)
    xf = bf16_to_f32(x).astype(np.float64).reshape(512, 8, 128)
    q = out["xq"].reshape(512, 8, 128)
    s = out["sa"].T.reshape(512, 8, 1).astype(np.float64)
    amax_pos = np.abs(xf).argmax(axis=2)
    assert np.all(np.take_along_axis(q, amax_pos[..., None], 2)[..., 0] & 0x7F == 0x7E)
    deq = dq(oracle, q) * s
    y = np.abs(xf) / s
    normal = y >= 2.0 ** -6
    rel = np.abs(deq - xf)[normal] / np.abs(xf)[normal]
    assert rel.max() <= 2.0 ** -4
    # subnormal outputs: absolute error at most half the subnormal step
    assert np.all(np.abs(deq - xf)[~normal] <= 2.0 ** -10 * np.broadcast_to(s, xf.shape)[~normal])


def test_zero_tile_has_unit_scale_and_keeps_sign(oracle):
    x = np.zeros((2, 256), np.uint16)
    x[1, 128:] = 0x8000            # -0.0 tile
    x[0, 128] = bf16_bits([3.0])[0]
    out = oracle.quantize_act(x, None, 1)
    assert out["sa"][0, 0] == 1.0 and out["sa"][0, 1] == 1.0
    assert np.all(out["xq"][0, :128] == 0) and np.all(out["xq"][1, :128] == 0)
    assert np.all(out["xq"][1, 128:] == 0x80)
    assert out["sa"][1, 1] == 1.0


@pytest.mark.parametrize("m", [-20, -3, 0, 5])
def test_power_of_two_scale_reduces_to_plain_cast(oracle, m):
    """amax = 448 * 2^m gives s = 2^m exactly, and then q = e4m3(x * 2^-m): the
    result equals torch's float8_e4m3fn cast of the exactly rescaled values."""
    rng = np.random.default_rng(100 + m)
    v = rng.standard_normal((64, 128)) * 100 * 2.0 ** m
    v[:, 7] = 448 * 2.0 ** m
    x = bf16_bits(v)
    assert np.all(bf16_to_f32(x)[:, 7] == np.float32(448 * 2.0 ** m))
    x = np.where(np.abs(bf16_to_f32(x)) > np.float32(448 * 2.0 ** m), bf16_bits([0.0])[0], x)
    out = oracle.quantize_act(x, None, 1)
    assert np.all(out["sa"] == np.float32(2.0 ** m))
    scaled = torch.from_numpy(bf16_to_f32(x).astype(np.float64) * 2.0 ** -m).to(torch.float32)
    ref = scaled.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(out["xq"], ref)


def test_tiny_tiles_brute_force(oracle):
    """Tiles with 1-3 non-zero values: every code is the exact nearest E4M3
    value (ties to even) of fp32(x / s), found by exhaustive search in
    rationals, and s is the correctly rounded fp32 quotient amax / 448."""
    mags = [Fraction(float(v)) for v in oracle.e4m3_decode_table()[:127]]
    rng = np.random.default_rng(11)
    for trial in range(40):
        n = 1 + trial % 3
        x = np.zeros((1, 128), np.uint16)
        pos = rng.choice(128, n, replace=False)
        x[0, pos] = bf16_bits(rng.standard_normal(n) * 10.0 ** rng.integers(-6, 6))
        out = oracle.quantize_act(x, None, 1)
        xf = bf16_to_f32(x)[0]
        amax = Fraction(float(np.abs(xf).max()))
        s = np.float32(out["sa"][0, 0])
        d = abs(Fraction(float(s)) - amax / 448)
        for nb in (np.nextafter(s, np.float32(np.inf)), np.nextafter(s, np.float32(0))):
            assert d <= abs(Fraction(float(nb)) - amax / 448)
        for i in range(128):
            y = np.float32(xf[i]) / s          # the fp32 quotient
            a = Fraction(abs(float(y)))
            sign = 0x80 if math.copysign(1.0, float(y)) < 0 else 0
            if a >= 448:
                want = 0x7E | sign
            else:
                best = min(range(127), key=lambda c: (abs(a - mags[c]), c % 2))
                want = best | sign
            assert out["xq"][0, i] == want, (trial, i, float(y))


# --------------------------------------------------------------------------
# permute
# --------------------------------------------------------------------------

@pytest.mark.parametrize("name", ["tiny", "kanana", "dsv3"])
def test_route_is_stable_bijection(oracle, name):
    cfg = W.CONFIGS[name]
    ids = W.route(cfg)
    r = oracle.route(ids, cfg.E)
    T, k = ids.shape
    assert r["bad"] == 0
    assert np.array_equal(r["counts"], np.bincount(ids.ravel(), minlength=cfg.E))
    assert r["offsets"][-1] == T * k
    tr = r["token_row"]
    assert np.array_equal(np.sort(tr), np.arange(T * k))          # bijection
    assert np.array_equal(r["row_token"][tr], np.repeat(np.arange(T), k))
    # rows of each expert in ascending (token, slot) order
    flat_e = ids.ravel()
    order = np.lexsort((np.arange(T * k), flat_e))                 # by expert, then (t, j)
    assert np.array_equal(tr[order], np.arange(T * k))
    if name == "dsv3":
        assert (r["counts"] == 0).sum() == 16


def test_route_single_expert_is_identity(oracle):
    ids = np.zeros((100, 1), np.int32)
    r = oracle.route(ids, 1)
    assert np.array_equal(r["token_row"], np.arange(100))
    assert np.array_equal(r["row_token"], np.arange(100))


def test_route_bad_ids_are_dropped_and_counted(oracle):
    ids = np.array([[0, 5], [-1, 1], [1, 0]], np.int32)
    r = oracle.route(ids, 2)
    assert r["bad"] == 2
    assert r["token_row"][1] == -1 and r["token_row"][2] == -1
    assert list(r["offsets"]) == [0, 2, 4]
    assert list(r["row_token"]) == [0, 2, 1, 2, -1, -1]


def test_quantize_then_permute_equals_permute_then_quantize(oracle):
    cfg = W.CONFIGS["tiny"]
    x = W.gen_x(cfg)
    ids = W.route(cfg)
    fused = oracle.quantize_act(x, ids, cfg.E)
    plain = oracle.quantize_act(x, None, cfg.E)
    rt = fused["row_token"]
    assert np.array_equal(fused["xq"], plain["xq"][rt])
    assert np.array_equal(fused["sa"], plain["sa"][:, rt])


def test_duplicate_ids_in_one_token_each_get_a_row(oracle):
    ids = np.array([[1, 1], [0, 1]], np.int32)
    x = rand_bf16((2, 128), 5)
    out = oracle.quantize_act(x, ids, 2)
    assert list(out["offsets"]) == [0, 1, 4]
    assert list(out["row_token"]) == [1, 0, 0, 1]
    assert np.array_equal(out["xq"][1], out["xq"][2])


# --------------------------------------------------------------------------
# column-wise (token axis) quantisation
# --------------------------------------------------------------------------

def test_colwise_equals_rowwise_of_transposed_padded_segments(oracle):
    rng = np.random.default_rng(21)
    counts = np.array([0, 1, 127, 128, 129, 300, 0, 5])
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    R, C = int(offsets[-1]), 256
    y = rand_bf16((R, C), 22)
    out = oracle.quantize_act_colwise(y, offsets)
    padoff = out["padoff"]
    assert list(np.diff(padoff)) == [int(math.ceil(c / 128) * 128) for c in counts]
    for e in range(len(counts)):
        seg = y[offsets[e]:offsets[e + 1]]                       # [Te, C]
        Tp = padoff[e + 1] - padoff[e]
        if Tp == 0:
            continue
        padded = np.zeros((Tp, C), np.uint16)
        padded[:seg.shape[0]] = seg
        rowq = oracle.quantize_act(np.ascontiguousarray(padded.T), None, 1)   # [C, Tp]
        got = out["xqT"][:, padoff[e]:padoff[e + 1]]
        assert np.array_equal(got, rowq["xq"])
        assert np.array_equal(out["sT"][padoff[e] // 128:padoff[e + 1] // 128], rowq["sa"])
        assert np.all(got[:, seg.shape[0]:] == 0)


def test_colwise_gather_equals_colwise_of_gathered(oracle):
    cfg = W.CONFIGS["tiny"]
    x = W.gen_x(cfg)
    ids = W.route(cfg)
    r = oracle.route(ids, cfg.E)
    a = oracle.quantize_act_colwise(x, r["offsets"], row_map=r["row_token"])
    xg = oracle._u16(x)[r["row_token"]]
    b = oracle.quantize_act_colwise(np.ascontiguousarray(xg), r["offsets"])
    for key in ("xqT", "sT", "padoff"):
        assert np.array_equal(a[key], b[key])


# --------------------------------------------------------------------------
# weights and transpose
# --------------------------------------------------------------------------

def test_weight_blocks_equal_rowwise_of_flattened_blocks(oracle):
    """A 128x128 block quantised as a block equals the same 16384 values
    quantised as one tile with the scale of the whole block: check it via the
    max-element invariant and the dequantisation bound per block."""
    w = rand_bf16((2, 256, 384), 31, 0.02)
    wq, sw = oracle.quantize_weight(w)
    wf = bf16_to_f32(w).astype(np.float64)
    for e in range(2):
        for nb in range(2):
            for kb in range(3):
                blk = wf[e, nb * 128:(nb + 1) * 128, kb * 128:(kb + 1) * 128]
                q = wq[e, nb * 128:(nb + 1) * 128, kb * 128:(kb + 1) * 128]
                s = float(sw[e, nb, kb])
                i = np.unravel_index(np.abs(blk).argmax(), blk.shape)
                assert q[i] & 0x7F == 0x7E
                assert np.all(q & 0x7F <= 0x7E)
                deq = dq(oracle, q) * s
                normal = np.abs(blk) / s >= 2.0 ** -6
                assert np.max(np.abs(deq - blk)[normal] / np.abs(blk)[normal]) <= 2.0 ** -4


def test_transpose_commutes_with_dequantisation_and_requantisation(oracle):
    w = rand_bf16((3, 256, 384), 41, 0.02)
    w[1, :128, :128] = 0                          # an all-zero block
    wq, sw = oracle.quantize_weight(w)
    wqT, swT = oracle.transpose_blockq(wq, sw)
    assert wqT.shape == (3, 384, 256) and swT.shape == (3, 3, 2)
    scale_full = np.repeat(np.repeat(sw, 128, 1), 128, 2).astype(np.float64)
    scale_fullT = np.repeat(np.repeat(swT, 128, 1), 128, 2).astype(np.float64)
    deq = dq(oracle, wq) * scale_full
    deqT = dq(oracle, wqT) * scale_fullT
    assert np.array_equal(deqT, deq.transpose(0, 2, 1))      # exact, square blocks
    # quantising the transposed bf16 weight gives the same bytes (square blocks)
    wq2, sw2 = oracle.quantize_weight(np.ascontiguousarray(w.transpose(0, 2, 1)))
    assert np.array_equal(wq2, wqT) and np.array_equal(sw2, swT)
    # transposing twice is the identity
    wqTT, swTT = oracle.transpose_blockq(wqT, swT)
    assert np.array_equal(wqTT, wq) and np.array_equal(swTT, sw)


# --------------------------------------------------------------------------
# GEMM references
# --------------------------------------------------------------------------

def _int_tile_operands(rng, rows, K):
    """bf16 operands whose every 1x128 tile / 128x128 block has amax 448 (so all
    scales are exactly 1) and whose other entries are small integers."""
    v = rng.integers(-6, 7, size=(rows, K)).astype(np.float64)
    v[:, ::128] = 448.0
    return bf16_bits(v), v


def test_gemm_unit_scales_small_integers_exact(oracle):
    rng = np.random.default_rng(51)
    E, N, K = 3, 256, 384
    counts = np.array([5, 0, 140])
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    M = int(offsets[-1])
    xa, va = _int_tile_operands(rng, M, K)
    wb, vb = _int_tile_operands(rng, E * N, K)
    act = oracle.quantize_act(xa, None, 1)
    wq, sw = oracle.quantize_weight(wb.reshape(E, N, K))
    assert np.all(act["sa"] == 1.0) and np.all(sw == 1.0)
    ref, bound = oracle.gemm_mgrouped_full(act["xq"], act["sa"], wq, sw, offsets)
    ia = va.astype(np.int64)
    ib = vb.astype(np.int64).reshape(E, N, K)
    for e in range(E):
        r0, r1 = offsets[e], offsets[e + 1]
        exact = ia[r0:r1] @ ib[e].T
        assert np.array_equal(ref[r0:r1], exact.astype(np.float64))
        assert np.array_equal(bound[r0:r1], (np.abs(ia[r0:r1]) @ np.abs(ib[e]).T).astype(np.float64))


def test_gemm_single_expert_equals_fp64_matmul_of_dequantised(oracle):
    rng = np.random.default_rng(61)
    M, N, K = 130, 256, 512
    x = rand_bf16((M, K), 62)
    w = rand_bf16((1, N, K), 63, 0.02)
    act = oracle.quantize_act(x, None, 1)
    wq, sw = oracle.quantize_weight(w)
    A = dq(oracle, act["xq"]) * np.repeat(act["sa"].T, 128, 1).astype(np.float64)
    B = dq(oracle, wq[0]) * np.repeat(np.repeat(sw[0], 128, 0), 128, 1).astype(np.float64)
    want = A @ B.T
    ref, bound = oracle.gemm_mgrouped_full(act["xq"], act["sa"], wq, sw,
                                           np.array([0, M], np.int32))
    assert np.all(np.abs(ref - want) <= 1e-12 * bound)
    assert np.allclose(bound, np.abs(A) @ np.abs(B).T, rtol=1e-12)
    # the quantised product approximates the bf16 product
    exact = bf16_to_f32(x).astype(np.float64) @ bf16_to_f32(w[0]).astype(np.float64).T
    assert np.linalg.norm(ref - exact) / np.linalg.norm(exact) < 0.05


def test_gemm_grouped_rows_use_their_own_expert(oracle):
    """Each segment of the grouped product equals a one-expert product of the
    same rows with that expert's weights alone; the empty segment is skipped."""
    E, N, K = 3, 128, 256
    offsets = np.array([0, 40, 40, 100], np.int32)
    x = rand_bf16((100, K), 72)
    w = rand_bf16((E, N, K), 73, 0.02)
    act = oracle.quantize_act(x, None, 1)
    wq, sw = oracle.quantize_weight(w)
    ref, _ = oracle.gemm_mgrouped_full(act["xq"], act["sa"], wq, sw, offsets)
    for e in (0, 2):
        r0, r1 = offsets[e], offsets[e + 1]
        sub = oracle.quantize_act(np.ascontiguousarray(x[r0:r1]), None, 1)
        one, _ = oracle.gemm_mgrouped_full(sub["xq"], sub["sa"], wq[e:e + 1], sw[e:e + 1],
                                           np.array([0, r1 - r0], np.int32))
        assert np.array_equal(ref[r0:r1], one)
    other, _ = oracle.gemm_mgrouped_full(act["xq"], act["sa"], wq[[2, 1, 0]], sw[[2, 1, 0]],
                                         offsets)
    assert not np.array_equal(ref[:40], other[:40])


def test_gemm_kgrouped_equals_per_expert_fp64_matmul(oracle):
    counts = np.array([3, 0, 200, 128])
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    R = int(offsets[-1])
    dy = rand_bf16((R, 256), 81)
    xx = rand_bf16((R, 384), 82)
    A = oracle.quantize_act_colwise(dy, offsets)
    B = oracle.quantize_act_colwise(xx, offsets)
    assert np.array_equal(A["padoff"], B["padoff"])
    padoff = A["padoff"]
    for e in range(len(counts)):
        m, n = np.meshgrid(np.arange(256), np.arange(384), indexing="ij")
        ref, bound = oracle.gemm_kgrouped_entries(A["xqT"], A["sT"], B["xqT"], B["sT"], padoff,
                                                  np.full(m.size, e), m.ravel(), n.ravel())
        ref = ref.reshape(256, 384)
        p0, p1 = padoff[e], padoff[e + 1]
        if p0 == p1:
            assert np.all(ref == 0)
            continue
        sa = np.repeat(A["sT"][p0 // 128:p1 // 128].T, 128, 1).astype(np.float64)
        sb = np.repeat(B["sT"][p0 // 128:p1 // 128].T, 128, 1).astype(np.float64)
        Ad = dq(oracle, A["xqT"][:, p0:p1]) * sa
        Bd = dq(oracle, B["xqT"][:, p0:p1]) * sb
        want = Ad @ Bd.T
        assert np.all(np.abs(ref - want) <= 1e-12 * bound.reshape(256, 384) + 1e-300)
        # and it approximates dY_e^T X_e of the bf16 inputs
        seg = slice(offsets[e], offsets[e + 1])
        exact = bf16_to_f32(dy[seg]).astype(np.float64).T @ bf16_to_f32(xx[seg]).astype(np.float64)
        assert np.linalg.norm(ref - exact) / np.linalg.norm(exact) < 0.05
