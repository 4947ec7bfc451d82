"""GPU parity of the bandwidth kernels against the CPU oracle, bit for bit:
1x128 activation quantization with the permute (and its identity and
column-wise modes), 128x128 weight quantization, and the block transpose.

Inputs come from the seeded generators; expected values from `oracle/` only.
Small configurations are compared in full; the DeepSeek-V3-shaped workload is
run at full size in the launch configuration the benchmark times and checked
in full where the oracle is fast enough, else on sampled blocks/experts."""

import numpy as np
import pytest
import torch

from fp8_fine_grained_permute_b200 import build as fbuild
from fp8_fine_grained_permute_b200 import fg8
from fp8_fine_grained_permute_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    fbuild.build()
    fg8.lib()
    torch.cuda.init()


def u16(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def bf16_from_bits(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(bits.astype(np.uint16).view(np.int16)).view(torch.bfloat16)


# --------------------------------------------------------------------------
# weight blocks
# --------------------------------------------------------------------------

def edge_weight(E=2, N=256, K=384, seed=5):
    """bf16 weights whose blocks span the whole bf16 range, plus special blocks."""
    rng = np.random.default_rng(seed)
    v = rng.standard_normal((E, N, K)).astype(np.float32)
    exps = rng.integers(-130, 125, size=(E, N // 128, K // 128))
    v *= np.exp2(np.repeat(np.repeat(exps, 128, 1), 128, 2)).astype(np.float32)
    t = torch.from_numpy(v).to(torch.bfloat16)
    t[0, :128, :128] = 0.0                                   # zero block -> s = 1
    t[0, :128, 128:256] = -0.0                               # -0 block -> 0x80 codes
    t[1, 128:, :128] = 0.0
    t[1, 128 + 5, 77] = 448.0 * 2.0 ** -20                   # power-of-two amax
    t[1, 128:, 128:256].view(torch.int16)[:] = torch.arange(1, 1 + 128 * 128, dtype=torch.int32)\
        .remainder(0x7F80).to(torch.int16).view(128, 128)      # every small bf16 pattern
    return t


@pytest.mark.parametrize("shape", ["tiny", "dense4096", "edge"])
def test_quantize_weight_bit_exact(oracle, shape):
    if shape == "edge":
        w = edge_weight()
    else:
        cfg = W.CONFIGS[shape]
        w = W.gen_w_up(cfg)
    wq, sw = fg8.quantize_weight(w.cuda())
    torch.cuda.synchronize()
    owq, osw = oracle.quantize_weight(w)
    assert np.array_equal(wq.cpu().numpy(), owq)
    assert np.array_equal(sw.cpu().numpy().view(np.uint32), osw.view(np.uint32))


def test_quantize_weight_kanana_sampled_experts(oracle):
    cfg = W.CONFIGS["kanana"]
    w = W.gen_w_up(cfg, device="cuda")
    wq, sw = fg8.quantize_weight(w)
    torch.cuda.synchronize()
    for e in (0, 17, 63):
        ow = W.gen_w_up(cfg, experts=[e])
        owq, osw = oracle.quantize_weight(ow)
        assert np.array_equal(wq[e].cpu().numpy(), owq[0])
        assert np.array_equal(sw[e].cpu().numpy(), osw[0])


def test_quantize_weight_dsv3_full_size_sampled_blocks(oracle):
    """Both DeepSeek-V3-shaped weights at full size, 48 sampled blocks each."""
    cfg = W.CONFIGS["dsv3"]
    rng = np.random.default_rng(99)
    for name, (N, K), sid in (("up", (cfg.n_up, cfg.hidden), W.SID_W_UP),
                              ("down", (cfg.hidden, cfg.inter), W.SID_W_DOWN)):
        w = W.gen_normal_bf16((cfg.E, N, K), W.SIGMA_W, cfg.seed, sid, device="cuda")
        wq, sw = fg8.quantize_weight(w)
        torch.cuda.synchronize()
        del w
        blocks = [(0, 0, 0), (cfg.E - 1, N // 128 - 1, K // 128 - 1)] + [
            (int(rng.integers(cfg.E)), int(rng.integers(N // 128)), int(rng.integers(K // 128)))
            for _ in range(46)]
        for e, nb, kb in blocks:
            rows = np.arange(nb * 128, nb * 128 + 128)
            cols = np.arange(kb * 128, kb * 128 + 128)
            idx = (e * N + rows[:, None]) * K + cols[None, :]
            blk = W.gen_normal_bf16_at(torch.from_numpy(idx.ravel()), W.SIGMA_W, cfg.seed, sid)
            owq, osw = oracle.quantize_weight(blk.view(1, 128, 128))
            got = wq[e, nb * 128:(nb + 1) * 128, kb * 128:(kb + 1) * 128].cpu().numpy()
            assert np.array_equal(got, owq[0]), (name, e, nb, kb)
            assert sw[e, nb, kb].item() == osw[0, 0, 0], (name, e, nb, kb)
        del wq, sw
        torch.cuda.empty_cache()


def test_quantize_fast_path_exhaustive_bf16_by_scales(oracle):
    """Every finite bf16 value x against ~400 tile maxima spanning the bf16 range
    (including subnormal maxima): each row is a 1x128 tile holding its amax and
    127 of the values with |x| <= amax, quantized by the GPU row kernel and by
    the oracle.  Exercises the reciprocal fast path and every fallback."""
    allbits = np.arange(0x10000, dtype=np.uint32)
    vals = (allbits << 16).view(np.float32)
    finite = np.isfinite(vals)
    bits = allbits[finite].astype(np.uint16)
    mags = np.abs((bits.astype(np.uint32) << 16).view(np.float32))
    amax_bits = np.unique(np.concatenate([
        np.linspace(1, 0x7F7F, 300).astype(np.uint16),
        np.random.default_rng(12).integers(1, 0x7F80, 100).astype(np.uint16),
        np.array([0x0001, 0x0002, 0x007F, 0x0080, 0x3F80, 0x43E0, 0x7F7F], np.uint16)]))
    rows = []
    for ab in amax_bits:
        amax = float((np.array([ab], np.uint32) << 16).view(np.float32)[0])
        cand = bits[mags <= amax]
        n = (cand.size + 126) // 127
        pad = np.resize(cand, n * 127).reshape(n, 127)
        rows.append(np.concatenate([np.full((n, 1), ab, np.uint16), pad], axis=1))
    x = np.concatenate(rows)
    xq, sa = fg8.quantize_act_rows(bf16_from_bits(x).cuda())
    torch.cuda.synchronize()
    ref = oracle.quantize_act(x, None, 1)
    got = xq.cpu().numpy()
    bad = np.argwhere(got != ref["xq"])
    assert bad.size == 0, f"{len(bad)} mismatches, first {bad[:5]}"
    assert np.array_equal(sa.cpu().numpy(), ref["sa"])


# --------------------------------------------------------------------------
# activation permute + quantize
# --------------------------------------------------------------------------

def _check_permute(oracle, x_cpu, ids, E, out):
    ref = oracle.route(ids, E)
    assert np.array_equal(out["offsets"].cpu().numpy(), ref["offsets"])
    assert np.array_equal(out["token_row"].cpu().numpy(), ref["token_row"])
    assert np.array_equal(out["row_token"].cpu().numpy(), ref["row_token"])
    # codes and scales: the oracle's row-wise quantization of each token row,
    # placed at every row the token is routed to (1x128 tiles never span
    # tokens, so quantize-then-permute equals the fused result; pinned in the
    # oracle tests)
    q = oracle.quantize_act(x_cpu, None, 1)
    rt = ref["row_token"]
    assert np.array_equal(out["xq"].cpu().numpy(), q["xq"][rt])
    assert np.array_equal(out["sa"].cpu().numpy(), q["sa"][:, rt])
    assert out["status"].item() == 0


def test_quantize_act_tiny_matches_fused_oracle(oracle):
    cfg = W.CONFIGS["tiny"]
    x = W.gen_x(cfg)
    ids = W.route(cfg)
    out = fg8.quantize_act(x.cuda(), torch.from_numpy(ids).cuda(), cfg.E)
    torch.cuda.synchronize()
    ref = oracle.quantize_act(x, ids, cfg.E)       # the fused oracle itself
    for key in ("xq", "sa", "row_token", "token_row", "offsets"):
        assert np.array_equal(out[key].cpu().numpy(), ref[key]), key
    assert out["status"].item() == 0


@pytest.mark.parametrize("name", ["kanana", "dsv3"])
def test_quantize_act_permute_full(oracle, name):
    cfg = W.CONFIGS[name]
    x = W.gen_x(cfg)
    ids = W.route(cfg)
    out = fg8.quantize_act(x.cuda(), torch.from_numpy(ids).cuda(), cfg.E)
    torch.cuda.synchronize()
    _check_permute(oracle, x, ids, cfg.E, out)


def test_quantize_act_ragged_and_degenerate(oracle):
    rng = np.random.default_rng(3)
    # T not a multiple of anything, K = 128 (single tile per row), experts with 0 rows
    T, K, E, k = 301, 384, 9, 3
    x = W.gen_normal_bf16((T, K), 1.0, 7, 1)
    ids = np.stack([rng.choice([0, 2, 3, 8], size=k, replace=False) for _ in range(T)]).astype(np.int32)
    out = fg8.quantize_act(x.cuda(), torch.from_numpy(ids).cuda(), E)
    torch.cuda.synchronize()
    _check_permute(oracle, x, ids, E, out)
    # one token
    x1 = W.gen_normal_bf16((1, 128), 1.0, 7, 2)
    ids1 = np.array([[2, 0]], np.int32)
    out1 = fg8.quantize_act(x1.cuda(), torch.from_numpy(ids1).cuda(), 4)
    torch.cuda.synchronize()
    _check_permute(oracle, x1, ids1, 4, out1)
    # duplicate ids inside a token, single expert
    x2 = W.gen_normal_bf16((50, 256), 1.0, 7, 3)
    ids2 = np.zeros((50, 2), np.int32)
    out2 = fg8.quantize_act(x2.cuda(), torch.from_numpy(ids2).cuda(), 1)
    torch.cuda.synchronize()
    _check_permute(oracle, x2, ids2, 1, out2)


def test_quantize_act_bad_expert_id_reports_and_skips(oracle):
    T, K, E = 40, 256, 4
    x = W.gen_normal_bf16((T, K), 1.0, 8, 1)
    ids = np.tile(np.array([[0, 1]], np.int32), (T, 1))
    ids[7, 1] = 4
    ids[9, 0] = -3
    out = fg8.quantize_act(x.cuda(), torch.from_numpy(ids).cuda(), E)
    torch.cuda.synchronize()
    assert out["status"].item() == fg8.FG8_ERR_BAD_EXPERT_ID
    ref = oracle.route(ids, E)
    assert np.array_equal(out["offsets"].cpu().numpy(), ref["offsets"])
    assert np.array_equal(out["token_row"].cpu().numpy(), ref["token_row"])
    nvalid = ref["offsets"][-1]
    assert np.array_equal(out["row_token"].cpu().numpy()[:nvalid], ref["row_token"][:nvalid])


def test_quantize_act_empty_input():
    x = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    ids = torch.empty((0, 2), dtype=torch.int32, device="cuda")
    out = fg8.quantize_act(x, ids, 3)
    torch.cuda.synchronize()
    assert out["offsets"].cpu().tolist() == [0, 0, 0, 0]


def test_quantize_rows_dsv3_down_input_full(oracle):
    """Identity mode on the down-projection input rows (already in expert order)."""
    cfg = W.CONFIGS["dsv3"]
    h = W.gen_h(cfg)
    xq, sa = fg8.quantize_act_rows(h.cuda())
    torch.cuda.synchronize()
    ref = oracle.quantize_act(h, None, 1)
    assert np.array_equal(xq.cpu().numpy(), ref["xq"])
    assert np.array_equal(sa.cpu().numpy(), ref["sa"])


# --------------------------------------------------------------------------
# column-wise (weight-gradient operands)
# --------------------------------------------------------------------------

def test_colwise_ragged_full(oracle):
    counts = np.array([0, 1, 127, 128, 129, 300, 0, 5, 256])
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    R, C = int(offsets[-1]), 384
    y = W.gen_grad_bf16((R, C), 11, 5)
    xqT, saT, padoff = fg8.quantize_act_colwise(y.cuda(), torch.from_numpy(offsets).cuda())
    torch.cuda.synchronize()
    ref = oracle.quantize_act_colwise(y, offsets)
    P = int(ref["padoff"][-1])
    assert np.array_equal(padoff.cpu().numpy(), ref["padoff"])
    assert np.array_equal(xqT.cpu().numpy()[:, :P], ref["xqT"][:, :P])
    assert np.array_equal(saT.cpu().numpy()[:P // 128], ref["sT"][:P // 128])


def test_colwise_gather_tiny_full(oracle):
    cfg = W.CONFIGS["tiny"]
    x = W.gen_x(cfg)
    ids = W.route(cfg)
    r = oracle.route(ids, cfg.E)
    xqT, saT, padoff = fg8.quantize_act_colwise(
        x.cuda(), torch.from_numpy(r["offsets"]).cuda(), k=cfg.k,
        row_token=torch.from_numpy(r["row_token"]).cuda())
    torch.cuda.synchronize()
    ref = oracle.quantize_act_colwise(x, r["offsets"], row_map=r["row_token"])
    P = int(ref["padoff"][-1])
    assert np.array_equal(padoff.cpu().numpy(), ref["padoff"])
    assert np.array_equal(xqT.cpu().numpy()[:, :P], ref["xqT"][:, :P])
    assert np.array_equal(saT.cpu().numpy()[:P // 128], ref["sT"][:P // 128])


def test_colwise_dsv3_full_size_sampled_experts(oracle):
    """dY [R, 4096] and X gathered through row_token [R, 7168] at full size;
    8 experts (largest, smallest non-empty, random) compared against the oracle
    run on those experts' rows alone."""
    cfg = W.CONFIGS["dsv3"]
    ids = W.route(cfg)
    r = oracle.route(ids, cfg.E)
    offs = r["offsets"]
    counts = np.diff(offs)
    nz = np.nonzero(counts)[0]
    rng = np.random.default_rng(5)
    pick = sorted(set([int(nz[np.argmax(counts[nz])]), int(nz[np.argmin(counts[nz])])] +
                      [int(e) for e in rng.choice(nz, 6, replace=False)]))
    offs_d = torch.from_numpy(offs).cuda()
    dy = W.gen_dy(cfg, device="cuda")
    dT, dS, dpad = fg8.quantize_act_colwise(dy, offs_d)
    x = W.gen_x(cfg, device="cuda")
    xT, xS, xpad = fg8.quantize_act_colwise(x, offs_d, k=cfg.k,
                                            row_token=torch.from_numpy(r["row_token"]).cuda())
    torch.cuda.synchronize()
    x_cpu = W.gen_x(cfg)
    padoff = dpad.cpu().numpy()
    assert np.array_equal(padoff, xpad.cpu().numpy())
    assert np.array_equal(np.diff(padoff), (counts + 127) // 128 * 128)
    for e in pick:
        o0, o1 = int(offs[e]), int(offs[e + 1])
        p0, p1 = int(padoff[e]), int(padoff[e + 1])
        sub_off = np.array([0, o1 - o0], np.int32)
        dref = oracle.quantize_act_colwise(W.gen_dy(cfg, row0=o0, rows=o1 - o0), sub_off)
        assert np.array_equal(dT[:, p0:p1].cpu().numpy(), dref["xqT"][:, :p1 - p0]), e
        assert np.array_equal(dS[p0 // 128:p1 // 128].cpu().numpy(), dref["sT"][:(p1 - p0) // 128]), e
        xg = np.ascontiguousarray(u16(x_cpu)[r["row_token"][o0:o1]])
        xref = oracle.quantize_act_colwise(xg, sub_off)
        assert np.array_equal(xT[:, p0:p1].cpu().numpy(), xref["xqT"][:, :p1 - p0]), e
        assert np.array_equal(xS[p0 // 128:p1 // 128].cpu().numpy(), xref["sT"][:(p1 - p0) // 128]), e


# --------------------------------------------------------------------------
# transpose of block-quantized weights
# --------------------------------------------------------------------------

def test_transpose_blockq_matches_oracle_small(oracle):
    cfg = W.CONFIGS["kanana"]
    w = W.gen_w_down(cfg, experts=[0, 5, 9])                  # [3, 2048, 768]
    owq, osw = oracle.quantize_weight(w)
    wqT, swT = fg8.transpose_blockq(torch.from_numpy(owq).cuda(), torch.from_numpy(osw).cuda())
    torch.cuda.synchronize()
    rwqT, rswT = oracle.transpose_blockq(owq, osw)
    assert np.array_equal(wqT.cpu().numpy(), rwqT)
    assert np.array_equal(swT.cpu().numpy(), rswT)


def test_transpose_blockq_dsv3_full_size_sampled(oracle):
    """All 256 experts of the up-projection shape [256, 4096, 7168] of random
    bytes and scales; 48 sampled blocks (and the whole scale grid) checked."""
    cfg = W.CONFIGS["dsv3"]
    E, N, K = cfg.E, cfg.n_up, cfg.hidden
    wq = W.gen_bytes((E, N, K), cfg.seed, 40, device="cuda")
    sw = W.gen_scales((E, N // 128, K // 128), cfg.seed, 41, device="cuda")
    wqT, swT = fg8.transpose_blockq(wq, sw)
    torch.cuda.synchronize()
    del wq
    osw = W.gen_scales((E, N // 128, K // 128), cfg.seed, 41)
    assert np.array_equal(swT.cpu().numpy(), osw.numpy().transpose(0, 2, 1))
    rng = np.random.default_rng(4)
    blocks = [(0, 0, 0), (E - 1, N // 128 - 1, K // 128 - 1)] + [
        (int(rng.integers(E)), int(rng.integers(N // 128)), int(rng.integers(K // 128)))
        for _ in range(46)]
    for e, nb, kb in blocks:
        rows = np.arange(nb * 128, nb * 128 + 128)
        idx = (e * N + rows[:, None]) * K + kb * 128 + np.arange(128)[None, :]
        blk = W.gen_bytes_at(torch.from_numpy(idx.ravel()), cfg.seed, 40)
        src = np.ascontiguousarray(blk.numpy().reshape(1, 128, 128))
        rT, _ = oracle.transpose_blockq(src, np.ones((1, 1, 1), np.float32))
        got = wqT[e, kb * 128:(kb + 1) * 128, nb * 128:(nb + 1) * 128].cpu().numpy()
        assert np.array_equal(got, rT[0]), (e, nb, kb)


def test_quantize_rows_ragged_row_count(oracle):
    """Identity mode with a row count that is not a multiple of the 128-row
    boxes (the last box reads past the end as zeros) and three column tiles."""
    x = W.gen_normal_bf16((300, 384), 1.0, 41, 1)
    xq, sa = fg8.quantize_act_rows(x.cuda())
    torch.cuda.synchronize()
    ref = oracle.quantize_act(x, None, 1)
    assert np.array_equal(xq.cpu().numpy(), ref["xq"])
    assert np.array_equal(sa.cpu().numpy(), ref["sa"])


def test_quantize_weight_reports_ok_status(oracle):
    """With a status word, a normal launch leaves it at FG8_OK."""
    w = W.gen_normal_bf16((3, 256, 384), 0.02, 43, 1)
    st = fg8.new_status()
    wq, sw = fg8.quantize_weight(w.cuda(), status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    rwq, rsw = oracle.quantize_weight(w)
    assert np.array_equal(wq.cpu().numpy(), rwq)
    assert np.array_equal(sw.cpu().numpy(), rsw)


@pytest.mark.parametrize("shape", [(3, 256, 384), (2, 512, 128)])
def test_quantize_weight_transposed_matches_oracle(oracle, shape):
    """The fused quantize + block transpose: wq, sw as fg8_quantize_weight,
    wqT, swT as the oracle's transpose of the oracle's quantization."""
    w = W.gen_normal_bf16(shape, 0.02, 47, 1)
    st = fg8.new_status()
    wq, sw, wqT, swT = fg8.quantize_weight_transposed(w.cuda(), status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    rwq, rsw = oracle.quantize_weight(w)
    rwqT, rswT = oracle.transpose_blockq(rwq, rsw)
    assert np.array_equal(wq.cpu().numpy(), rwq)
    assert np.array_equal(sw.cpu().numpy(), rsw)
    assert np.array_equal(wqT.cpu().numpy(), rwqT)
    assert np.array_equal(swT.cpu().numpy(), rswT)


def test_quantize_weight_transposed_dsv3_up_equals_separate_kernels():
    """At the DeepSeek-V3 up-projection size the fused kernel's transposed copy
    equals fg8_transpose_blockq applied to its forward copy, byte for byte."""
    cfg = W.CONFIGS["dsv3"]
    w = W.gen_w_up(cfg, "cuda")
    wq, sw, wqT, swT = fg8.quantize_weight_transposed(w)
    wq2, sw2 = fg8.quantize_weight(w)
    assert torch.equal(wq, wq2) and torch.equal(sw, sw2)
    del w, wq2, sw2
    wqT2, swT2 = fg8.transpose_blockq(wq, sw)
    torch.cuda.synchronize()
    assert torch.equal(wqT, wqT2) and torch.equal(swT, swT2)


# --------------------------------------------------------------------------
# groups whose fast path fails: exact rounding midpoints and subnormal scales
# --------------------------------------------------------------------------

def midpoint_values(shape, seed):
    """bf16 values that are exact midpoints between two neighbouring E4M3 codes
    (normal and subnormal ones), random signs: with a tile maximum of 448 the
    scale is 1 and every such value's quotient is a tie, so both brackets of
    the fast path disagree for every value of the tile."""
    rng = np.random.default_rng(seed)
    j = rng.integers(0, 8, size=shape)
    e = rng.integers(-6, 8, size=shape)                     # E4M3 normal binades below 448
    normal = (1.0 + (2 * j + 1) / 16.0) * np.exp2(e)
    sub = (2 * rng.integers(0, 8, size=shape) + 1) * 2.0 ** -10   # between subnormal codes
    v = np.where(rng.random(shape) < 0.1, sub, normal)
    v = np.where(v >= 448.0, 416.0 + 16.0, v)               # 432: the midpoint below 448
    v *= np.where(rng.random(shape) < 0.5, -1.0, 1.0)
    return torch.from_numpy(v.astype(np.float32)).to(torch.bfloat16)


def test_midpoint_values_are_bf16_ties():
    v = midpoint_values((4096,), 3).float().abs().numpy()
    assert np.all(v <= 432.0)
    codes = np.array([float(torch.tensor(c, dtype=torch.uint8).view(torch.float8_e4m3fn).float())
                      for c in range(0x7F)], dtype=np.float64)
    mids = (codes[:-1] + codes[1:]) / 2
    assert np.isin(v, mids).all()


def test_quantize_rows_all_ties_and_subnormal_scales(oracle):
    """Row tiles whose every value needs the exact path (ties at scale 1, and
    tiles with a subnormal scale): more failed groups per warp than its
    shared redo list holds."""
    x = midpoint_values((256, 512), 21)
    x[:, ::128] = 448.0                                     # every tile's maximum
    x[192:, :] = torch.from_numpy(np.full((64, 512), 3, np.int16)).view(torch.bfloat16)
    x[192:, 5] = torch.tensor(0x8007 - 0x10000, dtype=torch.int16).view(torch.bfloat16)   # -subnormal
    xq, sa = fg8.quantize_act_rows(x.cuda())
    torch.cuda.synchronize()
    ref = oracle.quantize_act(u16(x), None, 1)
    assert np.array_equal(xq.cpu().numpy(), ref["xq"])
    assert np.array_equal(sa.cpu().numpy(), ref["sa"])


def test_colwise_all_ties_and_subnormal_scales(oracle):
    counts = np.array([200, 300, 140])
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    R, C = int(offsets[-1]), 384
    y = midpoint_values((R, C), 22)
    for e in range(2):                                      # experts 0, 1: ties at scale 1
        for t0 in range(int(offsets[e]), int(offsets[e + 1]), 128):
            y[t0, :] = 448.0
    tiny = np.full((int(counts[2]), C), 2, np.int16)        # expert 2: bf16 subnormals
    tiny[::7] = 0x8005 - 0x10000                            # negative subnormals
    y[int(offsets[2]):] = torch.from_numpy(tiny).view(torch.bfloat16)
    xqT, saT, padoff = fg8.quantize_act_colwise(y.cuda(), torch.from_numpy(offsets).cuda())
    torch.cuda.synchronize()
    ref = oracle.quantize_act_colwise(y, offsets)
    P = int(ref["padoff"][-1])
    assert np.array_equal(padoff.cpu().numpy(), ref["padoff"])
    assert np.array_equal(xqT.cpu().numpy()[:, :P], ref["xqT"][:, :P])
    assert np.array_equal(saT.cpu().numpy()[:P // 128], ref["sT"][:P // 128])


@pytest.mark.parametrize("transposed", [False, True])
def test_quantize_weight_all_ties_and_subnormal_scales(oracle, transposed):
    w = midpoint_values((2, 256, 384), 23)
    w[:, ::128, ::128] = 448.0                              # every block's maximum
    tiny = np.full((128, 128), 1, np.int16)
    tiny[::3, ::5] = 0x8006 - 0x10000                       # negative subnormals
    w[1, 128:, 256:] = torch.from_numpy(tiny).view(torch.bfloat16)   # subnormal scale
    rwq, rsw = oracle.quantize_weight(w)
    if transposed:
        wq, sw, wqT, swT = fg8.quantize_weight_transposed(w.cuda())
        torch.cuda.synchronize()
        rwqT, rswT = oracle.transpose_blockq(rwq, rsw)
        assert np.array_equal(wqT.cpu().numpy(), rwqT)
        assert np.array_equal(swT.cpu().numpy(), rswT)
    else:
        wq, sw = fg8.quantize_weight(w.cuda())
        torch.cuda.synchronize()
    assert np.array_equal(wq.cpu().numpy(), rwq)
    assert np.array_equal(sw.cpu().numpy().view(np.uint32), rsw.view(np.uint32))
