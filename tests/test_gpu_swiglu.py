"""GPU parity of the up-projection with the fused gated activation and 1x128
re-quantization (fg8_grouped_gemm_swiglu_quant) against the oracle.

The oracle takes the fp64 up-projection (gate half G, up half U), forms
h = silu(G) * U in fp64 and quantizes its fp32 rounding.  The kernel forms h
from its fp32 accumulators, so h differs by the GEMM's rounding and codes can
differ where h / s sits next to a rounding midpoint.  The checks:
  * every scale: |448 sh - amax(h_ref)| within the tile's largest error bound,
    where a GEMM entry may be off by 1e-3 * sum_k |a_k b_k| (the GEMM parity
    tolerance) and the fp32 activation by 1e-5 relative (fast exp and divide);
  * every code: |dq(hq) sh - h_ref| <= half an E4M3 step of h_ref / sh, in
    scaled units, plus that error bound;
  * at most 1e-3 of the codes differ from the oracle's own (only values
    within ~1e-6 of a rounding midpoint may; a scale that differs from the
    oracle's in its last bits moves no other code);
  * rows outside [0, offsets[E]) untouched.
"""

import numpy as np
import pytest
import torch

from fp8_fine_grained_permute_b200 import build as fbuild
from fp8_fine_grained_permute_b200 import fg8
from fp8_fine_grained_permute_b200 import workloads as W

pytestmark = pytest.mark.gpu

GEMM_TOL = 1e-3
ACT_REL = 1e-5
CODE_MISMATCH = 1e-3


@pytest.fixture(scope="module", autouse=True)
def _lib():
    fbuild.build()
    fg8.lib()
    torch.cuda.init()


def e4m3_half_step(x):
    """Half the spacing of E4M3 values around |x| (in code units)."""
    ax = np.maximum(np.abs(x), 2.0 ** -6)
    e = np.floor(np.log2(ax))
    return 0.5 * 2.0 ** (e - 3)


def check_swiglu(oracle, hq, sh, G, U, bG, bU, what=""):
    """hq [R, I] u8, sh [I/128, R] f32 from the GPU; G, U, bG, bU fp64 [R, I]."""
    R, I = G.shape
    h_ref, hq_ref, _ = oracle.swiglu_quantize(G, U)
    silu = G / (1.0 + np.exp(-np.clip(G, -700, 700)))
    dh = 1.1 * np.abs(U) * GEMM_TOL * bG + np.abs(silu) * GEMM_TOL * bU + ACT_REL * np.abs(h_ref)
    dq = oracle.e4m3_decode_table()
    s = sh.T.astype(np.float64)                        # [R, I/128]
    s_e = np.repeat(s, 128, axis=1)
    # scales
    amax = np.abs(h_ref).reshape(R, I // 128, 128).max(axis=2)
    dmax = dh.reshape(R, I // 128, 128).max(axis=2)
    err_s = np.abs(448.0 * s - amax)
    lim_s = dmax + 2.0 ** -22 * amax + 1e-30
    assert np.all(err_s <= lim_s), f"{what}: scale off by {np.max(err_s - lim_s)}"
    # codes
    deq = dq[hq].astype(np.float64) * s_e
    x = np.maximum(np.abs(h_ref), np.abs(deq)) / s_e
    lim = e4m3_half_step(x) * s_e * (1 + 1e-9) + 2.0 * dh + 1e-30
    err = np.abs(deq - h_ref)
    bad = err > lim
    assert not bad.any(), f"{what}: {bad.sum()} codes outside the bound, worst {np.max(err - lim)}"
    assert np.mean(hq != hq_ref) <= CODE_MISMATCH, f"{what}: {np.mean(hq != hq_ref)} codes differ"


class Operands:
    """Row-grouped operands for a [gate; up] weight of 2I rows per expert.
    Scales in [2^-11, 2^-7) put the gate values mostly in |g| ~ 0.1 .. 20, so
    silu is exercised on both of its tails."""

    def __init__(self, counts, I, K, seed, extra_rows=0):
        self.counts = np.asarray(counts)
        self.E = len(counts)
        self.offsets = np.concatenate([[0], np.cumsum(self.counts)]).astype(np.int32)
        self.M = int(self.offsets[-1]) + extra_rows
        self.I, self.K = I, K
        self.a = W.gen_e4m3_codes((self.M, K), seed, 1)
        self.sa = W.gen_scales((K // 128, self.M), seed, 2, lo_exp=-11, hi_exp=-7)
        self.b = W.gen_e4m3_codes((self.E, 2 * I, K), seed, 3)
        self.sb = W.gen_scales((self.E, 2 * I // 128, K // 128), seed, 4, lo_exp=-11, hi_exp=-7)

    def run(self, hq_fill=0x5A, sh_fill=-3.0):
        hq = torch.full((self.M, self.I), hq_fill, dtype=torch.uint8, device="cuda")
        sh = torch.full((self.I // 128, self.M), sh_fill, dtype=torch.float32, device="cuda")
        st = fg8.new_status()
        fg8.grouped_gemm_swiglu_quant(self.a.cuda(), self.sa.cuda(), self.b.cuda(), self.sb.cuda(),
                                      torch.from_numpy(self.offsets).cuda(), dev_status=st,
                                      hq=hq, sh=sh)
        torch.cuda.synchronize()
        assert st.item() == 0
        return hq.cpu().numpy(), sh.cpu().numpy()

    def reference(self, oracle):
        ref, bound = oracle.gemm_mgrouped_full(self.a.numpy(), self.sa.numpy(), self.b.numpy(),
                                               self.sb.numpy(), self.offsets)
        I = self.I
        return ref[:, :I], ref[:, I:], bound[:, :I], bound[:, I:]


@pytest.mark.parametrize("case", [
    # ragged tiles, empty experts, rows past offsets[E]
    dict(counts=[0, 1, 127, 128, 129, 300, 0, 5], I=256, K=512, seed=31, extra=16),
    # one K block (the exchange buffers alternate every tile), three column tiles
    dict(counts=[200, 57, 0, 384], I=384, K=128, seed=32, extra=0),
    # odd number of K blocks, single expert
    dict(counts=[515], I=128, K=384, seed=33, extra=3),
])
def test_swiglu_quant_full_with_canaries(oracle, case):
    ops = Operands(case["counts"], case["I"], case["K"], case["seed"], extra_rows=case["extra"])
    hq, sh = ops.run()
    used = int(ops.offsets[-1])
    G, U, bG, bU = ops.reference(oracle)
    check_swiglu(oracle, hq[:used], sh[:, :used], G[:used], U[:used], bG[:used], bU[:used],
                 f"case {case['seed']}")
    assert np.all(hq[used:] == 0x5A)
    assert np.all(sh[:, used:] == -3.0)


def test_swiglu_quant_exact_case_matches_library_cast():
    """Unit scales and small-integer codes, built so that every gate entry is
    at least 64: then silu(g) == g in fp32 (1 + exp(-64) rounds to 1), h = g u
    is an exact integer, and the fused result must equal, bit for bit, the
    1x128 quantization of the exact integer product done with torch's fp32
    division and float8_e4m3fn cast on the CPU."""
    rng = np.random.default_rng(34)
    counts = [130, 0, 126]
    E, I, K = len(counts), 256, 256
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    M = int(offsets[-1])
    ia = np.zeros((M, K), np.int64)
    ia[:, 0] = rng.choice([8, 16], size=M)
    ia[:, 1] = rng.integers(-3, 4, M)
    ib = np.zeros((E, 2 * I, K), np.int64)
    ib[:, :I, 0] = rng.choice([8, 12, 16, 24], size=(E, I))     # gate: column 0 only
    ib[:, I:, 0] = rng.integers(-6, 7, (E, I))
    ib[:, I:, 1] = rng.integers(-2, 3, (E, I))
    codes = {v: int(torch.tensor(float(v)).to(torch.float8_e4m3fn).view(torch.uint8))
             for v in range(-24, 25)}
    a = np.vectorize(codes.get)(ia).astype(np.uint8)
    b = np.vectorize(codes.get)(ib).astype(np.uint8)
    h = np.zeros((M, I), np.int64)
    for e in range(E):
        r0, r1 = offsets[e], offsets[e + 1]
        y = ia[r0:r1] @ ib[e].T
        assert np.all(y[:, :I] >= 64)
        h[r0:r1] = y[:, :I] * y[:, I:]
    assert np.abs(h).max() < 2 ** 24
    ht = torch.from_numpy(h).to(torch.float32).view(M, I // 128, 128)
    amax = ht.abs().amax(dim=2)
    s = torch.where(amax == 0, torch.ones_like(amax), amax / 448.0)
    want_q = (ht / s[:, :, None]).view(M, I).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    want_s = s.T.contiguous().numpy()
    sa = torch.ones((K // 128, M), dtype=torch.float32, device="cuda")
    sb = torch.ones((E, 2 * I // 128, K // 128), dtype=torch.float32, device="cuda")
    st = fg8.new_status()
    hq, sh = fg8.grouped_gemm_swiglu_quant(torch.from_numpy(a).cuda(), sa,
                                           torch.from_numpy(b).cuda(), sb,
                                           torch.from_numpy(offsets).cuda(), dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    assert np.array_equal(sh.cpu().numpy().view(np.uint32), want_s.view(np.uint32))
    assert np.array_equal(hq.cpu().numpy(), want_q)


@pytest.mark.parametrize("name", ["kanana", "dsv3"])
def test_swiglu_quant_full_size_sampled_rows(oracle, name):
    """The full up-projection of a layer (routed rows of every expert), checked
    on sampled rows: their gate and up blocks are regenerated on the host."""
    cfg = W.CONFIGS[name]
    offsets = oracle.route(W.route(cfg), cfg.E)["offsets"]
    E, I, K = cfg.E, cfg.inter, cfg.hidden
    M = int(offsets[-1])
    seed = cfg.seed + 777
    a = W.gen_e4m3_codes((M, K), seed, 1, device="cuda")
    sa = W.gen_scales((K // 128 * M,), seed, 2, device="cuda", lo_exp=-11, hi_exp=-7).view(
        K // 128, M)
    b = W.gen_e4m3_codes((E, 2 * I, K), seed, 3, device="cuda")
    NB, KB = 2 * I // 128, K // 128
    sb = W.gen_scales((E * NB * KB,), seed, 4, device="cuda", lo_exp=-11, hi_exp=-7).view(
        E, NB, KB)
    st = fg8.new_status()
    hq, sh = fg8.grouped_gemm_swiglu_quant(a, sa, b, sb, torch.from_numpy(offsets).cuda(),
                                           dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    del a, b
    rng = np.random.default_rng(35)
    rows = sorted(set([0, M - 1, min(M - 1, int(offsets[E // 2]))] + [int(r) for r in rng.integers(0, M, 5)]))
    sa_all = sa.cpu()
    for r in rows:
        e = int(np.searchsorted(offsets, r, side="right") - 1)
        blocks = sorted(set([I // 128 - 1] + [int(x) for x in rng.integers(0, I // 128, 1)]))
        a_row = W.gen_e4m3_codes((1, K), seed, 1, index_offset=r * K).numpy()
        sa_row = sa_all[:, r:r + 1].contiguous().numpy()
        sb_e = W.gen_scales((NB * KB,), seed, 4, index_offset=e * NB * KB, lo_exp=-11,
                            hi_exp=-7).view(NB, KB)
        for c in blocks:
            rows_b = [c, I // 128 + c]     # gate block, up block
            b_rows = np.concatenate([
                W.gen_e4m3_codes((128, K), seed, 3, index_offset=(e * 2 * I + nb * 128) * K).numpy()
                for nb in rows_b])[None]
            sb_sub = sb_e[rows_b].contiguous().numpy()[None]
            ref, bound = oracle.gemm_mgrouped_full(a_row, sa_row, b_rows, sb_sub,
                                                   np.array([0, 1], np.int32))
            got_q = hq[r, 128 * c:128 * (c + 1)].cpu().numpy()[None]
            got_s = sh[c:c + 1, r:r + 1].cpu().numpy()
            check_swiglu(oracle, got_q, got_s, ref[:, :128], ref[:, 128:], bound[:, :128],
                         bound[:, 128:], f"{name} row {r} block {c}")


def test_swiglu_quant_rejects_bad_shapes():
    a = torch.zeros((128, 256), dtype=torch.uint8, device="cuda")
    sa = torch.ones((2, 128), device="cuda")
    b = torch.zeros((1, 192, 256), dtype=torch.uint8, device="cuda")   # I = 96
    sb = torch.ones((1, 2, 2), device="cuda")
    off = torch.tensor([0, 128], dtype=torch.int32, device="cuda")
    hq = torch.empty((128, 96), dtype=torch.uint8, device="cuda")
    sh = torch.empty((1, 128), device="cuda")
    with pytest.raises(fg8.FG8Error) as ei:
        fg8.fg8_grouped_gemm_swiglu_quant(a, sa, b, sb, off, 128, 96, 256, 1, hq, sh, None)
    assert ei.value.status == fg8.FG8_ERR_INVALID_ARG
