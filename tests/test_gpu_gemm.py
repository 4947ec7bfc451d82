"""GPU parity of the grouped FP8 GEMM (tcgen05) against the oracle's fp64
reference: per element |err| <= 1e-3 * sum_k |a_k b_k| and relative Frobenius
error <= 1e-4 on the fp32 output; the bf16 output must be the round-to-nearest-
even conversion of the fp32 output, bit for bit.

Operands are E4M3 codes and fp32 scales drawn directly by the seeded
generators (independent of the quantizers), except in the end-to-end test,
where both sides quantize the same bf16 inputs with their own code."""

import numpy as np
import pytest
import torch

from fp8_fine_grained_permute_b200 import build as fbuild
from fp8_fine_grained_permute_b200 import fg8
from fp8_fine_grained_permute_b200 import workloads as W

pytestmark = pytest.mark.gpu

ELEM_TOL = 1e-3
FRO_TOL = 1e-4


@pytest.fixture(scope="module", autouse=True)
def _lib():
    fbuild.build()
    fg8.lib()
    torch.cuda.init()


def check(got, ref, bound, what=""):
    got = np.asarray(got, np.float64)
    err = np.abs(got - ref)
    worst = np.max(err - ELEM_TOL * bound) if err.size else 0
    assert np.all(err <= ELEM_TOL * bound + 1e-30), f"{what}: element bound exceeded by {worst}"
    nref = np.linalg.norm(ref)
    if nref > 0:
        fro = np.linalg.norm(got - ref) / nref
        assert fro <= FRO_TOL, f"{what}: relative Frobenius {fro}"


def bf16_of(t32: torch.Tensor) -> np.ndarray:
    return t32.to(torch.bfloat16).view(torch.int16).cpu().numpy()


class Operands:
    """Row-grouped operands drawn from the generators."""

    def __init__(self, counts, N, K, seed, extra_rows=0, lo_exp=-12, hi_exp=0):
        self.counts = np.asarray(counts)
        self.E = len(counts)
        self.offsets = np.concatenate([[0], np.cumsum(self.counts)]).astype(np.int32)
        self.M = int(self.offsets[-1]) + extra_rows
        self.N, self.K = N, K
        self.seed = seed
        self.a = W.gen_e4m3_codes((self.M, K), seed, 1)
        self.sa = W.gen_scales((K // 128, self.M), seed, 2, lo_exp=lo_exp, hi_exp=hi_exp)
        self.b = W.gen_e4m3_codes((self.E, N, K), seed, 3)
        self.sb = W.gen_scales((self.E, N // 128, K // 128), seed, 4, lo_exp=lo_exp, hi_exp=hi_exp)

    def gpu(self):
        return [t.cuda() for t in (self.a, self.sa, self.b, self.sb)] + \
            [torch.from_numpy(self.offsets).cuda()]


def run_m(ops_gpu, out_dtype, M_alloc=None, fill=None):
    a, sa, b, sb, off = ops_gpu
    M, N = a.shape[0], b.shape[1]
    dt = torch.float32 if out_dtype == fg8.FG8_OUT_F32 else torch.bfloat16
    out = torch.empty((M, N), dtype=dt, device="cuda")
    if fill is not None:
        out.view(torch.int16 if dt == torch.bfloat16 else torch.int32).fill_(fill)
    st = fg8.new_status()
    fg8.grouped_gemm(a, sa, b, sb, off, out_dtype=out_dtype, out=out, dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    return out


def test_gemm_ragged_experts_full_with_canaries(oracle):
    """Experts of 0, 1, 127, 128, 129, 300, 0, 5 rows (ragged tiles, empty
    experts), N = 384 (a half 256-column tile), 16 rows past offsets[E] that
    must stay untouched."""
    ops = Operands([0, 1, 127, 128, 129, 300, 0, 5], N=384, K=512, seed=11, extra_rows=16)
    g = ops.gpu()
    out32 = run_m(g, fg8.FG8_OUT_F32, fill=0x7FC00001)
    out16 = run_m(g, fg8.FG8_OUT_BF16, fill=0x7FC1)
    used = int(ops.offsets[-1])
    ref, bound = oracle.gemm_mgrouped_full(ops.a.numpy(), ops.sa.numpy(), ops.b.numpy(),
                                           ops.sb.numpy(), ops.offsets)
    check(out32[:used].cpu().numpy(), ref[:used], bound[:used], "ragged")
    assert np.array_equal(bf16_of(out32[:used]), out16[:used].view(torch.int16).cpu().numpy())
    assert np.all(out32[used:].view(torch.int32).cpu().numpy() == 0x7FC00001)
    assert np.all(out16[used:].view(torch.int16).cpu().numpy() == 0x7FC1)


def test_gemm_unit_scales_small_integers_exact():
    """All scales 1 and codes of the integers -8..8: every partial sum is an
    integer below 2^24, so the fp32 result must equal the int64 product."""
    rng = np.random.default_rng(5)
    counts = [130, 0, 77, 256]
    E, N, K = len(counts), 384, 768
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    M = int(offsets[-1])
    ints = np.arange(-8, 9)
    code_of = {int(v): int(torch.tensor(float(v)).to(torch.float8_e4m3fn).view(torch.uint8))
               for v in ints}
    ia = rng.choice(ints, size=(M, K))
    ib = rng.choice(ints, size=(E, N, K))
    a = np.vectorize(code_of.get)(ia).astype(np.uint8)
    b = np.vectorize(code_of.get)(ib).astype(np.uint8)
    sa = torch.ones((K // 128, M), dtype=torch.float32)
    sb = torch.ones((E, N // 128, K // 128), dtype=torch.float32)
    out = fg8.grouped_gemm(torch.from_numpy(a).cuda(), sa.cuda(), torch.from_numpy(b).cuda(),
                           sb.cuda(), torch.from_numpy(offsets).cuda(), out_dtype=fg8.FG8_OUT_F32)
    torch.cuda.synchronize()
    got = out.cpu().numpy()
    for e in range(E):
        r0, r1 = offsets[e], offsets[e + 1]
        assert np.array_equal(got[r0:r1], (ia[r0:r1] @ ib[e].T).astype(np.float32)), e


def test_gemm_tiny_end_to_end(oracle):
    """bf16 X, W of the tiny config: GPU permute+quantize -> GPU grouped GEMM,
    against oracle permute+quantize -> oracle fp64 GEMM."""
    cfg = W.CONFIGS["tiny"]
    x = W.gen_x(cfg)
    ids = W.route(cfg)
    w = W.gen_w_up(cfg)
    act = fg8.quantize_act(x.cuda(), torch.from_numpy(ids).cuda(), cfg.E)
    wq, sw = fg8.quantize_weight(w.cuda())
    out = fg8.grouped_gemm(act["xq"], act["sa"], wq, sw, act["offsets"], out_dtype=fg8.FG8_OUT_F32)
    torch.cuda.synchronize()
    oa = oracle.quantize_act(x, ids, cfg.E)
    owq, osw = oracle.quantize_weight(w)
    ref, bound = oracle.gemm_mgrouped_full(oa["xq"], oa["sa"], owq, osw, oa["offsets"])
    check(out.cpu().numpy(), ref, bound, "tiny e2e")
    # and the quantized product approximates the bf16 product
    xf = x.double().numpy()[oa["row_token"]]
    wf = w.double().numpy()
    exact = np.concatenate([xf[oa["offsets"][e]:oa["offsets"][e + 1]] @ wf[e].T
                            for e in range(cfg.E)])
    assert np.linalg.norm(out.cpu().numpy() - exact) / np.linalg.norm(exact) < 0.05


def _sampled_rows_check(oracle, cfg_seed, a_gpu_out, offsets, N, K, E, rows, a_sid, b_sid,
                        sa_sid, sb_sid, n_blocks=2, what=""):
    """Check sampled rows of a row-grouped product whose operands were drawn by
    the generators on the device: regenerate the sampled rows, their experts'
    weights for n_blocks 128-column blocks, and their scales on the host."""
    rng = np.random.default_rng(len(rows))
    M_total = a_gpu_out.shape[0]
    NB, KB = N // 128, K // 128
    sa_all = W.gen_scales((KB * M_total,), cfg_seed, sa_sid).view(KB, M_total)
    for r in rows:
        e = int(np.searchsorted(offsets, r, side="right") - 1)
        blocks = sorted(set([NB - 1] + [int(b) for b in rng.integers(0, NB, n_blocks - 1)]))
        a_row = W.gen_e4m3_codes((1, K), cfg_seed, a_sid, index_offset=r * K).numpy()
        sa_row = sa_all[:, r:r + 1].contiguous().numpy()
        b_rows = np.concatenate([
            W.gen_e4m3_codes((128, K), cfg_seed, b_sid, index_offset=(e * N + nb * 128) * K).numpy()
            for nb in blocks])[None]
        sb_e = W.gen_scales((NB * KB,), cfg_seed, sb_sid, index_offset=e * NB * KB).view(NB, KB)
        sb_sub = sb_e[blocks].contiguous().numpy()[None]
        ref, bound = oracle.gemm_mgrouped_full(a_row, sa_row, b_rows, sb_sub,
                                               np.array([0, 1], np.int32))
        cols = np.concatenate([np.arange(nb * 128, nb * 128 + 128) for nb in blocks])
        got = a_gpu_out[r, torch.from_numpy(cols).cuda()].float().cpu().numpy()[None]
        check(got, ref, bound, f"{what} row {r} expert {e}")


@pytest.mark.parametrize("shape", ["dense4096", "kanana_up", "kanana_down", "dsv3_up",
                                   "dsv3_down", "dsv3_dgrad"])
def test_gemm_full_size_sampled_rows(oracle, shape):
    name, which = (shape.split("_") + [""])[:2]
    cfg = W.CONFIGS["dense4096" if name == "dense4096" else name]
    if name == "dense4096":
        N, K = 4096, 4096
        offsets = np.array([0, 4096], np.int32)
    else:
        r = oracle.route(W.route(cfg), cfg.E)
        offsets = r["offsets"]
        N, K = {"up": (cfg.n_up, cfg.hidden), "down": (cfg.hidden, cfg.inter),
                "dgrad": (cfg.hidden, cfg.n_up)}[which]
    E = offsets.size - 1
    M = int(offsets[-1])
    seed = cfg.seed + 1000 * len(shape)
    a = W.gen_e4m3_codes((M, K), seed, 1, device="cuda")
    sa = W.gen_scales((K // 128 * M,), seed, 2, device="cuda").view(K // 128, M)
    b = W.gen_e4m3_codes((E, N, K), seed, 3, device="cuda")
    sb = W.gen_scales((E * (N // 128) * (K // 128),), seed, 4, device="cuda").view(
        E, N // 128, K // 128)
    off_d = torch.from_numpy(offsets).cuda()
    st = fg8.new_status()
    out32 = fg8.grouped_gemm(a, sa, b, sb, off_d, out_dtype=fg8.FG8_OUT_F32, dev_status=st)
    out16 = fg8.grouped_gemm(a, sa, b, sb, off_d, out_dtype=fg8.FG8_OUT_BF16, dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    del a, b
    # bf16 output = RNE(fp32 output), checked on all rows
    assert torch.equal(out32.to(torch.bfloat16).view(torch.int16), out16.view(torch.int16))
    del out16
    counts = np.diff(offsets)
    nz = np.nonzero(counts)[0]
    rng = np.random.default_rng(7)
    rows = set()
    for e in sorted(set([int(nz[np.argmax(counts[nz])]), int(nz[np.argmin(counts[nz])])] +
                        [int(e) for e in rng.choice(nz, min(14, nz.size), replace=False)])):
        rows.update([int(offsets[e]), int(offsets[e + 1] - 1)])
    rows.update(int(x) for x in rng.integers(0, M, 24))
    _sampled_rows_check(oracle, seed, out32, offsets, N, K, E, sorted(rows), 1, 3, 2, 4,
                        what=shape)


def test_gemm_kgrouped_ragged_full(oracle):
    """Contraction-grouped (weight gradient) with experts of 3, 0, 200, 128, 0,
    257 tokens: padded contraction ranges, zero-token experts give zeros."""
    counts = np.array([3, 0, 200, 128, 0, 257])
    padded = (counts + 127) // 128 * 128
    padoff = np.concatenate([[0], np.cumsum(padded)]).astype(np.int32)
    E, M, N = len(counts), 256, 384
    P = fg8.fg8_colwise_capacity(int(counts.sum()), E)
    a = W.gen_e4m3_codes((M, P), 21, 1)
    b = W.gen_e4m3_codes((N, P), 21, 2)
    sa = W.gen_scales((P // 128, M), 21, 3)
    sb = W.gen_scales((P // 128, N), 21, 4)
    out = fg8.grouped_gemm(a.cuda(), sa.cuda(), b.cuda(), sb.cuda(),
                           torch.from_numpy(padoff).cuda(), out_dtype=fg8.FG8_OUT_F32,
                           group_mode=fg8.FG8_GROUP_K)
    torch.cuda.synchronize()
    got = out.cpu().numpy()
    m, n = np.meshgrid(np.arange(M), np.arange(N), indexing="ij")
    for e in range(E):
        ref, bound = oracle.gemm_kgrouped_entries(a.numpy(), sa.numpy(), b.numpy(), sb.numpy(),
                                                  padoff, np.full(m.size, e), m.ravel(), n.ravel())
        if counts[e] == 0:
            assert np.all(got[e] == 0)
        check(got[e].ravel(), ref, bound, f"kgrouped expert {e}")


def test_gemm_kgrouped_dsv3_wgrad_full_size_sampled(oracle):
    """dW[e] = dY_e^T X_e shapes of the DeepSeek-V3-shaped layer at full size:
    A [4096, P], B [7168, P], P = capacity(65536, 256), fp32 out [256, 4096, 7168];
    64 sampled entries in each of 10 experts (incl. empty ones)."""
    cfg = W.CONFIGS["dsv3_bwd"]
    r = oracle.route(W.route(cfg), cfg.E)
    counts = np.diff(r["offsets"])
    padoff = np.concatenate([[0], np.cumsum((counts + 127) // 128 * 128)]).astype(np.int32)
    M, N, E = cfg.n_up, cfg.hidden, cfg.E
    P = fg8.fg8_colwise_capacity(cfg.R, E)
    seed = cfg.seed + 77
    a = W.gen_e4m3_codes((M, P), seed, 1, device="cuda")
    b = W.gen_e4m3_codes((N, P), seed, 2, device="cuda")
    sa = W.gen_scales((P // 128 * M,), seed, 3, device="cuda").view(P // 128, M)
    sb = W.gen_scales((P // 128 * N,), seed, 4, device="cuda").view(P // 128, N)
    st = fg8.new_status()
    out = fg8.grouped_gemm(a, sa, b, sb, torch.from_numpy(padoff).cuda(),
                           out_dtype=fg8.FG8_OUT_F32, group_mode=fg8.FG8_GROUP_K, dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    del a, b
    rng = np.random.default_rng(8)
    zero = np.nonzero(counts == 0)[0]
    nz = np.nonzero(counts)[0]
    experts = [int(zero[0]), int(nz[np.argmax(counts[nz])]), int(nz[np.argmin(counts[nz])])] + \
        [int(e) for e in rng.choice(nz, 7, replace=False)]
    ms = np.sort(rng.choice(M, 16, replace=False))
    ns = np.sort(rng.choice(N, 16, replace=False))
    a_sub = torch.cat([W.gen_e4m3_codes((1, P), seed, 1, index_offset=int(m) * P) for m in ms]).numpy()
    b_sub = torch.cat([W.gen_e4m3_codes((1, P), seed, 2, index_offset=int(n) * P) for n in ns]).numpy()
    sa_sub = W.gen_scales((P // 128 * M,), seed, 3).view(P // 128, M)[:, ms].contiguous().numpy()
    sb_sub = W.gen_scales((P // 128 * N,), seed, 4).view(P // 128, N)[:, ns].contiguous().numpy()
    mi, ni = np.meshgrid(np.arange(16), np.arange(16), indexing="ij")
    for e in experts:
        ref, bound = oracle.gemm_kgrouped_entries(a_sub, sa_sub, b_sub, sb_sub, padoff,
                                                  np.full(mi.size, e), mi.ravel(), ni.ravel())
        got = out[e][torch.from_numpy(ms).cuda()][:, torch.from_numpy(ns).cuda()].cpu().numpy()
        if counts[e] == 0:
            assert np.all(got == 0)
        check(got.ravel(), ref, bound, f"wgrad expert {e}")


def _kgrouped_operands(counts, M, N, seed):
    counts = np.asarray(counts)
    padoff = np.concatenate([[0], np.cumsum((counts + 127) // 128 * 128)]).astype(np.int32)
    P = fg8.fg8_colwise_capacity(int(counts.sum()), len(counts))
    a = W.gen_e4m3_codes((M, P), seed, 1)
    b = W.gen_e4m3_codes((N, P), seed, 2)
    sa = W.gen_scales((P // 128, M), seed, 3)
    sb = W.gen_scales((P // 128, N), seed, 4)
    return padoff, a, b, sa, sb


def test_gemm_kgrouped_interleaved_order_full(oracle):
    """Contraction-grouped with E divisible by 4, so tiles of four experts of
    different sizes are interleaved at run time: 8 experts (two empty, one with
    five K blocks), every output entry against the oracle."""
    counts = [0, 700, 1, 130, 0, 64, 390, 128]
    M, N, E = 256, 512, len(counts)
    padoff, a, b, sa, sb = _kgrouped_operands(counts, M, N, 31)
    st = fg8.new_status()
    out = fg8.grouped_gemm(a.cuda(), sa.cuda(), b.cuda(), sb.cuda(), torch.from_numpy(padoff).cuda(),
                           out_dtype=fg8.FG8_OUT_F32, group_mode=fg8.FG8_GROUP_K, dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    got = out.cpu().numpy()
    m, n = np.meshgrid(np.arange(M), np.arange(N), indexing="ij")
    for e in range(E):
        ref, bound = oracle.gemm_kgrouped_entries(a.numpy(), sa.numpy(), b.numpy(), sb.numpy(),
                                                  padoff, np.full(m.size, e), m.ravel(), n.ravel())
        if counts[e] == 0:
            assert np.all(got[e] == 0)
        check(got[e].ravel(), ref, bound, f"interleaved expert {e}")


def test_gemm_kgrouped_workspaces_reused_and_concurrent():
    """The contraction-grouped GEMM hands out tiles from a counter in the
    caller's workspace.  One workspace reused by 10 launches in a row on one
    stream, and 72 launches spread over 4 streams with a workspace each (more
    than any fixed pool of counters would hold), must all equal the first
    result bit for bit (the kernel is deterministic) with a clean status."""
    counts = [5, 300, 0, 129, 77, 256, 1, 40]
    M, N = 128, 256
    padoff, a, b, sa, sb = _kgrouped_operands(counts, M, N, 33)
    args = [t.cuda() for t in (a, sa, b, sb)] + [torch.from_numpy(padoff).cuda()]
    need = fg8.fg8_grouped_gemm_workspace(fg8.FG8_GROUP_K)
    st = fg8.new_status()

    def run(ws, stream=None):
        return fg8.grouped_gemm(*args, out_dtype=fg8.FG8_OUT_F32, group_mode=fg8.FG8_GROUP_K,
                                dev_status=st, stream=stream, workspace=ws)

    ws0 = torch.empty(need, dtype=torch.uint8, device="cuda")
    first = run(ws0)
    torch.cuda.synchronize()
    outs = [run(ws0) for _ in range(10)]
    streams = [torch.cuda.Stream() for _ in range(4)]
    wss = [torch.empty(need, dtype=torch.uint8, device="cuda") for _ in range(72)]
    torch.cuda.synchronize()
    for i, ws in enumerate(wss):
        s_ = streams[i % 4]
        with torch.cuda.stream(s_):
            outs.append(run(ws, s_.cuda_stream))
    torch.cuda.synchronize()
    assert st.item() == 0
    for o in outs:
        assert torch.equal(o, first)
