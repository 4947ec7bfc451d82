"""Full-size parity of the bandwidth kernels and of the dense GEMM against the
oracle, in full (no sampling), at the sizes of the benchmark's workloads.

The inputs come from the seeded generators, run on the device for speed and
copied back to the host one slice at a time (every slice is also checked
against the same generator run on the CPU at sampled indices, so the oracle's
input is the generator's, not anything the kernels produced).  The oracle runs
through its threaded drivers (plain loops on disjoint experts, rows or column
groups), streamed over expert chunks so that host memory stays bounded.

  * 128x128 weight quantization, the fused quantize + block transpose and the
    standalone block transpose: every expert of both Kanana-scale weights and
    both DeepSeek-V3-shaped weights, bit for bit;
  * column-wise (token-axis) quantization of dY and of X gathered through the
    permutation: every expert of the DeepSeek-V3-shaped and Kanana-scale
    layers, bit for bit;
  * identity-mode row quantization of the DeepSeek-V3 dY [65536, 4096];
  * the single-group dense GEMM M = N = K = 4096: both operands quantized on
    the device (bit-exact against the oracle), then every output entry within
    |err| <= 1e-3 sum|a b| and relative Frobenius <= 1e-4 of the fp64
    reference, and the bf16 output equal to the RNE of the fp32 output."""

import numpy as np
import pytest
import torch

from fp8_fine_grained_permute_b200 import build as fbuild
from fp8_fine_grained_permute_b200 import fg8
from fp8_fine_grained_permute_b200 import workloads as W

pytestmark = pytest.mark.gpu

HOST_CHUNK_BYTES = 1 << 30     # bf16 bytes of one streamed slice


@pytest.fixture(scope="module", autouse=True)
def _lib():
    fbuild.build()
    fg8.lib()
    torch.cuda.init()


def _spot_check_generator(chunk_u16: np.ndarray, flat0: int, sigma: float, seed: int, sid: int):
    """The device-generated slice equals the CPU generator at 4096 sampled indices."""
    flat = chunk_u16.reshape(-1)
    idx = np.random.default_rng(flat0 % 1000003).integers(0, flat.size, 4096)
    cpu = W.gen_normal_bf16_at(torch.from_numpy(idx + flat0), sigma, seed, sid)
    assert np.array_equal(flat[idx], cpu.view(torch.int16).numpy().view(np.uint16))


def _u16(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


WEIGHTS = [("kanana", "up"), ("kanana", "down"), ("dsv3", "up"), ("dsv3", "down")]


@pytest.mark.parametrize("name,which", WEIGHTS, ids=[f"{c}-{w}" for c, w in WEIGHTS])
def test_weight_quantize_fused_transpose_and_k3_full(oracle, name, which):
    """Every block of the weight: fg8_quantize_weight, the fused
    fg8_quantize_weight_transposed (both copies) and fg8_transpose_blockq of
    the forward copy, all equal to the oracle's quantization and transpose."""
    cfg = W.CONFIGS[name]
    if which == "up":
        E, N, K, sid = cfg.E, cfg.n_up, cfg.hidden, W.SID_W_UP
    else:
        E, N, K, sid = cfg.E, cfg.hidden, cfg.inter, W.SID_W_DOWN
    w = W.gen_normal_bf16((E, N, K), W.SIGMA_W, cfg.seed, sid, device="cuda")
    st = fg8.new_status()
    wq_f, sw_f, wqT_f, swT_f = fg8.quantize_weight_transposed(w, status=st)
    wq_p, sw_p = fg8.quantize_weight(w, status=st)
    wqT_k3, swT_k3 = fg8.transpose_blockq(wq_p, sw_p)
    torch.cuda.synchronize()
    assert st.item() == 0
    per = max(1, HOST_CHUNK_BYTES // (2 * N * K))
    for e0 in range(0, E, per):
        e1 = min(E, e0 + per)
        wc = _u16(w[e0:e1])
        _spot_check_generator(wc, e0 * N * K, W.SIGMA_W, cfg.seed, sid)
        owq, osw = oracle.quantize_weight_threaded(wc)
        owqT, oswT = oracle.transpose_blockq_threaded(owq, osw)
        for tag, (q, s) in (("K2", (wq_p, sw_p)), ("fused", (wq_f, sw_f))):
            assert np.array_equal(q[e0:e1].cpu().numpy(), owq), (tag, e0)
            assert np.array_equal(s[e0:e1].cpu().numpy().view(np.uint32), osw.view(np.uint32)), (tag, e0)
        for tag, (q, s) in (("fused^T", (wqT_f, swT_f)), ("K3", (wqT_k3, swT_k3))):
            assert np.array_equal(q[e0:e1].cpu().numpy(), owqT), (tag, e0)
            assert np.array_equal(s[e0:e1].cpu().numpy().view(np.uint32), oswT.view(np.uint32)), (tag, e0)


@pytest.mark.parametrize("name", ["kanana", "dsv3"])
def test_colwise_all_experts_full(oracle, name):
    """Weight-gradient operands of every expert: dY [R, n_up] in expert order
    and X [T, hidden] gathered through row_token, quantized along the token
    axis in 128-token tiles; codes, scales and padded offsets bit for bit."""
    cfg = W.CONFIGS[name]
    r = oracle.route(W.route(cfg), cfg.E)
    offs = r["offsets"]
    offs_d = torch.from_numpy(offs).cuda()
    dy = W.gen_dy(cfg, device="cuda")
    dT, dS, dpad = fg8.quantize_act_colwise(dy, offs_d)
    x = W.gen_x(cfg, device="cuda")
    xT, xS, xpad = fg8.quantize_act_colwise(x, offs_d, k=cfg.k,
                                            row_token=torch.from_numpy(r["row_token"]).cuda())
    torch.cuda.synchronize()
    P = fg8.fg8_colwise_capacity(cfg.R, cfg.E)
    dyh = _u16(dy)
    xh = _u16(x)
    _spot_check_generator(xh, 0, W.SIGMA_X, cfg.seed, W.SID_X)
    # dY comes from the Student-t generator: spot-check through its slice call
    assert np.array_equal(dyh[:4], _u16(W.gen_dy(cfg, row0=0, rows=4)))
    assert np.array_equal(dyh[-4:], _u16(W.gen_dy(cfg, row0=cfg.R - 4, rows=4)))
    dref = oracle.quantize_act_colwise_threaded(dyh, offs, P_cap=P)
    xref = oracle.quantize_act_colwise_threaded(xh, offs, row_map=r["row_token"], P_cap=P)
    used = int(dref["padoff"][-1])
    for got, pad, ref in ((dT, dpad, dref), (xT, xpad, xref)):
        assert np.array_equal(pad.cpu().numpy(), ref["padoff"])
        assert np.array_equal(got[:, :used].cpu().numpy(), ref["xqT"][:, :used])
    assert np.array_equal(dS[:used // 128].cpu().numpy(), dref["sT"][:used // 128])
    assert np.array_equal(xS[:used // 128].cpu().numpy(), xref["sT"][:used // 128])


def test_rows_dsv3_dy_full(oracle):
    """Identity-mode 1x128 quantization of the DeepSeek-V3 backward dY
    [65536, 4096] (Student-t with outlier tiles), every code and scale."""
    cfg = W.CONFIGS["dsv3_bwd"]
    dy = W.gen_dy(cfg, device="cuda")
    xq, sa = fg8.quantize_act_rows(dy)
    torch.cuda.synchronize()
    dyh = _u16(dy)
    assert np.array_equal(dyh[-3:], _u16(W.gen_dy(cfg, row0=cfg.R - 3, rows=3)))
    oxq, osa = oracle.quantize_rows_threaded(dyh)
    assert np.array_equal(xq.cpu().numpy(), oxq)
    assert np.array_equal(sa.cpu().numpy().view(np.uint32), osa.view(np.uint32))


def test_dense4096_quantize_and_gemm_full(oracle):
    """Config M = N = K = 4096, one group: X and W quantized on the device
    (1x128 and 128x128, bit-exact against the oracle), then the FP8 GEMM;
    all 16.7 M outputs against the fp64 product of the oracle's operands."""
    cfg = W.CONFIGS["dense4096"]
    x = W.gen_x(cfg, device="cuda")
    w = W.gen_w_up(cfg, device="cuda")
    xq, sa = fg8.quantize_act_rows(x)
    wq, sw = fg8.quantize_weight(w)
    offsets = torch.tensor([0, cfg.T], dtype=torch.int32, device="cuda")
    st = fg8.new_status()
    y32 = fg8.grouped_gemm(xq, sa, wq, sw, offsets, out_dtype=fg8.FG8_OUT_F32, dev_status=st)
    y16 = fg8.grouped_gemm(xq, sa, wq, sw, offsets, out_dtype=fg8.FG8_OUT_BF16, dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    xh, wh = _u16(x), _u16(w)
    _spot_check_generator(xh, 0, W.SIGMA_X, cfg.seed, W.SID_X)
    _spot_check_generator(wh, 0, W.SIGMA_W, cfg.seed, W.SID_W_UP)
    oxq, osa = oracle.quantize_rows_threaded(xh)
    owq, osw = oracle.quantize_weight_threaded(wh)
    assert np.array_equal(xq.cpu().numpy(), oxq) and np.array_equal(sa.cpu().numpy(), osa)
    assert np.array_equal(wq.cpu().numpy(), owq) and np.array_equal(sw.cpu().numpy(), osw)
    ref, bound = oracle.gemm_dense_fp64(oxq, osa, owq, osw)
    got = y32.cpu().numpy().astype(np.float64)
    err = np.abs(got - ref)
    assert np.all(err <= 1e-3 * bound + 1e-30), float(np.max(err - 1e-3 * bound))
    assert np.linalg.norm(got - ref) <= 1e-4 * np.linalg.norm(ref)
    assert torch.equal(y16.view(torch.int16), y32.to(torch.bfloat16).view(torch.int16))
