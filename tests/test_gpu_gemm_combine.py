"""GPU parity of fg8_grouped_gemm_combine (the down-projection with the combine
in its epilogue) against the oracle's gemm_combine_entries: per entry
|err| <= 1e-3 * bound + 2^-20 * sum |w Y| (the GEMM's stated tolerance on
every weighted row, plus fp32 rounding of the products and of the k
reductions, whose order is not fixed), and close to the unfused GPU path
(the fp32 GEMM output through fg8_unpermute_combine with fp32 output)."""

import numpy as np
import pytest
import torch

from fp8_fine_grained_permute_b200 import build as fbuild
from fp8_fine_grained_permute_b200 import fg8
from fp8_fine_grained_permute_b200 import workloads as W

pytestmark = pytest.mark.gpu

ELEM_TOL = 1e-3
ROUND_TOL = 2.0 ** -20


@pytest.fixture(scope="module", autouse=True)
def _lib():
    fbuild.build()
    fg8.lib()
    torch.cuda.init()


def _layer(oracle, T, E, k, N, K, seed, extra_rows=0):
    rng = np.random.default_rng(seed)
    ids = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    r = oracle.route(ids, E)
    R = int(r["offsets"][-1]) + extra_rows
    a = W.gen_e4m3_codes((R, K), seed, 1)
    sa = W.gen_scales((K // 128, R), seed, 2)
    b = W.gen_e4m3_codes((E, N, K), seed, 3)
    sb = W.gen_scales((E, N // 128, K // 128), seed, 4)
    aff = W.gen_uniform_f32((T, k), seed, 5)
    row_token = np.full(R, -1, np.int32)
    row_token[:int(r["offsets"][-1])] = r["row_token"]
    return dict(a=a, sa=sa, b=b, sb=sb, offsets=r["offsets"], row_token=row_token,
                token_row=r["token_row"].copy(), aff=aff.numpy() if torch.is_tensor(aff) else aff)


def _run(L, normalize=True):
    dev = "cuda"
    g = lambda x: (x if torch.is_tensor(x) else torch.from_numpy(np.ascontiguousarray(x))).to(dev)  # noqa: E731
    st = fg8.new_status()
    out = fg8.grouped_gemm_combine(g(L["a"]), g(L["sa"]), g(L["b"]), g(L["sb"]), g(L["offsets"]),
                                   g(L["row_token"]), g(L["token_row"]), g(L["aff"]),
                                   normalize=normalize, dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    return out.cpu().numpy().astype(np.float64)


def _check(oracle, L, got, tokens=None, normalize=True):
    T, N = got.shape
    if tokens is None:
        tokens = np.arange(T)
    t, c = np.meshgrid(tokens, np.arange(N), indexing="ij")
    ref, bound, mag = oracle.gemm_combine_entries(
        L["a"], L["sa"], L["b"], L["sb"], L["offsets"], L["token_row"], L["aff"],
        t.ravel(), c.ravel(), normalize=normalize)
    g = got[tokens].ravel()
    err = np.abs(g - ref)
    lim = ELEM_TOL * bound + ROUND_TOL * mag + 1e-30
    assert np.all(err <= lim), f"worst excess {np.max(err - lim)}"


@pytest.mark.parametrize("normalize", [True, False])
def test_gemm_combine_matches_oracle(oracle, normalize):
    L = _layer(oracle, T=300, E=6, k=3, N=384, K=256, seed=31, extra_rows=5)
    got = _run(L, normalize)
    _check(oracle, L, got, normalize=normalize)


def test_gemm_combine_dropped_slots_and_empty_tokens(oracle):
    L = _layer(oracle, T=200, E=5, k=4, N=256, K=384, seed=32)
    tr = L["token_row"].reshape(200, 4)
    tr[3, 2] = -1          # a slot without a row
    tr[7, :] = -1          # a token without rows: zeros
    L["aff"] = L["aff"].copy()
    L["aff"][11, :] = 0.0  # kept affinities summing to 0: zeros
    L["token_row"] = tr.ravel()
    got = _run(L)
    assert np.all(got[7] == 0) and np.all(got[11] == 0)
    _check(oracle, L, got)


def test_gemm_combine_close_to_unfused_path(oracle):
    """The same rows from the plain GEMM (fp32 output), weighted and summed on
    the host in fp64: only the fp32 rounding of the products and of the
    reductions may differ."""
    T, k = 512, 4
    L = _layer(oracle, T=T, E=8, k=k, N=512, K=512, seed=33)
    got = _run(L)
    g = lambda x: (x if torch.is_tensor(x) else torch.from_numpy(np.ascontiguousarray(x))).cuda()  # noqa: E731
    y = fg8.grouped_gemm(g(L["a"]), g(L["sa"]), g(L["b"]), g(L["sb"]), g(L["offsets"]),
                         out_dtype=fg8.FG8_OUT_F32)
    yn = y.double().cpu().numpy()
    tr = L["token_row"].reshape(T, k)
    kept = (tr >= 0) & (tr < int(L["offsets"][-1]))
    aff = np.where(kept, L["aff"].astype(np.float64), 0.0)
    w = aff / np.where(aff.sum(1) == 0, 1.0, aff.sum(1))[:, None]
    want = np.stack([(w[t][kept[t], None] * yn[tr[t][kept[t]]]).sum(0) for t in range(T)])
    rel = np.linalg.norm(got - want) / np.linalg.norm(want)
    assert rel <= 1e-6, rel


def test_gemm_combine_kanana_down_sampled_tokens(oracle):
    cfg = W.CONFIGS["kanana"]
    ids = W.route(cfg)
    r = oracle.route(ids, cfg.E)
    R, K, N = cfg.R, cfg.inter, cfg.hidden
    L = dict(a=W.gen_e4m3_codes((R, K), 41, 1), sa=W.gen_scales((K // 128, R), 41, 2),
             b=W.gen_e4m3_codes((cfg.E, N, K), 41, 3), sb=W.gen_scales((cfg.E, N // 128, K // 128), 41, 4),
             offsets=r["offsets"], row_token=r["row_token"], token_row=r["token_row"],
             aff=W.gen_affinity(cfg).numpy())
    got = _run(L)
    tokens = np.random.default_rng(7).choice(cfg.T, 48, replace=False)
    _check(oracle, L, got, tokens=np.sort(tokens))


def test_gemm_combine_rejects_bad_arguments():
    dev = "cuda"
    a = torch.zeros((128, 128), dtype=torch.uint8, device=dev)
    sa = torch.ones((1, 128), device=dev)
    b = torch.zeros((1, 128, 128), dtype=torch.uint8, device=dev)
    sb = torch.ones((1, 1, 1), device=dev)
    off = torch.tensor([0, 128], dtype=torch.int32, device=dev)
    rt = torch.zeros(128, dtype=torch.int32, device=dev)
    tr = torch.zeros(128, dtype=torch.int32, device=dev)
    aff = torch.ones((128, 1), device=dev)
    out = torch.empty((128, 128), device=dev)
    ws = torch.empty(16, dtype=torch.uint8, device=dev)   # too small for 128 rows
    st = fg8.new_status()
    with pytest.raises(fg8.FG8Error):
        fg8.fg8_grouped_gemm_combine(a, sa, b, sb, off, 128, 128, 128, 1, rt, tr, aff, 128, 1, 1,
                                     out, ws, ws.numel(), st)
    with pytest.raises(fg8.FG8Error):   # k out of range
        fg8.fg8_grouped_gemm_combine(a, sa, b, sb, off, 128, 128, 128, 1, rt, tr, aff, 128, 17, 1,
                                     out, ws, ws.numel(), st)
