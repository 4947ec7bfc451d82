"""GPU parity of the unpermute + combine kernel against the oracle's fp64 sum.

The kernel sums in fp32, every operation rounded to nearest: the affinity sum
(k - 1 additions), one division per weight, one product and one addition per
slot.  Its fp32 result is therefore within (2k + 4) * 2^-24 * sum_j |w_j y_j|
of the exact value (first-order bound); the bf16 output adds half a bf16 ulp
(2^-8 of the magnitude at most).  Also: at least 99% of the bf16 outputs equal
the oracle's value rounded to bf16, rows of dropped slots contribute nothing,
and the argument checks of the ABI.
"""

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


def check(got, ref, bound, k, bf16_out, what=""):
    got = np.asarray(got, np.float64)
    lim = (2 * k + 4) * 2.0 ** -24 * bound
    if bf16_out:
        lim = lim + 2.0 ** -8 * (np.abs(ref) + lim)
    err = np.abs(got - ref)
    assert np.all(err <= lim + 1e-38), f"{what}: worst excess {np.max(err - lim)}"
    if bf16_out:
        want = torch.from_numpy(ref).to(torch.float32).to(torch.bfloat16).to(torch.float64).numpy()
        # the fp64 -> fp32 -> bf16 double rounding can differ from the kernel's
        # only at ties; the kernel's own fp32 error moves a few more
        assert np.mean(got == want) >= 0.99, f"{what}: {np.mean(got != want)} differ"


def run(y, token_row, aff, normalize, out_dtype, fill=None):
    T, k = aff.shape
    dt = torch.float32 if out_dtype == fg8.FG8_OUT_F32 else torch.bfloat16
    out = torch.empty((T, y.shape[1]), dtype=dt, device="cuda")
    if fill is not None:
        out.view(torch.int16 if dt == torch.bfloat16 else torch.int32).fill_(fill)
    fg8.unpermute_combine(y.cuda(), torch.from_numpy(token_row).cuda(),
                          torch.from_numpy(aff).cuda(), normalize=normalize, out_dtype=out_dtype,
                          out=out)
    torch.cuda.synchronize()
    return out.float().cpu().numpy()


@pytest.mark.parametrize("k,C", [(6, 256), (8, 72), (1, 8), (16, 136), (3, 2048)])
@pytest.mark.parametrize("normalize", [True, False])
def test_combine_matches_oracle(oracle, k, C, normalize):
    rng = np.random.default_rng(1000 * k + C)
    T, E = 300, 7
    ids = rng.integers(0, E, (T, k)).astype(np.int32)
    ids[rng.random((T, k)) < 0.03] = E          # a few bad ids: no row
    r = oracle.route(ids, E)
    R = int(r["offsets"][-1])
    y = W.gen_normal_bf16((R, C), 1.0, 4242, k)
    aff = rng.uniform(0.0, 1.0, (T, k)).astype(np.float32)
    if not normalize:
        aff -= 0.5                               # signed weights
    ref, bound = oracle.unpermute_combine(y, r["token_row"], aff, normalize=normalize)
    for od in (fg8.FG8_OUT_F32, fg8.FG8_OUT_BF16):
        got = run(y, r["token_row"], aff, normalize, od)
        check(got, ref, bound, k, od == fg8.FG8_OUT_BF16, f"k={k} C={C} norm={normalize} od={od}")


def test_combine_dropped_and_out_of_range_rows(oracle):
    rng = np.random.default_rng(77)
    R, C, T, k = 64, 32, 40, 4
    y = W.gen_normal_bf16((R, C), 1.0, 4243, 1)
    rows = rng.integers(0, R, (T, k)).astype(np.int32)
    rows[:, 2] = -1
    rows[5, :] = -1                              # a token with no rows: zeros
    rows[6, 1] = R                               # out of range: dropped
    rows[7, 3] = np.iinfo(np.int32).max
    aff = rng.uniform(0.1, 1.0, (T, k)).astype(np.float32)
    ref, bound = oracle.unpermute_combine(y, rows.ravel(), aff, normalize=True)
    got = run(y, rows.ravel(), aff, True, fg8.FG8_OUT_F32, fill=0x7FC00001)
    check(got, ref, bound, k, False, "dropped")
    assert not got[5].any()


def test_combine_no_rows_at_all():
    T, k, C = 10, 2, 16
    y = torch.empty((0, C), dtype=torch.bfloat16)
    rows = np.full(T * k, -1, np.int32)
    aff = np.ones((T, k), np.float32)
    out = torch.full((T, C), 7.0, device="cuda")
    fg8.fg8_unpermute_combine(None, 0, C, torch.from_numpy(rows).cuda(),
                              torch.from_numpy(aff).cuda(), T, k, 1, fg8.FG8_OUT_F32, out)
    torch.cuda.synchronize()
    assert not out.any()


@pytest.mark.parametrize("name", ["kanana", "dsv3"])
def test_combine_full_size_sampled_tokens(oracle, name):
    """A full layer (every routed row of the down-projection output) on the
    device; sampled tokens are checked against the oracle on their own rows,
    regenerated on the host."""
    cfg = W.CONFIGS[name]
    r = oracle.route(W.route(cfg), cfg.E)
    T, k, C, R = cfg.T, cfg.k, cfg.hidden, cfg.R
    y = W.gen_y_down(cfg, "cuda")
    aff = W.gen_affinity(cfg, "cuda")
    tr = torch.from_numpy(r["token_row"]).cuda()
    out32 = fg8.unpermute_combine(y, tr, aff, out_dtype=fg8.FG8_OUT_F32)
    out16 = fg8.unpermute_combine(y, tr, aff, out_dtype=fg8.FG8_OUT_BF16)
    torch.cuda.synchronize()
    del y
    # bf16 output = RNE of the fp32 output, on every token
    assert torch.equal(out32.to(torch.bfloat16).view(torch.int16), out16.view(torch.int16))
    aff_h = W.gen_affinity(cfg).numpy()
    rng = np.random.default_rng(78)
    for t in sorted(set([0, T - 1] + [int(x) for x in rng.integers(0, T, 6)])):
        rows = r["token_row"][t * k:(t + 1) * k]
        y_rows = torch.stack([W.gen_normal_bf16((C,), 1.0, cfg.seed, W.SID_Y_DOWN,
                                                index_offset=int(row) * C) for row in rows])
        ref, bound = oracle.unpermute_combine(y_rows, np.arange(k, dtype=np.int32),
                                              aff_h[t:t + 1], normalize=True)
        check(out32[t].cpu().numpy()[None], ref, bound, k, False, f"{name} token {t}")


def test_combine_rejects_bad_arguments():
    y = torch.zeros((8, 16), dtype=torch.int16, device="cuda")
    rows = torch.zeros(4 * 17, dtype=torch.int32, device="cuda")
    aff = torch.ones((4, 17), device="cuda")
    out = torch.empty((4, 16), device="cuda")
    for args in [(y, 8, 16, rows, aff, 4, 17, 1, fg8.FG8_OUT_F32, out),   # k > 16
                 (y, 8, 12, rows, aff, 4, 2, 1, fg8.FG8_OUT_F32, out),    # C % 8
                 (y, 8, 16, rows, aff, 4, 2, 2, fg8.FG8_OUT_F32, out)]:   # normalize flag
        with pytest.raises(fg8.FG8Error) as ei:
            fg8.fg8_unpermute_combine(*args)
        assert ei.value.status == fg8.FG8_ERR_INVALID_ARG
