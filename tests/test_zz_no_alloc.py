"""The allocation-free permuting quantizer, fg8_quantize_act_noalloc.

It is meant for callers that cannot allocate device memory (a plugin whose
host framework owns all allocations, or a path that must not enter the
allocator): its scratch is an array inside the library.  This test calls it
through the C ABI twice in a row and checks each result bit for bit against
the oracle (the routing maps and the 1x128 codes and scales of every routed
row) and against the regular entry point, fg8_quantize_act, which uses a
caller-provided workspace.  The cases include an expert count that is not a
multiple of 64, so the scratch layout's rounding is exercised at the array's
end (E = 255 of at most 256).

The file is named so that pytest collects it last."""

import numpy as np
import pytest
import torch

from fp8_fine_grained_permute_b200 import build as fbuild
from fp8_fine_grained_permute_b200 import fg8
from fp8_fine_grained_permute_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _noalloc(x, ids, E):
    T, K = x.shape
    k = ids.shape[1]
    R = T * k
    dev = x.device
    out = dict(xq=torch.empty((R, K), dtype=torch.uint8, device=dev),
               sa=torch.empty((K // 128, R), dtype=torch.float32, device=dev),
               row_token=torch.empty(R, dtype=torch.int32, device=dev),
               token_row=torch.empty(T * k, dtype=torch.int32, device=dev),
               offsets=torch.empty(E + 1, dtype=torch.int32, device=dev),
               status=torch.zeros(1, dtype=torch.int32, device=dev))
    st = fg8.lib().fg8_quantize_act_noalloc(
        x.view(torch.int16).data_ptr(), T, K, ids.data_ptr(), k, E, out["xq"].data_ptr(),
        out["sa"].data_ptr(), out["row_token"].data_ptr(), out["token_row"].data_ptr(),
        out["offsets"].data_ptr(), out["status"].data_ptr(),
        torch.cuda.current_stream().cuda_stream)
    assert st == fg8.FG8_OK, fg8.status_name(st)
    return out


def _case(name):
    if name == "E255":
        T, K, E, k = 777, 512, 255, 8
        rng = np.random.default_rng(255)
        ids = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
        return W.gen_normal_bf16((T, K), 1.0, 255, 1), ids, E
    cfg = W.CONFIGS[name]
    return W.gen_x(cfg), W.route(cfg), cfg.E


@pytest.mark.parametrize("name", ["tiny", "E255", "dsv3"])
def test_noalloc_matches_oracle_and_workspace_entry_point_twice(oracle, name):
    fbuild.build()
    fg8.lib()
    x_cpu, ids_np, E = _case(name)
    x = x_cpu.cuda()
    ids = torch.from_numpy(ids_np).cuda()
    r = oracle.route(ids_np, E)
    q = oracle.quantize_act(x_cpu, None, 1)          # each token row, 1x128 tiles
    rt = r["row_token"]
    expect = dict(xq=q["xq"][rt], sa=q["sa"][:, rt], row_token=rt, token_row=r["token_row"],
                  offsets=r["offsets"])
    ref = fg8.quantize_act(x, ids, E)
    for _ in range(2):
        got = _noalloc(x, ids, E)
        torch.cuda.synchronize()
        assert got["status"].item() == 0 and ref["status"].item() == 0
        for key in ("xq", "sa", "row_token", "token_row", "offsets"):
            assert np.array_equal(got[key].cpu().numpy(), expect[key]), key
            assert torch.equal(got[key], ref[key]), key


def test_noalloc_rejects_too_many_experts():
    fbuild.build()
    x = torch.zeros((4, 128), dtype=torch.bfloat16, device="cuda")
    ids = torch.zeros((4, 1), dtype=torch.int32, device="cuda")
    with pytest.raises(fg8.FG8Error) as e:
        fg8.fg8_quantize_act_noalloc(x.view(torch.int16), 4, 128, ids, 1, 257, None, None, None,
                                     None, None, None)
    assert e.value.status == fg8.FG8_ERR_UNSUPPORTED
