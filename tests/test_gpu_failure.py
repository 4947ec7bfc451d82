"""Failure detection on the GPU without a fault: the library's bounded waits
(the permuting quantizer's grid barrier, the GEMM pipeline's mbarrier wait)
are made to run out on a condition nothing satisfies; each must report
FG8_ERR_TIMEOUT through the status word and return, leaving the context
usable for the next launch."""

import time

import numpy as np
import pytest
import torch

from fp8_fine_grained_permute_b200 import build as fbuild
from fp8_fine_grained_permute_b200 import fg8
from fp8_fine_grained_permute_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("which", [0, 1])
def test_bounded_wait_times_out_and_context_survives(oracle, which):
    fbuild.build()
    st = fg8.new_status()
    scratch = torch.zeros(1, dtype=torch.int32, device="cuda")
    t0 = time.monotonic()
    fg8.fg8_selftest_wait_timeout(which, scratch, st)
    torch.cuda.synchronize()
    elapsed = time.monotonic() - t0
    assert st.item() == fg8.FG8_ERR_TIMEOUT
    assert 1.5 < elapsed < 30.0
    # the context is still usable: a regular launch produces oracle-exact output
    cfg = W.CONFIGS["tiny"]
    x = W.gen_x(cfg)
    ids = W.route(cfg)
    out = fg8.quantize_act(x.cuda(), torch.from_numpy(ids).cuda(), cfg.E)
    torch.cuda.synchronize()
    ref = oracle.quantize_act(x, ids, cfg.E)
    assert out["status"].item() == 0
    assert np.array_equal(out["xq"].cpu().numpy(), ref["xq"])
