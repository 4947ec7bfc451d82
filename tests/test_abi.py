"""The C-ABI library loads on the host, exports every symbol that
include/fg8.h declares, and rejects bad arguments before touching the GPU.
(No compute call is made: this file runs without a GPU.)"""

import ctypes

import pytest

from fp8_fine_grained_permute_b200 import build as fbuild
from fp8_fine_grained_permute_b200 import fg8


@pytest.fixture(scope="module")
def L():
    fbuild.build()
    return fg8.lib()


def test_every_declared_symbol_is_exported(L):
    names = fg8.declared_symbols()
    assert {"fg8_quantize_act", "fg8_quantize_act_workspace", "fg8_colwise_capacity",
            "fg8_quantize_weight", "fg8_transpose_blockq", "fg8_grouped_gemm",
            "fg8_status_string"} <= set(names)
    for n in names:
        assert hasattr(L, n), n
        assert isinstance(getattr(L, n), ctypes._CFuncPtr)


def test_binding_has_the_c_names():
    for n in fg8.declared_symbols():
        assert callable(getattr(fg8, n)), n


def test_status_strings(L):
    for code, name in [(0, "FG8_OK"), (1, "FG8_ERR_INVALID_ARG"), (2, "FG8_ERR_UNSUPPORTED"),
                       (3, "FG8_ERR_CUDA"), (4, "FG8_ERR_BAD_EXPERT_ID"), (5, "FG8_ERR_TIMEOUT")]:
        assert fg8.status_name(code) == name
    assert fg8.status_name(99) == "FG8_UNKNOWN_STATUS"


def test_sizes(L):
    assert fg8.fg8_colwise_capacity(0, 4) == 512
    assert fg8.fg8_colwise_capacity(128, 1) == 256
    assert fg8.fg8_colwise_capacity(65536, 256) == 65536 + 127 * 256     # already a multiple of 128
    assert fg8.fg8_colwise_capacity(100, 3) == 512                       # 100 + 381 -> 512
    assert fg8.fg8_quantize_act_workspace(8192, 8, 256) >= 4 * 256
    assert fg8.fg8_quantize_act_workspace(8192, 8, 0) == 0


def test_null_and_shape_arguments_rejected_on_host(L):
    INV = fg8.FG8_ERR_INVALID_ARG
    # null pointers / bad sizes return before any CUDA call
    assert L.fg8_quantize_weight(None, 1, 128, 128, None, None, None, None) == INV
    assert L.fg8_quantize_weight(16, 1, 100, 128, 16, 16, None, None) == INV        # N % 128
    assert L.fg8_quantize_weight(16, 0, 128, 128, 16, 16, None, None) == INV        # E < 1
    assert L.fg8_transpose_blockq(None, None, 1, 128, 128, None, None, None) == INV
    assert L.fg8_transpose_blockq(16, 16, 1, 128, 130, 16, 16, None) == INV  # K % 128
    assert L.fg8_grouped_gemm(None, None, None, None, None, 128, 128, 128, 1, 0, 0, 0, None,
                              None, 0, None, None) == INV
    assert L.fg8_grouped_gemm(16, 16, 16, 16, 16, 128, 128, 128, 1, 0, 0, 7, 16, None, 0, None,
                              None) == INV                                    # out dtype
    # contraction-grouped: the tile counter's workspace is required, aligned, large enough
    need = fg8.fg8_grouped_gemm_workspace(fg8.FG8_GROUP_K)
    assert need >= 12 and fg8.fg8_grouped_gemm_workspace(fg8.FG8_GROUP_M) == 0
    assert L.fg8_grouped_gemm(16, 16, 16, 16, 16, 128, 128, 128, 1, 1, 1, 1, 16, None, need, None,
                              None) == INV
    assert L.fg8_grouped_gemm(16, 16, 16, 16, 16, 128, 128, 128, 1, 1, 1, 1, 16, 16, need - 1,
                              None, None) == INV
    assert L.fg8_grouped_gemm(16, 16, 16, 16, 16, 128, 128, 128, 1, 1, 1, 1, 16, 20, need, None,
                              None) == INV
    assert L.fg8_quantize_act(None, 10, 128, None, 1, 1, None, 1, 16, 16, None, None, None,
                              None, None, None, 0, None, None) == INV         # x null
    assert L.fg8_quantize_act(16, 10, 100, None, 1, 1, None, 1, 16, 16, None, None, None,
                              None, None, None, 0, None, None) == INV         # K % 128
    # misaligned FP8 / bf16 buffers
    assert L.fg8_quantize_weight(18, 1, 128, 128, 16, 16, None, None) == INV
    assert L.fg8_grouped_gemm(17, 16, 16, 16, 16, 128, 128, 128, 1, 0, 0, 0, 16, None, 0, None,
                              None) == INV
    # unsupported combinations
    assert L.fg8_grouped_gemm(16, 16, 16, 16, 16, 128, 128, 128, 1, 0, 1, 0, 16, None, 0, None,
                              None) == fg8.FG8_ERR_UNSUPPORTED               # M-grouped + row scales
    assert L.fg8_quantize_act(16, 10, 128, 16, 33, 4, None, 1, 16, 16, 16, 16, 16, None, None,
                              16, 1 << 20, None, None) == fg8.FG8_ERR_UNSUPPORTED  # k > 32


def test_next_entry_points_reject_bad_arguments_on_host(L):
    INV, OK = fg8.FG8_ERR_INVALID_ARG, fg8.FG8_OK
    F32 = fg8.FG8_OUT_F32
    # gated-activation up-projection: I % 128, K % 128, null outputs, misaligned codes
    assert L.fg8_grouped_gemm_swiglu_quant(16, 16, 16, 16, 16, 128, 96, 128, 1, 16, 16, None,
                                           None) == INV
    assert L.fg8_grouped_gemm_swiglu_quant(16, 16, 16, 16, 16, 128, 128, 100, 1, 16, 16, None,
                                           None) == INV
    assert L.fg8_grouped_gemm_swiglu_quant(16, 16, 16, 16, 16, 128, 128, 128, 1, None, 16, None,
                                           None) == INV
    assert L.fg8_grouped_gemm_swiglu_quant(16, 16, 16, 16, 16, 128, 128, 128, 1, 24, 16, None,
                                           None) == INV
    assert L.fg8_grouped_gemm_swiglu_quant(16, 16, 16, 16, 16, 128, 128, 128, 2000, 16, 16, None,
                                           None) == fg8.FG8_ERR_UNSUPPORTED       # E > 1024
    assert L.fg8_grouped_gemm_swiglu_quant(16, 16, 16, 16, 16, 0, 128, 128, 1, 16, 16, None,
                                           None) == OK                            # no rows
    # combine: slots, row width, flags, dtype; an empty batch is a no-op
    assert L.fg8_unpermute_combine(16, 8, 16, 16, 16, 4, 17, 1, F32, 16, None) == INV
    assert L.fg8_unpermute_combine(16, 8, 12, 16, 16, 4, 2, 1, F32, 16, None) == INV
    assert L.fg8_unpermute_combine(16, 8, 16, 16, 16, 4, 2, 2, F32, 16, None) == INV
    assert L.fg8_unpermute_combine(16, 8, 16, 16, 16, 4, 2, 1, 5, 16, None) == INV
    assert L.fg8_unpermute_combine(16, 8, 16, None, 16, 4, 2, 1, F32, 16, None) == INV
    assert L.fg8_unpermute_combine(16, 8, 16, 16, 16, 4, 2, 1, F32, 24, None) == INV   # out align
    assert L.fg8_unpermute_combine(None, 0, 16, None, None, 0, 2, 1, F32, None, None) == OK
    # routing: k within [1, min(16, E)], E <= 1024; an empty batch is a no-op
    assert L.fg8_route_topk(16, 16, 4, 8, 9, 16, 16, None) == INV
    assert L.fg8_route_topk(16, 16, 4, 64, 17, 16, 16, None) == INV
    assert L.fg8_route_topk(16, 16, 4, 2000, 4, 16, 16, None) == INV
    assert L.fg8_route_topk(16, 16, 4, 64, 0, 16, 16, None) == INV
    assert L.fg8_route_topk(None, 16, 4, 64, 4, 16, 16, None) == INV
    assert L.fg8_route_topk(18, 16, 4, 64, 4, 16, 16, None) == INV                     # align
    assert L.fg8_route_topk(None, None, 0, 64, 4, None, None, None) == OK
    # fused routing + permute-quantize: k, E, K checks; null outputs; empty batch
    assert L.fg8_route_quantize_act(16, 16, 16, 4, 256, 17, 64, 16, 16, 16, 16, 16, 16, 16, 16,
                                    1 << 20, None, None) == INV              # k > 16
    assert L.fg8_route_quantize_act(16, 16, 16, 4, 256, 4, 2000, 16, 16, 16, 16, 16, 16, 16, 16,
                                    1 << 20, None, None) == INV              # E > 1024
    assert L.fg8_route_quantize_act(16, 16, 16, 4, 200, 4, 64, 16, 16, 16, 16, 16, 16, 16, 16,
                                    1 << 20, None, None) == INV              # K % 128
    assert L.fg8_route_quantize_act(16, 16, 16, 4, 256, 4, 64, None, 16, 16, 16, 16, 16, 16, 16,
                                    1 << 20, None, None) == INV              # ids null
    assert L.fg8_route_quantize_act(16, 16, 16, 4, 256, 4, 64, 16, 16, 16, 16, 16, 16, 16, 16,
                                    8, None, None) == INV                    # workspace small


def test_binding_refuses_cpu_tensors(L):
    import torch
    w = torch.zeros((1, 128, 128), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        fg8.quantize_weight(w)
