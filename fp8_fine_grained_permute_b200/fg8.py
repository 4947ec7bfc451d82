"""Python binding of libfg8 (the C ABI declared in include/fg8.h).

Argument marshalling only: every step of the path runs in the CUDA kernels of
libfg8.so.  PyTorch supplies device memory and streams.  There is no CPU
fallback: if the library is missing, or a tensor is not on a CUDA device,
these functions raise.

Two layers:
  * `fg8_*` functions with the C names and arguments (tensors or None in place
    of pointers), raising FG8Error on a non-OK status;
  * small helpers (`quantize_act`, `quantize_weight`, ...) that allocate the
    output tensors with torch and call the former.
"""

from __future__ import annotations

import ctypes
import os
import re

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libfg8.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "fg8.h")

FG8_OK = 0
FG8_ERR_INVALID_ARG = 1
FG8_ERR_UNSUPPORTED = 2
FG8_ERR_CUDA = 3
FG8_ERR_BAD_EXPERT_ID = 4
FG8_ERR_TIMEOUT = 5
FG8_ERR_WORKSPACE_SHARED = 6
FG8_ROWWISE = 1
FG8_COLWISE = 2
FG8_OUT_BF16 = 0
FG8_OUT_F32 = 1
FG8_GROUP_M = 0
FG8_GROUP_K = 1
FG8_BSCALE_BLOCK128 = 0
FG8_BSCALE_ROW128 = 1


class FG8Error(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {status_name(status)} ({status})")
        self.status = status


_lib = None
_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I = ctypes.c_int
_SZ = ctypes.c_size_t


def lib() -> ctypes.CDLL:
    """Load libfg8.so (built in-tree by fp8_fine_grained_permute_b200.build)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libfg8.so is not built ({LIB_PATH}); run "
                               "`python -m fp8_fine_grained_permute_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        L.fg8_quantize_act.restype = _I
        L.fg8_quantize_act.argtypes = [_P, _I64, _I64, _P, _I, _I, _P, _I, _P, _P, _P, _P, _P,
                                       _P, _P, _P, _SZ, _P, _P]
        L.fg8_route_quantize_act.restype = _I
        L.fg8_route_quantize_act.argtypes = [_P, _P, _P, _I64, _I64, _I, _I, _P, _P, _P, _P, _P,
                                             _P, _P, _P, _SZ, _P, _P]
        L.fg8_quantize_act_noalloc.restype = _I
        L.fg8_quantize_act_noalloc.argtypes = [_P, _I64, _I64, _P, _I, _I, _P, _P, _P, _P, _P,
                                               _P, _P]
        L.fg8_quantize_act_workspace.restype = _SZ
        L.fg8_quantize_act_workspace.argtypes = [_I64, _I, _I]
        L.fg8_colwise_capacity.restype = _I64
        L.fg8_colwise_capacity.argtypes = [_I64, _I]
        L.fg8_quantize_weight.restype = _I
        L.fg8_quantize_weight.argtypes = [_P, _I, _I, _I, _P, _P, _P, _P]
        L.fg8_quantize_weight_transposed.restype = _I
        L.fg8_quantize_weight_transposed.argtypes = [_P, _I, _I, _I, _P, _P, _P, _P, _P, _P]
        L.fg8_transpose_blockq.restype = _I
        L.fg8_transpose_blockq.argtypes = [_P, _P, _I, _I, _I, _P, _P, _P]
        L.fg8_grouped_gemm.restype = _I
        L.fg8_grouped_gemm.argtypes = [_P, _P, _P, _P, _P, _I64, _I, _I, _I, _I, _I, _I, _P, _P,
                                       _SZ, _P, _P]
        L.fg8_grouped_gemm_workspace.restype = _SZ
        L.fg8_grouped_gemm_workspace.argtypes = [_I]
        L.fg8_grouped_gemm_swiglu_quant.restype = _I
        L.fg8_grouped_gemm_swiglu_quant.argtypes = [_P, _P, _P, _P, _P, _I64, _I, _I, _I, _P, _P,
                                                    _P, _P]
        L.fg8_route_topk.restype = _I
        L.fg8_route_topk.argtypes = [_P, _P, _I64, _I, _I, _P, _P, _P]
        L.fg8_unpermute_combine.restype = _I
        L.fg8_unpermute_combine.argtypes = [_P, _I64, _I, _P, _P, _I64, _I, _I, _I, _P, _P]
        L.fg8_grouped_gemm_combine_workspace.restype = _SZ
        L.fg8_grouped_gemm_combine_workspace.argtypes = [_I64]
        L.fg8_grouped_gemm_combine.restype = _I
        L.fg8_grouped_gemm_combine.argtypes = [_P, _P, _P, _P, _P, _I64, _I, _I, _I, _P, _P, _P,
                                               _I64, _I, _I, _P, _P, _SZ, _P, _P]
        L.fg8_ep_pack_scales.restype = _I
        L.fg8_ep_pack_scales.argtypes = [_P, _I64, _I64, _P, _P]
        L.fg8_ep_unpack.restype = _I
        L.fg8_ep_unpack.argtypes = [_P, _P, _P, _I, _I, _I64, _I64, _P, _P, _P, _P, _P, _P]
        L.fg8_gather_rows.restype = _I
        L.fg8_gather_rows.argtypes = [_P, _I64, _I64, _P, _I64, _P, _P, _P]
        L.fg8_selftest_wait_timeout.restype = _I
        L.fg8_selftest_wait_timeout.argtypes = [_I, _P, _P, _P]
        L.fg8_status_string.restype = ctypes.c_char_p
        L.fg8_status_string.argtypes = [_I]
        _lib = L
    return _lib


def declared_symbols() -> list[str]:
    """Names of the functions include/fg8.h declares."""
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:[\w\s\*]+?)\b(fg8_\w+)\s*\(", text, flags=re.M)))


def status_name(status: int) -> str:
    return lib().fg8_status_string(int(status)).decode()


def _check(status: int, what: str) -> None:
    if status != FG8_OK:
        raise FG8Error(status, what)


def _ptr(t):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch.Tensor or None")
    if not t.is_cuda:
        raise ValueError("libfg8 takes CUDA tensors only (no CPU fallback)")
    if not t.is_contiguous():
        raise ValueError("libfg8 takes contiguous tensors")
    return t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


# --------------------------------------------------------------------------
# C-named entry points
# --------------------------------------------------------------------------

def fg8_quantize_act(x, T, K, topk_ids, k, E, offsets_in, layout, xq, sa, row_token, token_row,
                     offsets_out, xqT, saT, workspace, ws_bytes, dev_status, stream=None):
    _check(lib().fg8_quantize_act(_ptr(x), T, K, _ptr(topk_ids), k, E, _ptr(offsets_in), layout,
                                  _ptr(xq), _ptr(sa), _ptr(row_token), _ptr(token_row),
                                  _ptr(offsets_out), _ptr(xqT), _ptr(saT), _ptr(workspace),
                                  ws_bytes, _ptr(dev_status), _stream(stream)),
           "fg8_quantize_act")


def fg8_route_quantize_act(logits, bias, x, T, K, k, E, topk_ids, affinity, xq, sa, row_token,
                           token_row, offsets_out, workspace, ws_bytes, dev_status, stream=None):
    _check(lib().fg8_route_quantize_act(_ptr(logits), _ptr(bias), _ptr(x), T, K, k, E,
                                        _ptr(topk_ids), _ptr(affinity), _ptr(xq), _ptr(sa),
                                        _ptr(row_token), _ptr(token_row), _ptr(offsets_out),
                                        _ptr(workspace), ws_bytes, _ptr(dev_status),
                                        _stream(stream)),
           "fg8_route_quantize_act")


def fg8_quantize_act_noalloc(x, T, K, topk_ids, k, E, xq, sa, row_token, token_row, offsets_out,
                             dev_status, stream=None):
    """Permute + 1x128 quantize using the library's built-in scratch (no
    workspace argument, nothing allocated; E <= 256)."""
    _check(lib().fg8_quantize_act_noalloc(_ptr(x), T, K, _ptr(topk_ids), k, E, _ptr(xq), _ptr(sa),
                                          _ptr(row_token), _ptr(token_row), _ptr(offsets_out),
                                          _ptr(dev_status), _stream(stream)),
           "fg8_quantize_act_noalloc")


def fg8_quantize_act_workspace(T: int, k: int, E: int) -> int:
    return lib().fg8_quantize_act_workspace(T, k, E)


def fg8_colwise_capacity(R: int, E: int) -> int:
    return lib().fg8_colwise_capacity(R, E)


def fg8_quantize_weight_transposed(w, E, N, K, wq, sw, wqT, swT, dev_status=None, stream=None):
    _check(lib().fg8_quantize_weight_transposed(_ptr(w), E, N, K, _ptr(wq), _ptr(sw), _ptr(wqT),
                                                _ptr(swT), _ptr(dev_status), _stream(stream)),
           "fg8_quantize_weight_transposed")


def fg8_quantize_weight(w, E, N, K, wq, sw, dev_status=None, stream=None):
    _check(lib().fg8_quantize_weight(_ptr(w), E, N, K, _ptr(wq), _ptr(sw), _ptr(dev_status),
                                     _stream(stream)),
           "fg8_quantize_weight")


def fg8_transpose_blockq(wq, sw, E, N, K, wqT, swT, stream=None):
    _check(lib().fg8_transpose_blockq(_ptr(wq), _ptr(sw), E, N, K, _ptr(wqT), _ptr(swT),
                                      _stream(stream)),
           "fg8_transpose_blockq")


def fg8_grouped_gemm(a, sa, b, sb, offsets, M_total, N, K, E, group_mode, bscale_mode,
                     out_dtype, out, workspace, ws_bytes, dev_status, stream=None):
    _check(lib().fg8_grouped_gemm(_ptr(a), _ptr(sa), _ptr(b), _ptr(sb), _ptr(offsets), M_total,
                                  N, K, E, group_mode, bscale_mode, out_dtype, _ptr(out),
                                  _ptr(workspace), ws_bytes, _ptr(dev_status), _stream(stream)),
           "fg8_grouped_gemm")


def fg8_grouped_gemm_workspace(group_mode: int) -> int:
    return int(lib().fg8_grouped_gemm_workspace(group_mode))


def fg8_grouped_gemm_swiglu_quant(a, sa, b, sb, offsets, M_total, I, K, E, hq, sh, dev_status,
                                  stream=None):
    _check(lib().fg8_grouped_gemm_swiglu_quant(_ptr(a), _ptr(sa), _ptr(b), _ptr(sb), _ptr(offsets),
                                               M_total, I, K, E, _ptr(hq), _ptr(sh),
                                               _ptr(dev_status), _stream(stream)),
           "fg8_grouped_gemm_swiglu_quant")


def fg8_route_topk(logits, bias, T, E, k, ids, affinity, stream=None):
    _check(lib().fg8_route_topk(_ptr(logits), _ptr(bias), T, E, k, _ptr(ids), _ptr(affinity),
                                _stream(stream)),
           "fg8_route_topk")


def fg8_unpermute_combine(y, R, C, token_row, affinity, T, k, normalize, out_dtype, out,
                          stream=None):
    _check(lib().fg8_unpermute_combine(_ptr(y), R, C, _ptr(token_row), _ptr(affinity), T, k,
                                       normalize, out_dtype, _ptr(out), _stream(stream)),
           "fg8_unpermute_combine")


def fg8_grouped_gemm_combine_workspace(M_total: int) -> int:
    return int(lib().fg8_grouped_gemm_combine_workspace(M_total))


def fg8_grouped_gemm_combine(a, sa, b, sb, offsets, M_total, N, K, E, row_token, token_row,
                             affinity, T, k, normalize, out, workspace, ws_bytes, dev_status,
                             stream=None):
    _check(lib().fg8_grouped_gemm_combine(_ptr(a), _ptr(sa), _ptr(b), _ptr(sb), _ptr(offsets),
                                          M_total, N, K, E, _ptr(row_token), _ptr(token_row),
                                          _ptr(affinity), T, k, normalize, _ptr(out),
                                          _ptr(workspace), ws_bytes, _ptr(dev_status),
                                          _stream(stream)),
           "fg8_grouped_gemm_combine")


def fg8_ep_pack_scales(sa, R, K, sa_rows, stream=None):
    _check(lib().fg8_ep_pack_scales(_ptr(sa), R, K, _ptr(sa_rows), _stream(stream)),
           "fg8_ep_pack_scales")


def fg8_ep_unpack(recv_xq, recv_sa, counts, W, E_loc, R_recv, K, xq, sa, offsets, recv_to_local,
                  dev_status, stream=None):
    _check(lib().fg8_ep_unpack(_ptr(recv_xq), _ptr(recv_sa), _ptr(counts), W, E_loc, R_recv, K,
                               _ptr(xq), _ptr(sa), _ptr(offsets), _ptr(recv_to_local),
                               _ptr(dev_status), _stream(stream)),
           "fg8_ep_unpack")


def fg8_gather_rows(inp, n_in, row_bytes, map_, n, out, dev_status, stream=None):
    _check(lib().fg8_gather_rows(_ptr(inp), n_in, row_bytes, _ptr(map_), n, _ptr(out),
                                 _ptr(dev_status), _stream(stream)),
           "fg8_gather_rows")


def fg8_selftest_wait_timeout(which, scratch, dev_status, stream=None):
    _check(lib().fg8_selftest_wait_timeout(which, _ptr(scratch), _ptr(dev_status), _stream(stream)),
           "fg8_selftest_wait_timeout")


def fg8_status_string(status: int) -> str:
    return status_name(status)


# --------------------------------------------------------------------------
# allocate-and-call helpers
# --------------------------------------------------------------------------

def _u16(x: torch.Tensor) -> torch.Tensor:
    if x.dtype == torch.bfloat16:
        return x.view(torch.int16)
    if x.dtype in (torch.int16, torch.uint16):
        return x
    raise TypeError("expected bf16 data")


def new_status(device=None) -> torch.Tensor:
    return torch.zeros(1, dtype=torch.int32, device=device or "cuda")


def quantize_act(x: torch.Tensor, topk_ids: torch.Tensor, E: int, dev_status=None,
                 workspace=None, stream=None):
    """Permute + 1x128 quantize.  Returns dict(xq, sa, row_token, token_row, offsets)."""
    T, K = x.shape
    k = topk_ids.shape[1]
    R = T * k
    dev = x.device
    out = dict(
        xq=torch.empty((R, K), dtype=torch.uint8, device=dev),
        sa=torch.empty((K // 128, R), dtype=torch.float32, device=dev),
        row_token=torch.empty(R, dtype=torch.int32, device=dev),
        token_row=torch.empty(T * k, dtype=torch.int32, device=dev),
        offsets=torch.empty(E + 1, dtype=torch.int32, device=dev),
    )
    ws_bytes = fg8_quantize_act_workspace(T, k, E)
    if workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    st = dev_status if dev_status is not None else new_status(dev)
    fg8_quantize_act(_u16(x), T, K, topk_ids, k, E, None, FG8_ROWWISE, out["xq"], out["sa"],
                     out["row_token"], out["token_row"], out["offsets"], None, None, workspace,
                     ws_bytes, st, stream)
    out["status"] = st
    return out


def route_quantize_act(logits: torch.Tensor, bias: torch.Tensor, x: torch.Tensor, k: int,
                       dev_status=None, workspace=None, stream=None):
    """Routing (sigmoid + bias top-k) fused with permute + 1x128 quantize.
    Returns dict(ids, affinity, xq, sa, row_token, token_row, offsets, status)."""
    T, K = x.shape
    E = logits.shape[1]
    R = T * k
    dev = x.device
    out = dict(
        ids=torch.empty((T, k), dtype=torch.int32, device=dev),
        affinity=torch.empty((T, k), dtype=torch.float32, device=dev),
        xq=torch.empty((R, K), dtype=torch.uint8, device=dev),
        sa=torch.empty((K // 128, R), dtype=torch.float32, device=dev),
        row_token=torch.empty(R, dtype=torch.int32, device=dev),
        token_row=torch.empty(T * k, dtype=torch.int32, device=dev),
        offsets=torch.empty(E + 1, dtype=torch.int32, device=dev),
    )
    ws_bytes = fg8_quantize_act_workspace(T, k, E)
    if workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    st = dev_status if dev_status is not None else new_status(dev)
    fg8_route_quantize_act(logits, bias, _u16(x), T, K, k, E, out["ids"], out["affinity"],
                           out["xq"], out["sa"], out["row_token"], out["token_row"],
                           out["offsets"], workspace, ws_bytes, st, stream)
    out["status"] = st
    return out


def quantize_act_rows(x: torch.Tensor, stream=None):
    """1x128 quantize of rows already in expert order -> (xq [R,K], sa [K/128,R])."""
    R, K = x.shape
    xq = torch.empty((R, K), dtype=torch.uint8, device=x.device)
    sa = torch.empty((K // 128, R), dtype=torch.float32, device=x.device)
    fg8_quantize_act(_u16(x), R, K, None, 1, 1, None, FG8_ROWWISE, xq, sa, None, None, None,
                     None, None, None, 0, None, stream)
    return xq, sa


def quantize_act_colwise(x: torch.Tensor, offsets: torch.Tensor, k: int = 1,
                         row_token: torch.Tensor | None = None, stream=None):
    """Token-axis 1x128 quantization per expert -> (xqT [C,P], saT [P/128,C], padded offsets)."""
    T, C = x.shape
    E = offsets.numel() - 1
    R = T * k
    P = fg8_colwise_capacity(R, E)
    xqT = torch.empty((C, P), dtype=torch.uint8, device=x.device)
    saT = torch.empty((P // 128, C), dtype=torch.float32, device=x.device)
    padoff = torch.empty(E + 1, dtype=torch.int32, device=x.device)
    fg8_quantize_act(_u16(x), T, C, None, k, E, offsets, FG8_COLWISE, None, None, row_token,
                     None, padoff, xqT, saT, None, 0, None, stream)
    return xqT, saT, padoff


def quantize_weight(w: torch.Tensor, status=None, stream=None):
    """128x128 block quantize of bf16 w [E,N,K] -> (wq, sw [E,N/128,K/128])."""
    E, N, K = w.shape
    wq = torch.empty((E, N, K), dtype=torch.uint8, device=w.device)
    sw = torch.empty((E, N // 128, K // 128), dtype=torch.float32, device=w.device)
    fg8_quantize_weight(_u16(w), E, N, K, wq, sw, status, stream)
    return wq, sw


def quantize_weight_transposed(w: torch.Tensor, status=None, stream=None):
    """128x128 block quantize of bf16 w [E,N,K] plus its block-transposed copy
    -> (wq, sw, wqT [E,K,N], swT [E,K/128,N/128])."""
    E, N, K = w.shape
    wq = torch.empty((E, N, K), dtype=torch.uint8, device=w.device)
    sw = torch.empty((E, N // 128, K // 128), dtype=torch.float32, device=w.device)
    wqT = torch.empty((E, K, N), dtype=torch.uint8, device=w.device)
    swT = torch.empty((E, K // 128, N // 128), dtype=torch.float32, device=w.device)
    fg8_quantize_weight_transposed(_u16(w), E, N, K, wq, sw, wqT, swT, status, stream)
    return wq, sw, wqT, swT


def transpose_blockq(wq: torch.Tensor, sw: torch.Tensor, stream=None):
    E, N, K = wq.shape
    wqT = torch.empty((E, K, N), dtype=torch.uint8, device=wq.device)
    swT = torch.empty((E, K // 128, N // 128), dtype=torch.float32, device=wq.device)
    fg8_transpose_blockq(wq, sw, E, N, K, wqT, swT, stream)
    return wqT, swT


def grouped_gemm(a, sa, b, sb, offsets, out_dtype=FG8_OUT_BF16, group_mode=FG8_GROUP_M,
                 dev_status=None, out=None, stream=None, workspace=None):
    """Row-grouped: a [M,K], b [E,N,K] -> out [M,N].  Contraction-grouped:
    a [M,P], b [N,P] -> out [E,M,N] (its tile counter lives in `workspace`,
    allocated here when not given)."""
    M_total, K = a.shape
    E = offsets.numel() - 1
    if group_mode == FG8_GROUP_M:
        N = b.shape[1]
        shape = (M_total, N)
        bmode = FG8_BSCALE_BLOCK128
    else:
        N = b.shape[0]
        shape = (E, M_total, N)
        bmode = FG8_BSCALE_ROW128
    if out is None:
        dt = torch.float32 if out_dtype == FG8_OUT_F32 else torch.bfloat16
        out = torch.empty(shape, dtype=dt, device=a.device)
    ws_bytes = fg8_grouped_gemm_workspace(group_mode)
    if workspace is None and ws_bytes:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=a.device)
    fg8_grouped_gemm(a, sa, b, sb, offsets, M_total, N, K, E, group_mode, bmode, out_dtype, out,
                     workspace, ws_bytes if workspace is not None else 0, dev_status, stream)
    return out


def grouped_gemm_swiglu_quant(a, sa, b, sb, offsets, dev_status=None, hq=None, sh=None,
                              stream=None):
    """a [M,K] E4M3, b [E,2I,K] E4M3 (gate rows then up rows) -> (hq [M,I]
    E4M3, sh [I/128,M] fp32): the 1x128 quantization of silu(gate) * up."""
    M_total, K = a.shape
    E = offsets.numel() - 1
    I = b.shape[1] // 2
    if hq is None:
        hq = torch.empty((M_total, I), dtype=torch.uint8, device=a.device)
    if sh is None:
        sh = torch.empty((I // 128, M_total), dtype=torch.float32, device=a.device)
    fg8_grouped_gemm_swiglu_quant(a, sa, b, sb, offsets, M_total, I, K, E, hq, sh, dev_status,
                                  stream)
    return hq, sh


def grouped_gemm_combine(a, sa, b, sb, offsets, row_token, token_row, affinity, normalize=True,
                         dev_status=None, out=None, stream=None, workspace=None):
    """Row-grouped GEMM a [M,K] x b [E,N,K] with the combine in its epilogue:
    -> out fp32 [T, N], each token's rows weighted by its gate weights."""
    M_total, K = a.shape
    E, N = offsets.numel() - 1, b.shape[1]
    T, k = affinity.shape
    dev = a.device
    if out is None:
        out = torch.empty((T, N), dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = torch.empty(max(16, fg8_grouped_gemm_combine_workspace(M_total)),
                                dtype=torch.uint8, device=dev)
    st = dev_status if dev_status is not None else new_status(dev)
    fg8_grouped_gemm_combine(a, sa, b, sb, offsets, M_total, N, K, E, row_token, token_row,
                             affinity, T, k, int(bool(normalize)), out, workspace,
                             workspace.numel(), st, stream)
    return out


def unpermute_combine(y, token_row, affinity, normalize=True, out_dtype=FG8_OUT_BF16, out=None,
                      stream=None):
    """y bf16 [R, C] (permuted rows), token_row int32 [T*k], affinity fp32 [T, k]
    -> out [T, C]: each token's rows summed with its (normalized) gate weights."""
    R, C = y.shape
    T, k = affinity.shape
    if out is None:
        dt = torch.float32 if out_dtype == FG8_OUT_F32 else torch.bfloat16
        out = torch.empty((T, C), dtype=dt, device=affinity.device)
    yv = y.view(torch.int16) if y.dtype == torch.bfloat16 else y
    fg8_unpermute_combine(yv, R, C, token_row, affinity, T, k, int(bool(normalize)), out_dtype,
                          out, stream)
    return out


def route_topk(logits, bias, k, ids=None, affinity=None, stream=None):
    """logits fp32 [T, E], bias fp32 [E] -> (ids int32 [T, k], affinity fp32 [T, k])."""
    T, E = logits.shape
    if ids is None:
        ids = torch.empty((T, k), dtype=torch.int32, device=logits.device)
    if affinity is None:
        affinity = torch.empty((T, k), dtype=torch.float32, device=logits.device)
    fg8_route_topk(logits, bias, T, E, k, ids, affinity, stream)
    return ids, affinity
