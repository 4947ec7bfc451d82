"""CPU oracle for the FP8 fine-grained MoE path (test infrastructure only).

This package wraps `fg8_oracle.c`, a plain scalar C implementation of what the
path computes (see the header of that file for the definition and the
passages of the Kanana-2 and DeepSeek-V3 pages it follows).  Only the test
suite, the smoke check and the benchmark's CPU-baseline / reference leg may
import it.  It shares no code with the CUDA library and never calls it.

All arrays are numpy arrays on the host; bf16 data is passed as its uint16
bit pattern, E4M3 data as uint8.
"""

from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fg8_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math"]


def build(force: bool = False) -> str:
    """Compile fg8_oracle.c into liboracle.so next to it (gcc)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None

_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I = ctypes.c_int


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        L = _lib
        L.fg8o_e4m3_decode.restype = ctypes.c_double
        L.fg8o_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.fg8o_e4m3_encode.restype = ctypes.c_uint8
        L.fg8o_e4m3_encode.argtypes = [ctypes.c_float]
        L.fg8o_e4m3_encode_array.argtypes = [_P, _I64, _P]
        L.fg8o_tile_scale.restype = ctypes.c_float
        L.fg8o_tile_scale.argtypes = [ctypes.c_float]
        L.fg8o_route.restype = _I64
        L.fg8o_route.argtypes = [_P, _I64, _I, _I, _P, _P, _P, _P]
        L.fg8o_quantize_act_rowwise.restype = _I64
        L.fg8o_quantize_act_rowwise.argtypes = [_P, _I64, _I64, _P, _I, _I, _P, _P, _P, _P, _P]
        L.fg8o_quantize_act_colwise.argtypes = [_P, _I64, _P, _P, _I, _I64, _P, _P, _P]
        L.fg8o_quantize_weight.argtypes = [_P, _I64, _I64, _I64, _P, _P]
        L.fg8o_transpose_blockq.argtypes = [_P, _P, _I64, _I64, _I64, _P, _P]
        L.fg8o_gemm_mgrouped_entries.argtypes = [_P, _P, _I64, _P, _P, _P, _I, _I64, _I64,
                                                 _P, _P, _I64, _P, _P]
        L.fg8o_gemm_kgrouped_entries.argtypes = [_P, _P, _P, _P, _P, _I, _I64, _I64, _I64,
                                                 _P, _P, _P, _I64, _P, _P]
        L.fg8o_swiglu_quantize.argtypes = [_P, _P, _I64, _I64, _P, _P, _P]
        L.fg8o_unpermute_combine.argtypes = [_P, _I64, _I64, _P, _P, _I64, _I, _I, _P, _P]
        L.fg8o_route_topk.argtypes = [_P, _P, _I64, _I, _I, _P, _P, _P]
    return _lib


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data


def _u16(x) -> np.ndarray:
    """bf16 data (torch bf16 tensor or uint16/int16 array) -> uint16 array."""
    if hasattr(x, "view") and hasattr(x, "dtype") and str(x.dtype) == "torch.bfloat16":
        import torch
        return x.contiguous().view(torch.int16).numpy().view(np.uint16)
    a = np.ascontiguousarray(x)
    return a.view(np.uint16)


# --------------------------------------------------------------------------
# E4M3
# --------------------------------------------------------------------------

def e4m3_decode(code: int) -> float:
    return lib().fg8o_e4m3_decode(int(code))


def e4m3_decode_table() -> np.ndarray:
    return np.array([e4m3_decode(c) for c in range(256)], dtype=np.float64)


def e4m3_encode(v: float) -> int:
    return lib().fg8o_e4m3_encode(float(v))


def e4m3_encode_array(v: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.empty(v.shape, dtype=np.uint8)
    lib().fg8o_e4m3_encode_array(_ptr(v), v.size, _ptr(out))
    return out


def tile_scale(amax: float) -> float:
    return lib().fg8o_tile_scale(float(amax))


# --------------------------------------------------------------------------
# permute + quantize
# --------------------------------------------------------------------------

def route(ids: np.ndarray, E: int):
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    T, k = ids.shape
    counts = np.zeros(E, np.int32)
    offsets = np.zeros(E + 1, np.int32)
    row_token = np.full(T * k, -1, np.int32)
    token_row = np.full(T * k, -1, np.int32)
    bad = lib().fg8o_route(_ptr(ids), T, k, E, _ptr(counts), _ptr(offsets),
                           _ptr(row_token), _ptr(token_row))
    return dict(counts=counts, offsets=offsets, row_token=row_token,
                token_row=token_row, bad=int(bad))


def quantize_act(x, ids: np.ndarray | None, E: int):
    """Row-wise 1x128 quantization fused with the permute.

    x: bf16 [T, K].  ids: int32 [T, k] or None (identity).
    Returns dict(xq [R,K] u8, sa [K/128, R] f32, row_token, token_row, offsets, bad).
    """
    xu = _u16(x)
    T, K = xu.shape
    if ids is None:
        R, k, idp = T, 1, None
    else:
        ids = np.ascontiguousarray(ids, dtype=np.int32)
        k = ids.shape[1]
        R, idp = T * k, ids
    xq = np.zeros((R, K), np.uint8)
    sa = np.zeros((K // 128, R), np.float32)
    row_token = np.full(R, -1, np.int32)
    token_row = np.full(T * k, -1, np.int32)
    offsets = np.zeros(E + 1, np.int32)
    bad = lib().fg8o_quantize_act_rowwise(_ptr(xu), T, K, _ptr(idp), k, E, _ptr(xq), _ptr(sa),
                                          _ptr(row_token), _ptr(token_row), _ptr(offsets))
    return dict(xq=xq, sa=sa, row_token=row_token, token_row=token_row, offsets=offsets,
                bad=int(bad))


def colwise_capacity(R: int, E: int) -> int:
    """Width of the column-wise buffers: every expert padded to 128 rows."""
    return ((R + 127 * E + 127) // 128) * 128


def quantize_act_colwise(src, offsets: np.ndarray, row_map: np.ndarray | None = None,
                         P_cap: int | None = None):
    """Token-axis 1x128 quantization per expert (weight-gradient operands).

    src: bf16 [rows, C]; logical row r is src[row_map[r]] (or src[r]).
    Returns dict(xqT [C, P_cap] u8, sT [P_cap/128, C] f32, padoff [E+1] i32).
    """
    su = _u16(src)
    C = su.shape[1]
    offsets = np.ascontiguousarray(offsets, dtype=np.int32)
    E = offsets.size - 1
    R = int(offsets[E])
    if P_cap is None:
        P_cap = colwise_capacity(R, E)
    xqT = np.zeros((C, P_cap), np.uint8)
    sT = np.zeros((P_cap // 128, C), np.float32)
    padoff = np.zeros(E + 1, np.int32)
    rm = None if row_map is None else np.ascontiguousarray(row_map, dtype=np.int32)
    lib().fg8o_quantize_act_colwise(_ptr(su), C, _ptr(rm), _ptr(offsets), E, P_cap,
                                    _ptr(xqT), _ptr(sT), _ptr(padoff))
    return dict(xqT=xqT, sT=sT, padoff=padoff)


def quantize_weight(w):
    """128x128 block quantization of bf16 w [E, N, K] -> (wq u8, sw f32 [E, N/128, K/128])."""
    wu = _u16(w)
    E, N, K = wu.shape
    wq = np.zeros((E, N, K), np.uint8)
    sw = np.zeros((E, N // 128, K // 128), np.float32)
    lib().fg8o_quantize_weight(_ptr(wu), E, N, K, _ptr(wq), _ptr(sw))
    return wq, sw


def transpose_blockq(wq: np.ndarray, sw: np.ndarray):
    wq = np.ascontiguousarray(wq, dtype=np.uint8)
    sw = np.ascontiguousarray(sw, dtype=np.float32)
    E, N, K = wq.shape
    wqT = np.zeros((E, K, N), np.uint8)
    swT = np.zeros((E, K // 128, N // 128), np.float32)
    lib().fg8o_transpose_blockq(_ptr(wq), _ptr(sw), E, N, K, _ptr(wqT), _ptr(swT))
    return wqT, swT


# --------------------------------------------------------------------------
# GEMM references (fp64)
# --------------------------------------------------------------------------

def gemm_mgrouped_entries(a, sa, b, sb, offsets, rows, cols):
    """fp64 reference and |term| bound of the row-grouped product at (rows[i], cols[i])."""
    a = np.ascontiguousarray(a, np.uint8)
    sa = np.ascontiguousarray(sa, np.float32)
    b = np.ascontiguousarray(b, np.uint8)
    sb = np.ascontiguousarray(sb, np.float32)
    offsets = np.ascontiguousarray(offsets, np.int32)
    rows = np.ascontiguousarray(rows, np.int64)
    cols = np.ascontiguousarray(cols, np.int64)
    M_total, K = a.shape
    E, N, _ = b.shape
    ref = np.zeros(rows.size, np.float64)
    bound = np.zeros(rows.size, np.float64)
    lib().fg8o_gemm_mgrouped_entries(_ptr(a), _ptr(sa), M_total, _ptr(b), _ptr(sb),
                                     _ptr(offsets), E, N, K, _ptr(rows), _ptr(cols),
                                     rows.size, _ptr(ref), _ptr(bound))
    return ref, bound


def gemm_mgrouped_full(a, sa, b, sb, offsets):
    """All entries of the row-grouped product: ([M_total, N] ref, bound)."""
    M_total = a.shape[0]
    N = b.shape[1]
    r, c = np.meshgrid(np.arange(M_total), np.arange(N), indexing="ij")
    ref, bound = gemm_mgrouped_entries(a, sa, b, sb, offsets, r.ravel(), c.ravel())
    return ref.reshape(M_total, N), bound.reshape(M_total, N)


def swiglu_quantize(G, U):
    """h = silu(G) * U in fp64, quantized in 1x128 tiles from its fp32 rounding.

    G, U: fp64 [R, I].  Returns (h fp64 [R, I], hq u8 [R, I], sh f32 [I/128, R]).
    """
    G = np.ascontiguousarray(G, np.float64)
    U = np.ascontiguousarray(U, np.float64)
    R, I = G.shape
    h = np.zeros((R, I), np.float64)
    hq = np.zeros((R, I), np.uint8)
    sh = np.zeros((I // 128, R), np.float32)
    lib().fg8o_swiglu_quantize(_ptr(G), _ptr(U), R, I, _ptr(h), _ptr(hq), _ptr(sh))
    return h, hq, sh


def route_topk(logits, bias, k):
    """Sigmoid-affinity top-k with a per-expert bias, in fp64.

    logits fp32 [T, E], bias fp32 [E].  Returns (ids int32 [T, k],
    affinity fp64 [T, k], score fp64 [T, E] = sigmoid(logits) + bias).
    """
    logits = np.ascontiguousarray(logits, np.float32)
    bias = np.ascontiguousarray(bias, np.float32)
    T, E = logits.shape
    ids = np.zeros((T, k), np.int32)
    aff = np.zeros((T, k), np.float64)
    score = np.zeros((T, E), np.float64)
    lib().fg8o_route_topk(_ptr(logits), _ptr(bias), T, E, k, _ptr(ids), _ptr(aff), _ptr(score))
    return ids, aff, score


def unpermute_combine(y, token_row, affinity, normalize=True):
    """fp64 layer output of routed tokens and the |term| sum of every entry.

    y: bf16 [R, C] (uint16 bits or torch bf16); token_row int32 [T*k];
    affinity fp32 [T, k].  Returns (out fp64 [T, C], bound fp64 [T, C]).
    """
    yu = _u16(y)
    R, C = yu.shape
    affinity = np.ascontiguousarray(affinity, np.float32)
    token_row = np.ascontiguousarray(token_row, np.int32)
    T, k = affinity.shape
    out = np.zeros((T, C), np.float64)
    bound = np.zeros((T, C), np.float64)
    lib().fg8o_unpermute_combine(_ptr(yu), R, C, _ptr(token_row), _ptr(affinity), T, k,
                                 int(bool(normalize)), _ptr(out), _ptr(bound))
    return out, bound


def gemm_kgrouped_entries(a, sa, b, sb, padoff, experts, rows, cols):
    a = np.ascontiguousarray(a, np.uint8)
    sa = np.ascontiguousarray(sa, np.float32)
    b = np.ascontiguousarray(b, np.uint8)
    sb = np.ascontiguousarray(sb, np.float32)
    padoff = np.ascontiguousarray(padoff, np.int32)
    experts = np.ascontiguousarray(experts, np.int64)
    rows = np.ascontiguousarray(rows, np.int64)
    cols = np.ascontiguousarray(cols, np.int64)
    M, P_cap = a.shape
    N = b.shape[0]
    E = padoff.size - 1
    ref = np.zeros(rows.size, np.float64)
    bound = np.zeros(rows.size, np.float64)
    lib().fg8o_gemm_kgrouped_entries(_ptr(a), _ptr(sa), _ptr(b), _ptr(sb), _ptr(padoff), E,
                                     M, N, P_cap, _ptr(experts), _ptr(rows), _ptr(cols),
                                     rows.size, _ptr(ref), _ptr(bound))
    return ref, bound
