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


def gemm_combine_entries(a, sa, b, sb, offsets, token_row, affinity, tokens, cols,
                         normalize=True):
    """The down-projection followed by the combine, at (tokens[i], cols[i]):
        out[t][c] = sum over the token's kept slots j of w[t][j] * Y[row_j][c]
    with Y the row-grouped product (its fp64 reference, gemm_mgrouped_entries)
    and w the combine's gate weights (the kept affinities, normalized to sum 1
    over the kept slots when `normalize`; a slot is kept when its row is in
    [0, offsets[E])).  Returns (out fp64, bound fp64 = sum |w| * the GEMM's
    |term| bound, mag fp64 = sum |w * Y|) per requested entry."""
    offsets = np.ascontiguousarray(offsets, np.int32)
    affinity = np.ascontiguousarray(affinity, np.float32)
    T, k = affinity.shape
    tr = np.ascontiguousarray(token_row, np.int32).reshape(T, k)
    tokens = np.asarray(tokens, np.int64)
    cols = np.asarray(cols, np.int64)
    R = int(offsets[-1])
    kept = (tr >= 0) & (tr < R)
    aff = affinity.astype(np.float64)
    sums = np.where(kept, aff, 0.0).sum(axis=1)
    if normalize:
        w = np.where(kept & (sums[:, None] != 0), aff / np.where(sums == 0, 1.0, sums)[:, None], 0.0)
    else:
        w = np.where(kept, aff, 0.0)
    # one GEMM entry per (requested entry, kept slot)
    ent, slot = np.nonzero(kept[tokens])
    rows = tr[tokens[ent], slot].astype(np.int64)
    ref, bnd = gemm_mgrouped_entries(a, sa, b, sb, offsets, rows, cols[ent])
    wt = w[tokens[ent], slot]
    out = np.zeros(tokens.size, np.float64)
    bound = np.zeros(tokens.size, np.float64)
    mag = np.zeros(tokens.size, np.float64)
    np.add.at(out, ent, wt * ref)
    np.add.at(bound, ent, np.abs(wt) * bnd)
    np.add.at(mag, ent, np.abs(wt * ref))
    return out, bound, mag


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


# --------------------------------------------------------------------------
# threaded drivers
#
# The same C functions as above, each called on disjoint slices of the input
# from a pool of threads (ctypes releases the GIL for the duration of a call,
# so the calls run in parallel).  Every thread runs the plain scalar loop of
# the function it calls; the drivers only cut the work into independent pieces
# (experts, rows or 128-column groups, which the method never couples) and
# place each piece's results where the single call would have put them.
# --------------------------------------------------------------------------

def threads() -> int:
    """Threads the drivers use: FG8_ORACLE_THREADS, else the usable cores."""
    env = os.environ.get("FG8_ORACLE_THREADS")
    if env:
        return max(1, int(env))
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:
        return max(1, os.cpu_count() or 1)


def _run(jobs, nthreads=None):
    """Run the zero-argument callables `jobs` on a thread pool; re-raise errors."""
    from concurrent.futures import ThreadPoolExecutor
    n = nthreads or threads()
    if n <= 1 or len(jobs) <= 1:
        for j in jobs:
            j()
        return
    with ThreadPoolExecutor(max_workers=n) as ex:
        for f in [ex.submit(j) for j in jobs]:
            f.result()


def _pieces(n: int, parts: int, quantum: int = 1):
    """Split range(n) into at most `parts` contiguous pieces, boundaries on
    multiples of `quantum`."""
    units = (n + quantum - 1) // quantum
    parts = max(1, min(parts, units))
    cuts = [min(n, (units * i // parts) * quantum) for i in range(parts + 1)]
    return [(cuts[i], cuts[i + 1]) for i in range(parts) if cuts[i + 1] > cuts[i]]


def quantize_weight_threaded(w, nthreads=None):
    """quantize_weight over expert slices (E > 1) or 128-row slabs (E == 1)."""
    wu = _u16(w)
    E, N, K = wu.shape
    wq = np.zeros((E, N, K), np.uint8)
    sw = np.zeros((E, N // 128, K // 128), np.float32)
    n = nthreads or threads()
    jobs = []
    if E >= n:
        for e0, e1 in _pieces(E, 4 * n):
            jobs.append(lambda e0=e0, e1=e1: lib().fg8o_quantize_weight(
                _ptr(wu[e0:e1]), e1 - e0, N, K, _ptr(wq[e0:e1]), _ptr(sw[e0:e1])))
    else:
        for e in range(E):
            for n0, n1 in _pieces(N, 4 * n, 128):
                jobs.append(lambda e=e, n0=n0, n1=n1: lib().fg8o_quantize_weight(
                    _ptr(wu[e, n0:n1]), 1, n1 - n0, K, _ptr(wq[e, n0:n1]),
                    _ptr(sw[e, n0 // 128:n1 // 128])))
    _run(jobs, n)
    return wq, sw


def transpose_blockq_threaded(wq: np.ndarray, sw: np.ndarray, nthreads=None):
    """transpose_blockq over expert slices."""
    wq = np.ascontiguousarray(wq, dtype=np.uint8)
    sw = np.ascontiguousarray(sw, dtype=np.float32)
    E, N, K = wq.shape
    wqT = np.zeros((E, K, N), np.uint8)
    swT = np.zeros((E, K // 128, N // 128), np.float32)
    jobs = [lambda e=e: lib().fg8o_transpose_blockq(_ptr(wq[e]), _ptr(sw[e]), 1, N, K,
                                                    _ptr(wqT[e]), _ptr(swT[e]))
            for e in range(E)]
    _run(jobs, nthreads)
    return wqT, swT


def quantize_rows_threaded(x, nthreads=None):
    """Identity-mode quantize_act (rows already in expert order) over row slices:
    returns (xq [R, K] u8, sa [K/128, R] f32)."""
    xu = _u16(x)
    R, K = xu.shape
    xq = np.zeros((R, K), np.uint8)
    sa = np.zeros((K // 128, R), np.float32)
    n = nthreads or threads()

    def job(r0, r1):
        s = np.zeros((K // 128, r1 - r0), np.float32)
        rt = np.full(r1 - r0, -1, np.int32)
        tr = np.full(r1 - r0, -1, np.int32)
        off = np.zeros(2, np.int32)
        lib().fg8o_quantize_act_rowwise(_ptr(xu[r0:r1]), r1 - r0, K, None, 1, 1, _ptr(xq[r0:r1]),
                                        _ptr(s), _ptr(rt), _ptr(tr), _ptr(off))
        sa[:, r0:r1] = s
    _run([lambda r0=r0, r1=r1: job(r0, r1) for r0, r1 in _pieces(R, 4 * n)], n)
    return xq, sa


def quantize_act_colwise_threaded(src, offsets: np.ndarray, row_map: np.ndarray | None = None,
                                  P_cap: int | None = None, nthreads=None):
    """quantize_act_colwise over groups of 128 columns (every column is
    quantized on its own, so the groups are independent)."""
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
    n = nthreads or threads()

    def job(c0, c1):
        part = np.ascontiguousarray(su[:, c0:c1])
        s = np.zeros((P_cap // 128, c1 - c0), np.float32)
        pad = np.zeros(E + 1, np.int32)
        lib().fg8o_quantize_act_colwise(_ptr(part), c1 - c0, _ptr(rm), _ptr(offsets), E, P_cap,
                                        _ptr(xqT[c0:c1]), _ptr(s), _ptr(pad))
        sT[:, c0:c1] = s
        if c0 == 0:
            padoff[:] = pad
    _run([lambda c0=c0, c1=c1: job(c0, c1) for c0, c1 in _pieces(C, 4 * n, 128)], n)
    return dict(xqT=xqT, sT=sT, padoff=padoff)


def gemm_mgrouped_entries_threaded(a, sa, b, sb, offsets, rows, cols, nthreads=None):
    """gemm_mgrouped_entries over slices of the entry list."""
    rows = np.ascontiguousarray(rows, np.int64)
    cols = np.ascontiguousarray(cols, np.int64)
    a = np.ascontiguousarray(a, np.uint8)
    sa = np.ascontiguousarray(sa, np.float32)
    b = np.ascontiguousarray(b, np.uint8)
    sb = np.ascontiguousarray(sb, np.float32)
    offsets = np.ascontiguousarray(offsets, np.int32)
    M_total, K = a.shape
    E, N, _ = b.shape
    ref = np.zeros(rows.size, np.float64)
    bound = np.zeros(rows.size, np.float64)
    n = nthreads or threads()
    jobs = [lambda i0=i0, i1=i1: lib().fg8o_gemm_mgrouped_entries(
        _ptr(a), _ptr(sa), M_total, _ptr(b), _ptr(sb), _ptr(offsets), E, N, K,
        _ptr(rows[i0:i1]), _ptr(cols[i0:i1]), i1 - i0, _ptr(ref[i0:i1]), _ptr(bound[i0:i1]))
        for i0, i1 in _pieces(rows.size, 4 * n)]
    _run(jobs, n)
    return ref, bound


def gemm_dense_fp64(a, sa, b, sb):
    """All entries of the single-group product (E = 1) and their |term| sums:
        out[r][n] = sum_k dq(a[r][k]) sa[k/128][r] * dq(b[n][k]) sb[n/128][k/128]
    written as one fp64 matrix product of the dequantized operands (numpy's
    matmul is the library step).  Every dequantized operand is exact in fp64
    (a 4-bit code times a 24-bit scale); the products and the sum round at
    2^-53, far below the GEMM tolerance.

    a u8 [M, K], sa f32 [K/128, M], b u8 [N, K] (or [1, N, K]), sb f32
    [N/128, K/128] (or [1, ...]).  Returns (ref fp64 [M, N], bound fp64 [M, N]).
    """
    a = np.ascontiguousarray(a, np.uint8)
    b = np.ascontiguousarray(b, np.uint8).reshape(-1, a.shape[1])
    sa = np.asarray(sa, np.float32)
    sb = np.asarray(sb, np.float32).reshape(b.shape[0] // 128, a.shape[1] // 128)
    dq = e4m3_decode_table()
    A = dq[a] * np.repeat(sa.T.astype(np.float64), 128, axis=1)
    B = dq[b] * np.repeat(np.repeat(sb.astype(np.float64), 128, axis=0), 128, axis=1)
    return A @ B.T, np.abs(A) @ np.abs(B).T


# --------------------------------------------------------------------------
# expert-parallel exchange (index work, written out with plain loops)
# --------------------------------------------------------------------------

def ep_dispatch(sources, W: int):
    """Where every routed row lands when the E experts are spread over W ranks
    (rank r owns experts [r E/W, (r + 1) E/W)).

    sources: per source rank s, (xq u8 [R_s, K], sa f32 [K/128, R_s], offsets
    [E + 1]) of its rows grouped by expert.  Rank r receives, for each of its
    experts in ascending order, that expert's rows from source 0, then source
    1, ..., each source's rows in their own order.  Returns, per rank r,
    dict(xq [n, K], sa [K/128, n], offsets [E/W + 1], origin int64 [n, 2] =
    (source, source row) of each local row).
    """
    E = len(sources[0][2]) - 1
    EL = E // W
    K = sources[0][0].shape[1]
    out = []
    for r in range(W):
        origin = []
        offs = [0]
        for el in range(EL):
            e = r * EL + el
            for s, (_, _, off) in enumerate(sources):
                for i in range(int(off[e]), int(off[e + 1])):
                    origin.append((s, i))
            offs.append(len(origin))
        n = len(origin)
        xq = np.zeros((n, K), np.uint8)
        sa = np.zeros((K // 128, n), np.float32)
        for j, (s, i) in enumerate(origin):
            xq[j] = sources[s][0][i]
            sa[:, j] = sources[s][1][:, i]
        out.append(dict(xq=xq, sa=sa, offsets=np.array(offs, np.int32),
                        origin=np.array(origin, np.int64).reshape(n, 2)))
    return out


def ep_combine(y_locals, dispatched, rows_per_source):
    """The reverse trip: y_locals[r] [n_r, C] are rank r's outputs of its local
    rows (dispatched[r]["origin"] says where each came from).  Returns, per
    source s, [rows_per_source[s], C]: each of its rows' outputs in its own
    row order (rows that went nowhere stay zero)."""
    C = y_locals[0].shape[1:]
    back = [np.zeros((n,) + C, y_locals[0].dtype) for n in rows_per_source]
    for r, d in enumerate(dispatched):
        for j, (s, i) in enumerate(d["origin"]):
            back[s][i] = y_locals[r][j]
    return back
