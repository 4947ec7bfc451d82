#!/usr/bin/env python
"""Benchmark of the FP8 fine-grained MoE path on B200.

One step = one pass of the whole path over one batch of the DeepSeek-V3-shaped
MoE layer (256 experts, hidden 7168, inter 2048, 8192 tokens top-8, Zipf(1.2)
routing with 16 empty experts), forward and backward shapes:

  K1  permute + 1x128 quantize X [8192, 7168]            (fg8_quantize_act, rowwise)
  K2  128x128 quantize W_up [256, 4096, 7168], W_down [256, 7168, 2048]
  K4  fprop up    Y_up   = Xq  . Wq_up^T     -> bf16 [65536, 4096]
  K1  1x128 quantize H [65536, 2048] (down-projection input, in expert order)
  K4  fprop down  Y_down = Hq  . Wq_down^T   -> bf16 [65536, 7168]
  K3  transpose Wq_up -> WqT_up [256, 7168, 4096] (+ scale grid)
  K1  1x128 quantize dY [65536, 4096]
  K4  dgrad       dX     = dYq . WqT_up^T    -> bf16 [65536, 7168]
  K1  column-wise quantize dY and X (gathered by row) along tokens, per expert
  K4  wgrad       dW_e   = dY_e^T X_e        -> fp32 [256, 4096, 7168]

The printed `value` is the grouped FP8 GEMM throughput (algorithmic FLOPs of
the four GEMMs over their summed kernel time, CUDA events on the launching
stream); `quantize_gbs` is the same for the bandwidth kernels.  `roofline`
describes the kernel with the largest share of the step; `kernels` lists
every kernel against its own roofline.

`--impl reference` times the CPU oracle (the reference implementation of what
the path computes) on a bounded sample of the same workload.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from fp8_fine_grained_permute_b200 import workloads as W  # noqa: E402

METRIC = "grouped FP8 GEMM TFLOP/s + quantize GB/s, % of B200 FP8/HBM roofline"
FP8_OVER_BF16 = 2.0          # nominal dense FP8 / BF16 tensor throughput ratio on B200
# nominal B200 figures (context next to the measured peaks): HBM3e bandwidth
# and dense (non-sparse) FP8 tensor throughput
NOMINAL = {"hbm_gbs": 8000.0, "fp8_tflops": 4500.0}
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return dict(hbm_gbs=float(p["hbm_gbs"]), bf16=float(p["bf16_tflops"]),
                    bf16_sus=float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                    source="measured")
    return dict(hbm_gbs=FALLBACK["hbm_gbs"], bf16=FALLBACK["bf16_tflops"],
                bf16_sus=FALLBACK["bf16_tflops_sustained"], source="fallback")


# --------------------------------------------------------------------------
# algorithmic work per kernel launch (bytes the method must move, FLOPs it must do)
# --------------------------------------------------------------------------

def bytes_route_quant(T, K, k, E):
    R = T * k
    return 2 * T * K + R * K + 4 * R * K // 128 + 4 * T * k + 8 * R + 4 * (E + 1)


def bytes_rows_quant(R, K):
    return 2 * R * K + R * K + 4 * R * K // 128


def bytes_colwise(read_rows, C, padded_total):
    return 2 * read_rows * C + padded_total * C + 4 * padded_total * C // 128


def bytes_weight_quant(E, N, K):
    return 3 * E * N * K + 4 * E * N * K // 16384


def bytes_transpose(E, N, K):
    return 2 * (E * N * K + 4 * E * N * K // 16384)


def bytes_route_quantize(T, K, k, E):
    """Routing fused with the permuting quantizer: the router logits in, the
    ids and affinities out, plus the permute + quantize bytes."""
    return 4 * T * E + 4 * E + 8 * T * k + bytes_route_quant(T, K, k, E)


def bytes_combine(T, k, C):
    """Unpermute + combine: the k routed bf16 rows of every token in, its bf16
    row out, plus the row index and affinity of every slot."""
    return T * k * C * 2 + T * C * 2 + T * k * 8


def nominal_of(entry: dict) -> dict:
    """Add the fraction of the nominal peak beside the measured one."""
    nom = NOMINAL["hbm_gbs"] if entry["unit"] == "GB/s" else NOMINAL["fp8_tflops"]
    entry["nominal_peak"] = nom
    entry["frac_of_nominal"] = entry["achieved"] / nom
    if "tflops" in entry:     # an HBM-bound GEMM: its FLOP rate against the nominal FP8 peak too
        entry["tensor_frac_of_nominal"] = entry["tflops"] / NOMINAL["fp8_tflops"]
    return entry


def padded_total_of(cfg: W.MoEConfig) -> int:
    counts = np.bincount(W.route(cfg).ravel(), minlength=cfg.E)
    return int(((counts + 127) // 128 * 128).sum())


def work_of(cfg: W.MoEConfig, padded_total: int, fused_act: bool = False):
    """Per kernel family of one step: (bound, algorithmic amount) and, for the
    GEMMs, the bytes they must move at least (operands once, output once).
    fused_act: the up-projection emits the quantized gated activation (E4M3
    codes and 1x128 scales of H) instead of bf16 Y, and H is not quantized
    separately."""
    T, K, k, E, R, N, I = cfg.T, cfg.hidden, cfg.k, cfg.E, cfg.R, cfg.n_up, cfg.inter
    w = {
        "quant_act_permute": ("hbm", bytes_route_quant(T, K, k, E)),
        # up weight: quantized with its block-transposed copy written in the same
        # pass (one more byte per element and a scale per block)
        "quant_weight": ("hbm", bytes_weight_quant(E, N, K) + E * N * K + 4 * E * (N // 128) * (K // 128)
                         + (bytes_weight_quant(E, K, I) if I else 0)),
        "gemm_fprop_up": ("tensor", 2 * R * N * K),
        "quant_act_rows": ("hbm", bytes_rows_quant(R, N) + (bytes_rows_quant(R, I) if I else 0)),
        "gemm_dgrad": ("tensor", 2 * R * K * N),
        "quant_act_colwise": ("hbm", bytes_colwise(R, N, padded_total) + bytes_colwise(T, K, padded_total)),
        "gemm_wgrad": ("tensor", 2 * R * N * K),
    }
    gemm_bytes = {
        "gemm_fprop_up": R * K + E * N * K + 2 * R * N,
        "gemm_dgrad": R * N + E * K * N + 2 * R * K,
        "gemm_wgrad": (N + K) * padded_total + 4 * E * N * K,
    }
    if I:
        w["gemm_fprop_down"] = ("tensor", 2 * R * K * I)
        gemm_bytes["gemm_fprop_down"] = R * I + E * K * I + 2 * R * K
    if fused_act and I:
        del w["gemm_fprop_up"], gemm_bytes["gemm_fprop_up"]
        w["gemm_fprop_up_swiglu_quant"] = ("tensor", 2 * R * N * K)
        gemm_bytes["gemm_fprop_up_swiglu_quant"] = R * K + E * N * K + R * I + 4 * R * (I // 128)
        w["quant_act_rows"] = ("hbm", bytes_rows_quant(R, N))
    return w, gemm_bytes


# DRAM bytes (read + write) per kernel family of one step: the launch list of
# the DeepSeek-V3-shaped step (`ncu --metrics gpu__time_duration.sum,
# dram__bytes_read.sum,dram__bytes_write.sum`, one replay pass, the bench's own
# launches with `--steps 1 --warmup 1`; the standalone kernels' first launch).
# They are scaled to another workload by the ratio of algorithmic bytes, and
# dropped (traffic: null) when the kernel sources differ from the ones the
# counters were taken on (short sha1 of the code of the kernel file and shared
# headers, comments and whitespace removed).
TRAFFIC_CAPTURE = {
    "config": "dsv3",
    "fused_act": True,
    "families": {
        "quant_act_permute": (598.5e6, "quant_act", "c5187dc2015d"),
        "quant_weight": (41280.4e6, "quant_weight", "c5689f11fc37"),
        "gemm_fprop_up_swiglu_quant": (7836.7e6, "gemm", "7d78004fde39"),
        "quant_act_rows": (777.8e6, "quant_act", "c5187dc2015d"),
        "gemm_fprop_down": (4594.1e6, "gemm", "7d78004fde39"),
        "gemm_dgrad": (8393.9e6, "gemm", "7d78004fde39"),
        "quant_act_colwise": (1573.4e6, "quant_act", "c5187dc2015d"),
        "gemm_wgrad": (31920.1e6, "gemm", "7d78004fde39"),
        "transpose_blockq": (14976.3e6, "transpose", "3f2c2c5f91b7"),
        "gemm_fprop_up": (8460.5e6, "gemm", "7d78004fde39"),
        "unpermute_combine": (1044.5e6, "combine", "641810fdcb7b"),
    },
}
# the files each family's counters depend on; fg8_common.cuh is added unless
# the group lists its own headers (the transpose uses none of its device code
# but one unchanged load helper)
_SRC = {"quant_act": ["quant_act.cu", "fg8_tma.cuh"], "quant_weight": ["quant_weight.cu", "fg8_tma.cuh"],
        "transpose": ["transpose_blockq.cu"], "gemm": ["grouped_gemm.cu", "fg8_tma.cuh"],
        "combine": ["combine.cu"]}
_OWN_HEADERS = {"transpose"}


def code_of(text: str) -> str:
    """C/CUDA source without comments and blank space (what the counters
    depend on): string literals are kept, // and /* */ comments dropped, runs
    of whitespace folded."""
    import re
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c == '"':
            j = i + 1
            while j < n and text[j] != '"':
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    return re.sub(r"\s+", " ", "".join(out)).strip()


def source_hash(group: str) -> str:
    import hashlib
    h = hashlib.sha1()
    base = os.path.join(ROOT, "fp8_fine_grained_permute_b200", "csrc")
    for f in _SRC[group] + ([] if group in _OWN_HEADERS else ["fg8_common.cuh"]):
        with open(os.path.join(base, f), encoding="utf-8") as fh:
            h.update(code_of(fh.read()).encode())
    return h.hexdigest()[:12]


def algorithmic_bytes(family: str, cfg: W.MoEConfig, padded_total: int, fused_act: bool = True) -> float:
    """The bytes a family must move on `cfg` (GEMMs: operands + output once)."""
    if family == "transpose_blockq":
        return bytes_transpose(cfg.E, cfg.n_up, cfg.hidden)
    if family == "unpermute_combine":
        return bytes_combine(cfg.T, cfg.k, cfg.hidden)
    if family == "gemm_fprop_up_swiglu_quant":
        R, K, I = cfg.R, cfg.hidden, cfg.inter
        return R * K + cfg.E * cfg.n_up * K + R * I + 4 * R * (I // 128)
    if family == "gemm_fprop_up":   # bf16 Y out (in the step only without the fused activation)
        R, K, N = cfg.R, cfg.hidden, cfg.n_up
        return R * K + cfg.E * N * K + 2 * R * N
    w, gb = work_of(cfg, padded_total, fused_act)
    return gb.get(family, w[family][1])


def measured_traffic(family: str, cfg: W.MoEConfig, padded_total: int, fused_act: bool = True):
    entry = TRAFFIC_CAPTURE["families"].get(family)
    if entry is None:
        return None
    bytes_cap, group, sha = entry
    if source_hash(group) != sha:
        return None
    if family == "quant_act_rows" and fused_act != TRAFFIC_CAPTURE["fused_act"]:
        return None   # the other step variant quantizes a different set of rows
    cap = W.CONFIGS[TRAFFIC_CAPTURE["config"]]
    fa = TRAFFIC_CAPTURE["fused_act"]
    return bytes_cap * algorithmic_bytes(family, cfg, padded_total, fa) / \
        algorithmic_bytes(family, cap, padded_total_of(cap), fa)


# --------------------------------------------------------------------------
# the workload on one GPU
# --------------------------------------------------------------------------

class Step:
    """Device-resident inputs and outputs of one step; `run` launches the path."""

    def __init__(self, cfg: W.MoEConfig, dev, fused_act: bool = False):
        from fp8_fine_grained_permute_b200 import fg8
        self.fg8 = fg8
        self.cfg = cfg
        self.dev = dev
        self.fused_act = bool(fused_act and cfg.inter)
        T, K, k, E, R = cfg.T, cfg.hidden, cfg.k, cfg.E, cfg.R
        N, I = cfg.n_up, cfg.inter
        self.ids_np = W.route(cfg)
        counts = np.bincount(self.ids_np.ravel(), minlength=E)
        self.padded_total = int(((counts + 127) // 128 * 128).sum())
        u8, f32, i32, bf = torch.uint8, torch.float32, torch.int32, torch.bfloat16
        e = lambda shape, dt: torch.empty(shape, dtype=dt, device=dev)  # noqa: E731
        # inputs (generated on the device by the seeded counter-based generators)
        self.x = W.gen_x(cfg, dev)
        self.ids = torch.from_numpy(self.ids_np).to(dev)
        self.w_up = W.gen_w_up(cfg, dev)
        self.w_down = W.gen_w_down(cfg, dev) if I else None
        self.h = W.gen_h(cfg, dev) if I and not self.fused_act else None
        self.dy = W.gen_dy(cfg, dev)
        # outputs / intermediates
        self.xq, self.sa = e((R, K), u8), e((K // 128, R), f32)
        self.row_token, self.token_row = e(R, i32), e(T * k, i32)
        self.offsets = e(E + 1, i32)
        self.ws_bytes = fg8.fg8_quantize_act_workspace(T, k, E)
        self.ws = e(self.ws_bytes, u8)
        self.status = torch.zeros(1, dtype=i32, device=dev)
        self.wq_up, self.sw_up = e((E, N, K), u8), e((E, N // 128, K // 128), f32)
        self.y_up = e((R, N), bf) if not self.fused_act else None
        if I:
            self.wq_dn, self.sw_dn = e((E, K, I), u8), e((E, K // 128, I // 128), f32)
            self.hq, self.sh = e((R, I), u8), e((I // 128, R), f32)
            self.y_dn = e((R, K), bf)
        self.wqT_up, self.swT_up = e((E, K, N), u8), e((E, K // 128, N // 128), f32)
        self.dyq, self.sdy = e((R, N), u8), e((N // 128, R), f32)
        self.dx = e((R, K), bf)
        self.P = fg8.fg8_colwise_capacity(R, E)
        self.dyT, self.sdyT, self.pad_dy = e((N, self.P), u8), e((self.P // 128, N), f32), e(E + 1, i32)
        self.xT, self.sxT, self.pad_x = e((K, self.P), u8), e((self.P // 128, K), f32), e(E + 1, i32)
        self.dw = e((E, N, K), f32)
        self.gemm_ws = e(max(16, fg8.fg8_grouped_gemm_workspace(fg8.FG8_GROUP_K)), u8)
        self.launches_per_step = 0
        self.work, self.gemm_bytes = work_of(cfg, self.padded_total, self.fused_act)

    def run(self, stream, marks=None):
        """Launch one step on `stream`.  With `marks`, record an event pair
        around each kernel family: marks[name] -> list of (start, end)."""
        fg8, c = self.fg8, self.cfg
        T, K, k, E, R, N, I = c.T, c.hidden, c.k, c.E, c.R, c.n_up, c.inter
        sp = stream.cuda_stream
        n = [0]

        def timed(name, fn):
            if marks is not None:
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                fn()
                b.record(stream)
                marks.setdefault(name, []).append((a, b))
            else:
                fn()

        def launch(fn):
            def g():
                fn()
                n[0] += 1
            return g

        u16 = lambda t: t.view(torch.int16)  # noqa: E731
        timed("quant_act_permute", launch(lambda: fg8.fg8_quantize_act(
            u16(self.x), T, K, self.ids, k, E, None, fg8.FG8_ROWWISE, self.xq, self.sa,
            self.row_token, self.token_row, self.offsets, None, None, self.ws, self.ws_bytes,
            self.status, sp)))

        def wquant():
            fg8.fg8_quantize_weight_transposed(u16(self.w_up), E, N, K, self.wq_up, self.sw_up,
                                               self.wqT_up, self.swT_up, self.status, sp)
            n[0] += 1
            if I:
                fg8.fg8_quantize_weight(u16(self.w_down), E, K, I, self.wq_dn, self.sw_dn, self.status, sp)
                n[0] += 1
        timed("quant_weight", wquant)
        if self.fused_act:
            timed("gemm_fprop_up_swiglu_quant", launch(lambda: self.run_fused_up(stream)))
        else:
            timed("gemm_fprop_up", launch(lambda: fg8.fg8_grouped_gemm(
                self.xq, self.sa, self.wq_up, self.sw_up, self.offsets, R, N, K, E, fg8.FG8_GROUP_M,
                fg8.FG8_BSCALE_BLOCK128, fg8.FG8_OUT_BF16, self.y_up, None, 0, self.status, sp)))

        def rows():
            if I and not self.fused_act:
                fg8.fg8_quantize_act(u16(self.h), R, I, None, 1, 1, None, fg8.FG8_ROWWISE, self.hq,
                                     self.sh, None, None, None, None, None, None, 0, None, sp)
                n[0] += 1
            fg8.fg8_quantize_act(u16(self.dy), R, N, None, 1, 1, None, fg8.FG8_ROWWISE, self.dyq,
                                 self.sdy, None, None, None, None, None, None, 0, None, sp)
            n[0] += 1
        timed("quant_act_rows", rows)
        if I:
            timed("gemm_fprop_down", launch(lambda: fg8.fg8_grouped_gemm(
                self.hq, self.sh, self.wq_dn, self.sw_dn, self.offsets, R, K, I, E,
                fg8.FG8_GROUP_M, fg8.FG8_BSCALE_BLOCK128, fg8.FG8_OUT_BF16, self.y_dn,
                None, 0, self.status, sp)))
        timed("gemm_dgrad", launch(lambda: fg8.fg8_grouped_gemm(
            self.dyq, self.sdy, self.wqT_up, self.swT_up, self.offsets, R, K, N, E,
            fg8.FG8_GROUP_M, fg8.FG8_BSCALE_BLOCK128, fg8.FG8_OUT_BF16, self.dx, None, 0, self.status, sp)))

        def colwise():
            fg8.fg8_quantize_act(u16(self.dy), R, N, None, 1, E, self.offsets, fg8.FG8_COLWISE,
                                 None, None, None, None, self.pad_dy, self.dyT, self.sdyT, None, 0,
                                 None, sp)
            fg8.fg8_quantize_act(u16(self.x), T, K, None, k, E, self.offsets, fg8.FG8_COLWISE,
                                 None, None, self.row_token, None, self.pad_x, self.xT, self.sxT,
                                 None, 0, None, sp)
            n[0] += 2
        timed("quant_act_colwise", colwise)
        timed("gemm_wgrad", launch(lambda: fg8.fg8_grouped_gemm(
            self.dyT, self.sdyT, self.xT, self.sxT, self.pad_dy, N, K, self.P, E, fg8.FG8_GROUP_K,
            fg8.FG8_BSCALE_ROW128, fg8.FG8_OUT_F32, self.dw, self.gemm_ws, self.gemm_ws.numel(),
            self.status, sp)))
        self.launches_per_step = n[0]

    def run_up_alternative(self, stream):
        """The up-projection variant the step does not run (for a standalone
        timing on the same operands)."""
        c = self.cfg
        if self.fused_act:
            if not hasattr(self, "y_up_alt"):
                self.y_up_alt = torch.empty((c.R, c.n_up), dtype=torch.bfloat16, device=self.dev)
            self.fg8.fg8_grouped_gemm(self.xq, self.sa, self.wq_up, self.sw_up, self.offsets, c.R,
                                      c.n_up, c.hidden, c.E, self.fg8.FG8_GROUP_M,
                                      self.fg8.FG8_BSCALE_BLOCK128, self.fg8.FG8_OUT_BF16,
                                      self.y_up_alt, None, 0, self.status, stream.cuda_stream)
        else:
            self.run_fused_up(stream)

    def run_fused_up(self, stream):
        """Up-projection with the gated activation and its 1x128 quantization
        in the epilogue: X_q W_up -> (H_q, s_H), the down-projection's input."""
        c = self.cfg
        self.fg8.fg8_grouped_gemm_swiglu_quant(self.xq, self.sa, self.wq_up, self.sw_up,
                                               self.offsets, c.R, c.inter, c.hidden, c.E,
                                               self.hq, self.sh, self.status, stream.cuda_stream)

    def run_route(self, stream):
        """Sigmoid-affinity top-k routing of the step's tokens (ids and
        affinities for the permuting quantizer and the combine)."""
        c = self.cfg
        if not hasattr(self, "logits"):
            self.logits = W.gen_router_logits(c, self.dev)
            self.rbias = W.gen_expert_bias(c, self.dev)
            self.r_ids = torch.empty((c.T, c.k), dtype=torch.int32, device=self.dev)
            self.r_aff = torch.empty((c.T, c.k), dtype=torch.float32, device=self.dev)
        self.fg8.fg8_route_topk(self.logits, self.rbias, c.T, c.E, c.k, self.r_ids, self.r_aff,
                                stream.cuda_stream)

    def run_combine(self, stream):
        """Unpermute + combine of the down-projection output: each token's k
        rows summed with its normalized gate weights -> [T, hidden] bf16."""
        c = self.cfg
        if not hasattr(self, "comb_out"):
            self.affinity = W.gen_affinity(c, self.dev)
            self.comb_out = torch.empty((c.T, c.hidden), dtype=torch.bfloat16, device=self.dev)
        self.fg8.fg8_unpermute_combine(self.y_dn.view(torch.int16), c.R, c.hidden, self.token_row,
                                       self.affinity, c.T, c.k, 1, self.fg8.FG8_OUT_BF16,
                                       self.comb_out, stream.cuda_stream)

    def run_down_combine(self, stream):
        """The down-projection with the combine in its epilogue
        (fg8_grouped_gemm_combine) on the step's H and W_down: -> [T, hidden]
        fp32 token rows."""
        c = self.cfg
        if not hasattr(self, "dc_out"):
            if not hasattr(self, "affinity"):
                self.affinity = W.gen_affinity(c, self.dev)
            self.dc_out = torch.empty((c.T, c.hidden), dtype=torch.float32, device=self.dev)
            self.dc_ws = torch.empty(max(16, self.fg8.fg8_grouped_gemm_combine_workspace(c.R)),
                                     dtype=torch.uint8, device=self.dev)
        self.fg8.fg8_grouped_gemm_combine(self.hq, self.sh, self.wq_dn, self.sw_dn, self.offsets,
                                          c.R, c.hidden, c.inter, c.E, self.row_token,
                                          self.token_row, self.affinity, c.T, c.k, 1, self.dc_out,
                                          self.dc_ws, self.dc_ws.numel(), self.status,
                                          stream.cuda_stream)

    def ep_data_plane(self, W_ranks: int = 8):
        """One rank's data plane of a W-rank expert-parallel layer, emulated on
        this GPU with the step's own rows: the E experts read as W source ranks
        of E/W local experts each (counts from the seeded routing), so the
        permuted rows are exactly what this rank would receive, source after
        source.  Returns the three launches (scale repack before the send, the
        merge into local expert order after the receive, the gather of the
        expert outputs for the way back) with their algorithmic bytes.  The
        all-to-all itself is not part of it."""
        c, fg8 = self.cfg, self.fg8
        R, K, KB, EL = c.R, c.hidden, c.hidden // 128, c.E // W_ranks
        e = lambda shape, dt: torch.empty(shape, dtype=dt, device=self.dev)  # noqa: E731
        counts = (self.offsets[1:] - self.offsets[:-1]).to(torch.int32).view(W_ranks, EL).contiguous()
        sa_rows = e((R, KB), torch.float32)
        xq_l, sa_l = e((R, K), torch.uint8), e((KB, R), torch.float32)
        off_l, r2l = e(EL + 1, torch.int32), e(R, torch.int32)
        y_back = e((R, K), torch.bfloat16)
        y_in = self.y_dn if self.y_dn is not None else e((R, K), torch.bfloat16)

        def pack(sp):
            fg8.fg8_ep_pack_scales(self.sa, R, K, sa_rows, sp)

        def unpack(sp):
            fg8.fg8_ep_unpack(self.xq, sa_rows, counts, W_ranks, EL, R, K, xq_l, sa_l, off_l, r2l,
                              self.status, sp)

        def gather(sp):
            fg8.fg8_gather_rows(y_in, R, K * 2, r2l, R, y_back, self.status, sp)

        return [("ep_pack_scales", pack, 8 * R * KB),
                ("ep_unpack", unpack, 2 * (R * K + 4 * R * KB) + 8 * R + 4 * (EL + 1)),
                ("ep_gather_rows", gather, 4 * R * K + 4 * R)]

    def run_route_quantize(self, stream):
        """Routing fused with the permuting quantizer (fg8_route_quantize_act)
        on the step's X and seeded router logits."""
        c = self.cfg
        if not hasattr(self, "rq_ids"):
            if not hasattr(self, "logits"):
                self.logits = W.gen_router_logits(c, self.dev)
                self.rbias = W.gen_expert_bias(c, self.dev)
            e = lambda shape, dt: torch.empty(shape, dtype=dt, device=self.dev)  # noqa: E731
            self.rq_ids, self.rq_aff = e((c.T, c.k), torch.int32), e((c.T, c.k), torch.float32)
            self.rq_xq, self.rq_sa = e((c.R, c.hidden), torch.uint8), e((c.hidden // 128, c.R), torch.float32)
            self.rq_rt, self.rq_tr = e(c.R, torch.int32), e(c.R, torch.int32)
            self.rq_off = e(c.E + 1, torch.int32)
        self.fg8.fg8_route_quantize_act(self.logits, self.rbias, self.x.view(torch.int16), c.T,
                                        c.hidden, c.k, c.E, self.rq_ids, self.rq_aff, self.rq_xq,
                                        self.rq_sa, self.rq_rt, self.rq_tr, self.rq_off, self.ws,
                                        self.ws_bytes, self.status, stream.cuda_stream)

    def run_transpose(self, stream):
        """The standalone block transpose (fg8_transpose_blockq) of the up
        weight: the step gets WqT from the fused quantizer, this times the
        transpose kernel on its own, outside the step."""
        c = self.cfg
        self.fg8.fg8_transpose_blockq(self.wq_up, self.sw_up, c.E, c.n_up, c.hidden, self.wqT_up,
                                      self.swT_up, stream.cuda_stream)

    # --- end-to-end measurement: step inputs arrive from pinned host memory and
    # the forward output and dX go back.  Inputs and those outputs have two
    # device slots, so the copies of one step overlap the kernels of the next.
    IN_NAMES = ("x", "ids", "dy", "h")

    def out_names(self):
        return ("y_dn" if self.cfg.inter else "y_up", "dx")

    def make_slots(self):
        names = [n for n in self.IN_NAMES if getattr(self, n) is not None] + list(self.out_names())
        self.slots = [{n: getattr(self, n) for n in names},
                      {n: torch.empty_like(getattr(self, n)) for n in names}]
        pin = lambda t: t.cpu().pin_memory()  # noqa: E731
        ins = {n: pin(getattr(self, n)) for n in self.IN_NAMES if getattr(self, n) is not None}
        outs = {n: torch.empty(getattr(self, n).shape, dtype=getattr(self, n).dtype).pin_memory()
                for n in self.out_names()}
        return ins, outs

    def use_slot(self, i):
        for n, t in self.slots[i].items():
            setattr(self, n, t)


# --------------------------------------------------------------------------
# clocks
# --------------------------------------------------------------------------

class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline and the reference arm)
# --------------------------------------------------------------------------

class OracleBaseline:
    """The oracle, as it stands (never tuned for timing), on this host's cores,
    on the workload of the step: K1 (permute + 1x128 quantize of X, identity-
    mode rows of dY, column-wise dY and gathered X), K2 (both weights), K3 (the
    up weight) and the fp64 GEMM.  Rates use the algorithmic byte and FLOP
    formulas of the GPU line, so the numbers compare.

    The work is cut into units the method never couples (token slabs, row
    slabs, experts or 128-row slabs of an expert's weight, output rows); each
    unit is one call of the oracle's plain single-threaded function.
    `time_1t` runs a few units of every family on one thread; `time_all` runs
    each family over a pool of threads, one unit per thread at a time: over
    the whole configuration when the per-family time budget allows, else over
    the first units that fit (reported as the fraction `covered`).  The GEMM
    at full size would take hours in fp64 on the host: it is timed on sampled
    output rows and its full-size time extrapolated (labelled so).

    Inputs are the seeded generators' output, untimed: copied from the device
    tensors of the GPU step (`source`, whole experts), or generated on the
    host (`source` None: 128-row weight slabs and smaller activation slabs,
    prepared once and reused, for the reference arm's bounded steps)."""

    FAMILIES = ("quant_act_permute", "quant_act_rows", "quant_act_colwise", "quant_weight",
                "transpose_blockq")

    def __init__(self, cfg: W.MoEConfig, source=None):
        import oracle
        oracle.build()
        self.o = oracle
        self.cfg = cfg
        self.src = source
        self.small = source is None
        self.ids = W.route(cfg)
        self.route = oracle.route(self.ids, cfg.E)
        self.counts = np.diff(self.route["offsets"])
        self.nz = [int(e) for e in np.nonzero(self.counts)[0]]
        self._x = None

    # ---- inputs (bf16 bits as uint16 host arrays)
    @staticmethod
    def _bits(t: torch.Tensor) -> np.ndarray:
        return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)

    def _rows(self, name, lo, hi):
        c = self.cfg
        if self.src is not None:
            return self._bits(getattr(self.src, name)[lo:hi])
        if name == "x":
            return self._bits(W.gen_normal_bf16((hi - lo, c.hidden), W.SIGMA_X, c.seed, W.SID_X,
                                                index_offset=lo * c.hidden))
        return self._bits(W.gen_dy(c, row0=lo, rows=hi - lo))

    def _weight(self, which, e, n0, n1):
        """Rows [n0, n1) of expert e's weight, [1, n1 - n0, K]."""
        c = self.cfg
        N, K, sid = (c.n_up, c.hidden, W.SID_W_UP) if which == "up" else (c.hidden, c.inter, W.SID_W_DOWN)
        if self.src is not None:
            t = (self.src.w_up if which == "up" else self.src.w_down)[e:e + 1, n0:n1]
            return self._bits(t)
        return self._bits(W.gen_normal_bf16((1, n1 - n0, K), W.SIGMA_W, c.seed, sid,
                                            index_offset=(e * N + n0) * K))

    def _x_all(self):
        if self._x is None:
            self._x = self._rows("x", 0, self.cfg.T)
        return self._x

    # ---- units: (prepare() -> args, untimed; run(args) -> algorithmic amount)
    def units(self, family):
        c, o = self.cfg, self.o
        T, K, k, E, R, N, I = c.T, c.hidden, c.k, c.E, c.R, c.n_up, c.inter
        if family == "quant_act_permute":
            slab = 64 if self.small else 512

            def run(a):
                o.quantize_act(a[0], a[1], E)
                return bytes_route_quant(a[0].shape[0], K, k, E)
            return [(lambda t0=t0: (self._rows("x", t0, min(T, t0 + slab)),
                                    np.ascontiguousarray(self.ids[t0:t0 + slab])), run)
                    for t0 in range(0, T, slab)]
        if family == "quant_act_rows":
            rows = 256 if self.small else 2048

            def run(a):
                o.quantize_act(a, None, 1)
                return bytes_rows_quant(a.shape[0], N)
            return [(lambda r0=r0: self._rows("dy", r0, min(R, r0 + rows)), run)
                    for r0 in range(0, R, rows)]
        if family == "quant_act_colwise":
            offs, rt = self.route["offsets"], self.route["row_token"]

            def prep(e):
                o0, o1 = int(offs[e]), int(offs[e + 1])
                if self.small:       # at most 128 rows of the expert (one token tile)
                    o1 = min(o1, o0 + 128)
                sub = np.array([0, o1 - o0], np.int32)
                return (self._rows("dy", o0, o1), np.ascontiguousarray(self._x_all()[rt[o0:o1]]), sub)

            def run(a):
                o.quantize_act_colwise(a[0], a[2])
                o.quantize_act_colwise(a[1], a[2])
                pad = int((a[2][1] + 127) // 128 * 128)
                return bytes_colwise(int(a[2][1]), N, pad) + bytes_colwise(int(a[2][1]), K, pad)
            return [(lambda e=e: prep(e), run) for e in self.nz]

        def slabs(which, rows_total):
            step = 128 if self.small else rows_total
            return [(e, n0, n0 + step) for e in range(E) for n0 in range(0, rows_total, step)]
        if family == "quant_weight":
            def run(a):
                o.quantize_weight(a)
                return bytes_weight_quant(1, a.shape[1], a.shape[2])
            us = [(lambda u=u: self._weight("up", *u), run) for u in slabs("up", N)]
            if I:
                us += [(lambda u=u: self._weight("down", *u), run) for u in slabs("down", K)]
            return us
        if family == "transpose_blockq":
            def run(a):
                o.transpose_blockq(*a)
                return bytes_transpose(1, a[0].shape[1], a[0].shape[2])
            return [(lambda u=u: o.quantize_weight(self._weight("up", *u)), run)
                    for u in slabs("up", N)]
        raise ValueError(family)

    def _gemm_setup(self):
        """Operands of the up-projection GEMM for 64 rows of the largest
        expert, quantized by the oracle (untimed, once)."""
        if not hasattr(self, "_g"):
            c, o = self.cfg, self.o
            e = int(np.argmax(self.counts))
            o0 = int(self.route["offsets"][e])
            rows = self.route["row_token"][o0:o0 + 64]
            xq = o.quantize_act(np.ascontiguousarray(self._x_all()[rows]), None, 1)
            wq, sw = o.quantize_weight(self._weight("up", e, 0, c.n_up))
            self._g = (xq["xq"], xq["sa"], wq, sw)
        return self._g

    def gemm_rate(self, nthreads, budget_s):
        """fp64 oracle GEMM (all output columns of sampled rows): FLOP/s and rows."""
        a, sa, wq, sw = self._gemm_setup()
        N, K = wq.shape[1], wq.shape[2]
        off = np.array([0, a.shape[0]], np.int32)
        per = max(1, nthreads)
        done, t0 = 0, time.perf_counter()
        while done == 0 or time.perf_counter() - t0 < budget_s:
            rows = np.arange(done, done + per) % a.shape[0]
            r, cc = np.repeat(rows, N), np.tile(np.arange(N), per)
            self.o.gemm_mgrouped_entries_threaded(a, sa, wq, sw, off, r, cc, nthreads=nthreads)
            done += per
        return 2.0 * done * N * K / (time.perf_counter() - t0), done

    def time_1t(self, per_family=2, gemm_s=3.0):
        """One thread: the first units of each family, and the GEMM rate."""
        out, tot_b, tot_s = {}, 0.0, 0.0
        for fam in self.FAMILIES:
            us = self.units(fam)[:per_family]
            b = s = 0.0
            for prep, run in us:
                a = prep()
                t0 = time.perf_counter()
                b += run(a)
                s += time.perf_counter() - t0
            out[fam] = {"gbs": b / s / 1e9, "units": len(us)}
            tot_b, tot_s = tot_b + b, tot_s + s
        g, rows = self.gemm_rate(1, gemm_s)
        return {"threads": 1, "quantize_gbs": tot_b / tot_s / 1e9, "kernels": out,
                "gemm_tflops": g / 1e12, "gemm_rows": rows}

    def time_all(self, nthreads, family_s=60.0, gemm_s=4.0, max_units=None, cache=None):
        """`nthreads` threads over every family (at most family_s seconds of
        timed work each: the whole workload when it fits), then the GEMM rate
        on sampled rows (gemm_s seconds).
        max_units caps the units per family; `cache` (a dict) keeps prepared
        inputs between calls."""
        from concurrent.futures import ThreadPoolExecutor
        out, tot_b, tot_s = {}, 0.0, 0.0
        share = family_s
        with ThreadPoolExecutor(max_workers=nthreads) as ex:
            for fam in self.FAMILIES:
                us = self.units(fam)
                if max_units:
                    us = us[:max_units]
                b = s = 0.0
                n_done = 0
                while n_done < len(us):
                    batch = us[n_done:n_done + 2 * nthreads]
                    key = (fam, n_done)
                    if cache is not None and key in cache:
                        args = cache[key]
                    else:
                        args = list(ex.map(lambda u: u[0](), batch))
                        if cache is not None:
                            cache[key] = args
                    t0 = time.perf_counter()
                    b += sum(ex.map(lambda ua: ua[0][1](ua[1]), zip(batch, args)))
                    s += time.perf_counter() - t0
                    n_done += len(batch)
                    if s > share:
                        break
                out[fam] = {"gbs": b / s / 1e9, "units": n_done, "of_units": len(us),
                            "covered": n_done / len(self.units(fam))}
                tot_b, tot_s = tot_b + b, tot_s + s
        res = {"threads": nthreads, "quantize_gbs": tot_b / tot_s / 1e9, "kernels": out,
               "covered": min(v["covered"] for v in out.values())}
        if gemm_s > 0:
            g, rows = self.gemm_rate(nthreads, gemm_s)
            res.update(gemm_tflops=g / 1e12, gemm_rows=rows)
        return res


def host_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def cpu_baseline(cfg: W.MoEConfig, source=None, family_s: float = 60.0):
    """The cpu_baseline object of the JSON line (oracle at 1 thread and at all
    usable cores; `value` is the GEMM rate at all cores)."""
    ob = OracleBaseline(cfg, source)
    n = host_threads()
    one = ob.time_1t()
    allc = ob.time_all(n, family_s=family_s)
    gemm_total = sum(a for b, a in work_of(cfg, padded_total_of(cfg))[0].values() if b == "tensor")
    return {
        "value": allc["gemm_tflops"], "unit": "TFLOP/s", "cores": n, "kind": "oracle",
        "sample": (f"fp64 GEMM on {allc['gemm_rows']} sampled output rows (all {cfg.n_up} "
                   f"columns, K={cfg.hidden}) at {n} threads; K1-K3 over "
                   f"{100 * allc['covered']:.0f}% or more of the {cfg.name} workload at {n} "
                   "threads; one-thread rates on the first units of each kernel"),
        "quantize_gbs": allc["quantize_gbs"],
        "threads_1": one, "threads_all": allc,
        "gemm_full_step_s": {"value": gemm_total / (allc["gemm_tflops"] * 1e12),
                             "extrapolated": True,
                             "note": "the step's GEMM FLOPs over the sampled fp64 rate"},
    }


# --------------------------------------------------------------------------
# replicas (one process per GPU, each running the whole step)
# --------------------------------------------------------------------------

def all_max(pg, values, device):
    """Elementwise max over the ranks of `pg` (the values unchanged without one)."""
    if pg is None:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return t.tolist()


def job_rate(world: int, units_per_rank: float, slowest_ms: float) -> float:
    """Whole-job throughput of `world` replicas that each processed
    `units_per_rank`: all units over the slowest rank's time (units/s)."""
    return world * units_per_rank / (slowest_ms * 1e-3)


def run_reference(args):
    """The reference arm: the oracle on this host's cores (no GPU), each step a
    bounded sample of the workload -- one unit per thread of every K1-K3
    family (inputs prepared once) and a fixed time of the fp64 GEMM on
    sampled rows.  Under torchrun only rank 0 runs and prints."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    cfg = W.CONFIGS[args.config]
    ob = OracleBaseline(cfg)
    n = host_threads()
    cache = {}
    times, tf_list, gb_list = [], [], []
    res = None
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        res = ob.time_all(n, family_s=1e9, gemm_s=1.0, max_units=n, cache=cache)
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
            tf_list.append(res["gemm_tflops"])
            gb_list.append(res["quantize_gbs"])
    value = statistics.median(tf_list) if tf_list else res["gemm_tflops"]
    desc = (f"per step: {n} units of each K1-K3 kernel of the {cfg.name} workload (token slabs, "
            "row slabs, experts' token tiles, 128-row weight slabs) and 1 s of the fp64 GEMM on "
            f"sampled output rows (all {cfg.n_up} columns, K={cfg.hidden}), at {n} threads")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * statistics.median(times) if times else None,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": cfg.name, "description": cfg.description, "E": cfg.E, "T": cfg.T,
                   "k": cfg.k, "hidden": cfg.hidden, "n_up": cfg.n_up, "inter": cfg.inter,
                   "routed_rows": cfg.R, "parallelism": f"oracle on {n} host threads"},
        "quantize_gbs": statistics.median(gb_list) if gb_list else res["quantize_gbs"],
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": n, "kind": "oracle",
                         "sample": desc, "quantize_gbs_by_kernel":
                             {k_: v["gbs"] for k_, v in res["kernels"].items()}},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


# --------------------------------------------------------------------------
# GPU arm
# --------------------------------------------------------------------------

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="fg8", choices=["fg8", "reference"])
    ap.add_argument("--config", default="dsv3", choices=sorted(W.CONFIGS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=60.0,
                    help="cap, in seconds of timed oracle work, for each K1-K3 family of "
                         "cpu_baseline (the whole workload is covered when it fits)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--unfused-act", action="store_true",
                    help="forward through the plain up-projection (bf16 Y) and a separately "
                         "generated, row-quantized down-projection input H, instead of the "
                         "default up-projection with the gated activation and its 1x128 "
                         "quantization fused in the epilogue")
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)
    if args.config == "dsv3_bwd":
        args.config = "dsv3"

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
        pg = dist

    from fp8_fine_grained_permute_b200 import build as fbuild
    from fp8_fine_grained_permute_b200 import fg8
    if rank == 0:
        fbuild.build()
    if pg:
        pg.barrier()
    fg8.lib()

    cfg = W.CONFIGS[args.config]
    st = Step(cfg, dev, fused_act=not args.unfused_act)
    stream = torch.cuda.Stream(dev)
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            st.run(stream)
    torch.cuda.synchronize()
    if st.status.item() != 0:
        raise RuntimeError(f"device status {fg8.status_name(st.status.item())}")

    # ---------------- kernel-level timed region
    marks = {}
    clk = ClockSampler(local)
    clk.start()
    time.sleep(0.3)
    if pg:
        pg.barrier()
    torch.cuda.synchronize()
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for _ in range(args.steps):
        st.run(stream, marks)
    t_end.record(stream)
    torch.cuda.synchronize()
    if pg:
        pg.barrier()
    clocks = clk.stop()
    (total_ms,) = all_max(pg, [t_start.elapsed_time(t_end)], dev)
    ms_step = total_ms / args.steps
    kern_ms = {k: sum(a.elapsed_time(b) for a, b in v) / args.steps for k, v in marks.items()}

    pk = peaks()
    fp8_peak = pk["bf16_sus"] * FP8_OVER_BF16
    kernels = []
    gemm_flops = gemm_ms = q_bytes = q_ms = 0.0
    for name, (bound, amount) in st.work.items():
        ms = kern_ms[name]
        if bound == "tensor":
            ach = amount / (ms * 1e-3) / 1e12
            gbytes = st.gemm_bytes[name]
            t_tensor = amount / (fp8_peak * 1e12)
            t_hbm = gbytes / (pk["hbm_gbs"] * 1e9)
            if t_hbm > t_tensor:         # the output/operand traffic is the floor
                gb = gbytes / (ms * 1e-3) / 1e9
                entry = {"kernel": name, "bound": "hbm", "ms": ms, "achieved": gb,
                         "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": gb / pk["hbm_gbs"],
                         "tflops": ach, "tensor_frac": ach / fp8_peak}
            else:
                entry = {"kernel": name, "bound": "tensor", "ms": ms, "achieved": ach,
                         "peak": fp8_peak, "unit": "TFLOP/s", "frac": ach / fp8_peak}
            entry["floor_ms"] = 1e3 * max(t_tensor, t_hbm)
            gemm_flops += amount
            gemm_ms += ms
        else:
            ach = amount / (ms * 1e-3) / 1e9
            entry = {"kernel": name, "bound": "hbm", "ms": ms, "achieved": ach,
                     "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": ach / pk["hbm_gbs"]}
            q_bytes += amount
            q_ms += ms
        entry["share"] = ms / ms_step
        entry["traffic"] = measured_traffic(name, cfg, st.padded_total, st.fused_act)
        nominal_of(entry)
        kernels.append(entry)
    dom = max(kernels, key=lambda d: d["ms"])
    # K3 on its own (the step takes WqT from the fused quantizer): timed with
    # events around args.steps back-to-back launches, outside the step
    with torch.cuda.stream(stream):
        st.run_transpose(stream)
        tr0, tr1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        tr0.record(stream)
        for _ in range(args.steps):
            st.run_transpose(stream)
        tr1.record(stream)
    torch.cuda.synchronize()
    tr_ms = tr0.elapsed_time(tr1) / args.steps
    tr_gb = bytes_transpose(cfg.E, cfg.n_up, cfg.hidden) / (tr_ms * 1e-3) / 1e9
    kernels.append({"kernel": "transpose_blockq", "standalone": True, "bound": "hbm", "ms": tr_ms,
                    "achieved": tr_gb, "peak": pk["hbm_gbs"], "unit": "GB/s",
                    "frac": tr_gb / pk["hbm_gbs"], "share": None,
                    "traffic": measured_traffic("transpose_blockq", cfg, st.padded_total, st.fused_act),
                    "note": "not in the step: the step's WqT comes from the fused quantizer"})
    # the up-projection kernel that the step does not use, on its own and on
    # the same operands: the plain one (bf16 Y) when the step runs the fused
    # gated activation (the default), the fused one otherwise
    if cfg.inter:
        alt = "gemm_fprop_up" if st.fused_act else "gemm_fprop_up_swiglu_quant"
        with torch.cuda.stream(stream):
            st.run_up_alternative(stream)
            fu0, fu1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            fu0.record(stream)
            for _ in range(args.steps):
                st.run_up_alternative(stream)
            fu1.record(stream)
        torch.cuda.synchronize()
        fu_ms = fu0.elapsed_time(fu1) / args.steps
        fu_tf = 2.0 * cfg.R * cfg.n_up * cfg.hidden / (fu_ms * 1e-3) / 1e12
        in_step = "gemm_fprop_up_swiglu_quant" if st.fused_act else "gemm_fprop_up"
        kernels.append({"kernel": alt, "standalone": True,
                        "bound": "tensor", "ms": fu_ms, "achieved": fu_tf, "peak": fp8_peak,
                        "unit": "TFLOP/s", "frac": fu_tf / fp8_peak, "share": None,
                        "traffic": measured_traffic(alt, cfg, st.padded_total, st.fused_act),
                        "in_step_counterpart": in_step, "in_step_ms": kern_ms[in_step],
                        "note": "not in the step: back-to-back launches on the step's operands "
                                "(W_up alone exceeds L2); "
                                + ("the fused kernel in the step replaces it and the row "
                                   "quantization of H" if st.fused_act else
                                   "it would replace gemm_fprop_up and the row quantization of H")})
    # unpermute + combine of the down-projection output on its own
    if cfg.inter:
        with torch.cuda.stream(stream):
            st.run_combine(stream)
            cb0, cb1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            cb0.record(stream)
            for _ in range(args.steps):
                st.run_combine(stream)
            cb1.record(stream)
        torch.cuda.synchronize()
        cb_ms = cb0.elapsed_time(cb1) / args.steps
        cb_bytes = bytes_combine(cfg.T, cfg.k, cfg.hidden)
        cb_gb = cb_bytes / (cb_ms * 1e-3) / 1e9
        kernels.append({"kernel": "unpermute_combine", "standalone": True, "bound": "hbm",
                        "ms": cb_ms, "achieved": cb_gb, "peak": pk["hbm_gbs"], "unit": "GB/s",
                        "frac": cb_gb / pk["hbm_gbs"], "share": None,
                        "traffic": measured_traffic("unpermute_combine", cfg, st.padded_total, st.fused_act),
                        "note": "not in the step: the layer output after the down-projection "
                                "(T x hidden bf16 from R routed rows); back-to-back launches, "
                                "rows larger than L2"})
    # the down-projection with the combine fused into its epilogue, on its own
    if cfg.inter:
        with torch.cuda.stream(stream):
            st.run_down_combine(stream)
            dc0, dc1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            dc0.record(stream)
            for _ in range(args.steps):
                st.run_down_combine(stream)
            dc1.record(stream)
        torch.cuda.synchronize()
        dc_ms = dc0.elapsed_time(dc1) / args.steps
        dc_flops = 2 * cfg.R * cfg.hidden * cfg.inter
        dc_tf = dc_flops / (dc_ms * 1e-3) / 1e12
        kernels.append({"kernel": "gemm_fprop_down_combine", "standalone": True, "bound": "tensor",
                        "ms": dc_ms, "achieved": dc_tf, "peak": fp8_peak, "unit": "TFLOP/s",
                        "frac": dc_tf / fp8_peak, "share": None, "traffic": None,
                        "replaces_ms": kern_ms["gemm_fprop_down"] + cb_ms,
                        "note": "not in the step: fg8_grouped_gemm_combine (the combine's "
                                "weighted sum as fp32 reductions into the [T, hidden] output from "
                                "the down-projection epilogue); replaces gemm_fprop_down + "
                                "unpermute_combine"})
        if st.status.item() != 0:
            raise RuntimeError(f"fused down-projection + combine reported status {st.status.item()}")
    # expert-parallel data plane (one rank of 8, emulated) on its own
    if cfg.E % 8 == 0:
        for name, fn, nbytes in st.ep_data_plane(8):
            with torch.cuda.stream(stream):
                fn(stream.cuda_stream)
                ep0, ep1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                ep0.record(stream)
                for _ in range(args.steps):
                    fn(stream.cuda_stream)
                ep1.record(stream)
            torch.cuda.synchronize()
            ep_ms = ep0.elapsed_time(ep1) / args.steps
            ep_gb = nbytes / (ep_ms * 1e-3) / 1e9
            kernels.append({"kernel": name, "standalone": True, "bound": "hbm", "ms": ep_ms,
                            "achieved": ep_gb, "peak": pk["hbm_gbs"], "unit": "GB/s",
                            "frac": ep_gb / pk["hbm_gbs"], "share": None, "traffic": None,
                            "note": "not in the step: one rank's data plane of an 8-rank "
                                    "expert-parallel layer, emulated on this GPU with the step's "
                                    "rows (the all-to-all itself is not measured: one GPU)"})
        if st.status.item() != 0:
            raise RuntimeError(f"expert-parallel data plane reported status {st.status.item()}")
    # sigmoid-affinity top-k routing on its own
    with torch.cuda.stream(stream):
        st.run_route(stream)
        ro0, ro1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ro0.record(stream)
        for _ in range(args.steps):
            st.run_route(stream)
        ro1.record(stream)
    torch.cuda.synchronize()
    ro_ms = ro0.elapsed_time(ro1) / args.steps
    ro_gb = (cfg.T * cfg.E * 4 + cfg.E * 4 + cfg.T * cfg.k * 8) / (ro_ms * 1e-3) / 1e9
    kernels.append({"kernel": "route_topk", "standalone": True, "bound": "hbm", "ms": ro_ms,
                    "achieved": ro_gb, "peak": pk["hbm_gbs"], "unit": "GB/s",
                    "frac": ro_gb / pk["hbm_gbs"], "share": None, "traffic": None,
                    "note": "not in the step (its ids come from the seeded host routing): "
                            "T x E fp32 logits -> top-k ids and affinities; a few MB, "
                            "L2-resident between launches, so launch- and latency-bound"})
    # routing fused with the permute + 1x128 quantization, on its own
    with torch.cuda.stream(stream):
        st.run_route_quantize(stream)
        rq0, rq1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        rq0.record(stream)
        for _ in range(args.steps):
            st.run_route_quantize(stream)
        rq1.record(stream)
    torch.cuda.synchronize()
    rq_ms = rq0.elapsed_time(rq1) / args.steps
    rq_bytes = bytes_route_quantize(cfg.T, cfg.hidden, cfg.k, cfg.E)
    rq_gb = rq_bytes / (rq_ms * 1e-3) / 1e9
    kernels.append({"kernel": "route_quantize_act", "standalone": True, "bound": "hbm",
                    "ms": rq_ms, "achieved": rq_gb, "peak": pk["hbm_gbs"], "unit": "GB/s",
                    "frac": rq_gb / pk["hbm_gbs"], "share": None, "traffic": None,
                    "replaces_ms": ro_ms + kern_ms["quant_act_permute"],
                    "note": "not in the step (its ids come from the seeded host routing): router "
                            "logits -> top-k ids, affinities, permuted E4M3 rows and 1x128 scales "
                            "in one cooperative launch; replaces route_topk + quant_act_permute"})
    # write-only HBM rate on this GPU (fills of 8 GiB, no reads): the ceiling of
    # kernels that mostly write, e.g. the weight gradient's fp32 output.  torch's
    # fill runs at a rate that depends on the element width (1-byte elements
    # are not vectorized), so the widest view's rate is taken.
    fill = torch.empty(8 << 30, dtype=torch.uint8, device=dev)
    write_by_view = {}
    for dt in (torch.uint8, torch.int32, torch.int64):
        v = fill.view(dt)
        with torch.cuda.stream(stream):
            v.fill_(1)
            fw0, fw1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            fw0.record(stream)
            for i in range(3):
                v.fill_(i)
            fw1.record(stream)
        torch.cuda.synchronize()
        write_by_view[str(dt).replace("torch.", "")] = 3 * fill.numel() / (fw0.elapsed_time(fw1) * 1e-3) / 1e9
    write_gbs = max(write_by_view.values())
    del fill, v
    for kd in kernels:
        if kd["kernel"] == "gemm_wgrad" and kd["unit"] == "GB/s":
            kd["write_ceiling_gbs"] = write_gbs
            kd["frac_of_write_ceiling"] = kd["achieved"] / write_gbs
    for kd in kernels:
        if "nominal_peak" not in kd:
            nominal_of(kd)
    # whole job: every rank did the same work; divide by the slowest rank's time
    gemm_ms, q_ms = all_max(pg, [gemm_ms, q_ms], dev)
    gemm_tflops = job_rate(world, gemm_flops, gemm_ms) / 1e12
    quant_gbs = job_rate(world, q_bytes, q_ms) / 1e9

    # ---------------- end-to-end through the C ABI with host buffers
    # Step i uses device slot i % 2: its inputs are copied in on one copy stream
    # (once step i - 2 is done with the slot), the kernels run on the compute
    # stream, and the forward output and dX go back on another copy stream, so
    # host transfers in both directions overlap the kernels of the next step.
    e2e = None
    if not args.no_e2e:
        host_in, host_out = st.make_slots()
        h2d = sum(t.numel() * t.element_size() for t in host_in.values())
        d2h = sum(t.numel() * t.element_size() for t in host_out.values())
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev = lambda: torch.cuda.Event()  # noqa: E731
        comp_done, out_done = [None, None], [None, None]
        if pg:
            pg.barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        s_in.wait_event(e0)
        s_out.wait_event(e0)
        for i in range(args.steps):
            slot = i % 2
            dev_slot = st.slots[slot]
            in_done = ev()
            with torch.cuda.stream(s_in):
                if comp_done[slot] is not None:
                    s_in.wait_event(comp_done[slot])
                for n, h in host_in.items():
                    dev_slot[n].copy_(h, non_blocking=True)
                in_done.record(s_in)
            stream.wait_event(in_done)
            if out_done[slot] is not None:
                stream.wait_event(out_done[slot])
            st.use_slot(slot)
            st.run(stream)
            comp_done[slot] = ev()
            comp_done[slot].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(comp_done[slot])
                for n, h in host_out.items():
                    h.copy_(dev_slot[n], non_blocking=True)
                out_done[slot] = ev()
                out_done[slot].record(s_out)
        for d in out_done:
            if d is not None:
                stream.wait_event(d)
        e1.record(stream)
        torch.cuda.synchronize()
        st.use_slot(0)
        (e2e_ms,) = all_max(pg, [e0.elapsed_time(e1) / args.steps], dev)
        e2e = {"value": job_rate(world, gemm_flops, e2e_ms) / 1e12, "unit": "TFLOP/s",
               "ms_per_step": e2e_ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "note": "GEMM FLOPs per step over the whole step time including pinned-host "
                       f"copies of {', '.join(host_in)} in and {', '.join(host_out)} out; two "
                       "device slots, copies overlap the next step's kernels"}
    if st.status.item() != 0:
        raise RuntimeError(f"device status {fg8.status_name(st.status.item())}")

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(cfg, st, family_s=args.cpu_budget)

    if rank == 0:
        line = {
            "metric": METRIC, "value": gemm_tflops, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "e4m3 x e4m3 -> f32 (GEMM); bf16 -> e4m3 (quantize)",
            "data": "synthetic",
            "config": {"workload": cfg.name, "description": cfg.description,
                       "E": cfg.E, "T": cfg.T, "k": cfg.k, "hidden": cfg.hidden,
                       "n_up": cfg.n_up, "inter": cfg.inter, "routed_rows": cfg.R,
                       "parallelism": f"replicas x{world}",
                       "fused_act": st.fused_act,
                       "l2": "inputs larger than L2 (step working set > 50 GB)"},
            "quantize_gbs": quant_gbs,
            "gemm_frac_of_fp8_peak": gemm_tflops / world / fp8_peak,
            "quantize_frac_of_hbm": quant_gbs / world / pk["hbm_gbs"],
            "roofline": {"kernel": dom["kernel"], "bound": dom["bound"], "achieved": dom["achieved"],
                         "peak": dom["peak"], "unit": dom["unit"], "frac": dom["frac"],
                         "traffic": measured_traffic(dom["kernel"], cfg, st.padded_total, st.fused_act),
                         "traffic_source": f"ncu DRAM bytes (read + write) of the {TRAFFIC_CAPTURE['config']} "
                                           "step's launch list, scaled by algorithmic bytes; null if "
                                           "the kernel changed since",
                         "peak_source": f"{pk['source']}: HBM {pk['hbm_gbs']} GB/s; FP8 = "
                                        f"{FP8_OVER_BF16} x sustained BF16 {pk['bf16_sus']} TFLOP/s",
                         "nominal_peak": dom["nominal_peak"], "frac_of_nominal": dom["frac_of_nominal"]},
            "kernels": kernels,
            "hbm_write_only_gbs": {"value": write_gbs, "by_element": write_by_view,
                                   "source": "torch fill of 8 GiB timed with CUDA events in this "
                                   "run (no reads), fastest element width"},
            "cpu_baseline": cpu,
            "e2e": e2e,
            "clocks": clocks,
            "gpu_launches": st.launches_per_step * args.steps,
        }
        print(json.dumps(line))
    if pg:
        pg.barrier()
        pg.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
