"""Seeded synthetic inputs for the FP8 fine-grained MoE path.

This module only *generates inputs*: bf16 activations and weights, routing
ids and the per-config sizes.  It holds none of the method's arithmetic (no
scaling, no FP8 encoding, no permutation, no GEMM), so that both the CUDA
path and the CPU oracle can draw from it without sharing any of the code
they are checked on.

Element values are a pure function of (seed, stream id, flat index): a
counter-based integer hash picks an entry of a precomputed quantile table.
Because the hash uses only exact int64 arithmetic and the table lookup is a
gather, the same call yields bit-identical tensors on the CPU and on a GPU,
and any slice (one expert, one 128x128 block, one row) can be regenerated on
its own without generating the rest.  That is what lets the full-size parity
tests check sampled outputs against the oracle on the host.

Distributions (the workloads of the Kanana-2 and DeepSeek-V3 pages, with the
sizes of the five configurations below):
  * activations  X ~ N(0, 1)            rounded to bf16
  * weights      W ~ N(0, 0.02^2)       rounded to bf16
  * gradients   dY ~ Student-t(nu = 3), with a seeded 0.1 % of the entries
                multiplied by 100 (outlier tiles), rounded to bf16
The quantile tables have 2^20 entries at the probability midpoints
(i + 1/2) / 2^20, so the largest |N(0,1)| draw is about 4.9 sigma.

Routing ids (host side, numpy, seeded):
  * tiny:   top-2 of U(0,1) logits over 4 experts
  * kanana: top-6 of sigmoid(u) + b_e, u ~ N(0,1), b_e ~ U(-0.1, 0.1)
            (sigmoid affinity plus per-expert bias, DeepSeek-V3 page sec. 2.1)
  * dsv3:   Zipf(s = 1.2) popularity over a seeded expert permutation, with 16
            seeded experts forced to zero tokens, 8 distinct experts per token
            drawn by Gumbel-top-k on log p.
Ties in any top-k are broken towards the lower expert index.
"""

from __future__ import annotations

import dataclasses
import functools
import math

import numpy as np
import torch

TABLE_BITS = 20
_M32 = 0xFFFFFFFF


# --------------------------------------------------------------------------
# counter-based hash on int64 tensors (values kept in [0, 2^32))
# --------------------------------------------------------------------------

def _mul32(x: torch.Tensor, c: int) -> torch.Tensor:
    """(x * c) mod 2^32 for 0 <= x < 2^32, without any int64 overflow."""
    lo, hi = c & 0xFFFF, c >> 16
    return (x * lo + (((x * hi) & 0xFFFF) << 16)) & _M32


def _mix32(x: torch.Tensor) -> torch.Tensor:
    """A 32-bit integer finaliser (xor-shift / multiply rounds)."""
    x = x ^ (x >> 16)
    x = _mul32(x, 0x21F0AAAD)
    x = x ^ (x >> 15)
    x = _mul32(x, 0x735A2D97)
    x = x ^ (x >> 15)
    return x


def _mix32_int(x: int) -> int:
    x &= _M32
    x ^= x >> 16
    x = (x * 0x21F0AAAD) & _M32
    x ^= x >> 15
    x = (x * 0x735A2D97) & _M32
    x ^= x >> 15
    return x


def stream_key(seed: int, sid: int) -> tuple[int, int]:
    k1 = _mix32_int(seed ^ _mix32_int(sid * 0x9E3779B9 + 0x7F4A7C15))
    k2 = _mix32_int(k1 ^ 0x85EBCA6B)
    return k1, k2


def hash_index(idx: torch.Tensor, seed: int, sid: int) -> torch.Tensor:
    """32-bit hash of (seed, sid, idx) for int64 idx >= 0 (any device)."""
    k1, k2 = stream_key(seed, sid)
    lo = idx & _M32
    hi = idx >> 32
    h = _mix32(lo ^ k1)
    return _mix32(h ^ ((hi * 0x2545F491 + k2) & _M32))


# --------------------------------------------------------------------------
# quantile tables (bf16 bit patterns as int16)
# --------------------------------------------------------------------------

def _probs() -> torch.Tensor:
    n = 1 << TABLE_BITS
    return (torch.arange(n, dtype=torch.float64) + 0.5) / n


def _to_bf16_bits(v: torch.Tensor) -> torch.Tensor:
    return v.to(torch.float32).to(torch.bfloat16).view(torch.int16)


@functools.lru_cache(maxsize=None)
def normal_table(sigma: float) -> torch.Tensor:
    return _to_bf16_bits(torch.special.ndtri(_probs()) * sigma)


def _student_t3_ppf(p: torch.Tensor) -> torch.Tensor:
    """Quantiles of Student-t with 3 degrees of freedom, by bisection on the
    closed-form CDF F(t) = 1/2 + (1/pi) * (u/(1+u^2) + atan(u)), u = t/sqrt(3)."""
    lo = torch.full_like(p, -1e4)
    hi = torch.full_like(p, 1e4)
    for _ in range(80):
        mid = 0.5 * (lo + hi)
        u = mid / math.sqrt(3.0)
        cdf = 0.5 + (u / (1.0 + u * u) + torch.atan(u)) / math.pi
        below = cdf < p
        lo = torch.where(below, mid, lo)
        hi = torch.where(below, hi, mid)
    return 0.5 * (lo + hi)


@functools.lru_cache(maxsize=None)
def student_t3_tables() -> tuple[torch.Tensor, torch.Tensor]:
    """(plain table, outlier table = 100 x the same quantiles)."""
    q = _student_t3_ppf(_probs())
    return _to_bf16_bits(q), _to_bf16_bits(q * 100.0)


def _tables_on(device, *tabs):
    return [t.to(device) for t in tabs]


# --------------------------------------------------------------------------
# tensor generators
# --------------------------------------------------------------------------

def gen_normal_bf16(shape, sigma: float, seed: int, sid: int, device="cpu",
                    index_offset: int = 0, chunk: int = 1 << 26) -> torch.Tensor:
    """bf16 tensor of `shape` whose flat element i is draw (index_offset + i)
    of the N(0, sigma^2) stream (seed, sid)."""
    numel = math.prod(shape)
    out = torch.empty(numel, dtype=torch.int16, device=device)
    (tab,) = _tables_on(device, normal_table(sigma))
    for s in range(0, numel, chunk):
        n = min(chunk, numel - s)
        idx = torch.arange(index_offset + s, index_offset + s + n, dtype=torch.int64, device=device)
        h = hash_index(idx, seed, sid)
        out[s:s + n] = tab[h >> (32 - TABLE_BITS)]
    return out.view(torch.bfloat16).view(*shape)


def gen_normal_bf16_at(idx: torch.Tensor, sigma: float, seed: int, sid: int) -> torch.Tensor:
    """Draws of the N(0, sigma^2) stream at arbitrary flat indices (CPU)."""
    (tab,) = _tables_on(idx.device, normal_table(sigma))
    return tab[hash_index(idx, seed, sid) >> (32 - TABLE_BITS)].view(torch.bfloat16)


def gen_grad_bf16(shape, seed: int, sid: int, device="cpu", index_offset: int = 0,
                  outlier_frac: float = 1e-3, chunk: int = 1 << 26) -> torch.Tensor:
    """Student-t(3) bf16 tensor with a seeded `outlier_frac` of entries x100."""
    numel = math.prod(shape)
    out = torch.empty(numel, dtype=torch.int16, device=device)
    tab, tab100 = _tables_on(device, *student_t3_tables())
    thresh = int(outlier_frac * 2**32)
    for s in range(0, numel, chunk):
        n = min(chunk, numel - s)
        idx = torch.arange(index_offset + s, index_offset + s + n, dtype=torch.int64, device=device)
        h = hash_index(idx, seed, sid) >> (32 - TABLE_BITS)
        pick = hash_index(idx, seed, sid + 1000) < thresh
        out[s:s + n] = torch.where(pick, tab100[h], tab[h])
    return out.view(torch.bfloat16).view(*shape)


# --------------------------------------------------------------------------
# routing ids (host)
# --------------------------------------------------------------------------

def _topk_lowest_index_ties(score: np.ndarray, k: int) -> np.ndarray:
    # stable sort of -score keeps equal scores in ascending expert order
    order = np.argsort(-score, axis=1, kind="stable")
    return order[:, :k].astype(np.int32)


def route_uniform(T: int, E: int, k: int, seed: int) -> np.ndarray:
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, 1])))
    logits = rng.random((T, E))
    return _topk_lowest_index_ties(logits, k)


def route_sigmoid_bias(T: int, E: int, k: int, seed: int) -> np.ndarray:
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, 2])))
    u = rng.standard_normal((T, E))
    b = rng.uniform(-0.1, 0.1, size=E)
    score = 1.0 / (1.0 + np.exp(-u)) + b[None, :]
    return _topk_lowest_index_ties(score, k)


def zipf_popularity(E: int, s: float, n_zero: int, seed: int) -> np.ndarray:
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, 3])))
    perm = rng.permutation(E)
    p = np.empty(E)
    p[perm] = (np.arange(E) + 1.0) ** (-s)
    zero = rng.choice(E, size=n_zero, replace=False) if n_zero else np.array([], dtype=np.int64)
    p[zero] = 0.0
    return p / p.sum()


def route_zipf(T: int, E: int, k: int, seed: int, s: float = 1.2, n_zero: int = 16) -> np.ndarray:
    p = zipf_popularity(E, s, n_zero, seed)
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, 4])))
    with np.errstate(divide="ignore"):
        logp = np.log(p)
    gumbel = -np.log(-np.log(rng.random((T, E))))
    return _topk_lowest_index_ties(logp[None, :] + gumbel, k)


# --------------------------------------------------------------------------
# configurations
# --------------------------------------------------------------------------

@dataclasses.dataclass(frozen=True)
class MoEConfig:
    name: str
    E: int
    T: int
    k: int
    hidden: int          # K of the up projection, N of the down projection
    n_up: int            # N of the up projection (gate+up where applicable)
    inter: int           # K of the down projection (0: no down projection)
    routing: str         # "uniform" | "sigmoid_bias" | "zipf" | "identity"
    seed: int
    description: str

    @property
    def R(self) -> int:
        return self.T * self.k


CONFIGS = {
    "tiny": MoEConfig("tiny", E=4, T=64, k=2, hidden=256, n_up=256, inter=0,
                      routing="uniform", seed=20261202 + 1,
                      description="tiny MoE FFN up-proj: 4 experts, K=256, N=256, 64 tokens top-2"),
    "dense4096": MoEConfig("dense4096", E=1, T=4096, k=1, hidden=4096, n_up=4096, inter=0,
                           routing="identity", seed=20261202 + 2,
                           description="single-group dense FP8 block-scaled GEMM M=N=K=4096"),
    "kanana": MoEConfig("kanana", E=64, T=16384, k=6, hidden=2048, n_up=1536, inter=768,
                        routing="sigmoid_bias", seed=20261202 + 3,
                        description="Kanana-scale MoE layer: 64 experts, hidden 2048, inter 768, 16384 tokens top-6"),
    "dsv3": MoEConfig("dsv3", E=256, T=8192, k=8, hidden=7168, n_up=4096, inter=2048,
                      routing="zipf", seed=20261202 + 4,
                      description="DeepSeek-V3-shaped MoE layer: 256 experts, hidden 7168, inter 2048, 8192 tokens top-8, Zipf(1.2)"),
    "dsv3_bwd": MoEConfig("dsv3_bwd", E=256, T=8192, k=8, hidden=7168, n_up=4096, inter=2048,
                          routing="zipf", seed=20261202 + 4,
                          description="backward shapes of the DeepSeek-V3-shaped layer: dgrad through transposed block-quantized weights, wgrad per expert"),
}

# stream ids of the tensors of one configuration
SID_X, SID_W_UP, SID_W_DOWN, SID_H, SID_DY = 1, 2, 3, 4, 5
SID_Y_DOWN, SID_AFF, SID_LOGITS, SID_BIAS = 6, 7, 8, 9
SIGMA_X, SIGMA_W = 1.0, 0.02


def route(cfg: MoEConfig) -> np.ndarray:
    if cfg.routing == "uniform":
        return route_uniform(cfg.T, cfg.E, cfg.k, cfg.seed)
    if cfg.routing == "sigmoid_bias":
        return route_sigmoid_bias(cfg.T, cfg.E, cfg.k, cfg.seed)
    if cfg.routing == "zipf":
        return route_zipf(cfg.T, cfg.E, cfg.k, cfg.seed)
    if cfg.routing == "identity":
        return np.zeros((cfg.T, cfg.k), dtype=np.int32)
    raise ValueError(cfg.routing)


def gen_x(cfg: MoEConfig, device="cpu") -> torch.Tensor:
    return gen_normal_bf16((cfg.T, cfg.hidden), SIGMA_X, cfg.seed, SID_X, device)


def gen_w_up(cfg: MoEConfig, device="cpu", experts=None) -> torch.Tensor:
    """[E, n_up, hidden] (or only the listed experts, same values)."""
    per = cfg.n_up * cfg.hidden
    if experts is None:
        return gen_normal_bf16((cfg.E, cfg.n_up, cfg.hidden), SIGMA_W, cfg.seed, SID_W_UP, device)
    return torch.stack([gen_normal_bf16((cfg.n_up, cfg.hidden), SIGMA_W, cfg.seed, SID_W_UP,
                                        device, index_offset=e * per) for e in experts])


def gen_w_down(cfg: MoEConfig, device="cpu", experts=None) -> torch.Tensor:
    """[E, hidden, inter] (or only the listed experts, same values)."""
    per = cfg.hidden * cfg.inter
    if experts is None:
        return gen_normal_bf16((cfg.E, cfg.hidden, cfg.inter), SIGMA_W, cfg.seed, SID_W_DOWN, device)
    return torch.stack([gen_normal_bf16((cfg.hidden, cfg.inter), SIGMA_W, cfg.seed, SID_W_DOWN,
                                        device, index_offset=e * per) for e in experts])


def gen_h(cfg: MoEConfig, device="cpu", row0: int = 0, rows: int | None = None) -> torch.Tensor:
    """Down-projection input [R, inter], already in expert order (N(0,1))."""
    rows = cfg.R - row0 if rows is None else rows
    return gen_normal_bf16((rows, cfg.inter), SIGMA_X, cfg.seed, SID_H, device,
                           index_offset=row0 * cfg.inter)


def gen_dy(cfg: MoEConfig, device="cpu", row0: int = 0, rows: int | None = None) -> torch.Tensor:
    """Up-projection output gradient [R, n_up] in expert order (Student-t(3) + outliers)."""
    rows = cfg.R - row0 if rows is None else rows
    return gen_grad_bf16((rows, cfg.n_up), cfg.seed, SID_DY, device,
                         index_offset=row0 * cfg.n_up)


def gen_y_down(cfg: MoEConfig, device="cpu") -> torch.Tensor:
    """Down-projection output [R, hidden] in expert order (N(0, 1) bf16)."""
    return gen_normal_bf16((cfg.R, cfg.hidden), 1.0, cfg.seed, SID_Y_DOWN, device)


def gen_affinity(cfg: MoEConfig, device="cpu") -> torch.Tensor:
    """Sigmoid affinities of each token's chosen experts [T, k], fp32 in (0, 1)."""
    return gen_uniform_f32((cfg.T, cfg.k), cfg.seed, SID_AFF, device)


def gen_router_logits(cfg: MoEConfig, device="cpu") -> torch.Tensor:
    """Router logits [T, E] fp32 (N(0, 1) values on the bf16 grid)."""
    return gen_normal_bf16((cfg.T, cfg.E), 1.0, cfg.seed, SID_LOGITS, device).to(torch.float32)


def gen_expert_bias(cfg: MoEConfig, device="cpu") -> torch.Tensor:
    """Per-expert routing bias [E] fp32, uniform on (-0.1, 0.1)."""
    return (gen_uniform_f32((cfg.E,), cfg.seed, SID_BIAS, device) - 0.5) * 0.2


def gen_uniform_f32(shape, seed: int, sid: int, device="cpu", index_offset: int = 0) -> torch.Tensor:
    """fp32 values uniform on the 2^24-point grid (i + 0.5) / 2^24 of (0, 1)."""
    numel = math.prod(shape)
    idx = torch.arange(index_offset, index_offset + numel, dtype=torch.int64, device=device)
    u = (hash_index(idx, seed, sid) >> 8).to(torch.float64)
    return ((u + 0.5) / float(1 << 24)).to(torch.float32).view(*shape)


# --------------------------------------------------------------------------
# direct FP8 operands (for GEMM / transpose parity independent of quantization)
# --------------------------------------------------------------------------

def finite_e4m3_codes() -> torch.Tensor:
    """The 254 finite E4M3 bit patterns (all but S.1111.111), as uint8."""
    c = torch.arange(256, dtype=torch.int32)
    keep = (c & 0x7F) != 0x7F
    return c[keep].to(torch.uint8)


@functools.lru_cache(maxsize=None)
def _scale_table(lo_exp: int, hi_exp: int) -> torch.Tensor:
    """2^16 fp32 values log-uniform in [2^lo_exp, 2^hi_exp)."""
    n = 1 << 16
    e = lo_exp + (hi_exp - lo_exp) * (torch.arange(n, dtype=torch.float64) + 0.5) / n
    return torch.exp2(e).to(torch.float32)


def gen_e4m3_codes(shape, seed: int, sid: int, device="cpu", index_offset: int = 0,
                   chunk: int = 1 << 26) -> torch.Tensor:
    """uint8 tensor of uniformly drawn finite E4M3 codes."""
    numel = math.prod(shape)
    codes = finite_e4m3_codes().to(device)
    out = torch.empty(numel, dtype=torch.uint8, device=device)
    for s in range(0, numel, chunk):
        n = min(chunk, numel - s)
        idx = torch.arange(index_offset + s, index_offset + s + n, dtype=torch.int64, device=device)
        out[s:s + n] = codes[hash_index(idx, seed, sid) % codes.numel()]
    return out.view(*shape)


def gen_bytes(shape, seed: int, sid: int, device="cpu", index_offset: int = 0,
              chunk: int = 1 << 26) -> torch.Tensor:
    """uint8 tensor of uniform random bytes."""
    numel = math.prod(shape)
    out = torch.empty(numel, dtype=torch.uint8, device=device)
    for s in range(0, numel, chunk):
        n = min(chunk, numel - s)
        idx = torch.arange(index_offset + s, index_offset + s + n, dtype=torch.int64, device=device)
        out[s:s + n] = (hash_index(idx, seed, sid) & 0xFF).to(torch.uint8)
    return out.view(*shape)


def gen_bytes_at(idx: torch.Tensor, seed: int, sid: int) -> torch.Tensor:
    """The bytes gen_bytes draws at arbitrary flat indices."""
    return (hash_index(idx, seed, sid) & 0xFF).to(torch.uint8)


def gen_scales(shape, seed: int, sid: int, device="cpu", lo_exp: int = -12, hi_exp: int = 0,
               index_offset: int = 0) -> torch.Tensor:
    """fp32 tensor of positive scales, log-uniform in [2^lo_exp, 2^hi_exp)."""
    numel = math.prod(shape)
    tab = _scale_table(lo_exp, hi_exp).to(device)
    idx = torch.arange(index_offset, index_offset + numel, dtype=torch.int64, device=device)
    return tab[hash_index(idx, seed, sid) >> 16].view(*shape)
