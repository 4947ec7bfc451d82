"""Expert-parallel dispatch and combine of FP8 rows (host side).

With the experts spread over the W ranks of a process group (rank r owns the
E_loc = E / W experts [r E_loc, (r + 1) E_loc)), every routed row has to reach
the rank that owns its expert and the expert's output has to come back for
the combine: the all-to-all of expert parallelism, with the FP8 codes and
their 1x128 scales crossing the links instead of bf16 rows (DeepSeek-V3
summary sec. 2.2: FP8 training on NVLink / InfiniBand nodes; the Pangu/Ascend
article: the expert-parallel all-to-all).

Steps of `dispatch` (all tensors on the device, one process per GPU, NCCL):
  1. per-destination expert counts, exchanged with one small all-to-all;
  2. one device->host copy of the row totals (the split sizes of the uneven
     all-to-alls below must be known on the host);
  3. the scales repacked per row (fg8_ep_pack_scales), then the codes (as they
     are: the permute already made each destination's rows contiguous) and
     the scale rows exchanged;
  4. the received segments merged into local expert order (fg8_ep_unpack).
`combine` sends each expert output row back (fg8_gather_rows to the order of
arrival, then the reverse all-to-all), so every rank ends with its rows in its
own permuted order, the input of fg8_unpermute_combine.

The data-plane kernels come from `kernels` (default: libfg8's CUDA kernels
through the C ABI); the exchange uses torch.distributed collectives.
"""

from __future__ import annotations

import dataclasses

import torch
import torch.distributed as dist

from . import fg8


class CudaKernels:
    """The data plane of the exchange: libfg8's kernels (device tensors only)."""

    def pack_scales(self, sa: torch.Tensor, R: int, K: int) -> torch.Tensor:
        out = torch.empty((R, K // 128), dtype=torch.float32, device=sa.device)
        fg8.fg8_ep_pack_scales(sa, R, K, out)
        return out

    def unpack(self, recv_xq, recv_sa, counts, W, E_loc, R_recv, K):
        dev = recv_xq.device
        xq = torch.empty((R_recv, K), dtype=torch.uint8, device=dev)
        sa = torch.empty((K // 128, R_recv), dtype=torch.float32, device=dev)
        offsets = torch.empty(E_loc + 1, dtype=torch.int32, device=dev)
        r2l = torch.empty(R_recv, dtype=torch.int32, device=dev)
        st = fg8.new_status(dev)
        fg8.fg8_ep_unpack(recv_xq, recv_sa, counts, W, E_loc, R_recv, K, xq, sa, offsets, r2l, st)
        return xq, sa, offsets, r2l, st

    def gather_rows(self, inp: torch.Tensor, index: torch.Tensor, n: int) -> torch.Tensor:
        out = torch.empty((n,) + tuple(inp.shape[1:]), dtype=inp.dtype, device=inp.device)
        row_bytes = _row_bytes(inp)
        st = fg8.new_status(inp.device)
        fg8.fg8_gather_rows(inp, inp.shape[0], row_bytes, index, n, out, st)
        return out


@dataclasses.dataclass
class Dispatched:
    """What a rank holds after `dispatch`: its local experts' rows, and what
    `combine` needs to send the outputs back."""
    xq: torch.Tensor          # E4M3 [R_recv, K], local expert order
    sa: torch.Tensor          # fp32 [K/128, R_recv]
    offsets: torch.Tensor     # int32 [E_loc + 1]
    recv_to_local: torch.Tensor
    send_rows: list           # rows this rank sent to each rank
    recv_rows: list           # rows this rank received from each rank
    status: torch.Tensor | None = None


def _row_bytes(t: torch.Tensor) -> int:
    return int(torch.Size(t.shape[1:]).numel()) * t.element_size()


def _bytes(t: torch.Tensor) -> torch.Tensor:
    """A flat uint8 view of a contiguous tensor (every backend moves bytes)."""
    return t.contiguous().view(-1).view(torch.uint8)


class ExpertParallel:
    """Dispatch / combine over the process group `group` (None: the default
    group) for a layer of E experts, E divisible by the group size."""

    def __init__(self, E: int, group=None, kernels=None):
        self.group = group
        self.W = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        if E % self.W:
            raise ValueError(f"{E} experts do not split evenly over {self.W} ranks")
        self.E = E
        self.E_loc = E // self.W
        self.k = kernels if kernels is not None else CudaKernels()

    def local_experts(self) -> range:
        return range(self.rank * self.E_loc, (self.rank + 1) * self.E_loc)

    def dispatch(self, xq: torch.Tensor, sa: torch.Tensor, offsets: torch.Tensor) -> Dispatched:
        """xq [R, K] E4M3, sa [K/128, R], offsets [E + 1] from the permuting
        quantizer (rows grouped by expert).  Returns this rank's rows of its
        local experts, in local expert order, ready for the grouped GEMM."""
        W, EL, g = self.W, self.E_loc, self.group
        R, K = xq.shape
        counts = (offsets[1:] - offsets[:-1]).to(torch.int32).view(W, EL).contiguous()
        recv_counts = torch.empty_like(counts)
        dist.all_to_all_single(recv_counts, counts, group=g)
        sizes = torch.stack([counts.sum(1), recv_counts.sum(1)]).cpu()
        send_rows = [int(v) for v in sizes[0]]
        recv_rows = [int(v) for v in sizes[1]]
        R_valid, R_recv = sum(send_rows), sum(recv_rows)
        KB = K // 128
        sa_rows = self.k.pack_scales(sa, R, K)
        recv_xq = torch.empty((R_recv, K), dtype=torch.uint8, device=xq.device)
        recv_sa = torch.empty((R_recv, KB), dtype=torch.float32, device=xq.device)
        dist.all_to_all_single(_bytes(recv_xq), _bytes(xq[:R_valid]),
                               [n * K for n in recv_rows], [n * K for n in send_rows], group=g)
        dist.all_to_all_single(_bytes(recv_sa), _bytes(sa_rows[:R_valid]),
                               [n * KB * 4 for n in recv_rows], [n * KB * 4 for n in send_rows],
                               group=g)
        xq_l, sa_l, off_l, r2l, st = self.k.unpack(recv_xq, recv_sa, recv_counts, W, EL, R_recv, K)
        return Dispatched(xq_l, sa_l, off_l, r2l, send_rows, recv_rows, st)

    def combine(self, y_local: torch.Tensor, d: Dispatched) -> torch.Tensor:
        """y_local [R_recv, C]: the expert outputs of the rows `dispatch`
        returned, in local order.  Returns [R_valid, C]: every row of this
        rank's permuted order with its expert's output (fg8_unpermute_combine's
        y)."""
        R_recv = sum(d.recv_rows)
        y_send = self.k.gather_rows(y_local, d.recv_to_local, R_recv)
        row = _row_bytes(y_local)
        out = torch.empty((sum(d.send_rows),) + tuple(y_local.shape[1:]), dtype=y_local.dtype,
                          device=y_local.device)
        dist.all_to_all_single(_bytes(out), _bytes(y_send), [n * row for n in d.send_rows],
                               [n * row for n in d.recv_rows], group=self.group)
        return out
