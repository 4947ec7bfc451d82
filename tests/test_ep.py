"""Expert-parallel dispatch / combine of FP8 rows.

* `test_exchange_two_gloo_ranks` (CPU): two gloo ranks run the host logic of
  fp8_fine_grained_permute_b200.ep.ExpertParallel -- counts exchange, split
  sizes, the uneven all-to-alls of codes, scales and outputs -- with the data
  plane done by plain host code, and compare what each rank receives (and
  gets back from the combine) with the oracle's exchange.
* `test_cuda_data_plane_matches_oracle` (GPU): W ranks emulated on one device
  (the all-to-all replaced by slicing, no collective): every source's rows
  (random E4M3 codes and scales grouped by a seeded routing, some experts
  empty) through fg8_ep_pack_scales, fg8_ep_unpack and fg8_gather_rows, bit
  for bit against the oracle.
"""

import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _source(s, E, K, n_tok=37, k=3):
    """Source rank s's permuted rows: random codes and scales grouped by a
    seeded routing (some experts empty)."""
    rng = np.random.default_rng(100 + s)
    ids = np.stack([rng.choice(E, k, replace=False) for _ in range(n_tok)])
    expert_of_row = np.sort(ids.ravel())
    n = expert_of_row.size
    xq = rng.integers(0, 256, (n, K), dtype=np.uint8)
    sa = rng.random((K // 128, n), dtype=np.float32)
    off = np.concatenate([[0], np.cumsum(np.bincount(expert_of_row, minlength=E))]).astype(np.int32)
    return xq, sa, off, expert_of_row


class HostDataPlane:
    """The exchange's data plane in plain host code, so the host logic of
    ExpertParallel can run on CPU ranks."""

    def pack_scales(self, sa, R, K):
        return sa.t().contiguous()[:R]

    def unpack(self, recv_xq, recv_sa, counts, W, E_loc, R_recv, K):
        c = counts.numpy()
        src_start = np.concatenate([[0], np.cumsum(c.ravel())])[:-1].reshape(W, E_loc)
        order = [src_start[s, e] + i for e in range(E_loc) for s in range(W) for i in range(c[s, e])]
        order = torch.tensor(order, dtype=torch.long)
        r2l = torch.empty(R_recv, dtype=torch.int32)
        r2l[order] = torch.arange(R_recv, dtype=torch.int32)
        off = torch.tensor(np.concatenate([[0], np.cumsum(c.sum(0))]), dtype=torch.int32)
        return recv_xq[order], recv_sa[order].t().contiguous(), off, r2l, None

    def gather_rows(self, inp, index, n):
        return inp[index.long()]


def _rank_main(rank, world, port):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    sys.path.insert(0, ROOT)
    import oracle
    from fp8_fine_grained_permute_b200.ep import ExpertParallel
    E, K = 8, 256
    srcs = [_source(s, E, K) for s in range(world)]
    xq, sa, off, expert_of_row = srcs[rank]
    ep = ExpertParallel(E, kernels=HostDataPlane())
    d = ep.dispatch(torch.from_numpy(xq), torch.from_numpy(sa), torch.from_numpy(off))
    want = oracle.ep_dispatch([s[:3] for s in srcs], world)
    assert np.array_equal(d.xq.numpy(), want[rank]["xq"])
    assert np.array_equal(d.sa.numpy(), want[rank]["sa"])
    assert np.array_equal(d.offsets.numpy(), want[rank]["offsets"])
    # the experts' "outputs": a function of the row and of its expert
    local_expert = np.repeat(np.arange(ep.E_loc), np.diff(d.offsets.numpy())) + rank * ep.E_loc
    y = d.xq[:, :8].to(torch.float32) + 1000.0 * torch.from_numpy(local_expert[:, None].astype(np.float32))
    back = ep.combine(y, d)
    expect = xq[:, :8].astype(np.float32) + 1000.0 * expert_of_row[:, None]
    assert np.array_equal(back.numpy(), expect)
    dist.barrier()
    dist.destroy_process_group()


def test_exchange_two_gloo_ranks():
    mp.start_processes(_rank_main, args=(2, _free_port()), nprocs=2, start_method="spawn",
                       join=True)


@pytest.mark.gpu
def test_cuda_data_plane_matches_oracle(oracle):
    from fp8_fine_grained_permute_b200 import build as fbuild
    from fp8_fine_grained_permute_b200 import fg8
    fbuild.build()
    W, E, K, C = 4, 16, 512, 384
    srcs = [_source(s, E, K, n_tok=200 + 37 * s, k=4) for s in range(W)]
    want = oracle.ep_dispatch([s[:3] for s in srcs], W)
    EL = E // W
    # emulated exchange: every source's rows for rank r (contiguous), scale rows packed on the GPU
    packed = []
    for xq, sa, off, _ in srcs:
        R = xq.shape[0]
        sr = torch.empty((R, K // 128), dtype=torch.float32, device="cuda")
        fg8.fg8_ep_pack_scales(torch.from_numpy(sa).cuda(), R, K, sr)
        packed.append((torch.from_numpy(xq).cuda(), sr, off))
    torch.cuda.synchronize()
    for s, (xq_d, sr, off) in enumerate(packed):
        assert np.array_equal(sr.cpu().numpy(), srcs[s][1].T)
    ys, sends = [], []
    for r in range(W):
        parts_x, parts_s, counts = [], [], []
        for xq_d, sr, off in packed:
            a, b = int(off[r * EL]), int(off[(r + 1) * EL])
            parts_x.append(xq_d[a:b])
            parts_s.append(sr[a:b])
            counts.append(np.diff(off[r * EL:(r + 1) * EL + 1]))
        recv_xq = torch.cat(parts_x).contiguous()
        recv_sa = torch.cat(parts_s).contiguous()
        cnt = torch.from_numpy(np.stack(counts).astype(np.int32)).cuda()
        Rr = recv_xq.shape[0]
        xq_l = torch.empty((Rr, K), dtype=torch.uint8, device="cuda")
        sa_l = torch.empty((K // 128, Rr), dtype=torch.float32, device="cuda")
        off_l = torch.empty(EL + 1, dtype=torch.int32, device="cuda")
        r2l = torch.empty(Rr, dtype=torch.int32, device="cuda")
        st = fg8.new_status()
        fg8.fg8_ep_unpack(recv_xq, recv_sa, cnt, W, EL, Rr, K, xq_l, sa_l, off_l, r2l, st)
        torch.cuda.synchronize()
        assert st.item() == 0
        assert np.array_equal(xq_l.cpu().numpy(), want[r]["xq"])
        assert np.array_equal(sa_l.cpu().numpy(), want[r]["sa"])
        assert np.array_equal(off_l.cpu().numpy(), want[r]["offsets"])
        # combine: local outputs back to the received order
        y_loc = torch.randn((Rr, C), generator=torch.Generator().manual_seed(r)).to(torch.bfloat16).cuda()
        y_send = torch.empty_like(y_loc)
        fg8.fg8_gather_rows(y_loc, Rr, C * 2, r2l, Rr, y_send, st)
        torch.cuda.synchronize()
        assert st.item() == 0
        ys.append(y_loc.cpu().view(torch.int16).numpy())
        sends.append((y_send.cpu().view(torch.int16).numpy(), [int(c.sum()) for c in counts]))
    back = oracle.ep_combine(ys, want, [s[0].shape[0] for s in srcs])
    # the reverse exchange, emulated: source s takes its segment of every
    # rank's received-order outputs, ranks in order -> its own row order
    for s in range(W):
        segs = []
        for y_send, per_src in sends:
            a = sum(per_src[:s])
            segs.append(y_send[a:a + per_src[s]])
        assert np.array_equal(np.concatenate(segs), back[s])


@pytest.mark.gpu
def test_cuda_data_plane_rejects_inconsistent_counts():
    from fp8_fine_grained_permute_b200 import build as fbuild
    from fp8_fine_grained_permute_b200 import fg8
    fbuild.build()
    K, R = 256, 10
    recv_xq = torch.zeros((R, K), dtype=torch.uint8, device="cuda")
    recv_sa = torch.zeros((R, K // 128), dtype=torch.float32, device="cuda")
    cnt = torch.tensor([[3, 4], [1, 1]], dtype=torch.int32, device="cuda")   # sums to 9, not 10
    xq = torch.full((R, K), 7, dtype=torch.uint8, device="cuda")
    sa = torch.zeros((K // 128, R), device="cuda")
    off = torch.zeros(3, dtype=torch.int32, device="cuda")
    r2l = torch.zeros(R, dtype=torch.int32, device="cuda")
    st = fg8.new_status()
    fg8.fg8_ep_unpack(recv_xq, recv_sa, cnt, 2, 2, R, K, xq, sa, off, r2l, st)
    torch.cuda.synchronize()
    assert st.item() == fg8.FG8_ERR_INVALID_ARG
    assert torch.all(xq == 7)
