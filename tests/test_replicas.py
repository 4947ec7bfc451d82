"""The multi-GPU path of bench.py is N independent replicas (the
configurations fit one GPU; the expert-parallel exchange is out of this
path).  Its host logic -- slowest-rank timing and whole-job throughput --
is exercised here with two gloo ranks on the CPU, and the reference arm is
run under torchrun with two ranks: rank 0 alone prints its line."""

import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    sys.path.insert(0, ROOT)
    import bench
    # rank r "measured" r + 1 ms and 10 - r ms: the job takes the slowest of each
    got = bench.all_max(dist, [rank + 1.0, 10.0 - rank], "cpu")
    rate = bench.job_rate(world, 1e9, got[0])
    with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
        json.dump({"max": got, "rate": rate}, f)
    dist.barrier()
    dist.destroy_process_group()


def test_replica_aggregation_two_gloo_ranks(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    for r in range(world):
        d = json.load(open(tmp_path / f"r{r}.json"))
        assert d["max"] == [2.0, 10.0]
        # 2 ranks x 1e9 units over the slowest rank's 2 ms
        assert d["rate"] == pytest.approx(1e12)


def test_aggregation_without_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.all_max(None, [3, 4.5], "cpu") == [3.0, 4.5]
    assert bench.job_rate(1, 5e9, 1000.0) == pytest.approx(5e9)


def test_reference_arm_two_ranks_prints_once():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py",
           "--impl", "reference", "--config", "tiny", "--gpus", "2", "--steps", "1",
           "--warmup", "0"]
    p = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [ln for ln in p.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0
