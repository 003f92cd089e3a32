"""The multi-rank path of bench.py on CPU, world size 2 over gloo (on GPUs the same calls run
over NCCL).  bench.py runs one replica per rank with no data-path collective; these tests
cover the host logic around the replicas: the slowest rank's time, the whole-job
throughput, and the reference arm under torchrun (rank 0 alone works and prints)."""
import datetime
import json
import os
import socket
import subprocess
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _max_worker(rank: int, world: int, port: int):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        got = bench.max_over_ranks(10.0 + 5.0 * rank, torch.device("cpu"))
        assert got == 10.0 + 5.0 * (world - 1), (rank, got)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_is_the_slowest_rank():
    mp.spawn(_max_worker, args=(2, _free_port()), nprocs=2, join=True)


def test_max_over_ranks_without_a_process_group_is_the_value():
    assert bench.max_over_ranks(3.5, torch.device("cpu")) == 3.5


def test_job_throughput_counts_every_replica():
    # 2 replicas x 5 steps x 131072 tokens in 1 s.
    assert bench.job_tokens_per_s(2, 131072, 5, 1000.0) == 2 * 5 * 131072


def test_reference_arm_under_torchrun_prints_once():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py",
           "--impl", "reference", "--workload", "tiny", "--steps", "1", "--warmup", "3",
           "--oracle-rows", "32"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [line for line in r.stdout.splitlines() if line.startswith("{")]
    assert len(lines) == 1, r.stdout[-2000:]
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["e2e"]["h2d_bytes_per_step"] == 0
