"""The multi-rank path of bench.py, on CPU: world size 2 over gloo.

Each rank of `bench.py --gpus N` is an independent replica.  The job's time is the slowest
rank's, and the rate counts every rank's tokens.  The reference arm runs on rank 0 alone
while the other ranks exit without output.  No GPU is involved.
"""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, ws, port, values, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=ws)
    got = bench.max_over_ranks(values[rank], ws, "cpu")
    out.put((rank, got))
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_gloo_world_size_2():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    values = [3.25, 7.5]
    port = free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, values, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = dict(q.get(timeout=10) for _ in range(2))
    assert res == {0: 7.5, 1: 7.5}


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(2.5, 1, "cpu") == 2.5


def test_whole_job_rate_counts_every_rank():
    # two ranks of 10 steps x 16 tokens in 2 ms (the slower rank's time)
    assert bench.whole_job_rate(2, 10, 16, 2.0) == pytest.approx(160000.0)
    assert bench.whole_job_rate(1, 10, 16, 2.0) == pytest.approx(80000.0)


def test_reference_arm_under_torchrun_world_size_2():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(free_port()), "bench.py",
           "--impl", "reference", "--workload", "tiny", "--gpus", "2", "--steps", "3",
           "--warmup", "3"]
    out = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1  # rank 0 alone prints
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
