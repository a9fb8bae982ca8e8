"""Multi-rank host logic of bench.py, on CPU (gloo, world size 2).

The benchmark shards independent problems over ranks (one problem per GPU,
weak scaling) with no data-path collective: ranks meet only at the barriers
around the timed region and in the maximum over ranks of the device time, and
rank 0 alone prints the JSON line.  These tests run that logic on two CPU
processes with the gloo backend, and the reference arm under torchrun.
"""
import datetime
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
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()
        # per-rank device times as a rank would measure them
        mine = [1.0 + rank, 5.0 - rank, 0.25 * rank]
        got = bench.max_over_ranks(mine, world, "cpu")
        dist.barrier()
        out.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_is_the_slowest_rank_on_every_rank():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(out.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    assert res[0] == res[1] == [2.0, 5.0, 0.25]


def test_single_rank_needs_no_process_group():
    assert not dist.is_initialized()
    assert bench.max_over_ranks([3.5, 1.0], 1, "cpu") == [3.5, 1.0]


def test_whole_job_throughput_counts_every_rank():
    # 284 MB per rank per step, slowest rank 0.1 ms: 2.84 TB/s per rank
    assert bench.whole_job_gbs(284e6, 1, 0.1) == pytest.approx(2840.0)
    assert bench.whole_job_gbs(284e6, 2, 0.1) == pytest.approx(5680.0)
    assert bench.whole_job_gbs(284e6, 8, 0.2) == pytest.approx(11360.0)


def test_reference_arm_under_torchrun_prints_once_from_rank_0():
    env = dict(os.environ, OMP_NUM_THREADS="2")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3", "--workload", "tiny_h1_L4k"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(x) for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    line = lines[0]
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["value"] > 0 and line["e2e"]["h2d_bytes_per_step"] == 0
