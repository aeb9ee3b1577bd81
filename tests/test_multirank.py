"""The multi-GPU bench path is replicas only (tokens are independent; no
data-path collective): each rank runs its own batch through its own layer,
and rank 0 reports the whole job's tokens over the slowest rank's time.
These CPU tests run that host logic on world-size-2 gloo process groups and
the reference arm's rank handling, without a GPU."""
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
from mixture_experts_layer_64_b200 import workloads  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, ws, port, out):
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=ws)
    try:
        # each rank's own timing: the job takes the slowest
        mine = [3.5, 5.25][rank]
        worst = bench.max_over_ranks(dist, mine, "cpu")
        # each rank draws its own batch from the same weights
        w = workloads.WORKLOADS["tiny-fp32"]
        x = workloads.make_x(bench.replica_workload(w, rank))
        digest = float(x.double().sum())
        got = [None] * ws
        dist.all_gather_object(got, digest)
        dist.barrier()
        out.put((rank, worst, got))
    finally:
        dist.destroy_process_group()


def test_replicas_take_the_slowest_rank_and_distinct_batches():
    ws, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, ws, port, q)) for r in range(ws)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(ws)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, worst, digests in res:
        assert worst == 5.25                      # max over ranks, on every rank
        assert digests[0] != digests[1]           # rank-specific batches
    # whole-job throughput: both ranks' tokens over the slowest rank's time
    assert bench.job_throughput(64, 2, 5.25 / 10) == pytest.approx(64 * 2 / 0.000525)
    assert bench.max_over_ranks(None, 1.5, "cpu") == 1.5


def test_reference_arm_rank_handling():
    """Under torchrun only rank 0 runs the reference arm; other ranks exit 0
    without output.  Rank 0 prints one JSON line with the oracle's rate."""
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload",
                        "tiny-fp32", "--steps", "1", "--warmup", "3", "--gpus", "2"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload",
                        "tiny-fp32", "--steps", "2", "--warmup", "3"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0
    assert line["config"]["workload"] == "tiny-fp32"
