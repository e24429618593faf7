"""The multi-GPU path of bench.py on the CPU: two ranks over gloo.

bench.py runs N independent replicas (one process per GPU); its only collectives are the
barrier around the timed region and the max over ranks of the timing. These tests run that
plumbing as two gloo ranks, and launch the reference arm under torch.distributed.run with two
processes, where rank 0 alone prints the JSON line."""

from __future__ import annotations

import json
import multiprocessing as mp
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank: int, world: int, port: int, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank), CUDA_VISIBLE_DEVICES="")
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import bench

    w, r, _ = bench.dist_setup()
    try:
        bench.barrier(w)
        ms = bench.max_over_ranks(10.0 * (r + 1), w)  # rank-dependent "timings"
        bench.barrier(w)
        q.put((r, w, dist.get_backend(), ms))
    finally:
        dist.destroy_process_group()


def test_replica_plumbing_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    assert [g[0] for g in got] == [0, 1]
    assert all(g[1] == 2 and g[2] == "gloo" for g in got)
    assert all(g[3] == 20.0 for g in got)  # every rank sees the max over ranks


@pytest.mark.timeout(600)
def test_reference_arm_under_torchrun_two_ranks():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py",
           "--impl", "reference", "--gpus", "2", "--steps", "2", "--warmup", "3",
           "--workload", "fwd_b2h1n512d64"]
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="", OMP_NUM_THREADS="2")
    out = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=540)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, out.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["config"]["workload"] == "fwd_b2h1n512d64" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0
