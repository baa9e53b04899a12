"""The multi-rank path of bench.py on CPU (gloo, world_size 2).

bench.py runs one rank per GPU, each on its own batch of tokens (weak scaling, no
data-path collective). The host logic that crosses ranks — barriers, the max of
the ranks' elapsed times, the whole-job throughput, and "rank 0 alone prints" for
the reference arm — is exercised here with two CPU processes.
"""
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


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import datetime
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        w, r, lr = bench.dist_env()
        bench.barrier(w)
        ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
        worst = bench.max_over_ranks(ms, w)
        value = bench.tokens_per_second(4096, w, 20, worst)
        bench.barrier(w)
        q.put((rank, w, r, lr, worst, value))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_value():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    for rank, (r, w, r2, lr, worst, value) in enumerate(got):
        assert (r, w, r2, lr) == (rank, 2, rank, rank)
        assert worst == 15.0  # the slowest rank's time, on every rank
        # both ranks' tokens over the slowest rank's time
        assert value == pytest.approx(4096 * 2 * 20 / 0.015)


def test_single_rank_helpers_need_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    bench.barrier(1)
    assert bench.tokens_per_second(64, 1, 10, 2.0) == pytest.approx(64 * 10 / 0.002)


def test_reference_arm_under_torchrun_prints_once():
    """`torchrun --nproc-per-node 2 bench.py --impl reference`: rank 0 alone runs and
    prints one JSON line; rank 1 exits 0 without work."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr=127.0.0.1", f"--master-port={port}", os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--workload", "tiny", "--steps", "2", "--warmup", "3",
           "--gpus", "2"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2 and rec["value"] > 0
    assert rec["e2e"]["h2d_bytes_per_step"] == 0 and rec["cpu_baseline"]["kind"] == "oracle"
