"""Host logic of the data-parallel bench path, as two gloo ranks on the CPU.

The decode and prefill steps do not shard inside one batch: N GPUs run N
independent replicas, each on its own seeded batch, and the only collective
is the max over ranks of the timed region.  These tests run that logic with
world size 2 over gloo (no GPU).
"""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest

import bench
import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # per-rank device times differ; every rank must see the max
        ms = [3.25, 7.5][rank]
        t = bench.max_over_ranks(ms, world)
        w = bench.replica_workload(1, rank)
        tput = bench.job_throughput(world, w.T, 10, t)
        # a second reduction in the same order on every rank (e2e)
        t2 = bench.max_over_ranks(float(rank + 1), world)
        q.put((rank, t, t2, tput, w.seed, w.idx.tolist()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_max_and_use_own_batches():
    import multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    (_, t0, s0, v0, seed0, idx0), (_, t1, s1, v1, seed1, idx1) = res
    assert t0 == t1 == 7.5
    assert s0 == s1 == 2.0
    assert v0 == v1 == pytest.approx(2 * 256 * 10 / 7.5e-3)
    # replicas process different batches of the same shape
    assert seed0 != seed1 and len(idx0) == len(idx1) == 256
    assert idx0 != idx1
    # and a rank's batch is reproducible
    assert np.array_equal(bench.replica_workload(1, 1).idx, np.asarray(idx1))


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(4.0, 1) == 4.0
    assert bench.job_throughput(1, 256, 4, 2.0) == pytest.approx(512000.0)


def test_reference_arm_runs_on_rank0_only():
    class A:
        config, steps, warmup = 0, 1, 0
    assert bench.run_reference(A, 1, 2) is None


@pytest.mark.timeout(300)
def test_reference_arm_under_torchrun_two_ranks():
    """`bench.py --impl reference` launched as a two-process torchrun job:
    rank 0 prints one JSON line, rank 1 exits 0 without work."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
           "--steps", "1", "--warmup", "0", "--config", "0"]
    env = dict(os.environ, OMP_NUM_THREADS="1")
    out = subprocess.run(cmd, capture_output=True, text=True, timeout=280, env=env, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2
    assert rec["cpu_baseline"]["kind"] == "oracle" and rec["value"] > 0
    assert rec["e2e"]["h2d_bytes_per_step"] == 0
