"""Multi-process host logic of the benchmark on CPU (gloo, world size 2).

The block does not shard: with N GPUs every rank runs its own replica (weak scaling) and the
ranks only agree on the time of the job (the slowest rank) and on who prints.  These tests
run that host logic in two gloo processes; no GPU is involved.
"""
import json
import os
import socket
import subprocess
import sys
import time

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, times, results):
    import torch.distributed as dist

    import bench

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = bench.max_over_ranks(times[rank], world, "cpu")
        results[rank] = (ms, bench.job_tokens_per_s(world, 105, 10, ms))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_gloo():
    world, port = 2, _free_port()
    times = [3.0, 5.0]  # ms of the timed region on each rank
    with mp.Manager() as m:
        results = m.dict()
        mp.spawn(_worker, args=(world, port, times, results), nprocs=world, join=True)
        got = dict(results)
    for rank in range(world):
        ms, tps = got[rank]
        assert ms == 5.0  # every rank sees the slowest rank's time
        assert tps == pytest.approx(world * 105 * 10 / 0.005)


def test_single_rank_helpers_need_no_process_group():
    import bench

    assert bench.max_over_ranks(2.5, 1, "cpu") == 2.5
    assert bench.job_tokens_per_s(1, 105, 4, 2.0) == pytest.approx(105 * 4 / 0.002)


def test_reference_arm_prints_on_rank_zero_only():
    """Under torchrun the oracle arm runs on rank 0; the other ranks exit 0 without output."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0", "--workload", "tiny"]
    env = dict(os.environ, OMP_NUM_THREADS="1")
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0


def _worker_leaves(rank, world, port, q):
    from datetime import timedelta

    import torch.distributed as dist

    import bench

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=10))
    if rank == 1:
        os._exit(3)  # this rank dies between steps, before the timing collective
    t0 = time.time()
    try:
        bench.max_over_ranks(1.0, world, "cpu")
        q.put(("returned", time.time() - t0))
    except Exception as e:  # noqa: BLE001 -- any error from the collective is the expected outcome
        q.put((type(e).__name__, time.time() - t0))


def test_a_rank_that_leaves_makes_the_collective_fail_not_hang():
    """Failure handling between steps on the host: when a rank exits before the timing
    collective, the surviving rank's collective ends with an error within the process group's
    timeout instead of waiting for ever."""
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker_leaves, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    try:
        kind, secs = q.get(timeout=120)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert kind != "returned", "the collective returned although a rank had left"
    assert secs < 60.0
