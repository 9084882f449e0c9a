"""Host logic of the N > 1 path on CPU ranks (gloo, world size 2).

The operator has no exchange step (rows are independent), so multi-GPU runs
are independent replicas; the only cross-rank traffic is the benchmark's
barrier and its max-over-ranks timing reduction. These tests run that logic
in two gloo processes, and the reference arm under torchrun (rank 0 prints
one line, the other ranks exit 0 without work).
"""
import json
import os
import socket
import subprocess
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    w, r, local = bench.dist_setup()
    try:
        assert (w, r, local) == (world, rank, rank)
        bench.barrier(w)
        # each rank reports a different time; every rank receives the max
        t = bench.max_over_ranks(10.0 + 5.0 * rank, w, torch.device("cpu"))
        # aggregate throughput: all ranks' bytes over the slowest rank's time
        value = bench.step_bytes(8192, 3840) * 3 * w / (t / 1e3) / 1e9
        q.put((rank, t, value))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_barrier_gloo():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    assert [g[1] for g in got] == [15.0, 15.0]
    assert got[0][2] == got[1][2] > 0


def test_reference_arm_under_torchrun_prints_once():
    port = _free_port()
    env = dict(os.environ, PYTHONPATH=ROOT)
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py",
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0",
           "--reference-rows", "16"]
    out = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, out.stdout
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2
    assert rec["value"] > 0 and rec["unit"] == "GB/s"
    assert rec["e2e"]["h2d_bytes_per_step"] == 0 and rec["cpu_baseline"]["kind"] == "oracle"
