"""The multi-process (N > 1) plumbing of bench.py on CPU ranks over gloo: one process per rank,
a barrier and the max over ranks, rank 0 alone printing.  On the GPU machine the same code runs one
replica of the whole workload per GPU with NCCL (no data-path collective: the path shards into
independent replicas)."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_body(rank, world, port, out):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    ws, r = bench.init_dist("gloo")
    assert (ws, r) == (world, rank)
    bench.barrier()
    m = bench.max_over_ranks(10.0 * rank + 0.5)   # the slowest rank's time is the job's
    bench.barrier()
    out.put((rank, m))
    dist.destroy_process_group()


def test_max_over_ranks_and_barrier_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_body, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert got == [(0, 10.5), (1, 10.5)]


def test_reference_arm_under_torchrun_world2():
    # bench.py --impl reference launched as the driver launches it for N > 1: rank 0 times the
    # oracle and prints exactly one JSON line; the other rank exits 0 without work.
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl",
           "reference", "--gpus", "2", "--steps", "1", "--warmup", "0", "--cpu-budget", "1.5"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0
