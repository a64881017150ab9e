"""The benchmark's multi-rank host path on CPU with the gloo backend.

N GPUs run N independent replicas of the step (the simulated ranks live in
one GPU), so the only cross-rank operations are a barrier and the max over
ranks of the measured times; the reference (CPU oracle) arm runs on rank 0
alone.  World size 2, rendezvous on 127.0.0.1.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as tmp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    if not dist.is_initialized():
        dist.init_process_group("gloo", rank=rank, world_size=world)
    bench.barrier(world)
    m = bench.max_over_ranks(world, float(10 + rank))
    s = bench.sum_over_ranks(world, float(1 + rank))
    bench.barrier(world)
    q.put((rank, m, s))
    dist.destroy_process_group()


def test_max_and_sum_over_two_ranks():
    if torch.cuda.is_available():
        pytest.skip("host-path test (gloo); GPUs present")
    ctx = tmp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, m, s in out:
        assert m == 11.0 and s == 3.0


def test_reference_arm_rank0_only_under_torchrun():
    if torch.cuda.is_available():
        pytest.skip("host-path test (gloo); GPUs present")
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--workload", "tiny", "--gpus", "2", "--steps", "1", "--warmup", "3",
           "--ref-tokens", "64"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["unit"] == "GB/s"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0
