"""Expert parallelism's host path across processes, on CPU with gloo.

In expert parallelism every rank counts its own tokens' experts and the R
counts rows are all-gathered (the binding's ep_gather_counts, the one
collective of an expert-parallel plan); every rank then plans from the same
rows.  Here two processes (world size 2, rendezvous on 127.0.0.1) each hold
their half of one routing: after the all-gather both hold the same [R, E+1]
rows in rank order, and the plan tables each derives from them -- with the
CPU oracle, since the planner kernel needs a GPU -- are identical on both
ranks and equal the single-process plan of the whole routing.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as tmp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
TABLES = ("expert_count", "slot_expert", "slot_count", "slot_offset", "rep_expert", "rep_rank", "rep_slot",
          "rep_quota", "host_ptr", "host_rank", "host_slot", "host_start", "host_quota", "rep_home_list")


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _routing():
    """R = 2 ranks, E = 8 experts (4 home each), K = 2, S = 12 tokens per
    rank; rank 0's tokens lean on experts 0 and 1, so rank 1 receives
    replicas."""
    rng = np.random.default_rng(5)
    R, E, K, S = 2, 8, 2, 12
    logits = rng.standard_normal((R * S, E))
    logits[:, :2] += 2.0
    topk = np.argsort(-logits, axis=1, kind="stable")[:, :K].astype(np.int32)
    return dict(R=R, E=E, K=K, S=S, H=8, B=2), topk


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import oracle
    from load_balancing_moonep_b200 import moonep as mp
    dist.init_process_group("gloo", rank=rank, world_size=world)
    cfg, topk = _routing()
    E, S = cfg["E"], cfg["S"]
    mine = topk[rank * S:(rank + 1) * S]
    # this rank's counts row as moonep_ep_count defines it: pairs per expert,
    # then the ids outside [0, E)
    row = torch.zeros(E + 1, dtype=torch.int32)
    row[:E] = torch.from_numpy(np.bincount(mine.ravel(), minlength=E).astype(np.int32))
    counts_all = mp.ep_gather_counts(row)
    ca = counts_all.numpy()
    # any routing with these per-rank counts has the same plan tables: take
    # each rank's ids in expert order
    canon = np.concatenate([np.repeat(np.arange(E, dtype=np.int32), ca[r, :E]) for r in range(world)])
    p = oracle.plan(oracle.Config(**cfg), canon.reshape(-1, cfg["K"]))
    q.put((rank, ca.tolist(), {f: p[f].tolist() for f in TABLES}, p["info"][:7].tolist()))
    dist.barrier()
    dist.destroy_process_group()


def test_gathered_counts_give_identical_plans_on_both_ranks(oracle_lib, cuda_lib_path):
    if torch.cuda.is_available():
        pytest.skip("host-path test (gloo); GPUs present")
    import oracle
    ctx = tmp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    cfg, topk = _routing()
    E, S = cfg["E"], cfg["S"]
    expect_counts = [np.bincount(topk[r * S:(r + 1) * S].ravel(), minlength=E).tolist() + [0] for r in range(2)]
    whole = oracle.plan(oracle.Config(**cfg), topk)
    assert whole["info"][1] > 0  # the routing needs replicas
    for rank, ca, tables, info in out:
        assert ca == expect_counts, f"rank {rank}: gathered rows out of rank order"
        for f in TABLES:
            assert tables[f] == whole[f].tolist(), f"rank {rank}: {f}"
        assert info == whole["info"][:7].tolist()
    assert out[0][2] == out[1][2]
