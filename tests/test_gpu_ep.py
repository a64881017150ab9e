"""Expert parallelism across GPUs, with the R ranks simulated on one GPU.

Each simulated rank runs the expert-parallel calls exactly as one process per
GPU would: it counts its own S tokens' ids (moonep_ep_count), the counts rows
are stacked as an all-gather would leave them, every rank plans from them
(moonep_ep_plan), and the data calls reach the other ranks' buffers through
arrays of R device pointers -- here R separate allocations of one GPU, the
same addressing as peer memory.  The ranks' kernels never wait on one another
(every call only reads what an earlier call in the stream wrote), so running
them one after another on one GPU is the same computation.

Bars (the oracle is the single-GPU plan of the concatenated routing):
* every rank's plan tables equal the oracle's, field by field;
* the ranks' dst_pos rows, concatenated, equal the oracle's dst_pos, and
  their remote-pair counts add up to the oracle's;
* dispatch, combine, combine backward (dy_buf) and the replica-gradient
  reduce bit-exact; dw within the derived bound of the single-GPU tests.
"""
import numpy as np
import pytest
import torch

import oracle
from load_balancing_moonep_b200 import workloads as W

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
TABLES = ("expert_count", "slot_expert", "slot_count", "slot_offset", "rep_expert", "rep_rank", "rep_slot",
          "rep_quota", "host_ptr", "host_rank", "host_slot", "host_start", "host_quota", "rep_home_list",
          "host_local")


@pytest.fixture(scope="module")
def mp(oracle_lib, cuda_lib_path):
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    from load_balancing_moonep_b200 import moonep
    return moonep


@pytest.fixture(autouse=True, params=["one-kernel", "two-kernel"])
def plan_path(request, mp):
    """Every test runs under both expert-parallel planners
    (moonep_set_plan_path): one kernel in which every CTA plans from the
    gathered counts, and the planner CTA followed by the assignment grid."""
    prev = mp.set_plan_path(1 if request.param == "two-kernel" else 0)
    yield request.param
    mp.set_plan_path(prev)


def _ep_plans(mp, cfg, topk):
    """Count, gather (stacking the rows) and plan on every simulated rank."""
    R, S = cfg.R, cfg.S
    plans = [mp.Plan(cfg, DEV, ep=True) for _ in range(R)]
    counts_all = torch.full((R, cfg.E + 1), -7, dtype=torch.int32, device=DEV)
    torch.cuda.synchronize()  # plan blocks and workspaces are zero-filled on the default stream
    for r in range(R):
        mp.ep_count(cfg, topk[r * S:(r + 1) * S].contiguous(), plans[r], counts_row=counts_all[r])
    for r in range(R):
        mp.ep_plan(cfg, r, topk[r * S:(r + 1) * S].contiguous(), counts_all, plans[r])
    torch.cuda.synchronize()
    return plans, counts_all


def _check_plans(cfg, plans, counts_all, topk_np, op):
    R, S, K, E = cfg.R, cfg.S, cfg.K, cfg.E
    # the gathered counts: each rank's own histogram, no invalid ids
    ca = counts_all.cpu().numpy()
    for r in range(R):
        own = np.bincount(topk_np[r * S:(r + 1) * S].ravel(), minlength=E)
        assert np.array_equal(ca[r, :E], own) and ca[r, E] == 0
    remote = 0
    for r, p in enumerate(plans):
        g = p.to_numpy()
        for f in TABLES:
            assert np.array_equal(g[f], op[f]), f"rank {r}: plan field {f} differs"
        info, oinfo = g["info"], op["info"]
        assert np.array_equal(np.delete(info, 7), np.delete(oinfo, 7)), f"rank {r}: info differs"
        assert np.array_equal(g["dst_pos"].ravel()[: S * K], op["dst_pos"].ravel()[r * S * K:(r + 1) * S * K]), \
            f"rank {r}: dst_pos differs"
        remote += int(info[7])
    assert remote == int(op["info"][7])


def _ranks_data_check(mp, cfg, ocfg, plans, op, r_w, P=None, sample_rows=None):
    """Dispatch, combine, combine backward (and the reduce when P is given)
    through per-rank allocations, against the oracle's single-GPU results."""
    R, S, K, H, C = cfg.R, cfg.S, cfg.K, cfg.H, cfg.C
    wl = W.Workload("ep", R, cfg.E, K, S, H, cfg.B)
    hidden = W.hidden_states(wl, seed=1, device=DEV)
    bufs = [torch.full((C, H), float("nan"), dtype=torch.bfloat16, device=DEV) for _ in range(R)]
    bp = mp.pointer_array(bufs)
    for r in range(R):
        mp.ep_dispatch(cfg, plans[r], hidden[r * S:(r + 1) * S].contiguous(), bp)
    torch.cuda.synchronize()
    ob = np.zeros((R, C, H), np.uint16)
    oracle.dispatch(ocfg, op, W.bits(hidden), ob)
    got = np.stack([W.bits(b) for b in bufs])
    assert np.array_equal(got, ob), "dispatch differs"
    # combine on independent expert outputs
    ys = [W.bf16_normal((C, H), seed=20 + r, device=DEV) for r in range(R)]
    yp = mp.pointer_array(ys)
    w = r_w
    outs = [mp.ep_combine(cfg, plans[r], yp, w[r * S:(r + 1) * S].contiguous()) for r in range(R)]
    torch.cuda.synchronize()
    yb = np.stack([W.bits(y) for y in ys])
    oo = oracle.combine(ocfg, op, yb, w.cpu().numpy())
    assert np.array_equal(np.concatenate([W.bits(o) for o in outs]), oo), "combine differs"
    # combine backward
    dy = W.bf16_normal((R * S, H), seed=3, device=DEV)
    dbs = [torch.full((C, H), float("nan"), dtype=torch.bfloat16, device=DEV) for _ in range(R)]
    dp = mp.pointer_array(dbs)
    dws = [mp.ep_combine_backward(cfg, plans[r], dy[r * S:(r + 1) * S].contiguous(),
                                  w[r * S:(r + 1) * S].contiguous(), yp, dp) for r in range(R)]
    torch.cuda.synchronize()
    odyb = np.zeros((R, C, H), np.uint16)
    odw = np.zeros((R * S, K), np.float32)
    oracle.combine_backward(ocfg, op, W.bits(dy), w.cpu().numpy(), yb, odyb, odw)
    assert np.array_equal(np.stack([W.bits(b) for b in dbs]), odyb), "combine backward dy_buf differs"
    dw = np.concatenate([d.cpu().numpy() for d in dws])
    dya = dy.float().abs().cpu().numpy()
    ya = np.concatenate([y.float().abs().cpu().numpy() for y in ys])
    for t0 in range(0, R * S, 512):  # sum_h |dy * y| per pair, in token chunks
        t1 = min(R * S, t0 + 512)
        mag = np.einsum("th,tkh->tk", dya[t0:t1].astype(np.float64), ya[op["dst_pos"][t0:t1]].astype(np.float64))
        err = np.abs(dw[t0:t1].astype(np.float64) - odw[t0:t1])
        assert (err <= 1e-5 * mag + 1e-30).all(), "dw out of tolerance"
    for p in plans:
        assert p.info()["status"] & mp.ST_ROW_RANGE == 0
    if P is None or cfg.B == 0:
        return
    # reduce: rank r's buffer [B, P], its home experts' gradients [L, P]
    L, B = cfg.L, cfg.B
    rbs = [W.f32_normal((B, P), seed=40 + r, device=DEV, std=1e-3) for r in range(R)]
    hgs = [W.f32_normal((L, P), seed=80 + r, device=DEV, std=1e-3) for r in range(R)]
    orb = np.stack([t.cpu().numpy() for t in rbs])
    ohg = np.concatenate([t.cpu().numpy() for t in hgs])
    rp = mp.pointer_array(rbs)
    for r in range(R):
        mp.ep_reduce_replica_grads(cfg, r, plans[r], rp, hgs[r])
    torch.cuda.synchronize()
    oracle.reduce_replica_grads(ocfg, op, orb, ohg, P)
    assert np.array_equal(np.concatenate([t.cpu().numpy() for t in hgs]), ohg), "reduce differs"
    assert np.array_equal(np.stack([t.cpu().numpy() for t in rbs]), orb), "reduce zeroing differs"


@pytest.mark.parametrize("wname,mv,flags", [("tiny", 1.0, 0), ("tiny", 0.0, 0), ("mid", 2.0, 0), ("mid", 0.0, 0),
                                            ("decode", 5.0, 0), ("decode", 20.0, 0), ("ep8", 10.0, 0)])
def test_ep_plan_and_data_match_the_oracle(mp, wname, mv, flags):
    wl = W.WORKLOADS[wname]
    c = dict(R=wl.R, E=wl.E, K=wl.K, S=wl.S, H=wl.H, B=wl.B, flags=flags)
    if wname == "ep8":  # a shorter row keeps the oracle's data steps quick
        c["S"], c["H"] = 512, 256
        wl = wl.with_(S=512, H=256)
    cfg, ocfg = mp.Config(**c), oracle.Config(**c)
    r = W.routing(wl, mv, device=DEV)
    topk_np = r.topk_idx.cpu().numpy()
    op = oracle.plan(ocfg, topk_np)
    plans, counts_all = _ep_plans(mp, cfg, r.topk_idx)
    _check_plans(cfg, plans, counts_all, topk_np, op)
    _ranks_data_check(mp, cfg, ocfg, plans, op, r.weights, P=1000 if wname != "decode" else 64)


@pytest.mark.parametrize("wname,mv,flags", [("tiny", 1.0, 16), ("mid", 2.0, 16), ("mid", 3.0, 16 | 8),
                                            ("decode", 13.4, 16), ("ep8", 20.0, 16)])
def test_ep_locality_plan_and_data_match_the_oracle(mp, wname, mv, flags):
    """MOONEP_FLAG_LOCALITY (with the relay cascade too on one case): every
    rank's tables, including host_local and the leftover starts, the rows of
    its pairs, and the data steps through the per-rank buffers, against the
    oracle; and the ranks keep on their source rank exactly the pairs the
    oracle does, never fewer than without the flag."""
    wl = W.WORKLOADS[wname]
    c = dict(R=wl.R, E=wl.E, K=wl.K, S=wl.S, H=wl.H, B=wl.B, flags=flags)
    if wname == "ep8":
        c["S"], c["H"] = 512, 256
        wl = wl.with_(S=512, H=256)
    if flags & 8:
        c["B"] = 1
    cfg, ocfg = mp.Config(**c), oracle.Config(**c)
    r = W.routing(wl, mv, device=DEV)
    topk_np = r.topk_idx.cpu().numpy()
    op = oracle.plan(ocfg, topk_np)
    op0 = oracle.plan(oracle.Config(**{**c, "flags": flags & ~16}), topk_np)
    assert op["info"][7] <= op0["info"][7]
    plans, counts_all = _ep_plans(mp, cfg, r.topk_idx)
    _check_plans(cfg, plans, counts_all, topk_np, op)
    _ranks_data_check(mp, cfg, ocfg, plans, op, r.weights, P=256 if wname != "decode" else 64)


def test_ep_plan_large_training_shape(mp):
    """The large training shape (R = 32, E = 384, S = 4096): the whole plan
    of every rank, and dispatch through 32 separate allocations checked on
    sampled rows against the hidden rows the oracle's row_src names."""
    wl = W.WORKLOADS["large"]
    c = dict(R=wl.R, E=wl.E, K=wl.K, S=wl.S, H=wl.H, B=wl.B, flags=0)
    cfg, ocfg = mp.Config(**c), oracle.Config(**c)
    r = W.routing(wl, 3.0, device=DEV)
    topk_np = r.topk_idx.cpu().numpy()
    op = oracle.plan(ocfg, topk_np)
    plans, counts_all = _ep_plans(mp, cfg, r.topk_idx)
    _check_plans(cfg, plans, counts_all, topk_np, op)
    hidden = W.hidden_states(wl, seed=1, device=DEV)
    bufs = [torch.empty((wl.C, wl.H), dtype=torch.bfloat16, device=DEV) for _ in range(wl.R)]
    bp = mp.pointer_array(bufs)
    for k in range(wl.R):
        mp.ep_dispatch(cfg, plans[k], hidden[k * wl.S:(k + 1) * wl.S].contiguous(), bp)
    torch.cuda.synchronize()
    rows = np.random.default_rng(0).integers(0, wl.pairs, 4096)
    for g in rows:
        rank, j = divmod(int(g), wl.C)
        src = int(op["row_src"][g]) // wl.K
        assert torch.equal(bufs[rank][j], hidden[src]), f"row {g}"


def test_ep_cascade_plan(mp):
    """The relay cascade through the expert-parallel planner: the 31-replica
    counterexample (one empty rank) planned within B on every rank."""
    wl = W.WORKLOADS["large"].with_(S=256, H=64)
    c = dict(R=wl.R, E=wl.E, K=wl.K, S=wl.S, H=wl.H, B=wl.B, flags=oracle.FLAG_CASCADE)
    cfg, ocfg = mp.Config(**c), oracle.Config(**c)
    r = W.over_budget_routing(wl, seed=0, device=DEV)
    topk_np = r.topk_idx.cpu().numpy()
    op = oracle.plan(ocfg, topk_np)
    assert op["info"][5] <= wl.B and op["info"][8] > 0
    plans, counts_all = _ep_plans(mp, cfg, r.topk_idx)
    _check_plans(cfg, plans, counts_all, topk_np, op)
    _ranks_data_check(mp, cfg, ocfg, plans, op, r.weights, P=256)


def test_ep_bad_id_on_one_rank_empties_every_plan(mp):
    wl = W.WORKLOADS["tiny"]
    c = dict(R=wl.R, E=wl.E, K=wl.K, S=wl.S, H=wl.H, B=wl.B, flags=0)
    cfg, ocfg = mp.Config(**c), oracle.Config(**c)
    topk = W.routing(wl, 1.0, device=DEV).topk_idx.clone()
    topk[wl.S + 3, 1] = wl.E  # rank 1 holds the bad id
    plans, counts_all = _ep_plans(mp, cfg, topk)
    assert counts_all[1, wl.E].item() == 1 and counts_all[0, wl.E].item() == 0
    op = oracle.plan(ocfg, topk.cpu().numpy())
    for p in plans:
        g = p.to_numpy()
        assert g["info"][0] == mp.ST_EXPERT_ID_RANGE
        for f in TABLES:
            assert np.array_equal(g[f], op[f]), f
        assert (g["dst_pos"].ravel()[: wl.S * wl.K] == -1).all()
    # the data calls are no-ops on an empty plan
    bufs = [torch.zeros((wl.C, wl.H), dtype=torch.bfloat16, device=DEV) for _ in range(wl.R)]
    hidden = W.hidden_states(wl, seed=1, device=DEV)
    mp.ep_dispatch(cfg, plans[0], hidden[: wl.S].contiguous(), mp.pointer_array(bufs))
    torch.cuda.synchronize()
    assert all(int(b.view(torch.int16).abs().sum()) == 0 for b in bufs)


def test_ep_null_peer_pointer_is_skipped_and_reported(mp):
    """A null entry in the pointer array: rows bound for that rank are
    skipped (never dereferenced) and MOONEP_ST_ROW_RANGE is set; every other
    rank's rows are written as the oracle has them."""
    wl = W.WORKLOADS["tiny"]
    c = dict(R=wl.R, E=wl.E, K=wl.K, S=wl.S, H=wl.H, B=wl.B, flags=0)
    cfg, ocfg = mp.Config(**c), oracle.Config(**c)
    r = W.routing(wl, 1.0, device=DEV)
    op = oracle.plan(ocfg, r.topk_idx.cpu().numpy())
    plans, _ = _ep_plans(mp, cfg, r.topk_idx)
    hidden = W.hidden_states(wl, seed=1, device=DEV)
    bufs = [torch.zeros((wl.C, wl.H), dtype=torch.bfloat16, device=DEV) for _ in range(wl.R)]
    ptrs = mp.pointer_array([bufs[0], None, bufs[2], bufs[3]])
    for k in range(wl.R):
        mp.ep_dispatch(cfg, plans[k], hidden[k * wl.S:(k + 1) * wl.S].contiguous(), ptrs)
    torch.cuda.synchronize()
    ob = np.zeros((wl.R, wl.C, wl.H), np.uint16)
    oracle.dispatch(ocfg, op, W.bits(hidden), ob)
    for k in (0, 2, 3):
        assert np.array_equal(W.bits(bufs[k]), ob[k])
    assert not bufs[1].view(torch.int16).any()
    dp = op["dst_pos"].reshape(wl.R, wl.S * wl.K)
    for k in range(wl.R):
        sends_to_1 = ((dp[k] // wl.C) == 1).any()
        assert bool(plans[k].info()["status"] & mp.ST_ROW_RANGE) == bool(sends_to_1)


@pytest.mark.parametrize("wname,mv,B", [("tiny", 1.0, None), ("mid", 3.0, None), ("mid", 3.0, 1)])
def test_ep_prefetch_matches_the_oracle(mp, wname, mv, B):
    """Each rank pulls its prefetched replicas' weight rows from the home
    ranks' [L, P] weights (R separate allocations): its pool rows equal the
    oracle's pool[r], and its slot table is the oracle's in the rank's own
    row numbering (home s, pool L + b, overflow read-through L + B + e).
    B = 1 on the mid shape leaves overflow replicas."""
    wl = W.WORKLOADS[wname]
    Bv = wl.B if B is None else B
    c = dict(R=wl.R, E=wl.E, K=wl.K, S=wl.S, H=wl.H, B=Bv, flags=0)
    cfg, ocfg = mp.Config(**c), oracle.Config(**c)
    r = W.routing(wl, mv, device=DEV)
    op = oracle.plan(ocfg, r.topk_idx.cpu().numpy())
    plans, _ = _ep_plans(mp, cfg, r.topk_idx)
    R, E, L, P = wl.R, wl.E, wl.L, 1000
    weights = W.bf16_normal((E, P), seed=7, device=DEV)
    owners = [weights[h * L:(h + 1) * L].clone() for h in range(R)]  # each rank's home weights
    wp = mp.pointer_array(owners)
    pools = [torch.zeros((Bv, P), dtype=torch.bfloat16, device=DEV) for _ in range(R)]
    tables = [mp.ep_prefetch_replicas(cfg, k, plans[k], wp, pools[k]) for k in range(R)]
    torch.cuda.synchronize()
    opool = np.zeros((R, Bv, P), np.uint16)
    owrow = oracle.prefetch_replicas(ocfg, op, W.bits(weights), opool, P)
    if wname == "mid" and B == 1:
        assert op["info"][2] > 0  # overflow replicas present
    for k in range(R):
        assert np.array_equal(W.bits(pools[k]), opool[k]), f"rank {k}: pool differs"
        exp = np.full(E, -1, np.int32)
        for s in range(E):
            e, row = op["slot_expert"][k, s], owrow[k, s]
            if e < 0:
                continue
            if s < L:
                exp[s] = s
            elif row >= E:  # a prefetched replica: pool row E + k*B + b
                exp[s] = L + (row - E - k * Bv)
            else:  # overflow: read through from the home rank
                exp[s] = L + Bv + e
        assert np.array_equal(tables[k].cpu().numpy(), exp), f"rank {k}: slot table differs"
