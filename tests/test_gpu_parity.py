"""GPU parity: the CUDA library (through its C ABI) against the CPU oracle on
identical seeded inputs.

Bars: plan, counts, offsets, dst_pos, row_src and dispatched rows bit-exact;
combine and dy_buf bit-exact (same fp32 fused multiply-add order and one
round-to-nearest-even); replica-gradient reduce bit-exact (same fp32 add
order); dw within |dw - ref| <= 1e-5 * sum_h |dy*y| + 1e-30 (GPU reduction
tree in fp32 vs the oracle's fp64 sum; the tree's worst-case bound is
(8 + H/256 + 5) * 2^-24 relative to sum |dy*y|, under 1e-5 for H <= 37k).

Small cases compare every element; the full-size configurations (large
training shape, decode) compare the whole plan and sampled tokens / rows /
element ranges of the data steps, run in the launch configuration the
benchmark times.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from load_balancing_moonep_b200 import workloads as W
from plan_checks import check_invariants, check_water_filling

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
DEV = "cuda:0"


@pytest.fixture(scope="module")
def mp(oracle_lib, cuda_lib_path):
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    from load_balancing_moonep_b200 import moonep
    return moonep


@pytest.fixture(autouse=True, params=["one-kernel", "two-kernel"])
def plan_path(request, mp):
    """Every test runs under both planners (moonep_set_plan_path): the one
    kernel wherever its CTAs all fit on the GPU, and the two-kernel path."""
    prev = mp.set_plan_path(1 if request.param == "two-kernel" else 0)
    yield request.param
    mp.set_plan_path(prev)


def _cfgs(c: dict, mp):
    return mp.Config(**c), oracle.Config(**c)


def _plan_both(mp, c: dict, topk: np.ndarray):
    gcfg, ocfg = _cfgs(c, mp)
    t = torch.from_numpy(np.ascontiguousarray(topk, np.int32)).to(DEV)
    gp = mp.plan(gcfg, t)
    torch.cuda.synchronize()
    return gcfg, ocfg, gp, oracle.plan(ocfg, topk)


def _assert_plan_equal(gp, op):
    g = gp.to_numpy()
    for k, v in op.items():
        assert np.array_equal(g[k], v), f"plan field {k} differs"


def _wl_cfg(wl, **kw):
    d = dict(R=wl.R, E=wl.E, K=wl.K, S=wl.S, H=wl.H, B=wl.B, flags=0)
    d.update(kw)
    return d


# ------------------------------------------------------------------ plan

@pytest.mark.parametrize("name", ["plan_example_a", "plan_example_b"])
@pytest.mark.parametrize("flags", [0, 1])
def test_plan_golden(mp, name, flags):
    g = json.load(open(os.path.join(GOLDEN, name + ".json")))
    c = {**g["config"], "flags": flags}
    topk = np.array(g["topk_idx"], np.int32)
    gcfg, ocfg, gp, op = _plan_both(mp, c, topk)
    _assert_plan_equal(gp, op)
    for k, v in g["expect"].items():
        if k != "info":
            assert gp.fields[k].cpu().numpy().tolist() == v


@pytest.mark.parametrize("wname,mv,adv", [
    ("tiny", 0.0, False), ("tiny", 1.0, False), ("tiny", 1.0, True), ("tiny", 3.0, False),
    ("mid", 0.0, False), ("mid", 0.5, False), ("mid", 1.0, False), ("mid", 2.0, False),
    ("mid", 3.0, False), ("mid", 3.0, True),
    ("decode", 5.0, False), ("decode", 13.4, False), ("decode", 20.0, False),
])
def test_plan_workloads(mp, wname, mv, adv):
    wl = W.WORKLOADS[wname]
    r = W.routing(wl, mv, seed=0, adversarial=adv, device=DEV)
    topk = r.topk_idx.cpu().numpy()
    gcfg, ocfg, gp, op = _plan_both(mp, _wl_cfg(wl), topk)
    _assert_plan_equal(gp, op)
    check_invariants(ocfg, topk, gp.to_numpy())


@pytest.mark.parametrize("mv,adv", [(0.0, False), (1.0, False), (3.0, False), (3.0, True)])
def test_plan_large_full_size(mp, mv, adv):
    wl = W.WORKLOADS["large"]
    r = W.routing(wl, mv, seed=0, adversarial=adv, device=DEV)
    topk = r.topk_idx.cpu().numpy()
    gcfg, ocfg, gp, op = _plan_both(mp, _wl_cfg(wl), topk)
    _assert_plan_equal(gp, op)
    check_invariants(ocfg, topk, gp.to_numpy())
    check_water_filling(ocfg, topk, gp.to_numpy())


@pytest.mark.parametrize("seed", range(16))
def test_plan_random_shapes(mp, seed):
    # ragged shapes: token counts that are not multiples of the chunk size,
    # every L, B from 0 to E-L, heavy and light skew
    rng = np.random.default_rng(100 + seed)
    R = int(rng.choice([1, 2, 3, 5, 8, 16, 64]))
    L = int(rng.choice([1, 2, 3, 7, 12]))
    E = R * L
    if E > 1024:
        L = max(1, 1024 // R)
        E = R * L
    K = int(rng.integers(1, min(E, 9) + 1))
    S = int(rng.integers(1, 300))
    B = int(rng.integers(0, E - L + 1))
    skew = float(rng.uniform(0, 3))
    w = np.arange(1, E + 1, dtype=np.float64) ** (-skew)
    w = w[rng.permutation(E)]
    w /= w.sum()
    topk = np.stack([rng.choice(E, size=K, replace=False, p=w) for _ in range(R * S)]).astype(np.int32)
    c = dict(R=R, E=E, K=K, S=S, H=8, B=B, flags=int(rng.integers(0, 2)))
    gcfg, ocfg, gp, op = _plan_both(mp, c, topk)
    _assert_plan_equal(gp, op)
    check_invariants(ocfg, topk, gp.to_numpy())


def test_plan_duplicates_within_token(mp):
    # the pages are silent on repeated ids in one token's top-K: they are
    # independent pairs; both sides must agree
    rng = np.random.default_rng(5)
    topk = rng.integers(0, 8, size=(4 * 20, 3)).astype(np.int32)
    _, ocfg, gp, op = _plan_both(mp, dict(R=4, E=8, K=3, S=20, H=8, B=2), topk)
    _assert_plan_equal(gp, op)


def test_plan_all_on_one_expert_and_max_E(mp):
    topk = np.zeros((64 * 5, 1), np.int32)
    _, _, gp, op = _plan_both(mp, dict(R=64, E=128, K=1, S=5, H=8, B=2), topk)
    _assert_plan_equal(gp, op)
    assert gp.info()["n_rep"] == 63
    rng = np.random.default_rng(9)
    topk = rng.integers(0, 1024, size=(1024 * 4, 4)).astype(np.int32)
    topk[: 1024, :] = 0  # one very hot expert
    _, ocfg, gp, op = _plan_both(mp, dict(R=1024, E=1024, K=4, S=4, H=8, B=1), topk)
    _assert_plan_equal(gp, op)
    check_invariants(ocfg, topk, gp.to_numpy())


def test_plan_bad_ids_status_and_noop(mp):
    c = dict(R=4, E=16, K=2, S=64, H=64, B=2)
    rng = np.random.default_rng(1)
    topk = rng.integers(0, 16, size=(256, 2)).astype(np.int32)
    topk[77, 1] = 16
    gcfg, ocfg, gp, op = _plan_both(mp, c, topk)
    _assert_plan_equal(gp, op)
    assert gp.info()["status"] & mp.ST_EXPERT_ID_RANGE
    hidden = W.hidden_states(W.Workload("x", 4, 16, 2, 64, 64, 2), seed=3, device=DEV)
    buf = torch.full((4, 128, 64), 7.0, dtype=torch.bfloat16, device=DEV)
    mp.dispatch(gcfg, gp, hidden, buf)
    out = torch.full((256, 64), 5.0, dtype=torch.bfloat16, device=DEV)
    mp.combine(gcfg, gp, buf, torch.ones(256, 2, device=DEV), out)
    torch.cuda.synchronize()
    assert (buf == 7.0).all() and (out == 5.0).all()
    # a following valid plan with the same workspace is unaffected
    topk[77, 1] = 3
    t = torch.from_numpy(topk).to(DEV)
    gp2 = mp.plan(gcfg, t, out=gp)
    _assert_plan_equal(gp2, oracle.plan(ocfg, topk))


def test_plan_repeat_deterministic(mp):
    wl = W.WORKLOADS["mid"]
    r = W.routing(wl, 2.0, device=DEV)
    cfg = mp.Config(**_wl_cfg(wl))
    p1 = mp.plan(cfg, r.topk_idx).to_numpy()
    p = mp.Plan(cfg)
    for _ in range(3):
        p2 = mp.plan(cfg, r.topk_idx, out=p).to_numpy()
        for k in p1:
            assert np.array_equal(p1[k], p2[k])


def test_plan_alternating_routings_reuse_workspace(mp):
    """Many calls on one plan block and workspace, alternating two routings.
    Every call flips the group-count buffer (low bit of the call sequence),
    the assignment CTAs zero the other one, and the counts-ready mark of one
    call must never pass for the next: every plan must equal the oracle's."""
    wl = W.WORKLOADS["mid"]
    gcfg, ocfg = _cfgs(_wl_cfg(wl), mp)
    rs = [W.routing(wl, mv, device="cpu") for mv in (0.5, 3.0)]
    ops = [oracle.plan(ocfg, r.topk_idx.numpy()) for r in rs]
    tks = [r.topk_idx.to(DEV) for r in rs]
    p = mp.Plan(gcfg)
    for it in range(24):
        mp.plan(gcfg, tks[it % 2], out=p)
        _assert_plan_equal(p, ops[it % 2])


# ------------------------------------------------------- relay cascade

def _cascade_routing(rng, R, L, S, K=1):
    """Skewed routing with an empty expert or two, so water-filling overflows
    small budgets often; token order shuffled."""
    E = R * L
    w = rng.random(E) ** 3
    w[rng.integers(0, E, size=2)] = 0
    T = rng.multinomial(R * S * K, w / w.sum())
    ids = np.repeat(np.arange(E), T)
    rng.shuffle(ids)
    return ids.reshape(R * S, K).astype(np.int32)


@pytest.mark.parametrize("name", ["plan_example_cascade", "plan_example_cascade_relay", "plan_example_cascade_merge",
                                  "plan_example_cascade_chain", "plan_example_cascade_two_relays"])
def test_plan_cascade_golden(mp, name):
    g = json.load(open(os.path.join(GOLDEN, name + ".json")))
    topk = np.array(g["topk_idx"], np.int32)
    gcfg, ocfg, gp, op = _plan_both(mp, g["config"], topk)
    _assert_plan_equal(gp, op)
    for k, v in g["expect"].items():
        if k == "info":
            inf = gp.info()
            assert {f: inf[f] for f in v} == v
        else:
            assert gp.fields[k].cpu().numpy().tolist() == v, k


@pytest.mark.parametrize("name,caps", [("plan_example_cascade", (4, 3)),
                                       ("plan_example_cascade_chain", (5, 6, 7)),
                                       ("plan_example_cascade_merge", (4, 5))])
def test_plan_cascade_guard_at_lowered_capacities(mp, name, caps):
    """The cascade guard's comparison on the GPU: with the capacity lowered in
    both the CUDA planner and the oracle, steps exactly on the limit are
    taken and steps one over are skipped, identically, whole plan."""
    g = json.load(open(os.path.join(GOLDEN, name + ".json")))
    topk = np.array(g["topk_idx"], np.int32)
    try:
        for cap in caps:
            mp.set_cascade_capacity(cap)
            oracle.set_cascade_capacity(cap)
            gcfg, ocfg, gp, op = _plan_both(mp, g["config"], topk)
            _assert_plan_equal(gp, op)
            if name == "plan_example_cascade":
                assert op["info"][9] == (0 if cap == 4 else -1)
    finally:
        mp.set_cascade_capacity(0)
        oracle.set_cascade_capacity(0)


def test_plan_cascade_counterexample_and_data(mp):
    """The 31-replica counterexample: the cascade's plan, then dispatch and
    combine over it, element for element against the oracle."""
    R, E, S, B, H = 32, 384, 3100, 12, 16
    L = E // R
    T = np.zeros(E, np.int64)
    for r in range(1, R):
        T[r * L:(r + 1) * L] = [300] * 10 + [100] * 2
    ids = np.repeat(np.arange(E), T)
    np.random.default_rng(0).shuffle(ids)
    topk = ids.reshape(R * S, 1).astype(np.int32)
    c = dict(R=R, E=E, K=1, S=S, H=H, B=B, flags=mp.FLAG_CASCADE)
    gcfg, ocfg, gp, op = _plan_both(mp, c, topk)
    _assert_plan_equal(gp, op)
    assert gp.info()["status"] == 0 and gp.info()["max_rep_per_rank"] == B
    wl = W.Workload("cx", R, E, 1, S, H, B)
    hidden = W.hidden_states(wl, seed=1, device=DEV)
    buf = torch.full((R, S, H), float("nan"), dtype=torch.bfloat16, device=DEV)
    mp.dispatch(gcfg, gp, hidden, buf)
    ob = np.zeros((R, S, H), np.uint16)
    oracle.dispatch(ocfg, op, W.bits(hidden), ob)
    assert np.array_equal(W.bits(buf), ob)
    w = W.f32_normal((R * S, 1), seed=4, device=DEV)
    out = mp.combine(gcfg, gp, buf, w)
    assert np.array_equal(W.bits(out), oracle.combine(ocfg, op, ob, w.cpu().numpy()))


@pytest.mark.parametrize("seed", range(6))
def test_plan_cascade_random(mp, seed):
    """Random skewed routings over small budgets, with and without strict
    mode: the cascade plan (or the overflow it could not avoid) equals the
    oracle's."""
    rng = np.random.default_rng(300 + seed)
    for trial in range(6):
        R = int(rng.choice([4, 8, 16]))
        L = int(rng.choice([2, 3, 4]))
        K = int(rng.choice([1, 2]))
        S = int(rng.integers(8, 64))
        B = int(rng.choice([1, 2]))
        flags = mp.FLAG_CASCADE | (mp.FLAG_STRICT_BUDGET if trial % 3 == 0 else 0)
        topk = _cascade_routing(rng, R, L, S, K)
        c = dict(R=R, E=R * L, K=K, S=S, H=8, B=B, flags=flags)
        _, ocfg, gp, op = _plan_both(mp, c, topk)
        _assert_plan_equal(gp, op)
        check_invariants(ocfg, topk, gp.to_numpy())


def test_plan_cascade_within_budget_is_water_filling(mp):
    wl = W.WORKLOADS["mid"]
    r = W.routing(wl, 2.0, device=DEV)
    topk = r.topk_idx.cpu().numpy()
    _, _, g0, _ = _plan_both(mp, _wl_cfg(wl), topk)
    _, _, g1, o1 = _plan_both(mp, _wl_cfg(wl, flags=mp.FLAG_CASCADE), topk)
    _assert_plan_equal(g1, o1)
    a0, a1 = g0.to_numpy(), g1.to_numpy()
    for k in a0:
        assert np.array_equal(a0[k], a1[k]), k


@pytest.mark.parametrize("flags", [0, 8])
def test_plan_over_budget_full_size(mp, flags):
    """The large training shape with one empty rank: water-filling puts 31
    replicas on it; the cascade keeps every rank within B = 12.  Every plan
    field against the oracle."""
    wl = W.WORKLOADS["large"]
    topk = W.over_budget_routing(wl).topk_idx.numpy()
    _, ocfg, gp, op = _plan_both(mp, _wl_cfg(wl, flags=flags), topk)
    _assert_plan_equal(gp, op)
    inf = gp.info()
    assert inf["max_rep_per_rank"] == (wl.B if flags else wl.R - 1)
    check_invariants(ocfg, topk, gp.to_numpy())


@pytest.mark.parametrize("R,E,K,S,B", [(1024, 1024, 4, 64, 1), (256, 1024, 8, 256, 4), (64, 384, 8, 128, 4)])
def test_plan_cascade_wide_shapes(mp, R, E, K, S, B):
    """One empty rank among many: at E = R = 1024 the cascade makes 255
    repairs on the largest lists; at R = 64, B = 4 no plan within budget
    exists (rank 0 needs C rows from at most 4 replicas, each below C / 4)
    and the overflow stays.  Against the oracle, with the host invariants."""
    wl = W.Workload("wide", R, E, K, S, 8, B)
    topk = W.over_budget_routing(wl).topk_idx.numpy()
    _, ocfg, gp, op = _plan_both(mp, dict(R=R, E=E, K=K, S=S, H=8, B=B, flags=mp.FLAG_CASCADE), topk)
    _assert_plan_equal(gp, op)
    check_invariants(ocfg, topk, gp.to_numpy())


@pytest.mark.parametrize("R,E,K,S,B", [(32, 384, 1, 3100, 12), (16, 64, 2, 40, 4), (16, 128, 2, 64, 8)])
def test_cascade_plan_reduce_and_prefetch(mp, R, E, K, S, B):
    """The replica-gradient reduce and the weight prefetch over a cascade
    plan (relay replicas, merged replicas, returned quota), every element
    against the oracle."""
    wl = W.Workload("cx", R, E, K, S, 8, B)
    topk = W.over_budget_routing(wl).topk_idx.numpy()
    gcfg, ocfg, gp, op = _plan_both(mp, dict(R=R, E=E, K=K, S=S, H=8, B=B, flags=mp.FLAG_CASCADE), topk)
    _assert_plan_equal(gp, op)
    assert op["info"][0] == 0 and op["info"][2] == 0  # within budget, nothing overflows
    P = 72
    rb = W.f32_normal((R, B, P), seed=4, device=DEV, std=1e-3)
    hg = W.f32_normal((E, P), seed=5, device=DEV, std=1e-3)
    orb, ohg = rb.cpu().numpy(), hg.cpu().numpy()
    mp.reduce_replica_grads(gcfg, gp, rb, hg)
    oracle.reduce_replica_grads(ocfg, op, orb, ohg, P)
    assert np.array_equal(hg.cpu().numpy(), ohg)
    assert np.array_equal(rb.cpu().numpy(), orb)
    weights = W.bf16_normal((E, P), seed=6, device=DEV)
    pool = torch.full((R, B, P), float("nan"), dtype=torch.bfloat16, device=DEV)
    opool = W.bits(pool).copy()
    wrow = mp.prefetch_replicas(gcfg, gp, weights, pool)
    owrow = oracle.prefetch_replicas(ocfg, op, W.bits(weights), opool, P)
    assert np.array_equal(wrow.cpu().numpy(), owrow)
    assert np.array_equal(W.bits(pool), opool)


def test_plan_many_chunks_multi_wave(mp):
    """More token chunks (512, in 32 groups) than two CTAs per SM can hold at
    once: both planner grids run in several waves, and assignment CTAs wait
    for the counts-ready mark while later histogram CTAs still run.  The plan
    must equal the oracle's."""
    c = dict(R=64, E=256, K=8, S=4096, H=16, B=4, flags=0)
    T = c["R"] * c["S"]
    g = torch.Generator(device=DEV).manual_seed(7)
    bias = -1.2 * torch.log(torch.randperm(c["E"], generator=g, device=DEV).float() + 1.0)
    scores = torch.randn((T, c["E"]), generator=g, device=DEV) + bias
    topk = torch.topk(scores, c["K"], dim=1).indices.to(torch.int32).cpu().numpy()
    del scores
    gcfg, ocfg, gp, op = _plan_both(mp, c, topk)
    _assert_plan_equal(gp, op)
    assert op["info"][1] > 0  # the skew made replicas


def test_plan_in_cuda_graph_replays(mp):
    """The plan captured in a CUDA graph (its programmatic launch edge and
    counts-ready handshake replayed) with fresh routings written into the
    captured input between replays: every replay equals the oracle."""
    wl = W.WORKLOADS["decode"]
    gcfg, ocfg = _cfgs(_wl_cfg(wl), mp)
    rs = [W.routing(wl, mv, seed=sd, device="cpu") for sd, mv in ((0, 5.0), (1, 5.0), (2, 1.0))]
    ops = [oracle.plan(ocfg, r.topk_idx.numpy()) for r in rs]
    topk = rs[0].topk_idx.to(DEV).clone()
    p = mp.Plan(gcfg)
    torch.cuda.synchronize()  # the plan block was zero-filled on the default stream
    cs = torch.cuda.Stream()
    with torch.cuda.stream(cs):
        for _ in range(2):
            mp.plan(gcfg, topk, out=p)
    cs.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=cs, capture_error_mode="thread_local"):
        mp.plan(gcfg, topk, out=p)
    for it in range(6):
        topk.copy_(rs[it % 3].topk_idx.to(DEV))
        torch.cuda.synchronize()
        graph.replay()
        torch.cuda.synchronize()
        _assert_plan_equal(p, ops[it % 3])
    del graph


def test_host_errors(mp):
    with pytest.raises(mp.MoonepError):
        mp.plan(mp.Config(R=3, E=16, K=2, S=8, H=8, B=2), torch.zeros(24, 2, dtype=torch.int32, device=DEV))
    with pytest.raises(ValueError):
        mp.plan(mp.Config(R=4, E=16, K=2, S=8, H=8, B=2), torch.zeros(32, 3, dtype=torch.int32, device=DEV))
    cfg = mp.Config(R=4, E=16, K=2, S=8, H=8, B=2)
    p = mp.plan(cfg, torch.zeros(32, 2, dtype=torch.int32, device=DEV))
    h = torch.zeros(32 * 8 + 1, dtype=torch.bfloat16, device=DEV)[1:].view(32, 8)  # misaligned
    with pytest.raises(mp.MoonepError):
        mp.dispatch(cfg, p, h)
    big = mp.Config(R=4, E=64, K=17, S=8, H=8, B=2)
    pb = mp.plan(big, torch.zeros(32, 17, dtype=torch.int32, device=DEV))
    z = torch.zeros(32, 8, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(mp.MoonepError):
        mp.combine_backward(big, pb, z, torch.zeros(32, 17, device=DEV),
                            torch.zeros(4, 8 * 17, 8, dtype=torch.bfloat16, device=DEV))


# ------------------------------------------------------------- data steps

def _sub_plan(op, tokens, K):
    """Index plumbing for sampled parity: the sampled tokens' rows, renumbered
    0..n*K-1, so the oracle reads exactly the rows the GPU read."""
    dp = op["dst_pos"][tokens]                        # [n, K] original rows
    compact = np.arange(dp.size, dtype=np.int32).reshape(dp.shape)
    return {"dst_pos": compact, "info": op["info"]}, dp.ravel()


@pytest.mark.parametrize("wname,mv", [("tiny", 1.0), ("tiny", 0.0), ("mid", 0.0), ("mid", 1.0),
                                      ("mid", 3.0)])
def test_data_steps_full(mp, wname, mv):
    wl = W.WORKLOADS[wname]
    r = W.routing(wl, mv, device=DEV)
    topk = r.topk_idx.cpu().numpy()
    c = _wl_cfg(wl)
    gcfg, ocfg, gp, op = _plan_both(mp, c, topk)
    _assert_plan_equal(gp, op)
    hidden = W.hidden_states(wl, seed=1, device=DEV)
    # dispatch: every buffer row
    buf = torch.full((wl.R, wl.C, wl.H), float("nan"), dtype=torch.bfloat16, device=DEV)
    mp.dispatch(gcfg, gp, hidden, buf)
    ob = np.zeros((wl.R, wl.C, wl.H), np.uint16)
    oracle.dispatch(ocfg, op, W.bits(hidden), ob)
    assert np.array_equal(W.bits(buf), ob)
    # combine on independent expert outputs y
    y = W.bf16_normal((wl.R, wl.C, wl.H), seed=2, device=DEV)
    w = r.weights
    out = mp.combine(gcfg, gp, y, w)
    oo = oracle.combine(ocfg, op, W.bits(y), w.cpu().numpy())
    assert np.array_equal(W.bits(out), oo)
    # combine backward
    dy = W.bf16_normal((wl.tokens, wl.H), seed=3, device=DEV)
    dyb, dw = mp.combine_backward(gcfg, gp, dy, w, y)
    odyb = np.zeros_like(ob)
    odw = np.zeros((wl.tokens, wl.K), np.float32)
    oracle.combine_backward(ocfg, op, W.bits(dy), w.cpu().numpy(), W.bits(y), odyb, odw)
    assert np.array_equal(W.bits(dyb), odyb)
    dyf = dy.float().cpu().numpy().astype(np.float64)
    yf = y.float().cpu().numpy().reshape(-1, wl.H).astype(np.float64)
    mag = np.einsum("th,tkh->tk", np.abs(dyf), np.abs(yf[op["dst_pos"]]))
    assert (np.abs(dw.cpu().numpy().astype(np.float64) - odw) <= 1e-5 * mag + 1e-30).all()
    assert gp.info()["status"] == op["info"][0]  # no row-range fault raised by the data kernels


@pytest.mark.parametrize("K", [1, 3, 4, 5, 7, 12, 40])
def test_data_steps_every_k_path(mp, K):
    """The compile-time-K specialisations (1, 2, 4, 6, 8), the any-K kernels
    (3, 5, 7, 12) and K > 32 (destination rows beyond one warp's lanes), on a
    skewed routing with a ragged row (H = 136: 17 vectors, not a multiple of
    32 lanes), every element against the oracle."""
    c = dict(R=4, E=48, K=K, S=48, H=136, B=3, flags=0)
    rng = np.random.default_rng(100 + K)
    T = c["R"] * c["S"]
    bias = -1.5 * np.log(rng.permutation(np.arange(1, c["E"] + 1)))
    scores = rng.standard_normal((T, c["E"])) + bias
    topk = np.argsort(-scores, axis=1, kind="stable")[:, :K].astype(np.int32)
    gcfg, ocfg, gp, op = _plan_both(mp, c, topk)
    _assert_plan_equal(gp, op)
    check_invariants(ocfg, topk, gp.to_numpy())
    C = c["S"] * K
    wl = W.Workload("k", c["R"], c["E"], K, c["S"], c["H"], c["B"])
    hidden = W.hidden_states(wl, seed=1, device=DEV)
    buf = torch.full((c["R"], C, c["H"]), float("nan"), dtype=torch.bfloat16, device=DEV)
    mp.dispatch(gcfg, gp, hidden, buf)
    ob = np.zeros((c["R"], C, c["H"]), np.uint16)
    oracle.dispatch(ocfg, op, W.bits(hidden), ob)
    assert np.array_equal(W.bits(buf), ob)
    y = W.bf16_normal((c["R"], C, c["H"]), seed=2, device=DEV)
    w = torch.from_numpy(rng.random((T, K)).astype(np.float32)).to(DEV)
    out = mp.combine(gcfg, gp, y, w)
    assert np.array_equal(W.bits(out), oracle.combine(ocfg, op, W.bits(y), w.cpu().numpy()))
    dy = W.bf16_normal((T, c["H"]), seed=3, device=DEV)
    if K > 16:  # combine backward keeps a token's K dot products in registers
        with pytest.raises(mp.MoonepError) as ei:
            mp.combine_backward(gcfg, gp, dy, w, y)
        assert ei.value.code == 7
        return
    dyb, dw = mp.combine_backward(gcfg, gp, dy, w, y)
    odyb = np.zeros_like(ob)
    odw = np.zeros((T, K), np.float32)
    oracle.combine_backward(ocfg, op, W.bits(dy), w.cpu().numpy(), W.bits(y), odyb, odw)
    assert np.array_equal(W.bits(dyb), odyb)
    dyf = dy.float().cpu().numpy().astype(np.float64)
    yf = y.float().cpu().numpy().reshape(-1, c["H"]).astype(np.float64)
    mag = np.einsum("th,tkh->tk", np.abs(dyf), np.abs(yf[op["dst_pos"]]))
    assert (np.abs(dw.cpu().numpy().astype(np.float64) - odw) <= 1e-5 * mag + 1e-30).all()
    assert gp.info()["status"] == op["info"][0]


@pytest.mark.parametrize("wname,mv", [("large", 1.0), ("large", 3.0), ("decode", 5.0)])
def test_data_steps_full_size_sampled(mp, wname, mv):
    wl = W.WORKLOADS[wname]
    r = W.routing(wl, mv, device=DEV)
    topk = r.topk_idx.cpu().numpy()
    gcfg, ocfg, gp, op = _plan_both(mp, _wl_cfg(wl), topk)
    _assert_plan_equal(gp, op)
    rng = np.random.default_rng(0)
    tokens = np.unique(np.concatenate([rng.choice(wl.tokens, 192, replace=False),
                                       [0, wl.S - 1, wl.tokens - 1]]))
    n = len(tokens)
    sub, rows = _sub_plan(op, tokens, wl.K)
    scfg = oracle.Config(R=1, E=wl.E, K=wl.K, S=n, H=wl.H, B=0)
    hidden = W.hidden_states(wl, seed=1, device=DEV)
    buf = torch.empty((wl.R, wl.C, wl.H), dtype=torch.bfloat16, device=DEV)
    mp.dispatch(gcfg, gp, hidden, buf)
    # dispatch: the sampled tokens' K rows, and every row owner check via row_src
    hb = W.bits(hidden[torch.from_numpy(tokens).to(DEV)])
    ob = np.zeros((n * wl.K, wl.H), np.uint16)
    oracle.dispatch(scfg, sub, hb, ob)
    got = W.bits(buf.view(-1, wl.H)[torch.from_numpy(rows.astype(np.int64)).to(DEV)])
    assert np.array_equal(got, ob)
    # every buffer row holds the token that row_src says it holds
    rs = torch.from_numpy(op["row_src"].astype(np.int64)).to(DEV)
    sample_rows = torch.from_numpy(rng.choice(wl.pairs, 4096, replace=False)).to(DEV)
    assert torch.equal(buf.view(-1, wl.H)[sample_rows], hidden[rs[sample_rows] // wl.K])
    # combine and backward on independent y / dy, sampled tokens
    del buf
    y = W.bf16_normal((wl.R, wl.C, wl.H), seed=2, device=DEV)  # independent expert outputs
    w = r.weights
    out = mp.combine(gcfg, gp, y, w)
    tt = torch.from_numpy(tokens).to(DEV)
    yrows = W.bits(y.view(-1, wl.H)[torch.from_numpy(rows.astype(np.int64)).to(DEV)])
    ws = w[tt].cpu().numpy()
    oo = oracle.combine(scfg, sub, yrows, ws)
    assert np.array_equal(W.bits(out[tt]), oo)
    dy = W.bf16_normal((wl.tokens, wl.H), seed=3, device=DEV)
    dyb, dw = mp.combine_backward(gcfg, gp, dy, w, y)
    odyb = np.zeros((n * wl.K, wl.H), np.uint16)
    odw = np.zeros((n, wl.K), np.float32)
    oracle.combine_backward(scfg, sub, W.bits(dy[tt]), ws, yrows, odyb, odw)
    assert np.array_equal(W.bits(dyb.view(-1, wl.H)[torch.from_numpy(rows.astype(np.int64)).to(DEV)]), odyb)
    dyf = dy[tt].float().cpu().numpy().astype(np.float64)
    yf = y.view(-1, wl.H)[torch.from_numpy(rows.astype(np.int64)).to(DEV)].float().cpu().numpy()
    mag = np.einsum("th,tkh->tk", np.abs(dyf), np.abs(yf.astype(np.float64).reshape(n, wl.K, wl.H)))
    assert (np.abs(dw[tt].cpu().numpy().astype(np.float64) - odw) <= 1e-5 * mag + 1e-30).all()


# ---------------------------------------------------------------- reduce

@pytest.mark.parametrize("wname,mv,P", [("tiny", 1.0, 1000), ("tiny", 1.0, 1003), ("mid", 3.0, 4096),
                                        ("large", 3.0, 2048), ("decode", 13.4, 517)])
def test_reduce_full(mp, wname, mv, P):
    wl = W.WORKLOADS[wname]
    r = W.routing(wl, mv, device=DEV)
    topk = r.topk_idx.cpu().numpy()
    gcfg, ocfg, gp, op = _plan_both(mp, _wl_cfg(wl), topk)
    rb = W.f32_normal((wl.R, wl.B, P), seed=4, device=DEV, std=1e-3)
    hg = W.f32_normal((wl.E, P), seed=5, device=DEV, std=1e-3)
    orb, ohg = rb.cpu().numpy(), hg.cpu().numpy()
    mp.reduce_replica_grads(gcfg, gp, rb, hg)
    oracle.reduce_replica_grads(ocfg, op, orb, ohg, P)
    assert np.array_equal(hg.cpu().numpy(), ohg)
    assert np.array_equal(rb.cpu().numpy(), orb)
    assert gp.info()["n_rep_experts"] == op["info"][6]


def test_reduce_full_size_sampled(mp):
    # the large training shape's real gradient size (gate + up + down,
    # 3 * 7168 * 2048 fp32 per expert), compared on sampled element ranges
    wl = W.WORKLOADS["large"]
    P = wl.grad_elems
    need = 4 * P * (wl.R * wl.B + wl.E) * 1.1
    torch.cuda.empty_cache()
    free, _ = torch.cuda.mem_get_info()
    if need > free:
        pytest.skip(f"needs {need / 1e9:.0f} GB of device memory, {free / 1e9:.0f} GB free")
    r = W.routing(wl, 1.0, device=DEV)
    topk = r.topk_idx.cpu().numpy()
    gcfg, ocfg, gp, op = _plan_both(mp, _wl_cfg(wl), topk)
    rb = W.f32_normal((wl.R, wl.B, P), seed=4, device=DEV, std=1e-3)
    hg = W.f32_normal((wl.E, P), seed=5, device=DEV, std=1e-3)
    ranges = [(0, 4096), (P // 2 - 1000, P // 2 + 3001), (P - 5003, P)]
    before = [(rb[:, :, a:b].cpu().numpy().copy(), hg[:, a:b].cpu().numpy().copy()) for a, b in ranges]
    mp.reduce_replica_grads(gcfg, gp, rb, hg)
    for (a, b), (orb, ohg) in zip(ranges, before):
        orb = np.ascontiguousarray(orb)
        ohg = np.ascontiguousarray(ohg)
        oracle.reduce_replica_grads(ocfg, op, orb, ohg, b - a)
        assert np.array_equal(hg[:, a:b].cpu().numpy(), ohg)
        assert np.array_equal(rb[:, :, a:b].cpu().numpy(), orb)
    del rb, hg
    torch.cuda.empty_cache()


# -------------------------------------------------------------- prefetch

@pytest.mark.parametrize("wname,mv,P", [("tiny", 1.0, 1000), ("tiny", 3.0, 1003), ("mid", 3.0, 4096),
                                        ("large", 3.0, 2048), ("decode", 13.4, 517)])
def test_prefetch(mp, wname, mv, P):
    wl = W.WORKLOADS[wname]
    r = W.routing(wl, mv, device=DEV)
    topk = r.topk_idx.cpu().numpy()
    gcfg, ocfg, gp, op = _plan_both(mp, _wl_cfg(wl), topk)
    weights = W.bf16_normal((wl.E, P), seed=6, device=DEV)
    pool = torch.full((wl.R, wl.B, P), float("nan"), dtype=torch.bfloat16, device=DEV)
    opool = W.bits(pool).copy()
    wrow = mp.prefetch_replicas(gcfg, gp, weights, pool)
    owrow = oracle.prefetch_replicas(ocfg, op, W.bits(weights), opool, P)
    assert np.array_equal(wrow.cpu().numpy(), owrow)
    assert np.array_equal(W.bits(pool), opool)


def test_prefetch_bad_ids_and_no_budget(mp):
    c = dict(R=4, E=16, K=2, S=64, H=64, B=2)
    rng = np.random.default_rng(2)
    topk = rng.integers(0, 16, size=(256, 2)).astype(np.int32)
    topk[5, 0] = -3
    gcfg, ocfg, gp, op = _plan_both(mp, c, topk)
    weights = W.bf16_normal((16, 64), seed=6, device=DEV)
    pool = torch.full((4, 2, 64), 3.0, dtype=torch.bfloat16, device=DEV)
    wrow = mp.prefetch_replicas(gcfg, gp, weights, pool)
    assert (wrow.cpu() == -1).all() and (pool == 3.0).all()
    # B = 0: every replica is overflow and reads its home row
    c0 = dict(R=4, E=16, K=2, S=64, H=64, B=0)
    topk[5, 0] = 1
    gcfg, ocfg, gp, op = _plan_both(mp, c0, topk)
    wrow = mp.prefetch_replicas(gcfg, gp, weights, torch.empty((4, 0, 64), dtype=torch.bfloat16, device=DEV))
    owrow = oracle.prefetch_replicas(ocfg, op, W.bits(weights), np.zeros((4, 0, 64), np.uint16), 64)
    assert np.array_equal(wrow.cpu().numpy(), owrow)


def test_workspace_not_zeroed_is_detected(mp):
    # The workspace must start zero-filled; if its expert totals hold
    # garbage, the planner reports MOONEP_ST_WORKSPACE and an empty plan
    # (white-box: the totals follow the 256-byte header of the workspace).
    wl = W.WORKLOADS["tiny"]
    c = _wl_cfg(wl)
    cfg = mp.Config(**c)
    topk = W.routing(wl, 1.0, device=DEV).topk_idx
    p = mp.Plan(cfg)
    torch.cuda.synchronize()
    p.workspace[256:256 + 4 * wl.E] = 0x7F
    torch.cuda.synchronize()
    mp.plan(cfg, topk, out=p)
    info = p.info()
    assert info["status"] & mp.ST_WORKSPACE
    f = p.to_numpy()
    assert (f["dst_pos"] == -1).all() and (f["slot_count"] == 0).all() and info["n_rep"] == 0
    # dispatch is a no-op on an empty plan
    hidden = W.hidden_states(wl, seed=1, device=DEV)
    buf = torch.full((wl.R, wl.C, wl.H), 2.0, dtype=torch.bfloat16, device=DEV)
    mp.dispatch(cfg, p, hidden, buf)
    torch.cuda.synchronize()
    assert (buf == 2.0).all()
    # zero-filled again, the same workspace plans exactly as the oracle
    p.workspace.zero_()
    mp.plan(cfg, topk, out=p)
    _assert_plan_equal(p, oracle.plan(oracle.Config(**c), topk.cpu().numpy()))


@pytest.mark.parametrize("mv", [0.2, 1.0, 10.0, 20.0])
def test_pages_sweep_shape_plan_and_sampled_data(mp, mv):
    # the pages' EP=8 sweep shape (256 experts, top-8) up to maxvio 20
    wl = W.WORKLOADS["ep8"]
    r = W.routing(wl, mv, device=DEV)
    topk = r.topk_idx.cpu().numpy()
    gcfg, ocfg, gp, op = _plan_both(mp, _wl_cfg(wl), topk)
    _assert_plan_equal(gp, op)
    check_invariants(ocfg, topk, gp.to_numpy())
    # every rank still receives exactly S*K rows however hot the hottest expert
    assert (gp.slot_count.sum(dim=1).cpu() == wl.C).all()
    hidden = W.hidden_states(wl, seed=1, device=DEV)
    buf = mp.dispatch(gcfg, gp, hidden)
    out = mp.combine(gcfg, gp, buf, r.weights)
    rng = np.random.default_rng(4)
    tokens = np.unique(np.concatenate([rng.choice(wl.tokens, 64, replace=False), [0, wl.tokens - 1]]))
    sub, rows = _sub_plan(op, tokens, wl.K)
    n = len(tokens)
    scfg = oracle.Config(R=1, E=wl.E, K=wl.K, S=n, H=wl.H, B=0)
    tt = torch.from_numpy(tokens).to(DEV)
    ob = np.zeros((n * wl.K, wl.H), np.uint16)
    oracle.dispatch(scfg, sub, W.bits(hidden[tt]), ob)
    got = W.bits(buf.view(-1, wl.H)[torch.from_numpy(rows.astype(np.int64)).to(DEV)])
    assert np.array_equal(got, ob)
    oo = oracle.combine(scfg, sub, ob, r.weights[tt].cpu().numpy())
    assert np.array_equal(W.bits(out[tt]), oo)


def test_views_slices_match_slot_tables(mp):
    wl = W.WORKLOADS["tiny"]
    c = _wl_cfg(wl)
    r = W.routing(wl, 1.0, device=DEV)
    gcfg = mp.Config(**c)
    gp = mp.plan(gcfg, r.topk_idx)
    buf = mp.dispatch(gcfg, gp, W.hidden_states(wl, seed=1, device=DEV))
    v = mp.views(gcfg, gp, buf)
    se = gp.slot_expert.cpu().numpy()
    sc = gp.slot_count.cpu().numpy()
    rs = gp.row_src.cpu().numpy()
    topk = r.topk_idx.cpu().numpy().ravel()
    for rank, slots in enumerate(v):
        assert sum(x.shape[0] for _, x in slots) == wl.C
        row = rank * wl.C
        for s, (e, x) in enumerate(slots):
            assert e == se[rank, s] and x.shape[0] == sc[rank, s]
            # each row of the view holds a token routed to the slot's expert
            assert (topk[rs[row:row + x.shape[0]]] == e).all()
            row += x.shape[0]
