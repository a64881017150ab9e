"""The two planners of moonep_plan.

moonep_plan launches one kernel when every CTA of its grid fits on the GPU
at once (every CTA then computes the whole plan in its own shared memory),
and two kernels otherwise (a histogram pass whose last CTA plans, then an
assignment pass); moonep_set_plan_path(1) keeps it on the two.  The parity
and failure-path modules run every test under both; this one checks which
kernels a call launches, that one workspace may pass between the two from
call to call, and that a shape too large for the one kernel takes the two
without being asked.
"""
import numpy as np
import pytest
import torch
from torch.profiler import ProfilerActivity, profile

import oracle
from load_balancing_moonep_b200 import workloads as W

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module")
def mp(oracle_lib, cuda_lib_path):
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    from load_balancing_moonep_b200 import moonep
    return moonep


def _kernels(fn):
    """Names of the CUDA kernels fn launches (profiler trace)."""
    torch.cuda.synchronize()
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        fn()
        torch.cuda.synchronize()
    return [e.name for e in prof.events() if e.device_type == torch.autograd.DeviceType.CUDA]


def _cfg(mp, wl, flags=0):
    c = dict(R=wl.R, E=wl.E, K=wl.K, S=wl.S, H=wl.H, B=wl.B, flags=flags)
    return mp.Config(**c), oracle.Config(**c)


def _assert_equal(gp, op, label):
    g = gp.to_numpy()
    for k, v in op.items():
        assert np.array_equal(g[k], v), f"{label}: plan field {k} differs"


@pytest.mark.parametrize("wname", ["tiny", "decode", "large"])
def test_a_call_launches_the_chosen_planner(mp, wname):
    wl = W.WORKLOADS[wname]
    gcfg, _ = _cfg(mp, wl)
    topk = W.routing(wl, 1.0, device=DEV).topk_idx
    p = mp.Plan(gcfg)
    prev = mp.set_plan_path(0)
    try:
        one = _kernels(lambda: mp.plan(gcfg, topk, out=p))
        mp.set_plan_path(1)
        two = _kernels(lambda: mp.plan(gcfg, topk, out=p))
    finally:
        mp.set_plan_path(prev)
    assert any("plan_fused_kernel" in k for k in one), one
    assert not any("hist_plan_kernel" in k or "assign_kernel" in k for k in one), one
    assert any("hist_plan_kernel" in k for k in two) and any("assign_kernel" in k for k in two), two
    assert not any("plan_fused_kernel" in k for k in two), two


def test_one_workspace_alternates_between_the_planners(mp):
    # the two leave the workspace header in the same state after a call, so
    # a workspace may switch path from one call to the next
    wl = W.WORKLOADS["mid"]
    gcfg, ocfg = _cfg(mp, wl)
    routings = [W.routing(wl, mv, seed=s, device=DEV).topk_idx for s, mv in ((0, 0.5), (1, 3.0))]
    expect = [oracle.plan(ocfg, t.cpu().numpy()) for t in routings]
    p = mp.Plan(gcfg)
    prev = mp.set_plan_path(0)
    try:
        for call in range(8):
            mp.set_plan_path((call // 2) % 2)
            i = call % 2
            mp.plan(gcfg, routings[i], out=p)
            torch.cuda.synchronize()
            _assert_equal(p, expect[i], f"call {call} (path {(call // 2) % 2})")
    finally:
        mp.set_plan_path(prev)


def test_a_shape_too_large_for_one_kernel_takes_two(mp):
    # E = R = 1024 with the relay cascade: the planner's shared memory does
    # not fit two CTAs per SM beside the pass's, so the two kernels run
    c = dict(R=1024, E=1024, K=1, S=4, H=8, B=1, flags=8)
    gcfg, ocfg = mp.Config(**c), oracle.Config(**c)
    rng = np.random.default_rng(3)
    topk = rng.integers(0, 1024, size=(1024 * 4, 1)).astype(np.int32)
    t = torch.from_numpy(topk).to(DEV)
    holder = {}
    names = _kernels(lambda: holder.setdefault("p", mp.plan(gcfg, t)))
    assert any("hist_plan_kernel" in k for k in names), names
    assert not any("plan_fused_kernel" in k for k in names), names
    _assert_equal(holder["p"], oracle.plan(ocfg, topk), "E = R = 1024")


@pytest.mark.parametrize("wname,shift", [("mid", 1), ("mid", 3), ("large", 2)])
def test_ids_not_16_byte_aligned(mp, wname, shift):
    # the one-kernel planner reads the ids in 16-byte words when topk_idx is
    # 16-byte aligned, one by one otherwise: a view starting `shift` ints
    # into a buffer takes the second way, and the plan is the same
    wl = W.WORKLOADS[wname]
    gcfg, ocfg = _cfg(mp, wl)
    topk = W.routing(wl, 2.0, device=DEV).topk_idx
    buf = torch.empty(topk.numel() + 4, dtype=torch.int32, device=DEV)
    view = buf[shift:shift + topk.numel()].view(topk.shape)
    view.copy_(topk)
    assert view.data_ptr() % 16 != 0
    gp = mp.plan(gcfg, view)
    torch.cuda.synchronize()
    _assert_equal(gp, oracle.plan(ocfg, topk.cpu().numpy()), f"{wname} shift {shift}")


def test_expert_parallel_plan_launches_the_chosen_planner(mp):
    # moonep_ep_plan: one kernel by default (every CTA plans from the
    # gathered counts), the planner CTA then the assignment grid with path 1
    R, E, K, S = 8, 64, 4, 512
    cfg = mp.Config(R=R, E=E, K=K, S=S, H=64, B=4)
    gen = torch.Generator(device="cpu").manual_seed(7)
    topk = torch.stack([torch.randperm(E, generator=gen)[:K] for _ in range(R * S)]).to(torch.int32).to(DEV)
    plans = [mp.Plan(cfg, DEV, ep=True) for _ in range(R)]
    counts = torch.zeros((R, E + 1), dtype=torch.int32, device=DEV)
    torch.cuda.synchronize()
    for r in range(R):
        mp.ep_count(cfg, topk[r * S:(r + 1) * S].contiguous(), plans[r], counts_row=counts[r])
    prev = mp.set_plan_path(0)
    try:
        one = _kernels(lambda: mp.ep_plan(cfg, 0, topk[:S].contiguous(), counts, plans[0]))
        mp.set_plan_path(1)
        two = _kernels(lambda: mp.ep_plan(cfg, 0, topk[:S].contiguous(), counts, plans[0]))
    finally:
        mp.set_plan_path(prev)
    assert any("ep_fused_kernel" in k for k in one) and not any("ep_plan_kernel" in k for k in one), one
    assert any("ep_plan_kernel" in k for k in two) and any("ep_assign_kernel" in k for k in two), two


@pytest.mark.parametrize("path", [0, 1])
def test_plan_is_exact_while_other_streams_hold_sms(mp, path):
    # Sleeping one-block kernels on 140 other streams hold SMs (the one-kernel
    # planner's CTAs each need a whole SM) for about 20 ms while the plan
    # runs with a short wait bound: CTAs that cannot all be resident take the
    # fallback (the one kernel counts every pair itself, the two-kernel pass
    # waits for the histogram grid), and the plan must still be the oracle's
    # (MOONEP_ST_WAIT_TIMEOUT may be set, nothing else may differ; on a B200
    # the one-kernel planner's CTAs did time out in this setting).  Every wait
    # in the library is bounded, and nothing here waits on the plan.
    wl = W.WORKLOADS["large"]
    gcfg, ocfg = _cfg(mp, wl)
    topk = W.routing(wl, 1.0, device=DEV).topk_idx
    op = oracle.plan(ocfg, topk.cpu().numpy())
    p = mp.Plan(gcfg)
    streams = [torch.cuda.Stream() for _ in range(140)]
    torch.cuda.synchronize()
    prev_limit = mp.set_wait_limit(2000)
    prev_path = mp.set_plan_path(path)
    try:
        for s in streams:
            with torch.cuda.stream(s):
                torch.cuda._sleep(40_000_000)  # about 20 ms at 2 GHz
        mp.plan(gcfg, topk, out=p)
        torch.cuda.synchronize()
    finally:
        mp.set_wait_limit(prev_limit)
        mp.set_plan_path(prev_path)
    g = p.to_numpy()
    for k, v in op.items():
        if k == "info":
            assert g[k][0] & ~mp.ST_WAIT_TIMEOUT == v[0]
            assert np.array_equal(g[k][1:], v[1:])
        else:
            assert np.array_equal(g[k], v), f"plan field {k} differs"
    # and the next plan, with the SMs free again, is exact without the bit
    mp.set_plan_path(path)
    try:
        mp.plan(gcfg, topk, out=p)
        torch.cuda.synchronize()
    finally:
        mp.set_plan_path(prev_path)
    assert p.info()["status"] == op["info"][0]
