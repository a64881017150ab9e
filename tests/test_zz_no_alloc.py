"""The no-allocation planner entry point (moonep_plan_noalloc).

Some callers cannot give the planner a workspace: code inside a runtime that
owns every device allocation, or a hot path that must not call cudaMalloc.
For them the library keeps a fixed device array as scratch space.  These
tests call that entry point through the C ABI several times in a row -- with
different configurations, and after a call that leaves non-zero counts
behind, so later calls find earlier calls' leftovers in the shared array --
and check every plan field by field, bit for bit (the plan's tolerance),
against the CPU oracle and against the ordinary, workspace-based
moonep_plan.  A configuration whose workspace does not fit is refused before
anything is launched.  The file sorts last so a stop-at-first-failure run
has already run every other test when it gets here.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from load_balancing_moonep_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mp(cuda_lib_path):
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    from load_balancing_moonep_b200 import moonep
    return moonep


def _noalloc_via_cabi(mp, cfg, topk):
    out = mp.Plan(cfg)
    torch.cuda.synchronize()  # the plan block is zero-filled on the default stream
    c = cfg.c()
    rc = mp._lib.moonep_plan_noalloc(ctypes.byref(c), topk.data_ptr(), ctypes.byref(out.c_plan),
                                     torch.cuda.current_stream().cuda_stream)
    assert rc == 0, mp._lib.moonep_error_string(rc)
    torch.cuda.synchronize()
    return out.to_numpy()


def _check_against_oracle_and_planner(mp, cfg, topk, label):
    got = _noalloc_via_cabi(mp, cfg, topk)
    ocfg = oracle.Config(R=cfg.R, E=cfg.E, K=cfg.K, S=cfg.S, H=cfg.H, B=cfg.B, flags=cfg.flags)
    ref = oracle.plan(ocfg, topk.cpu().numpy())
    for k, v in ref.items():
        assert np.array_equal(got[k], v), f"{label}: plan field {k} differs from the oracle"
    ws = mp.plan(cfg, topk).to_numpy()
    for k in ws:
        assert np.array_equal(got[k], ws[k]), f"{label}: plan field {k} differs from moonep_plan"
    assert got["info"][0] & (mp.ST_WORKSPACE | mp.ST_ROW_RANGE | mp.ST_WAIT_TIMEOUT) == 0, label
    return got


def test_noalloc_matches_oracle_twice_across_layouts(mp):
    # different layouts of the shared array, one after the other
    for name, mv in [("large", 3.0), ("mid", 1.0)]:
        wl = W.WORKLOADS[name]
        cfg = mp.Config(R=wl.R, E=wl.E, K=wl.K, S=wl.S, H=wl.H, B=wl.B)
        topk = W.routing(wl, mv, device="cuda").topk_idx
        _check_against_oracle_and_planner(mp, cfg, topk, name)


def test_noalloc_after_a_call_that_leaves_counts_behind(mp):
    # a call with one expert id out of range plans nothing but leaves the
    # large layout's group counts (non-zero) and an advanced sequence number
    # in the array; the next calls, of other layouts and of the same one,
    # must still plan exactly
    wl = W.WORKLOADS["large"]
    cfg = mp.Config(R=wl.R, E=wl.E, K=wl.K, S=wl.S, H=wl.H, B=wl.B)
    bad = W.routing(wl, 1.0, device="cuda").topk_idx.clone()
    bad[wl.tokens // 2, 0] = wl.E
    got = _noalloc_via_cabi(mp, cfg, bad)
    assert got["info"][0] & mp.ST_EXPERT_ID_RANGE
    assert (got["dst_pos"] == -1).all()
    for name, mv in [("mid", 2.0), ("tiny", 1.0), ("large", 1.0), ("large", 0.0)]:
        w2 = W.WORKLOADS[name]
        c2 = mp.Config(R=w2.R, E=w2.E, K=w2.K, S=w2.S, H=w2.H, B=w2.B)
        topk = W.routing(w2, mv, device="cuda").topk_idx
        _check_against_oracle_and_planner(mp, c2, topk, f"{name} after leftovers")


def test_noalloc_same_config_back_to_back(mp):
    wl = W.WORKLOADS["tiny"]
    cfg = mp.Config(R=wl.R, E=wl.E, K=wl.K, S=wl.S, H=wl.H, B=wl.B)
    for mv in (1.0, 3.0):
        topk = W.routing(wl, mv, device="cuda").topk_idx
        _check_against_oracle_and_planner(mp, cfg, topk, f"tiny maxvio {mv}")


def test_noalloc_rejects_oversize(mp):
    # 1024 experts, 4096 tokens per rank on 256 ranks: a workspace far above 4 MiB
    cfg = mp.Config(R=256, E=1024, K=8, S=4096, H=8, B=4)
    _, ws = mp.plan_sizes(cfg)
    assert ws > mp.NOALLOC_WORKSPACE_BYTES
    c = cfg.c()
    cp = mp._CPlan()
    rc = mp._lib.moonep_plan_noalloc(ctypes.byref(c), 1 << 20, ctypes.byref(cp), None)
    assert rc == 9
    assert "no-allocation" in mp._lib.moonep_error_string(rc).decode()
