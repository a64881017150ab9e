"""The no-allocation planner entry point (moonep_plan_noalloc).

Some callers cannot give the planner a workspace: code inside a runtime that
owns every device allocation, or a hot path that must not call cudaMalloc.
For them the library keeps a fixed device array as scratch space.  This test
calls that entry point through the C ABI twice in a row -- with different
configurations, so the second call finds the first call's leftovers in the
shared array -- and checks each plan against the ordinary, workspace-based
moonep_plan, field by field and bit for bit (the plan's tolerance).  It also
checks that a configuration whose workspace does not fit is refused before
anything is launched.  The file sorts last so a stop-at-first-failure run has
already run every other test when it gets here.
"""
import ctypes

import numpy as np
import pytest
import torch

from load_balancing_moonep_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mp(cuda_lib_path):
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    from load_balancing_moonep_b200 import moonep
    return moonep


def _reference(mp, cfg, topk):
    return mp.plan(cfg, topk).to_numpy()


def _noalloc_via_cabi(mp, cfg, topk):
    out = mp.Plan(cfg)
    c = cfg.c()
    rc = mp._lib.moonep_plan_noalloc(ctypes.byref(c), topk.data_ptr(), ctypes.byref(out.c_plan),
                                     torch.cuda.current_stream().cuda_stream)
    assert rc == 0, mp._lib.moonep_error_string(rc)
    torch.cuda.synchronize()
    return out.to_numpy()


def test_noalloc_matches_workspace_planner_twice(mp):
    cases = [("large", 3.0), ("mid", 1.0)]   # different layouts of the shared array
    for name, mv in cases:
        wl = W.WORKLOADS[name]
        cfg = mp.Config(R=wl.R, E=wl.E, K=wl.K, S=wl.S, H=wl.H, B=wl.B)
        topk = W.routing(wl, mv, device="cuda").topk_idx
        got = _noalloc_via_cabi(mp, cfg, topk)
        ref = _reference(mp, cfg, topk)
        for k in ref:
            assert np.array_equal(got[k], ref[k]), f"{name}: plan field {k} differs"
        assert got["info"][0] & mp.ST_ROW_RANGE == 0


def test_noalloc_same_config_back_to_back(mp):
    wl = W.WORKLOADS["tiny"]
    cfg = mp.Config(R=wl.R, E=wl.E, K=wl.K, S=wl.S, H=wl.H, B=wl.B)
    for mv in (1.0, 3.0):
        topk = W.routing(wl, mv, device="cuda").topk_idx
        got = _noalloc_via_cabi(mp, cfg, topk)
        ref = _reference(mp, cfg, topk)
        for k in ref:
            assert np.array_equal(got[k], ref[k]), f"plan field {k} differs"


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
