"""The library's two defensive paths, driven on the GPU in forms that cannot
fault it.

* The assignment pass waits for two marks of the histogram/planner pass with
  a bounded spin; when a bound runs out it waits for the whole histogram
  grid instead (a grid that never depends on it) and reports
  MOONEP_ST_WAIT_TIMEOUT.  moonep_set_wait_limit(0) makes both bounds run
  out at once: the plan must still equal the oracle's, with only that bit
  added to the status.
* The data kernels range-check every buffer row they take from the plan
  before any access.  Here a copy of a valid plan gets out-of-range rows
  written into dst_pos on the host side of the test; dispatch, combine and
  combine backward must skip exactly those rows, set MOONEP_ST_ROW_RANGE and
  leave every other row as the oracle has it.
"""
import numpy as np
import pytest
import torch

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


@pytest.fixture(autouse=True, params=["one-kernel", "two-kernel"])
def plan_path(request, mp):
    """Every test runs under both planners (moonep_set_plan_path): the one
    kernel wherever its CTAs all fit on the GPU, and the two-kernel path."""
    prev = mp.set_plan_path(1 if request.param == "two-kernel" else 0)
    yield request.param
    mp.set_plan_path(prev)


def _cfg(mp, wl, flags=0):
    c = dict(R=wl.R, E=wl.E, K=wl.K, S=wl.S, H=wl.H, B=wl.B, flags=flags)
    return mp.Config(**c), oracle.Config(**c)


# ------------------------------------------------------------ WAIT_TIMEOUT

@pytest.mark.parametrize("wname,mv,flags", [("tiny", 1.0, 0), ("mid", 3.0, 0), ("large", 1.0, 0),
                                            ("decode", 5.0, 0), ("large", -1.0, 8)])
def test_wait_fallback_gives_the_exact_plan(mp, wname, mv, flags):
    wl = W.WORKLOADS[wname]
    gcfg, ocfg = _cfg(mp, wl, flags)
    if mv < 0:  # one empty rank: the relay cascade's slow path runs
        topk = W.over_budget_routing(wl, seed=0, device=DEV).topk_idx
    else:
        topk = W.routing(wl, mv, device=DEV).topk_idx
    op = oracle.plan(ocfg, topk.cpu().numpy())
    hidden = W.hidden_states(wl, seed=1, device=DEV)
    prev = mp.set_wait_limit(0)
    try:
        gp = mp.plan(gcfg, topk)
        buf = mp.dispatch(gcfg, gp, hidden)
        torch.cuda.synchronize()
    finally:
        mp.set_wait_limit(prev)
    g = gp.to_numpy()
    for k, v in op.items():
        if k == "info":
            assert g[k][0] == v[0] | mp.ST_WAIT_TIMEOUT
            assert np.array_equal(g[k][1:], v[1:])
        else:
            assert np.array_equal(g[k], v), f"plan field {k} differs"
    # the data kernels treat the plan as valid
    rows = np.random.default_rng(0).integers(0, wl.pairs, 256)
    src = g["row_src"][rows]
    assert np.array_equal(W.bits(buf.view(-1, wl.H)[torch.from_numpy(rows).to(DEV)]),
                          W.bits(hidden[torch.from_numpy(src // wl.K).to(DEV)]))
    # the default bound is back: the next plan waits for the marks again
    gp2 = mp.plan(gcfg, topk)
    torch.cuda.synchronize()
    assert gp2.info()["status"] == op["info"][0]


# --------------------------------------------------------------- ROW_RANGE

def _combine_without(ocfg, wl, y_bits, w, rows, keep):
    """The oracle's combine of one token over its kept pairs only: the same
    fp32 fused multiply-add chain in k order with the skipped terms left out."""
    n = len(keep)
    scfg = oracle.Config(R=1, E=wl.E, K=n, S=1, H=wl.H, B=0)
    sub = {"dst_pos": np.arange(n, dtype=np.int32).reshape(1, n),
           "info": np.zeros(16, np.int32)}
    yy = np.ascontiguousarray(y_bits.reshape(-1, wl.H)[rows[keep]]).reshape(1, n, wl.H)
    return oracle.combine(scfg, sub, yy, np.ascontiguousarray(w[keep].reshape(1, n)))[0]


@pytest.mark.parametrize("wname", ["tiny", "mid"])
def test_out_of_range_rows_are_skipped_and_reported(mp, wname):
    wl = W.WORKLOADS[wname]
    gcfg, ocfg = _cfg(mp, wl)
    r = W.routing(wl, 1.0, device=DEV)
    topk = r.topk_idx
    op = oracle.plan(ocfg, topk.cpu().numpy())
    gp = mp.plan(gcfg, topk)
    torch.cuda.synchronize()
    status0 = int(op["info"][0])
    assert gp.info()["status"] == status0
    # three pairs get rows outside [0, R*S*K): one past the end, -1 and
    # INT32_MAX; they are written into the device plan's dst_pos
    NP = wl.pairs
    bad = [(3, 0, NP), (wl.tokens // 2, wl.K - 1, -1), (wl.tokens - 1, 1 % wl.K, 2**31 - 1)]
    for t, k, v in bad:
        gp.dst_pos[t, k] = v
    torch.cuda.synchronize()
    skipped_rows = [int(op["dst_pos"][t, k]) for t, k, _ in bad]

    hidden = W.hidden_states(wl, seed=1, device=DEV)
    sentinel = torch.full((wl.R, wl.C, wl.H), float("nan"), dtype=torch.bfloat16, device=DEV)
    sbits = W.bits(sentinel[0, 0, :1])[0]

    # dispatch: every row as the oracle has it, except the skipped ones
    buf = sentinel.clone()
    mp.dispatch(gcfg, gp, hidden, buf)
    torch.cuda.synchronize()
    assert gp.info()["status"] == status0 | mp.ST_ROW_RANGE
    ob = np.zeros((wl.R, wl.C, wl.H), np.uint16)
    oracle.dispatch(ocfg, op, W.bits(hidden), ob)
    ob = ob.reshape(-1, wl.H)
    ob[skipped_rows] = sbits
    assert np.array_equal(W.bits(buf).reshape(-1, wl.H), ob)

    # combine: tokens with a bad row sum over their other pairs only
    y = W.bf16_normal((wl.R, wl.C, wl.H), seed=2, device=DEV)
    w = r.weights.cpu().numpy()
    out = W.bits(mp.combine(gcfg, gp, y, r.weights))
    yb = W.bits(y)
    oo = oracle.combine(ocfg, op, yb, w)
    for t, k, _ in bad:
        keep = np.array([j for j in range(wl.K) if j != k])
        oo[t] = _combine_without(ocfg, wl, yb, w[t], op["dst_pos"][t], keep)
    assert np.array_equal(out, oo)

    # combine backward: the skipped rows of dy_buf keep their old contents
    # and the skipped pairs' dw is 0
    dy = W.bf16_normal((wl.tokens, wl.H), seed=3, device=DEV)
    dyb = sentinel.clone()
    dwt = torch.full((wl.tokens, wl.K), 7.0, dtype=torch.float32, device=DEV)
    mp.combine_backward(gcfg, gp, dy, r.weights, y, dyb, dwt)
    torch.cuda.synchronize()
    odyb = np.zeros((wl.R, wl.C, wl.H), np.uint16)
    odw = np.zeros((wl.tokens, wl.K), np.float32)
    oracle.combine_backward(ocfg, op, W.bits(dy), w, yb, odyb, odw)
    odyb = odyb.reshape(-1, wl.H)
    odyb[skipped_rows] = sbits
    assert np.array_equal(W.bits(dyb).reshape(-1, wl.H), odyb)
    dw = dwt.cpu().numpy()
    dyf = dy.float().cpu().numpy().astype(np.float64)
    yf = y.float().cpu().numpy().reshape(-1, wl.H).astype(np.float64)
    mag = np.einsum("th,tkh->tk", np.abs(dyf), np.abs(yf[op["dst_pos"]]))
    ok = np.abs(dw.astype(np.float64) - odw) <= 1e-5 * mag + 1e-30
    for t, k, _ in bad:
        assert dw[t, k] == 0.0
        ok[t, k] = True
    assert ok.all()
    assert gp.info()["status"] == status0 | mp.ST_ROW_RANGE
