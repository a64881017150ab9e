"""Properties every plan must satisfy, checked from first principles.

These hold for any output of the planner (oracle or CUDA) and do not reuse
the planner's arithmetic: they re-derive loads, deficits and orders with
numpy and compare.  Sources: the exact S*K invariant, redundant experts
planned from the router output ("Moonshot AI Open-Sources MoonEP: A
Perfectly Balanced Expert Parallelism Library for MoE Training", "The core
idea: dynamic redundant experts"); at most B prefetched replica slots per
rank (same page, explainer memory tab).
"""
from __future__ import annotations

import numpy as np

ST_EXPERT_ID_RANGE, ST_OVERFLOW, ST_STRICT = 1, 2, 4


def check_invariants(cfg, topk, p) -> dict:
    """Assert the constraints the pages fix plus the structural properties of
    the water-filling plan (with the locality flag, of its host intervals).
    Returns a few derived quantities."""
    locality = bool(getattr(cfg, "flags", 0) & 16)
    R, E, K, S, B = cfg.R, cfg.E, cfg.K, cfg.S, cfg.B
    L, C = E // R, S * K
    topk = np.asarray(topk).reshape(R * S, K)
    T = np.bincount(topk.ravel(), minlength=E)
    assert (p["expert_count"] == T).all()
    info = p["info"]
    n_rep = int(info[1])

    # every rank receives exactly S*K slots
    sc = p["slot_count"]
    assert (sc.sum(axis=1) == C).all()
    so = p["slot_offset"]
    assert (so[:, 0] == 0).all() and (so[:, E] == C).all()
    assert (np.diff(so, axis=1) == sc).all()

    # home slots
    for r in range(R):
        assert (p["slot_expert"][r, :L] == np.arange(r * L, (r + 1) * L)).all()

    # replicas: list, slots, never on home, never two of one expert on a rank
    reps = [(int(p["rep_expert"][q]), int(p["rep_rank"][q]), int(p["rep_slot"][q]),
             int(p["rep_quota"][q])) for q in range(n_rep)]
    assert (p["rep_expert"][n_rep:] == -1).all() and (p["rep_quota"][n_rep:] == 0).all()
    seen = set()
    per_rank = np.zeros(R, np.int64)
    for (e, r, s, q) in reps:
        assert 0 <= e < E and 0 <= r < R and q > 0
        assert r != e // L, "replica on its home rank"
        assert (e, r) not in seen, "two replicas of one expert on one rank"
        seen.add((e, r))
        assert s == L + per_rank[r], "replica slots are taken in creation order"
        per_rank[r] += 1
        assert p["slot_expert"][r, s] == e and p["slot_count"][r, s] == q
    n_over = sum(1 for (e, r, s, q) in reps if s - L >= B)
    assert info[2] == n_over
    assert info[5] == (per_rank.max() if R else 0)
    for r in range(R):
        used = L + per_rank[r]
        assert (p["slot_expert"][r, used:] == -1).all()
        assert (p["slot_count"][r, used:] == 0).all()
    st = int(info[0])
    assert bool(st & ST_OVERFLOW) == (n_over > 0)

    # host intervals: home + replicas, ascending rank, quotas sum to T[e]
    hp = p["host_ptr"]
    assert hp[0] == 0 and hp[E] == E + n_rep
    for e in range(E):
        hs = range(hp[e], hp[e + 1])
        ranks = [int(p["host_rank"][h]) for h in hs]
        assert ranks == sorted(ranks) and len(set(ranks)) == len(ranks)
        assert e // L in ranks
        start, n_loc = 0, 0
        for h in hs:
            assert p["host_start"][h] == start
            r, s = int(p["host_rank"][h]), int(p["host_slot"][h])
            assert p["slot_expert"][r, s] == e
            q = int(p["host_quota"][h])
            assert q == p["slot_count"][r, s]
            loc = int(p["host_local"][h])
            if locality:  # its own rank's pairs first, as many as its quota takes
                assert loc == min(q, int((topk[r * S:(r + 1) * S] == e).sum()))
            else:
                assert loc == 0
            start += q - loc
            n_loc += loc
        assert start + n_loc == T[e]

    # pair placement: every pair on a rank hosting its expert; row_src is the
    # inverse permutation; each slot holds its expert's pairs in (t, k) order
    dst = p["dst_pos"].reshape(-1)
    rs = p["row_src"]
    assert np.array_equal(np.sort(dst), np.arange(R * C))
    assert np.array_equal(rs[dst], np.arange(R * S * K))
    d_rank = dst // C
    d_row = dst % C
    slot_of = np.empty(R * S * K, np.int64)
    for r in range(R):
        m = d_rank == r
        slot_of[m] = np.searchsorted(so[r], d_row[m], side="right") - 1
    assert (p["slot_expert"][d_rank, slot_of] == topk.ravel()).all()
    row = np.arange(R * C)
    r_rank = row // C
    r_slot = np.empty(R * C, np.int64)
    for r in range(R):
        m = r_rank == r
        r_slot[m] = np.searchsorted(so[r], row[m] % C, side="right") - 1
    same = (r_rank[1:] == r_rank[:-1]) & (r_slot[1:] == r_slot[:-1])
    src_rank = (np.arange(R * S * K) // K) // S
    if not locality:
        assert (rs[1:][same] > rs[:-1][same]).all(), "slot rows not in (t, k) order"
        # for each expert, destination ranks are non-decreasing over (t, k)
        flat = topk.ravel()
        by_e = np.argsort(flat, kind="stable")
        same_e = flat[by_e][1:] == flat[by_e][:-1]
        assert (np.diff(d_rank[by_e])[same_e] >= 0).all()
    else:
        # a slot holds its own rank's pairs first, then leftover pairs, each
        # part in (t, k) order; the local pairs are exactly those
        local_row = src_rank[rs] == r_rank
        part_same = same & (local_row[1:] == local_row[:-1])
        assert (rs[1:][part_same] > rs[:-1][part_same]).all(), "slot parts not in (t, k) order"
        starts = np.r_[True, ~same]
        # no local row after a leftover row within a slot
        seen_left = False
        for i in range(R * C):
            if starts[i]:
                seen_left = False
            if not local_row[i]:
                seen_left = True
            else:
                assert not seen_left, "a local pair after a leftover pair in a slot"
        assert int(local_row.sum()) == int(p["host_local"].sum())

    # remote-pair statistic
    assert info[7] == int((src_rank != d_rank).sum())

    # reduce work list: experts with a prefetched replica, ascending
    pref = sorted({e for (e, r, s, q) in reps if s - L < B})
    assert info[6] == len(pref)
    assert list(p["rep_home_list"][:len(pref)]) == pref
    assert (p["rep_home_list"][len(pref):] == -1).all()
    return {"T": T, "reps": reps, "n_over": n_over}


def check_water_filling(cfg, topk, p):
    """The greedy's own structure: largest-first shedding, receivers and
    pieces taken in (value desc, index asc) order, north-west-corner merge."""
    R, E, K, S = cfg.R, cfg.E, cfg.K, cfg.S
    L, C = E // R, S * K
    T = np.bincount(np.asarray(topk).ravel(), minlength=E)
    Hl = T.reshape(R, L).sum(axis=1)
    X = np.maximum(Hl - C, 0)
    D = np.maximum(C - Hl, 0)
    n_rep = int(p["info"][1])
    reps = [(int(p["rep_expert"][q]), int(p["rep_rank"][q]), int(p["rep_quota"][q]))
            for q in range(n_rep)]
    shed = np.zeros(E, np.int64)
    recv = np.zeros(R, np.int64)
    for e, r, q in reps:
        shed[e] += q
        recv[r] += q
    # every deficit filled exactly, every excess shed exactly
    assert np.array_equal(recv, D)
    assert np.array_equal(shed.reshape(R, L).sum(axis=1), X)
    # largest-first: at most one partially shed expert per donor, and every
    # shed expert is at least as large as every kept-whole expert
    for r in range(R):
        if X[r] == 0:
            assert shed[r * L:(r + 1) * L].sum() == 0
            continue
        ex = list(range(r * L, (r + 1) * L))
        shed_set = [e for e in ex if shed[e] > 0]
        rest = [e for e in ex if shed[e] == 0]
        partial = [e for e in shed_set if shed[e] < T[e]]
        assert len(partial) <= 1
        if shed_set and rest:
            lo = min((T[e], -e) for e in shed_set)
            hi = max((T[e], -e) for e in rest)
            assert lo > hi
    P = int((shed > 0).sum())
    N = int((D > 0).sum())
    assert p["info"][3] == P and p["info"][4] == N
    if P:
        assert max(P, N) <= n_rep <= P + N - 1
    else:
        assert n_rep == 0
    # orders: pieces by (shed desc, e asc), receivers by (D desc, r asc)
    pieces = sorted([e for e in range(E) if shed[e] > 0], key=lambda e: (-shed[e], e))
    recvs = sorted([r for r in range(R) if D[r] > 0], key=lambda r: (-D[r], r))
    # north-west corner: the merge walks both lists monotonically
    jpos = [pieces.index(e) for e, _, _ in reps]
    ipos = [recvs.index(r) for _, r, _ in reps]
    if reps:
        assert jpos[0] == 0 and ipos[0] == 0
        assert jpos[-1] == len(pieces) - 1 and ipos[-1] == len(recvs) - 1
    for a in range(1, len(reps)):
        dj, di = jpos[a] - jpos[a - 1], ipos[a] - ipos[a - 1]
        assert (dj, di) in ((0, 1), (1, 0), (1, 1))
    # segment count is the number of distinct interior breakpoints plus one
    ps = set(np.cumsum([shed[e] for e in pieces])[:-1].tolist()) if pieces else set()
    qs = set(np.cumsum([D[r] for r in recvs])[:-1].tolist()) if recvs else set()
    if pieces:
        assert n_rep == len(ps | qs) + 1
    return P, N
