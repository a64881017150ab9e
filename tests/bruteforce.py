"""Brute-force minimum-replica placement on micro inputs (test helper).

Independent of the oracle's greedy: it enumerates replica sets
``{(e, r) : r != home(e)}`` by increasing size and accepts the first set for
which a max-flow (source -> expert e with capacity T_e, expert -> every rank
hosting it, rank -> sink with capacity C) saturates R*C.  That smallest size
is the optimum number of replicas that gives every rank exactly C slots.
"""
from __future__ import annotations

import itertools
from collections import deque


def _max_flow(n, edges, s, t):
    cap = {}
    adj = [[] for _ in range(n)]
    for u, v, c in edges:
        if (u, v) not in cap:
            adj[u].append(v)
            adj[v].append(u)
            cap[(u, v)] = 0
            cap.setdefault((v, u), 0)
        cap[(u, v)] += c
    flow = 0
    while True:
        par = [-1] * n
        par[s] = s
        dq = deque([s])
        while dq and par[t] < 0:
            u = dq.popleft()
            for v in adj[u]:
                if par[v] < 0 and cap[(u, v)] > 0:
                    par[v] = u
                    dq.append(v)
        if par[t] < 0:
            return flow
        aug = float("inf")
        v = t
        while v != s:
            aug = min(aug, cap[(par[v], v)])
            v = par[v]
        v = t
        while v != s:
            cap[(par[v], v)] -= aug
            cap[(v, par[v])] += aug
            v = par[v]
        flow += aug


def feasible(T, R, L, C, replicas) -> bool:
    E = len(T)
    src, snk = E + R, E + R + 1
    edges = [(src, e, T[e]) for e in range(E) if T[e] > 0]
    for e in range(E):
        edges.append((e, E + e // L, T[e]))
    for (e, r) in replicas:
        edges.append((e, E + r, T[e]))
    for r in range(R):
        edges.append((E + r, snk, C))
    return _max_flow(E + R + 2, edges, src, snk) == R * C


def min_replicas(T, R, L, C, max_size=None) -> int:
    E = len(T)
    cand = [(e, r) for e in range(E) for r in range(R) if r != e // L and T[e] > 0]
    top = len(cand) if max_size is None else max_size
    for k in range(top + 1):
        for combo in itertools.combinations(cand, k):
            if feasible(T, R, L, C, combo):
                return k
    return -1


def feasible_within_budget(T, R, L, C, B) -> bool:
    """Whether some replica set with at most B replicas on every rank gives
    every rank exactly C slots (sets enumerated by increasing size)."""
    E = len(T)
    cand = [(e, r) for e in range(E) for r in range(R) if r != e // L and T[e] > 0]
    for k in range(len(cand) + 1):
        for combo in itertools.combinations(cand, k):
            per = [0] * R
            for _, r in combo:
                per[r] += 1
            if max(per) <= B and feasible(T, R, L, C, combo):
                return True
    return False


def min_cover_count(values, target) -> int:
    """Fewest of ``values`` whose sum reaches ``target`` (brute force)."""
    if target <= 0:
        return 0
    n = len(values)
    for k in range(1, n + 1):
        for combo in itertools.combinations(values, k):
            if sum(combo) >= target:
                return k
    return -1
