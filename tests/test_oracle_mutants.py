"""Planted mistakes in the relay cascade of the oracle, each of which the
hand-worked cascade plans (tests/golden/plan_example_cascade*.json) must
reject.  Each mutant is a copy of oracle/moonep_oracle.c with one rule of
the cascade changed, compiled with the oracle's own flags into a temporary
directory; the test then plans every cascade golden with it and requires at
least one expected field to differ.  Nothing here touches the CUDA library.

Not pinned: the capacity guard's threshold (a step is skipped when the live
list plus m + B - 1 would exceed E + R - 1).  It binds only when the list is
within one step of full, which no small routing reaches."""
import importlib.util
import json
import os
import shutil
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
GOLDEN = os.path.join(ROOT, "tests", "golden")
CASCADE_GOLDENS = ["plan_example_cascade", "plan_example_cascade_relay", "plan_example_cascade_merge",
                   "plan_example_cascade_chain", "plan_example_cascade_two_relays"]

EXTRA_CMP = """
static int cmp_val_desc_idx_desc(const void *a, const void *b)
{
    const vi_t *x = (const vi_t *)a, *y = (const vi_t *)b;
    if (x->val != y->val) return x->val > y->val ? -1 : 1;
    return (x->idx < y->idx) - (x->idx > y->idx);
}
static int cmp_val_asc_idx_asc(const void *a, const void *b)
{
    const vi_t *x = (const vi_t *)a, *y = (const vi_t *)b;
    if (x->val != y->val) return x->val < y->val ? -1 : 1;
    return (x->idx > y->idx) - (x->idx < y->idx);
}
"""
CMP_ANCHOR = "typedef struct { int32_t rank, slot, quota, is_home; } host_t;"

# name -> [(text in the oracle, replacement)]
MUTANTS = {
    "relay ties broken by the higher expert": [
        ("qsort(cand, (size_t)nc, sizeof(vi_t), cmp_val_desc_idx_asc);",
         "qsort(cand, (size_t)nc, sizeof(vi_t), cmp_val_desc_idx_desc);")],
    "relays may already sit on the rank": [
        ("if (keep[e] > 0 && h != rs && !closed[h] && !on_r[e])", "if (keep[e] > 0 && h != rs && !closed[h])")],
    "relays may share a home rank": [("if (home_used[h]) continue;", "")],
    "relays may live on a closed rank": [
        ("if (keep[e] > 0 && h != rs && !closed[h] && !on_r[e])", "if (keep[e] > 0 && h != rs && !on_r[e])")],
    "moved quota never returns home": [
        ("if (ek / L == h) {\n                keep[ek] += (int32_t)amt;", "if (0) {\n                keep[ek] += (int32_t)amt;")],
    "rank's replicas by ascending quota": [
        ("qsort(S, (size_t)n, sizeof(vi_t), cmp_val_desc_idx_asc);\n        /* relay",
         "qsort(S, (size_t)n, sizeof(vi_t), cmp_val_asc_idx_asc);\n        /* relay")],
    "rank's quota ties by descending list position": [
        ("qsort(S, (size_t)n, sizeof(vi_t), cmp_val_desc_idx_asc);\n        /* relay",
         "qsort(S, (size_t)n, sizeof(vi_t), cmp_val_desc_idx_desc);\n        /* relay")],
    "rank ties go to the higher rank": [
        ("(rs < 0 || cnt[r] > cnt[rs])) rs = r;", "(rs < 0 || cnt[r] >= cnt[rs])) rs = r;")],
    "the rank with the fewest replicas first": [
        ("(rs < 0 || cnt[r] > cnt[rs])) rs = r;", "(rs < 0 || cnt[r] < cnt[rs])) rs = r;")],
    "kept replicas grow on closed homes": [
        ("room += closed[e / L] ? 0 : keep[e];", "room += keep[e];"),
        ("const int64_t capk = (pq[k] >= 0 && closed[e / L] && e / L != rs) ? 0 : keep[e];",
         "const int64_t capk = keep[e];")],
    "m starts at 1": [
        ("for (int32_t m = 0; m <= B && m_found < 0; ++m) {", "for (int32_t m = 1; m <= B && m_found < 0; ++m) {")],
    "the largest workable m": [
        ("for (int32_t m = 0; m <= B && m_found < 0; ++m) {", "for (int32_t m = 0; m <= B; ++m) {")],
    "moved quota never joins an existing replica": [
        ("if (found >= 0) {\n                    rq[found]", "if (0) {\n                    rq[found]")],
    "list order reversed after a step": [
        ("if (alive[q]) { re[w] = re[q]; rr[w] = rr[q]; rq[w] = rq[q]; alive[w] = 1; ++w; }\n        *nl = w;",
         "if (alive[q]) { re[w] = re[q]; rr[w] = rr[q]; rq[w] = rq[q]; alive[w] = 1; ++w; }\n        *nl = w;\n"
         "        for (int32_t i = 0, j = w - 1; i < j; ++i, --j) { int32_t t; t = re[i]; re[i] = re[j]; re[j] = t;"
         " t = rr[i]; rr[i] = rr[j]; rr[j] = t; t = rq[i]; rq[i] = rq[j]; rq[j] = t; }")],
}


def _load_mutant(tmp, tag, edits):
    d = os.path.join(tmp, "oracle_" + tag)
    shutil.copytree(os.path.join(ROOT, "oracle"), d, ignore=shutil.ignore_patterns("*.so", "__pycache__"))
    src_path = os.path.join(d, "moonep_oracle.c")
    s = open(src_path).read().replace(CMP_ANCHOR, EXTRA_CMP + CMP_ANCHOR)
    for old, new in edits:
        assert s.count(old) == 1, f"the oracle no longer contains: {old!r}"
        s = s.replace(old, new)
    open(src_path, "w").write(s)
    name = "oracle_mutant_" + tag
    spec = importlib.util.spec_from_file_location(name, os.path.join(d, "__init__.py"), submodule_search_locations=[d])
    mod = importlib.util.module_from_spec(spec)
    sys.modules[name] = mod
    spec.loader.exec_module(mod)
    mod.build(force=True)
    return mod


def _golden_holds(mod, g):
    topk = np.array(g["topk_idx"], np.int32)
    try:
        p = mod.plan(mod.Config(**g["config"]), topk)
    except Exception:
        return False
    for k, v in g["expect"].items():
        if k == "info":
            inf = mod.info_dict(p)
            if {f: inf[f] for f in v} != v:
                return False
        elif p[k].tolist() != v:
            return False
    return True


@pytest.fixture(scope="module")
def goldens():
    return [json.load(open(os.path.join(GOLDEN, n + ".json"))) for n in CASCADE_GOLDENS]


def test_unmutated_copy_holds_every_golden(tmp_path, goldens):
    mod = _load_mutant(str(tmp_path), "none", [])
    assert all(_golden_holds(mod, g) for g in goldens)


@pytest.mark.parametrize("what", sorted(MUTANTS))
def test_planted_mistake_is_caught(tmp_path, goldens, what):
    tag = "".join(c if c.isalnum() else "_" for c in what)
    mod = _load_mutant(str(tmp_path), tag, MUTANTS[what])
    held = [n for n, g in zip(CASCADE_GOLDENS, goldens) if _golden_holds(mod, g)]
    assert len(held) < len(goldens), f"'{what}' passes every hand-worked cascade plan"
