"""Planted mistakes in the oracle, each of which its pins must reject.

Each mutant is a copy of oracle/moonep_oracle.c with one plausible mistake
(a reversed order or tie-break, a dropped rule or term, an off-by-one, a
missing rounding or a wrong accumulation type), compiled with the oracle's
own flags into a temporary directory.
* Relay cascade mutants: every hand-worked cascade plan
  (tests/golden/plan_example_cascade*.json) is planned with the mutant and
  at least one expected field must differ.
* Core plan, data-step, rounding and configuration mutants: the pin of
  tests/test_oracle_pins.py that covers the step is run against the mutant
  (the module's oracle swapped for it) and must fail.
Nothing here touches the CUDA library.

The cascade's capacity guard (a step is skipped when the live list plus
m + B - 1 would exceed E + R - 1) is pinned in two parts.  Its arithmetic:
the slack it computes is reported in the plan's info, hand-worked in every
cascade golden, so the mutants below that change the sum or the capacity are
caught there.  Its comparison: with the capacity lowered (a test setting of
both the oracle and the CUDA planner), the hand-worked plan_example_cascade
puts its one step exactly on the limit and one over it, so a threshold moved
either way is caught (on every routing the tests enumerate the default
capacity leaves a slack of at least 3).

Not pinned, with the reason:
* water-filling loops nested receiver-major instead of piece-major: an
  equivalent program, since the north-west-corner overlaps form a staircase
  rising in both the piece and the receiver index, so both nestings list
  the replicas in the same order;
* dropping the reduce's skip of the home host: equivalent, since the home
  host's slot is below L and the prefetched-ordinal check skips it too;
* starting the cascade, or picking a rank to repair, at exactly B replicas
  instead of above B: equivalent, since a rank at B is picked only once no
  open rank is over B, and its repair moves nothing."""
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
static int cmp_host_rank_desc(const void *a, const void *b)
{
    const host_t *x = (const host_t *)a, *y = (const host_t *)b;
    return (x->rank < y->rank) - (x->rank > y->rank);
}
"""
CMP_ANCHOR = "static int64_t min64(int64_t a, int64_t b)"

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
    "moved replicas water-filled in reverse order": [
        ("        int32_t mk = k0, pi = 0;\n        int64_t a_left = mk < n ? sv_q[mk] : 0, c_left = np > 0 ? pa[0] : 0;",
         "        for (int32_t i = k0, j = n - 1; i < j; ++i, --j) { int32_t t = sv_e[i]; sv_e[i] = sv_e[j]; sv_e[j] = t;"
         " t = sv_q[i]; sv_q[i] = sv_q[j]; sv_q[j] = t; }\n"
         "        int32_t mk = k0, pi = 0;\n        int64_t a_left = mk < n ? sv_q[mk] : 0, c_left = np > 0 ? pa[0] : 0;")],
    "providers in reverse order": [
        ("        /* pour Q into the providers */",
         "        for (int32_t i = 0, j = np - 1; i < j; ++i, --j) { int32_t t = pe[i]; pe[i] = pe[j]; pe[j] = t;"
         " t = pq[i]; pq[i] = pq[j]; pq[j] = t; }\n        /* pour Q into the providers */")],
    "moved quota summed over the kept end of the order": [
        ("            for (int32_t k = B - m; k < n; ++k) Q += S[k].val;",
         "            for (int32_t k = 0; k < n - (B - m); ++k) Q += S[k].val;")],
    "guard counts the step's growth as m + B": [
        ("const int32_t slack = cap - (*nl + m_found + B - 1);", "const int32_t slack = cap - (*nl + m_found + B);")],
    "guard leaves the relays out": [
        ("const int32_t slack = cap - (*nl + m_found + B - 1);", "const int32_t slack = cap - (*nl + B - 1);")],
    "guard counts the rank's replicas instead of the list": [
        ("const int32_t slack = cap - (*nl + m_found + B - 1);", "const int32_t slack = cap - (n + m_found + B - 1);")],
    "guard capacity E + R": [
        ("const int32_t slack = cap - (*nl + m_found + B - 1);", "const int32_t slack = cap + 1 - (*nl + m_found + B - 1);")],
    "guard slack kept from the last step, not the least": [
        ("if (*n_guard == 0 || slack < *min_slack) *min_slack = slack;", "*min_slack = slack;")],
    "list order reversed after a step": [
        ("if (alive[q]) { re[w] = re[q]; rr[w] = rr[q]; rq[w] = rq[q]; alive[w] = 1; ++w; }\n        *nl = w;",
         "if (alive[q]) { re[w] = re[q]; rr[w] = rr[q]; rq[w] = rq[q]; alive[w] = 1; ++w; }\n        *nl = w;\n"
         "        for (int32_t i = 0, j = w - 1; i < j; ++i, --j) { int32_t t; t = re[i]; re[i] = re[j]; re[j] = t;"
         " t = rr[i]; rr[i] = rr[j]; rr[j] = t; t = rq[i]; rq[i] = rq[j]; rq[j] = t; }")],
}

# name -> (edits, [(pin in test_oracle_pins, its arguments besides oracle_lib)])
GOLDEN_A = [("test_golden_plan", {"name": "plan_example_a"})]
GOLDEN_B = [("test_golden_plan", {"name": "plan_example_b"})]
CASCADE_PINS = [("test_golden_cascade_plan", {"name": "plan_example_cascade", "over_greedy": 3}),
                ("test_golden_cascade_plan", {"name": "plan_example_cascade_merge", "over_greedy": 2}),
                ("test_golden_cascade_plan", {"name": "plan_example_cascade_chain", "over_greedy": 3})]
GUARD_PINS = [("test_cascade_guard_threshold_at_and_over_a_lowered_capacity", {})]
LOCALITY_PINS = [("test_golden_locality_plan", {}),
                 ("test_locality_reaches_the_bound_for_its_placement", {"wname": "mid", "mv": 2.0})]
CORE_MUTANTS = {
    "O3 sheds the smallest experts first": (
        [("qsort(order, (size_t)L, sizeof(vi_t), cmp_val_desc_idx_asc);",
          "qsort(order, (size_t)L, sizeof(vi_t), cmp_val_asc_idx_asc);")], GOLDEN_A + CASCADE_PINS),
    "O3 shedding ties by the higher expert": (
        [("qsort(order, (size_t)L, sizeof(vi_t), cmp_val_desc_idx_asc);",
          "qsort(order, (size_t)L, sizeof(vi_t), cmp_val_desc_idx_desc);")], GOLDEN_A),
    "O4 pieces left in expert order": (
        [("qsort(pieces, (size_t)nP, sizeof(vi_t), cmp_val_desc_idx_asc);", "")], GOLDEN_B),
    "O4 piece ties by the higher expert": (
        [("qsort(pieces, (size_t)nP, sizeof(vi_t), cmp_val_desc_idx_asc);",
          "qsort(pieces, (size_t)nP, sizeof(vi_t), cmp_val_desc_idx_desc);")], CASCADE_PINS),
    "O4 receivers left in rank order": (
        [("qsort(recv, (size_t)nN, sizeof(vi_t), cmp_val_desc_idx_asc);", "")], CASCADE_PINS),
    "O4 receiver ties by the higher rank": (
        [("qsort(recv, (size_t)nN, sizeof(vi_t), cmp_val_desc_idx_asc);",
          "qsort(recv, (size_t)nN, sizeof(vi_t), cmp_val_desc_idx_desc);")], CASCADE_PINS),
    "O2 deficit off by one": (
        [("        D[r] = h < C ? C - h : 0;", "        D[r] = h <= C ? C - h + 1 : 0;")], GOLDEN_B),
    "O5 replica slots without the home offset": (
        [("            rep_slot[nrep] = L + nrep_on[r];", "            rep_slot[nrep] = nrep_on[r];")], GOLDEN_A),
    "O6 home slots count T instead of what stays home": (
        [("            slot_count[(int64_t)r * E + j] = keep[r * L + j];",
          "            slot_count[(int64_t)r * E + j] = T[r * L + j];")], GOLDEN_A),
    "O7 home host first instead of rank order": (
        [("        qsort(hosts, (size_t)nh, sizeof(host_t), cmp_host_rank);\n", "")], GOLDEN_B),
    "O7 hosts in descending rank": (
        [("        qsort(hosts, (size_t)nh, sizeof(host_t), cmp_host_rank);\n",
          "        qsort(hosts, (size_t)nh, sizeof(host_t), cmp_host_rank_desc);\n")], GOLDEN_A),
    "O8 pairs in (k, t) order": (
        [("    for (int64_t p = 0; p < NP; ++p) {\n        const int32_t e = topk[p];\n        const int32_t g = gcount[e]++;",
          "    for (int64_t pp = 0; pp < NP; ++pp) {\n        int64_t p = (pp % ((int64_t)R * S)) * K + pp / ((int64_t)R * S);\n"
          "        const int32_t e = topk[p];\n        const int32_t g = gcount[e]++;")], GOLDEN_B),
    "remote pairs: source rank without dividing by K": (
        [("        if (s_rank != r) ++n_remote;", "        if ((int32_t)(p / S) != r) ++n_remote;")], GOLDEN_B),
    "overflow only above B": (
        [("        if (rep_ord[q] >= B) ++n_over;", "        if (rep_ord[q] > B) ++n_over;")], GOLDEN_B),
    "work list includes overflow replicas": (
        [("            if (rep_expert[q] == e && rep_ord[q] < B) has = 1;",
          "            if (rep_expert[q] == e) has = 1;")], GOLDEN_B),
    "strict flag ignored": (
        [("        if (c->flags & OR_FLAG_STRICT_BUDGET) status |= OR_ST_STRICT_VIOLATION;", "")],
        [("test_golden_b_strict_flag", {})]),
    "combine sums k in reverse": (
        [("            for (int64_t k = 0; k < K; ++k) {\n                int64_t d = dst_pos[t * K + k];\n                acc = fmaf(",
          "            for (int64_t k = K - 1; k >= 0; --k) {\n                int64_t d = dst_pos[t * K + k];\n                acc = fmaf(")],
        [("test_combine_uses_fused_multiply_add", {})]),
    "combine without fused multiply-add": (
        [("acc = fmaf(w[t * K + k], bf16_to_f32(y[d * H + h]), acc);",
          "acc = acc + w[t * K + k] * bf16_to_f32(y[d * H + h]);")], [("test_combine_uses_fused_multiply_add", {})]),
    "combine rounds to bf16 after every k": (
        [("acc = fmaf(w[t * K + k], bf16_to_f32(y[d * H + h]), acc);",
          "acc = bf16_to_f32(or_f32_to_bf16(fmaf(w[t * K + k], bf16_to_f32(y[d * H + h]), acc)));")],
        [("test_combine_error_bound", {})]),
    "combine backward sums dw in fp32": (
        [("            double s = 0.0;", "            float s = 0.0f;"),
         ("                s += (double)g * (double)bf16_to_f32(y[d * H + h]);",
          "                s += g * bf16_to_f32(y[d * H + h]);")], [("test_combine_backward_library", {})]),
    "combine backward never scales dy": (
        [("dy_buf[d * H + h] = unscaled ? dy[t * H + h] : or_f32_to_bf16(w[p] * g);",
          "dy_buf[d * H + h] = dy[t * H + h];")], [("test_combine_backward_library", {})]),
    "combine backward unscaled flag inverted": (
        [("dy_buf[d * H + h] = unscaled ? dy[t * H + h] : or_f32_to_bf16(w[p] * g);",
          "dy_buf[d * H + h] = !unscaled ? dy[t * H + h] : or_f32_to_bf16(w[p] * g);")],
        [("test_combine_backward_library", {})]),
    "reduce in descending rank order": (
        [("        for (int32_t h = host_ptr[e]; h < host_ptr[e + 1]; ++h) {\n            int32_t r = host_rank[h], b = host_slot[h] - L;\n"
          "            if (r == e / L) continue; /* the home copy */",
          "        for (int32_t h = host_ptr[e + 1] - 1; h >= host_ptr[e]; --h) {\n            int32_t r = host_rank[h], b = host_slot[h] - L;\n"
          "            if (r == e / L) continue; /* the home copy */")], [("test_reduce_order_is_rank_ascending", {})]),
    "reduce leaves the replica rows": (
        [("#pragma omp parallel for schedule(static)\n            for (int64_t i = i0; i < i1; ++i) src[i] = 0.0f;", "")],
        [("test_reduce_exact_integers", {})]),
    "reduce includes overflow replicas": (
        [("            if (b < 0 || b >= B) continue; /* overflow replica: no reduce rows */", "            if (b < 0) continue;")],
        [("test_reduce_exact_integers", {})]),
    "prefetch without read-through for overflow": (
        [("                    row = e; /* overflow: read through to the home copy */", "                    row = -1;")],
        [("test_prefetch_hand_worked", {})]),
    "bf16 by truncation": ([("    u += 0x7fffu + lsb;", "    (void)lsb;")], [("test_bf16_rounding_matches_torch", {})]),
    "bf16 ties away from zero": (
        [("    u += 0x7fffu + lsb;", "    (void)lsb; u += 0x8000u;")], [("test_bf16_rounding_matches_torch", {})]),
    "dispatch writes only the first k": (
        [("        for (int64_t k = 0; k < K; ++k) {\n            int64_t d = dst_pos[t * K + k];\n            for (int64_t h = 0; h < H; ++h) buf",
          "        for (int64_t k = 0; k < 1; ++k) {\n            int64_t d = dst_pos[t * K + k];\n            for (int64_t h = 0; h < H; ++h) buf")],
        [("test_dispatch_rows", {})]),
    "B range check against E": (
        [("    if (c->B > c->E - L) return OR_ERR_B_RANGE;", "    if (c->B > c->E) return OR_ERR_B_RANGE;")],
        [("test_config_errors", {})]),
    "training budget rule ignored": (
        [("    if ((c->flags & OR_FLAG_TRAIN_B_RULE) && c->B != L) return OR_ERR_BUDGET_RULE;", "")],
        [("test_config_errors", {})]),
    "O3 sheds whole experts": (
        [("            int64_t s = min64(T[e], rem);", "            int64_t s = T[e];")], GOLDEN_A),
    "O3 home quota not reduced": (
        [("            keep[e] = T[e] - (int32_t)s;", "            keep[e] = T[e];")], GOLDEN_A),
    "O4 pieces include experts that shed nothing": (
        [("        if (shed[e] > 0) { pieces[nP].val", "        if (shed[e] >= 0 && T[e] > 0) { pieces[nP].val")],
        GOLDEN_A),
    "O5 zero-length overlaps kept": (
        [("            if (len <= 0) continue;", "            if (len < 0) continue;")],
        [("test_invariants_random", {"seed": s}) for s in range(12)]),
    "O5 overlap start from the smaller end": (
        [("int64_t len = min64(PS[j + 1], QS[i + 1]) - max64(PS[j], QS[i]);",
          "int64_t len = min64(PS[j + 1], QS[i + 1]) - min64(PS[j], QS[i]);")], GOLDEN_B),
    "O6 slot offsets inclusive": (
        [("            slot_offset[(int64_t)r * (E + 1) + s] = (int32_t)acc;\n            acc += slot_count[(int64_t)r * E + s];",
          "            acc += slot_count[(int64_t)r * E + s];\n            slot_offset[(int64_t)r * (E + 1) + s] = (int32_t)acc;")],
        GOLDEN_A),
    "O7 host starts not accumulated": (
        [("            start += q - loc;", "")], GOLDEN_A),
    "O8 host interval closed at its end": (
        [("if (host_start[h] <= u && u < host_start[h] + host_quota[h] - host_local[h]) {",
          "if (host_start[h] <= u && u <= host_start[h] + host_quota[h] - host_local[h]) {")], GOLDEN_A),
    "O8 row without the slot offset": (
        [("        int64_t d = (int64_t)r * C + slot_offset[(int64_t)r * (E + 1) + host_slot[found]] + off;",
          "        int64_t d = (int64_t)r * C + off;")], GOLDEN_A),
    "O8 row without subtracting the host start": (
        [("                    off = host_local[h] + (u - host_start[h]);", "                    off = host_local[h] + u;")],
        GOLDEN_A),
    "row_src names the token instead of the pair": (
        [("        row_src[d] = (int32_t)p;", "        row_src[d] = (int32_t)(p / K);")], GOLDEN_B),
    "remote pairs never counted": (
        [("        if (s_rank != r) ++n_remote;", "")], GOLDEN_A),
    "largest replica count only over B": (
        [("        if (nrep_on[r] > max_rep) max_rep = nrep_on[r];",
          "        if (nrep_on[r] > max_rep && nrep_on[r] > B) max_rep = nrep_on[r];")], GOLDEN_A),
    "overflow bit not set": (
        [("        status |= OR_ST_OVERFLOW;\n", "")], GOLDEN_B),
    "work list in reverse expert order": (
        [("        if (has) rep_home_list[n_rep_experts++] = e;", "        if (has) rep_home_list[n_rep_experts++] = E - 1 - e;")],
        GOLDEN_A),
    "combine uses the first weight for every k": (
        [("acc = fmaf(w[t * K + k], bf16_to_f32(y[d * H + h]), acc);", "acc = fmaf(w[t * K], bf16_to_f32(y[d * H + h]), acc);")],
        [("test_combine_closed_forms", {})]),
    "combine backward dots dy with the wrong row": (
        [("                s += (double)g * (double)bf16_to_f32(y[d * H + h]);",
          "                s += (double)g * (double)bf16_to_f32(y[t * H + h]);")], [("test_combine_backward_library", {})]),
    "prefetch pool row strided by L instead of B": (
        [("                    row = E + r * B + b;", "                    row = E + r * L + b;")],
        [("test_prefetch_budget_above_L", {})]),
    "cascade guard refuses a step at zero slack": (
        [("        if (slack < 0) continue; /* the list could outgrow the plan's arrays */",
          "        if (slack <= 0) continue; /* the list could outgrow the plan's arrays */")], GUARD_PINS),
    "cascade guard takes a step one over the capacity": (
        [("        if (slack < 0) continue; /* the list could outgrow the plan's arrays */",
          "        if (slack < -1) continue; /* the list could outgrow the plan's arrays */")], GUARD_PINS),
    "cascade guard ignores a lowered capacity": (
        [("            const int32_t cap = NREP_MAX - 1 < or_cascade_cap_limit ? NREP_MAX - 1 : or_cascade_cap_limit;",
          "            const int32_t cap = NREP_MAX - 1;")], GUARD_PINS),
    "locality takes the whole quota locally": (
        [("const int32_t loc = locality ? (int32_t)min64(q, src_count[(int64_t)hosts[h].rank * E + e]) : 0;",
          "const int32_t loc = locality ? q : 0;")], LOCALITY_PINS),
    "locality counts the next rank's pairs": (
        [("const int32_t loc = locality ? (int32_t)min64(q, src_count[(int64_t)hosts[h].rank * E + e]) : 0;",
          "const int32_t loc = locality ? (int32_t)min64(q, src_count[(int64_t)((hosts[h].rank + 1) % R) * E + e]) : 0;")],
        LOCALITY_PINS),
    "leftover starts count the whole quota": (
        [("            start += q - loc;", "            start += q;")], LOCALITY_PINS),
    "local pairs before a pair leave out its own rank": (
        [("if (host_rank[h] <= s_rank) before += host_local[h];", "if (host_rank[h] < s_rank) before += host_local[h];")],
        LOCALITY_PINS),
    "leftover offset without the local rows": (
        [("                    off = host_local[h] + (u - host_start[h]);", "                    off = (u - host_start[h]);")],
        LOCALITY_PINS),
    "local test on the expert-wide index": (
        [("        if (own >= 0 && gs < host_local[own]) {\n            found = own;\n            off = gs;",
          "        if (own >= 0 && g < host_local[own]) {\n            found = own;\n            off = g;")],
        LOCALITY_PINS),
    "bf16 NaN truncated without forcing the quiet bit": (
        [("        return (uint16_t)((u >> 16) | 0x0040u);", "        return (uint16_t)(u >> 16);")],
        [("test_bf16_nan_patterns", {})]),
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
    mod.build(force=True, openmp=False)
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


@pytest.mark.parametrize("what", sorted(CORE_MUTANTS))
def test_planted_core_mistake_is_caught(tmp_path, monkeypatch, what):
    import test_oracle_pins as pins
    edits, killers = CORE_MUTANTS[what]
    tag = "".join(c if c.isalnum() else "_" for c in what)
    mod = _load_mutant(str(tmp_path), tag, edits)
    monkeypatch.setattr(pins, "oracle", mod)
    caught = []
    for fn, kw in killers:
        try:
            getattr(pins, fn)(mod, **kw)
        except Exception:  # a failed assertion, or the mutant oracle refusing its own plan
            caught.append(fn)
    assert caught, f"'{what}' passes {[fn for fn, _ in killers]}"


def test_unmutated_copy_passes_every_core_pin(tmp_path, monkeypatch):
    import test_oracle_pins as pins
    mod = _load_mutant(str(tmp_path), "none_core", [])
    monkeypatch.setattr(pins, "oracle", mod)
    seen = set()
    for _, killers in CORE_MUTANTS.values():
        for fn, kw in killers:
            key = (fn, tuple(sorted(kw.items())))
            if key not in seen:
                seen.add(key)
                getattr(pins, fn)(mod, **kw)
