/*
 * moonep_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, single-threaded CPU statement of what the MoonEP hot path
 * computes: the online redundant-expert plan, the zero-copy permute
 * (dispatch), the weighted unpermute (combine), its backward, and the
 * replica-gradient reduction.  It exists so that the CUDA library can be
 * checked against it.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load it; the product path never does.
 * It shares no code, header or table with the CUDA library.
 *
 * Sources (web pages on MoonEP; cited by page title and section):
 *   [P1] "Moonshot AI Open-Sources MoonEP: A Perfectly Balanced Expert
 *        Parallelism Library for MoE Training" -- sections "The problem
 *        MoonEP targets", "The core idea: dynamic redundant experts", and the
 *        interactive explainer's tabs (invariant, memory, maxvio, pillars).
 *   [P2] "Moonshot AI 开源 MoonEP，面向分布式 MoE 工作负载优化通信" (news
 *        aggregator) -- the README excerpt on zero copy and the three
 *        properties.
 *   [P4] "Moonshot Open-Sources MoonEP for MoE Distributed Communication and
 *        Load Balancing" -- "Core Technical Approach".
 *
 * What the pages fix: every rank receives exactly S*K token slots however
 * skewed the routing is [P1 core idea; P4]; this is achieved by a small
 * number of redundant experts planned online from the router output [P1
 * core idea]; tokens are written straight into expert-grouped positions and
 * views of a fixed S*K buffer are handed to compute [P1 core idea; P2];
 * at most B prefetched replica slots per rank, B = E/R in training [P1
 * explainer, memory tab]; duplicated experts' gradients are summed back to
 * their home experts and the replica buffer is zeroed [P1 explainer, memory
 * tab, training branch].
 *
 * What the pages leave open (the planning algorithm is only called
 * "near-optimal" [P1 core idea]) is filled with the plainest reading of a
 * histogram / scan / water-filling planner, in these steps:
 *   O1 histogram T[e];
 *   O2 home loads Hl[r], excess X[r] = max(0, Hl-C), deficit D[r];
 *   O3 each donor sheds its largest experts first (T desc, e asc) until its
 *      excess is gone -> pieces (e, shed[e]);
 *   O4 pieces ordered by (shed desc, e asc), receivers by (D desc, r asc),
 *      and their prefix sums PS, QS;
 *   O5 water-filling: every positive overlap of piece j's interval with
 *      receiver i's interval is one replica of expert e(p_j) on rank r(q_i),
 *      created in (j, i) order; a rank's replicas take slots L, L+1, ... in
 *      creation order; ordinal >= B means overflow (read-through);
 *   O5b (only with the cascade flag, and only when O5 left a rank with more
 *      than B replicas) relay cascade, described at or_cascade below;
 *   O6 per-rank slot tables (home slots 0..L-1, then replicas);
 *   O7 per-expert host intervals, hosts in ascending rank order (with
 *      OR_FLAG_LOCALITY each host first serves the pairs of its own rank);
 *   O8 pairs in global (t, k) order fill their expert's host intervals.
 *
 * Floating point: the precision is the one the method fixes -- bf16 data,
 * fp32 combine accumulation in k order with fused multiply-add, fp32
 * non-fused adds for the gradient reduction; the combine-backward dot
 * product is taken in fp64 and rounded once to fp32.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <math.h>

#define OR_FLAG_STRICT_BUDGET 1u
#define OR_FLAG_TRAIN_B_RULE 2u
#define OR_FLAG_BWD_UNSCALED 4u
#define OR_FLAG_CASCADE 8u
#define OR_FLAG_LOCALITY 16u

#define OR_ST_EXPERT_ID_RANGE 1
#define OR_ST_OVERFLOW 2
#define OR_ST_STRICT_VIOLATION 4

#define OR_OK 0
#define OR_ERR_ARG 1
#define OR_ERR_E_NOT_DIVISIBLE 2
#define OR_ERR_BUDGET_RULE 3
#define OR_ERR_B_RANGE 4
#define OR_ERR_NOMEM 6

/* info[] fields */
#define OR_INFO_STATUS 0
#define OR_INFO_N_REP 1
#define OR_INFO_N_OVERFLOW 2
#define OR_INFO_N_PIECES 3
#define OR_INFO_N_RECEIVERS 4
#define OR_INFO_MAX_REP_PER_RANK 5
#define OR_INFO_N_REP_EXPERTS 6
#define OR_INFO_N_REMOTE_PAIRS 7
#define OR_INFO_CASCADE_GUARD_STEPS 8
#define OR_INFO_CASCADE_GUARD_SLACK 9
#define OR_INFO_LEN 16

typedef struct {
    int32_t R, E, K, S, H, B;
    uint32_t flags;
} or_config;

/* ---------------------------------------------------------------- bf16 -- */

/* bf16 -> fp32 is exact: the bf16 pattern is the top half of the fp32 one. */
static float bf16_to_f32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* fp32 -> bf16, round to nearest, ties to even, on bit 16.  A NaN stays a
 * NaN (sign and top payload bits kept, quiet bit forced). */
uint16_t or_f32_to_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu) != 0u)
        return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

float or_bf16_to_f32(uint16_t b) { return bf16_to_f32(b); }

/* ------------------------------------------------------------ checks ---- */

int or_check_config(const or_config *c)
{
    if (!c) return OR_ERR_ARG;
    if (c->R <= 0 || c->E <= 0 || c->K <= 0 || c->S <= 0 || c->H <= 0 || c->B < 0)
        return OR_ERR_ARG;
    if (c->K > c->E) return OR_ERR_ARG;
    if ((int64_t)c->R * c->S * c->K > INT32_MAX) return OR_ERR_ARG;
    if (c->flags & ~(OR_FLAG_STRICT_BUDGET | OR_FLAG_TRAIN_B_RULE | OR_FLAG_BWD_UNSCALED | OR_FLAG_CASCADE |
                     OR_FLAG_LOCALITY))
        return OR_ERR_ARG;
    /* the explainer flags E % R != 0 as a configuration error [P1 explainer] */
    if (c->E % c->R != 0) return OR_ERR_E_NOT_DIVISIBLE;
    int32_t L = c->E / c->R;
    /* training requires B = E/R [P1 explainer, memory tab] */
    if ((c->flags & OR_FLAG_TRAIN_B_RULE) && c->B != L) return OR_ERR_BUDGET_RULE;
    /* a rank can never host more than E-L distinct foreign experts */
    if (c->B > c->E - L) return OR_ERR_B_RANGE;
    return OR_OK;
}

/* ------------------------------------------------------------- plan ----- */

typedef struct { int32_t val, idx; } vi_t;

/* order: value descending, then index ascending */
static int cmp_val_desc_idx_asc(const void *a, const void *b)
{
    const vi_t *x = (const vi_t *)a, *y = (const vi_t *)b;
    if (x->val != y->val) return x->val > y->val ? -1 : 1;
    return (x->idx > y->idx) - (x->idx < y->idx);
}

typedef struct { int32_t rank, slot, quota, is_home; } host_t;

static int cmp_host_rank(const void *a, const void *b)
{
    const host_t *x = (const host_t *)a, *y = (const host_t *)b;
    return (x->rank > y->rank) - (x->rank < y->rank);
}

static int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }
static int64_t max64(int64_t a, int64_t b) { return a > b ? a : b; }

/* O5b, relay cascade.  The pages require at most B = E/R prefetched replica
 * slots per rank in training [P1 explainer, memory tab] and give no
 * algorithm; water-filling can exceed B when a rank with a large deficit is
 * filled from many small pieces.  This step repairs such ranks one at a
 * time, always the rank with the most replicas (ties: lowest rank) among
 * those over B and not yet closed:
 *   - its replicas are ordered by (quota desc, list position asc); for the
 *     smallest m in 0..B it keeps the first B-m and moves the rest (total
 *     Q) away, provided the providers can carry Q.  The providers are, in
 *     order, the kept replicas (each can grow by its expert's remaining home
 *     quota keep[e], unless its home rank is closed) and then m relay
 *     experts: those with keep > 0 whose home rank is not this rank, not
 *     closed and not already a relay home, and that have no replica on this
 *     rank, taken in (keep desc, expert asc) order;
 *   - Q is poured into the providers in that order, each taking min(its
 *     capacity, what is left): a kept replica's quota grows, a relay becomes
 *     a new replica on this rank (appended to the list), and the provider's
 *     home keeps that much less;
 *   - the moved quotas are water-filled, in the moved order, into the
 *     providers' home ranks in provider order (capacity = what each took):
 *     an amount of expert e landing on e's own home returns to keep[e]; on a
 *     rank that already holds a replica of e it is added to that replica;
 *     otherwise it is a new replica appended to the list;
 *   - the rank is closed.  A rank no m works for is closed unchanged.
 * Every step keeps every rank's total at C and every expert's hosts summing
 * to T[e]; it closes one rank, so there are at most R steps.  A step adds at
 * most m + B - 1 live replicas (the relays, and the water-fill's splits
 * beyond the moved replicas it replaces); a step for which the live count
 * plus m + B - 1 would exceed cap is not taken (the rank is closed over B),
 * so the list never outgrows the plan's replica arrays.  Replicas keep list
 * order (dead entries are dropped after each step); ordinals are re-derived
 * by the caller.  re/rr/rq/alive: list arrays of capacity
 * lcap >= 2 * cap + 2 * B + 2; *nl: entries used. */
/* The capacity the cascade's guard compares with: the plan's E + R - 1
 * replica entries, or less when a test lowers it (or_set_cascade_capacity)
 * to put a step exactly on the limit. */
static int32_t or_cascade_cap_limit = INT32_MAX;

int32_t or_set_cascade_capacity(int32_t c)
{
    const int32_t prev = or_cascade_cap_limit;
    or_cascade_cap_limit = c > 0 ? c : INT32_MAX;
    return prev == INT32_MAX ? 0 : prev;
}

static int or_cascade(int32_t R, int32_t E, int32_t L, int32_t B, int32_t cap, int32_t *keep,
                      int32_t *re, int32_t *rr, int32_t *rq, int32_t *alive, int32_t *nl, int32_t lcap,
                      int32_t *n_guard, int32_t *min_slack)
{
    int32_t *cnt = calloc((size_t)R, sizeof(int32_t));
    int32_t *closed = calloc((size_t)R, sizeof(int32_t));
    int32_t *on_r = calloc((size_t)E, sizeof(int32_t));
    int32_t *home_used = calloc((size_t)R, sizeof(int32_t));
    vi_t *S = calloc((size_t)lcap, sizeof(vi_t));
    vi_t *cand = calloc((size_t)E, sizeof(vi_t));
    int32_t *pe = calloc((size_t)lcap + B + 1, sizeof(int32_t));   /* provider expert */
    int32_t *pq = calloc((size_t)lcap + B + 1, sizeof(int32_t));   /* kept replica index, -1 for a relay */
    int32_t *pa = calloc((size_t)lcap + B + 1, sizeof(int32_t));   /* amount taken */
    int32_t *sv_e = calloc((size_t)lcap, sizeof(int32_t)), *sv_q = calloc((size_t)lcap, sizeof(int32_t));
    int rc = OR_OK;
    if (!cnt || !closed || !on_r || !home_used || !S || !cand || !pe || !pq || !pa || !sv_e || !sv_q) {
        rc = OR_ERR_NOMEM;
        goto done;
    }
    for (;;) {
        for (int32_t r = 0; r < R; ++r) cnt[r] = 0;
        for (int32_t q = 0; q < *nl; ++q)
            if (alive[q]) cnt[rr[q]] += 1;
        int32_t rs = -1;
        for (int32_t r = 0; r < R; ++r)
            if (!closed[r] && cnt[r] > B && (rs < 0 || cnt[r] > cnt[rs])) rs = r;
        if (rs < 0) break;
        /* the rank's replicas by (quota desc, list position asc) */
        int32_t n = 0;
        for (int32_t e = 0; e < E; ++e) on_r[e] = 0;
        for (int32_t q = 0; q < *nl; ++q)
            if (alive[q] && rr[q] == rs) { S[n].val = rq[q]; S[n].idx = q; ++n; on_r[re[q]] = 1; }
        qsort(S, (size_t)n, sizeof(vi_t), cmp_val_desc_idx_asc);
        /* relay candidates by (keep desc, expert asc) */
        int32_t nc = 0;
        for (int32_t e = 0; e < E; ++e) {
            const int32_t h = e / L;
            if (keep[e] > 0 && h != rs && !closed[h] && !on_r[e]) { cand[nc].val = keep[e]; cand[nc].idx = e; ++nc; }
        }
        qsort(cand, (size_t)nc, sizeof(vi_t), cmp_val_desc_idx_asc);
        /* the smallest m whose providers carry the moved quota */
        int32_t m_found = -1, np = 0;
        int64_t Q = 0;
        for (int32_t m = 0; m <= B && m_found < 0; ++m) {
            Q = 0;
            for (int32_t k = B - m; k < n; ++k) Q += S[k].val;
            int64_t room = 0;
            np = 0;
            for (int32_t k = 0; k < B - m; ++k) {
                const int32_t e = re[S[k].idx];
                pe[np] = e;
                pq[np] = S[k].idx;
                room += closed[e / L] ? 0 : keep[e];
                ++np;
            }
            for (int32_t r = 0; r < R; ++r) home_used[r] = 0;
            int32_t got = 0;
            for (int32_t c = 0; c < nc && got < m; ++c) {
                const int32_t h = cand[c].idx / L;
                if (home_used[h]) continue;
                home_used[h] = 1;
                pe[np] = cand[c].idx;
                pq[np] = -1;
                room += cand[c].val;
                ++np;
                ++got;
            }
            if (got < m) break; /* fewer distinct relay homes than m: no larger m works either */
            if (room >= Q) m_found = m;
        }
        closed[rs] = 1;
        if (m_found < 0) continue;
        /* the guard: the step may add m + B - 1 live replicas; its slack is
         * recorded (the smallest over the steps that reach it) */
        const int32_t slack = cap - (*nl + m_found + B - 1);
        if (*n_guard == 0 || slack < *min_slack) *min_slack = slack;
        *n_guard += 1;
        if (slack < 0) continue; /* the list could outgrow the plan's arrays */
        /* the moved replicas' experts and quotas, before anything changes */
        for (int32_t k = 0; k < n; ++k) { sv_e[k] = re[S[k].idx]; sv_q[k] = rq[S[k].idx]; }
        int overfull = 0;
        /* pour Q into the providers */
        int64_t rem = Q;
        for (int32_t k = 0; k < np; ++k) {
            const int32_t e = pe[k];
            const int64_t capk = (pq[k] >= 0 && closed[e / L] && e / L != rs) ? 0 : keep[e];
            const int64_t amt = min64(capk, rem);
            pa[k] = (int32_t)amt;
            rem -= amt;
            if (amt <= 0) continue;
            keep[e] -= (int32_t)amt;
            if (pq[k] >= 0) {
                rq[pq[k]] += (int32_t)amt;
            } else if (*nl < lcap) {
                re[*nl] = e; rr[*nl] = rs; rq[*nl] = (int32_t)amt; alive[*nl] = 1; *nl += 1;
            } else {
                overfull = 1;
            }
        }
        /* the moved replicas leave this rank ... */
        const int32_t k0 = B - m_found;
        for (int32_t k = k0; k < n; ++k) alive[S[k].idx] = 0;
        /* ... and are water-filled into the providers' homes */
        int32_t mk = k0, pi = 0;
        int64_t a_left = mk < n ? sv_q[mk] : 0, c_left = np > 0 ? pa[0] : 0;
        while (!overfull && mk < n && pi < np) {
            if (c_left <= 0) { ++pi; c_left = pi < np ? pa[pi] : 0; continue; }
            if (a_left <= 0) { ++mk; a_left = mk < n ? sv_q[mk] : 0; continue; }
            const int64_t amt = min64(a_left, c_left);
            const int32_t ek = sv_e[mk], h = pe[pi] / L;
            if (ek / L == h) {
                keep[ek] += (int32_t)amt;
            } else {
                int32_t found = -1;
                for (int32_t q = 0; q < *nl; ++q)
                    if (alive[q] && re[q] == ek && rr[q] == h) { found = q; break; }
                if (found >= 0) {
                    rq[found] += (int32_t)amt;
                } else if (*nl < lcap) {
                    re[*nl] = ek; rr[*nl] = h; rq[*nl] = (int32_t)amt; alive[*nl] = 1; *nl += 1;
                } else {
                    overfull = 1;
                }
            }
            a_left -= amt;
            c_left -= amt;
        }
        if (overfull) { rc = OR_ERR_ARG; goto done; } /* cannot happen: lcap covers a step */
        /* drop the dead entries, keeping list order */
        int32_t w = 0;
        for (int32_t q = 0; q < *nl; ++q)
            if (alive[q]) { re[w] = re[q]; rr[w] = rr[q]; rq[w] = rq[q]; alive[w] = 1; ++w; }
        *nl = w;
    }
done:
    free(cnt); free(closed); free(on_r); free(home_used); free(S); free(cand); free(pe); free(pq); free(pa);
    free(sv_e); free(sv_q);
    return rc;
}

/*
 * Array sizes (all int32, caller-allocated):
 *   T[E]; slot_expert[R*E]; slot_count[R*E]; slot_offset[R*(E+1)];
 *   rep_expert/rep_rank/rep_slot/rep_quota[E+R];
 *   host_ptr[E+1]; host_rank/host_slot/host_start/host_quota[2E+R];
 *   rep_home_list[E]; dst_pos[R*S*K]; row_src[R*S*K]; info[16].
 */
int or_plan(const or_config *c, const int32_t *topk,
            int32_t *T, int32_t *slot_expert, int32_t *slot_count, int32_t *slot_offset,
            int32_t *rep_expert, int32_t *rep_rank, int32_t *rep_slot, int32_t *rep_quota,
            int32_t *host_ptr, int32_t *host_rank, int32_t *host_slot, int32_t *host_start,
            int32_t *host_quota, int32_t *host_local, int32_t *rep_home_list, int32_t *dst_pos,
            int32_t *row_src, int32_t *info)
{
    int rc = or_check_config(c);
    if (rc != OR_OK) return rc;
    const int32_t R = c->R, E = c->E, K = c->K, S = c->S, B = c->B;
    const int32_t L = E / R;
    const int64_t C = (int64_t)S * K;      /* slots per rank [P1 core idea] */
    const int64_t NP = (int64_t)R * S * K; /* number of (token, k) pairs */
    const int32_t NREP_MAX = E + R, NHOST_MAX = 2 * E + R;
    int32_t n_guard = 0, min_slack = 0; /* cascade steps that reached the capacity guard, its least slack */

    /* default (empty) outputs */
    for (int64_t i = 0; i < (int64_t)R * E; ++i) { slot_expert[i] = -1; slot_count[i] = 0; }
    for (int64_t i = 0; i < (int64_t)R * (E + 1); ++i) slot_offset[i] = 0;
    for (int32_t i = 0; i < NREP_MAX; ++i) { rep_expert[i] = -1; rep_rank[i] = -1; rep_slot[i] = -1; rep_quota[i] = 0; }
    for (int32_t i = 0; i <= E; ++i) host_ptr[i] = 0;
    for (int32_t i = 0; i < NHOST_MAX; ++i) {
        host_rank[i] = -1; host_slot[i] = -1; host_start[i] = 0; host_quota[i] = 0; host_local[i] = 0;
    }
    for (int32_t i = 0; i < E; ++i) rep_home_list[i] = -1;
    for (int64_t p = 0; p < NP; ++p) { dst_pos[p] = -1; row_src[p] = -1; }
    for (int i = 0; i < OR_INFO_LEN; ++i) info[i] = 0;

    /* O1: histogram; an id outside [0, E) invalidates the plan */
    int bad = 0;
    for (int32_t e = 0; e < E; ++e) T[e] = 0;
    for (int64_t p = 0; p < NP; ++p) {
        int32_t e = topk[p];
        if (e < 0 || e >= E) { bad = 1; continue; }
        T[e] += 1;
    }
    if (bad) { info[OR_INFO_STATUS] = OR_ST_EXPERT_ID_RANGE; return OR_OK; }

    int64_t *Hl = calloc((size_t)R, sizeof(int64_t));
    int64_t *X = calloc((size_t)R, sizeof(int64_t));
    int64_t *D = calloc((size_t)R, sizeof(int64_t));
    int32_t *shed = calloc((size_t)E, sizeof(int32_t));
    int32_t *keep = calloc((size_t)E, sizeof(int32_t));
    vi_t *order = calloc((size_t)(E > R ? E : R), sizeof(vi_t));
    vi_t *pieces = calloc((size_t)E, sizeof(vi_t));
    vi_t *recv = calloc((size_t)R, sizeof(vi_t));
    int64_t *PS = calloc((size_t)E + 1, sizeof(int64_t));
    int64_t *QS = calloc((size_t)R + 1, sizeof(int64_t));
    int32_t *nrep_on = calloc((size_t)R, sizeof(int32_t));
    int32_t *rep_ord = calloc((size_t)NREP_MAX, sizeof(int32_t));
    host_t *hosts = calloc((size_t)R + 1, sizeof(host_t));
    int32_t *gcount = calloc((size_t)E, sizeof(int32_t));
    int32_t *src_count = NULL, *src_seen = NULL;  /* [R][E]: pairs per (source rank, expert) */
    if (!Hl || !X || !D || !shed || !keep || !order || !pieces || !recv || !PS || !QS ||
        !nrep_on || !rep_ord || !hosts || !gcount) {
        rc = OR_ERR_NOMEM;
        goto out;
    }

    /* O2: home loads, excess, deficit.  home(e) = floor(e / L). */
    for (int32_t r = 0; r < R; ++r) {
        int64_t h = 0;
        for (int32_t j = 0; j < L; ++j) h += T[r * L + j];
        Hl[r] = h;
        X[r] = h > C ? h - C : 0;
        D[r] = h < C ? C - h : 0;
    }

    /* O3: a donor sheds its largest experts first until its excess is gone */
    for (int32_t e = 0; e < E; ++e) { shed[e] = 0; keep[e] = T[e]; }
    for (int32_t r = 0; r < R; ++r) {
        if (X[r] <= 0) continue;
        for (int32_t j = 0; j < L; ++j) { order[j].val = T[r * L + j]; order[j].idx = r * L + j; }
        qsort(order, (size_t)L, sizeof(vi_t), cmp_val_desc_idx_asc);
        int64_t rem = X[r];
        for (int32_t j = 0; j < L && rem > 0; ++j) {
            int32_t e = order[j].idx;
            int64_t s = min64(T[e], rem);
            shed[e] = (int32_t)s;
            keep[e] = T[e] - (int32_t)s;
            rem -= s;
        }
    }

    /* O4: pieces by (shed desc, e asc); receivers by (D desc, r asc) */
    int32_t nP = 0, nN = 0;
    for (int32_t e = 0; e < E; ++e)
        if (shed[e] > 0) { pieces[nP].val = shed[e]; pieces[nP].idx = e; ++nP; }
    qsort(pieces, (size_t)nP, sizeof(vi_t), cmp_val_desc_idx_asc);
    for (int32_t r = 0; r < R; ++r)
        if (D[r] > 0) { recv[nN].val = (int32_t)D[r]; recv[nN].idx = r; ++nN; }
    qsort(recv, (size_t)nN, sizeof(vi_t), cmp_val_desc_idx_asc);
    PS[0] = 0;
    for (int32_t j = 0; j < nP; ++j) PS[j + 1] = PS[j] + pieces[j].val;
    QS[0] = 0;
    for (int32_t i = 0; i < nN; ++i) QS[i + 1] = QS[i] + recv[i].val;

    /* O5: water-filling -- every positive overlap is one replica */
    int32_t nrep = 0;
    for (int32_t j = 0; j < nP; ++j) {
        for (int32_t i = 0; i < nN; ++i) {
            int64_t len = min64(PS[j + 1], QS[i + 1]) - max64(PS[j], QS[i]);
            if (len <= 0) continue;
            int32_t r = recv[i].idx;
            rep_expert[nrep] = pieces[j].idx;
            rep_rank[nrep] = r;
            rep_ord[nrep] = nrep_on[r];
            rep_slot[nrep] = L + nrep_on[r];
            rep_quota[nrep] = (int32_t)len;
            nrep_on[r] += 1;
            ++nrep;
        }
    }

    /* O5b: relay cascade, only with the flag and only over the budget */
    if ((c->flags & OR_FLAG_CASCADE) && B > 0) {
        int32_t mx = 0;
        for (int32_t r = 0; r < R; ++r)
            if (nrep_on[r] > mx) mx = nrep_on[r];
        if (mx > B) {
            const int32_t lcap = 2 * NREP_MAX + 2 * B + 2;
            int32_t *le = calloc((size_t)lcap, sizeof(int32_t)), *lr = calloc((size_t)lcap, sizeof(int32_t));
            int32_t *lq = calloc((size_t)lcap, sizeof(int32_t)), *la = calloc((size_t)lcap, sizeof(int32_t));
            if (!le || !lr || !lq || !la) {
                free(le); free(lr); free(lq); free(la);
                rc = OR_ERR_NOMEM;
                goto out;
            }
            for (int32_t q = 0; q < nrep; ++q) { le[q] = rep_expert[q]; lr[q] = rep_rank[q]; lq[q] = rep_quota[q]; la[q] = 1; }
            int32_t nl = nrep;
            const int32_t cap = NREP_MAX - 1 < or_cascade_cap_limit ? NREP_MAX - 1 : or_cascade_cap_limit;
            rc = or_cascade(R, E, L, B, cap, keep, le, lr, lq, la, &nl, lcap, &n_guard, &min_slack);
            if (rc == OR_OK) {
                /* the final list, ordinals re-derived in list order */
                for (int32_t r = 0; r < R; ++r) nrep_on[r] = 0;
                for (int32_t q = 0; q < NREP_MAX; ++q) { rep_expert[q] = -1; rep_rank[q] = -1; rep_slot[q] = -1; rep_quota[q] = 0; }
                for (int32_t q = 0; q < nl; ++q) {
                    rep_expert[q] = le[q];
                    rep_rank[q] = lr[q];
                    rep_quota[q] = lq[q];
                    rep_ord[q] = nrep_on[lr[q]];
                    rep_slot[q] = L + nrep_on[lr[q]];
                    nrep_on[lr[q]] += 1;
                }
                nrep = nl;
            }
            free(le); free(lr); free(lq); free(la);
            if (rc != OR_OK) goto out;
        }
    }

    /* O6: slot tables.  Home slot j of rank r is expert r*L + j. */
    for (int32_t r = 0; r < R; ++r)
        for (int32_t j = 0; j < L; ++j) {
            slot_expert[(int64_t)r * E + j] = r * L + j;
            slot_count[(int64_t)r * E + j] = keep[r * L + j];
        }
    for (int32_t q = 0; q < nrep; ++q) {
        slot_expert[(int64_t)rep_rank[q] * E + rep_slot[q]] = rep_expert[q];
        slot_count[(int64_t)rep_rank[q] * E + rep_slot[q]] = rep_quota[q];
    }
    for (int32_t r = 0; r < R; ++r) {
        int64_t acc = 0;
        for (int32_t s = 0; s < E; ++s) {
            slot_offset[(int64_t)r * (E + 1) + s] = (int32_t)acc;
            acc += slot_count[(int64_t)r * E + s];
        }
        slot_offset[(int64_t)r * (E + 1) + E] = (int32_t)acc;
    }

    /* O7: host intervals per expert, hosts in ascending rank order.  Without
     * OR_FLAG_LOCALITY host h serves the pairs g in [start_h, start_h + q_h)
     * of its expert, the quotas laid out in rank order.  With it, host h
     * first serves loc_h = min(q_h, pairs of the expert from h's own rank)
     * of its own rank's pairs (the first ones, in (t, k) order), and the
     * pairs left over, in (t, k) order, fill the rest of the quotas
     * q_h - loc_h in rank order: host_start then holds where host h's share
     * of the leftover pairs starts and host_local holds loc_h. */
    const int locality = (c->flags & OR_FLAG_LOCALITY) != 0;
    if (locality) {
        src_count = calloc((size_t)R * E, sizeof(int32_t));
        if (!src_count) { rc = OR_ERR_NOMEM; goto out; }
        for (int64_t p = 0; p < NP; ++p) src_count[((p / K) / S) * E + topk[p]] += 1;
    }
    int32_t hcur = 0;
    for (int32_t e = 0; e < E; ++e) {
        int32_t nh = 0;
        hosts[nh].rank = e / L;
        hosts[nh].slot = e % L;
        hosts[nh].quota = keep[e];
        hosts[nh].is_home = 1;
        ++nh;
        for (int32_t q = 0; q < nrep; ++q)
            if (rep_expert[q] == e) {
                hosts[nh].rank = rep_rank[q];
                hosts[nh].slot = rep_slot[q];
                hosts[nh].quota = rep_quota[q];
                hosts[nh].is_home = 0;
                ++nh;
            }
        qsort(hosts, (size_t)nh, sizeof(host_t), cmp_host_rank);
        host_ptr[e] = hcur;
        int32_t start = 0;
        for (int32_t h = 0; h < nh; ++h) {
            const int32_t q = hosts[h].quota;
            const int32_t loc = locality ? (int32_t)min64(q, src_count[(int64_t)hosts[h].rank * E + e]) : 0;
            host_rank[hcur] = hosts[h].rank;
            host_slot[hcur] = hosts[h].slot;
            host_start[hcur] = start;
            host_quota[hcur] = q;
            host_local[hcur] = loc;
            start += q - loc;
            ++hcur;
        }
    }
    host_ptr[E] = hcur;

    /* O8: pairs in global (t, k) order.  The g-th pair of expert e, the
     * gs-th of e among the pairs of its own source rank s: if the host on
     * rank s serves gs among its local pairs (gs < loc), it takes the pair
     * at offset gs; otherwise the pair is leftover number
     * u = g - (local pairs of the hosts on ranks <= s), and the host whose
     * leftover share [start, start + q - loc) holds u takes it at offset
     * loc + (u - start).  Without the flag loc = 0: u = g, the plain
     * interval layout. */
    int64_t n_remote = 0;
    src_seen = calloc((size_t)R * E, sizeof(int32_t));
    if (!src_seen) { rc = OR_ERR_NOMEM; goto out; }
    for (int32_t e = 0; e < E; ++e) gcount[e] = 0;
    for (int64_t p = 0; p < NP; ++p) {
        const int32_t e = topk[p];
        const int32_t g = gcount[e]++;
        const int32_t s_rank = (int32_t)((p / K) / S);
        const int32_t gs = src_seen[(int64_t)s_rank * E + e]++;
        int32_t found = -1, own = -1;
        int64_t off = 0, before = 0;
        for (int32_t h = host_ptr[e]; h < host_ptr[e + 1]; ++h) {
            if (host_rank[h] <= s_rank) before += host_local[h];
            if (host_rank[h] == s_rank) own = h;
        }
        if (own >= 0 && gs < host_local[own]) {
            found = own;
            off = gs;
        } else {
            const int64_t u = g - before;
            for (int32_t h = host_ptr[e]; h < host_ptr[e + 1]; ++h)
                if (host_start[h] <= u && u < host_start[h] + host_quota[h] - host_local[h]) {
                    found = h;
                    off = host_local[h] + (u - host_start[h]);
                    break;
                }
        }
        if (found < 0) { rc = OR_ERR_ARG; goto out; } /* cannot happen: quotas sum to T[e] */
        int32_t r = host_rank[found];
        int64_t d = (int64_t)r * C + slot_offset[(int64_t)r * (E + 1) + host_slot[found]] + off;
        if (d < 0 || d >= (int64_t)R * C) { rc = OR_ERR_ARG; goto out; } /* cannot happen */
        dst_pos[p] = (int32_t)d;
        row_src[d] = (int32_t)p;
        if (s_rank != r) ++n_remote;
    }

    /* statistics and the reduce work list */
    int32_t n_over = 0, max_rep = 0, n_rep_experts = 0;
    for (int32_t q = 0; q < nrep; ++q)
        if (rep_ord[q] >= B) ++n_over;
    for (int32_t r = 0; r < R; ++r)
        if (nrep_on[r] > max_rep) max_rep = nrep_on[r];
    for (int32_t e = 0; e < E; ++e) {
        int has = 0;
        for (int32_t q = 0; q < nrep; ++q)
            if (rep_expert[q] == e && rep_ord[q] < B) has = 1;
        if (has) rep_home_list[n_rep_experts++] = e;
    }
    int32_t status = 0;
    if (n_over > 0) {
        status |= OR_ST_OVERFLOW;
        if (c->flags & OR_FLAG_STRICT_BUDGET) status |= OR_ST_STRICT_VIOLATION;
    }
    info[OR_INFO_STATUS] = status;
    info[OR_INFO_N_REP] = nrep;
    info[OR_INFO_N_OVERFLOW] = n_over;
    info[OR_INFO_N_PIECES] = nP;
    info[OR_INFO_N_RECEIVERS] = nN;
    info[OR_INFO_MAX_REP_PER_RANK] = max_rep;
    info[OR_INFO_N_REP_EXPERTS] = n_rep_experts;
    info[OR_INFO_N_REMOTE_PAIRS] = (int32_t)n_remote;
    info[OR_INFO_CASCADE_GUARD_STEPS] = n_guard;
    info[OR_INFO_CASCADE_GUARD_SLACK] = min_slack;

out:
    free(Hl); free(X); free(D); free(shed); free(keep); free(order); free(pieces);
    free(recv); free(PS); free(QS); free(nrep_on); free(rep_ord); free(hosts); free(gcount);
    free(src_count); free(src_seen);
    return rc;
}

/* --------------------------------------------------------- data steps --- */

/* The data steps' token (or element) loops carry OpenMP pragmas.  The
 * oracle proper is compiled without OpenMP, so they are single-threaded
 * loops; a second build with OpenMP, used only to time a multi-core CPU
 * baseline, runs the same loops over the host's cores.  Each iteration
 * writes its own outputs, so both builds compute identical results.
 * or_omp_threads(n) sets the thread count (n > 0) and returns the count in
 * use: always 1 without OpenMP. */
#ifdef _OPENMP
#include <omp.h>
int or_omp_threads(int n)
{
    if (n > 0) omp_set_num_threads(n);
    return omp_get_max_threads();
}
#else
int or_omp_threads(int n)
{
    (void)n;
    return 1;
}
#endif

/* Dispatch (zero-copy permute) [P1 core idea; P2 README]: the row of token t
 * is written, unchanged, into the buffer row dst_pos[t*K+k] for every k.
 * Tokens [t0, t1) only; buf is the [R, S*K, H] buffer as R*S*K rows. */
int or_dispatch(const or_config *c, const int32_t *dst_pos, const int32_t *info,
                const uint16_t *hidden, uint16_t *buf, int64_t t0, int64_t t1)
{
    if (info[OR_INFO_STATUS] & OR_ST_EXPERT_ID_RANGE) return OR_OK;
    const int64_t K = c->K, H = c->H;
#pragma omp parallel for schedule(static)
    for (int64_t t = t0; t < t1; ++t)
        for (int64_t k = 0; k < K; ++k) {
            int64_t d = dst_pos[t * K + k];
            for (int64_t h = 0; h < H; ++h) buf[d * H + h] = hidden[t * H + h];
        }
    return OR_OK;
}

/* Combine (weighted unpermute): out[t,h] = bf16(sum_k w[t,k] * y[dst_pos[t,k], h]),
 * the sum an fp32 fused multiply-add chain from 0 in k order, one rounding
 * to bf16 at the end. */
int or_combine(const or_config *c, const int32_t *dst_pos, const int32_t *info,
               const uint16_t *y, const float *w, uint16_t *out, int64_t t0, int64_t t1)
{
    if (info[OR_INFO_STATUS] & OR_ST_EXPERT_ID_RANGE) return OR_OK;
    const int64_t K = c->K, H = c->H;
#pragma omp parallel for schedule(static)
    for (int64_t t = t0; t < t1; ++t)
        for (int64_t h = 0; h < H; ++h) {
            float acc = 0.0f;
            for (int64_t k = 0; k < K; ++k) {
                int64_t d = dst_pos[t * K + k];
                acc = fmaf(w[t * K + k], bf16_to_f32(y[d * H + h]), acc);
            }
            out[t * H + h] = or_f32_to_bf16(acc);
        }
    return OR_OK;
}

/* Combine backward (the exact gradient of the combine above):
 *   dy_buf[dst_pos[t,k], h] = bf16(w[t,k] * dy[t,h])   (fp32 product)
 *   dw[t,k] = sum_h dy[t,h] * y[dst_pos[t,k], h]        (fp64 sum, one fp32 rounding)
 * With OR_FLAG_BWD_UNSCALED the dispatched rows are dy itself. */
int or_combine_backward(const or_config *c, const int32_t *dst_pos, const int32_t *info,
                        const uint16_t *dy, const float *w, const uint16_t *y,
                        uint16_t *dy_buf, float *dw, int64_t t0, int64_t t1)
{
    if (info[OR_INFO_STATUS] & OR_ST_EXPERT_ID_RANGE) return OR_OK;
    const int64_t K = c->K, H = c->H;
    const int unscaled = (c->flags & OR_FLAG_BWD_UNSCALED) != 0;
    for (int64_t t = t0; t < t1; ++t)
        for (int64_t k = 0; k < K; ++k) {
            int64_t p = t * K + k;
            int64_t d = dst_pos[p];
            double s = 0.0;
            for (int64_t h = 0; h < H; ++h) {
                float g = bf16_to_f32(dy[t * H + h]);
                dy_buf[d * H + h] = unscaled ? dy[t * H + h] : or_f32_to_bf16(w[p] * g);
                s += (double)g * (double)bf16_to_f32(y[d * H + h]);
            }
            dw[p] = (float)s;
        }
    return OR_OK;
}

/* Replica-gradient reduction [P1 explainer, memory tab, training branch]:
 * for every expert, in ascending host rank order, each prefetched replica
 * (ordinal b = slot - L < B) adds its fp32 gradient rows reduce_buf[r, b]
 * into home_grad[e] (one non-fused fp32 add per element per replica), and
 * the replica rows are then zeroed for the next microbatch.  Elements
 * [i0, i1) of each gradient only. */
int or_reduce_replica_grads(const or_config *c, const int32_t *host_ptr,
                            const int32_t *host_rank, const int32_t *host_slot,
                            const int32_t *info, float *reduce_buf, float *home_grad,
                            int64_t P, int64_t i0, int64_t i1)
{
    if (info[OR_INFO_STATUS] & OR_ST_EXPERT_ID_RANGE) return OR_OK;
    const int32_t E = c->E, L = c->E / c->R, B = c->B;
    for (int32_t e = 0; e < E; ++e) {
        for (int32_t h = host_ptr[e]; h < host_ptr[e + 1]; ++h) {
            int32_t r = host_rank[h], b = host_slot[h] - L;
            if (r == e / L) continue; /* the home copy */
            if (b < 0 || b >= B) continue; /* overflow replica: no reduce rows */
            float *src = reduce_buf + ((int64_t)r * B + b) * P;
            float *dst = home_grad + (int64_t)e * P;
#pragma omp parallel for schedule(static)
            for (int64_t i = i0; i < i1; ++i) dst[i] = dst[i] + src[i];
        }
    }
    for (int32_t e = 0; e < E; ++e)
        for (int32_t h = host_ptr[e]; h < host_ptr[e + 1]; ++h) {
            int32_t r = host_rank[h], b = host_slot[h] - L;
            if (r == e / L || b < 0 || b >= B) continue;
            float *src = reduce_buf + ((int64_t)r * B + b) * P;
#pragma omp parallel for schedule(static)
            for (int64_t i = i0; i < i1; ++i) src[i] = 0.0f;
        }
    return OR_OK;
}

/* Replica weight prefetch [P1 explainer, memory tab]: duplicated experts are
 * copied before expert compute into the rank's prefetch slots, rows [L, L+B)
 * of its [L+B, ...] weight pool (the page's [E, E+B) with E read as the
 * rank's L home experts).  pool[r][b][:] = weights[e][:] for every replica
 * of expert e on rank r with ordinal b = slot - L < B; overflow replicas are
 * not copied -- they read the home copy (inference read-through).
 * slot_wrow[r][s] names the weight row each used slot computes with, in the
 * concatenated row space [weights (E rows) | pool (R*B rows)]:
 *   home slot -> e;  prefetched replica -> E + r*B + b;  overflow -> e;
 * unused slots -> -1.  Elements [i0, i1) of each row are copied. */
int or_prefetch_replicas(const or_config *c, const int32_t *slot_expert, const int32_t *info,
                         const uint16_t *weights, uint16_t *pool, int32_t *slot_wrow,
                         int64_t P, int64_t i0, int64_t i1)
{
    const int32_t R = c->R, E = c->E, L = c->E / c->R, B = c->B;
    const int invalid = (info[OR_INFO_STATUS] & OR_ST_EXPERT_ID_RANGE) != 0;
    for (int32_t r = 0; r < R; ++r)
        for (int32_t s = 0; s < E; ++s) {
            int32_t e = invalid ? -1 : slot_expert[(int64_t)r * E + s];
            int32_t row = -1;
            if (e >= 0) {
                if (s < L) {
                    row = e;
                } else if (s - L < B) {
                    int32_t b = s - L;
                    row = E + r * B + b;
                    uint16_t *dst = pool + ((int64_t)r * B + b) * P;
                    const uint16_t *src = weights + (int64_t)e * P;
                    for (int64_t i = i0; i < i1; ++i) dst[i] = src[i];
                } else {
                    row = e; /* overflow: read through to the home copy */
                }
            }
            slot_wrow[(int64_t)r * E + s] = row;
        }
    return OR_OK;
}
