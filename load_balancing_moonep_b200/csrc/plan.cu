// Online redundant-expert planner (sm_100a).
//
// The MoonEP article ("Moonshot AI Open-Sources MoonEP: A Perfectly Balanced
// Expert Parallelism Library for MoE Training", "The core idea: dynamic
// redundant experts") fixes what the plan must achieve -- every rank gets
// exactly S*K token slots, by replicating a few experts online from the
// router output -- and calls the planner near-optimal without giving it.
// This file implements the water-filling plan described in moonep.h:
//
//   hist_plan_kernel  one CTA per token chunk: shared-memory histogram of the
//                     chunk (per-chunk counts kept for the assignment pass,
//                     totals accumulated with global atomics).  The CTA that
//                     finishes last (atomic ticket, no waiting) runs the whole
//                     planner as one 1024-thread block: loads, largest-first
//                     shedding, (value desc, index asc) orders by counting
//                     rank, prefix sums, water-filling as a parallel merge of
//                     the two prefix-sum partitions, slot tables and
//                     rank-ordered host intervals.
//   assign_kernel     one CTA per token chunk: the stable within-expert rank g
//                     of every (t, k) pair from the chunk prefix of the
//                     per-chunk counts, per-warp counters and warp match/popc,
//                     then the host interval holding g gives the buffer row.
//
// Nothing waits on another CTA, so no launch can hang.
#include "common.cuh"

namespace moonep {

struct PlanParams {
    Dims d;
    const int32_t *topk;
    moonep_plan_t p;
    int *ticket;
    int *status;
    int *gs;
    int *gp;
    int *cc;
    int *host_dst0;
};

constexpr int PLAN_THREADS = 1024;
constexpr int ASSIGN_THREADS = 512;
constexpr int ASSIGN_WARPS = ASSIGN_THREADS / 32;

// ints of dynamic shared memory used by the planner block
__host__ __device__ inline int plan_smem_ints(int E, int R)
{
    const int mx = E > R ? E : R;
    return 3 * E /*T, shed, flag2*/ + 2 * R /*X, D*/ + (mx + 1) /*scr*/ + 2 * E + (E + 1) /*pe pv PS*/ +
           2 * R + (R + 1) /*qr qv QS*/ + E + (E + 1) /*pilo segb*/ + 3 * R /*jlo nrr ridx*/ +
           E /*pof*/ + (R + 1) /*rbase*/ + (2 * E + R) /*offc*/ + (E + 1) /*hcnt*/ + 32 + 16;
}

__host__ __device__ inline int assign_smem_ints(int E, int R, int max_pairs)
{
    return E + ASSIGN_WARPS * E + 2 * max_pairs + (E + 1) + 2 * (2 * E + R) + 32;
}

// quota of the overlap of piece j with receiver i
__device__ __forceinline__ int seg_quota(const int *PS, const int *QS, int j, int i)
{
    return min(PS[j + 1], QS[i + 1]) - max(PS[j], QS[i]);
}

__device__ void write_empty_plan(const PlanParams &a, int status)
{
    const Dims &d = a.d;
    const int E = d.E, R = d.R, tid = threadIdx.x, nt = blockDim.x;
    for (int i = tid; i < R * E; i += nt) {
        a.p.slot_expert[i] = -1;
        a.p.slot_count[i] = 0;
    }
    for (int i = tid; i < R * (E + 1); i += nt) a.p.slot_offset[i] = 0;
    for (int i = tid; i < E + R; i += nt) {
        a.p.rep_expert[i] = -1;
        a.p.rep_rank[i] = -1;
        a.p.rep_slot[i] = -1;
        a.p.rep_quota[i] = 0;
    }
    for (int i = tid; i <= E; i += nt) a.p.host_ptr[i] = 0;
    for (int i = tid; i < 2 * E + R; i += nt) {
        a.p.host_rank[i] = -1;
        a.p.host_slot[i] = -1;
        a.p.host_start[i] = 0;
        a.p.host_quota[i] = 0;
    }
    for (int i = tid; i < E; i += nt) a.p.rep_home_list[i] = -1;
    for (int i = tid; i < MOONEP_INFO_LEN; i += nt) a.p.info[i] = (i == MOONEP_INFO_STATUS) ? status : 0;
}

// The planner, run by the last CTA of hist_plan_kernel (blockDim = 1024).
__device__ void plan_block(const PlanParams &a, int *sm)
{
    const Dims &d = a.d;
    const int E = d.E, R = d.R, L = d.L, C = d.C, B = d.B;
    const int tid = threadIdx.x, nt = blockDim.x;
    const int mx = E > R ? E : R;

    int *T = sm;
    int *shed = T + E;
    int *flag2 = shed + E;
    int *X = flag2 + E;
    int *D = X + R;
    int *scr = D + R;          // mx + 1
    int *pe = scr + mx + 1;    // E  pieces: expert, sorted
    int *pv = pe + E;          // E  pieces: shed, sorted
    int *PS = pv + E;          // E + 1
    int *qr = PS + E + 1;      // R  receivers: rank, sorted
    int *qv = qr + R;          // R  receivers: deficit, sorted
    int *QS = qv + R;          // R + 1
    int *pilo = QS + R + 1;    // E  first receiver of piece j
    int *segb = pilo + E;      // E + 1 first replica index of piece j
    int *jlo = segb + E + 1;   // R  first piece of receiver i
    int *nrr = jlo + R;        // R  replicas on rank r
    int *ridx = nrr + R;       // R  receiver index of rank r, -1 if none
    int *pof = ridx + R;       // E  piece index of expert e, -1 if none
    int *rbase = pof + E;      // R + 1 compact base of rank r's used slots
    int *offc = rbase + R + 1; // 2E + R slot offsets of used slots
    int *hcnt = offc + 2 * E + R;  // E + 1
    int *wsum = hcnt + E + 1;      // 32
    int *misc = wsum + 32;         // 16: 0 status 1 n_rep 2 n_over 3 max_rep 4 nP 5 nN 6 n_rep_experts

    for (int i = tid; i < 16; i += nt) misc[i] = 0;
    __syncthreads();

    // ---- totals from the histogram pass: exclusive prefix of the group
    // counts for the assignment pass; leave the group counts zeroed
    const int ng = d.ngroups;
    for (int e = tid; e < E; e += nt) {
        int run = 0;
        for (int g = 0; g < ng; ++g) {
            const int v = ld_cg(a.gs + (size_t)g * E + e);
            a.gs[(size_t)g * E + e] = 0;
            a.gp[(size_t)g * E + e] = run;
            run += v;
        }
        T[e] = run;
        a.p.expert_count[e] = run;
    }
    if (tid == 0) {
        misc[0] = ld_cg(a.status);
        *a.status = 0;
        *a.ticket = 0;
    }
    __syncthreads();
    const int status_in = misc[0];
    if (status_in & MOONEP_ST_EXPERT_ID_RANGE) {
        write_empty_plan(a, status_in);
        return;
    }

    // ---- home loads, excess X and deficit D per rank
    for (int r = tid; r < R; r += nt) {
        int h = 0;
        for (int j = 0; j < L; ++j) h += T[r * L + j];
        X[r] = h > C ? h - C : 0;
        D[r] = h < C ? C - h : 0;
    }
    __syncthreads();

    // ---- largest-first shedding: expert e's share of its rank's excess is
    // what remains after all larger (T desc, e asc) experts of the rank
    for (int e = tid; e < E; e += nt) {
        const int r = e / L, v = T[e];
        int s = 0;
        if (X[r] > 0) {
            int before = 0;
            for (int j = r * L; j < r * L + L; ++j) {
                const int tj = T[j];
                if (tj > v || (tj == v && j < e)) before += tj;
            }
            const int rem = X[r] - before;
            s = rem > 0 ? min(v, rem) : 0;
        }
        shed[e] = s;
    }
    __syncthreads();

    // ---- pieces, compacted then ordered by (shed desc, e asc)
    for (int e = tid; e < E; e += nt) scr[e] = shed[e] > 0;
    __syncthreads();
    const int nP = block_exscan(scr, E, wsum);
    int *tv = pilo, *ti = segb;  // temporaries
    for (int e = tid; e < E; e += nt)
        if (shed[e] > 0) {
            tv[scr[e]] = shed[e];
            ti[scr[e]] = e;
        }
    __syncthreads();
    for (int i = tid; i < nP; i += nt) {
        const int v = tv[i], id = ti[i];
        int pos = 0;
        for (int j = 0; j < nP; ++j) pos += (tv[j] > v) || (tv[j] == v && ti[j] < id);
        pe[pos] = id;
        pv[pos] = v;
    }
    __syncthreads();

    // ---- receivers, compacted then ordered by (deficit desc, r asc)
    for (int r = tid; r < R; r += nt) scr[r] = D[r] > 0;
    __syncthreads();
    const int nN = block_exscan(scr, R, wsum);
    int *uv = jlo, *ui = nrr;  // temporaries
    for (int r = tid; r < R; r += nt)
        if (D[r] > 0) {
            uv[scr[r]] = D[r];
            ui[scr[r]] = r;
        }
    __syncthreads();
    for (int i = tid; i < nN; i += nt) {
        const int v = uv[i], id = ui[i];
        int pos = 0;
        for (int j = 0; j < nN; ++j) pos += (uv[j] > v) || (uv[j] == v && ui[j] < id);
        qr[pos] = id;
        qv[pos] = v;
    }
    __syncthreads();

    // ---- prefix sums PS over pieces, QS over receivers
    for (int j = tid; j <= nP; j += nt) PS[j] = j < nP ? pv[j] : 0;
    for (int i = tid; i <= nN; i += nt) QS[i] = i < nN ? qv[i] : 0;
    for (int e = tid; e < E; e += nt) pof[e] = -1;
    for (int r = tid; r < R; r += nt) {
        nrr[r] = 0;
        ridx[r] = -1;
    }
    __syncthreads();
    block_exscan(PS, nP + 1, wsum);
    block_exscan(QS, nN + 1, wsum);

    // ---- water-filling: piece j overlaps receivers pilo[j] .. last; receiver
    // i overlaps pieces jlo[i] .. last.  Replicas are numbered in (j, i) order.
    for (int j = tid; j < nP; j += nt) {
        const int ilo = last_le(QS, nN, PS[j]);
        const int ihi = last_le(QS, nN, PS[j + 1] - 1);
        pilo[j] = ilo;
        segb[j] = ihi - ilo + 1;
        pof[pe[j]] = j;
    }
    if (tid == 0) segb[nP] = 0;
    for (int i = tid; i < nN; i += nt) {
        const int jl = last_le(PS, nP, QS[i]);
        const int jh = last_le(PS, nP, QS[i + 1] - 1);
        jlo[i] = jl;
        nrr[qr[i]] = jh - jl + 1;
        ridx[qr[i]] = i;
    }
    __syncthreads();
    const int n_rep = block_exscan(segb, nP + 1, wsum);

    // ---- replica list
    for (int q = tid; q < E + R; q += nt) {
        if (q < n_rep) {
            const int j = last_le(segb, nP, q);
            const int i = pilo[j] + (q - segb[j]);
            const int ord = j - jlo[i];
            a.p.rep_expert[q] = pe[j];
            a.p.rep_rank[q] = qr[i];
            a.p.rep_slot[q] = L + ord;
            a.p.rep_quota[q] = seg_quota(PS, QS, j, i);
            if (ord >= B) atomicAdd(&misc[2], 1);
        } else {
            a.p.rep_expert[q] = -1;
            a.p.rep_rank[q] = -1;
            a.p.rep_slot[q] = -1;
            a.p.rep_quota[q] = 0;
        }
    }

    // ---- slot tables: compact per-rank offsets of the used slots first
    for (int r = tid; r <= R; r += nt) rbase[r] = r < R ? L + nrr[r] : 0;
    __syncthreads();
    block_exscan(rbase, R + 1, wsum);
    for (int r = tid; r < R; r += nt) {
        const int used = L + nrr[r];
        int off = 0;
        for (int s = 0; s < used; ++s) {
            offc[rbase[r] + s] = off;
            int cnt;
            if (s < L) {
                cnt = T[r * L + s] - shed[r * L + s];
            } else {
                const int i = ridx[r];
                cnt = seg_quota(PS, QS, jlo[i] + (s - L), i);
            }
            off += cnt;
        }
        atomicMax(&misc[3], nrr[r]);
    }
    __syncthreads();
    for (int idx = tid; idx < R * E; idx += nt) {
        const int r = idx / E, s = idx - r * E, used = L + nrr[r];
        int ex = -1, cnt = 0;
        if (s < L) {
            ex = r * L + s;
            cnt = T[ex] - shed[ex];
        } else if (s < used) {
            const int i = ridx[r], j = jlo[i] + (s - L);
            ex = pe[j];
            cnt = seg_quota(PS, QS, j, i);
        }
        a.p.slot_expert[idx] = ex;
        a.p.slot_count[idx] = cnt;
    }
    for (int idx = tid; idx < R * (E + 1); idx += nt) {
        const int r = idx / (E + 1), s = idx - r * (E + 1), used = L + nrr[r];
        a.p.slot_offset[idx] = s < used ? offc[rbase[r] + s] : C;
    }

    // ---- host intervals: home + replicas of e, ascending rank
    for (int e = tid; e <= E; e += nt) {
        int c = 0;
        if (e < E) {
            c = 1;
            if (pof[e] >= 0) c += segb[pof[e] + 1] - segb[pof[e]];
        }
        hcnt[e] = c;
    }
    __syncthreads();
    block_exscan(hcnt, E + 1, wsum);
    for (int e = tid; e <= E; e += nt) a.p.host_ptr[e] = hcnt[e];
    for (int x = tid; x < 2 * E + R; x += nt) {
        if (x >= E + n_rep) {
            a.p.host_rank[x] = -1;
            a.p.host_slot[x] = -1;
            a.p.host_start[x] = 0;
            a.p.host_quota[x] = 0;
            continue;
        }
        int e, r0, slot, quota, j, pos;
        if (x < E) {
            e = x;
            r0 = e / L;
            slot = e - r0 * L;
            quota = T[e] - shed[e];
            j = pof[e];
            pos = 0;
        } else {
            const int q = x - E;
            j = last_le(segb, nP, q);
            const int i = pilo[j] + (q - segb[j]);
            e = pe[j];
            r0 = qr[i];
            slot = L + (j - jlo[i]);
            quota = seg_quota(PS, QS, j, i);
            pos = (e / L) < r0 ? 1 : 0;
        }
        if (j >= 0) {
            const int ns = segb[j + 1] - segb[j];
            for (int s = 0; s < ns; ++s) pos += qr[pilo[j] + s] < r0;
        }
        const int h = hcnt[e] + pos;
        a.p.host_rank[h] = r0;
        a.p.host_slot[h] = slot;
        a.p.host_quota[h] = quota;
    }
    __syncthreads();
    for (int e = tid; e < E; e += nt) {
        int st = 0;
        for (int h = hcnt[e]; h < hcnt[e + 1]; ++h) {
            const int r = a.p.host_rank[h], slot = a.p.host_slot[h];
            a.p.host_start[h] = st;
            a.host_dst0[h] = r * C + offc[rbase[r] + slot] - st;
            st += a.p.host_quota[h];
        }
    }

    // ---- experts with a prefetched replica (reduce work list)
    for (int e = tid; e < E; e += nt) {
        int f = 0;
        const int j = pof[e];
        if (j >= 0) {
            const int ns = segb[j + 1] - segb[j];
            for (int s = 0; s < ns; ++s)
                if (j - jlo[pilo[j] + s] < B) f = 1;
        }
        flag2[e] = f;
        scr[e] = f;
    }
    __syncthreads();
    const int n_rep_experts = block_exscan(scr, E, wsum);
    for (int e = tid; e < E; e += nt) {
        if (flag2[e]) a.p.rep_home_list[scr[e]] = e;
        if (e >= n_rep_experts) a.p.rep_home_list[e] = -1;
    }

    if (tid == 0) {
        const int n_over = misc[2];
        int st = 0;
        if (n_over > 0) {
            st |= MOONEP_ST_OVERFLOW;
            if (d.flags & MOONEP_FLAG_STRICT_BUDGET) st |= MOONEP_ST_STRICT_VIOLATION;
        }
        a.p.info[MOONEP_INFO_STATUS] = st;
        a.p.info[MOONEP_INFO_N_REP] = n_rep;
        a.p.info[MOONEP_INFO_N_OVERFLOW] = n_over;
        a.p.info[MOONEP_INFO_N_PIECES] = nP;
        a.p.info[MOONEP_INFO_N_RECEIVERS] = nN;
        a.p.info[MOONEP_INFO_MAX_REP_PER_RANK] = misc[3];
        a.p.info[MOONEP_INFO_N_REP_EXPERTS] = n_rep_experts;
        for (int i = MOONEP_INFO_N_REMOTE_PAIRS; i < MOONEP_INFO_LEN; ++i) a.p.info[i] = 0;
    }
}

__global__ void __launch_bounds__(PLAN_THREADS, 1) hist_plan_kernel(PlanParams a)
{
    extern __shared__ int sm[];
    __shared__ int s_last;
    const Dims &d = a.d;
    const int E = d.E, K = d.K, tid = threadIdx.x, nt = blockDim.x;
    const int lane = tid & 31, warp = tid >> 5;

    int *hist = sm;
    for (int e = tid; e < E; e += nt) hist[e] = 0;
    __syncthreads();

    const int chunk = blockIdx.x;
    const int t0 = chunk * d.chunk_tokens;
    const int t1 = min(t0 + d.chunk_tokens, d.tokens);
    const int p0 = t0 * K, p1 = t1 * K;
    int bad = 0;
    for (int base = p0 + warp * 32; base < p1; base += nt) {
        const int p = base + lane;
        const bool valid = p < p1;
        const int e = valid ? __ldg(a.topk + p) : -1;
        const bool ok = valid && e >= 0 && e < E;
        if (valid && !ok) bad = 1;
        const unsigned peers = __match_any_sync(FULL_MASK, ok ? e : E + lane);
        if (ok && lane == __ffs(peers) - 1) atomicAdd(&hist[e], __popc(peers));
    }
    bad = __syncthreads_or(bad);
    const int grp = chunk / CHUNK_GROUP;
    for (int e = tid; e < E; e += nt) {
        const int c = hist[e];
        a.cc[(size_t)chunk * E + e] = c;
        if (c) atomicAdd(a.gs + (size_t)grp * E + e, c);  // commutative: order-free
    }
    if (bad && tid == 0) atomicOr(a.status, MOONEP_ST_EXPERT_ID_RANGE);
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = (atomicAdd(a.ticket, 1) == (int)gridDim.x - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    plan_block(a, sm);
}

struct AssignParams {
    Dims d;
    const int32_t *topk;
    moonep_plan_t p;
    const int *cc;
    const int *gp;
    const int *host_dst0;
};

__global__ void __launch_bounds__(ASSIGN_THREADS) assign_kernel(AssignParams a)
{
    extern __shared__ int sm[];
    const Dims &d = a.d;
    const int E = d.E, K = d.K, R = d.R, C = d.C, S = d.S;
    const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31, warp = tid >> 5;
    const int chunk = blockIdx.x;
    const int t0 = chunk * d.chunk_tokens;
    const int t1 = min(t0 + d.chunk_tokens, d.tokens);
    const int p0 = t0 * K, n = (t1 - t0) * K;
    const int max_pairs = d.chunk_tokens * K;
    const int nh = 2 * E + R;

    const int status = a.p.info[MOONEP_INFO_STATUS];
    if (status & MOONEP_ST_EXPERT_ID_RANGE) {
        for (int i = tid; i < n; i += nt) {
            a.p.dst_pos[p0 + i] = -1;
            a.p.row_src[p0 + i] = -1;
        }
        return;
    }

    int *base = sm;                        // E
    int *cnt = base + E;                   // ASSIGN_WARPS * E
    int *ids = cnt + ASSIGN_WARPS * E;     // max_pairs
    int *lr = ids + max_pairs;             // max_pairs
    int *hptr = lr + max_pairs;            // E + 1
    int *hstart = hptr + E + 1;            // nh
    int *hdst = hstart + nh;               // nh
    int *red = hdst + nh;                  // 32

    for (int e = tid; e <= E; e += nt) hptr[e] = a.p.host_ptr[e];
    for (int h = tid; h < nh; h += nt) {
        hstart[h] = a.p.host_start[h];
        hdst[h] = a.host_dst0[h];
    }
    // pairs of each expert in earlier chunks: group prefix + earlier chunks
    // of this chunk's group (at most CHUNK_GROUP - 1 independent loads)
    {
        const int grp = chunk / CHUNK_GROUP, c0 = grp * CHUNK_GROUP;
        for (int e = tid; e < E; e += nt) {
            int s = __ldg(a.gp + (size_t)grp * E + e);
            int v[CHUNK_GROUP - 1];
#pragma unroll
            for (int j = 0; j < CHUNK_GROUP - 1; ++j)
                v[j] = (c0 + j < chunk) ? __ldg(a.cc + (size_t)(c0 + j) * E + e) : 0;
#pragma unroll
            for (int j = 0; j < CHUNK_GROUP - 1; ++j) s += v[j];
            base[e] = s;
        }
    }
    for (int i = tid; i < ASSIGN_WARPS * E; i += nt) cnt[i] = 0;
    for (int i = tid; i < n; i += nt) ids[i] = __ldg(a.topk + p0 + i);
    __syncthreads();

    // pass 1: rank of each pair among earlier pairs of its expert inside the
    // warp's contiguous sub-range
    const int per = (n + ASSIGN_WARPS - 1) / ASSIGN_WARPS;
    {
        const int beg = min(warp * per, n), end = min(beg + per, n);
        int *wc = cnt + warp * E;
        for (int b = beg; b < end; b += 32) {
            const int i = b + lane;
            const bool valid = i < end;
            const int e = valid ? ids[i] : -1;
            const bool ok = valid && e >= 0 && e < E;
            const unsigned peers = __match_any_sync(FULL_MASK, ok ? e : E + lane);
            int r0 = 0;
            if (ok) {
                r0 = wc[e];
                lr[i] = r0 + __popc(peers & lanemask_lt());
            }
            __syncwarp();
            if (ok && lane == __ffs(peers) - 1) wc[e] = r0 + __popc(peers);
            __syncwarp();
        }
    }
    __syncthreads();
    // warp bases: chunk prefix plus earlier warps of this chunk
    for (int e = tid; e < E; e += nt) {
        int run = base[e];
        for (int w = 0; w < ASSIGN_WARPS; ++w) {
            const int t = cnt[w * E + e];
            cnt[w * E + e] = run;
            run += t;
        }
    }
    __syncthreads();

    // pass 2: host interval holding g gives the buffer row
    int remote = 0;
    for (int i = tid; i < n; i += nt) {
        const int e = ids[i];
        if (e < 0 || e >= E) continue;
        const int w = i / per;
        const int g = cnt[w * E + e] + lr[i];
        int h = hptr[e];
        const int hend = hptr[e + 1];
        while (h + 1 < hend && hstart[h + 1] <= g) ++h;
        const int dst = hdst[h] + g;
        const int p = p0 + i;
        if (dst < 0 || dst >= R * C) {  // cannot happen for a consistent plan
            atomicOr(a.p.info + MOONEP_INFO_STATUS, MOONEP_ST_ROW_RANGE);
            a.p.dst_pos[p] = -1;
            continue;
        }
        a.p.dst_pos[p] = dst;
        a.p.row_src[dst] = p;
        remote += (dst / C) != ((p / K) / S);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) remote += __shfl_xor_sync(FULL_MASK, remote, o);
    if (lane == 0) red[warp] = remote;
    __syncthreads();
    if (tid == 0) {
        int s = 0;
        for (int w = 0; w < (nt >> 5); ++w) s += red[w];
        if (s) atomicAdd(a.p.info + MOONEP_INFO_N_REMOTE_PAIRS, s);
    }
}

// ---------------------------------------------------------------- launch

int launch_plan(const Dims &d, const int32_t *topk, const moonep_plan_t &p, void *ws, cudaStream_t st)
{
    const WsLayout wl = ws_layout(d);
    char *w = static_cast<char *>(ws);
    PlanParams a;
    a.d = d;
    a.topk = topk;
    a.p = p;
    a.ticket = reinterpret_cast<int *>(w + wl.ticket);
    a.status = reinterpret_cast<int *>(w + wl.status);
    a.gs = reinterpret_cast<int *>(w + wl.gs);
    a.gp = reinterpret_cast<int *>(w + wl.gp);
    a.cc = reinterpret_cast<int *>(w + wl.cc);
    a.host_dst0 = reinterpret_cast<int *>(w + wl.host_dst0);

    const size_t smem1 = sizeof(int) * (size_t)plan_smem_ints(d.E, d.R);
    if (cudaFuncSetAttribute(hist_plan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem1) !=
        cudaSuccess)
        return MOONEP_ERR_CUDA;
    hist_plan_kernel<<<d.nchunk, PLAN_THREADS, smem1, st>>>(a);
    if (cudaGetLastError() != cudaSuccess) return MOONEP_ERR_CUDA;

    AssignParams b;
    b.d = d;
    b.topk = topk;
    b.p = p;
    b.cc = a.cc;
    b.gp = a.gp;
    b.host_dst0 = a.host_dst0;
    const size_t smem2 = sizeof(int) * (size_t)assign_smem_ints(d.E, d.R, d.chunk_tokens * d.K);
    if (cudaFuncSetAttribute(assign_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem2) !=
        cudaSuccess)
        return MOONEP_ERR_CUDA;
    assign_kernel<<<d.nchunk, ASSIGN_THREADS, smem2, st>>>(b);
    if (cudaGetLastError() != cudaSuccess) return MOONEP_ERR_CUDA;
    return MOONEP_OK;
}

size_t plan_smem_bytes_max(const Dims &d)
{
    const size_t a = sizeof(int) * (size_t)plan_smem_ints(d.E, d.R);
    const size_t b = sizeof(int) * (size_t)assign_smem_ints(d.E, d.R, d.chunk_tokens * d.K);
    return a > b ? a : b;
}

}  // namespace moonep
