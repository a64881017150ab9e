// Online redundant-expert planner (sm_100a).
//
// The MoonEP article ("Moonshot AI Open-Sources MoonEP: A Perfectly Balanced
// Expert Parallelism Library for MoE Training", "The core idea: dynamic
// redundant experts") fixes what the plan must achieve -- every rank gets
// exactly S*K token slots, by replicating a few experts online from the
// router output -- and calls the planner near-optimal without giving it.
// This file implements the water-filling plan described in moonep.h, with no
// host synchronisation, in one of two ways that give the same plan:
//
//   plan_fused_kernel (the default) one CTA per SM and token chunk: every CTA
//                     counts its chunk, takes a ticket, sums the totals once
//                     every chunk's counts are in, runs the planner (plan_core)
//                     in its own shared memory and places its own pairs from
//                     its own host tables; ep_fused_kernel is its expert-
//                     parallel form, which needs no ticket (the gathered
//                     counts are complete before it starts).
//
// or, where the planner's shared memory does not fit beside a chunk, in two
// launches:
//
//   hist_plan_kernel  one CTA per token chunk stages the chunk's ids in
//                     shared memory and counts them with shared-memory
//                     atomics (a token's K experts are distinct, so few lanes
//                     of a warp collide), stores the counts for the second
//                     pass and adds them to the counts of its group of
//                     CHUNK_GROUP chunks with global atomics (sums:
//                     order-free, so deterministic).
//                     The CTA that finishes last (atomic ticket) runs the
//                     planner: expert totals from the group counts, loads,
//                     largest-first shedding, (value desc, index asc) orders
//                     by counting rank, prefix sums, water-filling as a
//                     parallel merge of the two prefix-sum partitions,
//                     per-rank slot lists, rank-ordered host intervals.  Its
//                     primitives are shuffle scans and warp ballots: on
//                     sm_100 a runtime-bound shared-memory loop costs a full
//                     load latency per step.  It writes the used slots of the
//                     padded [R][E] tables, the replica list, the host CSR
//                     and the reduce work list.
//   assign_kernel     one CTA per token chunk, launched with programmatic
//                     dependent launch, so every histogram CTA is resident
//                     before it starts.  On its ids alone (pass A) each warp
//                     walks a contiguous sub-range in (t, k) order ranking
//                     equal experts with ballots, which gives every pair its
//                     rank within the sub-range and every warp its counts.
//                     After a bounded wait for the READY mark that the last
//                     histogram CTA sets once all counts are in, a prefix
//                     over earlier groups, chunks and warps gives every warp
//                     its base -- all of this while the planner CTA runs.
//                     Only pass B waits for the grid: g = base + rank is the
//                     pair's rank among all pairs of its expert, and the host
//                     interval holding g gives the buffer row.  (The
//                     histogram CTAs write the tables' empty defaults
//                     before the planner writes over them, so no pass fills
//                     the unused rest afterwards.)
#include <atomic>
#include <climits>
#include <mutex>

#include "common.cuh"

namespace moonep {

constexpr int PLAN_THREADS = 512;
constexpr int ASSIGN_THREADS = 512;
constexpr int READY_SPIN_LIMIT = 1 << 16;  // x 100 ns sleeps: far beyond any histogram pass
constexpr int ASSIGN_WARPS = ASSIGN_THREADS / 32;
// pass A packs (rank in the warp's sub-range, expert) into one int
constexpr int PACK_BITS = 10, PACK_MASK = (1 << PACK_BITS) - 1;
static_assert((1 << PACK_BITS) >= MOONEP_MAX_E, "expert ids need more pack bits");

struct PlanParams {
    Dims d;
    const int32_t *topk;
    moonep_plan_t p;
    int *hdr;        // ticket, status, call sequence, counts-ready mark, arrivals
    int *gs;         // [2][ngroups][E] (expert parallelism: the gathered counts [R][E+1])
    int gs_stride;   // ints between the count rows of gs: E (E + 1 for the gathered counts)
    int gs_buf;      // ints of one of the two group-count buffers as the workspace lays them out
    int *cc;         // [nchunk][E]
    int *host_dst0;  // [2E+R]
    FastDiv fC, fL;  // divisions by C and L
    int spin_limit;  // iterations of each bounded wait of the assignment pass
    int cascade_cap; // the relay cascade guard's replica capacity: E + R - 1, or less in a test
};

// Where the planner's results go.  In the two-kernel path one planner CTA
// computes the plan, writes every table and the info block, keeps the host
// rows in the workspace for the assignment CTAs and sets the marks they wait
// for (legacy).  In the one-kernel path every CTA computes the same plan in
// its own shared memory and keeps the host tables there for its own pass B;
// one CTA (writer) stores the plan tables, and the info values are left in
// the planner's misc words for the CTA that finishes last.
struct PlanSink {
    bool legacy;
    bool writer;
    int *hptr, *hstart, *hdst;  // one-kernel path: [E+1], [2E+R], [2E+R] in shared memory
    int *hloc = nullptr, *hq = nullptr, *hr = nullptr;  // and, if set, each host's local pairs, quota and rank
};

// The planner's misc words (16 ints of shared memory): 0 status in, 2
// replicas over the budget, 3 most replicas on a rank, 4-5 the cascade
// guard's steps and least slack, 6 replicas, 7 pieces, 8 receivers, 9
// experts with a prefetched replica, 10 the plan's status bits.
enum { MISC_STATUS_IN = 0, MISC_N_OVER = 2, MISC_MAX_REP = 3, MISC_GUARD_STEPS = 4, MISC_GUARD_SLACK = 5,
       MISC_N_REP = 6, MISC_N_PIECES = 7, MISC_N_RECEIVERS = 8, MISC_N_REP_EXPERTS = 9, MISC_PLAN_STATUS = 10 };

// The bound of the assignment pass's two waits, for every later launch in
// the process (moonep_set_wait_limit).
static std::atomic<int> g_wait_limit{READY_SPIN_LIMIT};

int set_wait_limit(int iterations)
{
    return g_wait_limit.exchange(iterations < 0 ? READY_SPIN_LIMIT : iterations);
}

// The replica capacity the cascade's guard compares with, for every later
// launch (moonep_set_cascade_capacity): the plan's E + R - 1 by default.
static std::atomic<int> g_cascade_cap{0};

int set_cascade_capacity(int c)
{
    return g_cascade_cap.exchange(c > 0 ? c : 0);
}

static int cascade_cap_for(const Dims &d)
{
    const int full = d.E + d.R - 1, c = g_cascade_cap.load(std::memory_order_relaxed);
    return c > 0 && c < full ? c : full;
}

// ints of dynamic shared memory used by the planner block
__host__ __device__ inline int plan_smem_ints(int E, int R)
{
    const int nh = 2 * E + R;
    return 3 * E /*T shed keep*/ + 2 * R /*X D*/ + (E + R + 2) /*scr*/ + E /*pe*/ + R /*qr*/ +
           (E + R + 4) /*A: PS | QS*/ + E /*pilo*/ + (E + R + 4) /*Bs: segments | per rank*/ + R /*jlo*/ +
           E /*pof*/ + 3 * nh /*cexp ccnt cspare*/ + 3 * nh /*hr hs hq, then Z*/ +
           E /*flag*/ + 32 + 16;
}

__host__ __device__ inline int assign_smem_ints(int E, int R, int max_pairs)
{
    return ASSIGN_WARPS * E + max_pairs + (E + 1) + 2 * (2 * E + R) + 32;
}

// The relay cascade's shared memory.  Its step lists take a region of their
// own after the planner's (allocated only with MOONEP_FLAG_CASCADE); its host
// and per-expert tables reuse the planner's arrays from jlo to flag, which are
// dead once water-filling has been counted, when they fit there.
// lc: the list's capacity; a step never makes it longer than E + R - 1.
__host__ __device__ inline int cascade_list_cap(int E, int R) { return E + R; }
__host__ __device__ inline int plan_dead_ints(int E, int R) { return R + E + 6 * (2 * E + R) + E; }
__host__ __device__ inline int cascade_table_ints(int E, int R)
{
    return 4 * (2 * E + R) /*hosts*/ + E /*on_r*/ + 3 * R /*cnt closed hused*/ + E /*home slot offset*/ +
           2 * (E + 1) /*host counts, flag prefix*/ + E /*flag*/;
}
__host__ __device__ inline bool cascade_tables_in_dead(int E, int R)
{
    return cascade_table_ints(E, R) <= plan_dead_ints(E, R);
}
__host__ __device__ inline int cascade_smem_ints(int E, int R, int B)
{
    const int lc = cascade_list_cap(E, R);
    return 7 * lc /*le lr lq la, order, moved experts and quotas*/ + 4 * (B + 1) /*providers, relays*/ +
           (cascade_tables_in_dead(E, R) ? 0 : cascade_table_ints(E, R)) + 16;
}

__host__ __device__ inline int hist_smem_ints(int E, int R, int max_pairs, unsigned flags, int B)
{
    const int a = plan_smem_ints(E, R) + ((flags & MOONEP_FLAG_CASCADE) ? cascade_smem_ints(E, R, B) : 0);
    const int b = E + max_pairs;
    return a > b ? a : b;
}

// p[0] + p[stride] + ... + p[(n-1) stride], read through L2 with BATCH
// loads in flight at a time (one round trip for n <= BATCH)
template <int BATCH>
__device__ __forceinline__ int sum_strided(const int *p, int stride, int n)
{
    int s = 0;
    for (int g0 = 0; g0 < n; g0 += BATCH) {
        int v[BATCH];
#pragma unroll
        for (int j = 0; j < BATCH; ++j) v[j] = g0 + j < n ? ld_cg(p + (size_t)(g0 + j) * stride) : 0;
#pragma unroll
        for (int j = 0; j < BATCH; ++j) s += v[j];
    }
    return s;
}

__device__ __forceinline__ void pdl_launch_dependents()
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// ------------------------------------------------ relay cascade (slow path)

// The planner's tail when MOONEP_FLAG_CASCADE is set and water-filling left
// some rank with more than B replicas.  It keeps such ranks within B by the
// relay cascade: repeatedly, the rank with the most replicas (ties: lowest
// rank) among those over B and not yet closed keeps its B - m largest
// replicas (quota desc, list position asc) for the smallest m in 0..B whose
// providers can carry the rest; the providers are those kept replicas (each
// can grow by its expert's remaining home quota, unless that home is closed)
// and then m relay experts (home quota left, home not this rank, not closed
// and not yet a relay home, no replica on this rank), chosen by largest home
// quota, lowest expert first.  The moved quota is poured into the providers
// in that order, and the moved replicas are water-filled into the providers'
// home ranks: an amount on its own expert's home returns there, one on a
// rank already holding the expert joins that replica, any other is a new
// replica at the end of the list.  The rank is then closed; a step that
// could make the list longer than E + R - 1 live entries is not taken.
// The steps are inherently one after another and run on one warp over
// shared-memory lists (searches, sums and compaction by ballot and shuffle;
// the water-fill one provider at a time, through a per-expert tag of the
// entries on the provider's home rank); the tables are then rebuilt from the
// list by the whole CTA.  Every index the step loops use is bounded by the
// list capacity.
__device__ void cascade_tail(const PlanParams &a, int *cz, int *dead, int *keep, const int *pe, const int *qr,
                             const int *segb, const int *pilo, const int *PS, const int *QSr, int qbase,
                             int n_rep, int nP, int nN, int *misc, int *wsum, int seq, const PlanSink &sink)
{
    const Dims &d = a.d;
    const int E = d.E, R = d.R, L = d.L, C = d.C, B = d.B;
    const int tid = threadIdx.x;
    constexpr int nt = PLAN_THREADS;
    const int cap = a.cascade_cap, lc = cascade_list_cap(E, R), nh = 2 * E + R;
    int *le = cz, *lr = le + lc, *lq = lr + lc, *la = lq + lc;  // list: expert, rank, quota, alive
    int *ordx = la + lc;                                          // a rank's replicas in step order
    int *me = ordx + lc, *mq = me + lc;                           // their experts and quotas
    int *pve = mq + lc, *pvq = pve + B + 1, *pva = pvq + B + 1;   // providers: expert, kept entry or -1, amount
    int *rel = pva + B + 1;                                       // relays in pick order
    int *tb = cascade_tables_in_dead(E, R) ? dead : rel + B + 1;
    int *xr = tb, *xs = xr + nh, *xq = xs + nh, *xo = xq + nh;    // hosts: rank, slot, quota, slot offset
    int *on_r = xo + nh;                                          // E
    int *cnt = on_r + E, *closed = cnt + R, *hused = closed + R;  // R each
    int *hoff = hused + R;                                        // E: home slot offset
    int *hc = hoff + E, *fpre = hc + E + 1, *fl = fpre + E + 1;   // host counts, flag prefix, flags
    int *lo = ordx, *loff = me;                                   // after the steps: ordinal, slot offset per entry
    __shared__ int s_nl;

    // announce the slow path: the assignment CTAs stop spinning on the
    // plan-ready mark and wait for this grid to finish
    if (sink.legacy && tid == 0) st_release(a.hdr + WS_SLOW, seq + 1);
    const bool wr = sink.writer;
    // the water-filling list in creation order
#pragma unroll 1
    for (int q = tid; q < min(n_rep, lc); q += nt) {
        const int j = last_le(segb, nP, q);
        const int i = pilo[j] + (q - segb[j]);
        le[q] = pe[j];
        lr[q] = qr[i];
        lq[q] = min(PS[j + 1], QSr[i + 1] - qbase) - max(PS[j], QSr[i] - qbase);
        la[q] = 1;
    }
#pragma unroll 1
    for (int r = tid; r < R; r += nt) closed[r] = 0;
    __syncthreads();

    if (tid < 32) {
        // warp 0 runs the steps: every lane holds the same step state, lane 0
        // makes the scalar writes, searches and sums use the whole warp
        const int lane = tid;
        const unsigned lt = lanemask_lt();
        if (lane == 0) {  // every thread has passed the branch that read misc[3]: recount it
            misc[2] = 0;
            misc[3] = 0;
        }
        int nl = min(n_rep, lc);
        int n_guard = 0, min_slack = 0;  // steps that reached the capacity guard, its least slack
#pragma unroll 1
        for (int step = 0; step <= R; ++step) {
#pragma unroll 1
            for (int r = lane; r < R; r += 32) cnt[r] = 0;
            __syncwarp();
#pragma unroll 1
            for (int q = lane; q < nl; q += 32)
                if (la[q]) atomicAdd(&cnt[lr[q]], 1);
            __syncwarp();
            // the open rank over B with the most replicas, lowest rank on ties
            int bc = -1, br = R;
#pragma unroll 1
            for (int r = lane; r < R; r += 32) {
                const int c = cnt[r];
                if (!closed[r] && c > B && c > bc) {
                    bc = c;
                    br = r;
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const int oc = __shfl_xor_sync(FULL_MASK, bc, o), orr = __shfl_xor_sync(FULL_MASK, br, o);
                if (oc > bc || (oc == bc && orr < br)) {
                    bc = oc;
                    br = orr;
                }
            }
            if (bc < 0) break;
            const int rs = br;
            // its replicas: positions in list order (in mq), then ranked by
            // (quota desc, position asc) into ordx
#pragma unroll 1
            for (int e = lane; e < E; e += 32) on_r[e] = 0;
#pragma unroll 1
            for (int r = lane; r < R; r += 32) hused[r] = 0;
            int n = 0;
#pragma unroll 1
            for (int q0 = 0; q0 < nl; q0 += 32) {
                const int q = q0 + lane;
                const bool mine = q < nl && la[q] && lr[q] == rs;
                const unsigned b = __ballot_sync(FULL_MASK, mine);
                const int k = n + __popc(b & lt);
                if (mine && k < lc) mq[k] = q;
                n += __popc(b);
            }
            n = min(n, lc);
            __syncwarp();
#pragma unroll 1
            for (int k = lane; k < n; k += 32) {
                const int qk = mq[k], vk = lq[qk];
                int rk = 0;
#pragma unroll 1
                for (int j = 0; j < n; ++j) {
                    const int v = lq[mq[j]];
                    rk += (v > vk) || (v == vk && j < k);
                }
                ordx[rk] = qk;
                on_r[le[qk]] = 1;
            }
            __syncwarp();
            // the smallest m whose providers carry the moved quota
            int npick = 0, m_found = -1;
#pragma unroll 1
            for (int m = 0; m <= B; ++m) {
                while (npick < m) {  // next relay: largest home quota, lowest expert
                    int bk = 0, be = E;
#pragma unroll 1
                    for (int e = lane; e < E; e += 32) {
                        const int h = (int)fdiv((uint32_t)e, a.fL), kv = keep[e];
                        if (kv > bk && h != rs && !closed[h] && !on_r[e] && !hused[h]) {
                            bk = kv;
                            be = e;
                        }
                    }
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) {
                        const int ok = __shfl_xor_sync(FULL_MASK, bk, o), oe = __shfl_xor_sync(FULL_MASK, be, o);
                        if (ok > bk || (ok == bk && oe < be)) {
                            bk = ok;
                            be = oe;
                        }
                    }
                    if (be >= E) break;
                    if (lane == 0) {
                        rel[npick] = be;
                        hused[fdiv((uint32_t)be, a.fL)] = 1;
                    }
                    ++npick;
                    __syncwarp();
                }
                if (npick < m) break;  // fewer distinct relay homes than m
                long long Q = 0, room = 0;
#pragma unroll 1
                for (int k = B - m + lane; k < n; k += 32) Q += lq[ordx[k]];
#pragma unroll 1
                for (int k = lane; k < B - m; k += 32) {
                    const int e = le[ordx[k]];
                    room += closed[fdiv((uint32_t)e, a.fL)] ? 0 : keep[e];
                }
#pragma unroll 1
                for (int k = lane; k < m; k += 32) room += keep[rel[k]];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    Q += __shfl_xor_sync(FULL_MASK, Q, o);
                    room += __shfl_xor_sync(FULL_MASK, room, o);
                }
                if (room >= Q) {
                    m_found = m;
                    break;
                }
            }
            if (lane == 0) closed[rs] = 1;
            __syncwarp();
            if (m_found < 0) continue;
            // the step may add m + B - 1 live replicas: the list could
            // outgrow the plan's arrays when the slack is negative
            const int slack = cap - (nl + m_found + B - 1);
            if (n_guard == 0 || slack < min_slack) min_slack = slack;
            ++n_guard;
            if (slack < 0) continue;
            const int k0 = B - m_found;
            // the rank's replicas by step order: experts and quotas; a kept
            // replica's position once the moved ones are dropped
#pragma unroll 1
            for (int k = lane; k < n; k += 32) {
                const int q = ordx[k];
                me[k] = le[q];
                mq[k] = lq[q];
                if (k < k0) {
                    int before = 0;
#pragma unroll 1
                    for (int j = k0; j < n; ++j) before += ordx[j] < q;
                    pvq[k] = q - before;
                }
            }
            __syncwarp();
#pragma unroll 1
            for (int k = k0 + lane; k < n; k += 32) la[ordx[k]] = 0;  // the moved replicas leave this rank
            __syncwarp();
            // drop them, keeping list order (a destination never lies past its
            // source, so a chunk only writes where its reads are done)
            int w = 0;
#pragma unroll 1
            for (int q0 = 0; q0 < nl; q0 += 32) {
                const int q = q0 + lane;
                const bool alive = q < nl && la[q];
                int ve = 0, vr = 0, vq = 0;
                if (alive) {
                    ve = le[q];
                    vr = lr[q];
                    vq = lq[q];
                }
                const unsigned b = __ballot_sync(FULL_MASK, alive);
                __syncwarp();
                if (alive) {
                    const int dd = w + __popc(b & lt);
                    le[dd] = ve;
                    lr[dd] = vr;
                    lq[dd] = vq;
                    la[dd] = 1;
                }
                w += __popc(b);
                __syncwarp();
            }
            nl = w;
            // providers: the kept replicas, then the relays; pour the moved
            // quota into them (lane 0)
            int np = 0;
            if (lane == 0) {
                long long rem = 0;
#pragma unroll 1
                for (int k = k0; k < n; ++k) rem += mq[k];
#pragma unroll 1
                for (int k = 0; k < k0; ++k) pve[np++] = me[k];
#pragma unroll 1
                for (int k = 0; k < m_found; ++k) {
                    pve[np] = rel[k];
                    pvq[np] = -1;
                    ++np;
                }
#pragma unroll 1
                for (int k = 0; k < np; ++k) {
                    const int e = pve[k];
                    const long long capk = (pvq[k] >= 0 && closed[fdiv((uint32_t)e, a.fL)]) ? 0 : keep[e];
                    const int amt = (int)(capk < rem ? capk : rem);
                    pva[k] = amt;
                    rem -= amt;
                    if (amt <= 0) continue;
                    keep[e] -= amt;
                    if (pvq[k] >= 0) {
                        lq[pvq[k]] += amt;
                    } else if (nl < lc) {
                        le[nl] = e;
                        lr[nl] = rs;
                        lq[nl] = amt;
                        la[nl] = 1;
                        ++nl;
                    }
                }
            }
            np = __shfl_sync(FULL_MASK, np, 0);
            nl = __shfl_sync(FULL_MASK, nl, 0);
            __syncwarp();
            // water-fill the moved replicas into the providers' home ranks:
            // the moved quota [MS[i], MS[i+1]) of replica k0 + i meets
            // provider p's [PV[p], PV[p+1]); each overlap, in (p, i) order,
            // returns home, joins the replica of that expert already on the
            // home rank (found through a per-expert tag of the rank's
            // entries), or is appended
            const int nm = n - k0;
            int *MS = ordx, *PV = pvq, *tag = on_r;  // free by now: order, kept positions, relay marks
            {
                int run = 0;
#pragma unroll 1
                for (int b0 = 0; b0 < nm; b0 += 32) {
                    const int i = b0 + lane, v = i < nm ? mq[k0 + i] : 0;
                    int x = v;
#pragma unroll
                    for (int o = 1; o < 32; o <<= 1) {
                        const int y = __shfl_up_sync(FULL_MASK, x, o);
                        if (lane >= o) x += y;
                    }
                    if (i < nm) MS[i] = run + x - v;
                    run += __shfl_sync(FULL_MASK, x, 31);
                }
                if (lane == 0) MS[nm] = run;
                run = 0;
#pragma unroll 1
                for (int b0 = 0; b0 < np; b0 += 32) {
                    const int i = b0 + lane, v = i < np ? pva[i] : 0;
                    int x = v;
#pragma unroll
                    for (int o = 1; o < 32; o <<= 1) {
                        const int y = __shfl_up_sync(FULL_MASK, x, o);
                        if (lane >= o) x += y;
                    }
                    if (i < np) PV[i] = run + x - v;
                    run += __shfl_sync(FULL_MASK, x, 31);
                }
                if (lane == 0) PV[np] = run;
            }
#pragma unroll 1
            for (int e = lane; e < E; e += 32) tag[e] = -1;
            __syncwarp();
#pragma unroll 1
            for (int pi = 0; pi < np; ++pi) {
                const int lo = PV[pi], hi = PV[pi + 1];
                if (hi <= lo || nm <= 0) continue;
                const int h = (int)fdiv((uint32_t)pve[pi], a.fL);
                const int i_lo = warp_last_le(MS, nm, lo), i_hi = warp_last_le(MS, nm, hi - 1);
                const int nl0 = nl;
#pragma unroll 1
                for (int q = lane; q < nl0; q += 32)
                    if (lr[q] == h) tag[le[q]] = q;
                __syncwarp();
#pragma unroll 1
                for (int i0 = i_lo; i0 <= i_hi; i0 += 32) {
                    const int i = i0 + lane;
                    bool fresh = false;
                    int ek = 0, amt = 0;
                    if (i <= i_hi) {
                        ek = me[k0 + i];
                        amt = min(MS[i + 1], hi) - max(MS[i], lo);
                        if ((int)fdiv((uint32_t)ek, a.fL) == h) {
                            keep[ek] += amt;
                        } else {
                            const int t = tag[ek];
                            if (t >= 0) lq[t] += amt;
                            else fresh = true;
                        }
                    }
                    const unsigned b = __ballot_sync(FULL_MASK, fresh);
                    const int pos = nl + __popc(b & lt);
                    if (fresh && pos < lc) {
                        le[pos] = ek;
                        lr[pos] = h;
                        lq[pos] = amt;
                        la[pos] = 1;
                    }
                    nl = min(nl + __popc(b), lc);
                }
                __syncwarp();
#pragma unroll 1
                for (int q = lane; q < nl0; q += 32)
                    if (lr[q] == h) tag[le[q]] = -1;
                __syncwarp();
            }
        }
        if (lane == 0) {
            s_nl = nl;
            misc[4] = n_guard;
            misc[5] = min_slack;
        }
    }
    __syncthreads();
    const int nl = s_nl;

    // ordinals in list order, slot offsets and the used slots of every rank
    // (in the one-kernel path each rank's row is written by the CTA that owns
    // the rank, r mod gridDim.x, empty slots included)
#pragma unroll 1
    for (int r = tid; r < R; r += nt) {
        const bool own = sink.legacy ? wr : (int)(r % gridDim.x) == (int)blockIdx.x;
        int off = 0;
#pragma unroll 1
        for (int sl = 0; sl < L; ++sl) {
            const int e = r * L + sl;
            hoff[e] = off;
            if (own) {
                a.p.slot_expert[(size_t)r * E + sl] = e;
                a.p.slot_count[(size_t)r * E + sl] = keep[e];
                a.p.slot_offset[(size_t)r * (E + 1) + sl] = off;
            }
            off += keep[e];
        }
        int ord = 0;
#pragma unroll 1
        for (int q = 0; q < nl; ++q) {
            if (lr[q] != r) continue;
            lo[q] = ord;
            loff[q] = off;
            const int sl = min(L + ord, E - 1);
            if (own) {
                a.p.slot_expert[(size_t)r * E + sl] = le[q];
                a.p.slot_count[(size_t)r * E + sl] = lq[q];
                a.p.slot_offset[(size_t)r * (E + 1) + sl] = off;
            }
            off += lq[q];
            ++ord;
        }
        atomicMax(&misc[3], ord);
        cnt[r] = min(L + ord, E);  // used slots of rank r (cnt is free after the steps)
    }
    __syncthreads();
    if (!sink.legacy)
#pragma unroll 1
        for (int r = blockIdx.x; r < R; r += gridDim.x)
#pragma unroll 1
            for (int sl = cnt[r] + tid; sl <= E; sl += nt) {
                if (sl < E) {
                    a.p.slot_expert[(size_t)r * E + sl] = -1;
                    a.p.slot_count[(size_t)r * E + sl] = 0;
                }
                a.p.slot_offset[(size_t)r * (E + 1) + sl] = C;
            }
#pragma unroll 1
    for (int q = tid; q < nl; q += nt) {
        if (wr) {
            a.p.rep_expert[q] = le[q];
            a.p.rep_rank[q] = lr[q];
            a.p.rep_slot[q] = L + lo[q];
            a.p.rep_quota[q] = lq[q];
        }
        if (lo[q] >= B) atomicAdd(&misc[2], 1);
    }
    if (wr && !sink.legacy)  // the one-kernel path writes no defaults beforehand
#pragma unroll 1
        for (int q = nl + tid; q < E + R; q += nt) {
            a.p.rep_expert[q] = -1;
            a.p.rep_rank[q] = -1;
            a.p.rep_slot[q] = -1;
            a.p.rep_quota[q] = 0;
        }
    // hosts per expert (home + its replicas) and the work-list flags
#pragma unroll 1
    for (int e = tid; e < E; e += nt) {
        int c = 1, f = 0;
#pragma unroll 1
        for (int q = 0; q < nl; ++q)
            if (le[q] == e) {
                ++c;
                f |= lo[q] < B;
            }
        hc[e] = c;
        fl[e] = f;
        fpre[e] = f;
    }
    if (tid == 0) {
        hc[E] = 0;
        fpre[E] = 0;
    }
    __syncthreads();
    block_exscan(hc, E + 1, wsum);
    const int n_rep_experts = block_exscan(fpre, E + 1, wsum);
#pragma unroll 1
    for (int e = tid; e <= E; e += nt) {
        if (wr) a.p.host_ptr[e] = hc[e];
        if (!sink.legacy) sink.hptr[e] = hc[e];
    }
    if (wr && !sink.legacy)
#pragma unroll 1
        for (int h = hc[E] + tid; h < nh; h += nt) {
            a.p.host_rank[h] = -1;
            a.p.host_slot[h] = -1;
            a.p.host_start[h] = 0;
            a.p.host_quota[h] = 0;
            a.p.host_local[h] = 0;
        }
    if (wr)
#pragma unroll 1
        for (int e = tid; e < E; e += nt) {
            if (fl[e]) a.p.rep_home_list[fpre[e]] = e;
            if (e >= n_rep_experts) a.p.rep_home_list[e] = -1;
        }
    // host intervals: the hosts of e in ascending rank, starts in that order
#pragma unroll 1
    for (int e = tid; e < E; e += nt) {
        const int b0 = hc[e], b1 = min(hc[e + 1], nh);
        int k = b0;
        if (k < b1) {
            xr[k] = e / L;
            xs[k] = e - (e / L) * L;
            xq[k] = keep[e];
            xo[k] = hoff[e];
            ++k;
        }
#pragma unroll 1
        for (int q = 0; q < nl && k < b1; ++q)
            if (le[q] == e) {
                xr[k] = lr[q];
                xs[k] = L + lo[q];
                xq[k] = lq[q];
                xo[k] = loff[q];
                ++k;
            }
#pragma unroll 1
        for (int x = b0 + 1; x < k; ++x) {  // insertion sort by rank (ranks are distinct)
            const int vr = xr[x], vs = xs[x], vq = xq[x], vo = xo[x];
            int y = x;
            while (y > b0 && xr[y - 1] > vr) {
                xr[y] = xr[y - 1];
                xs[y] = xs[y - 1];
                xq[y] = xq[y - 1];
                xo[y] = xo[y - 1];
                --y;
            }
            xr[y] = vr;
            xs[y] = vs;
            xq[y] = vq;
            xo[y] = vo;
        }
        int st = 0;
#pragma unroll 1
        for (int h = b0; h < k; ++h) {
            // the locality flag as in the water-filling tail
            const int loc = (d.flags & MOONEP_FLAG_LOCALITY)
                                ? min(xq[h], ld_cg(a.gs + (size_t)xr[h] * a.gs_stride + e))
                                : 0;
            if (wr) {
                a.p.host_rank[h] = xr[h];
                a.p.host_slot[h] = xs[h];
                a.p.host_quota[h] = xq[h];
                a.p.host_start[h] = st;
                a.p.host_local[h] = loc;
            }
            const int dst0 = xr[h] * C + xo[h] - st;
            if (sink.legacy) {
                a.host_dst0[h] = dst0;
            } else {
                sink.hstart[h] = st;
                sink.hdst[h] = dst0;
                if (sink.hloc) {
                    sink.hloc[h] = loc;
                    sink.hq[h] = xq[h];
                    sink.hr[h] = xr[h];
                }
            }
            st += xq[h] - loc;
        }
    }
    __syncthreads();
    if (tid == 0) {
        const int n_over = misc[2];
        int st = 0;
        if (n_over > 0) {
            st |= MOONEP_ST_OVERFLOW;
            if (d.flags & MOONEP_FLAG_STRICT_BUDGET) st |= MOONEP_ST_STRICT_VIOLATION;
        }
        misc[MISC_N_REP] = nl;
        misc[MISC_N_PIECES] = nP;
        misc[MISC_N_RECEIVERS] = nN;
        misc[MISC_N_REP_EXPERTS] = n_rep_experts;
        misc[MISC_PLAN_STATUS] = st;
        if (sink.legacy) {
            a.p.info[MOONEP_INFO_STATUS] = st;
            a.p.info[MOONEP_INFO_N_REP] = nl;
            a.p.info[MOONEP_INFO_N_OVERFLOW] = n_over;
            a.p.info[MOONEP_INFO_N_PIECES] = nP;
            a.p.info[MOONEP_INFO_N_RECEIVERS] = nN;
            a.p.info[MOONEP_INFO_MAX_REP_PER_RANK] = misc[3];
            a.p.info[MOONEP_INFO_N_REP_EXPERTS] = n_rep_experts;
#pragma unroll 1
            for (int i = MOONEP_INFO_N_REMOTE_PAIRS; i < MOONEP_INFO_LEN; ++i) a.p.info[i] = 0;
            a.p.info[MOONEP_INFO_CASCADE_GUARD_STEPS] = misc[4];
            a.p.info[MOONEP_INFO_CASCADE_GUARD_SLACK] = misc[5];
        }
    }
    // every thread's plan writes precede the plan-ready mark
    __syncthreads();
    if (sink.legacy && tid == 0) {
        __threadfence();
        st_release(a.hdr + WS_PLANNED, seq + 1);
    }
}

// ------------------------------------------------------------- planner CTA

// The planner's shared-memory layout, from the base sm (plan_smem_ints(E, R)
// ints): the expert totals T come first, the misc words last.
__device__ __forceinline__ int *plan_misc(int *sm, int E, int R) { return sm + plan_smem_ints(E, R) - 16; }

__device__ void plan_core(const PlanParams &a, int *sm, int seq, const PlanSink &sink);

// The two-kernel path's planner CTA: the expert totals from this call's
// group counts, the checks that empty the plan, then the plan itself.
__device__ void plan_block(const PlanParams &a, int *sm, int seq)
{
    const int parity = seq & 1;
    const Dims &d = a.d;
    const int E = d.E, R = d.R;
    const int tid = threadIdx.x;
    constexpr int nt = PLAN_THREADS;
    const int lane = tid & 31, warp = tid >> 5;
    constexpr int nwarp = PLAN_THREADS / 32;
    int *T = sm;
    int *misc = plan_misc(sm, E, R);

    __shared__ unsigned s_part[2][32];
    // every other CTA has arrived: take the status (the load is issued here
    // and waited for after the totals' loads) and reset the header
    int st_hdr = 0;
    if (tid == 0) st_hdr = ld_cg(a.hdr + WS_STATUS);
    // ---- totals: the sum of this call's group counts (one atomic sum per
    // chunk and expert lands in a group of CHUNK_GROUP chunks, so no address
    // takes more than CHUNK_GROUP atomics; per-expert totals accumulated
    // by every CTA serialised some 300 atomics per address)
    static_assert(MOONEP_MAX_E <= 2 * PLAN_THREADS, "at most two experts per planner thread");
    unsigned part = 0;  // <= 2 values < 2^31 each (negative ones are flagged)
    int negative = 0;
    {
        const int *gsb = a.gs + (size_t)parity * d.ngroups * a.gs_stride;
        for (int e = tid; e < E; e += nt) {
            const int v = sum_strided<32>(gsb + e, a.gs_stride, d.ngroups);
            T[e] = v;
            a.p.expert_count[e] = v;
            negative |= v < 0;
            part += (unsigned)v;
        }
    }
    if (tid == 0) {
        misc[MISC_STATUS_IN] = st_hdr;
        a.hdr[WS_STATUS] = 0;
        a.hdr[WS_TICKET] = 0;
    }
    // exact 64-bit total from 16-bit halves, each warp sum by one reduction
    {
        const unsigned lo = __reduce_add_sync(FULL_MASK, part & 0xffffu);
        const unsigned hi = __reduce_add_sync(FULL_MASK, part >> 16);
        if (lane == 0) {
            s_part[0][warp] = lo;
            s_part[1][warp] = hi;
        }
    }
    negative = __syncthreads_or(negative);
    int status_in = misc[MISC_STATUS_IN];
    long long total;
    {
        const unsigned lo = __reduce_add_sync(FULL_MASK, lane < nwarp ? s_part[0][lane] : 0u);
        const unsigned hi = __reduce_add_sync(FULL_MASK, lane < nwarp ? s_part[1][lane] : 0u);
        total = ((long long)hi << 16) + (long long)lo;
    }
    // with every id valid the totals must be non-negative and add up to the
    // number of pairs; anything else means the workspace was not zeroed
    if (!(status_in & MOONEP_ST_EXPERT_ID_RANGE) && (negative || total != (long long)d.pairs))
        status_in |= MOONEP_ST_WORKSPACE;
    if (status_in & ST_EMPTY_PLAN) {
        if (tid == 0) {
            a.p.info[MOONEP_INFO_STATUS] = status_in;
            for (int i = 1; i < MOONEP_INFO_LEN; ++i) a.p.info[i] = 0;
            __threadfence();
            st_release(a.hdr + WS_PLANNED, seq + 1);
        }
        return;  // the assignment pass writes the empty tables
    }
    __syncthreads();  // misc[0] read by every thread before plan_core clears it
    plan_core(a, sm, seq, PlanSink{true, true, nullptr, nullptr, nullptr});
}

// The plan from the expert totals T = sm[0..E) (every id valid, the totals
// adding up to the pairs), by the whole CTA: loads, shedding, orders,
// water-filling, slot lists and host intervals, or the relay cascade.
// Its loops (and the cascade's) are kept rolled: the steps run one after
// another, each on data already in shared memory, and the unrolled code did
// not fit the instruction caches -- after a kernel that streams through L2,
// every step then waited on instruction fetch from memory.
__device__ void plan_core(const PlanParams &a, int *sm, int seq, const PlanSink &sink)
{
    const Dims &d = a.d;
    const int E = d.E, R = d.R, L = d.L, C = d.C, B = d.B;
    // PLAN_THREADS threads, a compile-time stride for every loop below
    const int tid = threadIdx.x;
    constexpr int nt = PLAN_THREADS;
    const int lane = tid & 31, warp = tid >> 5;
    constexpr int nwarp = PLAN_THREADS / 32;
    const int nh = 2 * E + R;
    const bool wr = sink.writer;

    int *T = sm;
    int *shed = T + E;
    int *keep = shed + E;
    int *X = keep + E;
    int *D = X + R;
    int *scr = D + R;              // E + R + 2
    int *pe = scr + E + R + 2;     // E   pieces: expert, sorted
    int *qr = pe + E;              // R   receivers: rank, sorted
    int *A = qr + R;               // E + R + 4: sorted sizes, then PS (nP+1) and QS (nN+1)
    int *pilo = A + E + R + 4;     // E   first receiver of piece j
    int *Bs = pilo + E;            // E + R + 4: segments per piece (nP+1) | replicas per rank (R+1)
    int *jlo = Bs + E + R + 4;     // R   first piece of receiver i
    int *pof = jlo + R;            // E   piece index of expert e, -1 if none
    int *cexp = pof + E;           // nh  compact used slots: expert
    int *ccnt = cexp + nh;         // nh  rows
    int *cspare = ccnt + nh;       // nh  receiver ids while sorting, then the rank of each used slot
    int *hr = cspare + nh;         // nh  piece rows, while sorting
    int *hs = hr + nh;             // nh  piece experts, while sorting
    int *hq = hs + nh;             // nh  receiver deficits, while sorting
    int *flag = hq + nh;           // E
    int *wsum = flag + E;          // 32
    int *misc = wsum + 32;         // 16 (MISC_*)
#pragma unroll 1
    for (int i = tid; i < 16; i += nt) misc[i] = 0;

    // ---- home loads, excess X and deficit D per rank
#pragma unroll 1
    for (int r = tid; r < R; r += nt) {
        int h = 0;
#pragma unroll 4
        for (int j = 0; j < L; ++j) h += T[r * L + j];
        X[r] = h > C ? h - C : 0;
        D[r] = h < C ? C - h : 0;
    }
    __syncthreads();

    // ---- largest-first shedding: expert e sheds what remains of its rank's
    // excess after all larger (T desc, e asc) experts of the rank
#pragma unroll 1
    for (int e = tid; e < E; e += nt) {
        const int r = (int)fdiv((uint32_t)e, a.fL), v = T[e];
        int s = 0;
        if (X[r] > 0) {
            int before = 0;
#pragma unroll 4
            for (int j = r * L; j < r * L + L; ++j) {
                const int tj = T[j];
                if (tj > v || (tj == v && j < e)) before += tj;
            }
            const int rem = X[r] - before;
            s = rem > 0 ? min(v, rem) : 0;
        }
        shed[e] = s;
        keep[e] = v - s;
        scr[e] = s > 0;
        pof[e] = -1;
    }
#pragma unroll 1
    for (int r = tid; r < R; r += nt) scr[E + r] = D[r] > 0;
    __syncthreads();

    // ---- compact pieces and receivers with one scan over [E experts | R ranks]
    const int nPN = block_exscan(scr, E + R, wsum);
    const int nP = scr[E];
    const int nN = nPN - nP;
#pragma unroll 1
    for (int e = tid; e < E; e += nt)
        if (shed[e] > 0) {
            hr[scr[e]] = shed[e];
            hs[scr[e]] = e;
        }
#pragma unroll 1
    for (int r = tid; r < R; r += nt)
        if (D[r] > 0) {
            hq[scr[E + r] - nP] = D[r];
            cspare[scr[E + r] - nP] = r;
        }
    __syncthreads();
    // counting-rank sorts, one warp per element: pieces by (shed desc,
    // e asc), receivers by (D desc, r asc); an element's position is the
    // number of entries ordered before it, counted 32 at a time by ballot
#pragma unroll 1
    for (int x = warp; x < nP + nN; x += nwarp) {
        const bool piece = x < nP;
        const int m = piece ? nP : nN, xi = piece ? x : x - nP;
        const int *val = piece ? hr : hq, *key = piece ? hs : cspare;
        const int v = val[xi], id = key[xi];
        int pos = 0;
#pragma unroll 4
        for (int j0 = 0; j0 < m; j0 += 32) {
            const int j = j0 + lane;
            bool before = false;
            if (j < m) {
                const int vj = val[j];
                before = vj > v || (vj == v && key[j] < id);
            }
            pos += __popc(__ballot_sync(FULL_MASK, before));
        }
        if (lane == 0) {  // A = [sorted piece sizes, 0, sorted deficits, 0]
            if (piece) {
                pe[pos] = id;
                A[pos] = v;
            } else {
                qr[pos] = id;
                A[nP + 1 + pos] = v;
            }
        }
    }
    if (tid == 0) {
        A[nP] = 0;
        A[nP + nN + 1] = 0;
    }
    int *segb = Bs;          // nP + 1: replicas per piece, then their prefix
    int *rpr = Bs + nP + 1;  // R + 1: replicas per rank, then prefix + n_rep
#pragma unroll 1
    for (int r = tid; r <= R; r += nt) rpr[r] = 0;
    __syncthreads();

    // ---- prefix sums: A scanned gives PS = A[0..nP] and QS[i] =
    // A[nP+1+i] - qbase, qbase being the pieces' total
    block_exscan(A, nP + nN + 2, wsum);
    const int *PS = A;
    const int *QSr = A + nP + 1;
    const int qbase = QSr[0];
    auto seg_q = [&](int j, int i) {  // rows of the overlap of piece j and receiver i
        return min(PS[j + 1], QSr[i + 1] - qbase) - max(PS[j], QSr[i] - qbase);
    };

    // ---- water-filling: piece j meets receivers pilo[j].. ; receiver i meets
    // pieces jlo[i].. ; replicas are numbered in (j, i) order
    // (one warp per piece or receiver, searching by ballot)
#pragma unroll 1
    for (int x = warp; x < nP + nN; x += nwarp) {
        if (x < nP) {
            const int j = x;
            const int ilo = warp_last_le(QSr, nN, PS[j] + qbase);
            const int ihi = warp_last_le(QSr, nN, PS[j + 1] - 1 + qbase);
            if (lane == 0) {
                pilo[j] = ilo;
                segb[j] = ihi - ilo + 1;
                pof[pe[j]] = j;
            }
        } else {
            const int i = x - nP;
            const int jl = warp_last_le(PS, nP, QSr[i] - qbase);
            const int jh = warp_last_le(PS, nP, QSr[i + 1] - 1 - qbase);
            if (lane == 0) {
                const int r = qr[i];
                jlo[i] = jl;
                rpr[r] = jh - jl + 1;
                atomicMax(&misc[3], jh - jl + 1);  // read after later barriers
            }
        }
    }
    if (tid == 0) segb[nP] = 0;
    __syncthreads();
    // one scan over [replicas per piece | replicas per rank]
    block_exscan(Bs, nP + 1 + R + 1, wsum);
    const int n_rep = Bs[nP];
    // over the budget with the cascade asked for: the slow path plans the rest
    if ((d.flags & MOONEP_FLAG_CASCADE) && B > 0 && misc[3] > B) {
        cascade_tail(a, sm + plan_smem_ints(E, R), jlo, keep, pe, qr, segb, pilo, PS, QSr, qbase, n_rep, nP, nN,
                     misc, wsum, seq, sink);
        return;
    }
    auto rank_base = [&](int r) { return r * L + rpr[r] - n_rep; };  // first compact slot of rank r

    // ---- replica list (creation order), the compact used-slot lists and
    // the per-expert host counts, all into one array Z for one scan:
    //   Z = [rows of each used slot (E + n_rep) | hosts per expert (E) | 0 |
    //        prefetched-replica flag per expert (E) | 0]
    // Rank r's used slots sit at rank_base(r) .. (home slots, then replicas).
    int *Z = hr;     // 4E + R + 2 <= 3 nh ints, free after the sort
    const int zh = E + n_rep, zf = zh + E + 1, nz = zf + E + 1;
#pragma unroll 1
    for (int q = tid; q < n_rep; q += nt) {
        const int j = last_le(segb, nP, q);
        const int i = pilo[j] + (q - segb[j]);
        const int ord = j - jlo[i];
        const int r = qr[i];
        const int quota = seg_q(j, i);
        if (wr) {
            a.p.rep_expert[q] = pe[j];
            a.p.rep_rank[q] = r;
            a.p.rep_slot[q] = L + ord;
            a.p.rep_quota[q] = quota;
        }
        const int cs = rank_base(r) + L + ord;
        cexp[cs] = pe[j];
        ccnt[cs] = quota;
        Z[cs] = quota;
        cspare[cs] = r;
        if (ord >= B) atomicAdd(&misc[2], 1);
    }
#pragma unroll 1
    for (int e = tid; e < E; e += nt) {
        const int r = (int)fdiv((uint32_t)e, a.fL);
        const int cs = rank_base(r) + (e - r * L);
        cexp[cs] = e;
        ccnt[cs] = keep[e];
        Z[cs] = keep[e];
        cspare[cs] = r;
        // hosts: home + one per replica; flag: a replica within the budget
        int c = 1, f = 0;
        const int j = pof[e];
        if (j >= 0) {
            const int ns = segb[j + 1] - segb[j], i0 = pilo[j];
            c += ns;
#pragma unroll 1
            for (int s = 0; s < ns; ++s)
                if (j - jlo[i0 + s] < B) {
                    f = 1;
                    break;
                }
        }
        Z[zh + e] = c;
        Z[zf + e] = f;
        flag[e] = f;
    }
    if (tid == 0) {
        Z[zh + E] = 0;
        Z[zf + E] = 0;
    }
    __syncthreads();
    block_exscan(Z, nz, wsum);
    // slot offset = prefix minus that of the rank's first slot; host_ptr[e]
    // and the work-list position likewise relative to their part's start
    const int zh0 = Z[zh], zf0 = Z[zf];
    const int n_hosts = E + n_rep;                  // == Z[zh + E] - zh0
    const int n_rep_experts = Z[zf + E] - zf0;
    auto hptr = [&](int e) { return Z[zh + e] - zh0; };
    // ---- host intervals first: they are all the assignment CTAs wait for.
    // The hosts of e in ascending rank; a host's start is the rows of the
    // hosts of e on lower ranks.
    // With MOONEP_FLAG_LOCALITY (expert parallelism, where the count rows are
    // the ranks' own counts) a host first takes min(quota, its rank's pairs
    // of e), and its start is in the order of the pairs left over.
    const bool locality = (d.flags & MOONEP_FLAG_LOCALITY) != 0;
    auto own_pairs = [&](int r, int e) { return ld_cg(a.gs + (size_t)r * a.gs_stride + e); };
    // host h of e: rank r0, slot, quota, start st, local pairs loc
    auto put_host = [&](int e, int h, int r0, int slot, int quota, int st, int loc) {
        const int b0 = rank_base(r0);
        if (wr) {
            a.p.host_rank[h] = r0;
            a.p.host_slot[h] = slot;
            a.p.host_quota[h] = quota;
            a.p.host_start[h] = st;
            a.p.host_local[h] = loc;
        }
        const int dst0 = r0 * C + Z[b0 + slot] - Z[b0] - st;
        if (sink.legacy) {
            a.host_dst0[h] = dst0;
        } else {
            sink.hstart[h] = st;
            sink.hdst[h] = dst0;
            if (sink.hloc) {
                sink.hloc[h] = loc;
                sink.hq[h] = quota;
                sink.hr[h] = r0;
            }
        }
    };
    // an expert with no replica: its home is its one host, at start 0
#pragma unroll 1
    for (int e = tid; e < E; e += nt) {
        if (pof[e] >= 0) continue;
        const int r0 = (int)fdiv((uint32_t)e, a.fL);
        put_host(e, hptr(e), r0, e - r0 * L, keep[e], 0, locality ? min(keep[e], own_pairs(r0, e)) : 0);
    }
    // a replicated expert (piece j): one warp, its hosts (the home, then the
    // piece's receivers) as lanes, 32 at a time; a host's position and start
    // are the count and the quota sum of the expert's hosts on lower ranks,
    // broadcast 32 at a time by shuffles (a hot expert has tens of hosts; one
    // thread per host walking all of them took 6 µs at the decode shape)
    auto host_of_piece = [&](int j, int e, int home, int k, int &r, int &q) {
        if (k == 0) {
            r = home;
            q = keep[e];
        } else {
            const int i = pilo[j] + k - 1;
            r = qr[i];
            q = seg_q(j, i);
        }
    };
#pragma unroll 1
    for (int j = warp; j < nP; j += nwarp) {
        const int e = pe[j], home = (int)fdiv((uint32_t)e, a.fL);
        const int nhost = segb[j + 1] - segb[j] + 1;
#pragma unroll 1
        for (int k0 = 0; k0 < nhost; k0 += 32) {
            const int k = k0 + lane;
            int rk = 0, qk = 0;
            if (k < nhost) host_of_piece(j, e, home, k, rk, qk);
            int pos = 0, st = 0, locsum = 0;
#pragma unroll 1
            for (int m0 = 0; m0 < nhost; m0 += 32) {
                const int m = m0 + lane;
                int rm = INT_MAX, qm = 0, lm = 0;
                if (m < nhost) {
                    host_of_piece(j, e, home, m, rm, qm);
                    if (locality) lm = min(qm, own_pairs(rm, e));
                }
                const int tn = min(32, nhost - m0);  // the hosts in this round (warp-uniform)
#pragma unroll 4
                for (int t = 0; t < tn; ++t) {
                    const int r_ = __shfl_sync(FULL_MASK, rm, t), q_ = __shfl_sync(FULL_MASK, qm, t);
                    const int l_ = locality ? __shfl_sync(FULL_MASK, lm, t) : 0;
                    if (r_ < rk) {
                        ++pos;
                        st += q_;
                        locsum += l_;
                    }
                }
            }
            if (k < nhost) {
                const int slot = k == 0 ? e - home * L : L + (j - jlo[pilo[j] + k - 1]);
                const int loc = locality ? min(qk, own_pairs(rk, e)) : 0;
                put_host(e, hptr(e) + pos, rk, slot, qk, st - locsum, loc);
            }
        }
    }
#pragma unroll 1
    for (int x = tid; x <= E; x += nt) {
        if (wr) a.p.host_ptr[x] = hptr(x);
        if (!sink.legacy) sink.hptr[x] = hptr(x);
    }

    if (tid == 0) {
        const int n_over = misc[2];
        int st = 0;
        if (n_over > 0) {
            st |= MOONEP_ST_OVERFLOW;
            if (d.flags & MOONEP_FLAG_STRICT_BUDGET) st |= MOONEP_ST_STRICT_VIOLATION;
        }
        misc[MISC_N_REP] = n_rep;
        misc[MISC_N_PIECES] = nP;
        misc[MISC_N_RECEIVERS] = nN;
        misc[MISC_N_REP_EXPERTS] = n_rep_experts;
        misc[MISC_PLAN_STATUS] = st;
        if (sink.legacy) {
            a.p.info[MOONEP_INFO_STATUS] = st;
            a.p.info[MOONEP_INFO_N_REP] = n_rep;
            a.p.info[MOONEP_INFO_N_OVERFLOW] = n_over;
            a.p.info[MOONEP_INFO_N_PIECES] = nP;
            a.p.info[MOONEP_INFO_N_RECEIVERS] = nN;
            a.p.info[MOONEP_INFO_MAX_REP_PER_RANK] = misc[3];
            a.p.info[MOONEP_INFO_N_REP_EXPERTS] = n_rep_experts;
#pragma unroll 1
            for (int i = MOONEP_INFO_N_REMOTE_PAIRS; i < MOONEP_INFO_LEN; ++i) a.p.info[i] = 0;
        }
    }
    // the host tables and the status precede the plan-ready mark
    __syncthreads();
    if (sink.legacy && tid == 0) {
        __threadfence();
        st_release(a.hdr + WS_PLANNED, seq + 1);
    }
    if (!sink.legacy)
        // the one-kernel path: the rows of the padded slot tables of this
        // CTA's ranks (r mod gridDim.x), used and empty slots alike, so every
        // entry is written once and no defaults precede them
#pragma unroll 1
        for (int r = blockIdx.x; r < R; r += gridDim.x) {
            const int b0 = rank_base(r), ns = rank_base(r + 1) - b0;
#pragma unroll 1
            for (int sl = tid; sl <= E; sl += nt) {
                const bool used = sl < ns;
                if (sl < E) {
                    a.p.slot_expert[(size_t)r * E + sl] = used ? cexp[b0 + sl] : -1;
                    a.p.slot_count[(size_t)r * E + sl] = used ? ccnt[b0 + sl] : 0;
                }
                a.p.slot_offset[(size_t)r * (E + 1) + sl] = used ? Z[b0 + sl] - Z[b0] : C;
            }
        }
    if (!wr) return;
    if (sink.legacy) {
        // ---- then, while the assignment CTAs place the pairs, the used
        // slots of the padded [R][E] tables (read only by later kernels,
        // which start after this grid has finished)
#pragma unroll 1
        for (int x = tid; x < E + n_rep; x += nt) {
            const int r = cspare[x], b0 = rank_base(r), sl = x - b0;
            a.p.slot_expert[(size_t)r * E + sl] = cexp[x];
            a.p.slot_count[(size_t)r * E + sl] = ccnt[x];
            a.p.slot_offset[(size_t)r * (E + 1) + sl] = Z[x] - Z[b0];
        }
    } else {
        // the writer: the empty rest of the replica and host tables
#pragma unroll 1
        for (int q = n_rep + tid; q < E + R; q += nt) {
            a.p.rep_expert[q] = -1;
            a.p.rep_rank[q] = -1;
            a.p.rep_slot[q] = -1;
            a.p.rep_quota[q] = 0;
        }
#pragma unroll 1
        for (int h = n_hosts + tid; h < nh; h += nt) {
            a.p.host_rank[h] = -1;
            a.p.host_slot[h] = -1;
            a.p.host_start[h] = 0;
            a.p.host_quota[h] = 0;
            a.p.host_local[h] = 0;
        }
    }
    // the reduce work list
#pragma unroll 1
    for (int x = tid; x < E; x += nt) {
        if (flag[x]) a.p.rep_home_list[Z[zf + x] - zf0] = x;
        if (x >= n_rep_experts) a.p.rep_home_list[x] = -1;
    }
}

// The plan tables' empty defaults (unused slots, replica and host entries),
// entries x0, x0 + g, ...: the grid's share of the calling thread, or the
// CTA's.  The planner writes the used entries over them afterwards, so no
// later pass fills the unused rest.
__device__ __forceinline__ void write_table_defaults(const PlanParams &a, int x0, int g)
{
    const Dims &d = a.d;
    const int E = d.E, R = d.R, nh = 2 * E + R;
    for (int x = x0; x < R * E; x += g) {
        a.p.slot_expert[x] = -1;
        a.p.slot_count[x] = 0;
    }
    for (int x = x0; x < R * (E + 1); x += g) a.p.slot_offset[x] = d.C;
    for (int x = x0; x < E + R; x += g) {
        a.p.rep_expert[x] = -1;
        a.p.rep_rank[x] = -1;
        a.p.rep_slot[x] = -1;
        a.p.rep_quota[x] = 0;
    }
    for (int x = x0; x < nh; x += g) {
        a.p.host_rank[x] = -1;
        a.p.host_slot[x] = -1;
        a.p.host_start[x] = 0;
        a.p.host_quota[x] = 0;
        a.p.host_local[x] = 0;
    }
}

// An empty plan: every table empty, spread over the grid, and dst_pos (and,
// with rows, row_src) -1 for this CTA's pairs [p0, p0 + n) (the rows are as
// many as the pairs, so the CTAs cover row_src too).
__device__ __forceinline__ void write_empty_plan(const PlanParams &a, int p0, int n, bool rows = true)
{
    const Dims &d = a.d;
    const int E = d.E, R = d.R, nh = 2 * E + R;
    const int g = gridDim.x * blockDim.x, x0 = blockIdx.x * blockDim.x + threadIdx.x;
    for (int x = x0; x < R * E; x += g) {
        a.p.slot_expert[x] = -1;
        a.p.slot_count[x] = 0;
    }
    for (int x = x0; x < R * (E + 1); x += g) a.p.slot_offset[x] = 0;
    for (int x = x0; x < E + R; x += g) {
        a.p.rep_expert[x] = -1;
        a.p.rep_rank[x] = -1;
        a.p.rep_slot[x] = -1;
        a.p.rep_quota[x] = 0;
    }
    for (int x = x0; x < nh; x += g) {
        a.p.host_rank[x] = -1;
        a.p.host_slot[x] = -1;
        a.p.host_start[x] = 0;
        a.p.host_quota[x] = 0;
        a.p.host_local[x] = 0;
    }
    for (int x = x0; x <= E; x += g) a.p.host_ptr[x] = 0;
    for (int x = x0; x < E; x += g) a.p.rep_home_list[x] = -1;
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        a.p.dst_pos[p0 + i] = -1;
        if (rows) a.p.row_src[p0 + i] = -1;
    }
}

__global__ void __launch_bounds__(PLAN_THREADS) hist_plan_kernel(PlanParams a)
{
    extern __shared__ int sm[];
    __shared__ int s_last, s_seq;
    const Dims &d = a.d;
    const int E = d.E, K = d.K, tid = threadIdx.x, nt = blockDim.x;
    // launched with programmatic dependent launch after whatever the stream
    // ran before (the router, or the last reader of this plan): its CTAs may
    // be placed while that kernel drains, and wait here for its completion
    // before touching any memory
    pdl_wait();
    // the assignment kernel may be scheduled now: it reads the counts after
    // the READY mark and the plan after the PLANNED mark
    pdl_launch_dependents();

    const int chunk = blockIdx.x;
    const int t0 = chunk * d.chunk_tokens;
    const int t1 = min(t0 + d.chunk_tokens, d.tokens);
    const int p0 = t0 * K, n = (t1 - t0) * K;
    int *hist = sm;       // E
    int *ids = sm + E;    // chunk_tokens * K
    // this CTA's share of the defaults; the planner CTA writes the used
    // entries after every CTA's ticket
    write_table_defaults(a, blockIdx.x * nt + tid, gridDim.x * nt);
    for (int e = tid; e < E; e += nt) hist[e] = 0;
    for (int i = tid; i < n; i += nt) ids[i] = __ldg(a.topk + p0 + i);  // all loads in flight
    if (tid == 0) s_seq = ld_cg(a.hdr + WS_SEQ);
    __syncthreads();
    const int seq = s_seq, parity = seq & 1;
    // distinct experts within a token: at most 32/K lanes of a warp collide
    int bad = 0;
    for (int i = tid; i < n; i += nt) {
        const int e = ids[i];
        if (e < 0 || e >= E) bad = 1;
        else atomicAdd(&hist[e], 1);
    }
    bad = __syncthreads_or(bad);
    int *gsb = a.gs + ((size_t)parity * d.ngroups + chunk / CHUNK_GROUP) * E;
    for (int e = tid; e < E; e += nt) {
        const int c = hist[e];
        a.cc[(size_t)chunk * E + e] = c;
        if (c) atomicAdd(gsb + e, c);  // sums: order-free
    }
    // release: the CTA barrier orders every thread's writes before thread 0's
    // device-scope fence and ticket increment; the last CTA's thread 0
    // fences again (acquire) before the barrier that lets the CTA read
    __syncthreads();
    if (tid == 0) {
        if (bad) atomicOr(a.hdr + WS_STATUS, MOONEP_ST_EXPERT_ID_RANGE);
        __threadfence();
        const bool last = atomicAdd(a.hdr + WS_TICKET, 1) == (int)gridDim.x - 1;
        if (last) {
            __threadfence();
            // every chunk's counts are in: open them to the assignment CTAs
            a.hdr[WS_ARRIVED] = 0;
            st_release(a.hdr + WS_READY, seq + 1);
        }
        s_last = last;
    }
    __syncthreads();
    if (!s_last) return;
    plan_block(a, sm, seq);
}

// ---------------------------------------------------------- assignment

// The host of rank g among an expert's hosts [h0, hend) (hend > h0): the last
// h with hstart[h] <= g (hstart[h0] = 0 <= g; starts are non-decreasing in
// rank order, equal where a host takes no rows), by bisection -- a hot expert
// has tens of hosts, and a linear walk over them held back its warp.
__device__ __forceinline__ int host_of(const int *hstart, int h0, int hend, int g)
{
    int lo = h0, hi = hend;  // the answer is in [lo, hi)
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (hstart[mid] <= g) lo = mid;
        else hi = mid;
    }
    return lo;
}

// Pass A, on the ids alone: the calling warp walks its contiguous sub-range
// [wbeg, wend) of the staged ids in (t, k) order, ranking equal experts with
// ballots, so loc is the pair's rank among the sub-range's earlier pairs of
// its expert and the warp's counters wc[E] end as its per-expert counts.
// ids[i] becomes loc << PACK_BITS | e.  (Out-of-range ids are left as they
// are; they make the plan empty.)
__device__ __forceinline__ void assign_pass_a(int *ids, int *wc, int wbeg, int wend, int E, int ebits)
{
    const int lane = threadIdx.x & 31;
    for (int b = wbeg; b < wend; b += 32) {
        const int i = b + lane;
        const bool valid = i < wend;
        const int e = valid ? ids[i] : 0;
        const bool ok = valid && e >= 0 && e < E;
        const unsigned peers = peers_of(ok ? e : 0, ok, ebits);
        int loc = 0;
        if (ok) loc = wc[e] + __popc(peers & lanemask_lt());
        __syncwarp();
        if (ok && lane == __ffs(peers) - 1) wc[e] += __popc(peers);
        __syncwarp();
        if (ok) ids[i] = (loc << PACK_BITS) | e;
    }
}

// Pass A as above, with the lanes of a batch that hold the same expert found
// by one shared-memory atomicOr per pair into a lane mask per expert (mk: the
// warp's E words, zero on entry and again on exit) instead of one ballot per
// id bit: the vote unit's throughput, not latency, bounds the ballot form
// when all warps of an SM run it.  Same ranks, bit for bit.
__device__ __forceinline__ void assign_pass_a_mask(int *ids, int *wc, unsigned *mk, int wbeg, int wend, int E)
{
    const int lane = threadIdx.x & 31;
    for (int b = wbeg; b < wend; b += 32) {
        const int i = b + lane;
        const int e = i < wend ? ids[i] : -1;
        const bool ok = e >= 0 && e < E;
        if (ok) atomicOr(&mk[e], 1u << lane);
        __syncwarp();
        unsigned peers = 0;
        int base = 0;
        if (ok) {
            peers = mk[e];
            base = wc[e];
        }
        __syncwarp();  // every lane has read its expert's words before the first lane updates them
        if (ok) {
            if (lane == __ffs(peers) - 1) {
                wc[e] = base + __popc(peers);
                mk[e] = 0;
            }
            ids[i] = ((base + __popc(peers & lanemask_lt())) << PACK_BITS) | e;
        }
        __syncwarp();
    }
}

// Pass B for the calling warp's sub-range: g = warp base wb[e] + loc is the
// pair's rank among all pairs of its expert in (t, k) order; the host
// interval holding g gives the buffer row hdst[h] + g, a global row in
// [0, rows).  Pair i of the sub-range is pair p0 + i of dst_pos; row_src
// (may be null) gets the inverse; a row out of range sets MOONEP_ST_ROW_RANGE
// in *status.  Returns the number of the warp's pairs that land on another
// rank than their source rank: src_rank >= 0 is the source rank of every pair
// (one rank's pairs), -1 derives it as p / C.
__device__ __forceinline__ int assign_pass_b(const int *ids, const int *wb, const int *hptr, const int *hstart,
                                             const int *hdst, int wbeg, int wend, int p0, int E, int rows, int C,
                                             const FastDiv &fC, int src_rank, int *dst_pos, int *row_src,
                                             int *status)
{
    const int lane = threadIdx.x & 31;
    int remote = 0;
    for (int i = wbeg + lane; i < wend; i += 32) {
        const int v = ids[i];
        const int e = v & PACK_MASK, loc = v >> PACK_BITS;
        if (v < 0 || e >= E) continue;  // cannot happen in a non-empty plan
        const int g = wb[e] + loc;
        const int h = host_of(hstart, hptr[e], hptr[e + 1], g);
        const int dst = hdst[h] + g;
        const int p = p0 + i;
        if (dst < 0 || dst >= rows) {  // cannot happen for a consistent plan
            atomicOr(status, MOONEP_ST_ROW_RANGE);
            dst_pos[p] = -1;
            continue;
        }
        dst_pos[p] = dst;
        if (row_src) row_src[dst] = p;
        // the source rank's first row: the rank of pair p is p / (S*K) = p / C
        const uint32_t src0 = (src_rank >= 0 ? (uint32_t)src_rank : fdiv((uint32_t)p, fC)) * (uint32_t)C;
        remote += (uint32_t)dst - src0 >= (uint32_t)C;
    }
    return remote;
}

// Pass B of the one-kernel planner.  dw (per warp and expert) = the row of
// rank wb (the warp base) in the expert's first host; dlim (per expert) = the
// first row past the first host (INT_MAX when the expert has one host).  A
// pair of rank loc in the warp's sub-range thus has row dw + loc, unless that
// is past the first host, where the host intervals give it: two
// shared-memory loads per pair on the common path, where the generic pass
// makes about six.  Their random expert index makes them conflict, but
// halving them did not shorten this pass: the host search and the scattered
// row_src stores take its time.  (Staging row_src in shared memory in (expert,
// rank) order, so that its stores coalesce, measured 1.9 µs slower at the
// large shape than these scattered stores.)
// src_rank >= 0: the source rank of every pair (one rank's pairs, whose
// row_src is null); -1 derives it as p / C.
__device__ __forceinline__ int assign_pass_b_fused(const int *ids, const int *dw, const int *dlim, const int *hptr,
                                                   const int *hstart, const int *hdst, int wbeg, int wend, int p0,
                                                   int E, int rows, int C, const FastDiv &fC, int src_rank,
                                                   int *dst_pos, int *row_src, int *status)
{
    const int lane = threadIdx.x & 31;
    int remote = 0;
    for (int i = wbeg + lane; i < wend; i += 32) {
        const int v = ids[i];
        const int e = v & PACK_MASK, loc = v >> PACK_BITS;
        if (v < 0 || e >= E) continue;  // cannot happen in a non-empty plan
        int dst = dw[e] + loc;
        if (dst >= dlim[e]) {  // past the expert's first host
            const int h0 = hptr[e];
            const int g = dst - hdst[h0];
            dst = hdst[host_of(hstart, h0, hptr[e + 1], g)] + g;
        }
        const int p = p0 + i;
        if (dst < 0 || dst >= rows) {  // cannot happen for a consistent plan
            atomicOr(status, MOONEP_ST_ROW_RANGE);
            dst_pos[p] = -1;
            continue;
        }
        dst_pos[p] = dst;
        if (row_src) row_src[dst] = p;
        const uint32_t src0 = (src_rank >= 0 ? (uint32_t)src_rank : fdiv((uint32_t)p, fC)) * (uint32_t)C;
        remote += (uint32_t)dst - src0 >= (uint32_t)C;
    }
    return remote;
}

__global__ void __launch_bounds__(ASSIGN_THREADS, 2) assign_kernel(PlanParams a)
{
    extern __shared__ int sm[];
    const Dims &d = a.d;
    const int E = d.E, K = d.K, R = d.R, C = d.C;
    const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31, warp = tid >> 5;
    const int chunk = blockIdx.x;
    const int t0 = chunk * d.chunk_tokens;
    const int t1 = min(t0 + d.chunk_tokens, d.tokens);
    const int p0 = t0 * K, n = (t1 - t0) * K;
    const int max_pairs = d.chunk_tokens * K;
    const int nh = 2 * E + R;

    int *cnt = sm;                         // ASSIGN_WARPS * E
    int *ids = cnt + ASSIGN_WARPS * E;     // max_pairs
    int *hptr = ids + max_pairs;           // E + 1
    int *hstart = hptr + E + 1;            // nh
    int *hdst = hstart + nh;               // nh
    int *red = hdst + nh;                  // 32
    __shared__ int s_seq, s_ready, s_planned;

    // prologue on inputs only, overlapping the histogram/planner grid
    for (int i = tid; i < ASSIGN_WARPS * E; i += nt) cnt[i] = 0;
    for (int i = tid; i < n; i += nt) ids[i] = __ldg(a.topk + p0 + i);
    __syncthreads();

    // pass A, on the ids alone: each warp walks its contiguous sub-range in
    // (t, k) order, ranking equal experts with ballots, so loc is the pair's
    // rank among the sub-range's earlier pairs of its expert and the warp's
    // counters end as its per-expert counts.  ids[i] becomes loc << 10 | e.
    // (Out-of-range ids are left as they are; they make the plan empty.)
    const int per = (n + ASSIGN_WARPS - 1) / ASSIGN_WARPS;
    const int wbeg = min(warp * per, n), wend = min(wbeg + per, n);
    assign_pass_a(ids, cnt + warp * E, wbeg, wend, E, d.ebits);

    // ---- the counts are complete once the last histogram CTA has set READY;
    // the planner CTA is still running then, and the chunk bases and warp
    // counts below overlap it.  Every histogram CTA is resident before this
    // grid starts, so the mark comes; the bounded wait falls back to the
    // grid dependency, which implies it.
    if (tid == 0) {
        const int seq = ld_cg(a.hdr + WS_SEQ);
        int ok = 0;
        for (int it = 0; it < a.spin_limit; ++it) {
            if (ld_acquire(a.hdr + WS_READY) == seq + 1) {
                ok = 1;
                break;
            }
            __nanosleep(100);
        }
        s_seq = seq;
        s_ready = ok;
    }
    __syncthreads();
    if (!s_ready) {  // complete either way; report that the mark came late
        pdl_wait();
        if (tid == 0) atomicOr(a.p.info + MOONEP_INFO_STATUS, MOONEP_ST_WAIT_TIMEOUT);
    }
    const int seq = s_seq;
    if (tid == 0) {  // the last CTA past this point advances the sequence
        if (atomicAdd(a.hdr + WS_ARRIVED, 1) == (int)gridDim.x - 1) {
            a.hdr[WS_ARRIVED] = 0;
            a.hdr[WS_SEQ] = seq + 1;
        }
    }

    // the previous call's group-count buffer is read by nobody now; zero it
    // for the next call, which accumulates into it
    {
        int *old = a.gs + (size_t)((seq & 1) ^ 1) * d.ngroups * E;
        const int n_gs = d.ngroups * E;
        for (int i = blockIdx.x * nt + tid; i < n_gs; i += gridDim.x * nt) old[i] = 0;
    }

    // pairs of each expert in earlier chunks: earlier groups + earlier chunks
    // of this chunk's group, all loads of a batch in flight together, then
    // the warp bases
    {
        const int grp = chunk / CHUNK_GROUP, c0 = grp * CHUNK_GROUP;
        const int *gsb = a.gs + (size_t)(seq & 1) * d.ngroups * E;  // the buffer this call filled
        for (int e = tid; e < E; e += nt) {
            int s = 0;
            for (int g0 = 0; g0 < grp; g0 += 32) {
                int v[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) v[j] = (g0 + j < grp) ? ld_cg(gsb + (size_t)(g0 + j) * E + e) : 0;
                int w[CHUNK_GROUP - 1];
                if (g0 == 0) {
#pragma unroll
                    for (int j = 0; j < CHUNK_GROUP - 1; ++j)
                        w[j] = (c0 + j < chunk) ? ld_cg(a.cc + (size_t)(c0 + j) * E + e) : 0;
#pragma unroll
                    for (int j = 0; j < CHUNK_GROUP - 1; ++j) s += w[j];
                }
#pragma unroll
                for (int j = 0; j < 32; ++j) s += v[j];
            }
            if (grp == 0) {
                int w[CHUNK_GROUP - 1];
#pragma unroll
                for (int j = 0; j < CHUNK_GROUP - 1; ++j)
                    w[j] = (c0 + j < chunk) ? ld_cg(a.cc + (size_t)(c0 + j) * E + e) : 0;
#pragma unroll
                for (int j = 0; j < CHUNK_GROUP - 1; ++j) s += w[j];
            }
            // warp bases: this prefix plus the earlier warps' counts of
            // this chunk (pass A's counters are past the barrier above)
            for (int w = 0; w < ASSIGN_WARPS; ++w) {
                const int t = cnt[w * E + e];
                cnt[w * E + e] = s;
                s += t;
            }
        }
    }

    // ---- the plan is complete once the planner CTA has set PLANNED (a
    // bounded wait, as for READY: the planner CTA is resident, and the grid
    // dependency implies the mark).  Every load below is issued before any
    // of its results is used (one round trip), and every count or index read
    // back is clamped, so even a plan block of garbage cannot steer an
    // access out of its array.
    // A slow path announced by the planner is waited for through the grid
    // dependency, without a timeout report.
    if (tid == 0) {
        int ok = 0;
        for (int it = 0; it < a.spin_limit; ++it) {
            if (ld_acquire(a.hdr + WS_PLANNED) == seq + 1) {
                ok = 1;
                break;
            }
            if (ld_acquire(a.hdr + WS_SLOW) == seq + 1) {
                ok = 2;
                break;
            }
            __nanosleep(64);
        }
        s_planned = ok;
    }
    __syncthreads();
    if (s_planned != 1) {
        pdl_wait();
        if (tid == 0 && s_planned == 0) atomicOr(a.p.info + MOONEP_INFO_STATUS, MOONEP_ST_WAIT_TIMEOUT);
    }
    const int status = ld_cg(a.p.info + MOONEP_INFO_STATUS);
    // host tables of the whole array; only entries inside the clamped
    // [host_ptr[e], host_ptr[e+1]) are used
    for (int e = tid; e <= E; e += nt) hptr[e] = min(max(ld_cg(a.p.host_ptr + e), 0), nh);
    for (int h = tid; h < nh; h += nt) {
        hstart[h] = ld_cg(a.p.host_start + h);
        hdst[h] = ld_cg(a.host_dst0 + h);
    }
    const bool empty = (status & ST_EMPTY_PLAN) != 0;

    // ---- an empty plan: every table empty, spread over the CTAs.  (For a
    // plan, the histogram CTAs wrote the empty defaults before the planner
    // wrote its entries over them.)
    if (empty) {
        write_empty_plan(a, p0, n);
        pdl_wait();  // as below: finish after the histogram grid
        return;
    }
    __syncthreads();

    // pass B: g = warp base + loc is the pair's rank among all pairs of its
    // expert in (t, k) order; the host interval holding g gives the buffer row
    int remote = assign_pass_b(ids, cnt + warp * E, hptr, hstart, hdst, wbeg, wend, p0, E, R * C, C, a.fC, -1,
                               a.p.dst_pos, a.p.row_src, a.p.info + MOONEP_INFO_STATUS);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) remote += __shfl_xor_sync(FULL_MASK, remote, o);
    if (lane == 0) red[warp] = remote;
    __syncthreads();
    if (tid == 0) {
        int s = 0;
        for (int w = 0; w < (nt >> 5); ++w) s += red[w];
        if (s) atomicAdd(a.p.info + MOONEP_INFO_N_REMOTE_PAIRS, s);
    }
    // this grid finishes only after the histogram grid: the planner CTA
    // writes its last tables after the plan-ready mark, and a kernel that
    // follows the plan in the stream must see them
    pdl_wait();
}

// The chunk's ids [p0, p0 + n) of topk into shared memory, by the calling
// CTA: 16-byte loads, all of a thread's in flight together (from pair p0 & ~3
// on, into ids_raw, so the loads are aligned; the few before p0 belong to the
// previous chunk and are not used), then the last < 4 one by one; every pair
// one by one when topk is not 16-byte aligned.  ids = ids_raw + (p0 & 3).
// Returns whether this thread saw an id outside [0, E).
__device__ __forceinline__ int stage_ids(const int32_t *topk, int p0, int n, int E, int *ids_raw, int *ids)
{
    const int tid = threadIdx.x, nt = blockDim.x;
    int bad = 0;
    const int q0 = p0 >> 2, q1 = (p0 + n) >> 2;  // 16-byte words wholly or partly before p0 + n
    const bool vec = (reinterpret_cast<uintptr_t>(topk) & 15) == 0;
    const int nv = vec ? q1 - q0 : 0;
    const int4 *src = reinterpret_cast<const int4 *>(topk) + q0;
    constexpr int VB = 4;
    for (int k0 = tid; k0 < nv; k0 += VB * nt) {
        int4 v[VB];
#pragma unroll
        for (int j = 0; j < VB; ++j)
            if (k0 + j * nt < nv) v[j] = __ldg(src + k0 + j * nt);
#pragma unroll
        for (int j = 0; j < VB; ++j) {
            const int k = k0 + j * nt;
            if (k < nv) {
                reinterpret_cast<int4 *>(ids_raw)[k] = v[j];
                const int q = 4 * (q0 + k);  // pair of v[j].x
                const int x[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    if (q + c >= p0) bad |= x[c] < 0 || x[c] >= E;
            }
        }
    }
    for (int i = (vec ? max(4 * q1 - p0, 0) : 0) + tid; i < n; i += nt) {
        const int e = __ldg(topk + p0 + i);
        ids[i] = e;
        bad |= e < 0 || e >= E;
    }
    return bad;
}

// ------------------------------------------------------- one-kernel planner
//
// When one CTA per SM can hold a chunk of about tokens / SMs tokens beside
// the planner's shared memory, one launch does the whole plan.  Every CTA
// stages its chunk's ids, ranks them (pass A), adds the chunk's counts to its
// group's and takes a ticket.  Once every chunk's counts are in, it sums the
// expert totals and its chunk's base, runs the planner on them in its own
// shared memory -- every CTA computes the same plan, so no CTA waits for
// another's tables -- and places its pairs from its own copy of the host
// tables (pass B).  Each CTA writes the slot-table rows of the ranks it owns
// (r mod chunks), one CTA (the last chunk's, which has the fewest pairs) the
// other tables, and the CTA that finishes last writes the info block and
// resets the header for the next call.  One CTA per SM,
// not two with half the tokens each: the planner is a chain of short
// dependent steps, and two of them on one SM take nearly twice as long.
// The chunking is this kernel's own (at most one chunk per SM); the group
// counts use the workspace's buffers at its layout (gs_buf), so a workspace
// may pass between this path and the two-kernel one.
// The wait for the ticket is bounded: a CTA that gives up (its peers not all
// resident) counts every pair of the call itself, which is slower but gives
// the same totals and base, and reports MOONEP_ST_WAIT_TIMEOUT.  A ticket past
// the chunk count can only come from a workspace that was not zero-filled.
__host__ __device__ inline int fused_smem_ints(int E, int R, int max_pairs, unsigned flags, int B)
{
    // (pass A's lane masks, ASSIGN_WARPS * E words, fit in the planner's
    // 22 E + 13 R + 58 ints, which are idle until the totals)
    static_assert(ASSIGN_WARPS <= 22, "pass A's lane masks alias the planner's shared memory");
    return ASSIGN_WARPS * E + (max_pairs + 4) + (E + 1) + 2 * (2 * E + R) + 32 + (E + 1) + plan_smem_ints(E, R) +
           ((flags & MOONEP_FLAG_CASCADE) ? cascade_smem_ints(E, R, B) : 0);
}

__global__ void __launch_bounds__(PLAN_THREADS, 1) plan_fused_kernel(PlanParams a)
{
    extern __shared__ __align__(16) int sm[];
    const Dims &d = a.d;
    const int E = d.E, K = d.K, R = d.R, C = d.C;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr int nt = PLAN_THREADS;
    static_assert(PLAN_THREADS == ASSIGN_THREADS, "one block size for the planner and the passes");
    const int chunk = blockIdx.x, nchunk = gridDim.x;
    const int t0 = chunk * d.chunk_tokens;
    const int t1 = min(t0 + d.chunk_tokens, d.tokens);
    const int p0 = t0 * K, n = (t1 - t0) * K;
    const int max_pairs = d.chunk_tokens * K;
    const int nh = 2 * E + R;

    int *cnt = sm;                           // ASSIGN_WARPS * E: warp counts, then warp bases
    int *ids_raw = cnt + ASSIGN_WARPS * E;   // max_pairs + 4, 16-byte aligned: from pair p0 & ~3 on
    int *ids = ids_raw + (p0 & 3);           // the chunk's pairs
    int *hptr = ids_raw + max_pairs + 4;     // E + 1
    int *hstart = hptr + E + 1;              // nh
    int *hdst = hstart + nh;                 // nh; first each expert's pairs in earlier chunks
    int *red = hdst + nh;                    // 32
    int *dlim = red + 32;                    // E (+1 pad): pass B's first row past each expert's first host
    int *psm = dlim + E + 1;                 // the planner's; first pass A's lane masks (ASSIGN_WARPS * E)
    unsigned *mk = reinterpret_cast<unsigned *>(psm);
    int *T = psm;
    const int *misc = plan_misc(psm, E, R);
    __shared__ int s_seq, s_wait, s_status;

    // placed while the stream's previous kernel drains: wait for it before
    // touching memory
    pdl_wait();
    for (int i = tid; i < ASSIGN_WARPS * E; i += nt) {
        cnt[i] = 0;
        mk[i] = 0;
    }
    const int bad = stage_ids(a.topk, p0, n, E, ids_raw, ids);
    if (tid == 0) s_seq = ld_cg(a.hdr + WS_SEQ);
    const int any_bad = __syncthreads_or(bad);
    const int seq = s_seq, parity = seq & 1;
    {  // the previous call's group counts are read by nobody now: zero them for the next call
        int *old = a.gs + (size_t)(parity ^ 1) * a.gs_buf;
        for (int i = chunk * nt + tid; i < a.gs_buf; i += nchunk * nt) old[i] = 0;
    }

    // pass A, then the chunk's counts (column sums of the warp counters)
    const int per = (n + ASSIGN_WARPS - 1) / ASSIGN_WARPS;
    const int wbeg = min(warp * per, n), wend = min(wbeg + per, n);
    assign_pass_a_mask(ids, cnt + warp * E, mk + warp * E, wbeg, wend, E);
    __syncthreads();
    {
        int *gsb = a.gs + (size_t)parity * a.gs_buf + (size_t)(chunk / CHUNK_GROUP) * E;
        for (int e = tid; e < E; e += nt) {
            int c = 0;
#pragma unroll 4
            for (int w = 0; w < ASSIGN_WARPS; ++w) c += cnt[w * E + e];
            a.cc[(size_t)chunk * E + e] = c;
            if (c) atomicAdd(gsb + e, c);  // sums: order-free
        }
    }
    // release the counts with the ticket, then wait (bounded) for every chunk's
    __syncthreads();
    int mine = 0;
    if (tid == 0) {
        if (any_bad) atomicOr(a.hdr + WS_STATUS, MOONEP_ST_EXPERT_ID_RANGE);
        __threadfence();
        mine = atomicAdd(a.hdr + WS_TICKET, 1) + 1;
    }
    if (tid == 0) {
        int w = 0, st = 0;  // w: 0 gave up, 1 every chunk in, 2 ticket past the chunk count
        if (mine == nchunk) w = 1;
        else if (mine > nchunk || mine <= 0) w = 2;
        for (int it = 0; w == 0 && it < a.spin_limit; ++it) {
            const int tk = ld_acquire(a.hdr + WS_TICKET);
            if (tk == nchunk) w = 1;
            else if (tk > nchunk || tk <= 0) w = 2;
            else __nanosleep(32);
        }
        if (w == 1) {
            __threadfence();
            st = ld_cg(a.hdr + WS_STATUS);
        }
        s_wait = w;
        s_status = st;
    }
    __syncthreads();
    const int wstate = s_wait;
    int status_in = s_status;

    // ---- the expert totals T and this chunk's base (pairs of each expert in
    // earlier chunks, into hdst for now)
    const int grp = chunk / CHUNK_GROUP, c0 = grp * CHUNK_GROUP;
    unsigned part = 0;  // <= 2 values < 2^31 each (negative ones are flagged)
    int negative = 0;
    if (wstate == 1) {
        const int *gsb = a.gs + (size_t)parity * a.gs_buf;
        for (int e = tid; e < E; e += nt) {
            int w[CHUNK_GROUP - 1];
#pragma unroll
            for (int j = 0; j < CHUNK_GROUP - 1; ++j)
                w[j] = (c0 + j < chunk) ? ld_cg(a.cc + (size_t)(c0 + j) * E + e) : 0;
            int tot = 0, before = 0;
            for (int g0 = 0; g0 < d.ngroups; g0 += 32) {
                int v[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) v[j] = (g0 + j < d.ngroups) ? ld_cg(gsb + (size_t)(g0 + j) * E + e) : 0;
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    tot += v[j];
                    before += (g0 + j < grp) ? v[j] : 0;
                }
            }
#pragma unroll
            for (int j = 0; j < CHUNK_GROUP - 1; ++j) before += w[j];
            T[e] = tot;
            hdst[e] = before;
            negative |= tot < 0;
            part += (unsigned)tot;
        }
    } else {
        for (int e = tid; e < E; e += nt) {
            T[e] = 0;
            hdst[e] = 0;
        }
        if (wstate == 0) {  // gave up waiting: count every pair of the call here
            __syncthreads();
            int bad_any = 0;
            for (int p = tid; p < d.pairs; p += nt) {
                const int e = __ldg(a.topk + p);
                if (e < 0 || e >= E) {
                    bad_any = 1;
                    continue;
                }
                atomicAdd(&T[e], 1);
                if (p < p0) atomicAdd(&hdst[e], 1);
            }
            bad_any = __syncthreads_or(bad_any);
            status_in = bad_any ? MOONEP_ST_EXPERT_ID_RANGE : 0;
            if (tid == 0) atomicOr(a.hdr + WS_FLAGS, MOONEP_ST_WAIT_TIMEOUT);
        } else {
            status_in = MOONEP_ST_WORKSPACE;
        }
    }
    // with every id valid the summed totals must be non-negative and add up
    // to the pairs; anything else means the workspace was not zeroed (exact
    // 64-bit total from 16-bit halves, each warp sum by one reduction)
    {
        const unsigned lo = __reduce_add_sync(FULL_MASK, part & 0xffffu);
        const unsigned hi = __reduce_add_sync(FULL_MASK, part >> 16);
        if (lane == 0) {
            red[warp] = (int)lo;
            red[16 + warp] = (int)hi;
        }
    }
    negative = __syncthreads_or(negative);
    if (wstate == 1) {
        const unsigned lo = __reduce_add_sync(FULL_MASK, lane < ASSIGN_WARPS ? (unsigned)red[lane] : 0u);
        const unsigned hi = __reduce_add_sync(FULL_MASK, lane < ASSIGN_WARPS ? (unsigned)red[16 + lane] : 0u);
        const long long total = ((long long)hi << 16) + (long long)lo;
        if (!(status_in & MOONEP_ST_EXPERT_ID_RANGE) && (negative || total != (long long)d.pairs))
            status_in |= MOONEP_ST_WORKSPACE;
    }
    // warp bases: the chunk's base plus the earlier warps' counts
    for (int e = tid; e < E; e += nt) {
        int sb = hdst[e];
        for (int w = 0; w < ASSIGN_WARPS; ++w) {
            const int t = cnt[w * E + e];
            cnt[w * E + e] = sb;
            sb += t;
        }
    }
    const bool writer = chunk == nchunk - 1;
    if (writer)
        for (int e = tid; e < E; e += nt) a.p.expert_count[e] = T[e];
    __syncthreads();

    const bool empty = (status_in & ST_EMPTY_PLAN) != 0;
    int remote = 0;
    if (empty) {
        write_empty_plan(a, p0, n);
    } else {
        plan_core(a, psm, seq, PlanSink{false, writer, hptr, hstart, hdst});
        __syncthreads();
        // pass B's tables from this CTA's own host tables: dw over the warp
        // bases, and dlim
        int *dw = cnt;
        for (int e = tid; e < E; e += nt) {
            const int h0 = hptr[e], d0 = hdst[h0];
#pragma unroll 4
            for (int w = 0; w < ASSIGN_WARPS; ++w) dw[w * E + e] = d0 + cnt[w * E + e];
            dlim[e] = hptr[e + 1] - h0 > 1 ? d0 + hstart[h0 + 1] : INT_MAX;
        }
        __syncthreads();
        remote = assign_pass_b_fused(ids, dw + warp * E, dlim, hptr, hstart, hdst, wbeg, wend, p0, E, R * C, C, a.fC,
                                     -1, a.p.dst_pos, a.p.row_src, a.hdr + WS_FLAGS);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) remote += __shfl_xor_sync(FULL_MASK, remote, o);
    if (lane == 0) red[warp] = remote;
    __syncthreads();
    if (tid == 0) {
        int sr = 0;
        for (int w = 0; w < ASSIGN_WARPS; ++w) sr += red[w];
        if (sr) atomicAdd(a.hdr + WS_REMOTE, sr);
        // the CTA that finishes last: the info block, and the header reset
        // for the next call (which starts after this grid has finished)
        __threadfence();
        if (atomicAdd(a.hdr + WS_ARRIVED, 1) == nchunk - 1) {
            __threadfence();
            const int late = atomicExch(a.hdr + WS_FLAGS, 0);
            const int remote_all = atomicExch(a.hdr + WS_REMOTE, 0);
            int *info = a.p.info;
            for (int i = 1; i < MOONEP_INFO_LEN; ++i) info[i] = 0;
            if (empty) {
                info[MOONEP_INFO_STATUS] = status_in | late;
            } else {
                info[MOONEP_INFO_STATUS] = misc[MISC_PLAN_STATUS] | late;
                info[MOONEP_INFO_N_REP] = misc[MISC_N_REP];
                info[MOONEP_INFO_N_OVERFLOW] = misc[MISC_N_OVER];
                info[MOONEP_INFO_N_PIECES] = misc[MISC_N_PIECES];
                info[MOONEP_INFO_N_RECEIVERS] = misc[MISC_N_RECEIVERS];
                info[MOONEP_INFO_MAX_REP_PER_RANK] = misc[MISC_MAX_REP];
                info[MOONEP_INFO_N_REP_EXPERTS] = misc[MISC_N_REP_EXPERTS];
                info[MOONEP_INFO_N_REMOTE_PAIRS] = remote_all;
                info[MOONEP_INFO_CASCADE_GUARD_STEPS] = misc[MISC_GUARD_STEPS];
                info[MOONEP_INFO_CASCADE_GUARD_SLACK] = misc[MISC_GUARD_SLACK];
            }
            a.hdr[WS_TICKET] = 0;
            a.hdr[WS_STATUS] = 0;
            a.hdr[WS_ARRIVED] = 0;
            a.hdr[WS_READY] = seq + 1;
            a.hdr[WS_PLANNED] = seq + 1;
            a.hdr[WS_SEQ] = seq + 1;
        }
    }
}

// ---------------------------------------------------------------- launch

// Both planner kernels ask for the largest shared-memory carveout: an SM
// that runs histogram CTAs must also fit two assignment CTAs as the
// histogram CTAs retire (the carveout changes only when an SM is idle).
// The attributes are set once per device and kernel, and again only when a
// launch needs more dynamic shared memory than was allowed so far: the
// driver calls cost host time on every plan of a latency-bound layer.
constexpr int SMEM_CACHE_DEVICES = 64;
enum { K_HIST, K_ASSIGN, K_EP_COUNT, K_EP_PLAN, K_EP_ASSIGN, K_FUSED, K_EP_FUSED, K_N };
static std::atomic<size_t> g_smem_set[SMEM_CACHE_DEVICES][K_N];  // bytes allowed so far, 0 = never set

static bool set_smem(int which, const void *fn, size_t bytes)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    std::atomic<size_t> *slot = (dev >= 0 && dev < SMEM_CACHE_DEVICES) ? &g_smem_set[dev][which] : nullptr;
    if (slot && slot->load(std::memory_order_relaxed) >= bytes && bytes > 0) return true;
    const bool ok =
        cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) == cudaSuccess &&
        cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout,
                             (int)cudaSharedmemCarveoutMaxShared) == cudaSuccess;
    if (ok && slot) {
        size_t cur = slot->load(std::memory_order_relaxed);
        while (cur < bytes && !slot->compare_exchange_weak(cur, bytes, std::memory_order_relaxed)) {
        }
    }
    return ok;
}

// moonep_set_plan_path: 0 lets launch_plan choose, 1 keeps it on the
// two-kernel path (for tests that compare the two)
static std::atomic<int> g_plan_path{0};

int set_plan_path(int mode) { return g_plan_path.exchange(mode == 1 ? 1 : 0); }

// Resident CTAs per SM of the one-kernel planner with `smem` bytes of dynamic
// shared memory, on the current device (cached per device for the last few
// sizes: a plan call makes no occupancy query once its size has been seen).
constexpr int OCC_SLOTS = 4;
struct OccCache {
    std::mutex m;
    size_t smem[OCC_SLOTS] = {};
    int blocks[OCC_SLOTS] = {};
    int next = 0;
};
static OccCache g_occ[SMEM_CACHE_DEVICES];

static int fused_blocks_per_sm(size_t smem)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= SMEM_CACHE_DEVICES) return 0;
    OccCache &c = g_occ[dev];
    std::lock_guard<std::mutex> lock(c.m);
    for (int i = 0; i < OCC_SLOTS; ++i)
        if (c.smem[i] == smem && c.blocks[i] > 0) return c.blocks[i];
    int nb = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, plan_fused_kernel, PLAN_THREADS, smem) != cudaSuccess) {
        (void)cudaGetLastError();
        return 0;
    }
    c.smem[c.next] = smem;
    c.blocks[c.next] = nb;
    c.next = (c.next + 1) % OCC_SLOTS;
    return nb;
}

constexpr size_t MAX_BLOCK_SMEM = 227 * 1024;

int launch_plan(const Dims &d, const int32_t *topk, const moonep_plan_t &p, void *ws, cudaStream_t st)
{
    const WsLayout wl = ws_layout(d);
    char *w = static_cast<char *>(ws);
    PlanParams a;
    a.d = d;
    a.topk = topk;
    a.p = p;
    a.hdr = reinterpret_cast<int *>(w + wl.hdr);
    a.gs = reinterpret_cast<int *>(w + wl.gs);
    a.cc = reinterpret_cast<int *>(w + wl.cc);
    a.host_dst0 = reinterpret_cast<int *>(w + wl.host_dst0);
    a.gs_stride = d.E;
    a.gs_buf = d.ngroups * d.E;
    a.fC = make_fastdiv((uint32_t)d.C);
    a.fL = make_fastdiv((uint32_t)d.L);
    a.spin_limit = g_wait_limit.load(std::memory_order_relaxed);
    a.cascade_cap = cascade_cap_for(d);

    // both kernels with programmatic dependent launch: each may be placed
    // while its predecessor drains and waits (griddepcontrol.wait, or the
    // marks) before it reads anything the predecessor writes
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;

    // one kernel when one CTA per SM holds a chunk of tokens / SMs tokens (at
    // least 8) beside the planner: its chunking is coarser than the
    // two-kernel path's, so it fits in the workspace laid out for that
    if (g_plan_path.load(std::memory_order_relaxed) == 0) {
        PlanParams af = a;
        Dims &df = af.d;
        int ct = (d.tokens + d.nsm - 1) / d.nsm;
        if (ct < 8) ct = 8;
        if (ct > d.tokens) ct = d.tokens;
        df.chunk_tokens = ct;
        df.nchunk = (d.tokens + ct - 1) / ct;
        df.ngroups = (df.nchunk + CHUNK_GROUP - 1) / CHUNK_GROUP;
        const size_t smemf = sizeof(int) * (size_t)fused_smem_ints(d.E, d.R, ct * d.K, d.flags, d.B);
        if (df.nchunk <= d.nchunk && df.nchunk <= d.nsm && smemf <= MAX_BLOCK_SMEM &&
            set_smem(K_FUSED, (const void *)plan_fused_kernel, smemf) && fused_blocks_per_sm(smemf) >= 1) {
            cudaLaunchConfig_t cf = {};
            cf.gridDim = dim3(df.nchunk);
            cf.blockDim = dim3(PLAN_THREADS);
            cf.dynamicSmemBytes = smemf;
            cf.stream = st;
            cf.attrs = attr;
            cf.numAttrs = 1;
            return cudaLaunchKernelEx(&cf, plan_fused_kernel, af) == cudaSuccess ? MOONEP_OK : MOONEP_ERR_CUDA;
        }
        (void)cudaGetLastError();  // a refused attribute leaves the two-kernel path
    }

    const size_t smem1 = sizeof(int) * (size_t)hist_smem_ints(d.E, d.R, d.chunk_tokens * d.K, d.flags, d.B);
    if (!set_smem(K_HIST, (const void *)hist_plan_kernel, smem1)) return MOONEP_ERR_CUDA;
    cudaLaunchConfig_t c1 = {};
    c1.gridDim = dim3(d.nchunk);
    c1.blockDim = dim3(PLAN_THREADS);
    c1.dynamicSmemBytes = smem1;
    c1.stream = st;
    c1.attrs = attr;
    c1.numAttrs = 1;
    if (cudaLaunchKernelEx(&c1, hist_plan_kernel, a) != cudaSuccess) return MOONEP_ERR_CUDA;

    const size_t smem2 = sizeof(int) * (size_t)assign_smem_ints(d.E, d.R, d.chunk_tokens * d.K);
    if (!set_smem(K_ASSIGN, (const void *)assign_kernel, smem2)) return MOONEP_ERR_CUDA;
    cudaLaunchConfig_t c2 = c1;
    c2.blockDim = dim3(ASSIGN_THREADS);
    c2.dynamicSmemBytes = smem2;
    if (cudaLaunchKernelEx(&c2, assign_kernel, a) != cudaSuccess) return MOONEP_ERR_CUDA;
    return MOONEP_OK;
}

// ------------------------------------------------------- expert parallelism
//
// One process per GPU; rank `rank` of R owns S tokens (its topk rows [S, K]).
// The MoonEP article ("The core idea: dynamic redundant experts") writes
// every pair straight into its expert-grouped row on a remote rank; the plan
// needs every rank's per-expert counts, which are small ([E] per rank) and
// all-gathered by the caller between the count and the plan.  Every rank then
// runs the same planner on the same counts, so all ranks hold identical plan
// tables, and places its own pairs: the pair's rank g within its expert is
// the counts of the lower ranks plus its rank among this rank's own pairs,
// exactly the global (t, k) order of the single-GPU plan.  The per-rank
// chunking is over the S local tokens (d.nchunk, d.chunk_tokens); d.ngroups
// is R, the rows of the gathered counts.

// EP workspace header slots: the count kernel's ticket and invalid-id count,
// the planner's status word
enum { EP_TICKET = WS_TICKET, EP_STATUS = WS_STATUS, EP_BAD = WS_ARRIVED };

struct EpCountParams {
    Dims d;
    const int32_t *topk;  // [S, K]
    int *hdr, *cc;
    int32_t *counts_row;  // [E + 1]
};

// Per-chunk histograms of the rank's own ids (into the workspace, for the
// assignment), then, in the CTA that finishes last, their sums: the rank's
// counts row [E] and, in slot E, its number of ids outside [0, E).
__global__ void __launch_bounds__(PLAN_THREADS) ep_count_kernel(EpCountParams a)
{
    extern __shared__ int sm[];
    __shared__ int s_last;
    const Dims &d = a.d;
    const int E = d.E, K = d.K, tid = threadIdx.x, nt = blockDim.x;
    pdl_wait();  // the producer of the ids
    const int chunk = blockIdx.x;
    const int t0 = chunk * d.chunk_tokens, t1 = min(t0 + d.chunk_tokens, d.S);
    const int p0 = t0 * K, n = (t1 - t0) * K;
    int *hist = sm, *ids = sm + E;
    for (int e = tid; e < E; e += nt) hist[e] = 0;
    for (int i = tid; i < n; i += nt) ids[i] = __ldg(a.topk + p0 + i);
    __syncthreads();
    int bad = 0;
    for (int i = tid; i < n; i += nt) {
        const int e = ids[i];
        if (e < 0 || e >= E) ++bad;
        else atomicAdd(&hist[e], 1);
    }
    bad = __syncthreads_count(bad > 0) > 0 ? __reduce_add_sync(FULL_MASK, bad) : 0;
    if ((tid & 31) == 0 && bad) atomicAdd(a.hdr + EP_BAD, bad);
    for (int e = tid; e < E; e += nt) a.cc[(size_t)chunk * E + e] = hist[e];
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        const bool last = atomicAdd(a.hdr + EP_TICKET, 1) == (int)gridDim.x - 1;
        if (last) __threadfence();
        s_last = last;
    }
    __syncthreads();
    if (!s_last) return;
    for (int e = tid; e < E; e += nt) a.counts_row[e] = sum_strided<32>(a.cc + e, E, d.nchunk);
    if (tid == 0) {
        a.counts_row[E] = ld_cg(a.hdr + EP_BAD);
        a.hdr[EP_BAD] = 0;
        a.hdr[EP_TICKET] = 0;
    }
}

// The planner on the gathered counts [R][E+1], in one CTA: the tables'
// empty defaults, the status (an invalid id on any rank empties the plan),
// then the single-GPU planner with the counts as its R count rows.
__global__ void __launch_bounds__(PLAN_THREADS) ep_plan_kernel(PlanParams a)
{
    extern __shared__ int sm[];
    const Dims &d = a.d;
    const int E = d.E, R = d.R, tid = threadIdx.x;
    constexpr int nt = PLAN_THREADS;
    const int nh = 2 * E + R;
    // the assignment grid may start its prologue on the ids
    pdl_launch_dependents();
    for (int x = tid; x < R * E; x += nt) {
        a.p.slot_expert[x] = -1;
        a.p.slot_count[x] = 0;
    }
    for (int x = tid; x < R * (E + 1); x += nt) a.p.slot_offset[x] = d.C;
    for (int x = tid; x < E + R; x += nt) {
        a.p.rep_expert[x] = -1;
        a.p.rep_rank[x] = -1;
        a.p.rep_slot[x] = -1;
        a.p.rep_quota[x] = 0;
    }
    for (int x = tid; x < nh; x += nt) {
        a.p.host_rank[x] = -1;
        a.p.host_slot[x] = -1;
        a.p.host_start[x] = 0;
        a.p.host_quota[x] = 0;
        a.p.host_local[x] = 0;
    }
    if (tid < 32) {
        int bad = 0;
        for (int r = tid; r < R; r += 32) bad |= ld_cg(a.gs + (size_t)r * a.gs_stride + E) != 0;
        bad = __any_sync(FULL_MASK, bad);
        if (tid == 0) a.hdr[WS_STATUS] = bad ? MOONEP_ST_EXPERT_ID_RANGE : 0;
    }
    __syncthreads();
    plan_block(a, sm, 0);
    __syncthreads();
    // an empty plan: the tables as moonep_plan leaves them
    if (ld_cg(a.p.info + MOONEP_INFO_STATUS) & ST_EMPTY_PLAN) {
        for (int x = tid; x < R * (E + 1); x += nt) a.p.slot_offset[x] = 0;
        for (int x = tid; x <= E; x += nt) a.p.host_ptr[x] = 0;
        for (int x = tid; x < E; x += nt) a.p.rep_home_list[x] = -1;
    }
}

// The rank's own pairs: pass A on the ids while the planner runs, chunk
// bases from the lower ranks' counts and this rank's earlier chunks, then
// (after the planner grid) pass B.  dst_pos[0 .. S*K) gets global rows;
// row_src is not written (the rows of this rank's buffer are filled by every
// rank).  info[MOONEP_INFO_N_REMOTE_PAIRS] counts this rank's pairs placed
// on another rank.
__host__ __device__ inline int ep_assign_smem_ints(int E, int R, int max_pairs)
{
    const int nh = 2 * E + R;
    return assign_smem_ints(E, R, max_pairs) + 3 * nh /*local quota rank*/ + 3 * E /*own before G*/;
}

// Pass B with MOONEP_FLAG_LOCALITY for the calling warp's sub-range, all of
// whose pairs come from rank `rank`: the pair's rank g within its expert and
// gs within this rank's pairs of it (g - G[e]); the host on this rank takes
// it as local pair gs when gs < its local count, otherwise it is leftover
// number u = g - before[e] (the local pairs of the hosts on ranks <= rank),
// served by the host whose leftover share [start, start + quota - local)
// holds u, at row dst0 + local + u.
__device__ __forceinline__ int assign_pass_b_local(const int *ids, const int *wb, const int *hptr,
                                                   const int *hstart, const int *hdst, const int *hloc,
                                                   const int *hq, const int *own, const int *before,
                                                   const int *G, int wbeg, int wend, int p0, int E, int rows,
                                                   int C, int rank, int *dst_pos, int *status)
{
    const int lane = threadIdx.x & 31;
    int remote = 0;
    for (int i = wbeg + lane; i < wend; i += 32) {
        const int v = ids[i];
        const int e = v & PACK_MASK, loc = v >> PACK_BITS;
        if (v < 0 || e >= E) continue;  // cannot happen in a non-empty plan
        const int g = wb[e] + loc, gs = g - G[e], ho = own[e];
        int dst = -1;
        if (ho >= 0 && gs < hloc[ho]) {
            dst = hdst[ho] + hstart[ho] + gs;
        } else {
            const int u = g - before[e];
            for (int h = hptr[e]; h < hptr[e + 1]; ++h)
                if (hstart[h] <= u && u < hstart[h] + hq[h] - hloc[h]) {
                    dst = hdst[h] + hloc[h] + u;
                    break;
                }
        }
        const int p = p0 + i;
        if (dst < 0 || dst >= rows) {  // cannot happen for a consistent plan
            atomicOr(status, MOONEP_ST_ROW_RANGE);
            dst_pos[p] = -1;
            continue;
        }
        dst_pos[p] = dst;
        remote += (uint32_t)dst - (uint32_t)rank * (uint32_t)C >= (uint32_t)C;
    }
    return remote;
}

// The rank's own pairs: pass A on the ids while the planner runs, chunk
// bases from the lower ranks' counts and this rank's earlier chunks, then
// (after the planner grid) pass B.  dst_pos[0 .. S*K) gets global rows;
// row_src is not written (the rows of this rank's buffer are filled by every
// rank).  info[MOONEP_INFO_N_REMOTE_PAIRS] counts this rank's pairs placed
// on another rank.
__global__ void __launch_bounds__(ASSIGN_THREADS, 2) ep_assign_kernel(PlanParams a, int rank)
{
    extern __shared__ int sm[];
    const Dims &d = a.d;
    const int E = d.E, K = d.K, R = d.R, C = d.C;
    const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31, warp = tid >> 5;
    const int chunk = blockIdx.x;
    const int t0 = chunk * d.chunk_tokens, t1 = min(t0 + d.chunk_tokens, d.S);
    const int p0 = t0 * K, n = (t1 - t0) * K;
    const int max_pairs = d.chunk_tokens * K;
    const int nh = 2 * E + R;
    const bool locality = (d.flags & MOONEP_FLAG_LOCALITY) != 0;
    int *cnt = sm;                      // ASSIGN_WARPS * E
    int *ids = cnt + ASSIGN_WARPS * E;  // max_pairs
    int *hptr = ids + max_pairs;        // E + 1
    int *hstart = hptr + E + 1;         // nh
    int *hdst = hstart + nh;            // nh
    int *red = hdst + nh;               // 32
    int *hloc = red + 32;               // nh  (locality only, from here on)
    int *hq = hloc + nh;                // nh
    int *hr = hq + nh;                  // nh
    int *own = hr + nh;                 // E: the expert's host on this rank, or -1
    int *before = own + E;              // E: local pairs of the hosts on ranks <= rank
    int *G = before + E;                // E: the expert's pairs on lower ranks

    // on the ids and the counts only, overlapping the planner
    for (int i = tid; i < ASSIGN_WARPS * E; i += nt) cnt[i] = 0;
    for (int i = tid; i < n; i += nt) ids[i] = __ldg(a.topk + p0 + i);
    __syncthreads();
    const int per = (n + ASSIGN_WARPS - 1) / ASSIGN_WARPS;
    const int wbeg = min(warp * per, n), wend = min(wbeg + per, n);
    assign_pass_a(ids, cnt + warp * E, wbeg, wend, E, d.ebits);
    __syncthreads();
    // chunk base: pairs of e on lower ranks plus on this rank's earlier
    // chunks; then the warp bases
    for (int e = tid; e < E; e += nt) {
        const int lower = sum_strided<32>(a.gs + e, a.gs_stride, rank);
        G[e] = lower;
        int s = lower + sum_strided<32>(a.cc + e, E, chunk);
        for (int w = 0; w < ASSIGN_WARPS; ++w) {
            const int t = cnt[w * E + e];
            cnt[w * E + e] = s;
            s += t;
        }
    }
    // the plan is complete once the planner grid has finished
    pdl_wait();
    const int status = ld_cg(a.p.info + MOONEP_INFO_STATUS);
    for (int e = tid; e <= E; e += nt) hptr[e] = min(max(ld_cg(a.p.host_ptr + e), 0), nh);
    for (int h = tid; h < nh; h += nt) {
        hstart[h] = ld_cg(a.p.host_start + h);
        hdst[h] = ld_cg(a.host_dst0 + h);
        if (locality) {
            hloc[h] = ld_cg(a.p.host_local + h);
            hq[h] = ld_cg(a.p.host_quota + h);
            hr[h] = ld_cg(a.p.host_rank + h);
        }
    }
    if (status & ST_EMPTY_PLAN) {
        for (int i = tid; i < n; i += nt) a.p.dst_pos[p0 + i] = -1;
        return;
    }
    __syncthreads();
    int remote;
    if (locality) {
        for (int e = tid; e < E; e += nt) {
            int o = -1, b = 0;
            for (int h = hptr[e]; h < hptr[e + 1]; ++h) {
                if (hr[h] <= rank) b += hloc[h];
                if (hr[h] == rank) o = h;
            }
            own[e] = o;
            before[e] = b;
        }
        __syncthreads();
        remote = assign_pass_b_local(ids, cnt + warp * E, hptr, hstart, hdst, hloc, hq, own, before, G, wbeg, wend,
                                     p0, E, R * C, C, rank, a.p.dst_pos, a.p.info + MOONEP_INFO_STATUS);
    } else {
        remote = assign_pass_b(ids, cnt + warp * E, hptr, hstart, hdst, wbeg, wend, p0, E, R * C, C, a.fC, rank,
                               a.p.dst_pos, nullptr, a.p.info + MOONEP_INFO_STATUS);
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

// ------------------------------------------------- expert parallelism, one kernel
//
// In expert parallelism the plan's inputs, the gathered counts [R][E+1], are
// complete before the planner starts, so every CTA can plan at once: one
// launch over the rank's token chunks (the chunking of moonep_ep_count), each
// CTA staging its chunk's ids and ranking them (pass A), summing the expert
// totals and its chunk's base (the lower ranks' counts and this rank's
// earlier chunks') from the gathered rows, running the planner in its own
// shared memory and placing its pairs (pass B, or the locality-aware pass B).
// No CTA waits for another, so none needs the others resident.  One CTA (the
// last chunk's) writes the small tables, each CTA the slot-table rows of the
// ranks it owns (r mod chunks), and the CTA that finishes last (EP_DONE) the
// info block.
enum { EP_DONE = 9 };

__host__ __device__ inline int ep_fused_smem_ints(int E, int R, int max_pairs, unsigned flags, int B)
{
    const int nh = 2 * E + R;
    return ASSIGN_WARPS * E + (max_pairs + 4) + (E + 1) + 2 * nh + 32 + (E + 1) + 3 * nh + 3 * E +
           plan_smem_ints(E, R) + ((flags & MOONEP_FLAG_CASCADE) ? cascade_smem_ints(E, R, B) : 0);
}

__global__ void __launch_bounds__(PLAN_THREADS, 1) ep_fused_kernel(PlanParams a, int rank)
{
    extern __shared__ __align__(16) int sm[];
    const Dims &d = a.d;
    const int E = d.E, K = d.K, R = d.R, C = d.C;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr int nt = PLAN_THREADS;
    const int chunk = blockIdx.x, nchunk = gridDim.x;
    const int t0 = chunk * d.chunk_tokens, t1 = min(t0 + d.chunk_tokens, d.S);
    const int p0 = t0 * K, n = (t1 - t0) * K;
    const int max_pairs = d.chunk_tokens * K;
    const int nh = 2 * E + R;
    const bool locality = (d.flags & MOONEP_FLAG_LOCALITY) != 0;

    int *cnt = sm;                          // ASSIGN_WARPS * E: warp counts, then warp bases
    int *ids_raw = cnt + ASSIGN_WARPS * E;  // max_pairs + 4
    int *ids = ids_raw + (p0 & 3);
    int *hptr = ids_raw + max_pairs + 4;    // E + 1
    int *hstart = hptr + E + 1;             // nh
    int *hdst = hstart + nh;                // nh; first each expert's pairs before this chunk
    int *red = hdst + nh;                   // 32
    int *dlim = red + 32;                   // E + 1
    int *hloc = dlim + E + 1;               // nh: each host's local pairs, quota, rank
    int *hq = hloc + nh;                    // nh
    int *hr = hq + nh;                      // nh
    int *own = hr + nh;                     // E: the expert's host on this rank, or -1
    int *before = own + E;                  // E: local pairs of the hosts on ranks <= rank
    int *G = before + E;                    // E: the expert's pairs on lower ranks
    int *psm = G + E;                       // the planner's; first pass A's lane masks
    unsigned *mk = reinterpret_cast<unsigned *>(psm);
    int *T = psm;
    const int *misc = plan_misc(psm, E, R);

    pdl_wait();  // the producer of the ids and of the gathered counts
    for (int i = tid; i < ASSIGN_WARPS * E; i += nt) {
        cnt[i] = 0;
        mk[i] = 0;
    }
    stage_ids(a.topk, p0, n, E, ids_raw, ids);  // invalid ids are in the gathered counts' slot E
    __syncthreads();
    const int per = (n + ASSIGN_WARPS - 1) / ASSIGN_WARPS;
    const int wbeg = min(warp * per, n), wend = min(wbeg + per, n);
    assign_pass_a_mask(ids, cnt + warp * E, mk + warp * E, wbeg, wend, E);
    __syncthreads();

    // totals, the lower ranks' pairs and this chunk's base, from the gathered
    // rows and this rank's per-chunk counts
    int bad = 0, negative = 0;
    unsigned part = 0;  // <= 2 values < 2^31 each (negative ones are flagged)
    for (int r = tid; r < R; r += nt) bad |= ld_cg(a.gs + (size_t)r * a.gs_stride + E) != 0;
    for (int e = tid; e < E; e += nt) {
        int tot = 0, lower = 0;
        for (int r0 = 0; r0 < R; r0 += 32) {
            int v[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = r0 + j < R ? ld_cg(a.gs + (size_t)(r0 + j) * a.gs_stride + e) : 0;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                tot += v[j];
                lower += r0 + j < rank ? v[j] : 0;
            }
        }
        T[e] = tot;
        G[e] = lower;
        hdst[e] = lower + sum_strided<32>(a.cc + e, E, chunk);
        negative |= tot < 0;
        part += (unsigned)tot;
    }
    {
        const unsigned lo = __reduce_add_sync(FULL_MASK, part & 0xffffu);
        const unsigned hi = __reduce_add_sync(FULL_MASK, part >> 16);
        if (lane == 0) {
            red[warp] = (int)lo;
            red[16 + warp] = (int)hi;
        }
    }
    bad = __syncthreads_or(bad);
    negative = __syncthreads_or(negative);
    int status_in = bad ? MOONEP_ST_EXPERT_ID_RANGE : 0;
    {
        const unsigned lo = __reduce_add_sync(FULL_MASK, lane < ASSIGN_WARPS ? (unsigned)red[lane] : 0u);
        const unsigned hi = __reduce_add_sync(FULL_MASK, lane < ASSIGN_WARPS ? (unsigned)red[16 + lane] : 0u);
        const long long total = ((long long)hi << 16) + (long long)lo;
        if (!bad && (negative || total != (long long)d.pairs)) status_in |= MOONEP_ST_WORKSPACE;
    }
    for (int e = tid; e < E; e += nt) {
        int sb = hdst[e];
        for (int w = 0; w < ASSIGN_WARPS; ++w) {
            const int t = cnt[w * E + e];
            cnt[w * E + e] = sb;
            sb += t;
        }
    }
    const bool writer = chunk == nchunk - 1;
    if (writer)
        for (int e = tid; e < E; e += nt) a.p.expert_count[e] = T[e];
    __syncthreads();

    const bool empty = (status_in & ST_EMPTY_PLAN) != 0;
    int remote = 0;
    if (empty) {
        write_empty_plan(a, p0, n, false);  // row_src is not this rank's to write
    } else {
        PlanSink sink{false, writer, hptr, hstart, hdst};
        if (locality) {
            sink.hloc = hloc;
            sink.hq = hq;
            sink.hr = hr;
        }
        plan_core(a, psm, 0, sink);
        __syncthreads();
        if (locality) {
            for (int e = tid; e < E; e += nt) {
                int o = -1, b = 0;
                for (int h = hptr[e]; h < hptr[e + 1]; ++h) {
                    if (hr[h] <= rank) b += hloc[h];
                    if (hr[h] == rank) o = h;
                }
                own[e] = o;
                before[e] = b;
            }
            __syncthreads();
            remote = assign_pass_b_local(ids, cnt + warp * E, hptr, hstart, hdst, hloc, hq, own, before, G, wbeg,
                                         wend, p0, E, R * C, C, rank, a.p.dst_pos, a.hdr + WS_FLAGS);
        } else {
            int *dw = cnt;
            for (int e = tid; e < E; e += nt) {
                const int h0 = hptr[e], d0 = hdst[h0];
#pragma unroll 4
                for (int w = 0; w < ASSIGN_WARPS; ++w) dw[w * E + e] = d0 + cnt[w * E + e];
                dlim[e] = hptr[e + 1] - h0 > 1 ? d0 + hstart[h0 + 1] : INT_MAX;
            }
            __syncthreads();
            remote = assign_pass_b_fused(ids, dw + warp * E, dlim, hptr, hstart, hdst, wbeg, wend, p0, E, R * C, C,
                                         a.fC, rank, a.p.dst_pos, nullptr, a.hdr + WS_FLAGS);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) remote += __shfl_xor_sync(FULL_MASK, remote, o);
    if (lane == 0) red[warp] = remote;
    __syncthreads();
    if (tid == 0) {
        int sr = 0;
        for (int w = 0; w < ASSIGN_WARPS; ++w) sr += red[w];
        if (sr) atomicAdd(a.hdr + WS_REMOTE, sr);
        __threadfence();
        if (atomicAdd(a.hdr + EP_DONE, 1) == nchunk - 1) {
            __threadfence();
            const int late = atomicExch(a.hdr + WS_FLAGS, 0);
            const int remote_all = atomicExch(a.hdr + WS_REMOTE, 0);
            int *info = a.p.info;
            for (int i = 1; i < MOONEP_INFO_LEN; ++i) info[i] = 0;
            if (empty) {
                info[MOONEP_INFO_STATUS] = status_in | late;
            } else {
                info[MOONEP_INFO_STATUS] = misc[MISC_PLAN_STATUS] | late;
                info[MOONEP_INFO_N_REP] = misc[MISC_N_REP];
                info[MOONEP_INFO_N_OVERFLOW] = misc[MISC_N_OVER];
                info[MOONEP_INFO_N_PIECES] = misc[MISC_N_PIECES];
                info[MOONEP_INFO_N_RECEIVERS] = misc[MISC_N_RECEIVERS];
                info[MOONEP_INFO_MAX_REP_PER_RANK] = misc[MISC_MAX_REP];
                info[MOONEP_INFO_N_REP_EXPERTS] = misc[MISC_N_REP_EXPERTS];
                info[MOONEP_INFO_N_REMOTE_PAIRS] = remote_all;
                info[MOONEP_INFO_CASCADE_GUARD_STEPS] = misc[MISC_GUARD_STEPS];
                info[MOONEP_INFO_CASCADE_GUARD_SLACK] = misc[MISC_GUARD_SLACK];
            }
            a.hdr[EP_DONE] = 0;
        }
    }
}

int launch_ep_count(const Dims &d, const int32_t *topk, int32_t *counts_row, void *ws, cudaStream_t st)
{
    const EpWsLayout wl = ws_layout_ep(d);
    char *w = static_cast<char *>(ws);
    EpCountParams a;
    a.d = d;
    a.topk = topk;
    a.hdr = reinterpret_cast<int *>(w + wl.hdr);
    a.cc = reinterpret_cast<int *>(w + wl.cc);
    a.counts_row = counts_row;
    const size_t smem = sizeof(int) * (size_t)(d.E + d.chunk_tokens * d.K);
    if (!set_smem(K_EP_COUNT, (const void *)ep_count_kernel, smem)) return MOONEP_ERR_CUDA;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t c = {};
    c.gridDim = dim3(d.nchunk);
    c.blockDim = dim3(PLAN_THREADS);
    c.dynamicSmemBytes = smem;
    c.stream = st;
    c.attrs = attr;
    c.numAttrs = 1;
    return cudaLaunchKernelEx(&c, ep_count_kernel, a) == cudaSuccess ? MOONEP_OK : MOONEP_ERR_CUDA;
}

int launch_ep_plan(const Dims &d, int rank, const int32_t *topk, const int32_t *counts_all,
                   const moonep_plan_t &p, void *ws, cudaStream_t st)
{
    const EpWsLayout wl = ws_layout_ep(d);
    char *w = static_cast<char *>(ws);
    PlanParams a;
    a.d = d;
    a.d.ngroups = d.R;  // the planner sums R count rows
    a.topk = topk;
    a.p = p;
    a.hdr = reinterpret_cast<int *>(w + wl.hdr);
    a.gs = const_cast<int *>(counts_all);
    a.gs_stride = d.E + 1;
    a.gs_buf = 0;  // the gathered counts are one buffer, rewritten by the caller every call
    a.cc = reinterpret_cast<int *>(w + wl.cc);
    a.host_dst0 = reinterpret_cast<int *>(w + wl.host_dst0);
    a.fC = make_fastdiv((uint32_t)d.C);
    a.fL = make_fastdiv((uint32_t)d.L);
    a.spin_limit = 0;
    a.cascade_cap = cascade_cap_for(d);

    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;

    // one kernel wherever its shared memory fits (no CTA waits for another,
    // so residency does not matter)
    const size_t smemf = sizeof(int) * (size_t)ep_fused_smem_ints(d.E, d.R, d.chunk_tokens * d.K, d.flags, d.B);
    if (g_plan_path.load(std::memory_order_relaxed) == 0 && smemf <= MAX_BLOCK_SMEM &&
        set_smem(K_EP_FUSED, (const void *)ep_fused_kernel, smemf)) {
        cudaLaunchConfig_t cf = {};
        cf.gridDim = dim3(d.nchunk);
        cf.blockDim = dim3(PLAN_THREADS);
        cf.dynamicSmemBytes = smemf;
        cf.stream = st;
        cf.attrs = attr;
        cf.numAttrs = 1;
        return cudaLaunchKernelEx(&cf, ep_fused_kernel, a, rank) == cudaSuccess ? MOONEP_OK : MOONEP_ERR_CUDA;
    }
    (void)cudaGetLastError();

    const size_t smem1 = sizeof(int) * (size_t)(plan_smem_ints(d.E, d.R) +
                                                ((d.flags & MOONEP_FLAG_CASCADE) ? cascade_smem_ints(d.E, d.R, d.B) : 0));
    if (!set_smem(K_EP_PLAN, (const void *)ep_plan_kernel, smem1)) return MOONEP_ERR_CUDA;
    ep_plan_kernel<<<1, PLAN_THREADS, smem1, st>>>(a);
    if (cudaGetLastError() != cudaSuccess) return MOONEP_ERR_CUDA;

    const size_t smem2 = sizeof(int) * (size_t)ep_assign_smem_ints(d.E, d.R, d.chunk_tokens * d.K);
    if (!set_smem(K_EP_ASSIGN, (const void *)ep_assign_kernel, smem2)) return MOONEP_ERR_CUDA;
    cudaLaunchConfig_t c = {};
    c.gridDim = dim3(d.nchunk);
    c.blockDim = dim3(ASSIGN_THREADS);
    c.dynamicSmemBytes = smem2;
    c.stream = st;
    c.attrs = attr;
    c.numAttrs = 1;
    return cudaLaunchKernelEx(&c, ep_assign_kernel, a, rank) == cudaSuccess ? MOONEP_OK : MOONEP_ERR_CUDA;
}

size_t ep_smem_bytes_max(const Dims &d)
{
    const size_t a = sizeof(int) * (size_t)(plan_smem_ints(d.E, d.R) +
                                            ((d.flags & MOONEP_FLAG_CASCADE) ? cascade_smem_ints(d.E, d.R, d.B) : 0));
    const size_t b = sizeof(int) * (size_t)ep_assign_smem_ints(d.E, d.R, d.chunk_tokens * d.K);
    const size_t c = sizeof(int) * (size_t)(d.E + d.chunk_tokens * d.K);
    return a > b ? (a > c ? a : c) : (b > c ? b : c);
}

size_t plan_smem_bytes_max(const Dims &d)
{
    const size_t a = sizeof(int) * (size_t)hist_smem_ints(d.E, d.R, d.chunk_tokens * d.K, d.flags, d.B);
    const size_t b = sizeof(int) * (size_t)assign_smem_ints(d.E, d.R, d.chunk_tokens * d.K);
    return a > b ? a : b;
}

}  // namespace moonep
