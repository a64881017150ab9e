// Device-side helpers shared by the MoonEP kernels (sm_100a).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "moonep.h"

namespace moonep {

constexpr unsigned FULL_MASK = 0xffffffffu;

// Internal launch description shared by the host launchers.
struct Dims {
    int R, E, K, S, H, B, L;
    uint32_t flags;
    int C;        // S*K rows per rank
    int tokens;   // R*S
    int pairs;    // R*S*K
    int nchunk;   // planner token chunks
    int chunk_tokens;
    int ngroups;  // groups of CHUNK_GROUP consecutive chunks
    int ebits;    // bits of an expert id: 2^ebits >= E
    int nsm;      // SMs the chunking targets (the launch device's, at most 148)
};

// Chunks per group: the assignment pass sums at most CHUNK_GROUP - 1
// per-chunk counts on top of a group prefix.
constexpr int CHUNK_GROUP = 16;

// Workspace layout (bytes from the workspace base; 256-byte aligned parts).
struct WsLayout {
    size_t hdr;        // int32[16]: ticket, status, call sequence, counts-ready mark, arrivals, plan-ready mark,
                       // slow-path mark, late status bits, remote pairs
    size_t gs;         // int32 [2][ngroups][E]: per-group expert counts, double-buffered
    size_t cc;         // int32 [nchunk][E]: per-chunk expert counts
    size_t host_dst0;  // int32 [2E+R]: rank*C + slot_offset - host_start per host
    size_t total;
};
// The call sequence number SEQ counts completed plan calls on a workspace; its
// low bit selects the group-count buffer.  The last histogram CTA of a call
// sets READY = SEQ + 1 once every chunk's counts are in, and PLANNED = SEQ + 1
// once the plan is written; the assignment CTAs wait for those marks, and the
// last of them to arrive advances SEQ, so after a call READY == PLANNED == SEQ
// and a stale mark never passes for a fresh one.  SLOW = SEQ + 1 announces
// that the planner took a slow path (the relay cascade) whose length has no
// useful bound for a spin: the assignment CTAs then wait for the whole
// histogram grid instead.
// The one-kernel planner uses TICKET, STATUS, SEQ and ARRIVED the same way
// (TICKET: chunks whose counts are in; ARRIVED: CTAs done), and two words of
// its own that the CTA finishing last folds into the info block: FLAGS (status
// bits raised after the plan) and REMOTE (pairs placed off their source
// rank).  It leaves READY == PLANNED == SEQ too, so either path may follow it.
enum {
    WS_TICKET = 0, WS_STATUS = 1, WS_SEQ = 2, WS_READY = 3, WS_ARRIVED = 4, WS_PLANNED = 5, WS_SLOW = 6,
    WS_FLAGS = 7, WS_REMOTE = 8, WS_HDR_INTS = 16
};

// Status bits after which every later call treats the plan as empty.
constexpr int ST_EMPTY_PLAN = MOONEP_ST_EXPERT_ID_RANGE | MOONEP_ST_WORKSPACE;

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

__host__ inline WsLayout ws_layout(const Dims &d)
{
    WsLayout w;
    const size_t i4 = sizeof(int32_t), nh = (size_t)(2 * d.E + d.R);
    size_t o = 0;
    w.hdr = o; o = align256(o + WS_HDR_INTS * i4);
    w.gs = o; o = align256(o + i4 * 2 * (size_t)d.ngroups * d.E);
    w.cc = o; o = align256(o + i4 * (size_t)d.nchunk * d.E);
    w.host_dst0 = o; o = align256(o + i4 * nh);
    w.total = o;
    return w;
}

// Workspace of one rank in expert parallelism (moonep_ep_*): the header
// (the count kernel's ticket and invalid-id count, the planner's status
// word), this rank's per-chunk expert counts, and the host rows.
struct EpWsLayout {
    size_t hdr;        // int32[16]
    size_t cc;         // int32 [nchunk][E] over the rank's S tokens
    size_t host_dst0;  // int32 [2E+R]
    size_t total;
};

__host__ inline EpWsLayout ws_layout_ep(const Dims &d)
{
    EpWsLayout w;
    const size_t i4 = sizeof(int32_t);
    size_t o = 0;
    w.hdr = o; o = align256(o + WS_HDR_INTS * i4);
    w.cc = o; o = align256(o + i4 * (size_t)d.nchunk * d.E);
    w.host_dst0 = o; o = align256(o + i4 * (size_t)(2 * d.E + d.R));
    w.total = o;
    return w;
}

// Division by a run-time invariant 31-bit divisor with a multiply-high and a
// shift (Granlund & Montgomery, "Division by invariant integers using
// multiplication", 1994): for 0 <= n < 2^31 and d >= 1,
//   l = ceil(log2 d),  m = floor(2^32 (2^l - d) / d) + 1,
//   n / d = (umulhi(m, n) + n) >> l.
struct FastDiv {
    uint32_t d, m, l;
};

__host__ inline FastDiv make_fastdiv(uint32_t d)
{
    FastDiv f;
    f.d = d;
    uint32_t l = 0;
    while ((1ull << l) < d) ++l;
    f.l = l;
    f.m = (uint32_t)((((1ull << l) - d) << 32) / d + 1);
    return f;
}

__device__ __forceinline__ uint32_t fdiv(uint32_t n, const FastDiv &f)
{
    return (__umulhi(f.m, n) + n) >> f.l;
}

// Lanes holding the same key as this lane, from one ballot per key bit
// (keys in [0, 2^nbits), nbits <= MAX_KEY_BITS); lanes with valid == false
// match nobody.  The loop is unrolled; the bit guard is warp-uniform.
constexpr int MAX_KEY_BITS = 10;
static_assert((1 << MAX_KEY_BITS) >= MOONEP_MAX_E, "expert ids need more key bits");
__device__ __forceinline__ unsigned peers_of(int key, bool valid, int nbits)
{
    unsigned m = __ballot_sync(0xffffffffu, valid);
#pragma unroll
    for (int b = 0; b < MAX_KEY_BITS; ++b) {
        if (b < nbits) {
            const bool bit = (key >> b) & 1;
            const unsigned bb = __ballot_sync(0xffffffffu, bit);
            m &= bit ? bb : ~bb;
        }
    }
    return valid ? m : 0u;
}

__device__ __forceinline__ unsigned lanemask_lt()
{
    unsigned m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

__device__ __forceinline__ int ld_cg(const int *p) { return __ldcg(p); }

__device__ __forceinline__ int ld_acquire(const int *p)
{
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release(int *p, int v)
{
    asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Largest i in [0, n) with a[i] <= x, for non-decreasing a (a[0] <= x assumed).
__device__ __forceinline__ int last_le(const int *a, int n, int x)
{
    int lo = 0, hi = n;  // answer in [lo, hi)
    while (hi - lo > 1) {
        int mid = (lo + hi) >> 1;
        if (a[mid] <= x) lo = mid; else hi = mid;
    }
    return lo;
}

// Largest i in [0, n) with a[i] <= x, for non-decreasing a (a[0] <= x
// assumed), by one warp: every lane passes the same x and gets the result.
// Ballots count 32 entries at a time, stopping at the first chunk that is
// not all <= x.
__device__ __forceinline__ int warp_last_le(const int *a, int n, int x)
{
    const int lane = threadIdx.x & 31;
    int c = 0;
    for (int j0 = 0; j0 < n; j0 += 32) {
        const int j = j0 + lane;
        const unsigned b = __ballot_sync(FULL_MASK, j < n && a[j] <= x);
        c += __popc(b);
        if (b != FULL_MASK) break;
    }
    return c - 1;
}

// Exclusive prefix sum of a[0..n) in shared memory, in place; returns the
// total.  Every thread of the block must call it.  wsum: >= 32 ints of smem.
// Two barriers.  Each thread takes PER consecutive elements (PER fixed at
// compile time, fully unrolled; PER = 0: a runtime loop of per elements),
// the warps scan with shuffles, and every warp reads the warp totals with one
// load per lane and scans them with shuffles too: on sm_100 a small
// runtime-bound loop, or every thread reading every warp total, costs more
// than the whole scan.
template <int PER>
__device__ __forceinline__ int block_exscan_per(int *a, int n, int *wsum, int per)
{
    const int tid = threadIdx.x, nt = blockDim.x;
    const int lane = tid & 31, w = tid >> 5, nw = nt >> 5;
    constexpr int P = PER > 0 ? PER : 1;
    int v[P];
    int local = 0, beg;
    if (PER > 0) {
        beg = tid * PER;
#pragma unroll
        for (int k = 0; k < P; ++k) {
            v[k] = beg + k < n ? a[beg + k] : 0;
            local += v[k];
        }
    } else {
        beg = min(tid * per, n);
        const int end = min(beg + per, n);
        for (int i = beg; i < end; ++i) local += a[i];
    }
    int x = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(FULL_MASK, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) wsum[w] = x;
    __syncthreads();
    int s = lane < nw ? wsum[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(FULL_MASK, s, o);
        if (lane >= o) s += y;
    }
    const int total = __shfl_sync(FULL_MASK, s, 31);
    const int upto_w = __shfl_sync(FULL_MASK, s, w);  // warps 0..w
    const int own_w = __shfl_sync(FULL_MASK, x, 31);  // warp w alone
    int excl = x - local + upto_w - own_w;
    if (PER > 0) {
#pragma unroll
        for (int k = 0; k < P; ++k) {
            if (beg + k < n) a[beg + k] = excl;
            excl += v[k];
        }
    } else {
        const int end = min(beg + per, n);
        for (int i = beg; i < end; ++i) {
            const int u = a[i];
            a[i] = excl;
            excl += u;
        }
    }
    __syncthreads();
    return total;
}

// Out of line: the planner calls it at a dozen places, and five inlined
// variants at each made its code several times larger than the instruction
// caches, so that its one-after-another steps waited on instruction fetch.
static __device__ __noinline__ int block_exscan(int *a, int n, int *wsum)
{
    const int nt = blockDim.x;
    if (n <= nt) return block_exscan_per<1>(a, n, wsum, 1);
    if (n <= 2 * nt) return block_exscan_per<2>(a, n, wsum, 2);
    if (n <= 3 * nt) return block_exscan_per<3>(a, n, wsum, 3);
    if (n <= 4 * nt) return block_exscan_per<4>(a, n, wsum, 4);
    return block_exscan_per<0>(a, n, wsum, (n + nt - 1) / nt);
}

// Rows of the plan's prefetched replicas, grouped by expert, built by one
// block in shared memory (used by the replica-gradient reduce and the weight
// prefetch): for i < n (the return value), expert s_e[i] -- the plan's
// rep_home_list order, or -1 where take(e) rejects it -- has the replica
// rows s_row[s_off[i] .. s_off[i+1]) = r*B + b (b = slot - L < B) in
// ascending host rank order.  Every count and index read from the plan is
// clamped: s_row holds at most max_list rows.  An empty plan gives 0.
// Every thread of the block must call it (two barriers of its own, one of
// the scan's).  s_e: MOONEP_MAX_E ints, s_off: MOONEP_MAX_E + 1, wsum: 32.
template <typename Take>
__device__ int replica_lists(const moonep_plan_t &p, int E, int L, int B, int R, Take take, int *s_e, int *s_off,
                             int *s_row, int max_list, int *wsum)
{
    const int status = __ldg(p.info + MOONEP_INFO_STATUS);
    if (status & ST_EMPTY_PLAN) return 0;
    const int n_exp = min(max(__ldg(p.info + MOONEP_INFO_N_REP_EXPERTS), 0), E);
    if (n_exp == 0) return 0;
    const int tid = threadIdx.x, nh = 2 * E + R;
    for (int i = tid; i <= n_exp; i += blockDim.x) {
        int c = 0, e = -1;
        if (i < n_exp) {
            e = __ldg(p.rep_home_list + i);
            if (e >= 0 && e < E && !take(e)) e = -1;
            if (e >= 0 && e < E) {
                const int home = e / L;
                const int h0 = max(0, __ldg(p.host_ptr + e)), h1 = min(nh, __ldg(p.host_ptr + e + 1));
                for (int h = h0; h < h1; ++h) {
                    const int r = __ldg(p.host_rank + h), b = __ldg(p.host_slot + h) - L;
                    c += (r != home && r >= 0 && r < R && b >= 0 && b < B);
                }
            }
        }
        if (i < n_exp) s_e[i] = e;
        s_off[i] = c;
    }
    __syncthreads();
    block_exscan(s_off, n_exp + 1, wsum);
    for (int i = tid; i < n_exp; i += blockDim.x) {
        const int e = s_e[i];
        if (e < 0 || e >= E) continue;
        const int home = e / L;
        int o = s_off[i];
        const int h0 = max(0, __ldg(p.host_ptr + e)), h1 = min(nh, __ldg(p.host_ptr + e + 1));
        for (int h = h0; h < h1; ++h) {
            const int r = __ldg(p.host_rank + h), b = __ldg(p.host_slot + h) - L;
            if (r != home && r >= 0 && r < R && b >= 0 && b < B && o < max_list) s_row[o++] = r * B + b;
        }
    }
    __syncthreads();
    return n_exp;
}

}  // namespace moonep
