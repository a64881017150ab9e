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
};

// Chunks per group: the assignment pass sums at most CHUNK_GROUP - 1
// per-chunk counts on top of a group prefix.
constexpr int CHUNK_GROUP = 16;

// Workspace layout (bytes from the workspace base; 256-byte aligned parts).
struct WsLayout {
    size_t hdr;        // int32[4]: ticket, status, parity of the group buffers, spare
    size_t t_acc;      // int32 [E]: expert totals accumulated by the histogram pass
    size_t gs;         // int32 [2][ngroups][E]: per-group expert counts, double-buffered
    size_t cc;         // int32 [nchunk][E]: per-chunk expert counts
    size_t host_dst0;  // int32 [2E+R]: rank*C + slot_offset - host_start per host
    size_t sc_base;    // int32 [R+1]: first compact used slot of each rank
    size_t sc_exp;     // int32 [2E+R]: expert of each used slot (compact)
    size_t sc_cnt;     // int32 [2E+R]: rows of each used slot
    size_t sc_off;     // int32 [2E+R]: slot offset of each used slot
    size_t total;
};
enum { WS_TICKET = 0, WS_STATUS = 1, WS_PARITY = 2 };

// Status bits after which every later call treats the plan as empty.
constexpr int ST_EMPTY_PLAN = MOONEP_ST_EXPERT_ID_RANGE | MOONEP_ST_WORKSPACE;

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

__host__ inline WsLayout ws_layout(const Dims &d)
{
    WsLayout w;
    const size_t i4 = sizeof(int32_t), nh = (size_t)(2 * d.E + d.R);
    size_t o = 0;
    w.hdr = o; o = align256(o + 4 * i4);
    w.t_acc = o; o = align256(o + i4 * d.E);
    w.gs = o; o = align256(o + i4 * 2 * (size_t)d.ngroups * d.E);
    w.cc = o; o = align256(o + i4 * (size_t)d.nchunk * d.E);
    w.host_dst0 = o; o = align256(o + i4 * nh);
    w.sc_base = o; o = align256(o + i4 * (d.R + 1));
    w.sc_exp = o; o = align256(o + i4 * nh);
    w.sc_cnt = o; o = align256(o + i4 * nh);
    w.sc_off = o; o = align256(o + i4 * nh);
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
// (keys in [0, 2^nbits)); lanes with valid == false match nobody.
__device__ __forceinline__ unsigned peers_of(int key, bool valid, int nbits)
{
    unsigned m = __ballot_sync(0xffffffffu, valid);
    for (int b = 0; b < nbits; ++b) {
        const bool bit = (key >> b) & 1;
        const unsigned bb = __ballot_sync(0xffffffffu, bit);
        m &= bit ? bb : ~bb;
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

// Exclusive prefix sum of a[0..n) in shared memory, in place; returns the
// total.  Every thread of the block must call it.  wsum: >= 32 ints of smem.
// Two barriers: after the per-warp scans every thread reads all warp totals.
__device__ inline int block_exscan(int *a, int n, int *wsum)
{
    const int tid = threadIdx.x, nt = blockDim.x;
    const int lane = tid & 31, w = tid >> 5, nw = nt >> 5;
    const int per = (n + nt - 1) / nt;
    const int beg = min(tid * per, n), end = min(beg + per, n);
    int local = 0;
    for (int i = beg; i < end; ++i) local += a[i];
    int x = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(FULL_MASK, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) wsum[w] = x;
    __syncthreads();
    int before = 0, total = 0;
    for (int j = 0; j < nw; ++j) {
        const int v = wsum[j];
        total += v;
        before += j < w ? v : 0;
    }
    int excl = x - local + before;
    for (int i = beg; i < end; ++i) {
        const int v = a[i];
        a[i] = excl;
        excl += v;
    }
    __syncthreads();
    return total;
}

}  // namespace moonep
