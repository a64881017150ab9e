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
};

// Chunks per group: the assignment pass sums at most CHUNK_GROUP - 1
// per-chunk counts on top of a group prefix.
constexpr int CHUNK_GROUP = 16;

// Workspace layout (bytes from the workspace base; 256-byte aligned parts).
struct WsLayout {
    size_t ticket;     // int32: CTAs of the histogram kernel that finished
    size_t status;     // int32: status bits collected by the histogram kernel
    size_t gs;         // int32 [ngroups][E]: per-group expert counts (atomic sums)
    size_t gp;         // int32 [ngroups][E]: exclusive prefix of gs over groups
    size_t cc;         // int32 [nchunk][E]: per-chunk expert counts
    size_t host_dst0;  // int32 [2E+R]: rank*C + slot_offset - host_start per host
    size_t total;
};

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

__host__ inline WsLayout ws_layout(const Dims &d)
{
    WsLayout w;
    size_t o = 0;
    w.ticket = o; o += 4;
    w.status = o; o += 4;
    o = align256(o);
    w.gs = o; o = align256(o + sizeof(int32_t) * (size_t)d.ngroups * d.E);
    w.gp = o; o = align256(o + sizeof(int32_t) * (size_t)d.ngroups * d.E);
    w.cc = o; o = align256(o + sizeof(int32_t) * (size_t)d.nchunk * d.E);
    w.host_dst0 = o; o = align256(o + sizeof(int32_t) * (size_t)(2 * d.E + d.R));
    w.total = o;
    return w;
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
        int y = __shfl_up_sync(FULL_MASK, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) wsum[w] = x;
    __syncthreads();
    if (w == 0) {
        int v = lane < nw ? wsum[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int y = __shfl_up_sync(FULL_MASK, v, o);
            if (lane >= o) v += y;
        }
        if (lane < nw) wsum[lane] = v;
    }
    __syncthreads();
    int excl = x - local + (w > 0 ? wsum[w - 1] : 0);
    const int total = wsum[nw - 1];
    for (int i = beg; i < end; ++i) {
        int v = a[i];
        a[i] = excl;
        excl += v;
    }
    __syncthreads();
    return total;
}

}  // namespace moonep
