// Replica weight prefetch (sm_100a).
//
// MoonEP article ("Moonshot AI Open-Sources MoonEP: A Perfectly Balanced
// Expert Parallelism Library for MoE Training"), "The core idea": duplicated
// experts are prefetched before expert computation; explainer, memory tab:
// the prefetch slots are rows [E, E+B) of one contiguous weight pool per
// projection, and a rank needing more than B foreign experts reads the
// overflow from the home copy.  Here each rank's B prefetch rows form
// pool[r][0..B), the home experts stay in `weights`, and a per-slot table
// tells the expert computation which row to use.
//
// The copy is an HBM stream of 16-byte vectors over work items (expert with
// prefetched replicas, element chunk) taken from the plan on the device, so
// the launch needs no host synchronisation: each chunk of an expert's row is
// read once and written to every one of its prefetched replicas, so the
// bytes moved are the minimum, (experts with replicas + replicas) x row.
#include "common.cuh"

namespace moonep {

constexpr int PF_THREADS = 256;
constexpr int PF_UNROLL = 4;
constexpr int PF_MAX_LIST = 2048;  // >= E + R - 1 >= prefetched replicas

struct PrefetchParams {
    moonep_plan_t p;
    const uint8_t *weights;
    uint8_t *pool;
    int *slot_wrow;
    int R, E, L, B;
    long long row_bytes;  // P * 2
    long long chunk;      // bytes per work item
};

template <typename V>
__global__ void __launch_bounds__(PF_THREADS) prefetch_kernel(PrefetchParams a)
{
    __shared__ int s_e[MOONEP_MAX_E];
    __shared__ int s_off[MOONEP_MAX_E + 1];
    __shared__ int s_row[PF_MAX_LIST];
    __shared__ int s_wsum[32];
    const int status = __ldg(a.p.info + MOONEP_INFO_STATUS);
    const bool invalid = (status & ST_EMPTY_PLAN) != 0;
    const long long gtid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long gstride = (long long)gridDim.x * blockDim.x;

    // weight row of every slot: home e, pool E + r*B + b, overflow e (read-through)
    for (long long x = gtid; x < (long long)a.R * a.E; x += gstride) {
        const int r = (int)(x / a.E), s = (int)(x - (long long)r * a.E);
        const int e = invalid ? -1 : __ldg(a.p.slot_expert + x);
        int row = -1;
        if (e >= 0) row = (s < a.L) ? e : (s - a.L < a.B ? a.E + r * a.B + (s - a.L) : e);
        a.slot_wrow[x] = row;
    }
    // per block: every expert with prefetched replicas and their pool rows r*B + b
    const int n_exp = replica_lists(a.p, a.E, a.L, a.B, a.R, [](int) { return true; }, s_e, s_off, s_row,
                                    PF_MAX_LIST, s_wsum);
    if (n_exp == 0) return;

    constexpr int W = sizeof(V);
    const long long vrow = a.row_bytes / W;
    const long long vchunk = a.chunk / W;
    const long long nchunks = (vrow + vchunk - 1) / vchunk;
    const long long n_items = (long long)n_exp * nchunks;
    for (long long item = blockIdx.x; item < n_items; item += gridDim.x) {
        const int ei = (int)(item / nchunks);
        const long long ci = item - (long long)ei * nchunks;
        const int e = s_e[ei];
        if (e < 0 || e >= a.E) continue;
        const int r0 = s_off[ei], n = min(s_off[ei + 1], PF_MAX_LIST) - r0;
        const V *src = reinterpret_cast<const V *>(a.weights + (long long)e * a.row_bytes);
        const long long v0 = ci * vchunk, v1 = min(vrow, v0 + vchunk);
        for (long long v = v0 + threadIdx.x; v < v1; v += (long long)PF_THREADS * PF_UNROLL) {
            V t[PF_UNROLL];
#pragma unroll
            for (int u = 0; u < PF_UNROLL; ++u) {
                const long long x = v + (long long)u * PF_THREADS;
                if (x < v1) t[u] = src[x];
            }
            for (int m = 0; m < n; ++m) {
                V *dst = reinterpret_cast<V *>(a.pool + (long long)s_row[r0 + m] * a.row_bytes);
#pragma unroll
                for (int u = 0; u < PF_UNROLL; ++u) {
                    const long long x = v + (long long)u * PF_THREADS;
                    if (x < v1) dst[x] = t[u];
                }
            }
        }
    }
}

// Expert parallelism, on rank `rank`: each of its prefetched replicas (list
// entries on this rank with ordinal b < B) pulls its expert's weight row from
// the home rank's [L, P] weights (peer memory, through the pointer array)
// into the local pool row b.  The local slot table: home slot s -> s (own
// weights), prefetched replica -> L + b (own pool), overflow replica ->
// L + B + e (expert e read through from its home rank), unused -> -1.
struct EpPrefetchParams {
    moonep_plan_t p;
    const uint8_t *const *weights;  // [R] pointers to each rank's [L, P] bf16 weights
    uint8_t *pool;                  // this rank's [B, P]
    int *slot_wrow;                 // this rank's [E]
    int R, E, L, B, rank;
    long long row_bytes, chunk;
};

template <typename V>
__global__ void __launch_bounds__(PF_THREADS) ep_prefetch_kernel(EpPrefetchParams a)
{
    const int status = __ldg(a.p.info + MOONEP_INFO_STATUS);
    const bool invalid = (status & ST_EMPTY_PLAN) != 0;
    const long long gtid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long gstride = (long long)gridDim.x * blockDim.x;
    for (long long s = gtid; s < a.E; s += gstride) {
        const int e = invalid ? -1 : __ldg(a.p.slot_expert + (long long)a.rank * a.E + s);
        int row = -1;
        if (e >= 0 && e < a.E) row = (s < a.L) ? (int)s : (s - a.L < a.B ? (int)s : a.L + a.B + e);
        a.slot_wrow[s] = row;
    }
    if (invalid) return;
    const int n_rep = min(max(__ldg(a.p.info + MOONEP_INFO_N_REP), 0), a.E + a.R);
    constexpr int W = sizeof(V);
    const long long vrow = a.row_bytes / W, vchunk = a.chunk / W;
    const long long nchunks = (vrow + vchunk - 1) / vchunk;
    const long long n_items = (long long)n_rep * nchunks;
    for (long long item = blockIdx.x; item < n_items; item += gridDim.x) {
        const int q = (int)(item / nchunks);
        if (__ldg(a.p.rep_rank + q) != a.rank) continue;
        const int b = __ldg(a.p.rep_slot + q) - a.L, e = __ldg(a.p.rep_expert + q);
        if (b < 0 || b >= a.B || e < 0 || e >= a.E) continue;  // overflow: read through
        const int h = e / a.L;
        const uint8_t *wb = a.weights[h];
        if (wb == nullptr || (reinterpret_cast<uintptr_t>(wb) & (W - 1))) {
            if (threadIdx.x == 0) atomicOr(a.p.info + MOONEP_INFO_STATUS, MOONEP_ST_ROW_RANGE);
            continue;
        }
        const long long ci = item - (long long)q * nchunks;
        const V *src = reinterpret_cast<const V *>(wb + (long long)(e - h * a.L) * a.row_bytes);
        V *dst = reinterpret_cast<V *>(a.pool + (long long)b * a.row_bytes);
        const long long v0 = ci * vchunk, v1 = min(vrow, v0 + vchunk);
        for (long long v = v0 + threadIdx.x; v < v1; v += (long long)PF_THREADS * PF_UNROLL) {
            V t[PF_UNROLL];
#pragma unroll
            for (int u = 0; u < PF_UNROLL; ++u) {
                const long long x = v + (long long)u * PF_THREADS;
                if (x < v1) t[u] = src[x];
            }
#pragma unroll
            for (int u = 0; u < PF_UNROLL; ++u) {
                const long long x = v + (long long)u * PF_THREADS;
                if (x < v1) dst[x] = t[u];
            }
        }
    }
}

int launch_prefetch(const Dims &d, const moonep_plan_t &p, const uint16_t *weights, uint16_t *pool,
                    int32_t *slot_wrow, long long P, cudaStream_t st)
{
    static int sms[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) dev = 0;
    if (!sms[dev]) {
        int v = 0;
        cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
        sms[dev] = v > 0 ? v : 148;
    }
    PrefetchParams a;
    a.p = p;
    a.weights = reinterpret_cast<const uint8_t *>(weights);
    a.pool = reinterpret_cast<uint8_t *>(pool);
    a.slot_wrow = slot_wrow;
    a.R = d.R;
    a.E = d.E;
    a.L = d.L;
    a.B = d.B;
    a.row_bytes = P * 2;
    const bool vec = (a.row_bytes % 16 == 0) && (reinterpret_cast<uintptr_t>(weights) % 16 == 0) &&
                     (reinterpret_cast<uintptr_t>(pool) % 16 == 0);
    // eight waves of blocks: the block scheduler refills SMs as blocks
    // finish, which evens out the tail of the item loop (9 % over one wave)
    const int grid = sms[dev] * (2048 / PF_THREADS) * 8;
    if (vec) {
        a.chunk = 256 * 1024;
        prefetch_kernel<uint4><<<grid, PF_THREADS, 0, st>>>(a);
    } else {
        a.chunk = 64 * 1024;
        prefetch_kernel<uint16_t><<<grid, PF_THREADS, 0, st>>>(a);
    }
    return cudaGetLastError() == cudaSuccess ? MOONEP_OK : MOONEP_ERR_CUDA;
}

int launch_prefetch_ep(const Dims &d, int rank, const moonep_plan_t &p, const uint16_t *const *weights,
                       uint16_t *pool, int32_t *slot_wrow, long long P, cudaStream_t st)
{
    int dev = 0, sms = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (sms <= 0) sms = 148;
    EpPrefetchParams a;
    a.p = p;
    a.weights = reinterpret_cast<const uint8_t *const *>(weights);
    a.pool = reinterpret_cast<uint8_t *>(pool);
    a.slot_wrow = slot_wrow;
    a.R = d.R;
    a.E = d.E;
    a.L = d.L;
    a.B = d.B;
    a.rank = rank;
    a.row_bytes = P * 2;
    const bool vec = (a.row_bytes % 16 == 0) && (reinterpret_cast<uintptr_t>(pool) % 16 == 0);
    const int grid = sms * (2048 / PF_THREADS) * 8;
    if (vec) {
        a.chunk = 256 * 1024;
        ep_prefetch_kernel<uint4><<<grid, PF_THREADS, 0, st>>>(a);
    } else {
        a.chunk = 64 * 1024;
        ep_prefetch_kernel<uint16_t><<<grid, PF_THREADS, 0, st>>>(a);
    }
    return cudaGetLastError() == cudaSuccess ? MOONEP_OK : MOONEP_ERR_CUDA;
}

}  // namespace moonep
