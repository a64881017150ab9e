// Replica-gradient reduction (sm_100a).
//
// MoonEP article ("Moonshot AI Open-Sources MoonEP: A Perfectly Balanced
// Expert Parallelism Library for MoE Training"), explainer memory tab,
// training branch: duplicated experts' gradients land in an fp32 reduce
// buffer mapped as [R, B, ...]; they are pulled back to the home expert and
// the buffer rows are zeroed for the next microbatch.
//
// Work items are (expert with prefetched replicas, element chunk); the
// expert list and its hosts come from the plan on the device, so the launch
// needs no host synchronisation.  Each element is read from home_grad and
// every replica once, summed with separate fp32 adds in ascending host rank
// order, written once, and the replica elements are overwritten with zeros.
#include "common.cuh"

namespace moonep {

constexpr int REDUCE_THREADS = 256;
constexpr int REDUCE_UNROLL = 2;
constexpr int REDUCE_GROUP = 4;
constexpr int REDUCE_MAX_LIST = 2048;  // >= E + R - 1 >= prefetched replicas

struct ReduceParams {
    moonep_plan_t p;
    int *status;        // the plan's status word (for MOONEP_ST_ROW_RANGE)
    int L, B, E, R, n_hosts;
    long long P;        // elements per gradient row
    long long chunk;    // vectors per work item
};

// Where the gradient rows live.  The replica row of slot b of rank r is
// reduce-buffer row r * B + b.
// One GPU: reduce_buf [R, B, P] and home_grad [E, P], every expert reduced.
struct FlatGrads {
    static constexpr bool may_skip = false;  // rep() never returns null
    float *reduce_buf, *home_grad;
    __device__ __forceinline__ bool takes(int e) const { return true; }
    template <typename V>
    __device__ __forceinline__ V *home(int e, long long PV) const
    {
        return reinterpret_cast<V *>(home_grad) + (long long)e * PV;
    }
    template <typename V>
    __device__ __forceinline__ V *rep(int row, long long PV) const
    {
        return reinterpret_cast<V *>(reduce_buf) + (long long)row * PV;
    }
};

// Expert parallelism, on home rank `rank`: its own experts only, home_grad
// [L, P] local, each rank's reduce buffer [B, P] reached through a device
// array of R pointers (peer memory).  A null or misaligned pointer is
// reported (MOONEP_ST_ROW_RANGE) and its rows are skipped.
struct RankGrads {
    static constexpr bool may_skip = true;
    float *const *reduce_bufs;
    float *home_grad;
    int rank, L, B;
    FastDiv fB;
    __device__ __forceinline__ bool takes(int e) const { return e / L == rank; }
    template <typename V>
    __device__ __forceinline__ V *home(int e, long long PV) const
    {
        return reinterpret_cast<V *>(home_grad) + (long long)(e - rank * L) * PV;
    }
    template <typename V>
    __device__ __forceinline__ V *rep(int row, long long PV) const
    {
        const int r = (int)fdiv((uint32_t)row, fB);
        float *b = reduce_bufs[r];
        if (b == nullptr || (reinterpret_cast<uintptr_t>(b) & (sizeof(V) - 1))) return nullptr;
        return reinterpret_cast<V *>(b) + (long long)(row - r * B) * PV;
    }
};

template <typename V>
__device__ __forceinline__ V vadd(const V &a, const V &b);
template <>
__device__ __forceinline__ float4 vadd<float4>(const float4 &a, const float4 &b)
{
    return make_float4(__fadd_rn(a.x, b.x), __fadd_rn(a.y, b.y), __fadd_rn(a.z, b.z), __fadd_rn(a.w, b.w));
}
template <>
__device__ __forceinline__ float vadd<float>(const float &a, const float &b)
{
    return __fadd_rn(a, b);
}
template <typename V>
__device__ __forceinline__ V vzero();
template <>
__device__ __forceinline__ float4 vzero<float4>() { return make_float4(0.f, 0.f, 0.f, 0.f); }
template <>
__device__ __forceinline__ float vzero<float>() { return 0.f; }

template <typename V, typename G>
__global__ void __launch_bounds__(REDUCE_THREADS) reduce_kernel(ReduceParams a, G gr)
{
    // Per block, once: for every expert with prefetched replicas, the list
    // of its reduce_buf rows (r*B + b) in ascending host rank order.
    __shared__ int s_e[MOONEP_MAX_E];
    __shared__ int s_off[MOONEP_MAX_E + 1];
    __shared__ int s_row[REDUCE_MAX_LIST];
    __shared__ int s_wsum[32];
    const int tid = threadIdx.x;
    const int n_exp = replica_lists(a.p, a.E, a.L, a.B, a.R, [&](int e) { return gr.takes(e); }, s_e, s_off, s_row,
                                    REDUCE_MAX_LIST, s_wsum);
    if (n_exp == 0) return;

    constexpr int W = sizeof(V) / sizeof(float);
    const long long PV = a.P / W;  // vectors per row
    const long long nchunks = (PV + a.chunk - 1) / a.chunk;
    const long long n_items = (long long)n_exp * nchunks;

    // Phase 1: sums into home_grad.  Phase 2: zero the replica rows of the
    // same items.  Interleaving the zero stores with the summing loads per
    // element halves DRAM throughput on B200 (measured); separated phases
    // each stream at full rate.  The block zeroes only chunks it has itself
    // summed, so program order keeps every read before its zeroing store.
    for (long long item = blockIdx.x; item < n_items; item += gridDim.x) {
        const int ei = (int)(item / nchunks);
        const long long ci = item - (long long)ei * nchunks;
        const int e = s_e[ei];
        if (e < 0 || e >= a.E) continue;
        const int r0 = s_off[ei], n = min(s_off[ei + 1], REDUCE_MAX_LIST) - r0;
        V *home_row = gr.template home<V>(e, PV);
        const long long v0 = ci * a.chunk;
        const long long v1 = min(PV, v0 + a.chunk);
        for (long long v = v0 + tid; v < v1; v += (long long)REDUCE_THREADS * REDUCE_UNROLL) {
            V acc[REDUCE_UNROLL];
#pragma unroll
            for (int u = 0; u < REDUCE_UNROLL; ++u) {
                const long long x = v + (long long)u * REDUCE_THREADS;
                if (x < v1) acc[u] = home_row[x];
            }
            // replicas in groups of REDUCE_GROUP: every load of a group is in
            // flight before the adds, which keep ascending host rank order
            for (int m0 = 0; m0 < n; m0 += REDUCE_GROUP) {
                V r[REDUCE_GROUP][REDUCE_UNROLL];
                bool live[REDUCE_GROUP];
#pragma unroll
                for (int m = 0; m < REDUCE_GROUP; ++m) {
                    const V *rrow = gr.template rep<V>(s_row[r0 + min(m0 + m, n - 1)], PV);
                    live[m] = m0 + m < n && (!G::may_skip || rrow != nullptr);
#pragma unroll
                    for (int u = 0; u < REDUCE_UNROLL; ++u) {
                        const long long x = v + (long long)u * REDUCE_THREADS;
                        if (live[m] && x < v1) r[m][u] = rrow[x];
                    }
                }
#pragma unroll
                for (int m = 0; m < REDUCE_GROUP; ++m)
#pragma unroll
                    for (int u = 0; u < REDUCE_UNROLL; ++u) {
                        const long long x = v + (long long)u * REDUCE_THREADS;
                        if (live[m] && x < v1) acc[u] = vadd(acc[u], r[m][u]);
                    }
            }
#pragma unroll
            for (int u = 0; u < REDUCE_UNROLL; ++u) {
                const long long x = v + (long long)u * REDUCE_THREADS;
                if (x < v1) home_row[x] = acc[u];
            }
        }
    }
    for (long long item = blockIdx.x; item < n_items; item += gridDim.x) {
        const int ei = (int)(item / nchunks);
        const long long ci = item - (long long)ei * nchunks;
        const int e = s_e[ei];
        if (e < 0 || e >= a.E) continue;
        const int r0 = s_off[ei], n = min(s_off[ei + 1], REDUCE_MAX_LIST) - r0;
        const long long v0 = ci * a.chunk;
        const long long v1 = min(PV, v0 + a.chunk);
        for (int m = 0; m < n; ++m) {
            V *rrow = gr.template rep<V>(s_row[r0 + m], PV);
            if (G::may_skip && rrow == nullptr) {
                if (tid == 0 && ci == 0) atomicOr(a.status, MOONEP_ST_ROW_RANGE);
                continue;
            }
            for (long long v = v0 + tid; v < v1; v += (long long)REDUCE_THREADS * REDUCE_UNROLL) {
#pragma unroll
                for (int u = 0; u < REDUCE_UNROLL; ++u) {
                    const long long x = v + (long long)u * REDUCE_THREADS;
                    if (x < v1) rrow[x] = vzero<V>();
                }
            }
        }
    }
}

static int device_sms()
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
    return sms[dev];
}

template <typename G>
static int reduce_with(const Dims &d, const moonep_plan_t &p, const G &gr, bool vec, long long P, cudaStream_t st)
{
    ReduceParams a;
    a.p = p;
    a.status = p.info + MOONEP_INFO_STATUS;
    a.L = d.L;
    a.B = d.B;
    a.E = d.E;
    a.R = d.R;
    a.n_hosts = 2 * d.E + d.R;
    a.P = P;
    // eight waves of blocks: the block scheduler refills SMs as blocks
    // finish, which evens out the tail of the item loop (4 % over one wave)
    const int grid = device_sms() * (2048 / REDUCE_THREADS) * 8;
    if (vec) {
        a.chunk = (long long)REDUCE_THREADS * REDUCE_UNROLL * 8;
        reduce_kernel<float4, G><<<grid, REDUCE_THREADS, 0, st>>>(a, gr);
    } else {
        a.chunk = (long long)REDUCE_THREADS * REDUCE_UNROLL * 32;
        reduce_kernel<float, G><<<grid, REDUCE_THREADS, 0, st>>>(a, gr);
    }
    return cudaGetLastError() == cudaSuccess ? MOONEP_OK : MOONEP_ERR_CUDA;
}

int launch_reduce(const Dims &d, const moonep_plan_t &p, float *reduce_buf, float *home_grad, long long P,
                  cudaStream_t st)
{
    const bool vec = (P % 4 == 0) && (reinterpret_cast<uintptr_t>(reduce_buf) % 16 == 0) &&
                     (reinterpret_cast<uintptr_t>(home_grad) % 16 == 0);
    return reduce_with(d, p, FlatGrads{reduce_buf, home_grad}, vec, P, st);
}

// Expert parallelism: home rank `rank` pulls its experts' replica rows from
// every rank's reduce buffer (reduce_bufs: device array of R pointers, each
// 16-byte aligned for the vector path) into its local home_grad [L, P].
int launch_reduce_ep(const Dims &d, int rank, const moonep_plan_t &p, float *const *reduce_bufs,
                     float *home_grad, long long P, cudaStream_t st)
{
    const bool vec = (P % 4 == 0) && (reinterpret_cast<uintptr_t>(home_grad) % 16 == 0);
    RankGrads gr{reduce_bufs, home_grad, rank, d.L, d.B, make_fastdiv((uint32_t)d.B)};
    return reduce_with(d, p, gr, vec, P, st);
}

}  // namespace moonep
