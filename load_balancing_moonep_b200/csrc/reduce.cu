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
    float *reduce_buf;
    float *home_grad;
    const int *host_ptr, *host_rank, *host_slot, *rep_home_list, *info;
    int L, B, E, R, n_hosts;
    long long P;        // elements per gradient row
    long long chunk;    // vectors per work item
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

template <typename V>
__global__ void __launch_bounds__(REDUCE_THREADS) reduce_kernel(ReduceParams a)
{
    // Per block, once: for every expert with prefetched replicas, the list
    // of its reduce_buf rows (r*B + b) in ascending host rank order.
    __shared__ int s_e[MOONEP_MAX_E];
    __shared__ int s_off[MOONEP_MAX_E + 1];
    __shared__ int s_row[REDUCE_MAX_LIST];
    __shared__ int s_wsum[32];
    const int status = __ldg(a.info + MOONEP_INFO_STATUS);
    if (status & ST_EMPTY_PLAN) return;
    const int n_exp = min(max(__ldg(a.info + MOONEP_INFO_N_REP_EXPERTS), 0), a.E);
    if (n_exp == 0) return;
    const int tid = threadIdx.x;
    for (int i = tid; i <= n_exp; i += blockDim.x) {
        int c = 0, e = -1;
        if (i < n_exp) {
            e = __ldg(a.rep_home_list + i);
            if (e >= 0 && e < a.E) {
                const int home = e / a.L;
                const int h0 = max(0, __ldg(a.host_ptr + e)), h1 = min(a.n_hosts, __ldg(a.host_ptr + e + 1));
                for (int h = h0; h < h1; ++h) {
                    const int r = __ldg(a.host_rank + h), b = __ldg(a.host_slot + h) - a.L;
                    c += (r != home && r >= 0 && r < a.R && b >= 0 && b < a.B);
                }
            }
        }
        if (i < n_exp) s_e[i] = e;
        s_off[i] = c;
    }
    __syncthreads();
    block_exscan(s_off, n_exp + 1, s_wsum);
    for (int i = tid; i < n_exp; i += blockDim.x) {
        const int e = s_e[i];
        if (e < 0 || e >= a.E) continue;
        const int home = e / a.L;
        int o = s_off[i];
        const int h0 = max(0, __ldg(a.host_ptr + e)), h1 = min(a.n_hosts, __ldg(a.host_ptr + e + 1));
        for (int h = h0; h < h1; ++h) {
            const int r = __ldg(a.host_rank + h), b = __ldg(a.host_slot + h) - a.L;
            if (r != home && r >= 0 && r < a.R && b >= 0 && b < a.B && o < REDUCE_MAX_LIST)
                s_row[o++] = r * a.B + b;
        }
    }
    __syncthreads();

    constexpr int W = sizeof(V) / sizeof(float);
    const long long PV = a.P / W;  // vectors per row
    const long long nchunks = (PV + a.chunk - 1) / a.chunk;
    const long long n_items = (long long)n_exp * nchunks;
    V *rb = reinterpret_cast<V *>(a.reduce_buf);
    V *hg = reinterpret_cast<V *>(a.home_grad);

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
        V *home_row = hg + (long long)e * PV;
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
#pragma unroll
                for (int m = 0; m < REDUCE_GROUP; ++m) {
                    const V *rrow = rb + (long long)s_row[r0 + min(m0 + m, n - 1)] * PV;
#pragma unroll
                    for (int u = 0; u < REDUCE_UNROLL; ++u) {
                        const long long x = v + (long long)u * REDUCE_THREADS;
                        if (m0 + m < n && x < v1) r[m][u] = rrow[x];
                    }
                }
#pragma unroll
                for (int m = 0; m < REDUCE_GROUP; ++m)
#pragma unroll
                    for (int u = 0; u < REDUCE_UNROLL; ++u) {
                        const long long x = v + (long long)u * REDUCE_THREADS;
                        if (m0 + m < n && x < v1) acc[u] = vadd(acc[u], r[m][u]);
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
            V *rrow = rb + (long long)s_row[r0 + m] * PV;
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

int launch_reduce(const Dims &d, const moonep_plan_t &p, float *reduce_buf, float *home_grad, long long P,
                  cudaStream_t st)
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
    ReduceParams a;
    a.reduce_buf = reduce_buf;
    a.home_grad = home_grad;
    a.host_ptr = p.host_ptr;
    a.host_rank = p.host_rank;
    a.host_slot = p.host_slot;
    a.rep_home_list = p.rep_home_list;
    a.info = p.info;
    a.L = d.L;
    a.B = d.B;
    a.E = d.E;
    a.R = d.R;
    a.n_hosts = 2 * d.E + d.R;
    a.P = P;
    const bool vec = (P % 4 == 0) && (reinterpret_cast<uintptr_t>(reduce_buf) % 16 == 0) &&
                     (reinterpret_cast<uintptr_t>(home_grad) % 16 == 0);
    // eight waves of blocks: the block scheduler refills SMs as blocks
    // finish, which evens out the tail of the item loop (4 % over one wave)
    const int grid = sms[dev] * (2048 / REDUCE_THREADS) * 8;
    if (vec) {
        a.chunk = (long long)REDUCE_THREADS * REDUCE_UNROLL * 8;
        reduce_kernel<float4><<<grid, REDUCE_THREADS, 0, st>>>(a);
    } else {
        a.chunk = (long long)REDUCE_THREADS * REDUCE_UNROLL * 32;
        reduce_kernel<float><<<grid, REDUCE_THREADS, 0, st>>>(a);
    }
    return cudaGetLastError() == cudaSuccess ? MOONEP_OK : MOONEP_ERR_CUDA;
}

}  // namespace moonep
