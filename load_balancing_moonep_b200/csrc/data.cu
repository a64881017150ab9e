// Fused permute / unpermute and their backward (sm_100a).
//
// MoonEP article ("Moonshot AI Open-Sources MoonEP: A Perfectly Balanced
// Expert Parallelism Library for MoE Training", "The core idea: dynamic
// redundant experts", zero copy and static shapes): tokens are written
// straight into their expert-grouped rows of a fixed [R, S*K, H] buffer, and
// the unpermute reads them back from there, with no intermediate copy.
//
// All three kernels are HBM-bound streams of 16-byte vectors.  One warp owns
// one token at a time (grid sized to fill every SM): its K destination rows
// are fetched once by lanes 0..K-1 and broadcast with shuffles, then the
// token's row is walked in 16-byte vectors, U vectors per lane in flight.
//   dispatch     read the row once, store it K times;
//   combine      read K rows, fp32 fused multiply-add in k order, store once;
//   combine_bwd  read dy once and K expert-output rows, store K scaled rows
//                and K dot products (fp32, fixed reduction tree).
#include <cuda_bf16.h>

#include "common.cuh"

namespace moonep {

constexpr int DATA_THREADS = 256;

__device__ __forceinline__ uint4 ld_stream(const uint4 *p)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ void st_vec(uint4 *p, const uint4 &v)
{
    asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
                 "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ float bf_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf_hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

// two fp32 -> packed bf16x2, round to nearest even (lo in the low half)
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

__device__ __forceinline__ void unpack8(const uint4 &v, float f[8])
{
    f[0] = bf_lo(v.x); f[1] = bf_hi(v.x);
    f[2] = bf_lo(v.y); f[3] = bf_hi(v.y);
    f[4] = bf_lo(v.z); f[5] = bf_hi(v.z);
    f[6] = bf_lo(v.w); f[7] = bf_hi(v.w);
}

__device__ __forceinline__ uint4 pack8(const float f[8])
{
    uint4 v;
    v.x = pack_bf16x2(f[0], f[1]);
    v.y = pack_bf16x2(f[2], f[3]);
    v.z = pack_bf16x2(f[4], f[5]);
    v.w = pack_bf16x2(f[6], f[7]);
    return v;
}

__device__ __forceinline__ bool plan_invalid(const int *info)
{
    return (*(volatile const int *)(info + MOONEP_INFO_STATUS) & ST_EMPTY_PLAN) != 0;
}

// A row index from the plan outside [0, rows) is never dereferenced: the
// access is skipped and MOONEP_ST_ROW_RANGE is raised.
__device__ __forceinline__ bool row_ok(int row, int rows, int *info)
{
    if ((unsigned)row < (unsigned)rows) return true;
    atomicOr(info + MOONEP_INFO_STATUS, MOONEP_ST_ROW_RANGE);
    return false;
}

// ------------------------------------------------------ buffer addressing

// Where buffer row g (a global row in [0, R*S*K), rank g / (S*K)) lives.
// row() returns nullptr, and raises MOONEP_ST_ROW_RANGE, for a row outside
// [0, rows) or a buffer that cannot be addressed; the caller skips it.

// One allocation holds every rank's rows: the single-GPU layout [R, S*K, H]
// (its base is checked on the host).
template <typename T>
struct FlatRows {
    T *base;
    int vpr;  // 16-byte vectors per row
    __device__ __forceinline__ T *row(int g, int rows, int *info) const
    {
        return row_ok(g, rows, info) ? base + (size_t)g * vpr : nullptr;
    }
};

// Each rank's [S*K, H] buffer is its own allocation, reached through a
// device array of R pointers (peer memory of the other GPUs in expert
// parallelism): row g is local row g - r*C of rank r = g / C.  A null or
// misaligned pointer in the array is reported, never dereferenced.
template <typename T>
struct RankRows {
    T *const *bases;  // [R] device pointers
    FastDiv fC;       // division by C = S*K
    int C;
    int vpr;
    __device__ __forceinline__ T *row(int g, int rows, int *info) const
    {
        if (!row_ok(g, rows, info)) return nullptr;
        const int r = (int)fdiv((uint32_t)g, fC);
        T *b = bases[r];
        if (b == nullptr || (reinterpret_cast<uintptr_t>(b) & 15u)) {
            atomicOr(info + MOONEP_INFO_STATUS, MOONEP_ST_ROW_RANGE);
            return nullptr;
        }
        return b + (size_t)(g - r * C) * vpr;
    }
};

// --------------------------------------------------------------- dispatch

// One warp per token: the row is read once, in U 16-byte vectors per lane,
// and stored to each of the K destination rows (broadcast by shuffles).
// A compile-time K with the K row pointers held in registers measured
// slower on B200 (2.99 vs 2.80 ms at the large shape), so K stays run-time.
template <int U, typename Rows>
__global__ void __launch_bounds__(DATA_THREADS) dispatch_kernel(const uint4 *__restrict__ hidden,
                                                               const Rows buf,
                                                               const int *__restrict__ dst_pos,
                                                               int *info, int tokens, int K, int vpr,
                                                               int rows)
{
    if (plan_invalid(info)) return;
    const int lane = threadIdx.x & 31;
    const int wpb = blockDim.x >> 5;
    const int nw = gridDim.x * wpb;
    for (int t = blockIdx.x * wpb + (threadIdx.x >> 5); t < tokens; t += nw) {
        const int *dp = dst_pos + (size_t)t * K;
        const int dl = lane < K ? __ldg(dp + lane) : 0;
        const uint4 *src = hidden + (size_t)t * vpr;
        for (int c0 = 0; c0 < vpr; c0 += 32 * U) {
            uint4 v[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int c = c0 + u * 32 + lane;
                if (c < vpr) v[u] = ld_stream(src + c);
            }
            for (int k = 0; k < K; ++k) {
                const int dk = k < 32 ? __shfl_sync(FULL_MASK, dl, k) : __ldg(dp + k);
                uint4 *dst = buf.row(dk, rows, info);
                if (dst == nullptr) continue;
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int c = c0 + u * 32 + lane;
                    if (c < vpr) st_vec(dst + c, v[u]);
                }
            }
        }
    }
}

// ---------------------------------------------------------------- combine

// KT > 0: compile-time K (all K loads of a vector issued together);
// KT == 0: any K, one expert row at a time.
template <int KT, int U, typename Rows>
__global__ void __launch_bounds__(DATA_THREADS) combine_kernel(const Rows y,
                                                              const float *__restrict__ w,
                                                              uint4 *__restrict__ out,
                                                              const int *__restrict__ dst_pos, int *info,
                                                              int tokens, int K_rt, int vpr, int rows)
{
    if (plan_invalid(info)) return;
    const int K = KT > 0 ? KT : K_rt;
    const int lane = threadIdx.x & 31;
    const int wpb = blockDim.x >> 5;
    const int nw = gridDim.x * wpb;
    for (int t = blockIdx.x * wpb + (threadIdx.x >> 5); t < tokens; t += nw) {
        const int *dp = dst_pos + (size_t)t * K;
        const float *wp = w + (size_t)t * K;
        const int dl = lane < K ? __ldg(dp + lane) : 0;
        const float wl = lane < K ? __ldg(wp + lane) : 0.0f;
        for (int c0 = 0; c0 < vpr; c0 += 32 * U) {
            float acc[U][8];
#pragma unroll
            for (int u = 0; u < U; ++u)
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[u][j] = 0.0f;
            if constexpr (KT > 0) {
                uint4 v[KT][U];
#pragma unroll
                for (int k = 0; k < KT; ++k) {
                    const int dk = __shfl_sync(FULL_MASK, dl, k);
                    const uint4 *row = y.row(dk, rows, info);
                    const bool ok = row != nullptr;
#pragma unroll
                    for (int u = 0; u < U; ++u) {
                        const int c = c0 + u * 32 + lane;
                        v[k][u] = make_uint4(0u, 0u, 0u, 0u);
                        if (ok && c < vpr) v[k][u] = ld_stream(row + c);
                    }
                }
#pragma unroll
                for (int k = 0; k < KT; ++k) {
                    const float wk = __shfl_sync(FULL_MASK, wl, k);
#pragma unroll
                    for (int u = 0; u < U; ++u) {
                        float f[8];
                        unpack8(v[k][u], f);
#pragma unroll
                        for (int j = 0; j < 8; ++j) acc[u][j] = fmaf(wk, f[j], acc[u][j]);
                    }
                }
            } else {
                for (int k = 0; k < K; ++k) {
                    const int dk = k < 32 ? __shfl_sync(FULL_MASK, dl, k) : __ldg(dp + k);
                    const float wk = k < 32 ? __shfl_sync(FULL_MASK, wl, k) : __ldg(wp + k);
                    const uint4 *row = y.row(dk, rows, info);
                    if (row == nullptr) continue;
#pragma unroll
                    for (int u = 0; u < U; ++u) {
                        const int c = c0 + u * 32 + lane;
                        if (c < vpr) {
                            float f[8];
                            unpack8(ld_stream(row + c), f);
#pragma unroll
                            for (int j = 0; j < 8; ++j) acc[u][j] = fmaf(wk, f[j], acc[u][j]);
                        }
                    }
                }
            }
            uint4 *o = out + (size_t)t * vpr;
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int c = c0 + u * 32 + lane;
                if (c < vpr) st_vec(o + c, pack8(acc[u]));
            }
        }
    }
}

// ------------------------------------------------------- combine backward

__device__ __forceinline__ float dot8(const float a[8], const float b[8])
{
    // products of two bf16 values are exact in fp32; fixed pairwise tree
    const float p0 = a[0] * b[0], p1 = a[1] * b[1], p2 = a[2] * b[2], p3 = a[3] * b[3];
    const float p4 = a[4] * b[4], p5 = a[5] * b[5], p6 = a[6] * b[6], p7 = a[7] * b[7];
    return ((p0 + p1) + (p2 + p3)) + ((p4 + p5) + (p6 + p7));
}

template <int KT, int U, typename YRows, typename BRows>
__global__ void __launch_bounds__(DATA_THREADS) combine_bwd_kernel(
    const uint4 *__restrict__ dy, const float *__restrict__ w, const YRows y,
    const BRows dy_buf, float *__restrict__ dw, const int *__restrict__ dst_pos, int *info,
    int tokens, int vpr, int unscaled, int rows)
{
    if (plan_invalid(info)) return;
    constexpr int K = KT;
    const int lane = threadIdx.x & 31;
    const int wpb = blockDim.x >> 5;
    const int nw = gridDim.x * wpb;
    for (int t = blockIdx.x * wpb + (threadIdx.x >> 5); t < tokens; t += nw) {
        const int *dp = dst_pos + (size_t)t * K;
        const float *wp = w + (size_t)t * K;
        const int dl = lane < K ? __ldg(dp + lane) : 0;
        const float wl = lane < K ? __ldg(wp + lane) : 0.0f;
        float dacc[K];
#pragma unroll
        for (int k = 0; k < K; ++k) dacc[k] = 0.0f;
        const uint4 *g = dy + (size_t)t * vpr;
        for (int c0 = 0; c0 < vpr; c0 += 32 * U) {
            float gf[U][8];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int c = c0 + u * 32 + lane;
                if (c < vpr) unpack8(ld_stream(g + c), gf[u]);
            }
            // all K expert-output rows of this vector slice in flight first
            uint4 yv[K][U];
            unsigned okm = 0;
#pragma unroll
            for (int k = 0; k < K; ++k) {
                const int dk = __shfl_sync(FULL_MASK, dl, k);
                // a pair is taken only when both of its rows can be addressed
                const uint4 *yr = y.row(dk, rows, info);
                const bool ok = yr != nullptr && dy_buf.row(dk, rows, info) != nullptr;
                okm |= ok ? (1u << k) : 0u;
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int c = c0 + u * 32 + lane;
                    yv[k][u] = make_uint4(0u, 0u, 0u, 0u);
                    if (ok && c < vpr) yv[k][u] = ld_stream(yr + c);
                }
            }
#pragma unroll
            for (int k = 0; k < K; ++k) {
                const int dk = __shfl_sync(FULL_MASK, dl, k);
                const float wk = __shfl_sync(FULL_MASK, wl, k);
                if (!(okm & (1u << k))) continue;
                uint4 *br = dy_buf.row(dk, rows, info);
                if (br == nullptr) continue;
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int c = c0 + u * 32 + lane;
                    if (c < vpr) {
                        float yf[8];
                        unpack8(yv[k][u], yf);
                        dacc[k] += dot8(gf[u], yf);
                        float sc[8];
#pragma unroll
                        for (int j = 0; j < 8; ++j) sc[j] = unscaled ? gf[u][j] : __fmul_rn(wk, gf[u][j]);
                        st_vec(br + c, pack8(sc));
                    }
                }
            }
        }
#pragma unroll
        for (int k = 0; k < K; ++k) {
            float v = dacc[k];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(FULL_MASK, v, o);
            if (lane == k) dw[(size_t)t * K + k] = v;
        }
    }
}

// ----------------------------------------------------------------- launch

// One token per warp: a block of DATA_THREADS / 32 warps per group of
// tokens, as many blocks as that takes.  A grid of one resident wave
// (SMs x 2048 / DATA_THREADS blocks) walking the tokens left about 14 tokens
// per warp, and the warps that drew one more token set the kernel's tail:
// one token per warp, with the block scheduler refilling SMs, measured 5 %
// faster on dispatch and combine backward at the large shape.  The kernels
// keep their grid-stride loops, so any grid is correct.
static int data_grid(int tokens)
{
    const int wpb = DATA_THREADS / 32;
    const long long want = ((long long)tokens + wpb - 1) / wpb;
    return want < 1 ? 1 : (want > (1LL << 30) ? (1 << 30) : (int)want);
}

template <typename T>
static FlatRows<T> flat_rows(const Dims &d, T *base)
{
    return FlatRows<T>{base, d.H / 8};
}

template <typename T>
static RankRows<T> rank_rows(const Dims &d, T *const *bases)
{
    return RankRows<T>{bases, make_fastdiv((uint32_t)d.C), d.C, d.H / 8};
}

// tokens: the tokens this launch reads (R*S for one GPU, S for one rank);
// buffer rows are global rows in [0, R*S*K) either way
template <typename Rows>
static int dispatch_rows(const Dims &d, int tokens, const int *dst_pos, int *info, const uint16_t *hidden,
                         const Rows &buf, cudaStream_t st)
{
    dispatch_kernel<4, Rows><<<data_grid(tokens), DATA_THREADS, 0, st>>>(
        reinterpret_cast<const uint4 *>(hidden), buf, dst_pos, info, tokens, d.K, d.H / 8, d.pairs);
    return cudaGetLastError() == cudaSuccess ? MOONEP_OK : MOONEP_ERR_CUDA;
}

template <typename Rows>
static int combine_rows(const Dims &d, int T, const int *dst_pos, int *info, const Rows &yv, const float *w,
                        uint16_t *out, cudaStream_t st)
{
    const int vpr = d.H / 8, grid = data_grid(T), K = d.K, rows = d.pairs;
    uint4 *ov = reinterpret_cast<uint4 *>(out);
    switch (K) {
    case 1: combine_kernel<1, 4, Rows><<<grid, DATA_THREADS, 0, st>>>(yv, w, ov, dst_pos, info, T, K, vpr, rows); break;
    case 2: combine_kernel<2, 4, Rows><<<grid, DATA_THREADS, 0, st>>>(yv, w, ov, dst_pos, info, T, K, vpr, rows); break;
    case 4: combine_kernel<4, 2, Rows><<<grid, DATA_THREADS, 0, st>>>(yv, w, ov, dst_pos, info, T, K, vpr, rows); break;
    case 6: combine_kernel<6, 2, Rows><<<grid, DATA_THREADS, 0, st>>>(yv, w, ov, dst_pos, info, T, K, vpr, rows); break;
    case 8: combine_kernel<8, 2, Rows><<<grid, DATA_THREADS, 0, st>>>(yv, w, ov, dst_pos, info, T, K, vpr, rows); break;
    default: combine_kernel<0, 2, Rows><<<grid, DATA_THREADS, 0, st>>>(yv, w, ov, dst_pos, info, T, K, vpr, rows); break;
    }
    return cudaGetLastError() == cudaSuccess ? MOONEP_OK : MOONEP_ERR_CUDA;
}

template <int KT, typename YRows, typename BRows>
static void launch_bwd_k(const Dims &d, int T, const uint4 *dy, const float *w, const YRows &y, const BRows &dyb,
                         float *dw, const int *dst_pos, int *info, int unscaled, cudaStream_t st)
{
    constexpr int U = KT <= 8 ? 2 : 1;  // U = 1 measured slower at K = 8
    combine_bwd_kernel<KT, U, YRows, BRows><<<data_grid(T), DATA_THREADS, 0, st>>>(
        dy, w, y, dyb, dw, dst_pos, info, T, d.H / 8, unscaled, d.pairs);
}

template <typename YRows, typename BRows>
static int bwd_rows(const Dims &d, int T, const int *dst_pos, int *info, const uint16_t *dy, const float *w,
                    const YRows &yv, const BRows &bv, float *dw, cudaStream_t st)
{
    const uint4 *dyv = reinterpret_cast<const uint4 *>(dy);
    const int uns = (d.flags & MOONEP_FLAG_BWD_UNSCALED) ? 1 : 0;
    switch (d.K) {
#define MOONEP_BWD_CASE(k) \
    case k: launch_bwd_k<k>(d, T, dyv, w, yv, bv, dw, dst_pos, info, uns, st); break;
    MOONEP_BWD_CASE(1) MOONEP_BWD_CASE(2) MOONEP_BWD_CASE(3) MOONEP_BWD_CASE(4)
    MOONEP_BWD_CASE(5) MOONEP_BWD_CASE(6) MOONEP_BWD_CASE(7) MOONEP_BWD_CASE(8)
    MOONEP_BWD_CASE(9) MOONEP_BWD_CASE(10) MOONEP_BWD_CASE(11) MOONEP_BWD_CASE(12)
    MOONEP_BWD_CASE(13) MOONEP_BWD_CASE(14) MOONEP_BWD_CASE(15) MOONEP_BWD_CASE(16)
#undef MOONEP_BWD_CASE
    default: return MOONEP_ERR_LIMIT;
    }
    return cudaGetLastError() == cudaSuccess ? MOONEP_OK : MOONEP_ERR_CUDA;
}

// ---- one GPU: every rank's rows in one allocation

int launch_dispatch(const Dims &d, const int *dst_pos, int *info, const uint16_t *hidden, uint16_t *buf,
                    cudaStream_t st)
{
    return dispatch_rows(d, d.tokens, dst_pos, info, hidden, flat_rows(d, reinterpret_cast<uint4 *>(buf)), st);
}

int launch_combine(const Dims &d, const int *dst_pos, int *info, const uint16_t *y, const float *w,
                   uint16_t *out, cudaStream_t st)
{
    return combine_rows(d, d.tokens, dst_pos, info, flat_rows(d, reinterpret_cast<const uint4 *>(y)), w, out, st);
}

int launch_combine_backward(const Dims &d, const int *dst_pos, int *info, const uint16_t *dy, const float *w,
                            const uint16_t *y, uint16_t *dy_buf, float *dw, cudaStream_t st)
{
    return bwd_rows(d, d.tokens, dst_pos, info, dy, w, flat_rows(d, reinterpret_cast<const uint4 *>(y)),
                    flat_rows(d, reinterpret_cast<uint4 *>(dy_buf)), dw, st);
}

// ---- expert parallelism: one rank's S tokens, every rank's rows in its own
// allocation (peer memory), bases = device array of R row-buffer pointers

int launch_dispatch_ep(const Dims &d, const int *dst_pos, int *info, const uint16_t *hidden,
                       uint16_t *const *bufs, cudaStream_t st)
{
    return dispatch_rows(d, d.S, dst_pos, info, hidden, rank_rows(d, reinterpret_cast<uint4 *const *>(bufs)), st);
}

int launch_combine_ep(const Dims &d, const int *dst_pos, int *info, const uint16_t *const *ys, const float *w,
                      uint16_t *out, cudaStream_t st)
{
    return combine_rows(d, d.S, dst_pos, info, rank_rows(d, reinterpret_cast<const uint4 *const *>(ys)), w, out,
                        st);
}

int launch_combine_backward_ep(const Dims &d, const int *dst_pos, int *info, const uint16_t *dy, const float *w,
                               const uint16_t *const *ys, uint16_t *const *dy_bufs, float *dw, cudaStream_t st)
{
    return bwd_rows(d, d.S, dst_pos, info, dy, w, rank_rows(d, reinterpret_cast<const uint4 *const *>(ys)),
                    rank_rows(d, reinterpret_cast<uint4 *const *>(dy_bufs)), dw, st);
}

}  // namespace moonep
