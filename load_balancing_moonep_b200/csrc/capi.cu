// C ABI entry points (declared in include/moonep.h): host-side argument
// checks, plan layout and kernel launches.  No call allocates memory or
// synchronises the host.
#include <atomic>
#include <cstdint>
#include <cstring>

#include "common.cuh"

namespace moonep {
int launch_plan(const Dims &d, const int32_t *topk, const moonep_plan_t &p, void *ws, cudaStream_t st);
int set_wait_limit(int iterations);
int set_cascade_capacity(int c);
int set_plan_path(int mode);
size_t plan_smem_bytes_max(const Dims &d);
int launch_dispatch(const Dims &d, const int *dst_pos, int *info, const uint16_t *hidden, uint16_t *buf,
                    cudaStream_t st);
int launch_combine(const Dims &d, const int *dst_pos, int *info, const uint16_t *y, const float *w,
                   uint16_t *out, cudaStream_t st);
int launch_combine_backward(const Dims &d, const int *dst_pos, int *info, const uint16_t *dy, const float *w,
                            const uint16_t *y, uint16_t *dy_buf, float *dw, cudaStream_t st);
int launch_reduce(const Dims &d, const moonep_plan_t &p, float *reduce_buf, float *home_grad, long long P,
                  cudaStream_t st);
int launch_prefetch(const Dims &d, const moonep_plan_t &p, const uint16_t *weights, uint16_t *pool,
                    int32_t *slot_wrow, long long P, cudaStream_t st);
int launch_ep_count(const Dims &d, const int32_t *topk, int32_t *counts_row, void *ws, cudaStream_t st);
int launch_ep_plan(const Dims &d, int rank, const int32_t *topk, const int32_t *counts_all,
                   const moonep_plan_t &p, void *ws, cudaStream_t st);
size_t ep_smem_bytes_max(const Dims &d);
int launch_dispatch_ep(const Dims &d, const int *dst_pos, int *info, const uint16_t *hidden,
                       uint16_t *const *bufs, cudaStream_t st);
int launch_combine_ep(const Dims &d, const int *dst_pos, int *info, const uint16_t *const *ys, const float *w,
                      uint16_t *out, cudaStream_t st);
int launch_combine_backward_ep(const Dims &d, const int *dst_pos, int *info, const uint16_t *dy, const float *w,
                               const uint16_t *const *ys, uint16_t *const *dy_bufs, float *dw, cudaStream_t st);
int launch_reduce_ep(const Dims &d, int rank, const moonep_plan_t &p, float *const *reduce_bufs,
                     float *home_grad, long long P, cudaStream_t st);
int launch_prefetch_ep(const Dims &d, int rank, const moonep_plan_t &p, const uint16_t *const *weights,
                       uint16_t *pool, int32_t *slot_wrow, long long P, cudaStream_t st);

constexpr size_t MAX_DYN_SMEM = 227 * 1024;
constexpr int MAX_COMBINE_BWD_K = 16;

// SMs of a B200.  The planner's token chunking is sized for it: the
// workspace is laid out for that many chunks, so its size never depends on
// which device is current when it is sized.
constexpr int B200_SMS = 148;
constexpr int MAX_DEVICES = 64;

// SM count of the current device, cached per device (B200_SMS when no device
// can be queried, e.g. for host-only sizing on a machine without a GPU).
static int current_device_sms()
{
    static std::atomic<int> cache[MAX_DEVICES];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) {
        (void)cudaGetLastError();
        return B200_SMS;
    }
    int n = cache[dev].load(std::memory_order_relaxed);
    if (n > 0) return n;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
        (void)cudaGetLastError();
        n = B200_SMS;
    }
    cache[dev].store(n, std::memory_order_relaxed);
    return n;
}

// nsm: the SM count the chunking targets, at most B200_SMS (sizing uses
// B200_SMS; a launch uses min(device SMs, B200_SMS), which never gives more
// chunks than the sizing did, so the launch's workspace layout fits in the
// sized workspace).
static int make_dims(const moonep_config *c, Dims *d, int nsm = B200_SMS)
{
    const int rc = moonep_check_config(c);
    if (rc != MOONEP_OK) return rc;
    d->R = c->R;
    d->E = c->E;
    d->K = c->K;
    d->S = c->S;
    d->H = c->H;
    d->B = c->B;
    d->L = c->E / c->R;
    d->flags = c->flags;
    d->C = c->S * c->K;
    d->tokens = c->R * c->S;
    d->pairs = c->R * c->S * c->K;
    // at most 2 x SMs - 1 chunks: two assignment CTAs fit on each SM but one
    // slot is held by the planner CTA while they start, and all of them
    // should be resident then.  The chunking affects speed only, never the
    // plan.
    if (nsm < 1) nsm = 1;
    if (nsm > B200_SMS) nsm = B200_SMS;
    const int target = 2 * nsm - 1;
    int ct = (d->tokens + target - 1) / target;
    if (ct < 8) ct = 8;
    int cap = 4096 / d->K;
    if (cap < 1) cap = 1;
    if (ct > cap) ct = cap;
    if (ct > d->tokens) ct = d->tokens;
    d->chunk_tokens = ct;
    d->nchunk = (d->tokens + ct - 1) / ct;
    d->ngroups = (d->nchunk + CHUNK_GROUP - 1) / CHUNK_GROUP;
    d->ebits = 0;
    while ((1 << d->ebits) < d->E) ++d->ebits;
    d->nsm = nsm;
    if (plan_smem_bytes_max(*d) > MAX_DYN_SMEM) return MOONEP_ERR_LIMIT;
    return MOONEP_OK;
}

// Expert parallelism: the chunking covers one rank's S tokens (about 128
// chunks, at least 8 tokens and at most 4096 pairs each) and the planner sums
// the R rows of the gathered counts.
static int make_dims_ep(const moonep_config *c, Dims *d)
{
    const int rc = make_dims(c, d);
    if (rc != MOONEP_OK) return rc;
    int ct = (d->S + 127) / 128;
    if (ct < 8) ct = 8;
    int cap = 4096 / d->K;
    if (cap < 1) cap = 1;
    if (ct > cap) ct = cap;
    if (ct > d->S) ct = d->S;
    d->chunk_tokens = ct;
    d->nchunk = (d->S + ct - 1) / ct;
    d->ngroups = d->R;
    if (ep_smem_bytes_max(*d) > MAX_DYN_SMEM) return MOONEP_ERR_LIMIT;
    return MOONEP_OK;
}

static bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static bool plan_ok(const moonep_plan_t *p)
{
    return p && p->expert_count && p->slot_expert && p->slot_count && p->slot_offset && p->rep_expert &&
           p->rep_rank && p->rep_slot && p->rep_quota && p->host_ptr && p->host_rank && p->host_slot &&
           p->host_start && p->host_quota && p->rep_home_list && p->dst_pos && p->row_src && p->info &&
           p->host_local;
}

constexpr int PLAN_ARRAYS = 18;
struct PlanLayout {
    size_t off[PLAN_ARRAYS];
    size_t total;
};

static PlanLayout plan_layout(const Dims &d)
{
    const size_t E = d.E, R = d.R, NP = (size_t)d.pairs;
    const size_t n[PLAN_ARRAYS] = {E,         R * E,     R * E,     R * (E + 1), E + R,      E + R,
                                   E + R,     E + R,     E + 1,     2 * E + R,   2 * E + R,  2 * E + R,
                                   2 * E + R, E,         NP,        NP,          MOONEP_INFO_LEN, 2 * E + R};
    PlanLayout l;
    size_t o = 0;
    for (int i = 0; i < PLAN_ARRAYS; ++i) {
        l.off[i] = o;
        o = align256(o + n[i] * sizeof(int32_t));
    }
    l.total = o;
    return l;
}

// Bytes at the start of the workspace that a call must find zeroed when the
// workspace holds another configuration's leftovers: the header and both
// group-count buffers (the per-chunk counts and host rows after them are
// written in full before they are read).  Laid out for the current device.
int workspace_clear_bytes(const moonep_config *cfg, size_t *bytes)
{
    Dims d;
    const int rc = make_dims(cfg, &d, current_device_sms());
    if (rc != MOONEP_OK) return rc;
    *bytes = ws_layout(d).cc;
    return MOONEP_OK;
}

}  // namespace moonep

using namespace moonep;

extern "C" {

int moonep_abi_version(void) { return MOONEP_ABI_VERSION; }

int moonep_set_wait_limit(int iterations) { return set_wait_limit(iterations); }

int moonep_set_cascade_capacity(int capacity) { return set_cascade_capacity(capacity); }

int moonep_set_plan_path(int mode) { return set_plan_path(mode); }

const char *moonep_error_string(int code)
{
    switch (code) {
    case MOONEP_OK: return "ok";
    case MOONEP_ERR_ARG:
        return "invalid argument (null pointer, non-positive size, K > E, R*S*K >= 2^31, or an unknown flag bit)";
    case MOONEP_ERR_E_NOT_DIVISIBLE: return "E is not divisible by R";
    case MOONEP_ERR_BUDGET_RULE: return "training budget rule violated: B must equal E/R";
    case MOONEP_ERR_B_RANGE: return "replica budget B out of range [0, E - E/R]";
    case MOONEP_ERR_CUDA: return "CUDA launch failed";
    case MOONEP_ERR_LIMIT: return "size beyond a library limit (E > 1024, shared memory, or K > 16 in combine_backward)";
    case MOONEP_ERR_ALIGN: return "H must be a multiple of 8 and bf16 data pointers 16-byte aligned";
    case MOONEP_ERR_NOALLOC_SIZE:
        return "workspace larger than the fixed no-allocation array (MOONEP_NOALLOC_WORKSPACE_BYTES)";
    default: return "unknown error";
    }
}

const char *moonep_status_string(int status, char *buf, size_t len)
{
    static const char empty[1] = {0};
    if (!buf || len == 0) return empty;
    static const char *const names[6] = {"EXPERT_ID_RANGE", "OVERFLOW", "STRICT_VIOLATION",
                                         "ROW_RANGE",       "WAIT_TIMEOUT", "WORKSPACE"};
    size_t n = 0;
    auto put = [&](const char *t) {
        for (; *t && n + 1 < len; ++t) buf[n++] = *t;
    };
    if (status == 0) put("ok");
    for (int b = 0; b < 32; ++b) {
        if (!((unsigned)status & (1u << b))) continue;
        if (n > 0) put("|");
        if (b < 6) {
            put(names[b]);
        } else {
            char t[8] = {'b', 'i', 't', 0, 0, 0, 0, 0};
            t[3] = (char)('0' + b / 10);
            t[4] = (char)('0' + b % 10);
            if (b < 10) { t[3] = (char)('0' + b); t[4] = 0; }
            put(t);
        }
    }
    buf[n] = 0;
    return buf;
}

int moonep_check_config(const moonep_config *c)
{
    if (!c) return MOONEP_ERR_ARG;
    if (c->R <= 0 || c->E <= 0 || c->K <= 0 || c->S <= 0 || c->H <= 0) return MOONEP_ERR_ARG;
    if (c->K > c->E) return MOONEP_ERR_ARG;
    if ((int64_t)c->R * c->S * c->K > INT32_MAX) return MOONEP_ERR_ARG;
    if (c->flags & ~(MOONEP_FLAG_STRICT_BUDGET | MOONEP_FLAG_TRAIN_B_RULE | MOONEP_FLAG_BWD_UNSCALED |
                     MOONEP_FLAG_CASCADE | MOONEP_FLAG_LOCALITY))
        return MOONEP_ERR_ARG;
    if (c->E % c->R != 0) return MOONEP_ERR_E_NOT_DIVISIBLE;
    const int L = c->E / c->R;
    if ((c->flags & MOONEP_FLAG_TRAIN_B_RULE) && c->B != L) return MOONEP_ERR_BUDGET_RULE;
    if (c->B < 0 || c->B > c->E - L) return MOONEP_ERR_B_RANGE;
    if (c->E > MOONEP_MAX_E) return MOONEP_ERR_LIMIT;
    if (c->H % 8 != 0) return MOONEP_ERR_ALIGN;
    return MOONEP_OK;
}

int moonep_plan_sizes(const moonep_config *cfg, size_t *plan_bytes, size_t *workspace_bytes)
{
    Dims d;
    const int rc = make_dims(cfg, &d);
    if (rc != MOONEP_OK) return rc;
    if (plan_bytes) *plan_bytes = plan_layout(d).total;
    if (workspace_bytes) *workspace_bytes = ws_layout(d).total;
    return MOONEP_OK;
}

int moonep_plan_layout(const moonep_config *cfg, void *plan_base, moonep_plan_t *out)
{
    if (!plan_base || !out) return MOONEP_ERR_ARG;
    Dims d;
    const int rc = make_dims(cfg, &d);
    if (rc != MOONEP_OK) return rc;
    if (reinterpret_cast<uintptr_t>(plan_base) & 255u) return MOONEP_ERR_ALIGN;
    const PlanLayout l = plan_layout(d);
    char *b = static_cast<char *>(plan_base);
    int32_t **f[PLAN_ARRAYS] = {&out->expert_count, &out->slot_expert,   &out->slot_count, &out->slot_offset,
                                &out->rep_expert,   &out->rep_rank,      &out->rep_slot,   &out->rep_quota,
                                &out->host_ptr,     &out->host_rank,     &out->host_slot,  &out->host_start,
                                &out->host_quota,   &out->rep_home_list, &out->dst_pos,    &out->row_src,
                                &out->info,         &out->host_local};
    for (int i = 0; i < PLAN_ARRAYS; ++i) *f[i] = reinterpret_cast<int32_t *>(b + l.off[i]);
    return MOONEP_OK;
}

int moonep_plan(const moonep_config *cfg, const int32_t *topk_idx, const moonep_plan_t *plan, void *workspace,
                void *stream)
{
    Dims d;
    const int rc = make_dims(cfg, &d, current_device_sms());
    if (rc != MOONEP_OK) return rc;
    if (!topk_idx || !plan_ok(plan) || !workspace) return MOONEP_ERR_ARG;
    // one GPU holds every rank: no pair crosses a link, and the locality
    // flag's per-rank counts exist only in expert parallelism
    if (d.flags & MOONEP_FLAG_LOCALITY) return MOONEP_ERR_ARG;
    return launch_plan(d, topk_idx, *plan, workspace, static_cast<cudaStream_t>(stream));
}

int moonep_dispatch(const moonep_config *cfg, const moonep_plan_t *plan, const uint16_t *hidden, uint16_t *buf,
                    void *stream)
{
    Dims d;
    const int rc = make_dims(cfg, &d);
    if (rc != MOONEP_OK) return rc;
    if (!plan_ok(plan) || !hidden || !buf) return MOONEP_ERR_ARG;
    if (!aligned16(hidden) || !aligned16(buf)) return MOONEP_ERR_ALIGN;
    return launch_dispatch(d, plan->dst_pos, plan->info, hidden, buf, static_cast<cudaStream_t>(stream));
}

int moonep_combine(const moonep_config *cfg, const moonep_plan_t *plan, const uint16_t *y, const float *w,
                   uint16_t *out, void *stream)
{
    Dims d;
    const int rc = make_dims(cfg, &d);
    if (rc != MOONEP_OK) return rc;
    if (!plan_ok(plan) || !y || !w || !out) return MOONEP_ERR_ARG;
    if (!aligned16(y) || !aligned16(out) || (reinterpret_cast<uintptr_t>(w) & 3u)) return MOONEP_ERR_ALIGN;
    return launch_combine(d, plan->dst_pos, plan->info, y, w, out, static_cast<cudaStream_t>(stream));
}

int moonep_combine_backward(const moonep_config *cfg, const moonep_plan_t *plan, const uint16_t *dy,
                            const float *w, const uint16_t *y, uint16_t *dy_buf, float *dw, void *stream)
{
    Dims d;
    const int rc = make_dims(cfg, &d);
    if (rc != MOONEP_OK) return rc;
    if (!plan_ok(plan) || !dy || !w || !y || !dy_buf || !dw) return MOONEP_ERR_ARG;
    if (d.K > MAX_COMBINE_BWD_K) return MOONEP_ERR_LIMIT;
    if (!aligned16(dy) || !aligned16(y) || !aligned16(dy_buf) || (reinterpret_cast<uintptr_t>(w) & 3u) ||
        (reinterpret_cast<uintptr_t>(dw) & 3u))
        return MOONEP_ERR_ALIGN;
    return launch_combine_backward(d, plan->dst_pos, plan->info, dy, w, y, dy_buf, dw,
                                   static_cast<cudaStream_t>(stream));
}

int moonep_reduce_replica_grads(const moonep_config *cfg, const moonep_plan_t *plan, float *reduce_buf,
                                float *home_grad, int64_t P, void *stream)
{
    Dims d;
    const int rc = make_dims(cfg, &d);
    if (rc != MOONEP_OK) return rc;
    if (!plan_ok(plan) || !home_grad || P <= 0) return MOONEP_ERR_ARG;
    if (d.B > 0 && !reduce_buf) return MOONEP_ERR_ARG;
    if (d.B == 0) return MOONEP_OK;  // no prefetched replica can exist
    if ((reinterpret_cast<uintptr_t>(reduce_buf) & 3u) || (reinterpret_cast<uintptr_t>(home_grad) & 3u))
        return MOONEP_ERR_ALIGN;
    return launch_reduce(d, *plan, reduce_buf, home_grad, (long long)P, static_cast<cudaStream_t>(stream));
}

int moonep_prefetch_replicas(const moonep_config *cfg, const moonep_plan_t *plan, const uint16_t *weights,
                             uint16_t *pool, int32_t *slot_wrow, int64_t P, void *stream)
{
    Dims d;
    const int rc = make_dims(cfg, &d);
    if (rc != MOONEP_OK) return rc;
    if (!plan_ok(plan) || !weights || !slot_wrow || P <= 0) return MOONEP_ERR_ARG;
    if (d.B > 0 && !pool) return MOONEP_ERR_ARG;
    if ((reinterpret_cast<uintptr_t>(weights) & 1u) || (reinterpret_cast<uintptr_t>(pool) & 1u) ||
        (reinterpret_cast<uintptr_t>(slot_wrow) & 3u))
        return MOONEP_ERR_ALIGN;
    return launch_prefetch(d, *plan, weights, pool, slot_wrow, (long long)P, static_cast<cudaStream_t>(stream));
}

// ---- expert parallelism over several GPUs

int moonep_ep_sizes(const moonep_config *cfg, size_t *plan_bytes, size_t *workspace_bytes)
{
    Dims d;
    const int rc = make_dims_ep(cfg, &d);
    if (rc != MOONEP_OK) return rc;
    if (plan_bytes) *plan_bytes = plan_layout(d).total;
    if (workspace_bytes) *workspace_bytes = ws_layout_ep(d).total;
    return MOONEP_OK;
}

int moonep_ep_count(const moonep_config *cfg, const int32_t *topk_local, int32_t *counts_row, void *workspace,
                    void *stream)
{
    Dims d;
    const int rc = make_dims_ep(cfg, &d);
    if (rc != MOONEP_OK) return rc;
    if (!topk_local || !counts_row || !workspace) return MOONEP_ERR_ARG;
    return launch_ep_count(d, topk_local, counts_row, workspace, static_cast<cudaStream_t>(stream));
}

int moonep_ep_plan(const moonep_config *cfg, int32_t rank, const int32_t *topk_local, const int32_t *counts_all,
                   const moonep_plan_t *plan, void *workspace, void *stream)
{
    Dims d;
    const int rc = make_dims_ep(cfg, &d);
    if (rc != MOONEP_OK) return rc;
    if (rank < 0 || rank >= d.R || !topk_local || !counts_all || !plan_ok(plan) || !workspace)
        return MOONEP_ERR_ARG;
    return launch_ep_plan(d, rank, topk_local, counts_all, *plan, workspace, static_cast<cudaStream_t>(stream));
}

int moonep_ep_dispatch(const moonep_config *cfg, const moonep_plan_t *plan, const uint16_t *hidden_local,
                       uint16_t *const *bufs, void *stream)
{
    Dims d;
    const int rc = make_dims(cfg, &d);
    if (rc != MOONEP_OK) return rc;
    if (!plan_ok(plan) || !hidden_local || !bufs) return MOONEP_ERR_ARG;
    if (!aligned16(hidden_local)) return MOONEP_ERR_ALIGN;
    return launch_dispatch_ep(d, plan->dst_pos, plan->info, hidden_local, bufs, static_cast<cudaStream_t>(stream));
}

int moonep_ep_combine(const moonep_config *cfg, const moonep_plan_t *plan, const uint16_t *const *ys,
                      const float *w_local, uint16_t *out_local, void *stream)
{
    Dims d;
    const int rc = make_dims(cfg, &d);
    if (rc != MOONEP_OK) return rc;
    if (!plan_ok(plan) || !ys || !w_local || !out_local) return MOONEP_ERR_ARG;
    if (!aligned16(out_local) || (reinterpret_cast<uintptr_t>(w_local) & 3u)) return MOONEP_ERR_ALIGN;
    return launch_combine_ep(d, plan->dst_pos, plan->info, ys, w_local, out_local,
                             static_cast<cudaStream_t>(stream));
}

int moonep_ep_combine_backward(const moonep_config *cfg, const moonep_plan_t *plan, const uint16_t *dy_local,
                               const float *w_local, const uint16_t *const *ys, uint16_t *const *dy_bufs,
                               float *dw_local, void *stream)
{
    Dims d;
    const int rc = make_dims(cfg, &d);
    if (rc != MOONEP_OK) return rc;
    if (!plan_ok(plan) || !dy_local || !w_local || !ys || !dy_bufs || !dw_local) return MOONEP_ERR_ARG;
    if (d.K > MAX_COMBINE_BWD_K) return MOONEP_ERR_LIMIT;
    if (!aligned16(dy_local) || (reinterpret_cast<uintptr_t>(w_local) & 3u) ||
        (reinterpret_cast<uintptr_t>(dw_local) & 3u))
        return MOONEP_ERR_ALIGN;
    return launch_combine_backward_ep(d, plan->dst_pos, plan->info, dy_local, w_local, ys, dy_bufs, dw_local,
                                      static_cast<cudaStream_t>(stream));
}

int moonep_ep_reduce_replica_grads(const moonep_config *cfg, int32_t rank, const moonep_plan_t *plan,
                                   float *const *reduce_bufs, float *home_grad_local, int64_t P, void *stream)
{
    Dims d;
    const int rc = make_dims(cfg, &d);
    if (rc != MOONEP_OK) return rc;
    if (rank < 0 || rank >= d.R || !plan_ok(plan) || !home_grad_local || P <= 0) return MOONEP_ERR_ARG;
    if (d.B > 0 && !reduce_bufs) return MOONEP_ERR_ARG;
    if (d.B == 0) return MOONEP_OK;  // no prefetched replica can exist
    if (reinterpret_cast<uintptr_t>(home_grad_local) & 3u) return MOONEP_ERR_ALIGN;
    return launch_reduce_ep(d, rank, *plan, reduce_bufs, home_grad_local, (long long)P,
                            static_cast<cudaStream_t>(stream));
}

int moonep_ep_prefetch_replicas(const moonep_config *cfg, int32_t rank, const moonep_plan_t *plan,
                                const uint16_t *const *weights, uint16_t *pool_local, int32_t *slot_wrow_local,
                                int64_t P, void *stream)
{
    Dims d;
    const int rc = make_dims(cfg, &d);
    if (rc != MOONEP_OK) return rc;
    if (rank < 0 || rank >= d.R || !plan_ok(plan) || !weights || !slot_wrow_local || P <= 0) return MOONEP_ERR_ARG;
    if (d.B > 0 && !pool_local) return MOONEP_ERR_ARG;
    if ((reinterpret_cast<uintptr_t>(pool_local) & 1u) || (reinterpret_cast<uintptr_t>(slot_wrow_local) & 3u))
        return MOONEP_ERR_ALIGN;
    return launch_prefetch_ep(d, rank, *plan, weights, pool_local, slot_wrow_local, (long long)P,
                              static_cast<cudaStream_t>(stream));
}

}  // extern "C"
