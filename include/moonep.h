/*
 * moonep.h -- C ABI of the MoonEP redundant-expert planner and fused
 * permute/unpermute for NVIDIA B200 (sm_100a).
 *
 * The operation (cited by page title and section):
 *   "Moonshot AI Open-Sources MoonEP: A Perfectly Balanced Expert
 *   Parallelism Library for MoE Training" (MoonEP article below):
 *     - "The problem MoonEP targets": top-K routing is skewed; skew is
 *       measured by maxvio = max_e T_e / T_bar - 1.
 *     - "The core idea: dynamic redundant experts": every rank receives
 *       exactly S*K token slots however skewed the routing is; a small
 *       number of redundant experts is planned online from the current
 *       router output; tokens are written directly into expert-grouped
 *       positions of a fixed S*K buffer and views of it are handed to the
 *       computation; duplicated experts' gradients go back to their home.
 *     - interactive explainer, memory tab: at most B prefetched replica
 *       slots per rank (B = E/R in training), replica gradients in an fp32
 *       reduce buffer [R, B, ...] that is summed home and zeroed; in
 *       inference a rank needing more than B foreign experts reads the
 *       overflow from the home rank (correctness unaffected).
 *     - explainer, invariant tab: no host synchronisation per MoE layer.
 *
 * Scope: R expert-parallel ranks are simulated as R partitions of ONE
 * GPU's memory; no collective is issued.  Rank r owns tokens
 * [r*S, (r+1)*S) and rows [r*S*K, (r+1)*S*K) of the dispatch buffer.
 * Expert e's home rank is e / L with L = E / R (contiguous homes).
 *
 * Conventions for every call below:
 *   - All array pointers are DEVICE pointers unless stated otherwise and
 *     are caller-allocated; the library never allocates and never frees.
 *   - bf16 data are passed as uint16_t bit patterns.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Every
 *     call only enqueues kernels on it and returns; nothing synchronises
 *     the host.  Data-dependent problems are reported in the device-side
 *     status word plan->info[MOONEP_INFO_STATUS], which the caller may read
 *     back whenever it likes.
 *   - Return value: MOONEP_OK or a MOONEP_ERR_* code from the host-side
 *     argument checks (nothing is launched then) or MOONEP_ERR_CUDA if a
 *     launch failed.
 *   - Calls are stream-ordered; two plans or workspaces must not be shared
 *     by calls that can run concurrently.
 */
#ifndef MOONEP_H
#define MOONEP_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MOONEP_ABI_VERSION 2

#if defined(__GNUC__)
#define MOONEP_API __attribute__((visibility("default")))
#else
#define MOONEP_API
#endif

/* ---- configuration flags ---------------------------------------------- */
/* Overflow (a rank needs more than B replica slots) also sets
 * MOONEP_ST_STRICT_VIOLATION: training has no reduce rows for overflow. */
#define MOONEP_FLAG_STRICT_BUDGET 1u
/* Require B == E/R, the training rule of the explainer's memory tab. */
#define MOONEP_FLAG_TRAIN_B_RULE 2u
/* combine_backward dispatches dy unscaled instead of w * dy. */
#define MOONEP_FLAG_BWD_UNSCALED 4u
/* Relay cascade: when water-filling leaves a rank with more than B
 * replicas, repair such ranks one at a time (most replicas first): the rank
 * keeps its B - m largest replicas, grows them and adds m relay replicas of
 * other ranks' experts to carry the rest, and the moved replicas go to the
 * providers' home ranks, which may in turn be repaired.  Within the budget
 * the plan is exactly water-filling's.  Costs 7 (E + R) + 4 (B + 1) + 16
 * more ints of planner shared memory (MOONEP_ERR_LIMIT if the total does not
 * fit; at E = R = MOONEP_MAX_E it does) and a slow path, one warp stepping
 * through the repairs, when it runs.  Unknown flag bits are MOONEP_ERR_ARG. */
#define MOONEP_FLAG_CASCADE 8u
/* Locality-aware host intervals (expert parallelism: moonep_ep_plan only;
 * moonep_plan, where a pair on another rank costs no transfer, refuses it
 * with MOONEP_ERR_ARG).  Each host of an expert first takes up to its quota
 * of the pairs from its own rank (the first ones, in (t, k) order:
 * host_local[h] = min(quota, those pairs)); the pairs left over, in (t, k)
 * order, fill the rest of the quotas in ascending rank order, host_start[h]
 * being where host h's share of them starts.  The replicas, quotas and slots
 * are water-filling's; the pairs kept on their source rank are the most any
 * choice of intervals keeps for them.  A host's rows hold its local pairs
 * first, then its leftover ones, each part in (t, k) order. */
#define MOONEP_FLAG_LOCALITY 16u

/* ---- host return codes ------------------------------------------------- */
#define MOONEP_OK 0
#define MOONEP_ERR_ARG 1            /* null pointer, non-positive size, K > E, R*S*K >= 2^31, unknown flag bit */
#define MOONEP_ERR_E_NOT_DIVISIBLE 2 /* E % R != 0 (the explainer flags it) */
#define MOONEP_ERR_BUDGET_RULE 3    /* TRAIN_B_RULE set and B != E/R */
#define MOONEP_ERR_B_RANGE 4        /* B < 0 or B > E - L */
#define MOONEP_ERR_CUDA 5           /* a kernel launch failed */
#define MOONEP_ERR_LIMIT 7          /* E > MOONEP_MAX_E; K > 16 in moonep_combine_backward */
#define MOONEP_ERR_ALIGN 8          /* H % 8 != 0 or a data pointer not 16-byte aligned */
#define MOONEP_ERR_NOALLOC_SIZE 9   /* moonep_plan_noalloc: workspace above MOONEP_NOALLOC_WORKSPACE_BYTES */

#define MOONEP_MAX_E 1024

/* ---- device status bits (plan->info[MOONEP_INFO_STATUS]) -------------- */
/* An id outside [0, E): the plan is empty, dst_pos/row_src are -1, and
 * dispatch / combine / combine_backward / reduce / prefetch become no-ops.
 * (MOONEP_ST_WORKSPACE below empties the plan the same way.) */
#define MOONEP_ST_EXPERT_ID_RANGE 1
/* Some rank holds more than B replicas; the extra ones (ordinal >= B) are
 * still planned, so every rank still gets exactly S*K slots, but they have
 * no prefetch slot / reduce rows (read-through in inference). */
#define MOONEP_ST_OVERFLOW 2
#define MOONEP_ST_STRICT_VIOLATION 4
/* A buffer row taken from the plan was outside [0, R*S*K) (a corrupted or
 * mismatched plan); that row access was skipped. */
#define MOONEP_ST_ROW_RANGE 8
/* A bounded wait inside a kernel ran out of iterations (about 6 ms at the
 * bound).  In the two-kernel planner: one of the assignment pass's waits for
 * a mark of the histogram/planner pass (counts ready, plan ready); the pass
 * then waits for the whole histogram grid instead.  In the one-kernel
 * planner: a CTA's wait for every chunk's counts (its peers were not all
 * resident, e.g. because another stream's kernels held SMs); that CTA then
 * counts every pair of the call itself.  Either way the plan is still
 * complete and exact; the bit reports the slow path, or a workspace used by
 * two overlapping calls.  A relay cascade (MOONEP_FLAG_CASCADE), which can
 * run for milliseconds, announces itself in the two-kernel planner and is
 * waited for the same way without setting this bit. */
#define MOONEP_ST_WAIT_TIMEOUT 16
/* The planner workspace did not hold the zeros a call must start from (it
 * was not zero-filled before first use, or two calls used it at once): the
 * expert totals do not add up to R*S*K.  The plan is then empty, exactly as
 * for MOONEP_ST_EXPERT_ID_RANGE; zero-fill the workspace and plan again. */
#define MOONEP_ST_WORKSPACE 32

/* ---- plan->info[] fields (int32, device) ------------------------------ */
#define MOONEP_INFO_STATUS 0
#define MOONEP_INFO_N_REP 1            /* replicas created */
#define MOONEP_INFO_N_OVERFLOW 2       /* replicas with ordinal >= B */
#define MOONEP_INFO_N_PIECES 3         /* experts that shed load */
#define MOONEP_INFO_N_RECEIVERS 4      /* ranks with a deficit */
#define MOONEP_INFO_MAX_REP_PER_RANK 5
#define MOONEP_INFO_N_REP_EXPERTS 6    /* experts with >= 1 prefetched replica */
#define MOONEP_INFO_N_REMOTE_PAIRS 7   /* pairs whose buffer rank != source rank */
/* Relay cascade (MOONEP_FLAG_CASCADE) only, 0 otherwise: the repair steps
 * that found providers and so reached the capacity guard, and the least
 * slack the guard saw, (E + R - 1) - (live replicas + m + B - 1); a step
 * with negative slack is not taken. */
#define MOONEP_INFO_CASCADE_GUARD_STEPS 8
#define MOONEP_INFO_CASCADE_GUARD_SLACK 9
#define MOONEP_INFO_LEN 16

typedef struct moonep_config {
    int32_t R;      /* simulated expert-parallel ranks */
    int32_t E;      /* experts; E % R == 0, L = E / R home experts per rank */
    int32_t K;      /* routed experts per token (top-K) */
    int32_t S;      /* tokens per rank */
    int32_t H;      /* hidden size (bf16 elements per row), H % 8 == 0 */
    int32_t B;      /* replica (prefetch) slots per rank, 0 <= B <= E - L */
    uint32_t flags; /* MOONEP_FLAG_* */
} moonep_config;

/* The plan: device arrays, all int32, laid out by moonep_plan_layout().
 * Slot s of rank r: s < L is home expert r*L + s; s >= L is the rank's
 * (s-L)-th replica in creation order; unused slots hold expert -1, count 0.
 * Rows of rank r's buffer are grouped by slot: slot s occupies rows
 * [slot_offset[r][s], slot_offset[r][s+1]) and slot_offset[r][E] == S*K. */
typedef struct moonep_plan_s {
    int32_t *expert_count;  /* [E] T_e = pairs routed to e */
    int32_t *slot_expert;   /* [R][E] */
    int32_t *slot_count;    /* [R][E] rows per slot */
    int32_t *slot_offset;   /* [R][E+1] exclusive prefix of slot_count */
    int32_t *rep_expert;    /* [E+R] replica list in creation order ... */
    int32_t *rep_rank;      /* [E+R] ... rank holding the replica */
    int32_t *rep_slot;      /* [E+R] ... its slot (L + ordinal) */
    int32_t *rep_quota;     /* [E+R] ... rows it receives; entries >= n_rep: -1 / 0 */
    int32_t *host_ptr;      /* [E+1] CSR: hosts of expert e are [host_ptr[e], host_ptr[e+1]) */
    int32_t *host_rank;     /* [2E+R] hosts in ascending rank order (home copy included) */
    int32_t *host_slot;     /* [2E+R] */
    int32_t *host_start;    /* [2E+R] first within-expert rank g served by the host (with
                               MOONEP_FLAG_LOCALITY: the start of its share of the leftover pairs) */
    int32_t *host_quota;    /* [2E+R] number of g served by the host */
    int32_t *rep_home_list; /* [E] experts with >= 1 prefetched replica, ascending, then -1 */
    int32_t *dst_pos;       /* [R*S*K] buffer row of pair (t, k), index t*K + k */
    int32_t *row_src;       /* [R*S*K] inverse: pair t*K + k held by a buffer row */
    int32_t *info;          /* [MOONEP_INFO_LEN] status and statistics */
    int32_t *host_local;    /* [2E+R] pairs of the host's own rank it serves first (MOONEP_FLAG_LOCALITY), else 0 */
} moonep_plan_t;

/* Host-side validation of a configuration.  Returns MOONEP_OK or an error. */
MOONEP_API int moonep_check_config(const moonep_config *cfg);

/* Bytes of the plan block and of the planner workspace for `cfg`.
 * The workspace must be zero-filled once after allocation (for example
 * cudaMemset).  Every moonep_plan() call leaves it ready for the next call
 * with the SAME configuration (its counters and sequence marks advanced, the
 * count buffer of the next call zeroed); before it is used with a different
 * configuration it must be zero-filled again, or the planner reports
 * MOONEP_ST_WORKSPACE and returns an empty plan. */
MOONEP_API int moonep_plan_sizes(const moonep_config *cfg, size_t *plan_bytes, size_t *workspace_bytes);

/* Fills `out` with pointers into the device block `plan_base` of
 * plan_bytes bytes (256-byte aligned sub-arrays).  Host-only arithmetic. */
MOONEP_API int moonep_plan_layout(const moonep_config *cfg, void *plan_base, moonep_plan_t *out);

/* Online planning (MoonEP article, "The core idea: dynamic redundant
 * experts"; planner described as "near-optimal" with no algorithm given).
 * topk_idx: device int32 [R*S, K], row t = token t (rank t / S), k order as
 * produced by the router.  Computes, with no host synchronisation:
 *   histogram T_e; home loads and excess/deficit per rank; largest-first
 *   shedding by each overloaded rank (ties: lower expert id first);
 *   pieces ordered by (shed desc, e asc) and receivers by (deficit desc,
 *   rank asc); water-filling of pieces into deficits (every positive
 *   overlap of the two prefix-sum partitions is one replica, created in
 *   (piece, receiver) order; a rank's replicas take slots L, L+1, ...);
 *   slot tables; per-expert host intervals in ascending rank order; and for
 *   every pair in (t, k) order the buffer row
 *     dst_pos = rank*S*K + slot_offset[rank][slot] + (g - host_start)
 *   where g is the pair's rank among earlier pairs of the same expert.
 * plan: laid out by moonep_plan_layout; workspace: workspace_bytes bytes,
 * zero-filled before the first call.
 * One kernel launch when all of its CTAs (one per token chunk, at most two
 * per SM) fit on the device at once: every CTA counts its chunk, waits
 * (bounded) for the others' counts, computes the whole plan in its own
 * shared memory and places its own pairs.  Otherwise (shapes whose planner
 * needs more shared memory) two launches: a histogram pass whose last CTA
 * plans, and an assignment pass.  Both give the same plan, bit for bit. */
MOONEP_API int moonep_plan(const moonep_config *cfg, const int32_t *topk_idx, const moonep_plan_t *plan,
                void *workspace, void *stream);

/* Zero-copy permute (MoonEP article, "The core idea", zero copy and static
 * shapes): buf[dst_pos[t*K+k], :] = hidden[t, :] for every pair.
 * hidden: bf16 [R*S, H]; buf: bf16 [R, S*K, H] = R*S*K rows of H.  Every
 * buffer row is written exactly once; values are copied bit for bit. */
MOONEP_API int moonep_dispatch(const moonep_config *cfg, const moonep_plan_t *plan, const uint16_t *hidden,
                    uint16_t *buf, void *stream);

/* Weighted unpermute: out[t, h] = bf16_rne(sum_k w[t,k] * y[dst_pos[t*K+k], h])
 * accumulated in fp32 as acc = fmaf(w, y, acc) from 0.0f in k order.
 * y: bf16 [R, S*K, H] (expert outputs in buffer layout); w: fp32 [R*S, K];
 * out: bf16 [R*S, H]. */
MOONEP_API int moonep_combine(const moonep_config *cfg, const moonep_plan_t *plan, const uint16_t *y,
                   const float *w, uint16_t *out, void *stream);

/* Backward of combine:
 *   dy_buf[dst_pos[t*K+k], h] = bf16_rne(w[t,k] * dy[t,h])   (one fp32 product;
 *                                dy itself with MOONEP_FLAG_BWD_UNSCALED)
 *   dw[t, k] = sum_h dy[t,h] * y[dst_pos[t*K+k], h]          (fp32 accumulation)
 * dy: bf16 [R*S, H]; w: fp32 [R*S, K]; y: bf16 [R, S*K, H];
 * dy_buf: bf16 [R, S*K, H]; dw: fp32 [R*S, K].  K <= 16 (each of a token's
 * K dot products is kept in registers); MOONEP_ERR_LIMIT above that. */
MOONEP_API int moonep_combine_backward(const moonep_config *cfg, const moonep_plan_t *plan, const uint16_t *dy,
                            const float *w, const uint16_t *y, uint16_t *dy_buf, float *dw,
                            void *stream);

/* Replica-gradient reduction (MoonEP explainer, memory tab, training
 * branch: replica grads land in an fp32 reduce buffer mapped as
 * [R, B, ...]; they are pulled back to the home expert and zeroed for the
 * next microbatch).  For every expert with prefetched replicas, in
 * ascending host rank order:
 *   home_grad[e, i] = home_grad[e, i] + reduce_buf[r, slot - L, i]
 * (separate fp32 adds), then those reduce_buf rows are set to 0.
 * reduce_buf: fp32 [R, B, P]; home_grad: fp32 [E, P]; P > 0 elements per
 * expert gradient.  Overflow replicas have no rows and are skipped. */
MOONEP_API int moonep_reduce_replica_grads(const moonep_config *cfg, const moonep_plan_t *plan,
                                float *reduce_buf, float *home_grad, int64_t P, void *stream);

/* Replica weight prefetch (MoonEP article, "The core idea": duplicated
 * experts are prefetched before expert computation; explainer, memory tab:
 * the prefetch slots are rows [E, E+B) of one contiguous weight pool, E read
 * here as the rank's L home experts, and a rank needing more than B foreign
 * experts reads the overflow from the home copy).
 *   pool[r][b][:] = weights[e][:]  for every replica of expert e on rank r
 *                                  with ordinal b = slot - L < B
 *   slot_wrow[r][s] = weight row the expert computation of slot s of rank r
 *       uses, in the concatenated row space [weights (E rows) | pool (R*B rows)]:
 *       home slot -> e, prefetched replica -> E + r*B + b, overflow replica
 *       -> e (read-through), unused slot -> -1.
 * weights: bf16 [E, P] (one expert's weights per row, e.g. gate+up+down);
 * pool: bf16 [R, B, P] (may be NULL when B == 0); slot_wrow: int32 [R][E];
 * P > 0 elements per expert.  Pool rows of unused slots are left as they
 * are.  A plan with MOONEP_ST_EXPERT_ID_RANGE copies nothing and marks every
 * slot -1. */
MOONEP_API int moonep_prefetch_replicas(const moonep_config *cfg, const moonep_plan_t *plan,
                                        const uint16_t *weights, uint16_t *pool, int32_t *slot_wrow,
                                        int64_t P, void *stream);

/* ---- expert parallelism over several GPUs ---------------------------- */
/* The pages' deployment (MoonEP article, "The core idea: dynamic redundant
 * experts": tokens are written directly into their expert-grouped positions
 * on remote ranks; explainer, pillars tab: NVLink and symmetric memory;
 * memory tab: the home rank pulls its replicas' gradient rows back over
 * NVLink).  One process per GPU; rank `rank` of R owns its S tokens
 * (topk_local [S, K], hidden_local / out_local / dy_local [S, H], w_local and
 * dw_local [S, K]), its receive buffer [S*K, H] (row j is global row
 * rank*S*K + j of the single-GPU buffer), its reduce buffer [B, P] and the
 * gradients of its L home experts [L, P].  Other ranks' buffers are reached
 * through device arrays of R device pointers (index = rank; peer memory
 * mapped into this process, e.g. symmetric memory or CUDA IPC, or R
 * allocations of one GPU); each pointer must be 16-byte aligned, and a null
 * or misaligned one is skipped and reported as MOONEP_ST_ROW_RANGE.  Loads
 * and stores to peers are plain 16-byte vector accesses.
 * Per MoE layer:
 *   1. moonep_ep_count: this rank's counts row [E + 1] (pairs per expert,
 *      then the number of ids outside [0, E));
 *   2. the caller all-gathers the R rows into counts_all [R, E + 1] (row r
 *      from rank r; 4 (E + 1) bytes per rank, e.g. an NCCL all-gather);
 *   3. moonep_ep_plan: every rank plans from counts_all -- plan tables equal
 *      to moonep_plan's for the concatenation of all ranks' routings, on
 *      every rank -- and places its own pairs: plan->dst_pos[0 .. S*K) holds
 *      the global buffer rows of its pairs (t*K + k, t local); plan->row_src
 *      is not written, and info[MOONEP_INFO_N_REMOTE_PAIRS] counts this
 *      rank's pairs placed on other ranks;
 *   4. moonep_ep_dispatch / combine / combine_backward /
 *      reduce_replica_grads / prefetch_replicas move the data over the peer
 *      pointers.
 * No call synchronises the host, and none issues a collective.
 * Sizes: moonep_ep_sizes (the plan block is laid out by moonep_plan_layout;
 * the workspace, one per rank, is zero-filled once and left ready for the
 * next call with the same configuration). */
MOONEP_API int moonep_ep_sizes(const moonep_config *cfg, size_t *plan_bytes, size_t *workspace_bytes);

/* counts_row[e] = pairs of this rank's topk_local [S, K] routed to expert e;
 * counts_row[E] = its ids outside [0, E).  One launch. */
MOONEP_API int moonep_ep_count(const moonep_config *cfg, const int32_t *topk_local, int32_t *counts_row,
                               void *workspace, void *stream);

/* The plan from the gathered counts [R, E + 1] (an id outside [0, E) on any
 * rank empties the plan, as in moonep_plan; counts that do not add up to
 * R*S*K give MOONEP_ST_WORKSPACE), and the global rows of this rank's pairs:
 * a pair's rank within its expert is the lower ranks' counts of that expert
 * plus its rank among this rank's own pairs in (t, k) order, the global
 * order of moonep_plan.  Uses the per-chunk counts moonep_ep_count left in
 * `workspace`: call it with the same workspace and topk_local.  One launch
 * in which every CTA plans from the gathered counts and places its own
 * chunk's pairs (two launches, a planner CTA then the assignment grid, where
 * that does not fit one CTA's shared memory, or after
 * moonep_set_plan_path(1)). */
MOONEP_API int moonep_ep_plan(const moonep_config *cfg, int32_t rank, const int32_t *topk_local,
                              const int32_t *counts_all, const moonep_plan_t *plan, void *workspace,
                              void *stream);

/* bufs[r] + (g - r*S*K)*H receives hidden_local[t] for every pair (t, k) of
 * this rank with global row g = plan->dst_pos[t*K + k], r = g / (S*K). */
MOONEP_API int moonep_ep_dispatch(const moonep_config *cfg, const moonep_plan_t *plan,
                                  const uint16_t *hidden_local, uint16_t *const *bufs, void *stream);

/* out_local[t] = bf16_rne(sum_k w_local[t,k] * y[g]) with the rows y[g] read
 * from ys[r] as in moonep_ep_dispatch, fp32 fmaf in k order from 0. */
MOONEP_API int moonep_ep_combine(const moonep_config *cfg, const moonep_plan_t *plan, const uint16_t *const *ys,
                                 const float *w_local, uint16_t *out_local, void *stream);

/* The backward of moonep_ep_combine: dy_bufs rows get bf16_rne(w * dy)
 * (dy with MOONEP_FLAG_BWD_UNSCALED), dw_local[t,k] = sum_h dy * y; K <= 16. */
MOONEP_API int moonep_ep_combine_backward(const moonep_config *cfg, const moonep_plan_t *plan,
                                          const uint16_t *dy_local, const float *w_local,
                                          const uint16_t *const *ys, uint16_t *const *dy_bufs, float *dw_local,
                                          void *stream);

/* On home rank `rank`: for each of its experts e with prefetched replicas,
 * in ascending host rank order, home_grad_local[e - rank*L] += the replica's
 * row reduce_bufs[r] + (slot - L)*P (separate fp32 adds), then that remote
 * row is zeroed.  reduce_bufs: device array of R pointers to [B, P] fp32. */
MOONEP_API int moonep_ep_reduce_replica_grads(const moonep_config *cfg, int32_t rank, const moonep_plan_t *plan,
                                              float *const *reduce_bufs, float *home_grad_local, int64_t P,
                                              void *stream);

/* Replica weight prefetch on rank `rank` (the expert-parallel form of
 * moonep_prefetch_replicas): each prefetched replica of this rank (ordinal
 * b = slot - L < B) pulls its expert e's weight row from the home rank
 * h = e / L, weights[h] + (e - h*L)*P (each rank's [L, P] bf16 home weights,
 * through the pointer array), into pool_local[b] ([B, P] bf16).
 * slot_wrow_local [E] int32: home slot s -> s and prefetched replica -> L + b
 * (rows of this rank's [own weights | pool]); overflow replica of expert e
 * -> L + B + e (read through from its home rank); unused slot -> -1. */
MOONEP_API int moonep_ep_prefetch_replicas(const moonep_config *cfg, int32_t rank, const moonep_plan_t *plan,
                                           const uint16_t *const *weights, uint16_t *pool_local,
                                           int32_t *slot_wrow_local, int64_t P, void *stream);

/* Size of the fixed device array behind moonep_plan_noalloc (4 MiB).  The
 * large training shape (R=32, E=384, K=8, S=4096) needs about 0.5 MiB. */
#define MOONEP_NOALLOC_WORKSPACE_BYTES (4u << 20)

/* moonep_plan without a caller-supplied workspace -- the pages have no
 * counterpart; this is a convenience of this library.  It is for callers
 * that cannot allocate device memory themselves: code running inside a
 * runtime or framework that owns every device allocation (a preallocated
 * pool, a server that reserves all memory at start-up), or code that must
 * not call cudaMalloc on its hot path because it can synchronise the device.
 * The planner's scratch space is then a file-scope device array of
 * MOONEP_NOALLOC_WORKSPACE_BYTES that every GPU loading this library holds
 * until the process exits; this call allocates nothing.
 *  - Same inputs, outputs and results as moonep_plan (plan laid out by
 *    moonep_plan_layout); configurations whose workspace (moonep_plan_sizes)
 *    exceeds the array are rejected with MOONEP_ERR_NOALLOC_SIZE before any
 *    launch.
 *  - The first call on a device looks up the array's device address with
 *    cudaGetSymbolAddress (once per device, the device current); make that
 *    first call before any stream capture.  Host threads may make their
 *    first calls at the same time: the lookup is serialised and runs once.
 *  - Each call first clears the front of the array that must start at zero
 *    (the planner's counters and count buffers: an async memset on
 *    `stream`), because the array keeps the previous call's contents.
 *  - All calls on a device share the one array: calls that can overlap on
 *    the GPU (different streams without ordering) race and give wrong plans.
 */
MOONEP_API int moonep_plan_noalloc(const moonep_config *cfg, const int32_t *topk_idx,
                                   const moonep_plan_t *plan, void *stream);

/* Human-readable text for a MOONEP_* return code. */
MOONEP_API const char *moonep_error_string(int code);

/* Human-readable text for a device status word (plan->info[MOONEP_INFO_STATUS],
 * a set of MOONEP_ST_* bits): "ok" for 0, else the set bits' names joined by
 * '|' (unknown bits as "bit<n>").  The text is written into buf (at most len
 * bytes, always NUL-terminated when len > 0); the return value is buf, or an
 * empty static string when buf is NULL or len == 0.  Host-only. */
MOONEP_API const char *moonep_status_string(int status, char *buf, size_t len);

/* Iteration bound of the planner's bounded waits (about 100 ns per
 * iteration) for every moonep_plan / moonep_plan_noalloc call this process
 * makes afterwards: the two-kernel path's waits for the counts-ready and
 * plan-ready marks, the one-kernel path's wait for every chunk's counts.
 * Default 65536; a negative value restores it.  With 0 every wait gives up at
 * once and takes its fallback (the two-kernel path waits for the whole
 * histogram grid, which never depends on it; a one-kernel CTA counts every
 * pair itself), so the plan is still complete and exact, and
 * MOONEP_ST_WAIT_TIMEOUT is set.  This is how the fallbacks are tested
 * without making a mark late.  Host-only; returns the previous bound.  Calls
 * already enqueued keep the bound they were launched with. */
MOONEP_API int moonep_set_wait_limit(int iterations);

/* Which planner moonep_plan / moonep_plan_noalloc / moonep_ep_plan launch
 * afterwards in this process: 1 the two-kernel planner always; any other
 * value (0, the default) the one-kernel planner wherever it fits (for
 * moonep_plan: all of its CTAs on the device at once), else the two-kernel
 * one.  Both give the same plan; tests use 1 to compare them.  A workspace
 * may pass between the two.  Host-only; returns the previous setting (0 or
 * 1). */
MOONEP_API int moonep_set_plan_path(int mode);

/* The replica capacity the relay cascade's guard (MOONEP_FLAG_CASCADE)
 * compares with, for every moonep_plan / moonep_ep_plan call this process
 * makes afterwards: a repair step that could leave more live replicas than
 * this is not taken.  Default (capacity <= 0): the plan's E + R - 1, which
 * no tested routing comes within 3 of.  A smaller value only makes the
 * guard stricter (the plan's arrays keep their size), so tests use it to put
 * a step exactly on the limit and one over it.  Host-only; returns the
 * previous setting (0 for the default). */
MOONEP_API int moonep_set_cascade_capacity(int capacity);

/* MOONEP_ABI_VERSION of the loaded library. */
MOONEP_API int moonep_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MOONEP_H */
