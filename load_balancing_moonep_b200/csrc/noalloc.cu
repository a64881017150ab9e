// moonep_plan_noalloc: the planner with its scratch memory in a fixed,
// file-scope device array instead of a caller-supplied workspace.
//
// Some callers cannot hand the planner a workspace: code running under a
// framework or runtime that owns every device allocation (a preallocated
// memory pool, an inference server that reserves all device memory at
// start-up), or code that must not call cudaMalloc on the hot path because
// it can synchronise the device and fragment the pool.  For them this entry
// point allocates nothing: the scratch space is the array below, which every
// GPU that loads the library keeps until the process exits.
#include <atomic>
#include <cstdint>
#include <mutex>

#include "common.cuh"

namespace moonep {
int workspace_clear_bytes(const moonep_config *cfg, size_t *bytes);
}

// Scratch space shared by every moonep_plan_noalloc call on a device.
static __device__ __align__(256) unsigned char g_noalloc_ws[MOONEP_NOALLOC_WORKSPACE_BYTES];

namespace {

constexpr int MAX_DEVICES = 64;
// device address of g_noalloc_ws, per device; written once under the mutex,
// read without it afterwards
std::atomic<void *> g_ws_ptr[MAX_DEVICES];
std::mutex g_ws_mutex;

// Once per device, with that device current: the device address of the
// array (its name in host code is only a host-side stand-in).  Host threads
// that make their first call on a device at the same time are serialised by
// the mutex, so the lookup runs once per device.
int noalloc_setup(void **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) return MOONEP_ERR_CUDA;
    void *p = g_ws_ptr[dev].load(std::memory_order_acquire);
    if (!p) {
        std::lock_guard<std::mutex> lock(g_ws_mutex);
        p = g_ws_ptr[dev].load(std::memory_order_acquire);
        if (!p) {
            if (cudaGetSymbolAddress(&p, g_noalloc_ws) != cudaSuccess || !p) return MOONEP_ERR_CUDA;
            g_ws_ptr[dev].store(p, std::memory_order_release);
        }
    }
    *out = p;
    return MOONEP_OK;
}

}  // namespace

extern "C" {

int moonep_plan_noalloc(const moonep_config *cfg, const int32_t *topk_idx, const moonep_plan_t *plan,
                        void *stream)
{
    size_t plan_bytes = 0, ws_bytes = 0, clear_bytes = 0;
    const int rc = moonep_plan_sizes(cfg, &plan_bytes, &ws_bytes);
    if (rc != MOONEP_OK) return rc;
    if (ws_bytes > MOONEP_NOALLOC_WORKSPACE_BYTES) return MOONEP_ERR_NOALLOC_SIZE;
    if (!topk_idx || !plan) return MOONEP_ERR_ARG;
    if (cfg->flags & MOONEP_FLAG_LOCALITY) return MOONEP_ERR_ARG;  // as moonep_plan: expert parallelism only
    const int crc = moonep::workspace_clear_bytes(cfg, &clear_bytes);
    if (crc != MOONEP_OK) return crc;
    void *ws = nullptr;
    const int src = noalloc_setup(&ws);
    if (src != MOONEP_OK) return src;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // The array keeps whatever the previous call (of any configuration) left
    // there.  The planner needs its header and group counts zeroed on entry;
    // the per-chunk counts and host rows behind them are written in full
    // before they are read, so only the front of the region is cleared.
    if (cudaMemsetAsync(ws, 0, clear_bytes, st) != cudaSuccess) return MOONEP_ERR_CUDA;
    return moonep_plan(cfg, topk_idx, plan, ws, stream);
}

}  // extern "C"
