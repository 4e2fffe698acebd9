// sa_select_noalloc: the per-step selection for callers that cannot allocate
// device memory.
//
// Some callers have no way to obtain scratch: code running where cudaMalloc
// is forbidden or unsafe (inside an allocator's own hooks, in a process whose
// device memory is entirely pre-partitioned by another runtime, or in a
// plug-in that may only use the buffers it is handed).  This entry point takes
// the same inputs and outputs as sa_select but keeps its scratch in a fixed
// array compiled into the library, so it never allocates.
//
// The array (kNoAllocScratchBytes, 8 MiB) lives on every GPU that loads the
// library until the process exits.  It is shared by every call on a device and
// keeps whatever the last call left there, so:
//   * the completion counters at its start are cleared (cudaMemsetAsync on the
//     caller's stream) before every call;
//   * calls that overlap on the GPU (different streams, no ordering between
//     them) race on the array and must not be issued.
// The device address of the array is looked up once per device, on the first
// call made with that device current (cudaGetSymbolAddress); issue that first
// call before any stream capture.
#include <mutex>

#include "sa_internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = 8u << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_select_scratch[kNoAllocScratchBytes];

std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of this device's copy of the scratch array (looked up once).
sa_status scratch_for_current_device(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (g_scratch_ptr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_select_scratch) != cudaSuccess || p == nullptr) return SA_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return SA_OK;
}

}  // namespace

extern "C" {

sa_status sa_select_noalloc(const sa_shape* shape, const sa_select_params* params, const void* q,
                            const sa_stats* stats, const void* k, const void* v, const sa_selection* out,
                            float scale, void* stream) {
    // every argument check first: a rejected call enqueues nothing and leaves
    // the shared array as it was
    sa_status e = sa::check_select_call(shape, params, q, stats, k, v, out, scale);
    if (e != SA_OK) return e;
    const size_t need = sa_workspace_size(shape, params, SA_OP_SELECT);
    if (need == 0) return SA_ERR_INVALID_ARG;
    if (need > kNoAllocScratchBytes) return SA_ERR_WORKSPACE;     // shape too large for the fixed array
    void* ws = nullptr;
    e = scratch_for_current_device(&ws);
    if (e != SA_OK) return e;
    // the completion counters (two per unit: selection and CLT budget, at offset 0 of its
    // workspace) must start at zero; the array may hold a previous call's data
    const size_t counters = sa::align256(sizeof(unsigned) * 2 * (size_t)shape->B * (size_t)shape->Hkv);
    if (cudaMemsetAsync(ws, 0, counters, static_cast<cudaStream_t>(stream)) != cudaSuccess) return SA_ERR_CUDA;
    return sa_select(shape, params, q, stats, k, v, out, scale, ws, kNoAllocScratchBytes, stream);
}

}  // extern "C"
