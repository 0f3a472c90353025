// ssd_noalloc.cu -- ssd_prefill for callers that cannot allocate device memory.
//
// Some callers have no way to hand the library a workspace: code running
// inside a framework whose allocator is not exposed to it, plug-ins that may
// only call into pre-built libraries, or code paths where a cudaMalloc would
// synchronise the device or fail because memory is reserved up front.  For
// them, ssd_prefill_noalloc runs the same prefill with its scratch (the
// post-conv B and C channels of every token) in a fixed array that lives in
// this library's device image, so the call itself allocates nothing.
//
// The array is SSD_NOALLOC_SCRATCH_BYTES (16 MiB) and every GPU that loads
// the library holds it until the process exits.  Its device address is looked
// up once per device, on the first call made with that device current; make
// that first call before any stream capture.  The address is cached by device
// index for the life of the process: a cudaDeviceReset (or any other teardown
// of the device's primary context) between calls leaves it stale, so this
// entry point must not be used across a device reset in one process.  All calls share the one array:
// calls whose kernels overlap on the GPU (e.g. on two streams) race on it.
// Nothing in it has to start at zero: the B/C prologue writes every element
// that the chunk scan then reads, so leftovers from the previous call are
// never seen.
#include <mutex>

#include "ssd.h"
#include "ssd_common.cuh"
#include "ssd_internal.h"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[SSD_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_lock;
void* g_scratch_ptr[kMaxDevices] = {};

// The array's device address on the current device (looked up once per device).
ssd_status scratch_for_current_device(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SSD_ERR_CUDA;
    std::lock_guard<std::mutex> guard(g_lock);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return SSD_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return SSD_OK;
}

}  // namespace

extern "C" ssd_status ssd_prefill_noalloc(const ssd_dims* d, ssd_dtype dtype, const ssd_params* params,
                                          const void* x, const void* dt, const void* B, const void* C,
                                          const void* z, const float* init_state, const void* init_conv_state,
                                          void* y, float* final_state, void* conv_state, void* stream) {
    const int path = ssd_prefill_path(d, dtype);
    if (path < 0) return static_cast<ssd_status>(-path);
    const size_t need = ssd_prefill_workspace_bytes(d, dtype);
    if (need > (size_t)SSD_NOALLOC_SCRATCH_BYTES) return SSD_ERR_WORKSPACE;
    void* scratch = nullptr;
    if (need > 0) {
        const ssd_status st = scratch_for_current_device(&scratch);
        if (st != SSD_OK) return st;
    }
    return ssd_prefill(d, dtype, params, x, dt, B, C, z, init_state, init_conv_state, y, final_state, conv_state,
                       scratch, need, stream);
}
