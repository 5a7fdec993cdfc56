// Split-K decode with a scratch area compiled into the library.
//
// pa_decode's split-K modes keep their partial outputs and log-sum-exp values
// in a workspace the caller allocates.  Some callers cannot
// allocate device memory where they decode: an engine that has handed all free
// device memory to its KV block pool up front, or a host integration that has
// no device allocator of its own.  pa_decode_fixed_scratch serves them: it runs
// exactly pa_decode, with the workspace pointed at the fixed area below instead
// of a caller buffer.  Nothing is allocated by the library, and the call uses no
// allocating routine.
//
// The area is one file-scope __device__ array of PA_FIXED_SCRATCH_BYTES, so each
// device that loads this module holds one copy.  Because of that:
//   * the first call on a device does the setup: it looks up the array's device
//     address (cudaGetSymbolAddress, with that device current); make that first
//     call before any stream capture.  Nothing in the area needs clearing: every
//     value a call reads there was written earlier in the same call;
//   * all calls on one device share the one area, so calls that overlap on the
//     device (on different streams, or from different host threads without
//     ordering) race on it: issue them in one stream order;
//   * parameters whose workspace is larger than PA_FIXED_SCRATCH_BYTES are
//     rejected with PA_ERR_WORKSPACE before anything is launched;
//   * calls with different parameters share the area safely, for the same
//     reason;
//   * the device address is looked up once per device and kept for the process:
//     after cudaDeviceReset the library must not be used again (its kernel
//     attributes and encoded copy descriptors are per-context state as well).
#include <cuda_runtime.h>

#include <mutex>

#include "pa.h"
#include "pa_internal.h"

namespace pa {
namespace {

__device__ __align__(256) unsigned char g_fixed_scratch[PA_FIXED_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_ptr[kMaxDevices];  // device address of g_fixed_scratch per device, once set up

// Device address of the fixed area on the current device, looked up by the first
// call per device.
int fixed_scratch(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return PA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return PA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_scratch_ptr[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_fixed_scratch) != cudaSuccess || p == nullptr) return PA_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return PA_OK;
}

}  // namespace
}  // namespace pa

extern "C" int pa_decode_fixed_scratch(void *out, const void *q, const void *key_cache, const void *value_cache,
                                       const int32_t *block_tables, const int32_t *seq_lens, float scale,
                                       const pa_decode_params *p, pa_stream_t stream) {
    if (!p) return PA_ERR_NULL;
    pa_decode_params p2 = *p;
    p2.workspace = nullptr;
    p2.workspace_bytes = 0;
    const size_t need = pa_decode_workspace_size(&p2);
    if (need > PA_FIXED_SCRATCH_BYTES) return PA_ERR_WORKSPACE;
    if (need > 0) {
        void *ws = nullptr;
        const int rc = pa::fixed_scratch(&ws);
        if (rc != PA_OK) return rc;
        p2.workspace = ws;
        p2.workspace_bytes = PA_FIXED_SCRATCH_BYTES;
    }
    return pa_decode(out, q, key_cache, value_cache, block_tables, seq_lens, scale, &p2, stream);
}
