// reatt_step_fixed_scratch: the whole step without any device allocation by
// the caller.  Some callers cannot hand the library a workspace: a plugin
// interface that gives its kernels no allocator, or a latency-critical loop
// where calling cudaMalloc would synchronize the device.  For them the
// workspace is a file-scope __device__ array of fixed size that lives as long
// as the library is loaded (each GPU that loads the library holds it until the
// process exits).
#include <mutex>

#include <cuda_runtime.h>

#include "reatt.h"

namespace {

constexpr size_t kFixedScratchBytes = size_t(16) << 20;   // 16 MiB

// The scratch itself.  In host code this name is only a host-side stand-in:
// its device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_fixed_scratch[kFixedScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_ptr[kMaxDevices];

// Device address of the scratch on the current device; resolved once per
// device (the first call loads the module's globals on that device).
int scratch_on_current_device(void **out)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return REATT_ECUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_fixed_scratch) != cudaSuccess || !p) return REATT_ECUDA;
        g_ptr[dev] = p;
    }
    *out = g_ptr[dev];
    return REATT_OK;
}

}  // namespace

extern "C" REATT_API int reatt_step_fixed_scratch(const reatt_dims *dims, const void *q,
                                                  const void *k_cache, const void *v_cache,
                                                  const void *k_cur, const void *v_cur,
                                                  int32_t *sel_out, float *out,
                                                  reatt_stream stream)
{
    size_t need = 0;
    const int rc = reatt_workspace_bytes(dims, &need);
    if (rc != REATT_OK) return rc;
    if (need > kFixedScratchBytes) return REATT_EUNSUPPORTED;   // does not fit the fixed scratch
    void *ws = nullptr;
    const int sc = scratch_on_current_device(&ws);
    if (sc != REATT_OK) return sc;
    return reatt_step(dims, q, k_cache, v_cache, k_cur, v_cur, sel_out, out, ws, stream);
}
