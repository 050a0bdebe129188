// reatt_step_fixed_scratch: the whole step without any device allocation by
// the caller.  Some callers cannot hand the library a workspace: a plugin
// interface that gives its kernels no allocator, or a latency-critical loop
// where calling cudaMalloc would synchronize the device.  For them the
// workspace is a file-scope __device__ array of fixed size that lives as long
// as the library is loaded (each GPU that loads the library holds it until the
// process exits).
#include <cuda_runtime.h>

#include "reatt.h"

namespace {

constexpr size_t kFixedScratchBytes = size_t(16) << 20;   // 16 MiB

// The scratch itself.  In host code this name is only a host-side stand-in:
// its device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_fixed_scratch[kFixedScratchBytes];

// Device address of the scratch on the current device, looked up on every
// call (a lookup, no synchronisation).  Nothing is cached: after a
// cudaDeviceReset the library's globals are loaded again into the new context,
// possibly at another address, and a cached pointer would be stale.  The first
// lookup on a device loads the module's globals there.
int scratch_on_current_device(void **out)
{
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_fixed_scratch) != cudaSuccess || !p) return REATT_ECUDA;
    *out = p;
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

extern "C" REATT_API int reatt_fixed_scratch_address(void **ws_out)
{
    if (!ws_out) return REATT_EINVAL;
    return scratch_on_current_device(ws_out);
}
