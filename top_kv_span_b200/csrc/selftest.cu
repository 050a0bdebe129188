// Diagnostic: exercise the bounded-wait path of the kernels without any fault.
// One thread waits on an mbarrier that nothing ever arrives on; after the
// caller's limit it records REATT_ETIMEOUT in the workspace status word (the
// same helpers the ring kernels use) and returns, leaving the context usable.
#include "common.cuh"
#include "reatt.h"

namespace reatt {
namespace {

__global__ void bounded_wait_kernel(void *ws, uint64_t limit_ns)
{
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        mbar_init_fence();
    }
    __syncthreads();
    if (threadIdx.x == 0 && !mbar_wait_bounded(&bar, 0, limit_ns))
        report_status(ws, REATT_ETIMEOUT);
}

}  // namespace
}  // namespace reatt

extern "C" REATT_API int reatt_selftest_bounded_wait(void *ws, int64_t limit_ns, reatt_stream stream)
{
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 15u) != 0) return REATT_EINVAL;
    if (limit_ns <= 0 || limit_ns > int64_t(10) * 1000000000) return REATT_EINVAL;
    reatt::bounded_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        ws, uint64_t(limit_ns));
    return cudaGetLastError() == cudaSuccess ? REATT_OK : REATT_ECUDA;
}
