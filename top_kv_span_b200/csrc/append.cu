// Appending the current tokens' K and V rows to the caches: the caller's step
// between two calls of the decoding loop or of the chunked prefill
// (ReAttention OpenReview discussion, "Prefilling Phase" / "Decoding Phase"
// pseudocode: the chunk's or new token's key and value join the cache after
// the attention).  Needs caches allocated with T_cap >= T + C rows per
// (batch, KV head).
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"
#include "reatt.h"

namespace reatt {
namespace {

// One 16-byte word per thread: cur row c of (b, h) -> cache row T + c.
__global__ void append_kernel(Geom geo, const uint4 *__restrict__ kcur,
                              const uint4 *__restrict__ vcur, uint4 *__restrict__ kc,
                              uint4 *__restrict__ vc, int words_per_row)
{
    const int64_t per_bh = int64_t(geo.C) * words_per_row;
    const int64_t n = int64_t(geo.B) * geo.Hkv * per_bh;
    for (int64_t x = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; x < n;
         x += int64_t(gridDim.x) * blockDim.x) {
        const int64_t bh = x / per_bh, r = x - bh * per_bh;
        const int64_t c = r / words_per_row, w = r - c * words_per_row;
        const int64_t dst = (bh * geo.Ts + geo.T + c) * words_per_row + w;
        kc[dst] = kcur[x];
        vc[dst] = vcur[x];
    }
}

}  // namespace

cudaError_t launch_append(const Geom &g, void *k_cache, void *v_cache, const void *k_cur,
                          const void *v_cur, cudaStream_t st)
{
    const int row_bytes = g.d * (g.dtype == REATT_BF16 ? 2 : 4);
    const int words = row_bytes / 16;
    const int64_t n = int64_t(g.B) * g.Hkv * g.C * words;
    const int threads = 256;
    int64_t blocks = (n + threads - 1) / threads;
    const int64_t cap = int64_t(num_sms()) * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) return cudaSuccess;
    append_kernel<<<unsigned(blocks), threads, 0, st>>>(
        g, static_cast<const uint4 *>(k_cur), static_cast<const uint4 *>(v_cur),
        static_cast<uint4 *>(k_cache), static_cast<uint4 *>(v_cache), words);
    return cudaGetLastError();
}

}  // namespace reatt
