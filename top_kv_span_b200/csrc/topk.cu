// Top-k span selection (decoding pseudocode of the ReAttention OpenReview
// discussion: idx_recall = score.topk(...)), per (batch, KV head):
// the k_eff = min(k, NS) largest span scores, ties to the lower span id,
// emitted in ascending span order so the window keeps cache order.
//
// Scores are mapped to order-preserving uint32 codes.  A block radix select
// (4 passes of 8 bits, shared-memory histogram, one warp scans the bins) finds
// the code tau of the k-th largest and how many codes equal to tau are taken;
// a stable block compaction in index order then writes the chosen ids, which
// are therefore already ascending -- no sort is needed.
// NS <= kSlice: one CTA per head.  Larger NS: slice CTAs (kSlice scores each)
// emit their own top-k candidates in index order, and one merge CTA per head
// runs the same select on the candidates.  The global top-k under the total
// order (score desc, id asc) is always inside the union of the slices' top-k.
#include "common.cuh"
#include "kernels.h"

namespace reatt {

namespace {

constexpr int kTopkThreads = 512;
constexpr int kSlice = 4096;
constexpr int kMergeCap = 8192;

struct SelScratch {
    uint32_t hist[256];
    uint32_t bcast[2];
    uint32_t wsum[33];
};

// Exclusive block-wide prefix count of `flag`; *total receives the sum.
__device__ __forceinline__ int block_prefix(bool flag, uint32_t *wsum, int *total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const uint32_t bal = __ballot_sync(0xffffffffu, flag);
    const int pre = __popc(bal & ((1u << lane) - 1u));
    if (lane == 0) wsum[warp] = __popc(bal);
    __syncthreads();
    if (warp == 0) {
        const uint32_t v = lane < nw ? wsum[lane] : 0u;
        uint32_t inc = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t t = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += t;
        }
        if (lane < nw) wsum[lane] = inc - v;
        if (lane == 31) wsum[32] = inc;
    }
    __syncthreads();
    const int res = int(wsum[warp]) + pre;
    *total = int(wsum[32]);
    __syncthreads();
    return res;
}

// Radix select of the kk-th largest code among n (kk >= 1, kk <= number of
// real codes; padding codes are 0 and never reached).
template <class Get>
__device__ void radix_select(Get get, int n, uint32_t kk, SelScratch &sc, uint32_t &tau,
                             uint32_t &take_eq)
{
    uint32_t prefix = 0, mask = 0, remaining = kk;
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int i = threadIdx.x; i < 256; i += blockDim.x) sc.hist[i] = 0u;
        __syncthreads();
        for (int i = threadIdx.x; i < n; i += blockDim.x) {
            const uint32_t u = get(i);
            if ((u & mask) == prefix) atomicAdd(&sc.hist[(u >> shift) & 255u], 1u);
        }
        __syncthreads();
        if (threadIdx.x < 32) {
            const int lane = threadIdx.x;
            uint32_t c[8], tot = 0;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                c[e] = sc.hist[lane * 8 + e];
                tot += c[e];
            }
            uint32_t suf = tot;   // inclusive suffix over lanes >= lane
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t v = __shfl_down_sync(0xffffffffu, suf, o);
                if (lane + o < 32) suf += v;
            }
            const uint32_t above = suf - tot;
            if (above < remaining && remaining <= suf) {
                uint32_t acc = above;
                for (int e = 7; e >= 0; --e) {
                    if (acc + c[e] >= remaining) {
                        sc.bcast[0] = uint32_t(lane * 8 + e);
                        sc.bcast[1] = acc;
                        break;
                    }
                    acc += c[e];
                }
            }
        }
        __syncthreads();
        const uint32_t bin = sc.bcast[0], above = sc.bcast[1];
        remaining -= above;
        prefix |= bin << shift;
        mask |= 0xffu << shift;
        __syncthreads();
    }
    tau = prefix;
    take_eq = remaining;
}

// Stable compaction in index order: emit(pos, i) for every chosen i.
template <class Get, class Emit>
__device__ void compact(Get get, int n, uint32_t tau, uint32_t take_eq, SelScratch &sc, Emit emit)
{
    int out_base = 0, eq_base = 0;
    for (int start = 0; start < n; start += blockDim.x) {
        const int i = start + threadIdx.x;
        const uint32_t u = i < n ? get(i) : 0u;
        const bool gt = i < n && u > tau;
        const bool eq = i < n && u == tau;
        int eq_tot, sel_tot;
        const int eq_rank = block_prefix(eq, sc.wsum, &eq_tot);
        const bool chosen = gt || (eq && uint32_t(eq_base + eq_rank) < take_eq);
        const int pos = block_prefix(chosen, sc.wsum, &sel_tot);
        if (chosen) emit(out_base + pos, i);
        out_base += sel_tot;
        eq_base += eq_tot;
    }
}

__global__ void __launch_bounds__(kTopkThreads)
topk_slice_kernel(Geom geo, const float *__restrict__ scores, int32_t *__restrict__ sel,
                  uint32_t *__restrict__ cand_code, int32_t *__restrict__ cand_idx, int nslices,
                  int kkp, uint32_t *zero_words, int nzero)
{
    __shared__ uint32_t codes[kSlice];
    __shared__ SelScratch sc;
    const int64_t bh = blockIdx.y;
    const int slice = blockIdx.x;
    if (zero_words && slice == 0 && bh == 0)
        for (int i = threadIdx.x; i < nzero; i += blockDim.x) zero_words[i] = 0u;

    const int64_t s_begin = int64_t(slice) * kSlice;
    int n = int(geo.NS - s_begin < kSlice ? geo.NS - s_begin : kSlice);
    if (n < 0) n = 0;
    const float *src = scores + bh * geo.NS + s_begin;
    for (int i = threadIdx.x; i < n; i += blockDim.x) codes[i] = order_code(src[i]);
    __syncthreads();
    const int kk = geo.k < n ? geo.k : n;
    auto get = [&](int i) { return codes[i]; };
    if (nslices == 1) {
        int32_t *out = sel + bh * geo.k;
        if (kk > 0) {
            uint32_t tau, take;
            radix_select(get, n, uint32_t(kk), sc, tau, take);
            compact(get, n, tau, take, sc, [&](int pos, int i) { out[pos] = int32_t(i); });
        }
        for (int i = kk + threadIdx.x; i < geo.k; i += blockDim.x) out[i] = -1;
    } else {
        uint32_t *oc = cand_code + (bh * nslices + slice) * int64_t(kkp);
        int32_t *oi = cand_idx + (bh * nslices + slice) * int64_t(kkp);
        if (kk > 0) {
            uint32_t tau, take;
            radix_select(get, n, uint32_t(kk), sc, tau, take);
            compact(get, n, tau, take, sc, [&](int pos, int i) {
                oc[pos] = codes[i];
                oi[pos] = int32_t(s_begin + i);
            });
        }
        for (int i = kk + threadIdx.x; i < kkp; i += blockDim.x) {
            oc[i] = 0u;
            oi[i] = -1;
        }
    }
}

__global__ void __launch_bounds__(kTopkThreads)
topk_merge_kernel(Geom geo, const uint32_t *__restrict__ cand_code,
                  const int32_t *__restrict__ cand_idx, int32_t *__restrict__ sel, int ncand)
{
    __shared__ uint32_t codes[kMergeCap];
    __shared__ SelScratch sc;
    const int64_t bh = blockIdx.x;
    const uint32_t *gc = cand_code + bh * int64_t(ncand);
    const int32_t *gi = cand_idx + bh * int64_t(ncand);
    const bool in_smem = ncand <= kMergeCap;
    if (in_smem)
        for (int i = threadIdx.x; i < ncand; i += blockDim.x) codes[i] = gc[i];
    __syncthreads();
    const int keff = int(geo.k < geo.NS ? geo.k : geo.NS);
    int32_t *out = sel + bh * geo.k;
    if (keff > 0) {
        uint32_t tau, take;
        auto get = [&](int i) { return in_smem ? codes[i] : __ldg(gc + i); };
        radix_select(get, ncand, uint32_t(keff), sc, tau, take);
        compact(get, ncand, tau, take, sc, [&](int pos, int i) { out[pos] = gi[i]; });
    }
    for (int i = keff + threadIdx.x; i < geo.k; i += blockDim.x) out[i] = -1;
}

struct TopkPlan {
    int nslices, kkp;
};
TopkPlan topk_plan(const Geom &geo)
{
    TopkPlan p;
    p.nslices = geo.NS <= kSlice ? 1 : int((geo.NS + kSlice - 1) / kSlice);
    p.kkp = geo.k < kSlice ? geo.k : kSlice;
    return p;
}

}  // namespace

size_t topk_ws_bytes(const Geom &geo)
{
    const TopkPlan p = topk_plan(geo);
    if (p.nslices <= 1 || geo.k == 0) return 0;
    return size_t(geo.B) * geo.Hkv * p.nslices * p.kkp * (sizeof(uint32_t) + sizeof(int32_t));
}

cudaError_t launch_topk(const Geom &geo, const float *scores, int32_t *sel, void *scratch,
                        uint32_t *zero_words, int nzero, cudaStream_t st)
{
    const int BH = geo.B * geo.Hkv;
    if (geo.k == 0 && nzero == 0) return cudaSuccess;
    const TopkPlan p = topk_plan(geo);
    uint32_t *cc = static_cast<uint32_t *>(scratch);
    int32_t *ci = reinterpret_cast<int32_t *>(
        cc + (p.nslices > 1 ? size_t(BH) * p.nslices * p.kkp : 0));
    dim3 grid(unsigned(p.nslices), unsigned(BH));
    topk_slice_kernel<<<grid, kTopkThreads, 0, st>>>(geo, scores, sel, cc, ci, p.nslices, p.kkp,
                                                     zero_words, nzero);
    if (p.nslices > 1 && geo.k > 0)
        topk_merge_kernel<<<BH, kTopkThreads, 0, st>>>(geo, cc, ci, sel, p.nslices * p.kkp);
    return cudaGetLastError();
}

}  // namespace reatt
