// Top-k span selection (decoding pseudocode of the ReAttention OpenReview
// discussion: idx_recall = score.topk(...)), per (batch, KV head):
// the k_eff = min(k, NS) largest span scores, ties to the lower span id,
// emitted in ascending span order so the window keeps cache order.
//
// Scores are mapped to order-preserving uint32 codes.  A block radix select
// finds the code tau of the k-th largest and how many codes equal to tau are
// taken.  The path every slice and merge of up to 8192 codes takes keeps the
// codes in registers, skips the high bits that the block's largest and
// smallest code share, resolves the rest with 11-bit digits (2048-bin
// shared-memory histogram) and, once at most 32 codes share the digit prefix,
// lets one warp rank them directly.  Larger candidate sets fall back to a
// generic select of 4 passes of 8 bits read from memory.  A stable block
// compaction in index order then writes the chosen ids, which are therefore
// already ascending -- no sort is needed.
// CTAs of 1024 threads.  NS <= 4096: one CTA per head, 4 codes per thread;
// NS <= 8192: one CTA per head, 8 codes per thread (no second launch).
// Larger NS: slice CTAs (4096 scores each, 4 codes per thread: faster than
// 8192-score slices and a smaller merge) emit their own top-k candidates in index order, and one
// merge CTA per head runs the same select on the candidates.  The global
// top-k under the total order (score desc, id asc) is always inside the union
// of the slices' top-k.
#include "common.cuh"
#include "kernels.h"
#include "select.cuh"

namespace reatt {

namespace {

#ifndef REATT_TOPK_THREADS
#define REATT_TOPK_THREADS 1024
#endif
constexpr int kTopkThreads = REATT_TOPK_THREADS;
constexpr int kSlice = 4096;        // 4 codes per thread: small heads and every slice
constexpr int kSliceWide = 8192;    // 8 codes per thread: the largest head one CTA takes
constexpr int kMaxE = 16;           // codes per thread of the merge's register path

// cos/sin table of the window positions: tab[p*(d/2) + i] = (cos, sin) of
// p * base^(-2i/d), for p < Wmax.  Filled by spare CTAs of the top-k launch,
// kTabRows positions per CTA.
constexpr int kTabRows = 64;

__device__ void fill_rope_table(const Geom &geo, float2 *tab, int64_t chunk)
{
    __shared__ float2 freq[64];
    const int half = geo.d / 2;                 // 32 or 64
    if (threadIdx.x < half) freq[threadIdx.x] = make_float2(geo.rope_hi[threadIdx.x], geo.rope_lo[threadIdx.x]);
    __syncthreads();
    const int rows_per_pass = kTopkThreads / half;
    const int i = threadIdx.x % half;
    const float hi = freq[i].x, lo = freq[i].y;
    const int64_t p_end0 = (chunk + 1) * kTabRows;
    const int64_t p_end = p_end0 < geo.Wmax ? p_end0 : geo.Wmax;
    for (int64_t p = chunk * kTabRows + threadIdx.x / half; p < p_end; p += rows_per_pass) {
        float c, s;
        rope_cs(p, hi, lo, c, s);
        tab[p * half + i] = make_float2(c, s);
    }
}

template <int E>
__global__ void __launch_bounds__(kTopkThreads)
topk_slice_kernel(Geom geo, const float *__restrict__ scores, int32_t *__restrict__ sel,
                  uint32_t *__restrict__ cand_code, int32_t *__restrict__ cand_idx, int nslices,
                  int kkp, uint32_t *zero_words, int nzero, float2 *rope_tab, int codes)
{
    __shared__ sel::Scratch rs;
    auto bsync = [] { __syncthreads(); };
    const int t = threadIdx.x;
    const int BH = geo.B * geo.Hkv;
    pdl_wait();      // scores come from the preceding scan
    pdl_trigger();   // the attention may launch and wait in turn
    if (int(blockIdx.y) >= BH) {   // spare CTA: a chunk of the RoPE table
        fill_rope_table(geo, rope_tab, int64_t(blockIdx.y - BH) * nslices + blockIdx.x);
        return;
    }
    const int64_t bh = blockIdx.y;
    const int slice = blockIdx.x;
    if (zero_words && slice == 0 && bh == 0)
        for (int i = threadIdx.x; i < nzero; i += blockDim.x) zero_words[i] = 0u;

    constexpr int kS = E * kTopkThreads;   // scores of one slice
    const int64_t s_begin = int64_t(slice) * kS;
    int n = int(geo.NS - s_begin < kS ? geo.NS - s_begin : kS);
    if (n < 0) n = 0;
    const float *src = scores + bh * geo.NS + s_begin;
    const int i0 = int(threadIdx.x) * E;
    const int mine = n - i0 < 0 ? 0 : (n - i0 > E ? E : n - i0);
    uint32_t u[E];
#pragma unroll
    for (int e = 0; e < E; ++e)
        u[e] = e < mine ? (codes ? __float_as_uint(src[i0 + e]) : order_code(src[i0 + e])) : 0u;
    const int kk = geo.k < n ? geo.k : n;
    if (nslices == 1) {
        int32_t *out = sel + bh * geo.k;
        if (kk > 0) {
            uint32_t tau, take;
            sel::select_regs<kTopkThreads, E>(t, u, mine, uint32_t(kk), rs, tau, take, bsync);
            sel::compact_regs<kTopkThreads, E>(
                t, u, mine, tau, take, i0, rs, [&](int pos, int i) { out[pos] = int32_t(i); },
                bsync);
        }
        for (int i = kk + threadIdx.x; i < geo.k; i += blockDim.x) out[i] = -1;
    } else {
        uint32_t *oc = cand_code + (bh * nslices + slice) * int64_t(kkp);
        int32_t *oi = cand_idx + (bh * nslices + slice) * int64_t(kkp);
        if (kk > 0) {
            uint32_t tau, take;
            sel::select_regs<kTopkThreads, E>(t, u, mine, uint32_t(kk), rs, tau, take, bsync);
            sel::compact_regs<kTopkThreads, E>(
                t, u, mine, tau, take, i0, rs,
                [&](int pos, int i) {
                    oc[pos] = codes ? __float_as_uint(src[i]) : order_code(src[i]);
                    oi[pos] = int32_t(s_begin + i);
                },
                bsync);
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
    pdl_wait();
    pdl_trigger();
    const int64_t bh = blockIdx.x;
    const uint32_t *gc = cand_code + bh * int64_t(ncand);
    const int32_t *gi = cand_idx + bh * int64_t(ncand);
    const int keff = int(geo.k < geo.NS ? geo.k : geo.NS);
    int32_t *out = sel + bh * geo.k;
    auto bsync = [] { __syncthreads(); };
    const int t = threadIdx.x;
    if (ncand <= kTopkThreads * kMaxE) {
        __shared__ sel::Scratch rs;
        constexpr int E = kMaxE;
        const int per = (ncand + kTopkThreads - 1) / kTopkThreads;
        const int i0 = t * per;
        const int mine = ncand - i0 < 0 ? 0 : (ncand - i0 > per ? per : ncand - i0);
        uint32_t u[E];
#pragma unroll
        for (int e = 0; e < E; ++e) u[e] = e < mine ? gc[i0 + e] : 0u;
        if (keff > 0) {
            uint32_t tau, take;
            sel::select_regs<kTopkThreads, E>(t, u, mine, uint32_t(keff), rs, tau, take, bsync);
            sel::compact_regs<kTopkThreads, E>(
                t, u, mine, tau, take, i0, rs, [&](int pos, int i) { out[pos] = gi[i]; }, bsync);
        }
    } else {   // large candidate sets: the generic select straight from memory
        __shared__ sel::MemScratch sc;
        if (keff > 0) {
            uint32_t tau, take;
            auto get = [&](int i) { return __ldg(gc + i); };
            sel::select_mem<kTopkThreads>(t, get, ncand, uint32_t(keff), sc, tau, take, bsync);
            sel::compact_mem<kTopkThreads>(
                t, get, ncand, tau, take, sc, [&](int pos, int i) { out[pos] = gi[i]; }, bsync);
        }
    }
    for (int i = keff + threadIdx.x; i < geo.k; i += blockDim.x) out[i] = -1;
}

struct TopkPlan {
    int nslices, kkp;
    bool wide;   // one CTA with 8 codes per thread (4096 < NS <= 8192)
};
TopkPlan topk_plan(const Geom &geo)
{
    TopkPlan p;
    p.wide = geo.NS > kSlice && geo.NS <= kSliceWide;
    p.nslices = geo.NS <= kSliceWide ? 1 : int((geo.NS + kSlice - 1) / kSlice);
    p.kkp = geo.k < kSlice ? geo.k : kSlice;
    return p;
}

}  // namespace

cudaError_t launch_topk_merge(const Geom &geo, const uint32_t *codes, const int32_t *ids,
                              int32_t *sel, int ncand, cudaStream_t st)
{
    if (geo.k == 0) return cudaSuccess;
    topk_merge_kernel<<<unsigned(geo.B * geo.Hkv), kTopkThreads, 0, st>>>(geo, codes, ids, sel,
                                                                          ncand);
    return cudaGetLastError();
}

int topk_selecting_ctas(const Geom &geo)
{
    return geo.k == 0 ? 0 : geo.B * geo.Hkv * topk_plan(geo).nslices;
}

size_t topk_ws_bytes(const Geom &geo)
{
    const TopkPlan p = topk_plan(geo);
    if (p.nslices <= 1 || geo.k == 0) return 0;
    return size_t(geo.B) * geo.Hkv * p.nslices * p.kkp * (sizeof(uint32_t) + sizeof(int32_t));
}

cudaError_t launch_topk(const Geom &geo, const float *scores, int32_t *sel, void *scratch,
                        uint32_t *zero_words, int nzero, float2 *rope_tab, cudaStream_t st,
                        bool codes)
{
    const int BH = geo.B * geo.Hkv;
    if (geo.k == 0 && nzero == 0 && !rope_tab) return cudaSuccess;
    const TopkPlan p = topk_plan(geo);
    uint32_t *cc = static_cast<uint32_t *>(scratch);
    int32_t *ci = reinterpret_cast<int32_t *>(
        cc + (p.nslices > 1 ? size_t(BH) * p.nslices * p.kkp : 0));
    int64_t tab_rows = 0;
    if (rope_tab) {
        const int64_t chunks = (geo.Wmax + kTabRows - 1) / kTabRows;
        tab_rows = (chunks + p.nslices - 1) / p.nslices;
    }
    dim3 grid(unsigned(p.nslices), unsigned(BH + tab_rows));
    cudaError_t e =
        p.wide ? launch_pdl(topk_slice_kernel<kSliceWide / kTopkThreads>, grid, dim3(kTopkThreads),
                            0, st, geo, scores, sel, cc, ci, p.nslices, p.kkp, zero_words, nzero,
                            rope_tab, codes ? 1 : 0)
               : launch_pdl(topk_slice_kernel<kSlice / kTopkThreads>, grid, dim3(kTopkThreads), 0,
                            st, geo, scores, sel, cc, ci, p.nslices, p.kkp, zero_words, nzero,
                            rope_tab, codes ? 1 : 0);
    if (e != cudaSuccess) return e;
    if (p.nslices > 1 && geo.k > 0) {
        e = launch_pdl(topk_merge_kernel, dim3(BH), dim3(kTopkThreads), 0, st, geo,
                       static_cast<const uint32_t *>(cc), static_cast<const int32_t *>(ci), sel,
                       p.nslices * p.kkp);
        if (e != cudaSuccess) return e;
    }
    return cudaGetLastError();
}

}  // namespace reatt
