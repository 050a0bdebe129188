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
// NS <= kSlice: one CTA per head.  Larger NS: slice CTAs (kSlice scores each)
// emit their own top-k candidates in index order, and one merge CTA per head
// runs the same select on the candidates.  The global top-k under the total
// order (score desc, id asc) is always inside the union of the slices' top-k.
#include "common.cuh"
#include "kernels.h"

namespace reatt {

namespace {

#ifndef REATT_TOPK_THREADS
#define REATT_TOPK_THREADS 512
#endif
constexpr int kTopkThreads = REATT_TOPK_THREADS;
constexpr int kSlice = 4096;

struct SelScratch {
    uint32_t hist[256];
    uint32_t bcast[2];
    int wsum[33];
};

// Exclusive block-wide prefix sum of v; *total receives the block sum.
__device__ __forceinline__ int block_exclusive_sum(int v, int *wsum, int *total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    int inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += t;
    }
    if (lane == 31) wsum[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        const int w = lane < nw ? wsum[lane] : 0;
        int winc = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, winc, o);
            if (lane >= o) winc += t;
        }
        if (lane < nw) wsum[lane] = winc - w;
        if (lane == 31) wsum[32] = winc;
    }
    __syncthreads();
    const int res = wsum[warp] + inc - v;
    *total = wsum[32];
    __syncthreads();
    return res;
}

// Radix select of the kk-th largest code among n (kk >= 1, kk <= number of
// real codes; padding codes are 0 and never reached).  Histogram updates are
// aggregated per warp over lanes that hit the same bin (codes of similar
// scores share their high bytes, so plain atomics would serialise).
template <class Get>
__device__ void radix_select(Get get, int n, uint32_t kk, SelScratch &sc, uint32_t &tau,
                             uint32_t &take_eq)
{
    const int lane = threadIdx.x & 31;
    uint32_t prefix = 0, mask = 0, remaining = kk;
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int i = threadIdx.x; i < 256; i += blockDim.x) sc.hist[i] = 0u;
        __syncthreads();
        for (int base = 0; base < n; base += blockDim.x) {
            const int i = base + threadIdx.x;
            const uint32_t u = i < n ? get(i) : 0u;
            const bool hit = i < n && (u & mask) == prefix;
            const uint32_t bin = (u >> shift) & 255u;
            const unsigned peers = __match_any_sync(0xffffffffu, hit ? bin : 0x100u);
            if (hit && lane == __ffs(peers) - 1) atomicAdd(&sc.hist[bin], __popc(peers));
        }
        __syncthreads();
        if (threadIdx.x < 32) {
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

// ---- register-resident select (n <= kTopkThreads * kMaxE) ----
// Thread t holds codes t*E .. t*E+E-1 (contiguous, so compaction keeps index
// order).  The common high bits of the block's max and min code are skipped,
// and the rest is resolved with 11-bit digits (2048-bin histogram).
constexpr int kMaxE = 16;
constexpr int kBins = 2048;

constexpr int kWarpResolve = 32;   // candidates one warp ranks directly

struct RegScratch {
    uint32_t hist[kBins];
    uint32_t red[2][32];
    int wsum[33];
    uint32_t bcast[3];
    uint32_t cand[kWarpResolve];
    int ncand;
};

__device__ __forceinline__ void block_minmax(uint32_t mx, uint32_t mn, RegScratch &sc,
                                             uint32_t &omax, uint32_t &omin)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
        mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    }
    if (lane == 0) {
        sc.red[0][warp] = mx;
        sc.red[1][warp] = mn;
    }
    __syncthreads();
    mx = lane < nw ? sc.red[0][lane] : 0u;
    mn = lane < nw ? sc.red[1][lane] : 0xffffffffu;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
        mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    }
    omax = mx;
    omin = mn;
    __syncthreads();
}

// kk-th largest among the valid codes (1 <= kk <= valid count).
template <int E>
__device__ void select_regs(const uint32_t (&u)[E], int nvalid_mine, uint32_t kk, RegScratch &sc,
                            uint32_t &tau, uint32_t &take_eq)
{
    uint32_t lmax = 0u, lmin = 0xffffffffu;
#pragma unroll
    for (int e = 0; e < E; ++e)
        if (e < nvalid_mine) {
            lmax = max(lmax, u[e]);
            lmin = min(lmin, u[e]);
        }
    uint32_t gmax, gmin;
    block_minmax(lmax, lmin, sc, gmax, gmin);
    const uint32_t diff = gmax ^ gmin;
    if (diff == 0u) {   // all equal
        tau = gmax;
        take_eq = kk;
        return;
    }
    int hb = 31 - __clz(diff);                       // highest differing bit
    uint32_t mask = hb == 31 ? 0u : ~((2u << hb) - 1u);
    uint32_t prefix = gmax & mask;
    uint32_t remaining = kk;
    const int nt = blockDim.x;
    while (hb >= 0) {
        const int lo = hb >= 10 ? hb - 10 : 0;
        const int nb = hb - lo + 1;
        const uint32_t dmask = (1u << nb) - 1u;
        for (int i = threadIdx.x; i < (1 << nb); i += nt) sc.hist[i] = 0u;
        __syncthreads();
#pragma unroll
        for (int e = 0; e < E; ++e)
            if (e < nvalid_mine && (u[e] & mask) == prefix)
                atomicAdd(&sc.hist[(u[e] >> lo) & dmask], 1u);
        __syncthreads();
        // thread t owns bins in descending order: [(nt-1-t)*per, +per)
        const int per = ((1 << nb) + nt - 1) / nt;
        const int top = (nt - 1 - int(threadIdx.x)) * per;   // lowest bin of this thread
        uint32_t local = 0;
        for (int j = 0; j < per; ++j) {
            const int bin = top + j;
            if (bin < (1 << nb)) local += sc.hist[bin];
        }
        int tot;
        const uint32_t above = uint32_t(block_exclusive_sum(int(local), sc.wsum, &tot));
        if (above < remaining && remaining <= above + local) {
            uint32_t acc = above;
            for (int j = per - 1; j >= 0; --j) {
                const int bin = top + j;
                if (bin >= (1 << nb)) continue;
                const uint32_t c = sc.hist[bin];
                if (acc + c >= remaining) {
                    sc.bcast[0] = uint32_t(bin);
                    sc.bcast[1] = acc;
                    sc.bcast[2] = c;   // codes left with the new prefix
                    sc.ncand = 0;
                    break;
                }
                acc += c;
            }
        }
        __syncthreads();
        remaining -= sc.bcast[1];
        prefix |= sc.bcast[0] << lo;
        mask |= dmask << lo;
        hb = lo - 1;
        const uint32_t left = sc.bcast[2];
        __syncthreads();
        if (hb >= 0 && left <= uint32_t(kWarpResolve)) {
            // Few codes share the prefix: gather them and let one warp rank
            // them (the remaining-th largest is tau).
#pragma unroll
            for (int e = 0; e < E; ++e)
                if (e < nvalid_mine && (u[e] & mask) == prefix)
                    sc.cand[atomicAdd(&sc.ncand, 1)] = u[e];
            __syncthreads();
            if (threadIdx.x < 32) {
                const int lane = threadIdx.x, n = sc.ncand;
                const uint32_t v = lane < n ? sc.cand[lane] : 0u;
                uint32_t gt = 0, eq = 0;
                for (int j = 0; j < n; ++j) {
                    const uint32_t w = __shfl_sync(0xffffffffu, v, j);
                    gt += w > v;
                    eq += w == v;
                }
                if (lane < n && gt < remaining && remaining <= gt + eq) {
                    sc.bcast[0] = v;                 // every such lane writes the same
                    sc.bcast[1] = remaining - gt;
                }
            }
            __syncthreads();
            tau = sc.bcast[0];
            take_eq = sc.bcast[1];
            __syncthreads();
            return;
        }
    }
    tau = prefix;
    take_eq = remaining;
}

template <int E, class Emit>
__device__ void compact_regs(const uint32_t (&u)[E], int nvalid_mine, uint32_t tau,
                             uint32_t take_eq, int i0, RegScratch &sc, Emit emit)
{
    int n_gt = 0, n_eq = 0;
#pragma unroll
    for (int e = 0; e < E; ++e)
        if (e < nvalid_mine) {
            n_gt += u[e] > tau;
            n_eq += u[e] == tau;
        }
    // one scan of both counts (ties in the high half; totals stay below 2^16)
    int tot;
    const int before = block_exclusive_sum((n_eq << 16) | n_gt, sc.wsum, &tot);
    const int eq_before = before >> 16, gt_before = before & 0xffff;
    int take = int(take_eq) - eq_before;
    take = take < 0 ? 0 : (take > n_eq ? n_eq : take);
    int pos = gt_before + (eq_before < int(take_eq) ? eq_before : int(take_eq));
#pragma unroll
    for (int e = 0; e < E; ++e)
        if (e < nvalid_mine) {
            if (u[e] > tau) {
                emit(pos++, i0 + e);
            } else if (u[e] == tau && take > 0) {
                emit(pos++, i0 + e);
                --take;
            }
        }
}

// Stable compaction in index order: every thread owns a contiguous run of
// elements, so two block scans (ties, then chosen) place the output; emit(pos,
// i) is called for every chosen i with pos ascending in i.
template <class Get, class Emit>
__device__ void compact(Get get, int n, uint32_t tau, uint32_t take_eq, SelScratch &sc, Emit emit)
{
    const int per = (n + int(blockDim.x) - 1) / int(blockDim.x);
    const int i0 = int(threadIdx.x) * per;
    const int i1 = i0 + per < n ? i0 + per : n;
    int n_gt = 0, n_eq = 0;
    for (int i = i0; i < i1; ++i) {
        const uint32_t u = get(i);
        n_gt += u > tau;
        n_eq += u == tau;
    }
    int tot;
    const int eq_before = block_exclusive_sum(n_eq, sc.wsum, &tot);
    int take = int(take_eq) - eq_before;
    take = take < 0 ? 0 : (take > n_eq ? n_eq : take);
    int pos = block_exclusive_sum(n_gt + take, sc.wsum, &tot);
    for (int i = i0; i < i1; ++i) {
        const uint32_t u = get(i);
        if (u > tau) {
            emit(pos++, i);
        } else if (u == tau && take > 0) {
            emit(pos++, i);
            --take;
        }
    }
}

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

__global__ void __launch_bounds__(kTopkThreads)
topk_slice_kernel(Geom geo, const float *__restrict__ scores, int32_t *__restrict__ sel,
                  uint32_t *__restrict__ cand_code, int32_t *__restrict__ cand_idx, int nslices,
                  int kkp, uint32_t *zero_words, int nzero, float2 *rope_tab)
{
    __shared__ RegScratch rs;
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

    const int64_t s_begin = int64_t(slice) * kSlice;
    int n = int(geo.NS - s_begin < kSlice ? geo.NS - s_begin : kSlice);
    if (n < 0) n = 0;
    const float *src = scores + bh * geo.NS + s_begin;
    constexpr int E = kSlice / kTopkThreads;
    const int i0 = int(threadIdx.x) * E;
    const int mine = n - i0 < 0 ? 0 : (n - i0 > E ? E : n - i0);
    uint32_t u[E];
#pragma unroll
    for (int e = 0; e < E; ++e) u[e] = e < mine ? order_code(src[i0 + e]) : 0u;
    const int kk = geo.k < n ? geo.k : n;
    if (nslices == 1) {
        int32_t *out = sel + bh * geo.k;
        if (kk > 0) {
            uint32_t tau, take;
            select_regs<E>(u, mine, uint32_t(kk), rs, tau, take);
            compact_regs<E>(u, mine, tau, take, i0, rs, [&](int pos, int i) { out[pos] = int32_t(i); });
        }
        for (int i = kk + threadIdx.x; i < geo.k; i += blockDim.x) out[i] = -1;
    } else {
        uint32_t *oc = cand_code + (bh * nslices + slice) * int64_t(kkp);
        int32_t *oi = cand_idx + (bh * nslices + slice) * int64_t(kkp);
        if (kk > 0) {
            uint32_t tau, take;
            select_regs<E>(u, mine, uint32_t(kk), rs, tau, take);
            compact_regs<E>(u, mine, tau, take, i0, rs, [&](int pos, int i) {
                oc[pos] = order_code(src[i]);
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
    pdl_wait();
    pdl_trigger();
    const int64_t bh = blockIdx.x;
    const uint32_t *gc = cand_code + bh * int64_t(ncand);
    const int32_t *gi = cand_idx + bh * int64_t(ncand);
    const int keff = int(geo.k < geo.NS ? geo.k : geo.NS);
    int32_t *out = sel + bh * geo.k;
    if (ncand <= kTopkThreads * kMaxE) {
        __shared__ RegScratch rs;
        constexpr int E = kMaxE;
        const int per = (ncand + kTopkThreads - 1) / kTopkThreads;
        const int i0 = int(threadIdx.x) * per;
        const int mine = ncand - i0 < 0 ? 0 : (ncand - i0 > per ? per : ncand - i0);
        uint32_t u[E];
#pragma unroll
        for (int e = 0; e < E; ++e) u[e] = e < mine ? gc[i0 + e] : 0u;
        if (keff > 0) {
            uint32_t tau, take;
            select_regs<E>(u, mine, uint32_t(keff), rs, tau, take);
            compact_regs<E>(u, mine, tau, take, i0, rs, [&](int pos, int i) { out[pos] = gi[i]; });
        }
    } else {   // large candidate sets: the generic select straight from memory
        __shared__ SelScratch sc;
        if (keff > 0) {
            uint32_t tau, take;
            auto get = [&](int i) { return __ldg(gc + i); };
            radix_select(get, ncand, uint32_t(keff), sc, tau, take);
            compact(get, ncand, tau, take, sc, [&](int pos, int i) { out[pos] = gi[i]; });
        }
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
                        uint32_t *zero_words, int nzero, float2 *rope_tab, cudaStream_t st)
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
    cudaError_t e = launch_pdl(topk_slice_kernel, grid, dim3(kTopkThreads), 0, st, geo, scores, sel,
                               cc, ci, p.nslices, p.kkp, zero_words, nzero, rope_tab);
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
