// Pieces shared by the windowed-attention kernels: the window map of one
// (batch, KV head), the argument block, the split-K key ranges and merge,
// and the rotated query pairs (ReAttention OpenReview discussion, "Decoding
// Phase" pseudocode: global ++ recalled ++ local, then attention; research-map
// summary "Approach": RoPE after concatenation, window row p at position p,
// query c at W-C+c).
#pragma once

#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace reatt {
namespace {

struct WinMap {
    int64_t g_end, loc_begin, n_loc, nsel_rows, W;
};

__device__ __forceinline__ WinMap make_winmap(const Geom &geo, const int32_t *sel_bh)
{
    WinMap m;
    m.g_end = geo.g_end;
    m.loc_begin = geo.loc_begin;
    m.n_loc = geo.n_loc;
    const int64_t keff = geo.k < geo.NS ? geo.k : geo.NS;
    m.nsel_rows = keff * geo.S;
    if (keff > 0) {
        const int32_t last = sel_bh[keff - 1];
        const int64_t r = geo.M % geo.S;
        if (last == geo.NS - 1 && r != 0) m.nsel_rows -= geo.S - r;
    }
    m.W = m.g_end + m.nsel_rows + m.n_loc + geo.C;
    return m;
}

// Source of window row p: cache row (>= 0) or -(1 + c) for current token c.
// Span ids are clamped into range so a malformed selection stays in bounds.
__device__ __forceinline__ int64_t win_src(const Geom &geo, const WinMap &m, const int32_t *sel_bh,
                                           int64_t p)
{
    if (p < m.g_end) return p;
    p -= m.g_end;
    if (p < m.nsel_rows) {
        const int64_t j = p / geo.S, off = p - j * geo.S;
        int64_t sp = sel_bh[j];
        sp = sp < 0 ? 0 : (sp >= geo.NS ? geo.NS - 1 : sp);
        int64_t row = geo.G + sp * geo.S + off;
        return row < geo.T ? row : geo.T - 1;
    }
    p -= m.nsel_rows;
    if (p < m.n_loc) return m.loc_begin + p;
    return -(1 + (p - m.n_loc));
}

// ---------------------------------------------------------------- attention
__device__ __forceinline__ WinMap attn_winmap(const Geom &geo, const AttnArgs &a, bool virt,
                                              int64_t bh, const int32_t *sel_bh)
{
    if (virt) return make_winmap(geo, sel_bh);
    WinMap m;
    m.g_end = m.loc_begin = m.n_loc = m.nsel_rows = 0;
    const int64_t wl = a.win_len[bh];   // caller data: keep every read inside the window
    m.W = wl < geo.C ? geo.C : (wl > geo.Wmax ? geo.Wmax : wl);
    return m;
}

// Key range of one split (whole multiples of `gran` keys), clipped by the
// causal limit of the block's last query row.
__device__ __forceinline__ void split_range(const Geom &geo, int64_t W, int nsplit, int split,
                                            int r0, int nrows, int gran, int64_t &kbeg,
                                            int64_t &kend)
{
    int64_t chunk = (W + nsplit - 1) / nsplit;
    chunk = (chunk + gran - 1) / gran * gran;
    kbeg = int64_t(split) * chunk;
    kend = kbeg + chunk;
    if (kend > W) kend = W;
    const int last_row = r0 + nrows - 1;
    const int c_max = (last_row / geo.C == r0 / geo.C) ? last_row % geo.C : geo.C - 1;
    const int64_t lim = W - geo.C + c_max + 1;
    if (kend > lim) kend = lim;
}

// End of a CTA's work: its (max, sum, acc) per row sit in shared memory.  With
// one split the output is written directly; otherwise the split's partial
// goes to the workspace and the last CTA of (bh, qb) to finish (atomic ticket,
// no waiting) merges all splits.  `scratch` holds >= 4 * 6 * nrows * D/4
// floats when blockDim.x >= 2 * nrows * D/4 (shared memory of the caller).
template <int D, int QB>
__device__ void split_finish(const Geom &geo, const AttnArgs &a, int64_t bh, int qb, int split,
                             int nrows, const float *s_m, const float *s_l, const float *s_acc,
                             float *scratch, int *is_last)
{
    constexpr int D4 = D / 4;
    const int tid = threadIdx.x, nthr = blockDim.x;
    const int b = int(bh / geo.Hkv), h = int(bh % geo.Hkv), r0 = qb * QB;
    auto out4 = [&](int rr) {
        const int r = r0 + rr, j = h * geo.g + r / geo.C, c = r % geo.C;
        return reinterpret_cast<float4 *>(a.out + ((int64_t(b) * geo.Hq + j) * geo.C + c) * D);
    };
    if (a.nsplit == 1) {
        for (int x = tid; x < nrows * D4; x += nthr) {
            const int rr = x / D4, d4 = x % D4;
            const float il = 1.f / s_l[rr];
            const float4 v = reinterpret_cast<const float4 *>(s_acc)[rr * D4 + d4];
            out4(rr)[d4] = make_float4(v.x * il, v.y * il, v.z * il, v.w * il);
        }
        return;
    }
    const int64_t pbase = (bh * a.nqb + qb) * a.nsplit;
    float4 *pacc = reinterpret_cast<float4 *>(a.part_acc + (pbase + split) * int64_t(QB) * D);
    for (int x = tid; x < nrows * D4; x += nthr)
        pacc[x] = reinterpret_cast<const float4 *>(s_acc)[x];
    for (int rr = tid; rr < nrows; rr += nthr)
        a.part_ml[(pbase + split) * QB + rr] = make_float2(s_m[rr], s_l[rr]);
    // The barrier makes the CTA's partial writes precede thread 0's ticket
    // increment, whose gpu-scope release publishes them (cumulatively); the
    // last CTA's acquire on the same atomic makes every split's partial
    // visible to it.
    __syncthreads();
    if (tid == 0) {
        uint32_t prev;
        asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;"
                     : "=r"(prev)
                     : "l"(&a.ticket[bh * a.nqb + qb])
                     : "memory");
        *is_last = prev == uint32_t(a.nsplit - 1);
    }
    __syncthreads();
    if (!*is_last) return;
    // out = sum_s exp2(m_s - M) acc_s / sum_s exp2(m_s - M) l_s, merged online.
    // With few output elements, G groups of threads take every G-th split of
    // the same element (so all loads are in flight at once) and combine
    // through `scratch` (G * items * 6 floats).
    const int items = nrows * D4;
    int G = nthr / items;
    G = G < 1 ? 1 : (G > 4 ? 4 : G);
    const float2 *ml = a.part_ml + pbase * QB;
    const float4 *all = reinterpret_cast<const float4 *>(a.part_acc + pbase * int64_t(QB) * D);
    auto fold = [&](float &M, float &den, float4 &z, float m, float l, float4 c) {
        if (m == -INFINITY) return;
        const float mn = fmaxf(M, m);
        const float fo = M == -INFINITY ? 0.f : exp2f(M - mn), fn = exp2f(m - mn);
        den = den * fo + fn * l;
        z.x = z.x * fo + fn * c.x;
        z.y = z.y * fo + fn * c.y;
        z.z = z.z * fo + fn * c.z;
        z.w = z.w * fo + fn * c.w;
        M = mn;
    };
    for (int x0 = 0; x0 < items; x0 += nthr / G) {
        const int x = x0 + tid % (nthr / G), g = tid / (nthr / G);
        float M = -INFINITY, den = 0.f;
        float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
        if (x < items && g < G) {
            const int rr = x / D4;
            for (int s0 = g; s0 < a.nsplit; s0 += 8 * G) {
                float2 v[8];
                float4 c[8];
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    if (s0 + u * G < a.nsplit) {
                        v[u] = __ldcg(&ml[(s0 + u * G) * QB + rr]);
                        c[u] = __ldcg(all + int64_t(s0 + u * G) * QB * D4 + x);
                    }
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    if (s0 + u * G < a.nsplit) fold(M, den, z, v[u].x, v[u].y, c[u]);
            }
        }
        if (G > 1) {
            float *sx = scratch + (size_t(g) * items + (x < items ? x : 0)) * 6;
            if (x < items && g < G && g > 0) {
                sx[0] = M;
                sx[1] = den;
                sx[2] = z.x;
                sx[3] = z.y;
                sx[4] = z.z;
                sx[5] = z.w;
            }
            __syncthreads();
            if (x < items && g == 0)
                for (int g2 = 1; g2 < G; ++g2) {
                    const float *o = scratch + (size_t(g2) * items + x) * 6;
                    fold(M, den, z, o[0], o[1], make_float4(o[2], o[3], o[4], o[5]));
                }
            __syncthreads();
        }
        if (x < items && g == 0) {
            const int rr = x / D4;
            const float iden = 1.f / den;
            out4(rr)[x % D4] = make_float4(z.x * iden, z.y * iden, z.z * iden, z.w * iden);
        }
    }
    if (tid == 0) a.ticket[bh * a.nqb + qb] = 0u;   // ready for the next call
}

// Rotated, pre-scaled query element pair (i, i + D/2) of block row rr:
// log2(e)/sqrt(d) folds the softmax scale so logits live in the log2 domain.
template <typename T, int D>
__device__ __forceinline__ void query_pair(const Geom &geo, const float2 *freq, const void *q,
                                           int b, int h, int r, int64_t qpos0, int i, float &lo,
                                           float &hi)
{
    const float qscale = 1.4426950408889634f * rsqrtf(float(D));
    const int j = h * geo.g + r / geo.C, c = r % geo.C;
    const T *qr = static_cast<const T *>(q) + ((int64_t(b) * geo.Hq + j) * geo.C + c) * D;
    const float x0 = Elem<T>::one(qr, i), x1 = Elem<T>::one(qr, i + D / 2);
    float cs, sn;
    rope_cs(qpos0 + c, freq[i].x, freq[i].y, cs, sn);
    lo = (x0 * cs - x1 * sn) * qscale;
    hi = (x1 * cs + x0 * sn) * qscale;
}

}  // namespace
}  // namespace reatt
