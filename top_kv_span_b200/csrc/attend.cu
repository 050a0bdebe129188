// Window construction and windowed attention (ReAttention OpenReview
// discussion, "Decoding Phase" pseudocode: concatenation global ++ recalled
// ++ local, then flash_attention over it; research-map summary "Approach":
// positional embeddings are applied only after the concatenation, so window
// row p is rotated at position p and the query c at W-C+c).
//
// Window of one (batch, KV head), W = g_end + nsel_rows + n_loc + C rows:
//   [0, g_end)                   cache rows 0..g_end-1            (global)
//   next nsel_rows               rows of the chosen spans in sel order; only
//                                the last chosen span can be short (span NS-1)
//   next n_loc                   cache rows loc_begin..T-1        (local)
//   last C                       current tokens 0..C-1
//
// Attention: split-K over the window on CUDA cores in fp32.  A CTA owns one
// (b, h), a block of QB query rows of that head's group (rows ordered head
// then query position), and a contiguous key range.  Keys and values are
// staged through shared memory in tiles of 64 rows (rotated in fp32 on the
// way in when read from the un-rotated cache), softmax is online in the log2
// domain, and the CTAs of one (b, h, query block) combine their partial
// (max, sum, acc) through the workspace: the last CTA to finish (atomic
// ticket, no waiting) merges them and writes the output.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace reatt {

namespace {

constexpr int kAttnThreads = 256;
constexpr int kKT = 64;                 // keys per tile
constexpr int kTargetCtas = 296;        // 2 x 148 SMs: split-K target

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

// ---------------------------------------------------------------- gather + RoPE
constexpr int kGatherRows = 32;

template <typename T, int D>
__global__ void __launch_bounds__(256)
gather_rope_kernel(Geom geo, const T *__restrict__ kc, const T *__restrict__ vc,
                   const T *__restrict__ kcur, const T *__restrict__ vcur,
                   const int32_t *__restrict__ sel, float *__restrict__ kw, float *__restrict__ vw,
                   int32_t *__restrict__ win_len)
{
    constexpr int V = Elem<T>::kVec, HV = D / 2 / V;   // vectors per half row
    __shared__ double ifreq[D / 2];
    const int64_t bh = blockIdx.y;
    const int32_t *sel_bh = sel + bh * geo.k;
    const WinMap m = make_winmap(geo, sel_bh);
    for (int i = threadIdx.x; i < D / 2; i += blockDim.x)
        ifreq[i] = rope_inv_freq_over_pi(i, D, geo.base);
    if (blockIdx.x == 0 && threadIdx.x == 0) win_len[bh] = int32_t(m.W);
    __syncthreads();

    const int64_t row0 = int64_t(blockIdx.x) * kGatherRows;
    for (int x = threadIdx.x; x < kGatherRows * HV; x += blockDim.x) {
        const int64_t p = row0 + x / HV;
        const int v = x % HV;
        if (p >= m.W) continue;
        const int64_t s = win_src(geo, m, sel_bh, p);
        const T *kr, *vr;
        if (s >= 0) {
            kr = kc + (bh * geo.T + s) * D;
            vr = vc + (bh * geo.T + s) * D;
        } else {
            kr = kcur + (bh * geo.C + (-s - 1)) * D;
            vr = vcur + (bh * geo.C + (-s - 1)) * D;
        }
        float klo[V], khi[V], vlo[V], vhi[V];
        Elem<T>::unpack(*reinterpret_cast<const uint4 *>(kr + v * V), klo);
        Elem<T>::unpack(*reinterpret_cast<const uint4 *>(kr + D / 2 + v * V), khi);
        Elem<T>::unpack(*reinterpret_cast<const uint4 *>(vr + v * V), vlo);
        Elem<T>::unpack(*reinterpret_cast<const uint4 *>(vr + D / 2 + v * V), vhi);
        float *ko = kw + (bh * geo.Wmax + p) * D;
        float *vo = vw + (bh * geo.Wmax + p) * D;
#pragma unroll
        for (int e = 0; e < V; ++e) {
            const int i = v * V + e;
            float c, sn;
            rope_cs(p, ifreq[i], c, sn);
            ko[i] = klo[e] * c - khi[e] * sn;
            ko[i + D / 2] = khi[e] * c + klo[e] * sn;
            vo[i] = vlo[e];
            vo[i + D / 2] = vhi[e];
        }
    }
}

// ---------------------------------------------------------------- attention
template <int D, int QB>
struct AttnSmem {
    static constexpr size_t kQ = size_t(QB) * D * 4;
    static constexpr size_t kK = size_t(kKT) * (D + 1) * 4;
    static constexpr size_t kV = size_t(kKT) * D * 4;
    static constexpr size_t kP = size_t(QB) * kKT * 4;
    static constexpr size_t kRow = size_t(QB) * 4 * 3;   // m, l, corr
    static constexpr size_t kF = size_t(D / 2) * 8;
    static constexpr size_t kTotal = kQ + kK + kV + kP + kRow + kF + 64;
};

// Key/value row source for the two attention variants.
template <typename T, int D, bool VIRT>
struct KvSource;

// Virtual window: rows straight from the un-rotated cache / current tokens.
template <typename T, int D>
struct KvSource<T, D, true> {
    const T *kc, *vc, *kcur, *vcur;
    const int32_t *sel;
    static constexpr int V = Elem<T>::kVec;
    __device__ __forceinline__ void load(const Geom &geo, const WinMap &m, int64_t bh,
                                         const int32_t *sel_bh, int64_t p, int v,
                                         const double *ifreq, float (&klo)[V], float (&khi)[V],
                                         float (&vlo)[V], float (&vhi)[V]) const
    {
        const int64_t s = win_src(geo, m, sel_bh, p);
        const T *kr, *vr;
        if (s >= 0) {
            kr = kc + (bh * geo.T + s) * D;
            vr = vc + (bh * geo.T + s) * D;
        } else {
            kr = kcur + (bh * geo.C + (-s - 1)) * D;
            vr = vcur + (bh * geo.C + (-s - 1)) * D;
        }
        float a[V], b[V];
        Elem<T>::unpack(ldg_stream(kr + v * V), a);
        Elem<T>::unpack(ldg_stream(kr + D / 2 + v * V), b);
        Elem<T>::unpack(ldg_stream(vr + v * V), vlo);
        Elem<T>::unpack(ldg_stream(vr + D / 2 + v * V), vhi);
#pragma unroll
        for (int e = 0; e < V; ++e) {
            float c, sn;
            rope_cs(p, ifreq[v * V + e], c, sn);
            klo[e] = a[e] * c - b[e] * sn;
            khi[e] = b[e] * c + a[e] * sn;
        }
    }
};

// Materialised fp32 window (already rotated by gather_rope).
template <typename T, int D>
struct KvSource<T, D, false> {
    const float *kw, *vw;
    static constexpr int V = 4;
    __device__ __forceinline__ void load(const Geom &geo, const WinMap &, int64_t bh,
                                         const int32_t *, int64_t p, int v, const double *,
                                         float (&klo)[V], float (&khi)[V], float (&vlo)[V],
                                         float (&vhi)[V]) const
    {
        const float *kr = kw + (bh * geo.Wmax + p) * D;
        const float *vr = vw + (bh * geo.Wmax + p) * D;
        Elem<float>::unpack(ldg_stream(kr + v * V), klo);
        Elem<float>::unpack(ldg_stream(kr + D / 2 + v * V), khi);
        Elem<float>::unpack(ldg_stream(vr + v * V), vlo);
        Elem<float>::unpack(ldg_stream(vr + D / 2 + v * V), vhi);
    }
};

struct AttnArgs {
    const void *q;
    const int32_t *sel;       // virtual window
    const int32_t *win_len;   // materialised window
    float *out;
    float *part;              // [BH][nqb][nsplit][QB][D+2]
    uint32_t *ticket;         // [BH][nqb]
    int nqb, nsplit;
};

template <typename T, int D, int QB, bool VIRT>
__global__ void __launch_bounds__(kAttnThreads)
attend_kernel(Geom geo, AttnArgs a, KvSource<T, D, VIRT> src)
{
    using Sm = AttnSmem<D, QB>;
    constexpr int V = KvSource<T, D, VIRT>::V;
    constexpr int HV = D / 2 / V;
    constexpr int NACC = QB * D / kAttnThreads;
    constexpr int NLOG = QB * kKT / kAttnThreads;
    static_assert(NACC >= 1 && NLOG >= 1, "tile shape");
    extern __shared__ __align__(16) uint8_t smem[];
    float *Qs = reinterpret_cast<float *>(smem);
    float *Ks = reinterpret_cast<float *>(smem + Sm::kQ);
    float *Vs = reinterpret_cast<float *>(smem + Sm::kQ + Sm::kK);
    float *Ps = reinterpret_cast<float *>(smem + Sm::kQ + Sm::kK + Sm::kV);
    float *m_run = reinterpret_cast<float *>(smem + Sm::kQ + Sm::kK + Sm::kV + Sm::kP);
    float *l_run = m_run + QB;
    float *corr = l_run + QB;
    double *ifreq = reinterpret_cast<double *>(smem + Sm::kQ + Sm::kK + Sm::kV + Sm::kP + Sm::kRow);
    __shared__ int is_last;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int split = blockIdx.x, qb = blockIdx.y;
    const int64_t bh = blockIdx.z;
    const int b = int(bh / geo.Hkv), h = int(bh % geo.Hkv);
    const int R = geo.g * geo.C;
    const int r0 = qb * QB;
    const int nrows = R - r0 < QB ? R - r0 : QB;

    const int32_t *sel_bh = VIRT ? a.sel + bh * geo.k : nullptr;
    WinMap m;
    if (VIRT) {
        m = make_winmap(geo, sel_bh);
    } else {
        m.g_end = m.loc_begin = m.n_loc = m.nsel_rows = 0;
        int64_t wl = a.win_len[bh];   // caller data: keep every read inside the window
        m.W = wl < geo.C ? geo.C : (wl > geo.Wmax ? geo.Wmax : wl);
    }
    const int64_t W = m.W;
    const int64_t qpos0 = W - geo.C;                    // position of query c = 0

    for (int i = tid; i < D / 2; i += kAttnThreads)
        ifreq[i] = rope_inv_freq_over_pi(i, D, geo.base);
    for (int r = tid; r < QB; r += kAttnThreads) {
        m_run[r] = -INFINITY;
        l_run[r] = 0.f;
    }
    __syncthreads();

    // rotated, pre-scaled queries: log2(e)/sqrt(d) folds the softmax scale
    const float qscale = 1.4426950408889634f / sqrtf(float(D));
    for (int x = tid; x < QB * (D / 2); x += kAttnThreads) {
        const int rr = x / (D / 2), i = x % (D / 2);
        float lo = 0.f, hi = 0.f;
        if (rr < nrows) {
            const int r = r0 + rr, j = h * geo.g + r / geo.C, c = r % geo.C;
            const T *qr = static_cast<const T *>(a.q) + ((int64_t(b) * geo.Hq + j) * geo.C + c) * D;
            const float x0 = Elem<T>::one(qr, i), x1 = Elem<T>::one(qr, i + D / 2);
            float cs, sn;
            rope_cs(qpos0 + c, ifreq[i], cs, sn);
            lo = (x0 * cs - x1 * sn) * qscale;
            hi = (x1 * cs + x0 * sn) * qscale;
        }
        Qs[rr * D + i] = lo;
        Qs[rr * D + i + D / 2] = hi;
    }

    // key range of this split (multiple of the tile), clipped by causality
    int64_t chunk = (W + a.nsplit - 1) / a.nsplit;
    chunk = (chunk + kKT - 1) / kKT * kKT;
    const int64_t kbeg = int64_t(split) * chunk;
    int64_t kend = kbeg + chunk;
    if (kend > W) kend = W;
    const int last_row = r0 + nrows - 1;
    const int c_max = (last_row / geo.C == r0 / geo.C) ? last_row % geo.C : geo.C - 1;
    if (kend > qpos0 + c_max + 1) kend = qpos0 + c_max + 1;

    float acc[NACC];
#pragma unroll
    for (int u = 0; u < NACC; ++u) acc[u] = 0.f;

    for (int64_t t0 = kbeg; t0 < kend; t0 += kKT) {
        const int nk = int(kend - t0 < kKT ? kend - t0 : kKT);
        __syncthreads();
        for (int x = tid; x < kKT * HV; x += kAttnThreads) {
            const int key = x / HV, v = x % HV;
            float klo[V], khi[V], vlo[V], vhi[V];
            if (key < nk) {
                src.load(geo, m, bh, sel_bh, t0 + key, v, ifreq, klo, khi, vlo, vhi);
            } else {
#pragma unroll
                for (int e = 0; e < V; ++e) klo[e] = khi[e] = vlo[e] = vhi[e] = 0.f;
            }
#pragma unroll
            for (int e = 0; e < V; ++e) {
                const int i = v * V + e;
                Ks[key * (D + 1) + i] = klo[e];
                Ks[key * (D + 1) + i + D / 2] = khi[e];
                Vs[key * D + i] = vlo[e];
                Vs[key * D + i + D / 2] = vhi[e];
            }
        }
        __syncthreads();
        // logits (log2 domain), causal mask per row
#pragma unroll
        for (int u = 0; u < NLOG; ++u) {
            const int x = tid + u * kAttnThreads;
            const int rr = x / kKT, key = x % kKT;
            float s = -INFINITY;
            if (rr < nrows && key < nk) {
                const int c = (r0 + rr) % geo.C;
                if (t0 + key <= qpos0 + c) {
                    const float *qv = Qs + rr * D, *kv = Ks + key * (D + 1);
                    float z = 0.f;
#pragma unroll 16
                    for (int i = 0; i < D; ++i) z = fmaf(qv[i], kv[i], z);
                    s = z;
                }
            }
            Ps[rr * kKT + key] = s;
        }
        __syncthreads();
        // online softmax, one warp per row
        for (int rr = warp; rr < nrows; rr += kAttnThreads / 32) {
            float v0 = Ps[rr * kKT + lane], v1 = Ps[rr * kKT + lane + 32];
            float mx = fmaxf(v0, v1);
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            const float m_old = m_run[rr];
            const float m_new = fmaxf(m_old, mx);
            float cf, p0, p1;
            if (m_new == -INFINITY) {
                cf = 1.f;
                p0 = p1 = 0.f;
            } else {
                cf = exp2f(m_old - m_new);
                p0 = exp2f(v0 - m_new);
                p1 = exp2f(v1 - m_new);
            }
            Ps[rr * kKT + lane] = p0;
            Ps[rr * kKT + lane + 32] = p1;
            float sum = p0 + p1;
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
            __syncwarp();
            if (lane == 0) {
                m_run[rr] = m_new;
                l_run[rr] = l_run[rr] * cf + sum;
                corr[rr] = cf;
            }
        }
        __syncthreads();
        // acc = acc * corr + P V
#pragma unroll
        for (int u = 0; u < NACC; ++u) {
            const int x = tid + u * kAttnThreads;
            const int rr = x / D, i = x % D;
            if (rr < nrows) {
                float z = acc[u] * corr[rr];
                const float *pr = Ps + rr * kKT;
#pragma unroll 8
                for (int key = 0; key < nk; ++key) z = fmaf(pr[key], Vs[key * D + i], z);
                acc[u] = z;
            }
        }
    }
    __syncthreads();

    if (a.nsplit == 1) {
#pragma unroll
        for (int u = 0; u < NACC; ++u) {
            const int x = tid + u * kAttnThreads;
            const int rr = x / D, i = x % D;
            if (rr < nrows) {
                const int r = r0 + rr, j = h * geo.g + r / geo.C, c = r % geo.C;
                a.out[((int64_t(b) * geo.Hq + j) * geo.C + c) * D + i] = acc[u] / l_run[rr];
            }
        }
        return;
    }

    // partials of this split, then the last CTA of (bh, qb) combines
    const int64_t pbase = (bh * a.nqb + qb) * a.nsplit;
    float *mine = a.part + (pbase + split) * int64_t(QB) * (D + 2);
#pragma unroll
    for (int u = 0; u < NACC; ++u) {
        const int x = tid + u * kAttnThreads;
        const int rr = x / D, i = x % D;
        if (rr < nrows) mine[rr * (D + 2) + 2 + i] = acc[u];
    }
    for (int rr = tid; rr < nrows; rr += kAttnThreads) {
        mine[rr * (D + 2)] = m_run[rr];
        mine[rr * (D + 2) + 1] = l_run[rr];
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) {
        const uint32_t prev = atomicAdd(&a.ticket[bh * a.nqb + qb], 1u);
        is_last = prev == uint32_t(a.nsplit - 1);
    }
    __syncthreads();
    if (!is_last) return;
    __threadfence();
    const float *all = a.part + pbase * int64_t(QB) * (D + 2);
    for (int x = tid; x < nrows * D; x += kAttnThreads) {
        const int rr = x / D, i = x % D;
        float mx = -INFINITY;
        for (int s = 0; s < a.nsplit; ++s)
            mx = fmaxf(mx, __ldcg(all + (int64_t(s) * QB + rr) * (D + 2)));
        float den = 0.f, num = 0.f;
        for (int s = 0; s < a.nsplit; ++s) {
            const float *ps = all + (int64_t(s) * QB + rr) * (D + 2);
            const float ms = __ldcg(ps);
            if (ms == -INFINITY) continue;
            const float w = exp2f(ms - mx);
            den += w * __ldcg(ps + 1);
            num += w * __ldcg(ps + 2 + i);
        }
        const int r = r0 + rr, j = h * geo.g + r / geo.C, c = r % geo.C;
        a.out[((int64_t(b) * geo.Hq + j) * geo.C + c) * D + i] = num / den;
    }
    if (tid == 0) a.ticket[bh * a.nqb + qb] = 0u;   // ready for the next call
}

template <typename T, int D, int QB, bool VIRT>
cudaError_t launch_attn(const Geom &geo, const AttnArgs &a, const KvSource<T, D, VIRT> &src,
                        cudaStream_t st)
{
    using Sm = AttnSmem<D, QB>;
    auto kern = attend_kernel<T, D, QB, VIRT>;
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(Sm::kTotal));
    if (e != cudaSuccess) return e;
    dim3 grid(unsigned(a.nsplit), unsigned(a.nqb), unsigned(geo.B * geo.Hkv));
    kern<<<grid, kAttnThreads, Sm::kTotal, st>>>(geo, a, src);
    return cudaGetLastError();
}

template <typename T, int D, bool VIRT>
cudaError_t dispatch_qb(const Geom &geo, const AttnArgs &a, const KvSource<T, D, VIRT> &src,
                        int QB, cudaStream_t st)
{
    if (QB == 8) return launch_attn<T, D, 8, VIRT>(geo, a, src, st);
    return launch_attn<T, D, 64, VIRT>(geo, a, src, st);
}

}  // namespace

AttnPlan attn_plan(const Geom &geo)
{
    AttnPlan p;
    const int64_t R = int64_t(geo.g) * geo.C;
    p.QB = R <= 8 ? 8 : 64;
    p.nqb = int((R + p.QB - 1) / p.QB);
    const int64_t base = int64_t(geo.B) * geo.Hkv * p.nqb;
    const int64_t max_split = (geo.Wmax + kKT - 1) / kKT;
    int64_t ns = 1;
    if (base < kTargetCtas) ns = (kTargetCtas + base - 1) / base;
    if (ns > max_split) ns = max_split;
    if (ns < 1) ns = 1;
    p.nsplit = int(ns);
    return p;
}

size_t attend_ws_bytes(const Geom &geo, size_t *ticket_bytes)
{
    const AttnPlan p = attn_plan(geo);
    const size_t nt = size_t(geo.B) * geo.Hkv * p.nqb;
    *ticket_bytes = (nt * sizeof(uint32_t) + 255) / 256 * 256;
    if (p.nsplit == 1) return *ticket_bytes;
    return *ticket_bytes + nt * p.nsplit * p.QB * (geo.d + 2) * sizeof(float);
}

cudaError_t launch_gather_rope(const Geom &geo, const void *kc, const void *vc, const void *kcur,
                               const void *vcur, const int32_t *sel, float *kw, float *vw,
                               int32_t *win_len, cudaStream_t st)
{
    dim3 grid(unsigned((geo.Wmax + kGatherRows - 1) / kGatherRows), unsigned(geo.B * geo.Hkv));
#define REATT_GATHER(T, D)                                                                     \
    gather_rope_kernel<T, D><<<grid, 256, 0, st>>>(                                            \
        geo, static_cast<const T *>(kc), static_cast<const T *>(vc),                          \
        static_cast<const T *>(kcur), static_cast<const T *>(vcur), sel, kw, vw, win_len)
    if (geo_is_bf16(geo)) {
        if (geo.d == 128) REATT_GATHER(uint16_t, 128);
        else REATT_GATHER(uint16_t, 64);
    } else {
        if (geo.d == 128) REATT_GATHER(float, 128);
        else REATT_GATHER(float, 64);
    }
#undef REATT_GATHER
    return cudaGetLastError();
}

cudaError_t launch_attend(const Geom &geo, const void *q, const float *kw, const float *vw,
                          const int32_t *win_len, const void *kc, const void *vc,
                          const void *kcur, const void *vcur, const int32_t *sel, float *out,
                          void *scratch, bool virt, cudaStream_t st)
{
    const AttnPlan p = attn_plan(geo);
    size_t tb = 0;
    attend_ws_bytes(geo, &tb);
    AttnArgs a;
    a.q = q;
    a.sel = sel;
    a.win_len = win_len;
    a.out = out;
    a.ticket = static_cast<uint32_t *>(scratch);
    a.part = reinterpret_cast<float *>(static_cast<uint8_t *>(scratch) + tb);
    a.nqb = p.nqb;
    a.nsplit = p.nsplit;
#define REATT_ATT(T, D)                                                                        \
    do {                                                                                       \
        if (virt) {                                                                            \
            KvSource<T, D, true> s{static_cast<const T *>(kc), static_cast<const T *>(vc),     \
                                   static_cast<const T *>(kcur), static_cast<const T *>(vcur), \
                                   sel};                                                       \
            return dispatch_qb<T, D, true>(geo, a, s, p.QB, st);                               \
        }                                                                                      \
        KvSource<T, D, false> s{kw, vw};                                                       \
        return dispatch_qb<T, D, false>(geo, a, s, p.QB, st);                                  \
    } while (0)
    if (geo_is_bf16(geo)) {
        if (geo.d == 128) REATT_ATT(uint16_t, 128);
        REATT_ATT(uint16_t, 64);
    }
    if (geo.d == 128) REATT_ATT(float, 128);
    REATT_ATT(float, 64);
#undef REATT_ATT
}

}  // namespace reatt
