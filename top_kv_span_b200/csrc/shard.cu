// One sequence's cache split by token ranges over several GPUs ("shards"):
// per-shard span scoring and top-k candidates, the global selection from
// every shard's candidates, per-shard partial attention over the window rows
// the shard holds, and the log-sum-exp merge of the partials.
//
// The research-map summary ("Limitations") and the OpenReview discussion
// (reply on W4, "memory overhead tradeoff": 400K tokens on one GPU) name
// memory as the method's bound, so one sequence's cache may have to live on
// several GPUs.  The selection and the attention both decompose over token
// ranges:
//   * the global top-k under the order (score desc, id asc) is contained in
//     the union of every shard's own top-k under the same order;
//   * softmax attention over a union of disjoint key sets is the log-sum-exp
//     merge of the per-set partials (max m, sum l, unnormalised acc).
// Window positions stay those of the whole window (global ++ chosen ++ local
// ++ current), so every shard needs the full selection (phase 2) before it
// attends (decoding pseudocode of the OpenReview discussion; research-map
// summary "Approach": RoPE after the concatenation).
#include <math.h>

#include "attend_common.cuh"
#include "common.cuh"
#include "kernels.h"

namespace reatt {

namespace {

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t up256(size_t x) { return (x + 255) / 256 * 256; }
inline int cuda_status(cudaError_t e) { return e == cudaSuccess ? REATT_OK : REATT_ECUDA; }

// Rows of one shard and the middle spans it holds.
struct ShardGeom {
    Geom sub;            // the shard's spans as a geometry of their own (scan / top-k)
    int64_t t_begin, t_end, rows;
    int64_t s_lo, s_hi;  // whole-sequence span ids [s_lo, s_hi)
    int owns_current;
};

// Token t lies on an allowed shard boundary: outside the middle, or on a
// span boundary inside it.
inline bool boundary_ok(const Geom &g, int64_t t)
{
    if (t <= g.G || t >= g.G + g.M) return true;
    return (t - g.G) % g.S == 0;
}

// First span whose tokens start at or after token t (t on an allowed boundary).
inline int64_t span_at(const Geom &g, int64_t t)
{
    if (t <= g.G) return 0;
    if (t >= g.G + g.M) return g.NS;
    return (t - g.G) / g.S;
}

int make_shard(const Geom &g, const reatt_shard *sh, ShardGeom *sg)
{
    if (!sh) return REATT_EINVAL;
    if (sh->t_begin < 0 || sh->t_end < sh->t_begin || sh->t_end > g.T) return REATT_EINVAL;
    if (sh->owns_current != 0 && sh->owns_current != 1) return REATT_EINVAL;
    if (sh->reserved != 0) return REATT_EINVAL;
    const int64_t n = sh->t_end - sh->t_begin;
    const int64_t cap = sh->rows_cap ? sh->rows_cap : n;
    if (cap < n || cap >= (int64_t(1) << 31)) return REATT_EINVAL;
    if (!boundary_ok(g, sh->t_begin) || !boundary_ok(g, sh->t_end)) return REATT_EINVAL;
    sg->t_begin = sh->t_begin;
    sg->t_end = sh->t_end;
    sg->rows = cap;
    sg->owns_current = sh->owns_current;
    sg->s_lo = span_at(g, sh->t_begin);
    sg->s_hi = span_at(g, sh->t_end);
    if (sg->s_hi < sg->s_lo) sg->s_hi = sg->s_lo;
    Geom s = g;
    s.G = int(g.G + sg->s_lo * g.S);   // token of the shard's first span
    s.NS = sg->s_hi - sg->s_lo;
    const int64_t m_end = g.M < sg->s_hi * g.S ? g.M : sg->s_hi * g.S;
    s.M = s.NS > 0 ? m_end - sg->s_lo * g.S : 0;
    s.Ts = cap;
    sg->sub = s;
    return REATT_OK;
}

// Base pointer of a shard's cache as if it held rows from token 0: row t of
// (b, h) sits at base + ((b*Hkv + h)*rows + t)*d for t in [t_begin, t_end).
// Only addresses of held rows are ever formed from it on the device.
inline const void *shifted(const void *p, int64_t t_begin, int d, int elem)
{
    return reinterpret_cast<const void *>(reinterpret_cast<uintptr_t>(p) -
                                          uintptr_t(t_begin) * uintptr_t(d) * uintptr_t(elem));
}

// ---------------------------------------------------------------- phase 1
__global__ void shard_cands_kernel(int64_t NS_sub, int k, int64_t s_lo,
                                   const float *__restrict__ scores,
                                   const int32_t *__restrict__ sel_local,
                                   float *__restrict__ cand_score, int32_t *__restrict__ cand_id)
{
    const int64_t bh = blockIdx.x;
    for (int i = threadIdx.x; i < k; i += blockDim.x) {
        const int32_t s = NS_sub > 0 ? sel_local[bh * k + i] : -1;
        cand_id[bh * k + i] = s >= 0 ? int32_t(s + s_lo) : -1;
        cand_score[bh * k + i] = s >= 0 ? scores[bh * NS_sub + s] : -INFINITY;
    }
}

// ---------------------------------------------------------------- phase 2
// [n][BH][k] (score, id) -> per bh: order codes and ids of all n*k
// candidates, shard-major (so index order is ascending span id); empty
// entries get code 0, below every real score.
__global__ void shard_codes_kernel(int n, int64_t BH, int k, const float *__restrict__ score,
                                   const int32_t *__restrict__ id, uint32_t *__restrict__ code,
                                   int32_t *__restrict__ idx)
{
    const int64_t total = int64_t(n) * BH * k;
    for (int64_t x = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; x < total;
         x += int64_t(gridDim.x) * blockDim.x) {
        const int64_t i = x % k, bh = (x / k) % BH, r = x / (int64_t(k) * BH);
        const int32_t s = id[x];
        const int64_t dst = bh * (int64_t(n) * k) + r * k + i;
        code[dst] = s >= 0 ? order_code(score[x]) : 0u;
        idx[dst] = s;
    }
}

// ---------------------------------------------------------------- phase 3
constexpr int kShWarps = 8;
constexpr int kShQB = 8;          // query rows per CTA
constexpr int kShKI = 4;          // keys in flight per warp
constexpr int kShTargetCtas = 296;

struct ShardRuns {
    int64_t n[4];     // rows held: global, chosen, local, current
    int64_t pos0[4];  // window position of the first row of each part
    int64_t src0[4];  // first source row: token (global, local), chosen-row index, current token
    int64_t W;        // whole window length
};

// The window rows this shard holds, per part (computed by one thread).
__device__ ShardRuns shard_runs(const Geom &g, const int32_t *sel_bh, int64_t t_begin,
                                int64_t t_end, int64_t s_lo, int64_t s_hi, int owns_current)
{
    const WinMap m = make_winmap(g, sel_bh);
    ShardRuns r;
    r.W = m.W;
    // global rows [0, g_end): positions equal tokens
    {
        const int64_t a = t_begin, b = t_end < m.g_end ? t_end : m.g_end;
        r.n[0] = b > a ? b - a : 0;
        r.pos0[0] = a;
        r.src0[0] = a;
    }
    // chosen spans: sel is ascending, so the shard's spans are a run of it
    {
        const int64_t keff = g.k < g.NS ? g.k : g.NS;
        int64_t jl = 0, jh = 0;
        while (jl < keff && sel_bh[jl] < s_lo) ++jl;
        jh = jl;
        while (jh < keff && sel_bh[jh] < s_hi) ++jh;
        int64_t r1 = jh * g.S;
        if (r1 > m.nsel_rows) r1 = m.nsel_rows;
        const int64_t r0 = jl * g.S;
        r.n[1] = r1 > r0 ? r1 - r0 : 0;
        r.pos0[1] = m.g_end + r0;
        r.src0[1] = r0;
    }
    // local rows [loc_begin, T)
    {
        const int64_t lb = m.loc_begin > t_begin ? m.loc_begin : t_begin;
        const int64_t le = t_end;
        const bool any = m.n_loc > 0 && le > lb;
        r.n[2] = any ? le - lb : 0;
        r.pos0[2] = m.g_end + m.nsel_rows + (lb - m.loc_begin);
        r.src0[2] = lb;
    }
    r.n[3] = owns_current ? g.C : 0;
    r.pos0[3] = m.W - g.C;
    r.src0[3] = 0;
    return r;
}

template <typename T, int D>
__global__ void __launch_bounds__(kShWarps * 32)
shard_attend_kernel(Geom g, int64_t t_begin, int64_t t_end, int64_t rows, int64_t s_lo,
                    int64_t s_hi, int owns_current, const T *__restrict__ q,
                    const T *__restrict__ kc, const T *__restrict__ vc,
                    const T *__restrict__ kcur, const T *__restrict__ vcur,
                    const int32_t *__restrict__ sel, int nsplit, int nqb,
                    float *__restrict__ part_acc, float2 *__restrict__ part_ml,
                    uint32_t *__restrict__ ticket, float2 *__restrict__ out_ml,
                    float *__restrict__ out_acc)
{
    constexpr int E = D / 32;           // elements per lane: dims lane + 32e
    constexpr int HE = E / 2;           // pairs per lane: (e, e + HE)
    __shared__ ShardRuns runs;
    __shared__ float s_m[kShWarps][kShQB], s_l[kShWarps][kShQB];
    __shared__ float s_acc[kShWarps][kShQB][D];
    __shared__ int is_last;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int split = blockIdx.x, qb = blockIdx.y;
    const int64_t bh = blockIdx.z;
    const int b = int(bh / g.Hkv), h = int(bh % g.Hkv);
    const int32_t *sel_bh = sel + bh * g.k;
    if (tid == 0) runs = shard_runs(g, sel_bh, t_begin, t_end, s_lo, s_hi, owns_current);
    __syncthreads();
    const int nrows_all = g.g * g.C;
    const int r0 = qb * kShQB;
    const int nrows = nrows_all - r0 < kShQB ? nrows_all - r0 : kShQB;
    const int64_t n_own = runs.n[0] + runs.n[1] + runs.n[2] + runs.n[3];
    const int64_t chunk = (n_own + nsplit - 1) / nsplit;
    const int64_t kb = int64_t(split) * chunk;
    const int64_t ke = kb + chunk < n_own ? kb + chunk : n_own;

    // rotated, pre-scaled query rows (log2 domain)
    const float qscale = 1.4426950408889634f * rsqrtf(float(D));
    float qv[kShQB][E];
    int climit[kShQB];
#pragma unroll
    for (int r = 0; r < kShQB; ++r) {
        climit[r] = -1;
#pragma unroll
        for (int e = 0; e < E; ++e) qv[r][e] = 0.f;
        if (r < nrows) {
            const int row = r0 + r, j = h * g.g + row / g.C, c = row % g.C;
            const T *qr = q + ((int64_t(b) * g.Hq + j) * g.C + c) * D;
            const int64_t qpos = runs.W - g.C + c;
            climit[r] = int(qpos);
#pragma unroll
            for (int e = 0; e < HE; ++e) {
                const int i = lane + 32 * e;
                const float x0 = Elem<T>::one(qr, i), x1 = Elem<T>::one(qr, i + D / 2);
                float cs, sn;
                rope_cs(qpos, g.rope_hi[i], g.rope_lo[i], cs, sn);
                qv[r][e] = (x0 * cs - x1 * sn) * qscale;
                qv[r][e + HE] = (x1 * cs + x0 * sn) * qscale;
            }
        }
    }
    float m[kShQB], l[kShQB], acc[kShQB][E];
#pragma unroll
    for (int r = 0; r < kShQB; ++r) {
        m[r] = -INFINITY;
        l[r] = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) acc[r][e] = 0.f;
    }
    // key x of the held rows -> (window position, K row, V row)
    auto locate = [&](int64_t x, int64_t &pos, const T *&kr, const T *&vr) {
        int part = 0;
        while (part < 3 && x >= runs.n[part]) {
            x -= runs.n[part];
            ++part;
        }
        pos = runs.pos0[part] + x;
        if (part == 3) {
            kr = kcur + (bh * g.C + x) * D;
            vr = vcur + (bh * g.C + x) * D;
            return;
        }
        int64_t tok;
        if (part == 1) {
            const int64_t cr = runs.src0[1] + x;   // row among the chosen rows
            const int64_t jj = cr / g.S, off = cr - jj * g.S;
            int64_t sp = sel_bh[jj];   // inside [s_lo, s_hi) for a well-formed selection;
            sp = sp < s_lo ? s_lo : (sp >= s_hi ? s_hi - 1 : sp);   // clamped: reads stay in the shard
            tok = g.G + sp * g.S + off;
            if (tok >= t_end) tok = t_end - 1;
        } else {
            tok = runs.src0[part] + x;
        }
        kr = kc + (bh * rows + tok) * D;   // kc, vc are shifted so token indices address them
        vr = vc + (bh * rows + tok) * D;
    };

    for (int64_t x0 = kb + int64_t(warp) * kShKI; x0 < ke; x0 += int64_t(kShWarps) * kShKI) {
        float kx[kShKI][E], vx[kShKI][E];
        int64_t pos[kShKI];
#pragma unroll
        for (int u = 0; u < kShKI; ++u) {
            pos[u] = -1;
            if (x0 + u < ke) {
                const T *kr, *vr;
                locate(x0 + u, pos[u], kr, vr);
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    kx[u][e] = Elem<T>::one(kr, lane + 32 * e);
                    vx[u][e] = Elem<T>::one(vr, lane + 32 * e);
                }
            }
        }
#pragma unroll
        for (int u = 0; u < kShKI; ++u) {
            if (pos[u] < 0) continue;   // warp-uniform
            // rotate the key at its window position
#pragma unroll
            for (int e = 0; e < HE; ++e) {
                const int i = lane + 32 * e;
                float cs, sn;
                rope_cs(pos[u], g.rope_hi[i], g.rope_lo[i], cs, sn);
                const float x0v = kx[u][e], x1v = kx[u][e + HE];
                kx[u][e] = x0v * cs - x1v * sn;
                kx[u][e + HE] = x1v * cs + x0v * sn;
            }
#pragma unroll
            for (int r = 0; r < kShQB; ++r) {
                if (r >= nrows || pos[u] > climit[r]) continue;   // warp-uniform
                float s = 0.f;
#pragma unroll
                for (int e = 0; e < E; ++e) s = fmaf(qv[r][e], kx[u][e], s);
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
                const float mn = fmaxf(m[r], s);
                const float fo = exp2f(m[r] - mn), p = exp2f(s - mn);
                l[r] = l[r] * fo + p;
#pragma unroll
                for (int e = 0; e < E; ++e) acc[r][e] = fmaf(acc[r][e], fo, p * vx[u][e]);
                m[r] = mn;
            }
        }
    }
    // combine the warps
#pragma unroll
    for (int r = 0; r < kShQB; ++r) {
        if (lane == 0) {
            s_m[warp][r] = m[r];
            s_l[warp][r] = l[r];
        }
#pragma unroll
        for (int e = 0; e < E; ++e) s_acc[warp][r][lane + 32 * e] = acc[r][e];
    }
    __syncthreads();
    // thread -> (row, dim) pairs of the CTA's partial
    const int64_t pbase = (bh * nqb + qb) * nsplit;
    auto cta_partial = [&](int r, int i, float &M, float &L, float &A) {
        M = -INFINITY;
        for (int w2 = 0; w2 < kShWarps; ++w2) M = fmaxf(M, s_m[w2][r]);
        L = 0.f;
        A = 0.f;
        if (M == -INFINITY) return;
        for (int w2 = 0; w2 < kShWarps; ++w2) {
            const float f = exp2f(s_m[w2][r] - M);
            L = fmaf(s_l[w2][r], f, L);
            A = fmaf(s_acc[w2][r][i], f, A);
        }
    };
    auto out_row = [&](int r) {   // (b, j, c) row index of block row r
        const int row = r0 + r, j = h * g.g + row / g.C, c = row % g.C;
        return (int64_t(b) * g.Hq + j) * g.C + c;
    };
    if (nsplit == 1) {
        for (int x = tid; x < nrows * D; x += blockDim.x) {
            const int r = x / D, i = x % D;
            float M, L, A;
            cta_partial(r, i, M, L, A);
            out_acc[out_row(r) * D + i] = A;
            if (i == 0) out_ml[out_row(r)] = make_float2(M, L);
        }
        return;
    }
    for (int x = tid; x < nrows * D; x += blockDim.x) {
        const int r = x / D, i = x % D;
        float M, L, A;
        cta_partial(r, i, M, L, A);
        part_acc[((pbase + split) * kShQB + r) * D + i] = A;
        if (i == 0) part_ml[(pbase + split) * kShQB + r] = make_float2(M, L);
    }
    // the barrier orders the CTA's partial writes before thread 0's release
    // on the ticket; the last CTA's acquire makes every split's partial visible
    __syncthreads();
    if (tid == 0) {
        uint32_t prev;
        asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;"
                     : "=r"(prev)
                     : "l"(&ticket[bh * nqb + qb])
                     : "memory");
        is_last = prev == uint32_t(nsplit - 1);
    }
    __syncthreads();
    if (!is_last) return;
    for (int x = tid; x < nrows * D; x += blockDim.x) {
        const int r = x / D, i = x % D;
        float M = -INFINITY;
        for (int s = 0; s < nsplit; ++s) M = fmaxf(M, __ldcg(&part_ml[(pbase + s) * kShQB + r]).x);
        float L = 0.f, A = 0.f;
        if (M != -INFINITY)
            for (int s = 0; s < nsplit; ++s) {
                const float2 ml = __ldcg(&part_ml[(pbase + s) * kShQB + r]);
                const float f = exp2f(ml.x - M);
                L = fmaf(ml.y, f, L);
                A = fmaf(__ldcg(&part_acc[((pbase + s) * kShQB + r) * D + i]), f, A);
            }
        out_acc[out_row(r) * D + i] = A;
        if (i == 0) out_ml[out_row(r)] = make_float2(M, L);
    }
    if (tid == 0) ticket[bh * nqb + qb] = 0u;   // ready for the next call
}

struct ShardAttnPlan {
    int nqb, nsplit;
};
ShardAttnPlan shard_attn_plan(const Geom &g)
{
    ShardAttnPlan p;
    const int64_t rows = int64_t(g.g) * g.C;
    p.nqb = int((rows + kShQB - 1) / kShQB);
    const int64_t base = int64_t(g.B) * g.Hkv * p.nqb;
    int64_t ns = (kShTargetCtas + base - 1) / base;
    const int64_t max_split = (g.Wmax + 127) / 128;   // at least ~128 keys per split
    if (ns > max_split) ns = max_split;
    if (ns > 64) ns = 64;
    p.nsplit = int(ns < 1 ? 1 : ns);
    return p;
}

size_t shard_attn_ws_bytes(const Geom &g, size_t *ticket_bytes, size_t *ml_off)
{
    const ShardAttnPlan p = shard_attn_plan(g);
    const size_t nt = size_t(g.B) * g.Hkv * p.nqb;
    *ticket_bytes = up256(nt * sizeof(uint32_t));
    const size_t acc = up256(nt * p.nsplit * kShQB * g.d * sizeof(float));
    *ml_off = *ticket_bytes + acc;
    return *ticket_bytes + acc + nt * p.nsplit * kShQB * sizeof(float2);
}

// Workspace: [status header][attention: tickets, partials][scan: scores,
// local selection, top-k scratch, summed queries][select: codes, ids].  Every
// offset depends on dims only (the scan region is sized for all the
// sequence's spans, an upper bound for any shard), so each phase finds its
// region without knowing the shard or the shard count.
struct ShardWs {
    size_t att, att_ticket_bytes, att_ml, scores, sel_local, topk, qsum, codes, ids, total;
};
ShardWs shard_ws(const Geom &g, int n)
{
    ShardWs w;
    const size_t BH = size_t(g.B) * g.Hkv;
    size_t off = kWsHeader;
    w.att = off;
    size_t tb = 0, mo = 0;
    off = up256(off + shard_attn_ws_bytes(g, &tb, &mo));
    w.att_ticket_bytes = tb;
    w.att_ml = w.att + mo;
    w.scores = off;
    off = up256(off + BH * size_t(g.NS) * sizeof(float));
    w.sel_local = off;
    off = up256(off + BH * size_t(g.k) * sizeof(int32_t));
    w.topk = off;
    off = up256(off + topk_ws_bytes(g));
    w.qsum = off;
    off = up256(off + score_spans_ws_bytes(g));
    w.codes = off;
    off = up256(off + BH * size_t(n) * g.k * sizeof(uint32_t));
    w.ids = off;
    off = up256(off + BH * size_t(n) * g.k * sizeof(int32_t));
    w.total = off;
    return w;
}

inline uint8_t *at(void *ws, size_t off) { return static_cast<uint8_t *>(ws) + off; }

}  // namespace

int geom_of(const reatt_dims *d, Geom *g);   // abi.cu

}  // namespace reatt

using namespace reatt;

extern "C" {

int reatt_shard_plan(const reatt_dims *dims, int32_t n, reatt_shard *shards)
{
    Geom g;
    const int rc = geom_of(dims, &g);
    if (rc) return rc;
    if (n < 1 || n > 1024 || !shards) return REATT_EINVAL;
    // spans per shard as even as possible; the first shard starts at token 0
    // (global rows), the last ends at T (local rows, current tokens)
    int64_t prev = 0;
    for (int r = 0; r < n; ++r) {
        const int64_t s_end = g.NS * (r + 1) / n;   // spans [.., s_end) on shards 0..r
        int64_t t_end;
        if (r == n - 1) t_end = g.T;
        else if (g.NS == 0) t_end = g.T < g.G ? g.T : g.G;   // no middle: all rows to the last
        else t_end = g.G + s_end * g.S;
        if (t_end > g.T) t_end = g.T;
        if (t_end < prev) t_end = prev;
        shards[r].t_begin = prev;
        shards[r].t_end = t_end;
        shards[r].rows_cap = 0;
        shards[r].owns_current = r == n - 1 ? 1 : 0;
        shards[r].reserved = 0;
        prev = t_end;
    }
    return REATT_OK;
}

int reatt_shard_workspace_bytes(const reatt_dims *dims, const reatt_shard *shard,
                                int32_t n_shards, size_t *bytes)
{
    Geom g;
    int rc = geom_of(dims, &g);
    if (rc) return rc;
    if (n_shards < 1 || n_shards > 1024 || !bytes) return REATT_EINVAL;
    ShardGeom sg;
    rc = make_shard(g, shard, &sg);
    if (rc) return rc;
    *bytes = shard_ws(g, n_shards).total;
    return REATT_OK;
}

int reatt_shard_candidates(const reatt_dims *dims, const reatt_shard *shard, const void *q,
                           const void *k_cache, float *cand_score, int32_t *cand_id, void *ws,
                           reatt_stream stream)
{
    Geom g;
    int rc = geom_of(dims, &g);
    if (rc) return rc;
    ShardGeom sg;
    rc = make_shard(g, shard, &sg);
    if (rc) return rc;
    if (g.k == 0) return REATT_OK;
    if (!q || !ws || !cand_score || !cand_id || (sg.sub.NS > 0 && !k_cache)) return REATT_EINVAL;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(cand_score) || !aligned16(cand_id) ||
        !aligned16(ws))
        return REATT_EINVAL;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const ShardWs w = shard_ws(g, 1);
    float *scores = reinterpret_cast<float *>(at(ws, w.scores));
    int32_t *sel_local = reinterpret_cast<int32_t *>(at(ws, w.sel_local));
    if (sg.sub.NS > 0) {
        const int elem = g.dtype == REATT_BF16 ? 2 : 4;
        cudaError_t e = launch_score_spans(sg.sub, q, shifted(k_cache, sg.t_begin, g.d, elem),
                                           scores, ws, at(ws, w.qsum), nullptr, st,
                                           /*allow_tc=*/false);
        if (e != cudaSuccess) return REATT_ECUDA;
        e = launch_topk(sg.sub, scores, sel_local, at(ws, w.topk), nullptr, 0, nullptr, st);
        if (e != cudaSuccess) return REATT_ECUDA;
    }
    shard_cands_kernel<<<unsigned(g.B * g.Hkv), 128, 0, st>>>(sg.sub.NS, g.k, sg.s_lo, scores,
                                                             sel_local, cand_score, cand_id);
    return cuda_status(cudaGetLastError());
}

int reatt_shard_select(const reatt_dims *dims, int32_t n_shards, const float *cand_score_all,
                       const int32_t *cand_id_all, int32_t *sel, void *ws, reatt_stream stream)
{
    Geom g;
    const int rc = geom_of(dims, &g);
    if (rc) return rc;
    if (n_shards < 1 || n_shards > 1024) return REATT_EINVAL;
    if (g.k == 0) return REATT_OK;
    if (!cand_score_all || !cand_id_all || !sel || !ws) return REATT_EINVAL;
    if (!aligned16(cand_score_all) || !aligned16(cand_id_all) || !aligned16(sel) ||
        !aligned16(ws))
        return REATT_EINVAL;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const ShardWs w = shard_ws(g, n_shards);
    uint32_t *codes = reinterpret_cast<uint32_t *>(at(ws, w.codes));
    int32_t *ids = reinterpret_cast<int32_t *>(at(ws, w.ids));
    const int64_t total = int64_t(n_shards) * g.B * g.Hkv * g.k;
    int blocks = int((total + 255) / 256);
    if (blocks > 4096) blocks = 4096;
    shard_codes_kernel<<<blocks, 256, 0, st>>>(n_shards, int64_t(g.B) * g.Hkv, g.k,
                                               cand_score_all, cand_id_all, codes, ids);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return REATT_ECUDA;
    return cuda_status(launch_topk_merge(g, codes, ids, sel, n_shards * g.k, st));
}

int reatt_shard_attend(const reatt_dims *dims, const reatt_shard *shard, const void *q,
                       const void *k_cache, const void *v_cache, const void *k_cur,
                       const void *v_cur, const int32_t *sel, void *part_ml, float *part_acc,
                       void *ws, reatt_stream stream)
{
    Geom g;
    int rc = geom_of(dims, &g);
    if (rc) return rc;
    ShardGeom sg;
    rc = make_shard(g, shard, &sg);
    if (rc) return rc;
    if (!q || !part_ml || !part_acc || !ws) return REATT_EINVAL;
    if (sg.t_end > sg.t_begin && (!k_cache || !v_cache)) return REATT_EINVAL;
    if (sg.owns_current && (!k_cur || !v_cur)) return REATT_EINVAL;
    if (g.k > 0 && !sel) return REATT_EINVAL;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(k_cur) ||
        !aligned16(v_cur) || !aligned16(sel) || !aligned16(part_ml) || !aligned16(part_acc) ||
        !aligned16(ws))
        return REATT_EINVAL;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const ShardWs w = shard_ws(g, 1);
    const ShardAttnPlan p = shard_attn_plan(g);
    cudaError_t e = cudaMemsetAsync(at(ws, w.att), 0, w.att_ticket_bytes, st);
    if (e != cudaSuccess) return REATT_ECUDA;
    const int elem = g.dtype == REATT_BF16 ? 2 : 4;
    const void *kc = sg.t_end > sg.t_begin ? shifted(k_cache, sg.t_begin, g.d, elem) : nullptr;
    const void *vc = sg.t_end > sg.t_begin ? shifted(v_cache, sg.t_begin, g.d, elem) : nullptr;
    // a valid (never read) selection pointer when k == 0
    const int32_t *selp = g.k > 0 ? sel : reinterpret_cast<const int32_t *>(ws);
    dim3 grid(unsigned(p.nsplit), unsigned(p.nqb), unsigned(g.B * g.Hkv));
    uint32_t *ticket = reinterpret_cast<uint32_t *>(at(ws, w.att));
    float *pacc = reinterpret_cast<float *>(at(ws, w.att + w.att_ticket_bytes));
    float2 *pml = reinterpret_cast<float2 *>(at(ws, w.att_ml));
#define REATT_SHARD_ATT(T, D)                                                                  \
    shard_attend_kernel<T, D><<<grid, kShWarps * 32, 0, st>>>(                                 \
        g, sg.t_begin, sg.t_end, sg.rows, sg.s_lo, sg.s_hi, sg.owns_current,                   \
        static_cast<const T *>(q), static_cast<const T *>(kc), static_cast<const T *>(vc),     \
        static_cast<const T *>(k_cur), static_cast<const T *>(v_cur), selp, p.nsplit, p.nqb,   \
        pacc, pml, ticket, static_cast<float2 *>(part_ml), part_acc)
    if (g.dtype == REATT_BF16) {
        if (g.d == 128) REATT_SHARD_ATT(uint16_t, 128);
        else REATT_SHARD_ATT(uint16_t, 64);
    } else {
        if (g.d == 128) REATT_SHARD_ATT(float, 128);
        else REATT_SHARD_ATT(float, 64);
    }
#undef REATT_SHARD_ATT
    return cuda_status(cudaGetLastError());
}

}  // extern "C"

namespace reatt {
namespace {

__global__ void merge_partials_kernel(int n, int64_t rows, int D, const float2 *__restrict__ ml,
                                      const float *__restrict__ acc, float *__restrict__ out)
{
    const int64_t row = blockIdx.x;
    if (row >= rows) return;
    float M = -INFINITY;
    for (int r = 0; r < n; ++r) M = fmaxf(M, ml[int64_t(r) * rows + row].x);
    float L = 0.f;
    if (M != -INFINITY)
        for (int r = 0; r < n; ++r) {
            const float2 v = ml[int64_t(r) * rows + row];
            L = fmaf(v.y, exp2f(v.x - M), L);
        }
    for (int i = threadIdx.x; i < D; i += blockDim.x) {
        float A = 0.f;
        if (M != -INFINITY)
            for (int r = 0; r < n; ++r) {
                const float2 v = ml[int64_t(r) * rows + row];
                A = fmaf(acc[(int64_t(r) * rows + row) * D + i], exp2f(v.x - M), A);
            }
        out[row * D + i] = L > 0.f ? A / L : 0.f;
    }
}

}  // namespace
}  // namespace reatt

extern "C" int reatt_merge_partials(const reatt_dims *dims, int32_t n_parts,
                                    const void *part_ml_all, const float *part_acc_all,
                                    float *out, reatt_stream stream)
{
    Geom g;
    const int rc = geom_of(dims, &g);
    if (rc) return rc;
    if (n_parts < 1 || n_parts > 1024) return REATT_EINVAL;
    if (!part_ml_all || !part_acc_all || !out) return REATT_EINVAL;
    if (!aligned16(part_ml_all) || !aligned16(part_acc_all) || !aligned16(out))
        return REATT_EINVAL;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int64_t rows = int64_t(g.B) * g.Hq * g.C;
    if (rows > 0x7fffffff) return REATT_EUNSUPPORTED;
    merge_partials_kernel<<<unsigned(rows), 128, 0, st>>>(
        n_parts, rows, g.d, static_cast<const float2 *>(part_ml_all), part_acc_all, out);
    return cuda_status(cudaGetLastError());
}
