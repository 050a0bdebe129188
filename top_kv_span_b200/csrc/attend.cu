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

#include <type_traits>

#include "attend_common.cuh"
#include "common.cuh"
#include "kernels.h"

namespace reatt {

namespace {

constexpr int kAttnThreads = 256;
constexpr int kKT = 64;                 // keys per tile
constexpr int kTargetCtas = 296;        // tile kernel: ~2 CTAs per SM (148 SMs)
constexpr int kMinSplitKeys = 128;      // keys per split at least

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
    __shared__ float2 freq[D / 2];
    const int64_t bh = blockIdx.y;
    const int32_t *sel_bh = sel + bh * geo.k;
    const WinMap m = make_winmap(geo, sel_bh);
    if (blockIdx.x == 0 && threadIdx.x == 0) win_len[bh] = int32_t(m.W);
    if (threadIdx.x < D / 2) freq[threadIdx.x] = make_float2(geo.rope_hi[threadIdx.x], geo.rope_lo[threadIdx.x]);
    __syncthreads();

    const int64_t row0 = int64_t(blockIdx.x) * kGatherRows;
    for (int x = threadIdx.x; x < kGatherRows * HV; x += blockDim.x) {
        const int64_t p = row0 + x / HV;
        const int v = x % HV;
        if (p >= m.W) continue;
        const int64_t s = win_src(geo, m, sel_bh, p);
        const T *kr, *vr;
        if (s >= 0) {
            kr = kc + (bh * geo.Ts + s) * D;
            vr = vc + (bh * geo.Ts + s) * D;
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
        float rl[V], rh[V];
#pragma unroll
        for (int e = 0; e < V; ++e) {
            const int i = v * V + e;
            float c, sn;
            rope_cs(p, freq[i].x, freq[i].y, c, sn);
            rl[e] = klo[e] * c - khi[e] * sn;
            rh[e] = khi[e] * c + klo[e] * sn;
        }
#pragma unroll
        for (int e = 0; e < V; e += 4) {
            const int i = v * V + e;
            *reinterpret_cast<float4 *>(ko + i) = make_float4(rl[e], rl[e + 1], rl[e + 2], rl[e + 3]);
            *reinterpret_cast<float4 *>(ko + i + D / 2) = make_float4(rh[e], rh[e + 1], rh[e + 2], rh[e + 3]);
            *reinterpret_cast<float4 *>(vo + i) = make_float4(vlo[e], vlo[e + 1], vlo[e + 2], vlo[e + 3]);
            *reinterpret_cast<float4 *>(vo + i + D / 2) = make_float4(vhi[e], vhi[e + 1], vhi[e + 2], vhi[e + 3]);
        }
    }
}

// ---------------------------------------------------------------- decode attention
// For few query rows per KV head (R = g*C <= 8, padded to RP): one warp walks
// keys in batches of KB = 32/RP.  Lane l owns the RoPE pairs PD*l .. PD*l+PD-1
// (PD = D/64) and their partners at +D/2, so a key row is rotated in
// registers.  Per batch the KB x RP partial dot products are folded by one
// transposed shuffle reduction (lane i ends with pair (key i/RP, row i%RP)),
// softmax is online per row, and P.V accumulates in registers.  No shared
// memory is touched until the warps of the CTA merge their states.
// Raw (unconverted) words of one lane's PD elements of a row: loaded early,
// converted only when the batch is computed, so loads of the next keys are in
// flight meanwhile.
template <typename T, int PD> struct PairRaw;
template <> struct PairRaw<uint16_t, 2> {
    uint32_t w;
    __device__ __forceinline__ void ld(const uint16_t *p)
    {
        w = __ldg(reinterpret_cast<const unsigned int *>(p));
    }
    __device__ __forceinline__ void lds(const uint8_t *p) { w = *reinterpret_cast<const uint32_t *>(p); }
    __device__ __forceinline__ void get(float (&o)[2]) const
    {
        o[0] = bf16lo(w);
        o[1] = bf16hi(w);
    }
};
template <> struct PairRaw<uint16_t, 1> {
    uint32_t w;
    __device__ __forceinline__ void ld(const uint16_t *p)
    {
        w = __ldg(reinterpret_cast<const unsigned short *>(p));
    }
    __device__ __forceinline__ void lds(const uint8_t *p) { w = *reinterpret_cast<const uint16_t *>(p); }
    __device__ __forceinline__ void get(float (&o)[1]) const { o[0] = __uint_as_float(w << 16); }
};
template <> struct PairRaw<float, 2> {
    float2 w;
    __device__ __forceinline__ void ld(const float *p) { w = __ldg(reinterpret_cast<const float2 *>(p)); }
    __device__ __forceinline__ void lds(const uint8_t *p) { w = *reinterpret_cast<const float2 *>(p); }
    __device__ __forceinline__ void get(float (&o)[2]) const
    {
        o[0] = w.x;
        o[1] = w.y;
    }
};
template <> struct PairRaw<float, 1> {
    float w;
    __device__ __forceinline__ void ld(const float *p) { w = __ldg(p); }
    __device__ __forceinline__ void lds(const uint8_t *p) { w = *reinterpret_cast<const float *>(p); }
    __device__ __forceinline__ void get(float (&o)[1]) const { o[0] = w; }
};

// Window row p -> element offset of its K/V row: cache rows at (bh*T + s)*D,
// current token c at a separate base (flag bit 62 set), in 32-bit index math.
__device__ __forceinline__ int64_t win_row_offset(const Geom &geo, const WinMap &m,
                                                  const int32_t *sel_bh, int64_t bh, int p, int D)
{
    const int g_end = int(m.g_end), nsel = int(m.nsel_rows), nloc = int(m.n_loc);
    int s;
    if (p < g_end) {
        s = p;
    } else if (p - g_end < nsel) {
        const int q = p - g_end, j = q / geo.S, off = q - j * geo.S;
        int sp = sel_bh[j];
        sp = sp < 0 ? 0 : (sp >= int(geo.NS) ? int(geo.NS) - 1 : sp);
        s = geo.G + sp * geo.S + off;
        if (s >= int(geo.T)) s = int(geo.T) - 1;
    } else if (p - g_end - nsel < nloc) {
        s = int(m.loc_begin) + (p - g_end - nsel);
    } else {
        const int c = p - g_end - nsel - nloc;
        return (int64_t(1) << 62) | ((bh * geo.C + c) * D);
    }
    return (bh * geo.Ts + s) * D;
}

constexpr int kDecWarps = 8;

template <typename T, int D, int RP, bool VIRT>
__global__ void __launch_bounds__(kDecWarps * 32, 2)
attend_decode_kernel(Geom geo, AttnArgs a, const T *__restrict__ kc, const T *__restrict__ vc,
                     const T *__restrict__ kcur, const T *__restrict__ vcur,
                     const float *__restrict__ kw, const float *__restrict__ vw)
{
    constexpr int PD = D / 64;            // RoPE pairs per lane
    constexpr int KB = 32 / RP;           // keys per batch
    using RowT = typename std::conditional<VIRT, T, float>::type;
    __shared__ float s_m[kDecWarps][RP], s_l[kDecWarps][RP];
    __shared__ __align__(16) float s_acc[kDecWarps][RP][D];
    __shared__ float f_m[RP], f_l[RP];
    __shared__ float2 freq[D / 2];
    __shared__ int is_last;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid < D / 2) freq[tid] = make_float2(geo.rope_hi[tid], geo.rope_lo[tid]);
    pdl_wait();
    __syncthreads();
    const int split = blockIdx.x;
    const int64_t bh = blockIdx.z;
    const int b = int(bh / geo.Hkv), h = int(bh % geo.Hkv);
    const int nrows = geo.g * geo.C;     // <= RP (one query block)
    const int32_t *sel_bh = VIRT ? a.sel + bh * geo.k : nullptr;
    const WinMap m = attn_winmap(geo, a, VIRT, bh, sel_bh);
    const int64_t W = m.W, qpos0 = W - geo.C;
    int64_t kbeg, kend;
    split_range(geo, W, a.nsplit, split, 0, nrows, 32, kbeg, kend);

    // this lane's query pairs for every row (zero for padded rows)
    float qlo[RP][PD], qhi[RP][PD];
#pragma unroll
    for (int r = 0; r < RP; ++r)
#pragma unroll
        for (int e = 0; e < PD; ++e) {
            qlo[r][e] = qhi[r][e] = 0.f;
            if (r < nrows)
                query_pair<T, D>(geo, freq, a.q, b, h, r, qpos0, PD * lane + e, qlo[r][e], qhi[r][e]);
        }
    // causal limit of this lane's logit row (lane % RP) and of every row
    const int my_r = lane % RP;
    const int64_t my_lim = my_r < nrows ? qpos0 + my_r % geo.C : -1;

    float mrow[RP], lrow[RP], alo[RP][PD], ahi[RP][PD];
#pragma unroll
    for (int r = 0; r < RP; ++r) {
        mrow[r] = -INFINITY;
        lrow[r] = 0.f;
#pragma unroll
        for (int e = 0; e < PD; ++e) alo[r][e] = ahi[r][e] = 0.f;
    }
    float m_own = -INFINITY;

    constexpr int NB = KB <= 8 ? 2 : 1;   // batches whose loads go out together
    constexpr int KI = NB * KB;             // keys per warp iteration (<= 32)
    for (int64_t pi = kbeg + int64_t(warp) * KI; pi < kend; pi += int64_t(kDecWarps) * KI) {
        // lane kk < KI resolves the row of key pi + kk once; the others take
        // it by shuffle
        int64_t my_off = -1;
        if (lane < KI && pi + lane < kend) {
            if (VIRT) my_off = win_row_offset(geo, m, sel_bh, bh, int(pi + lane), D);
            else my_off = (bh * geo.Wmax + pi + lane) * D;
        }
        PairRaw<RowT, PD> rkl[KI], rkh[KI], rvl[KI], rvh[KI];
#pragma unroll
        for (int kk = 0; kk < KI; ++kk) {
            const int64_t off = __shfl_sync(0xffffffffu, my_off, kk);
            if (off >= 0) {
                const RowT *kr, *vr;
                if (VIRT) {
                    const int64_t o = off & ~(int64_t(1) << 62);
                    const bool cur = (off >> 62) != 0;
                    kr = reinterpret_cast<const RowT *>(cur ? kcur : kc) + o;
                    vr = reinterpret_cast<const RowT *>(cur ? vcur : vc) + o;
                } else {
                    kr = reinterpret_cast<const RowT *>(kw) + off;
                    vr = reinterpret_cast<const RowT *>(vw) + off;
                }
                rkl[kk].ld(kr + PD * lane);
                rkh[kk].ld(kr + D / 2 + PD * lane);
                rvl[kk].ld(vr + PD * lane);
                rvh[kk].ld(vr + D / 2 + PD * lane);
            }
        }
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
        const int64_t p0 = pi + nb * KB;
        float klo[KB][PD], khi[KB][PD], vlo[KB][PD], vhi[KB][PD];
#pragma unroll
        for (int kk = 0; kk < KB; ++kk) {
            const int64_t p = p0 + kk;
            if (p < kend) {
                rkl[nb * KB + kk].get(klo[kk]);
                rkh[nb * KB + kk].get(khi[kk]);
                rvl[nb * KB + kk].get(vlo[kk]);
                rvh[nb * KB + kk].get(vhi[kk]);
                if (VIRT) {   // rotate the key pair at window position p
                    const float2 *cs = a.tab + p * (D / 2) + PD * lane;
#pragma unroll
                    for (int e = 0; e < PD; ++e) {
                        const float2 t = __ldg(cs + e);
                        const float x0 = klo[kk][e], x1 = khi[kk][e];
                        klo[kk][e] = x0 * t.x - x1 * t.y;
                        khi[kk][e] = x1 * t.x + x0 * t.y;
                    }
                }
            } else {
#pragma unroll
                for (int e = 0; e < PD; ++e) klo[kk][e] = khi[kk][e] = vlo[kk][e] = vhi[kk][e] = 0.f;
            }
        }
        // partial dots part[kk*RP + r] over this lane's pairs
        float part[32];
#pragma unroll
        for (int kk = 0; kk < KB; ++kk)
#pragma unroll
            for (int r = 0; r < RP; ++r) {
                float z = 0.f;
#pragma unroll
                for (int e = 0; e < PD; ++e)
                    z = fmaf(qlo[r][e], klo[kk][e], fmaf(qhi[r][e], khi[kk][e], z));
                part[kk * RP + r] = z;
            }
        // transposed reduction: lane i ends with the full dot of index i
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            const bool upper = (lane & o) != 0;
#pragma unroll
            for (int i = 0; i < o; ++i) {
                const float send = upper ? part[i] : part[i + o];
                const float keep = upper ? part[i + o] : part[i];
                part[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
            }
        }
        const int64_t my_p = p0 + lane / RP;
        const float x = (my_p < kend && my_p <= my_lim) ? part[0] : -INFINITY;
        // batch max per row (lanes sharing lane % RP), new running max
        float bm = x;
#pragma unroll
        for (int o = RP; o < 32; o <<= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, o));
        const float mn_own = fmaxf(m_own, bm);
        const float pv = x == -INFINITY ? 0.f : exp2f(x - mn_own);
        m_own = mn_own;
        float bs = pv;
#pragma unroll
        for (int o = RP; o < 32; o <<= 1) bs += __shfl_xor_sync(0xffffffffu, bs, o);
#pragma unroll
        for (int r = 0; r < RP; ++r) {
            const float mn = fmaxf(mrow[r], __shfl_sync(0xffffffffu, bm, r));
            const float cf = mn == -INFINITY ? 1.f : exp2f(mrow[r] - mn);
            mrow[r] = mn;
            lrow[r] = lrow[r] * cf + __shfl_sync(0xffffffffu, bs, r);
#pragma unroll
            for (int e = 0; e < PD; ++e) {
                alo[r][e] *= cf;
                ahi[r][e] *= cf;
            }
        }
#pragma unroll
        for (int kk = 0; kk < KB; ++kk)
#pragma unroll
            for (int r = 0; r < RP; ++r) {
                const float pr = __shfl_sync(0xffffffffu, pv, kk * RP + r);
#pragma unroll
                for (int e = 0; e < PD; ++e) {
                    alo[r][e] = fmaf(pr, vlo[kk][e], alo[r][e]);
                    ahi[r][e] = fmaf(pr, vhi[kk][e], ahi[r][e]);
                }
            }
    }
    }

    // merge the warps of the CTA
#pragma unroll
    for (int r = 0; r < RP; ++r) {
        if (lane == 0) {
            s_m[warp][r] = mrow[r];
            s_l[warp][r] = lrow[r];
        }
#pragma unroll
        for (int e = 0; e < PD; ++e) {
            s_acc[warp][r][PD * lane + e] = alo[r][e];
            s_acc[warp][r][D / 2 + PD * lane + e] = ahi[r][e];
        }
    }
    __syncthreads();
    if (tid < RP) {
        float mx = -INFINITY;
        for (int w2 = 0; w2 < kDecWarps; ++w2) mx = fmaxf(mx, s_m[w2][tid]);
        float l = 0.f;
        for (int w2 = 0; w2 < kDecWarps; ++w2) {
            const float wt = s_m[w2][tid] == -INFINITY ? 0.f : exp2f(s_m[w2][tid] - mx);
            s_m[w2][tid] = wt;   // now a weight
            l += wt * s_l[w2][tid];
        }
        f_m[tid] = mx;
        f_l[tid] = l;
    }
    __syncthreads();
    for (int x = tid; x < RP * D; x += kDecWarps * 32) {
        const int r = x / D, i = x % D;
        float z = 0.f;
        for (int w2 = 0; w2 < kDecWarps; ++w2) z = fmaf(s_m[w2][r], s_acc[w2][r][i], z);
        s_acc[0][r][i] = z;   // row r of warp 0's slot is only read by this thread
    }
    __syncthreads();
    split_finish<D, RP>(geo, a, bh, 0, split, nrows, f_m, f_l, &s_acc[0][0][0], &s_acc[1][0][0],
                        &is_last);
}

// ---------------------------------------------------------------- staged decode attention
// The fused step's decode path.  One producer thread walks the CTA's key range
// of the virtual window in chunks that are contiguous in memory (<= 32 rows,
// never crossing the end of the global part, of a chosen span, of the local
// part) and bulk-copies each chunk's K and V rows into a shared-memory ring
// (cp.async.bulk, mbarrier completion).  Consumer warp w takes chunks w,
// w+NCW, ... (fixed stage -> warp map, so parity waits never run ahead) and
// computes as the register kernel above, reading its pair words from shared
// memory.  The step's RoPE cos/sin table rows for the chunk's positions come
// into the same ring stage.
constexpr int kTmaCW = 12;                 // consumer warps (13 warps: <= 128 registers)
constexpr int kTmaStages = 2 * kTmaCW;     // warp w owns stages w and w + kTmaCW

template <typename T, int D, int RP>
struct TmaShape {
    static constexpr int kRowBytes = D * Elem<T>::kBytes;
    static constexpr int kTabRowBytes = D / 2 * 8;                     // (cos, sin) per pair
    static constexpr int kChunk = (RP <= 4 && kRowBytes <= 256) ? 8 : 4;   // rows per stage
    // K rows, then V rows, then the rows' RoPE table entries
    static constexpr int kStageBytes = kChunk * (2 * kRowBytes + kTabRowBytes);
    static constexpr size_t kRing = size_t(kTmaStages) * kStageBytes;
};
static_assert(kTmaStages % kTmaCW == 0, "stage -> warp map must be fixed");

// Chunk of window rows starting at p: its length (contiguous source run).
__device__ __forceinline__ int chunk_len(const Geom &geo, const WinMap &m, int p, int kend,
                                         int chunk)
{
    const int g_end = int(m.g_end), nsel = int(m.nsel_rows), nloc = int(m.n_loc);
    int end;
    if (p < g_end) {
        end = g_end;
    } else if (p < g_end + nsel) {
        const int j = (p - g_end) / geo.S;
        end = g_end + (j + 1) * geo.S;
        if (end > g_end + nsel) end = g_end + nsel;
    } else if (p < g_end + nsel + nloc) {
        end = g_end + nsel + nloc;
    } else {
        end = int(m.W);
    }
    if (end > kend) end = kend;
    if (end > p + chunk) end = p + chunk;
    return end - p;
}

// The chosen span ids a CTA's key range touches, staged in shared memory so
// the producer's address computations do not wait on global loads.
constexpr int kSelCache = 512;

template <typename T, int D, int RP>
__global__ void __launch_bounds__((kTmaCW + 1) * 32, 1)
attend_staged_kernel(Geom geo, AttnArgs a, const T *__restrict__ kc, const T *__restrict__ vc,
                     const T *__restrict__ kcur, const T *__restrict__ vcur, void *ws)
{
    using Sh = TmaShape<T, D, RP>;
    constexpr int PD = D / 64;            // RoPE pairs per lane
    constexpr int KB = 32 / RP;           // keys per reduction batch
    constexpr int RB = Sh::kRowBytes;
    constexpr int CH = Sh::kChunk;
    constexpr int EB = Elem<T>::kBytes;
    static_assert(kTmaStages % kTmaCW == 0, "chunk ci -> stage ci % kTmaStages -> warp ci % kTmaCW");
    extern __shared__ __align__(128) uint8_t smem[];
    uint8_t *ring = smem;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + Sh::kRing);
    uint64_t *empty = full + kTmaStages;
    float *s_acc = reinterpret_cast<float *>(empty + kTmaStages);      // [kTmaCW][RP][D]
    float *s_m = s_acc + kTmaCW * RP * D;                               // [kTmaCW][RP]
    float *s_l = s_m + kTmaCW * RP;
    __shared__ float f_m[RP], f_l[RP];
    __shared__ float2 freq[D / 2];
    __shared__ __align__(16) float q_s[RP][D];     // rotated, scaled queries
    __shared__ int is_last, abort_flag;
    __shared__ int32_t sel_s[kSelCache];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        abort_flag = 0;
        for (int s = 0; s < kTmaStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init_fence();
    }
    if (tid < D / 2) freq[tid] = make_float2(geo.rope_hi[tid], geo.rope_lo[tid]);
    // With the window length known up front, the rows that do not depend on
    // the selection (local part and current token) are taken first, while the
    // top-k still runs; only the producer's copies of chosen rows and the
    // split merge wait for the preceding grid.  Otherwise everything waits.
    const bool early = a.w_known >= 0;
    if (!early) pdl_wait();

    const int split = blockIdx.x;
    const int64_t bh = blockIdx.z;
    const int b = int(bh / geo.Hkv), h = int(bh % geo.Hkv);
    const int nrows = geo.g * geo.C;
    const int32_t *sel_bh = a.sel + bh * geo.k;
    WinMap m;
    if (early) {
        m.g_end = geo.g_end;
        m.loc_begin = geo.loc_begin;
        m.n_loc = geo.n_loc;
        m.W = a.w_known;
        m.nsel_rows = m.W - m.g_end - m.n_loc - geo.C;
    } else {
        m = make_winmap(geo, sel_bh);
    }
    const int64_t W = m.W, qpos0 = W - geo.C;
    const int g_end = int(m.g_end), nsel = int(m.nsel_rows), nloc = int(m.n_loc);
    // This CTA's rows: a slice of the early range [g_end + nsel, W), then a
    // slice of the late range [0, g_end + nsel) (without early mode the late
    // range is the whole window), cut at multiples of CH; rows past the last
    // query's causal limit are dropped.
    const int r_mid = early ? g_end + nsel : int(W);
    int eb, ee, lb, le;
    {
        const int last_row = nrows - 1;
        const int c_max = (last_row / geo.C == 0) ? last_row % geo.C : geo.C - 1;
        const int lim = int(W) - geo.C + c_max + 1;
        auto part = [&](int r0, int r1, int &pb, int &pe) {
            int len = (r1 - r0 + a.nsplit - 1) / a.nsplit;
            len = (len + CH - 1) / CH * CH;
            pb = r0 + split * len;
            pe = pb + len;
            if (pe > r1) pe = r1;
            if (pe > lim) pe = lim;
            if (pb > pe) pb = pe;
        };
        part(r_mid, int(W), eb, ee);
        part(0, r_mid, lb, le);
    }
    const int nE = (ee - eb + CH - 1) / CH;
    const int nchunks = nE + (le - lb + CH - 1) / CH;
    // chunk ci -> first window row and row count
    auto chunk_at = [&](int ci, int &p0, int &n) {
        const int pend = ci < nE ? ee : le;
        p0 = ci < nE ? eb + ci * CH : lb + (ci - nE) * CH;
        n = pend - p0 < CH ? pend - p0 : CH;
    };
    // span ids of the chosen part inside the late slice
    int j0 = 0, jn = 0;
    {
        const int lo = lb > g_end ? lb : g_end;
        const int hi = le < g_end + nsel ? le : g_end + nsel;
        if (lo < hi) {
            j0 = (lo - g_end) / geo.S;
            jn = (hi - 1 - g_end) / geo.S - j0 + 1;
        }
    }
    const bool sel_cached = jn <= kSelCache;
    __syncthreads();   // freq visible to the query rotation
    for (int x = tid; x < RP * (D / 2); x += blockDim.x) {
        const int rr = x / (D / 2), i = x % (D / 2);
        float lo = 0.f, hi = 0.f;
        if (rr < nrows) query_pair<T, D>(geo, freq, a.q, b, h, rr, qpos0, i, lo, hi);
        q_s[rr][i] = lo;
        q_s[rr][i + D / 2] = hi;
    }
    __syncthreads();

    if (warp == kTmaCW) {
        // ------------------------------------------------ producer warp
        // chunk ci -> stage ci % kTmaStages; lane l issues every chunk of
        // stage l, in order, so each barrier has one waiter taking its phases
        // in turn.  A chunk crossing a region boundary is copied as several
        // runs.  Chunks of the early slice come first; before the first chunk
        // of the late slice the warp waits for the selection.
        static_assert(kTmaStages <= 32, "one producer lane per stage");
        int issued = 0, ci = lane;
        bool stop = lane >= kTmaStages;
        auto issue_until = [&](int c_end) {
            for (; !stop && ci < c_end; ci += kTmaStages, ++issued) {
                const int stage = lane;
                if (issued > 0 &&
                    (*(volatile int *)&abort_flag ||
                     !mbar_wait_bounded(&empty[stage], uint32_t((issued - 1) & 1), kWaitLimitNs))) {
                    report_status(ws, REATT_ETIMEOUT);
                    *(volatile int *)&abort_flag = 1;
                    stop = true;
                    break;
                }
                int p0, n;
                chunk_at(ci, p0, n);
                uint8_t *dst = ring + stage * Sh::kStageBytes;
                mbar_arrive_expect_tx(&full[stage], uint32_t(n) * (2u * RB + Sh::kTabRowBytes));
                bulk_load_plain(dst + 2 * CH * RB, a.tab + int64_t(p0) * (D / 2),
                                uint32_t(n) * Sh::kTabRowBytes, &full[stage]);
                for (int p = p0; p < p0 + n;) {
                    const int r = chunk_len(geo, m, p, p0 + n, CH);
                    bool cur = false;
                    int64_t o;
                    if (p < g_end) {
                        o = (bh * geo.Ts + p) * D;
                    } else if (p - g_end < nsel) {
                        const int q = p - g_end, j = q / geo.S, off = q - j * geo.S;
                        int sp = sel_cached ? sel_s[j - j0] : sel_bh[j];
                        sp = sp < 0 ? 0 : (sp >= int(geo.NS) ? int(geo.NS) - 1 : sp);
                        int srow = geo.G + sp * geo.S + off;
                        if (srow >= int(geo.T)) srow = int(geo.T) - 1;
                        o = (bh * geo.Ts + srow) * D;
                    } else if (p - g_end - nsel < nloc) {
                        o = (bh * geo.Ts + m.loc_begin + (p - g_end - nsel)) * D;
                    } else {
                        cur = true;
                        o = (bh * geo.C + (p - g_end - nsel - nloc)) * D;
                    }
                    const uint32_t bytes = uint32_t(r) * RB;
                    bulk_load_plain(dst + (p - p0) * RB, (cur ? kcur : kc) + o, bytes, &full[stage]);
                    bulk_load_plain(dst + (CH + p - p0) * RB, (cur ? vcur : vc) + o, bytes,
                                    &full[stage]);
                    p += r;
                }
            }
        };
        issue_until(nE);
        __syncwarp();
        pdl_wait();   // the selection comes from the preceding kernel
        if (sel_cached)
            for (int j = lane; j < jn; j += 32) sel_s[j] = sel_bh[j0 + j];
        __syncwarp();
        issue_until(nchunks);
        // drain: this stage's last issued copy has landed
        if (lane < kTmaStages && issued > 0 &&
            !mbar_wait_bounded(&full[lane], uint32_t((issued - 1) & 1), kWaitLimitNs))
            report_status(ws, REATT_ETIMEOUT);
    } else {
        // ---------------------------------------------------- consumers
        float qlo[RP][PD], qhi[RP][PD];
#pragma unroll
        for (int e = 0; e < PD; ++e) {
            const int i = PD * lane + e;
#pragma unroll
            for (int r = 0; r < RP; ++r) {
                qlo[r][e] = q_s[r][i];
                qhi[r][e] = q_s[r][i + D / 2];
            }
        }
        const int my_r = lane % RP;
        const int64_t my_lim = my_r < nrows ? qpos0 + my_r % geo.C : -1;
        float mrow[RP], lrow[RP], alo[RP][PD], ahi[RP][PD];
#pragma unroll
        for (int r = 0; r < RP; ++r) {
            mrow[r] = -INFINITY;
            lrow[r] = 0.f;
#pragma unroll
            for (int e = 0; e < PD; ++e) alo[r][e] = ahi[r][e] = 0.f;
        }
        float m_own = -INFINITY;

        for (int ci = warp; ci < nchunks; ci += kTmaCW) {
            const int stage = ci % kTmaStages;
            int p0, n;
            chunk_at(ci, p0, n);
            if (__any_sync(0xffffffffu, *(volatile int *)&abort_flag != 0)) break;
            const bool ok =
                mbar_wait_bounded(&full[stage], uint32_t((ci / kTmaStages) & 1), kWaitLimitNs);
            if (!__all_sync(0xffffffffu, ok)) {
                if (lane == 0) {
                    report_status(ws, REATT_ETIMEOUT);
                    *(volatile int *)&abort_flag = 1;
                }
                break;
            }
            const uint8_t *kb = ring + stage * Sh::kStageBytes;
            const uint8_t *vb = kb + CH * RB;
            const float2 *tb = reinterpret_cast<const float2 *>(kb + 2 * CH * RB);
            for (int sb = 0; sb < n; sb += KB) {
                float part[32];
#pragma unroll
                for (int kk = 0; kk < KB; ++kk) {
                    const int row = sb + kk;
                    float klo[PD], khi[PD];
                    if (row < n) {
                        PairRaw<T, PD> w0, w1;
                        w0.lds(kb + row * RB + PD * lane * EB);
                        w1.lds(kb + row * RB + (D / 2 + PD * lane) * EB);
                        w0.get(klo);
                        w1.get(khi);
                    } else {
#pragma unroll
                        for (int e = 0; e < PD; ++e) klo[e] = khi[e] = 0.f;
                    }
                    if (row < n) {   // rotate at window position p0 + row
#pragma unroll
                        for (int e = 0; e < PD; ++e) {
                            const float2 cs = tb[row * (D / 2) + PD * lane + e];
                            const float x0 = klo[e], x1 = khi[e];
                            klo[e] = x0 * cs.x - x1 * cs.y;
                            khi[e] = x1 * cs.x + x0 * cs.y;
                        }
                    }
#pragma unroll
                    for (int r = 0; r < RP; ++r) {
                        float z = 0.f;
#pragma unroll
                        for (int e = 0; e < PD; ++e)
                            z = fmaf(qlo[r][e], klo[e], fmaf(qhi[r][e], khi[e], z));
                        part[kk * RP + r] = z;
                    }
                }
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1) {
                    const bool upper = (lane & o) != 0;
#pragma unroll
                    for (int i = 0; i < o; ++i) {
                        const float send = upper ? part[i] : part[i + o];
                        const float keep = upper ? part[i + o] : part[i];
                        part[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
                    }
                }
                const int my_row = sb + lane / RP;
                const int64_t my_p = int64_t(p0) + my_row;
                const float x = (my_row < n && my_p <= my_lim) ? part[0] : -INFINITY;
                float bm = x;
#pragma unroll
                for (int o = RP; o < 32; o <<= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, o));
                const float mn_own = fmaxf(m_own, bm);
                const float pv = x == -INFINITY ? 0.f : exp2f(x - mn_own);
                m_own = mn_own;
                float bs = pv;
#pragma unroll
                for (int o = RP; o < 32; o <<= 1) bs += __shfl_xor_sync(0xffffffffu, bs, o);
#pragma unroll
                for (int r = 0; r < RP; ++r) {
                    const float mn = fmaxf(mrow[r], __shfl_sync(0xffffffffu, bm, r));
                    const float cf = mn == -INFINITY ? 1.f : exp2f(mrow[r] - mn);
                    mrow[r] = mn;
                    lrow[r] = lrow[r] * cf + __shfl_sync(0xffffffffu, bs, r);
#pragma unroll
                    for (int e = 0; e < PD; ++e) {
                        alo[r][e] *= cf;
                        ahi[r][e] *= cf;
                    }
                }
#pragma unroll
                for (int kk = 0; kk < KB; ++kk) {
                    const int row = sb + kk;
                    float vlo[PD], vhi[PD];
                    if (row < n) {
                        PairRaw<T, PD> w2, w3;
                        w2.lds(vb + row * RB + PD * lane * EB);
                        w3.lds(vb + row * RB + (D / 2 + PD * lane) * EB);
                        w2.get(vlo);
                        w3.get(vhi);
                    } else {
#pragma unroll
                        for (int e = 0; e < PD; ++e) vlo[e] = vhi[e] = 0.f;
                    }
#pragma unroll
                    for (int r = 0; r < RP; ++r) {
                        const float pr = __shfl_sync(0xffffffffu, pv, kk * RP + r);
#pragma unroll
                        for (int e = 0; e < PD; ++e) {
                            alo[r][e] = fmaf(pr, vlo[e], alo[r][e]);
                            ahi[r][e] = fmaf(pr, vhi[e], ahi[r][e]);
                        }
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[stage]);   // chunk consumed: hand the stage back
        }
        // this warp's state to shared memory
#pragma unroll
        for (int r = 0; r < RP; ++r) {
            if (lane == 0) {
                s_m[warp * RP + r] = mrow[r];
                s_l[warp * RP + r] = lrow[r];
            }
#pragma unroll
            for (int e = 0; e < PD; ++e) {
                s_acc[(warp * RP + r) * D + PD * lane + e] = alo[r][e];
                s_acc[(warp * RP + r) * D + D / 2 + PD * lane + e] = ahi[r][e];
            }
        }
    }
    pdl_wait();   // split partials and tickets: after the preceding grid (it clears the tickets)
    __syncthreads();
    // merge the consumer warps
    if (tid < RP) {
        float mx = -INFINITY;
        for (int w2 = 0; w2 < kTmaCW; ++w2) mx = fmaxf(mx, s_m[w2 * RP + tid]);
        float l = 0.f;
        for (int w2 = 0; w2 < kTmaCW; ++w2) {
            const float mv = s_m[w2 * RP + tid];
            const float wt = mv == -INFINITY ? 0.f : exp2f(mv - mx);
            s_m[w2 * RP + tid] = wt;
            l += wt * s_l[w2 * RP + tid];
        }
        f_m[tid] = mx;
        f_l[tid] = l;
    }
    __syncthreads();
    for (int x = tid; x < RP * D; x += blockDim.x) {
        const int r = x / D, i = x % D;
        float z = 0.f;
        for (int w2 = 0; w2 < kTmaCW; ++w2) z = fmaf(s_m[w2 * RP + r], s_acc[(w2 * RP + r) * D + i], z);
        s_acc[r * D + i] = z;   // slot (warp 0, r): only this thread touches element i
    }
    __syncthreads();
    split_finish<D, RP>(geo, a, bh, 0, split, nrows, f_m, f_l, s_acc, s_acc + RP * D, &is_last);
}

template <typename T, int D>
cudaError_t launch_staged_attn(const Geom &geo, const AttnArgs &a, int RP, const void *kc,
                               const void *vc, const void *kcur, const void *vcur, void *ws,
                               cudaStream_t st)
{
    dim3 grid(unsigned(a.nsplit), 1u, unsigned(geo.B * geo.Hkv));
    const T *k = static_cast<const T *>(kc), *v = static_cast<const T *>(vc);
    const T *kq = static_cast<const T *>(kcur), *vq = static_cast<const T *>(vcur);
#define REATT_STAGED(RPV)                                                                      \
    do {                                                                                       \
        using Sh = TmaShape<T, D, RPV>;                                                        \
        const size_t smem = Sh::kRing + 2 * kTmaStages * sizeof(uint64_t) +                   \
                            size_t(kTmaCW) * RPV * (D + 2) * sizeof(float);                    \
        auto kern = attend_staged_kernel<T, D, RPV>;                                           \
        cudaError_t e =                                                                        \
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)); \
        if (e != cudaSuccess) return e;                                                        \
        e = launch_pdl(kern, grid, dim3((kTmaCW + 1) * 32), smem, st, geo, a, k, v, kq, vq, ws); \
        if (e != cudaSuccess) return e;                                                        \
    } while (0)
    switch (RP) {
    case 1: REATT_STAGED(1); break;
    case 2: REATT_STAGED(2); break;
    case 4: REATT_STAGED(4); break;
    default: REATT_STAGED(8); break;
    }
#undef REATT_STAGED
    return cudaGetLastError();
}

// ---------------------------------------------------------------- tile attention
// Many query rows per KV head (chunked prefill): a CTA owns QB rows and stages
// key/value tiles of 64 rows through shared memory (rotated on the way in when
// read from the un-rotated cache), with register prefetch of the next tile.
template <int D, int QB>
struct AttnSmem {
    static constexpr int kKS = D + 4;                     // padded key row (floats)
    static constexpr size_t kQ = size_t(QB) * D * 4;
    static constexpr size_t kK = size_t(kKT) * kKS * 4;
    static constexpr size_t kV = size_t(kKT) * D * 4;
    static constexpr size_t kP = size_t(QB) * kKT * 4;
    static constexpr size_t kRow = size_t(QB) * 4 * 4;   // m, l, corr, spare
    static constexpr size_t kTotal = kQ + kK + kV + kP + kRow;
};

// Raw (unconverted) 16-byte vectors of one half-row item of K and V.
struct RawKV {
    uint4 klo, khi, vlo, vhi;
};

template <typename T, int D, bool VIRT>
struct KvSource;

// Virtual window: rows straight from the un-rotated cache / current tokens,
// rotated with the per-step cos/sin table.
template <typename T, int D>
struct KvSource<T, D, true> {
    const T *kc, *vc, *kcur, *vcur;
    const float2 *tab;
    static constexpr int V = Elem<T>::kVec;
    __device__ __forceinline__ RawKV fetch(const Geom &geo, const WinMap &m, int64_t bh,
                                           const int32_t *sel_bh, int64_t p, int v) const
    {
        const int64_t s = win_src(geo, m, sel_bh, p);
        const T *kr, *vr;
        if (s >= 0) {
            kr = kc + (bh * geo.Ts + s) * D;
            vr = vc + (bh * geo.Ts + s) * D;
        } else {
            kr = kcur + (bh * geo.C + (-s - 1)) * D;
            vr = vcur + (bh * geo.C + (-s - 1)) * D;
        }
        RawKV r;
        r.klo = ldg_stream(kr + v * V);
        r.khi = ldg_stream(kr + D / 2 + v * V);
        r.vlo = ldg_stream(vr + v * V);
        r.vhi = ldg_stream(vr + D / 2 + v * V);
        return r;
    }
    __device__ __forceinline__ void finish(const RawKV &r, int64_t p, int v, float (&klo)[V],
                                           float (&khi)[V], float (&vlo)[V], float (&vhi)[V]) const
    {
        float a[V], b[V];
        Elem<T>::unpack(r.klo, a);
        Elem<T>::unpack(r.khi, b);
        Elem<T>::unpack(r.vlo, vlo);
        Elem<T>::unpack(r.vhi, vhi);
        const float4 *cs = reinterpret_cast<const float4 *>(tab + p * (D / 2) + v * V);
#pragma unroll
        for (int e = 0; e < V; e += 2) {
            const float4 t = __ldg(cs + e / 2);   // (cos, sin) of elements e, e+1
            klo[e] = a[e] * t.x - b[e] * t.y;
            khi[e] = b[e] * t.x + a[e] * t.y;
            klo[e + 1] = a[e + 1] * t.z - b[e + 1] * t.w;
            khi[e + 1] = b[e + 1] * t.z + a[e + 1] * t.w;
        }
    }
};

// Materialised fp32 window (already rotated by gather_rope).
template <typename T, int D>
struct KvSource<T, D, false> {
    const float *kw, *vw;
    static constexpr int V = 4;
    __device__ __forceinline__ RawKV fetch(const Geom &geo, const WinMap &, int64_t bh,
                                           const int32_t *, int64_t p, int v) const
    {
        const float *kr = kw + (bh * geo.Wmax + p) * D;
        const float *vr = vw + (bh * geo.Wmax + p) * D;
        RawKV r;
        r.klo = ldg_stream(kr + v * V);
        r.khi = ldg_stream(kr + D / 2 + v * V);
        r.vlo = ldg_stream(vr + v * V);
        r.vhi = ldg_stream(vr + D / 2 + v * V);
        return r;
    }
    __device__ __forceinline__ void finish(const RawKV &r, int64_t, int, float (&klo)[V],
                                           float (&khi)[V], float (&vlo)[V], float (&vhi)[V]) const
    {
        Elem<float>::unpack(r.klo, klo);
        Elem<float>::unpack(r.khi, khi);
        Elem<float>::unpack(r.vlo, vlo);
        Elem<float>::unpack(r.vhi, vhi);
    }
};

template <typename T, int D, int QB, bool VIRT>
__global__ void __launch_bounds__(kAttnThreads)
attend_tile_kernel(Geom geo, AttnArgs a, KvSource<T, D, VIRT> src)
{
    using Sm = AttnSmem<D, QB>;
    constexpr int V = KvSource<T, D, VIRT>::V;
    constexpr int HV = D / 2 / V;                          // half-row vectors
    constexpr int NITEM = kKT * HV / kAttnThreads;         // load items per thread
    constexpr int NR = QB / 4;                             // logit rows per thread
    constexpr int D4 = D / 4;
    constexpr int NACC = (QB * D4 + kAttnThreads - 1) / kAttnThreads;
    constexpr int KS = Sm::kKS;
    static_assert(NITEM >= 1 && kKT * HV % kAttnThreads == 0, "tile shape");
    static_assert(kAttnThreads % kKT == 0 && QB % 4 == 0, "tile shape");
    extern __shared__ __align__(128) uint8_t smem[];
    float *Qs = reinterpret_cast<float *>(smem);
    float *Ks = reinterpret_cast<float *>(smem + Sm::kQ);
    float *Vs = reinterpret_cast<float *>(smem + Sm::kQ + Sm::kK);
    float *Ps = reinterpret_cast<float *>(smem + Sm::kQ + Sm::kK + Sm::kV);
    float *m_run = reinterpret_cast<float *>(smem + Sm::kQ + Sm::kK + Sm::kV + Sm::kP);
    float *l_run = m_run + QB;
    float *corr = l_run + QB;
    __shared__ int is_last;
    __shared__ float2 freq[D / 2];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid < D / 2) freq[tid] = make_float2(geo.rope_hi[tid], geo.rope_lo[tid]);
    pdl_wait();
    __syncthreads();
    const int split = blockIdx.x, qb = blockIdx.y;
    const int64_t bh = blockIdx.z;
    const int b = int(bh / geo.Hkv), h = int(bh % geo.Hkv);
    const int R = geo.g * geo.C;
    const int r0 = qb * QB;
    const int nrows = R - r0 < QB ? R - r0 : QB;

    const int32_t *sel_bh = VIRT ? a.sel + bh * geo.k : nullptr;
    const WinMap m = attn_winmap(geo, a, VIRT, bh, sel_bh);
    const int64_t W = m.W;
    const int64_t qpos0 = W - geo.C;                       // position of query c = 0
    int64_t kbeg, kend;
    split_range(geo, W, a.nsplit, split, r0, nrows, kKT, kbeg, kend);

    // first tile's loads go out before anything else
    RawKV raw[NITEM];
    auto fetch_tile = [&](int64_t t0) {
#pragma unroll
        for (int u = 0; u < NITEM; ++u) {
            const int x = tid + u * kAttnThreads, key = x / HV, v = x % HV;
            if (t0 + key < kend) raw[u] = src.fetch(geo, m, bh, sel_bh, t0 + key, v);
        }
    };
    if (kbeg < kend) fetch_tile(kbeg);

    for (int r = tid; r < QB; r += kAttnThreads) {
        m_run[r] = -INFINITY;
        l_run[r] = 0.f;
    }
    for (int x = tid; x < QB * (D / 2); x += kAttnThreads) {
        const int rr = x / (D / 2), i = x % (D / 2);
        float lo = 0.f, hi = 0.f;
        if (rr < nrows) query_pair<T, D>(geo, freq, a.q, b, h, r0 + rr, qpos0, i, lo, hi);
        Qs[rr * D + i] = lo;
        Qs[rr * D + i + D / 2] = hi;
    }

    float4 acc[NACC];
#pragma unroll
    for (int u = 0; u < NACC; ++u) acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);

    for (int64_t t0 = kbeg; t0 < kend; t0 += kKT) {
        const int nk = int(kend - t0 < kKT ? kend - t0 : kKT);
        __syncthreads();   // previous tile fully consumed
#pragma unroll
        for (int u = 0; u < NITEM; ++u) {
            const int x = tid + u * kAttnThreads, key = x / HV, v = x % HV;
            float klo[V], khi[V], vlo[V], vhi[V];
            if (key < nk) {
                src.finish(raw[u], t0 + key, v, klo, khi, vlo, vhi);
            } else {
#pragma unroll
                for (int e = 0; e < V; ++e) klo[e] = khi[e] = vlo[e] = vhi[e] = 0.f;
            }
#pragma unroll
            for (int e = 0; e < V; e += 4) {
                const int i = v * V + e;
                *reinterpret_cast<float4 *>(Ks + key * KS + i) =
                    make_float4(klo[e], klo[e + 1], klo[e + 2], klo[e + 3]);
                *reinterpret_cast<float4 *>(Ks + key * KS + i + D / 2) =
                    make_float4(khi[e], khi[e + 1], khi[e + 2], khi[e + 3]);
                *reinterpret_cast<float4 *>(Vs + key * D + i) =
                    make_float4(vlo[e], vlo[e + 1], vlo[e + 2], vlo[e + 3]);
                *reinterpret_cast<float4 *>(Vs + key * D + i + D / 2) =
                    make_float4(vhi[e], vhi[e + 1], vhi[e + 2], vhi[e + 3]);
            }
        }
        if (t0 + kKT < kend) fetch_tile(t0 + kKT);   // next tile in flight during compute
        __syncthreads();

        // logits (log2 domain) for rows rg, rg+4, ...; causal mask per row
        {
            const int key = tid % kKT, rg = tid / kKT;
            float lg[NR];
#pragma unroll
            for (int j = 0; j < NR; ++j) lg[j] = 0.f;
            const float4 *k4 = reinterpret_cast<const float4 *>(Ks + key * KS);
#pragma unroll 4
            for (int d4 = 0; d4 < D4; ++d4) {
                const float4 kv = k4[d4];
#pragma unroll
                for (int j = 0; j < NR; ++j) {
                    const float4 qv = reinterpret_cast<const float4 *>(Qs + (rg + 4 * j) * D)[d4];
                    lg[j] = fmaf(qv.x, kv.x, fmaf(qv.y, kv.y, fmaf(qv.z, kv.z, fmaf(qv.w, kv.w, lg[j]))));
                }
            }
#pragma unroll
            for (int j = 0; j < NR; ++j) {
                const int rr = rg + 4 * j;
                const int c = (r0 + rr) % geo.C;
                const bool ok = rr < nrows && key < nk && t0 + key <= qpos0 + c;
                Ps[rr * kKT + key] = ok ? lg[j] : -INFINITY;
            }
        }
        __syncthreads();
        // online softmax, one warp per row
        for (int rr = warp; rr < nrows; rr += kAttnThreads / 32) {
            const float v0 = Ps[rr * kKT + lane], v1 = Ps[rr * kKT + lane + 32];
            float mx = fmaxf(v0, v1);
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            const float m_old = m_run[rr];
            const float m_new = fmaxf(m_old, mx);
            float cf = 1.f, p0 = 0.f, p1 = 0.f;
            if (m_new != -INFINITY) {
                cf = exp2f(m_old - m_new);
                p0 = exp2f(v0 - m_new);
                p1 = exp2f(v1 - m_new);
            }
            Ps[rr * kKT + lane] = p0;
            Ps[rr * kKT + lane + 32] = p1;
            float sum = p0 + p1;
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
            if (lane == 0) {
                m_run[rr] = m_new;
                l_run[rr] = l_run[rr] * cf + sum;
                corr[rr] = cf;
            }
        }
        __syncthreads();
        // acc = acc * corr + P V, one (row, 4 dims) item per slot
#pragma unroll
        for (int u = 0; u < NACC; ++u) {
            const int x = tid + u * kAttnThreads;
            const int rr = x / D4, d4 = x % D4;
            if (x < QB * D4 && rr < nrows) {
                const float cf = corr[rr];
                float4 z = make_float4(acc[u].x * cf, acc[u].y * cf, acc[u].z * cf, acc[u].w * cf);
                const float *pr = Ps + rr * kKT;
                const float4 *v4 = reinterpret_cast<const float4 *>(Vs) + d4;
#pragma unroll 8
                for (int key = 0; key < nk; ++key) {
                    const float p = pr[key];
                    const float4 vv = v4[key * D4];
                    z.x = fmaf(p, vv.x, z.x);
                    z.y = fmaf(p, vv.y, z.y);
                    z.z = fmaf(p, vv.z, z.z);
                    z.w = fmaf(p, vv.w, z.w);
                }
                acc[u] = z;
            }
        }
    }
    __syncthreads();
    // accumulators to shared memory (the Q tile is free now), then finish
#pragma unroll
    for (int u = 0; u < NACC; ++u) {
        const int x = tid + u * kAttnThreads;
        if (x < QB * D4) reinterpret_cast<float4 *>(Qs)[x] = acc[u];
    }
    __syncthreads();
    split_finish<D, QB>(geo, a, bh, qb, split, nrows, m_run, l_run, Qs, Ks, &is_last);
}

template <typename T, int D, int QB, bool VIRT>
cudaError_t launch_tile(const Geom &geo, const AttnArgs &a, const KvSource<T, D, VIRT> &src,
                        cudaStream_t st)
{
    using Sm = AttnSmem<D, QB>;
    auto kern = attend_tile_kernel<T, D, QB, VIRT>;
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(Sm::kTotal));
    if (e != cudaSuccess) return e;
    dim3 grid(unsigned(a.nsplit), unsigned(a.nqb), unsigned(geo.B * geo.Hkv));
    e = launch_pdl(kern, grid, dim3(kAttnThreads), Sm::kTotal, st, geo, a, src);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <typename T, int D, bool VIRT>
cudaError_t launch_decode_attn(const Geom &geo, const AttnArgs &a, int RP, const void *kc,
                               const void *vc, const void *kcur, const void *vcur,
                               const float *kw, const float *vw, cudaStream_t st)
{
    dim3 grid(unsigned(a.nsplit), 1u, unsigned(geo.B * geo.Hkv));
    const T *k = static_cast<const T *>(kc), *v = static_cast<const T *>(vc);
    const T *kq = static_cast<const T *>(kcur), *vq = static_cast<const T *>(vcur);
#define REATT_DEC(RPV)                                                                         \
    do {                                                                                       \
        cudaError_t e = launch_pdl(attend_decode_kernel<T, D, RPV, VIRT>, grid,                \
                                   dim3(kDecWarps * 32), 0, st, geo, a, k, v, kq, vq, kw, vw); \
        if (e != cudaSuccess) return e;                                                        \
    } while (0)
    switch (RP) {
    case 1: REATT_DEC(1); break;
    case 2: REATT_DEC(2); break;
    case 4: REATT_DEC(4); break;
    default: REATT_DEC(8); break;
    }
#undef REATT_DEC
    return cudaGetLastError();
}

}  // namespace

AttnPlan attn_plan(const Geom &geo, int reserved_sms)
{
    AttnPlan p;
    const int64_t R = int64_t(geo.g) * geo.C;
    const int64_t BH = int64_t(geo.B) * geo.Hkv;
    if (R <= 8) {   // warp kernel: one query block of RP rows
        p.decode = true;
        p.QB = R <= 1 ? 1 : R <= 2 ? 2 : R <= 4 ? 4 : 8;
        p.nqb = 1;
        // one wave: the staged kernel holds one CTA per SM (on the SMs the
        // kernels running beside it leave free)
        int64_t ns = (num_sms() - reserved_sms) / BH;
        const int64_t max_split = (geo.Wmax + kMinSplitKeys - 1) / kMinSplitKeys;
        const int64_t cap = int64_t(kDecWarps - 1) * geo.d;   // combine scratch (floats / QB)
        if (ns > max_split) ns = max_split;
        if (ns > cap) ns = cap;
        p.nsplit = int(ns < 1 ? 1 : ns);
        return p;
    }
    p.decode = false;
    p.QB = 64;
    p.nqb = int((R + p.QB - 1) / p.QB);
    const int64_t base = BH * p.nqb;
    // at least kMinSplitKeys keys per split, about kTargetCtas CTAs in all, and
    // the combine's weights must fit the key tile (nsplit * QB <= kKT * (D+4))
    int64_t max_split = (geo.Wmax + kMinSplitKeys - 1) / kMinSplitKeys;
    const int64_t cap = int64_t(kKT) * (geo.d + 4) / p.QB;
    if (max_split > cap) max_split = cap;
    int64_t ns = 1;
    if (base < kTargetCtas) ns = (kTargetCtas + base - 1) / base;
    if (ns > max_split) ns = max_split;
    p.nsplit = int(ns < 1 ? 1 : ns);
    return p;
}

size_t attend_ws_bytes(const Geom &geo, size_t *ticket_bytes, size_t *ml_off)
{
    const AttnPlan p = attn_plan(geo);
    const size_t nt = size_t(geo.B) * geo.Hkv * p.nqb;
    *ticket_bytes = (nt * sizeof(uint32_t) + 255) / 256 * 256;
    if (p.nsplit == 1) {
        *ml_off = *ticket_bytes;
        return *ticket_bytes;
    }
    const size_t acc = (nt * p.nsplit * p.QB * geo.d * sizeof(float) + 255) / 256 * 256;
    *ml_off = *ticket_bytes + acc;
    return *ticket_bytes + acc + nt * p.nsplit * p.QB * sizeof(float2);
}

size_t rope_table_bytes(const Geom &geo)
{
    return size_t(geo.Wmax) * (geo.d / 2) * sizeof(float2);
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
                          const void *kcur, const void *vcur, const int32_t *sel,
                          const float2 *rope_tab, float *out, void *scratch, void *ws, bool virt,
                          cudaStream_t st, int64_t w_known)
{
    // Early mode: the selecting top-k CTAs run beside the attention, so the
    // split count leaves their SMs free (when they are few).
    int reserved = 0;
    if (w_known >= 0) {
        const int t = topk_selecting_ctas(geo);
        if (t < num_sms() / 2) reserved = t;
    }
    const AttnPlan p = attn_plan(geo, reserved);
    size_t tb = 0, mo = 0;
    attend_ws_bytes(geo, &tb, &mo);
    AttnArgs a;
    a.q = q;
    a.sel = sel;
    a.win_len = win_len;
    a.tab = rope_tab;
    a.out = out;
    a.ticket = static_cast<uint32_t *>(scratch);
    a.part_acc = reinterpret_cast<float *>(static_cast<uint8_t *>(scratch) + tb);
    a.part_ml = reinterpret_cast<float2 *>(static_cast<uint8_t *>(scratch) + mo);
    a.nqb = p.nqb;
    a.nsplit = p.nsplit;
    a.w_known = (p.decode && virt) ? w_known : -1;
#define REATT_ATT(T, D)                                                                        \
    do {                                                                                       \
        if (p.decode) {                                                                        \
            if (virt && decode_tc_eligible(geo))                                               \
                return launch_attend_decode_tc(geo, a, p.QB, kc, vc, kcur, vcur, ws, st);      \
            if (virt)                                                                          \
                return launch_staged_attn<T, D>(geo, a, p.QB, kc, vc, kcur, vcur, ws, st);     \
            return launch_decode_attn<T, D, false>(geo, a, p.QB, nullptr, nullptr, nullptr,    \
                                                   nullptr, kw, vw, st);                       \
        }                                                                                      \
        if (virt) {                                                                            \
            KvSource<T, D, true> s{static_cast<const T *>(kc), static_cast<const T *>(vc),     \
                                   static_cast<const T *>(kcur), static_cast<const T *>(vcur), \
                                   rope_tab};                                                  \
            return launch_tile<T, D, 64, true>(geo, a, s, st);                                 \
        }                                                                                      \
        KvSource<T, D, false> s{kw, vw};                                                       \
        return launch_tile<T, D, 64, false>(geo, a, s, st);                                    \
    } while (0)
    if (geo_is_bf16(geo)) {
        if (geo.d == 128) REATT_ATT(uint16_t, 128);
        REATT_ATT(uint16_t, 64);
    }
    if (geo.d == 128) REATT_ATT(float, 128);
    REATT_ATT(float, 64);
#undef REATT_ATT
}

int64_t decode_window_known(const Geom &geo)
{
    const int64_t keff = geo.k < geo.NS ? geo.k : geo.NS;
    if (keff > 0 && geo.M % geo.S != 0) return -1;   // the ragged last span may be chosen
    return geo.g_end + keff * geo.S + geo.n_loc + geo.C;
}

}  // namespace reatt
