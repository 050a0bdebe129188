// Span scoring on un-rotated keys (decoding pseudocode of the ReAttention
// OpenReview discussion: score = query . key[global:-local]^T; research-map
// summary "Approach": the dot product uses un-positioned keys).
//
//   span_scores[b,h,s] = max_{t in span s, c < C} sum_{j in group(h)} q[b,j,c,:].k[b,h,t,:]
//
// Decode (C == 1): the sum over the group's query heads is folded into one
// fp32 vector qs = sum_j q_j (linearity), so the scan is one HBM pass over
// the middle keys at ~1 flop/byte.  A persistent CTA per SM streams its
// contiguous range of spans through a shared-memory ring filled by
// cp.async.bulk (one elected producer thread, mbarrier completion), while 8
// consumer warps form the dot products on CUDA cores and fold them into span
// maxima.  No per-token score is written anywhere.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace reatt {

static int g_num_sms[64];

int num_sms()
{
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) dev = 0;
    if (g_num_sms[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        g_num_sms[dev] = n;
    }
    return g_num_sms[dev];
}


namespace {

// Ring shape (compile-time; the defaults are the measured best on B200).
#ifndef REATT_SCAN_CWARPS
#define REATT_SCAN_CWARPS 16     // consumer warps per CTA
#endif
#ifndef REATT_SCAN_RING_KB
#define REATT_SCAN_RING_KB 192   // shared-memory ring per CTA
#endif
#ifndef REATT_SCAN_CPS
#define REATT_SCAN_CPS 1         // CTAs per SM
#endif
#ifndef REATT_SCAN_SUB
#define REATT_SCAN_SUB 2         // 32-token passes per ring stage
#endif
constexpr int kConsumerWarps = REATT_SCAN_CWARPS;
constexpr int kConsumers = 32 * kConsumerWarps;
constexpr int kScanThreads = kConsumers + 32;       // + one producer warp
constexpr int kRingBytes = REATT_SCAN_RING_KB * 1024;
constexpr int kCtasPerSm = REATT_SCAN_CPS;
constexpr int kSub = REATT_SCAN_SUB;
constexpr int kMaxItemSpans = 4096 / kCtasPerSm;
constexpr int kPassTok = 32;                          // tokens per consumer pass
constexpr int kStageTok = kPassTok * kSub;            // tokens per ring stage

constexpr int gcd(int a, int b) { return b == 0 ? a : gcd(b, a % b); }
// Largest warp count (halving from cw) whose fixed stage map leaves >= 2 stages.
constexpr int eff_warps(int stages_raw, int cw)
{
    return (cw <= 1 || stages_raw / (cw / gcd(cw, kSub)) * (cw / gcd(cw, kSub)) >= 2)
               ? cw
               : eff_warps(stages_raw, cw / 2);
}

template <typename T, int D>
struct ScanShape {
    static constexpr int kRowBytes = D * Elem<T>::kBytes;
    static constexpr int kLpt = kRowBytes / 16;       // lanes per token row
    static constexpr int kNg = 32 / kLpt;             // rows per load round
    static constexpr int kVec = Elem<T>::kVec;        // elements per lane load
    static constexpr int kPassBytes = kPassTok * kRowBytes;
    static constexpr int kStageBytes = kStageTok * kRowBytes;
    // Pass slot (stage, j) of ring use u is consumed by warp (st*kSub + j) %
    // kConsumerWarps with st = stage + u*kStages.  The stage count is a
    // multiple of kWarpPeriod so that warp is the same for every use: each
    // full barrier then has a single waiter that takes its phases in order,
    // and a parity wait can never be two phases ahead (where it would pass at
    // once on the stale parity).
    // (Wide rows with many warps: fewer warps consume, the rest idle.)
    static constexpr int kCW = eff_warps(kRingBytes / kStageBytes, kConsumerWarps);
    static constexpr int kWarpPeriod = kCW / gcd(kCW, kSub);
    static constexpr int kStages = kRingBytes / kStageBytes / kWarpPeriod * kWarpPeriod;
    static constexpr size_t kSmem = size_t(kRingBytes) + 2 * kStages * sizeof(uint64_t) +
                                    kMaxItemSpans * sizeof(uint32_t) + D * sizeof(float) + 16;
    static_assert(kLpt * kNg == 32, "row must split evenly over a warp");
    static_assert(kStages >= 2, "ring too small");
    static_assert((kStages * kSub) % kCW == 0, "stage -> warp map must be fixed");
};

// Work of one CTA: global span ids [gs, ge) over the flattened (b*Hkv+h, span)
// space, cut into items that stay inside one head and hold <= kMaxItemSpans.
struct Item {
    int64_t bh, s0, s1, t_begin, t_end;
};
__device__ __forceinline__ bool next_item(const Geom &geo, int64_t &gs, int64_t ge, Item &it)
{
    if (gs >= ge)
        return false;
    it.bh = gs / geo.NS;
    it.s0 = gs % geo.NS;
    int64_t lim = geo.NS - it.s0;
    if (ge - gs < lim) lim = ge - gs;
    if (lim > kMaxItemSpans) lim = kMaxItemSpans;
    it.s1 = it.s0 + lim;
    it.t_begin = geo.G + it.s0 * geo.S;
    it.t_end = geo.G + it.s1 * geo.S;
    if (it.t_end > geo.G + geo.M) it.t_end = geo.G + geo.M;
    gs += lim;
    return true;
}

template <typename T, int D>
__global__ void __launch_bounds__(kScanThreads, kCtasPerSm)
scan_decode_kernel(Geom geo, const T *__restrict__ q, const T *__restrict__ kc,
                   float *__restrict__ scores, void *ws, int64_t spans_per_cta,
                   float2 *__restrict__ rope_tab)
{
    using Sh = ScanShape<T, D>;
    extern __shared__ __align__(128) uint8_t smem[];
    uint8_t *ring = smem;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + kRingBytes);
    uint64_t *empty = full + Sh::kStages;
    uint32_t *smax = reinterpret_cast<uint32_t *>(empty + Sh::kStages);
    float *qs = reinterpret_cast<float *>(smax + kMaxItemSpans);
    __shared__ int abort_flag;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t total = int64_t(geo.B) * geo.Hkv * geo.NS;
    const int64_t cta_begin = int64_t(blockIdx.x) * spans_per_cta;
    int64_t cta_end = cta_begin + spans_per_cta;
    if (cta_end > total) cta_end = total;

    pdl_trigger();   // the top-k may launch now; it waits for this grid to finish
    if (tid == 0) {
        abort_flag = 0;
        for (int s = 0; s < Sh::kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kSub);   // one release per pass slot
        }
        mbar_init_fence();
    }
    __syncthreads();

    if (warp == kConsumerWarps) {
        // ------------------------------------------------ producer (one thread)
        if (lane == 0) {
            // Stage index and use parity advance incrementally (no divisions in
            // the issue loop: one thread issues every copy of the CTA).
            const uint64_t pol = l2_evict_first_policy();
            int stage = 0;
            uint32_t phase = 0;         // parity of the current use of `stage`
            bool wrapped = false;       // every stage has been used once
            int64_t gs = cta_begin;
            Item it;
            bool stop = false;
            while (!stop && next_item(geo, gs, cta_end, it)) {
                const T *src = kc + (it.bh * geo.Ts + it.t_begin) * D;
                for (int64_t t = it.t_begin; t < it.t_end; t += kStageTok, src += kStageTok * D) {
                    if (wrapped) {
                        if (*(volatile int *)&abort_flag ||
                            !mbar_wait_bounded(&empty[stage], phase ^ 1u, kWaitLimitNs)) {
                            report_status(ws, REATT_ETIMEOUT);
                            *(volatile int *)&abort_flag = 1;
                            stop = true;
                            break;
                        }
                    }
                    const int64_t left = it.t_end - t;
                    const uint32_t bytes =
                        uint32_t(left < kStageTok ? left : kStageTok) * Sh::kRowBytes;
                    mbar_arrive_expect_tx(&full[stage], bytes);
                    bulk_load(ring + stage * Sh::kStageBytes, src, bytes, &full[stage], pol);
                    if (++stage == Sh::kStages) {
                        stage = 0;
                        phase ^= 1u;
                        wrapped = true;
                    }
                }
            }
            // Drain: every issued copy has landed before the CTA may exit.  The
            // last use of each stage (the most recent kStages issues) is waited
            // on with that use's parity.
            for (int k2 = 0; k2 < Sh::kStages; ++k2) {
                if (--stage < 0) {
                    stage = Sh::kStages - 1;
                    if (!wrapped) break;      // fewer than kStages issues in all
                    phase ^= 1u;
                }
                if (!mbar_wait_bounded(&full[stage], phase, kWaitLimitNs))
                    report_status(ws, REATT_ETIMEOUT);
            }
        }
        return;
    }

    // ---------------------------------------------------- consumers
    if (rope_tab) {
        // The step's RoPE cos/sin table (tab[p*(D/2) + i] for window positions
        // p < Wmax), written while the first ring stages are in flight so the
        // attention can use it without waiting for the selection.  The grid
        // stride is a multiple of D/2, so each thread keeps one frequency.
        constexpr int kHalf = D / 2;
        static_assert(kConsumers % kHalf == 0, "one frequency per consumer thread");
        const float fhi = geo.rope_hi[tid % kHalf], flo = geo.rope_lo[tid % kHalf];
        const int64_t n = geo.Wmax * kHalf;
        for (int64_t x = int64_t(blockIdx.x) * kConsumers + tid; x < n;
             x += int64_t(gridDim.x) * kConsumers) {
            float c, s;
            rope_cs(x / kHalf, fhi, flo, c, s);
            rope_tab[x] = make_float2(c, s);
        }
    }
    const int gq = lane / Sh::kLpt, p = lane % Sh::kLpt;
    int stage = 0;
    uint32_t phase = 0;
    int64_t gs = cta_begin;
    Item it;
    while (next_item(geo, gs, cta_end, it)) {
        // fp32 sum of the group's query vectors (query position 0)
        if (tid < D) {
            const int b = int(it.bh / geo.Hkv), h = int(it.bh % geo.Hkv);
            const T *qb = q + ((int64_t(b) * geo.Hq + int64_t(h) * geo.g) * geo.C) * D;
            float a = 0.f;
            for (int j = 0; j < geo.g; ++j)
                a += Elem<T>::one(qb, int64_t(j) * geo.C * D + tid);
            qs[tid] = a;
        }
        const int nsp = int(it.s1 - it.s0);
        for (int s = tid; s < nsp; s += kConsumers)
            smax[s] = 0u;
        named_sync(1, kConsumers);
        float qv[Sh::kVec];
#pragma unroll
        for (int e = 0; e < Sh::kVec; ++e)
            qv[e] = qs[p * Sh::kVec + e];

        for (int64_t t = it.t_begin; t < it.t_end; t += kStageTok) {
            const uint32_t par = phase;
            const int st_now = stage;
            if (++stage == Sh::kStages) {
                stage = 0;
                phase ^= 1u;
            }
            // fixed map: slot j of ring stage s belongs to warp (s*kSub + j) % kCW
#pragma unroll
            for (int j = 0; j < kSub; ++j) {
                if ((st_now * kSub + j) % Sh::kCW != warp)
                    continue;
                // warp-uniform abort / wait outcome (the shuffles below need all lanes)
                if (__any_sync(0xffffffffu, *(volatile int *)&abort_flag != 0))
                    continue;
                const bool ok = mbar_wait_bounded(&full[st_now], par, kWaitLimitNs);
                if (!__all_sync(0xffffffffu, ok)) {
                    if (lane == 0) {
                        report_status(ws, REATT_ETIMEOUT);
                        *(volatile int *)&abort_flag = 1;
                    }
                    continue;
                }
                const int64_t tp = t + int64_t(j) * kPassTok;
                int ntok = int(it.t_end - tp);
                if (ntok > kPassTok) ntok = kPassTok;
                if (ntok <= 0) {   // empty slot of a short last stage: release only
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&empty[st_now]);
                    continue;
                }
                const uint8_t *sb = ring + st_now * Sh::kStageBytes + j * Sh::kPassBytes;
                float acc[Sh::kLpt];
#pragma unroll
                for (int r = 0; r < Sh::kLpt; ++r) {
                    const uint4 raw = *reinterpret_cast<const uint4 *>(
                        sb + (r * Sh::kNg + gq) * Sh::kRowBytes + p * 16);
                    float e[Sh::kVec];
                    Elem<T>::unpack(raw, e);
                    float a = 0.f;
#pragma unroll
                    for (int i = 0; i < Sh::kVec; ++i)
                        a = fmaf(qv[i], e[i], a);
                    acc[r] = a;
                }
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&empty[st_now]);   // the pass is in registers: hand it back

                // Transposed reduction over the kLpt lanes of a row group: after
                // it lane (gq, p) holds the full dot product of row p*kNg + gq.
#pragma unroll
                for (int o = Sh::kLpt / 2; o >= 1; o >>= 1) {
                    const bool upper = (p & o) != 0;
#pragma unroll
                    for (int i = 0; i < o; ++i) {
                        const float send = upper ? acc[i] : acc[i + o];
                        const float keep = upper ? acc[i + o] : acc[i];
                        acc[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
                    }
                }
                const int row = p * Sh::kNg + gq;
                const bool valid = row < ntok;
                const int moff = int(tp - geo.G);                // middle offset of row 0
                const int sfirst = moff / geo.S, slast = (moff + ntok - 1) / geo.S;
                if (sfirst == slast) {
                    float m = valid ? acc[0] : -INFINITY;
#pragma unroll
                    for (int o = 16; o >= 1; o >>= 1)
                        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
                    if (lane == 0)
                        atomicMax(&smax[sfirst - int(it.s0)], order_code(m));
                } else if (valid) {
                    atomicMax(&smax[(moff + row) / geo.S - int(it.s0)], order_code(acc[0]));
                }
            }
        }
        named_sync(1, kConsumers);
        float *dst = scores + it.bh * geo.NS + it.s0;
        for (int s = tid; s < nsp; s += kConsumers)
            dst[s] = order_decode(smax[s]);
        named_sync(1, kConsumers);
    }
}

// ---------------------------------------------------------------- C > 1
// fp32 sum of each KV head's group of query vectors: qsum[bh][c][:].
template <typename T, int D>
__global__ void qsum_kernel(Geom geo, const T *__restrict__ q, float *__restrict__ qsum)
{
    const int64_t rows = int64_t(geo.B) * geo.Hkv * geo.C;
    for (int64_t x = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; x < rows * D;
         x += int64_t(gridDim.x) * blockDim.x) {
        const int64_t i = x % D, row = x / D;
        const int64_t c = row % geo.C, bh = row / geo.C;
        const int64_t b = bh / geo.Hkv, h = bh % geo.Hkv;
        float a = 0.f;
        for (int j = 0; j < geo.g; ++j)
            a += Elem<T>::one(q, ((b * geo.Hq + h * geo.g + j) * geo.C + c) * D + i);
        qsum[x] = a;
    }
}

// Generic multi-query scan on CUDA cores: a CTA owns whole spans (SPB of
// them, SPB*S <= 64 tokens when S <= 64), streams their tokens in tiles of
// 64 rows through shared memory and takes, per token, the max over all C
// summed queries.
constexpr int kMqTile = 64;
constexpr int kMqQ = 16;
template <typename T, int D>
__global__ void __launch_bounds__(256)
scan_multi_kernel(Geom geo, const float *__restrict__ qsum, const T *__restrict__ kc,
                  float *__restrict__ scores, int spb)
{
    __shared__ float Kt[kMqTile][D + 1];
    __shared__ float Qs[kMqQ][D];
    __shared__ float part[4][kMqTile];
    __shared__ uint32_t smax[kMqTile];
    const int tid = threadIdx.x;
    const int64_t bh = blockIdx.y;
    const int64_t s0 = int64_t(blockIdx.x) * spb;
    int64_t s1 = s0 + spb;
    if (s1 > geo.NS) s1 = geo.NS;
    if (s0 >= s1) return;
    const int64_t t_begin = geo.G + s0 * geo.S;
    int64_t t_end = geo.G + s1 * geo.S;
    if (t_end > geo.G + geo.M) t_end = geo.G + geo.M;
    for (int s = tid; s < kMqTile; s += 256) smax[s] = 0u;
    const float *qb = qsum + bh * int64_t(geo.C) * D;
    const T *kb = kc + bh * geo.Ts * D;

    for (int64_t t0 = t_begin; t0 < t_end; t0 += kMqTile) {
        const int ntok = int(t_end - t0 < kMqTile ? t_end - t0 : kMqTile);
        __syncthreads();
        for (int x = tid; x < kMqTile * D; x += 256) {
            const int r = x / D, i = x % D;
            Kt[r][i] = r < ntok ? Elem<T>::one(kb, (t0 + r) * D + i) : 0.f;
        }
        const int r = tid % kMqTile, quarter = tid / kMqTile;
        float best = -INFINITY;
        for (int c0 = 0; c0 < geo.C; c0 += kMqQ) {
            const int nq = geo.C - c0 < kMqQ ? geo.C - c0 : kMqQ;
            __syncthreads();
            for (int x = tid; x < kMqQ * D; x += 256) {
                const int c = x / D;
                Qs[c][x % D] = c < nq ? qb[int64_t(c0 + c) * D + x % D] : 0.f;
            }
            __syncthreads();
            for (int c = quarter; c < nq; c += 4) {
                float a = 0.f;
#pragma unroll 8
                for (int i = 0; i < D; ++i)
                    a = fmaf(Qs[c][i], Kt[r][i], a);
                best = fmaxf(best, a);
            }
        }
        part[quarter][r] = best;
        __syncthreads();
        if (tid < ntok) {
            const float m = fmaxf(fmaxf(part[0][tid], part[1][tid]), fmaxf(part[2][tid], part[3][tid]));
            const int sp = int((t0 + tid - geo.G) / geo.S - s0);
            atomicMax(&smax[sp], order_code(m));
        }
    }
    __syncthreads();
    for (int s = tid; s < int(s1 - s0); s += 256)
        scores[bh * geo.NS + s0 + s] = order_decode(smax[s]);
}

template <typename T, int D>
cudaError_t launch_decode(const Geom &geo, const void *q, const void *kc, float *scores, void *ws,
                          float2 *rope_tab, cudaStream_t st)
{
    using Sh = ScanShape<T, D>;
    const int64_t total = int64_t(geo.B) * geo.Hkv * geo.NS;
    int grid = num_sms() * kCtasPerSm;
    if (total < grid) grid = int(total);
    const int64_t per = (total + grid - 1) / grid;
    grid = int((total + per - 1) / per);
    cudaError_t e = cudaFuncSetAttribute(scan_decode_kernel<T, D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         int(Sh::kSmem));
    if (e != cudaSuccess) return e;
    scan_decode_kernel<T, D><<<grid, kScanThreads, Sh::kSmem, st>>>(
        geo, static_cast<const T *>(q), static_cast<const T *>(kc), scores, ws, per, rope_tab);
    return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_multi(const Geom &geo, const void *q, const void *kc, float *scores,
                         float *qsum_ws, cudaStream_t st)
{
    const int64_t n = int64_t(geo.B) * geo.Hkv * geo.C * D;
    int blocks = int((n + 255) / 256);
    if (blocks > 4096) blocks = 4096;
    qsum_kernel<T, D><<<blocks, 256, 0, st>>>(geo, static_cast<const T *>(q), qsum_ws);
    const int spb = geo.S >= kMqTile ? 1 : kMqTile / geo.S;
    dim3 grid(unsigned((geo.NS + spb - 1) / spb), unsigned(geo.B * geo.Hkv));
    scan_multi_kernel<T, D><<<grid, 256, 0, st>>>(geo, qsum_ws, static_cast<const T *>(kc), scores,
                                                  spb);
    return cudaGetLastError();
}

}  // namespace

size_t score_spans_ws_bytes(const Geom &geo)
{
    if (geo.C <= 1) return 0;
    const size_t qsum = size_t(geo.B) * geo.Hkv * geo.C * geo.d * sizeof(float);
    const size_t terms = prefill_tc_ws_bytes(geo);
    return qsum > terms ? qsum : terms;
}

cudaError_t launch_score_spans(const Geom &geo, const void *q, const void *kc, float *scores,
                               void *ws, void *scratch, float2 *rope_tab, cudaStream_t st,
                               bool allow_tc, bool *codes_left)
{
    if (codes_left) *codes_left = false;
    if (int64_t(geo.B) * geo.Hkv * geo.NS == 0) return cudaSuccess;
    if (geo.C == 1) {
        if (geo.d == 128)
            return geo_is_bf16(geo)
                       ? launch_decode<uint16_t, 128>(geo, q, kc, scores, ws, rope_tab, st)
                       : launch_decode<float, 128>(geo, q, kc, scores, ws, rope_tab, st);
        return geo_is_bf16(geo) ? launch_decode<uint16_t, 64>(geo, q, kc, scores, ws, rope_tab, st)
                                : launch_decode<float, 64>(geo, q, kc, scores, ws, rope_tab, st);
    }
    if (rope_tab) return cudaErrorInvalidValue;   // only the decode scan writes the table
    if (allow_tc && prefill_tc_eligible(geo))   // tensor-core contraction (tcgen05 / TMEM)
        return launch_prefill_tc(geo, q, kc, scores, ws, scratch, st, codes_left);
    float *qsum = static_cast<float *>(scratch);
    if (geo.d == 128)
        return geo_is_bf16(geo) ? launch_multi<uint16_t, 128>(geo, q, kc, scores, qsum, st)
                                : launch_multi<float, 128>(geo, q, kc, scores, qsum, st);
    return geo_is_bf16(geo) ? launch_multi<uint16_t, 64>(geo, q, kc, scores, qsum, st)
                            : launch_multi<float, 64>(geo, q, kc, scores, qsum, st);
}

}  // namespace reatt
