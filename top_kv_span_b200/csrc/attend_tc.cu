// Chunked-prefill attention over the window on the tensor cores (tcgen05 + TMEM).
//
// The window of one (batch, KV head) and the chunk's g*C query rows form a
// causal attention (ReAttention OpenReview discussion, "Prefilling Phase":
// flash_attention(query, key_recall, value_recall); research-map summary
// "Approach": RoPE applied after concatenation, window row p at position p,
// query c at W-C+c).  The rotated operands of the logits are split into bf16
// hi + lo to keep fp32-level accuracy with bf16 tensor-core operands:
//   S = Qh.Kh^T + Qh.Kl^T + Ql.Kh^T   (dropped Ql.Kl^T is ~2^-18 relative)
// and the probabilities P = exp2(S - m) <= 2^8 meet V in fp16 (11-bit
// significand, V converted from bf16):  O += P.V.
//
// prefill_prep_kernel writes, per KV head, the rotated+scaled query rows
// (hi/lo), the rotated window keys (hi/lo) and the window values transposed
// (fp16), from the un-rotated cache through the selection (the window is
// never materialised in fp32).  attend_prefill_tc_kernel then runs, per
// 128-row query block (TMEM lanes = query rows):
//   warp 0   TMA producer: 128-key tiles of K (hi, lo) and V^T, each in a
//            2-stage ring, each issued as soon as its stage is free (128B
//            swizzle, no multicast)
//   warp 1   TMEM allocation; one thread issues S(j) (M128 x N128 MMAs) into
//            one of two TMEM S tiles as soon as K(j) has landed and the tile
//            is free (its previous P.V has completed)
//   warp 10  one thread issues O += P(j).V(j) into the TMEM O accumulator
//            as soon as P(j) is written (a thread of its own: tcgen05.mma
//            issue stalls while the pipe is full, and a P.V must not wait
//            behind an S).  Both products read their A operand (the query
//            terms, P) from TMEM, so only K and V^T come from shared memory
//   warps 2-9 softmax: two warps per TMEM lane group, one per 64-column half
//            of the S tile; first each stores its rows' query term (hi or
//            lo) into TMEM.  A thread owns one query row's half: it reads its
//            64 S values from TMEM, masks (causal, window end), trades its
//            half-row max with the partner warp (a named barrier per pair),
//            keeps a running reference max that moves (and rescales its half
//            of O in TMEM) only when the row max grows by more than 2^8,
//            stores its half of P as fp16 pairs over the first half of the
//            same S tile, and finally divides its half of O by the row sum.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"

namespace reatt {

namespace {

using namespace tc;

constexpr int kFaSoftWarps = 8;          // two per TMEM lane group (warps 2..9)
constexpr int kFaPvWarp = 2 + kFaSoftWarps;   // issues the P.V products
constexpr int kFaThreads = (3 + kFaSoftWarps) * 32;
constexpr int kQRows = 128;   // query rows per CTA (TMEM lanes)
constexpr int kKeyTile = 128;  // keys per S tile (S columns, the N of its MMAs)
constexpr float kRescaleLog2 = 8.f;

struct WinMapTc {
    int64_t g_end, loc_begin, n_loc, nsel_rows, W;
};

__device__ __forceinline__ WinMapTc winmap_tc(const Geom &geo, const int32_t *sel_bh)
{
    WinMapTc m;
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

// Window row p -> element offset of its K/V row (bit 62: current token).
__device__ __forceinline__ int64_t row_src_tc(const Geom &geo, const WinMapTc &m,
                                              const int32_t *sel_bh, int64_t bh, int64_t p, int D)
{
    if (p < m.g_end) return (bh * geo.Ts + p) * D;
    p -= m.g_end;
    if (p < m.nsel_rows) {
        const int64_t j = p / geo.S, off = p - j * geo.S;
        int64_t sp = sel_bh[j];
        sp = sp < 0 ? 0 : (sp >= geo.NS ? geo.NS - 1 : sp);
        int64_t row = geo.G + sp * geo.S + off;
        if (row >= geo.T) row = geo.T - 1;
        return (bh * geo.Ts + row) * D;
    }
    p -= m.nsel_rows;
    if (p < m.n_loc) return (bh * geo.Ts + m.loc_begin + p) * D;
    return (int64_t(1) << 62) | ((bh * geo.C + (p - m.n_loc)) * D);
}

// 2^x on the special-function unit (ex2.approx.ftz: relative error ~2^-22;
// 2^-inf = 0), for the softmax numerators.
__device__ __forceinline__ float ex2_approx(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Operand buffers of one call, bf16, per KV head bh:
//   qh/ql [BH][Rp][D]  rotated queries x log2(e)/sqrt(d), rows >= R zero
//   kh/kl [BH][Wp][D]  rotated window keys, rows >= W zero
//   vt    [BH][D][Wp]  window values transposed, columns >= W zero
struct PrepOut {
    __nv_bfloat16 *qh, *ql, *kh, *kl;
    __half *vt;   // fp16: the P.V products take fp16 P
    int Rp, Wp;
};

constexpr int kPrepRows = 64;

// 8 floats -> 8 bf16 (16 bytes)
__device__ __forceinline__ uint4 pack8_bf16(const float (&v)[8])
{
    uint4 w;
    uint32_t *u = reinterpret_cast<uint32_t *>(&w);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const __nv_bfloat162 t = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
        u[e] = *reinterpret_cast<const uint32_t *>(&t);
    }
    return w;
}
__device__ __forceinline__ void unpack8_bf16(const uint4 &w, float (&v)[8])
{
    Elem<uint16_t>::unpack(w, v);
}

// One thread item = 8 consecutive RoPE pairs (dims i0..i0+7 and their
// partners at +D/2) of one row: 16-byte loads and stores throughout; the
// cos/sin come from the step's table (the query positions W-C+c are inside it).
template <int D>
__global__ void __launch_bounds__(256)
prefill_prep_kernel(Geom geo, const uint16_t *__restrict__ q, const uint16_t *__restrict__ kc,
                    const uint16_t *__restrict__ vc, const uint16_t *__restrict__ kcur,
                    const uint16_t *__restrict__ vcur, const int32_t *__restrict__ sel,
                    const float2 *__restrict__ tab, PrepOut po)
{
    constexpr int NCH = D / 2 / 8;   // 8-pair chunks per row
    __shared__ float vs[kPrepRows][D + 1];
    pdl_wait();   // the selection and the RoPE table come from the top-k launch
    const int64_t bh = blockIdx.y;
    const int b = int(bh / geo.Hkv), h = int(bh % geo.Hkv);
    const int32_t *sel_bh = sel + bh * geo.k;
    const WinMapTc m = winmap_tc(geo, sel_bh);
    const int nkb = po.Wp / kPrepRows;
    auto rot8 = [&](const uint4 &xw, const uint4 &yw, const float2 *cs, float (&lo)[8],
                    float (&hi)[8], float scale) {
        float x[8], y[8];
        unpack8_bf16(xw, x);
        unpack8_bf16(yw, y);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            lo[e] = (x[e] * cs[e].x - y[e] * cs[e].y) * scale;
            hi[e] = (y[e] * cs[e].x + x[e] * cs[e].y) * scale;
        }
    };
    auto split_store = [&](const float (&v)[8], __nv_bfloat16 *dh, __nv_bfloat16 *dl) {
        float hv[8], lv[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            hv[e] = __bfloat162float(__float2bfloat16_rn(v[e]));
            lv[e] = v[e] - hv[e];
        }
        *reinterpret_cast<uint4 *>(dh) = pack8_bf16(hv);
        *reinterpret_cast<uint4 *>(dl) = pack8_bf16(lv);
    };
    if (int(blockIdx.x) < nkb) {
        // ---- 64 window rows: rotated K hi/lo, V transposed
        const int64_t p0 = int64_t(blockIdx.x) * kPrepRows;
        for (int x = threadIdx.x; x < kPrepRows * NCH; x += blockDim.x) {
            const int r = x / NCH, i0 = (x % NCH) * 8;
            const int64_t p = p0 + r;
            float k0[8], k1[8], v0[8], v1[8];
            if (p < m.W) {
                const int64_t off = row_src_tc(geo, m, sel_bh, bh, p, D);
                const bool cur = (off >> 62) != 0;
                const int64_t o = off & ~(int64_t(1) << 62);
                const uint16_t *kr = (cur ? kcur : kc) + o, *vr = (cur ? vcur : vc) + o;
                const uint4 kx = *reinterpret_cast<const uint4 *>(kr + i0);
                const uint4 ky = *reinterpret_cast<const uint4 *>(kr + D / 2 + i0);
                unpack8_bf16(*reinterpret_cast<const uint4 *>(vr + i0), v0);
                unpack8_bf16(*reinterpret_cast<const uint4 *>(vr + D / 2 + i0), v1);
                float2 cs[8];
                const float4 *tr = reinterpret_cast<const float4 *>(tab + p * (D / 2) + i0);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float4 t4 = tr[e];
                    cs[2 * e] = make_float2(t4.x, t4.y);
                    cs[2 * e + 1] = make_float2(t4.z, t4.w);
                }
                rot8(kx, ky, cs, k0, k1, 1.f);
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) k0[e] = k1[e] = v0[e] = v1[e] = 0.f;
            }
            const int64_t kb = (bh * po.Wp + p) * D;
            split_store(k0, po.kh + kb + i0, po.kl + kb + i0);
            split_store(k1, po.kh + kb + D / 2 + i0, po.kl + kb + D / 2 + i0);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                vs[r][i0 + e] = v0[e];
                vs[r][D / 2 + i0 + e] = v1[e];
            }
        }
        __syncthreads();
        // V^T: 8 consecutive window rows of one dim per 16-byte store
        for (int x = threadIdx.x; x < D * (kPrepRows / 8); x += blockDim.x) {
            const int i = x / (kPrepRows / 8), r0 = (x % (kPrepRows / 8)) * 8;
            uint4 w;
            uint32_t *u = reinterpret_cast<uint32_t *>(&w);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const __half2 t = __floats2half2_rn(vs[r0 + 2 * e][i], vs[r0 + 2 * e + 1][i]);
                u[e] = *reinterpret_cast<const uint32_t *>(&t);
            }
            *reinterpret_cast<uint4 *>(po.vt + (bh * D + i) * po.Wp + p0 + r0) = w;
        }
    } else {
        // ---- 64 query rows: rotated at W-C+c, scaled, hi/lo
        const int64_t r0 = int64_t(int(blockIdx.x) - nkb) * kPrepRows;
        const int R = geo.g * geo.C;
        const float qscale = 1.4426950408889634f * rsqrtf(float(D));
        const int64_t qpos0 = m.W - geo.C;
        for (int x = threadIdx.x; x < kPrepRows * NCH; x += blockDim.x) {
            const int rr = x / NCH, i0 = (x % NCH) * 8;
            const int64_t r = r0 + rr;
            float lo[8], hi[8];
            if (r < R) {
                const int j = h * geo.g + int(r / geo.C), c = int(r % geo.C);
                const uint16_t *qr = q + ((int64_t(b) * geo.Hq + j) * geo.C + c) * D;
                float2 cs[8];
                const float4 *tr = reinterpret_cast<const float4 *>(tab + (qpos0 + c) * (D / 2) + i0);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float4 t4 = tr[e];
                    cs[2 * e] = make_float2(t4.x, t4.y);
                    cs[2 * e + 1] = make_float2(t4.z, t4.w);
                }
                rot8(*reinterpret_cast<const uint4 *>(qr + i0),
                     *reinterpret_cast<const uint4 *>(qr + D / 2 + i0), cs, lo, hi, qscale);
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) lo[e] = hi[e] = 0.f;
            }
            const int64_t qb = (bh * po.Rp + r) * D;
            split_store(lo, po.qh + qb + i0, po.ql + qb + i0);
            split_store(hi, po.qh + qb + D / 2 + i0, po.ql + qb + D / 2 + i0);
        }
    }
}

struct FaArgs {
    float *out;
    const int32_t *sel;
    const __nv_bfloat16 *qh, *ql;   // [BH][Rp][D] query operand terms
    int Rp, Wp;
};

constexpr int kKStages = 2;   // K tiles (hi | lo) in flight
constexpr int kVStages = 2;   // V^T tiles in flight

// Shared-memory plan (1024-byte aligned): K stages (hi | lo) | V^T stages |
// barriers.  The query terms and P live in TMEM.
template <int D>
struct FaSmem {
    static constexpr int NBOX = D / 64;
    static constexpr int kK = NBOX * kKeyTile * 128;     // one of Kh / Kl
    static constexpr int kV = D * kKeyTile * 2;          // V^T tile: kKeyTile/64 boxes of D rows x 64 keys
    static constexpr int oK = 0, oV = kKStages * 2 * kK, oBar = oV + kVStages * kV;
    static constexpr size_t kBytes = size_t(oBar) + 32 * 8 + 1024;
};

// TMEM columns of one CTA (128 lanes = the query rows): two S tiles, the O
// accumulator and the query terms (A operand of S: lane = row, two bf16 of
// the head width per column).  P(j) (A operand of P.V, two fp16 keys per
// column) overwrites the first half of its own S tile once both softmax warps
// of the lane group have read S(j); S(j+2) goes into that tile only after
// P(j).V(j) has completed.
constexpr uint32_t kSCol = 0, kOCol = 2 * kKeyTile, kQCol = kOCol + 128, kTmemCols = 512;

template <int D>
__global__ void __launch_bounds__(kFaThreads, 1)
attend_prefill_tc_kernel(const __grid_constant__ CUtensorMap khmap,
                         const __grid_constant__ CUtensorMap klmap,
                         const __grid_constant__ CUtensorMap vtmap, Geom geo, FaArgs fa, void *ws)
{
    using Sm = FaSmem<D>;
    constexpr int NBOX = Sm::NBOX;
    constexpr int KS = D / 16;                 // k-steps of S over the head width
    constexpr int PS = kKeyTile / 16;          // k-steps of P.V over a key tile
    static_assert(kOCol + D <= kQCol && kQCol + D <= kTmemCols, "TMEM plan");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Sm::oBar);
    uint64_t *qfull = bars, *kfull = bars + 1, *kempty = kfull + kKStages,
             *vfull = kempty + kKStages, *vempty = vfull + kVStages, *sfull = vempty + kVStages,
             *pfull = sfull + 2, *pvdone = pfull + 2, *done = pvdone + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(done + 2);
    __shared__ int abort_flag;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        abort_flag = 0;
        mbar_init(qfull, kFaSoftWarps);   // query terms stored in TMEM (one arrival per softmax warp)
        for (int s = 0; s < kKStages; ++s) {
            mbar_init(&kfull[s], 1);
            mbar_init(&kempty[s], 1);
        }
        for (int s = 0; s < kVStages; ++s) {
            mbar_init(&vfull[s], 1);
            mbar_init(&vempty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&sfull[s], 1);
            mbar_init(&pfull[s], kFaSoftWarps);   // P in tile s written (one arrival per softmax warp)
            mbar_init(&pvdone[s], 1);    // P.V of tile s done: tile s free again
        }
        mbar_init(&done[0], 1);   // all S products complete
        mbar_init(&done[1], 1);   // all P.V products complete
        mbar_init_fence();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    pdl_wait();   // operands come from the prep launch
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const int qb = blockIdx.x;
    const int64_t bh = blockIdx.y;
    const int b = int(bh / geo.Hkv), h = int(bh % geo.Hkv);
    const int R = geo.g * geo.C;
    const int r0 = qb * kQRows;
    const int nrows = R - r0 < kQRows ? R - r0 : kQRows;
    const WinMapTc m = winmap_tc(geo, fa.sel + bh * geo.k);
    const int64_t W = m.W, qpos0 = W - geo.C;
    const int last_row = r0 + nrows - 1;
    const int c_max = (last_row / geo.C == r0 / geo.C) ? last_row % geo.C : geo.C - 1;
    int64_t kend = qpos0 + c_max + 1;
    if (kend > W) kend = W;
    const int nt = int((kend + kKeyTile - 1) / kKeyTile);

    auto fail = [&]() {
        report_status(ws, REATT_ETIMEOUT);
        *(volatile int *)&abort_flag = 1;
    };
    auto aborted = [&]() { return *(volatile int *)&abort_flag != 0; };

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        // K and V^T tiles go through separate rings and are issued, in
        // tile order within each ring, as soon as a stage is free (K first:
        // the next S needs it before the next P.V needs its V).
        if (lane == 0) {
            bool ok = true;
            int jk = 0, jv = 0;
            IdleWatch watch;
            while (ok && (jk < nt || jv < nt)) {
                bool progressed = false;
                if (jk < nt) {
                    const int s = jk % kKStages, u = jk / kKStages;
                    if (u == 0 || mbar_test(&kempty[s], (u - 1) & 1)) {
                        const int ky = int(bh * fa.Wp + int64_t(jk) * kKeyTile);
                        uint8_t *kst = smem + Sm::oK + s * 2 * Sm::kK;
                        mbar_arrive_expect_tx(&kfull[s], 2 * Sm::kK);
                        for (int bx = 0; bx < NBOX; ++bx) {
                            tma_load_2d(kst + bx * kKeyTile * 128, &khmap, 64 * bx, ky, &kfull[s]);
                            tma_load_2d(kst + Sm::kK + bx * kKeyTile * 128, &klmap, 64 * bx, ky, &kfull[s]);
                        }
                        ++jk;
                        progressed = true;
                    }
                }
                if (jv < jk) {
                    const int s = jv % kVStages, u = jv / kVStages;
                    if (u == 0 || mbar_test(&vempty[s], (u - 1) & 1)) {
                        mbar_arrive_expect_tx(&vfull[s], Sm::kV);
                        for (int bx = 0; bx < kKeyTile / 64; ++bx)
                            tma_load_2d(smem + Sm::oV + s * Sm::kV + bx * D * 128, &vtmap,
                                        jv * kKeyTile + 64 * bx, int(bh * D), &vfull[s]);
                        ++jv;
                        progressed = true;
                    }
                }
                if (progressed) {
                    watch.progress();
                } else if (aborted() || watch.expired(kWaitLimitNs)) {
                    fail();
                    ok = false;
                } else {
                    __nanosleep(64);
                }
            }
            // drain the loads in flight (the last fill of each stage)
            for (int j = jk - kKStages < 0 ? 0 : jk - kKStages; j < jk; ++j)
                if (!mbar_wait_bounded(&kfull[j % kKStages], (j / kKStages) & 1, kWaitLimitNs)) fail();
            for (int j = jv - kVStages < 0 ? 0 : jv - kVStages; j < jv; ++j)
                if (!mbar_wait_bounded(&vfull[j % kVStages], (j / kVStages) & 1, kWaitLimitNs)) fail();
        }
    } else if (warp == 1) {
        // ------------------------------------------------ S issuer
        // S(js) as soon as K(js) has landed and S tile js&1 is free (the
        // P(js-2).V(js-2) that read it has completed).  tcgen05.mma issue stalls while the pipe is full, so the
        // P.V products have their own issuing thread (the last warp) and
        // never wait behind an S.
        if (lane == 0) {
            const uint32_t id_s = idesc_bf16(kQRows, kKeyTile);
            const uint32_t t_qh = tmem_base + kQCol, t_ql = t_qh + uint32_t(D / 2);
            bool ok = !aborted() && mbar_wait_bounded(qfull, 0, kWaitLimitNs);
            if (!ok) fail();
            tc_fence_after();
            for (int js = 0; ok && js < nt; ++js) {
                const int s = js & 1, ks_ = js % kKStages;
                if (aborted() || !mbar_wait_bounded(&kfull[ks_], (js / kKStages) & 1, kWaitLimitNs) ||
                    (js >= 2 && !mbar_wait_bounded(&pvdone[s], ((js >> 1) - 1) & 1, kWaitLimitNs))) {
                    fail();
                    ok = false;
                    break;
                }
                // S(js) = Q.K(js)^T (three hi/lo products; Q from TMEM; the
                // two products with Kh are issued back to back)
                tc_fence_after();
                const uint8_t *kst = smem + Sm::oK + ks_ * 2 * Sm::kK;
                const uint32_t d_s = tmem_base + kSCol + uint32_t(s * kKeyTile);
#pragma unroll
                for (int ks = 0; ks < KS; ++ks) {
                    const int bx = ks / 4, kin = ks % 4;
                    const uint64_t kh = sw128_desc(kst + bx * kKeyTile * 128) + uint64_t(kin * 2);
                    const uint64_t kl = sw128_desc(kst + Sm::kK + bx * kKeyTile * 128) + uint64_t(kin * 2);
                    const uint32_t qh = t_qh + uint32_t(ks * 8), ql = t_ql + uint32_t(ks * 8);
                    tc_mma_ts(d_s, qh, kh, id_s, ks > 0 ? 1u : 0u);
                    tc_mma_ts(d_s, ql, kh, id_s, 1u);
                    tc_mma_ts(d_s, qh, kl, id_s, 1u);
                }
                tc_commit(&sfull[s]);
                tc_commit(&kempty[ks_]);
            }
            tc_commit(&done[0]);
            if (!mbar_wait_bounded(&done[0], 0, kWaitLimitNs)) fail();
        }
    } else if (warp == kFaPvWarp) {
        // ------------------------------------------------ P.V issuer
        if (lane == 0) {
            const uint32_t id_o = idesc_f16(kQRows, D);
            bool ok = true;
            for (int jp = 0; ok && jp < nt; ++jp) {
                const int s = jp & 1, vs_ = jp % kVStages;
                if (aborted() || !mbar_wait_bounded(&pfull[s], (jp >> 1) & 1, kWaitLimitNs) ||
                    !mbar_wait_bounded(&vfull[vs_], (jp / kVStages) & 1, kWaitLimitNs)) {
                    fail();
                    ok = false;
                    break;
                }
                // O += P(jp).V(jp) (P from TMEM)
                tc_fence_after();
                const uint32_t d_o = tmem_base + kOCol;
                const uint32_t t_p = tmem_base + kSCol + uint32_t(s * kKeyTile);
                const uint8_t *vst = smem + Sm::oV + vs_ * Sm::kV;
#pragma unroll
                for (int ks = 0; ks < PS; ++ks) {
                    const uint64_t vd = sw128_desc(vst + (ks / 4) * D * 128) + uint64_t((ks % 4) * 2);
                    tc_mma_ts(d_o, t_p + uint32_t(ks * 8), vd, id_o, (jp > 0 || ks > 0) ? 1u : 0u);
                }
                tc_commit(&pvdone[s]);
                tc_commit(&vempty[vs_]);
            }
            tc_commit(&done[1]);
            if (!mbar_wait_bounded(&done[1], 0, kWaitLimitNs)) fail();
        }
    } else {
        // ------------------------------------------------ softmax warps (half a query row each)
        // The two warps of a lane group keep identical row state (same
        // maxima, same decisions) and leave the loop together: every tile
        // they trade their half-row maxima and their status through
        // shared memory (double-buffered by tile parity) across one named
        // barrier of the pair.
        __shared__ float xmax[2][4][2][32], xsum[4][2][32];
        __shared__ int xok[2][4][2];
        const int quad = warp & 3;               // TMEM lanes this warp may access
        const int half = (warp - 2) >> 2;        // S columns [64*half, 64*half + 64)
        const int row = quad * 32 + lane;
        const uint32_t lane_base = tmem_base + (uint32_t(quad * 32) << 16);
        const bool live = row < nrows;
        const int64_t qpos = live ? qpos0 + (r0 + row) % geo.C : -1;
        // last key this row sees (window end and causal limit); -1: none
        const int row_lim = live ? int((kend - 1 < qpos) ? kend - 1 : qpos) : -1;
        auto pair_sync = [&] { named_sync(1 + quad, 64); };
        float m_ref = -INFINITY, l = 0.f;
        bool ok = true;
        constexpr int HC = kKeyTile / 2;         // columns per warp
        {
            // this row's query term (half 0: hi, half 1: lo) into TMEM, the
            // A operand of S; rows >= R are zero in the prep's buffer
            const __nv_bfloat16 *src = (half ? fa.ql : fa.qh) + (bh * fa.Rp + r0 + row) * D;
            const uint32_t tq = lane_base + kQCol + uint32_t(half * (D / 2));
#pragma unroll
            for (int c = 0; c < D / 64; ++c) {
                float w[32];
                const uint4 *s4 = reinterpret_cast<const uint4 *>(src + c * 64);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const uint4 v = s4[i];
                    w[4 * i] = __uint_as_float(v.x);
                    w[4 * i + 1] = __uint_as_float(v.y);
                    w[4 * i + 2] = __uint_as_float(v.z);
                    w[4 * i + 3] = __uint_as_float(v.w);
                }
                tmem_st32(tq + uint32_t(c * 32), w);
            }
            asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(qfull);
        }
        for (int j = 0; j < nt; ++j) {
            const int s = j & 1;
            if (ok) {
                const bool got = !aborted() && mbar_wait_bounded(&sfull[s], (j >> 1) & 1, kWaitLimitNs);
                if (!__all_sync(0xffffffffu, got)) {
                    if (lane == 0) fail();
                    ok = false;
                }
            }
            float sv[HC];
            float mx = -INFINITY;
            if (ok) {
                tc_fence_after();
                {
                    uint32_t ra[32], rb[32];
                    const uint32_t ts = lane_base + kSCol + uint32_t(s * kKeyTile + half * HC);
                    tmem_ld32_nowait(ts, ra);
                    tmem_ld32_nowait(ts + 32u, rb);
                    tmem_wait_ld();
                    tmem_regs_after_wait(ra);
                    tmem_regs_after_wait(rb);
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        sv[i] = __uint_as_float(ra[i]);
                        sv[32 + i] = __uint_as_float(rb[i]);
                    }
                }
                // keys past this row's limit (window end, causal) are masked;
                // halves wholly inside the limit skip the per-key test
                const int kb = j * kKeyTile + half * HC;
                if (kb + HC - 1 > row_lim) {
#pragma unroll
                    for (int i = 0; i < HC; ++i)
                        if (kb + i > row_lim) sv[i] = -INFINITY;
                }
                // eight independent partial maxima (short dependency chains)
                float pm[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) pm[i] = sv[i];
#pragma unroll
                for (int i = 8; i < HC; ++i) pm[i & 7] = fmaxf(pm[i & 7], sv[i]);
                mx = fmaxf(fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])),
                           fmaxf(fmaxf(pm[4], pm[5]), fmaxf(pm[6], pm[7])));
            }
            xmax[s][quad][half][lane] = mx;
            if (lane == 0) xok[s][quad][half] = ok ? 1 : 0;
            pair_sync();
            if (!xok[s][quad][0] || !xok[s][quad][1]) break;   // both warps leave together
            mx = fmaxf(mx, xmax[s][quad][half ^ 1][lane]);
            const float m_new = fmaxf(m_ref, mx);
            const bool move = m_new != -INFINITY && (m_ref == -INFINITY || m_new > m_ref + kRescaleLog2);
            float fac = 1.f;
            if (move) {
                fac = m_ref == -INFINITY ? 0.f : exp2f(m_ref - m_new);
                m_ref = m_new;
                l *= fac;
            }
            if (j >= 1 && __any_sync(0xffffffffu, move && fac != 1.f)) {
                // O is quiescent once P(j-1).V(j-1) has completed (P(j).V is
                // issued only after this tile's P is written)
                const bool got = !aborted() &&
                                 mbar_wait_bounded(&pvdone[(j - 1) & 1], ((j - 1) >> 1) & 1, kWaitLimitNs);
                if (!__all_sync(0xffffffffu, got)) {
                    if (lane == 0) fail();
                    ok = false;
                    continue;
                }
                tc_fence_after();
                // rescale this row's half of O in TMEM (warp-collective accesses)
#pragma unroll
                for (int cb = 0; cb < D / 64; ++cb) {
                    float o[32];
                    const uint32_t ta = lane_base + kOCol + uint32_t(half * (D / 2) + cb * 32);
                    tmem_ld32(ta, o);
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] *= fac;
                    tmem_st32(ta, o);
                }
            }
            // P = exp2(S - m_ref) <= 2^8 as fp16 (11-bit significand) into
            // this row's lane of S tile j&1: keys [64*half, 64*half+64) as 32
            // columns of fp16 pairs at columns [32*half, 32*half+32) (the A
            // operand of P.V).  Both warps of the pair have read their S
            // columns before the exchange above, so nothing unread is
            // overwritten.
            const bool any_key = m_ref != -INFINITY;
            float rs4[4] = {0.f, 0.f, 0.f, 0.f};
            float pw[HC / 2];
#pragma unroll
            for (int e = 0; e < HC; e += 2) {
                // masked keys are -inf: ex2 gives 0; a row with no key seen
                // yet (m_ref = -inf) has only masked keys
                const float p0 = any_key ? ex2_approx(sv[e] - m_ref) : 0.f;
                const float p1 = any_key ? ex2_approx(sv[e + 1] - m_ref) : 0.f;
                rs4[(e / 2) & 3] += p0 + p1;   // four partial sums (short chains)
                const __half2 hv = __floats2half2_rn(p0, p1);
                pw[e / 2] = __uint_as_float(*reinterpret_cast<const uint32_t *>(&hv));
            }
            const float rs = (rs4[0] + rs4[1]) + (rs4[2] + rs4[3]);
            tmem_st32(lane_base + kSCol + uint32_t(s * kKeyTile + half * (HC / 2)), pw);
            l += rs;
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&pfull[s]);
        }
        // row sum over both halves (both warps reach this barrier: they leave
        // the loop at the same tile or finish it)
        xsum[quad][half][lane] = l;
        pair_sync();
        l += xsum[quad][half ^ 1][lane];
        if (ok && nt > 0) {
            const bool got = !aborted() &&
                             mbar_wait_bounded(&pvdone[(nt - 1) & 1], ((nt - 1) >> 1) & 1, kWaitLimitNs);
            if (!__all_sync(0xffffffffu, got)) {
                if (lane == 0) fail();
            } else {
                tc_fence_after();
                const int r = r0 + row;
                const int j = h * geo.g + (live ? r / geo.C : 0), c = live ? r % geo.C : 0;
                float *dst = fa.out + ((int64_t(b) * geo.Hq + j) * geo.C + c) * D + half * (D / 2);
                const float il = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
                for (int cb = 0; cb < D / 64; ++cb) {
                    float o[32];
                    tmem_ld32(lane_base + kOCol + uint32_t(half * (D / 2) + cb * 32), o);
                    if (live) {
#pragma unroll
                        for (int i = 0; i < 32; i += 4)
                            *reinterpret_cast<float4 *>(dst + cb * 32 + i) =
                                make_float4(o[i] * il, o[i + 1] * il, o[i + 2] * il, o[i + 3] * il);
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, kTmemCols);
}

PFN_cuTensorMapEncodeTiled_v12000 encoder()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// 2-D bf16 map: `rows` rows of `cols` elements, boxes of box_rows x 64.
bool map2d(CUtensorMap *mp, const void *base, uint64_t rows, uint64_t cols, uint32_t box_rows)
{
    auto enc = encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {cuuint64_t(cols), cuuint64_t(rows)};
    cuuint64_t strides[1] = {cuuint64_t(cols) * 2};
    cuuint32_t box[2] = {64, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return enc(mp, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides,
               box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct PrepPlan {
    int Rp, Wp;
    size_t q_bytes, k_bytes, v_bytes;
};
PrepPlan prep_plan(const Geom &geo)
{
    PrepPlan p;
    const int64_t R = int64_t(geo.g) * geo.C;
    p.Rp = int((R + kQRows - 1) / kQRows * kQRows);
    p.Wp = int((geo.Wmax + kKeyTile - 1) / kKeyTile * kKeyTile);
    const size_t BH = size_t(geo.B) * geo.Hkv;
    p.q_bytes = (BH * p.Rp * geo.d * 2 + 255) / 256 * 256;
    p.k_bytes = (BH * p.Wp * geo.d * 2 + 255) / 256 * 256;
    p.v_bytes = p.k_bytes;
    return p;
}

}  // namespace

bool encode_bf16_map(CUtensorMap *mp, const void *base, uint64_t rows, uint64_t cols,
                     uint32_t box_rows)
{
    return map2d(mp, base, rows, cols, box_rows);
}

bool prefill_attn_tc_eligible(const Geom &geo)
{
    const int64_t R = int64_t(geo.g) * geo.C;
    const int64_t BH = int64_t(geo.B) * geo.Hkv;
    const PrepPlan p = prep_plan(geo);
    return geo.dtype == REATT_BF16 && R > 8 && (geo.d == 64 || geo.d == 128) &&
           BH * p.Wp < (int64_t(1) << 31) && BH * p.Rp < (int64_t(1) << 31) &&
           BH * geo.d < (int64_t(1) << 31);
}

size_t prefill_attn_tc_ws_bytes(const Geom &geo)
{
    if (!prefill_attn_tc_eligible(geo)) return 0;
    const PrepPlan p = prep_plan(geo);
    return 2 * p.q_bytes + 2 * p.k_bytes + p.v_bytes;
}

cudaError_t launch_attend_prefill_tc(const Geom &geo, const void *q, const void *kc,
                                     const void *vc, const void *kcur, const void *vcur,
                                     const int32_t *sel, const float2 *tab, float *out,
                                     void *scratch, void *ws, cudaStream_t st)
{
    const PrepPlan pp = prep_plan(geo);
    uint8_t *base = static_cast<uint8_t *>(scratch);
    PrepOut po;
    po.qh = reinterpret_cast<__nv_bfloat16 *>(base);
    po.ql = reinterpret_cast<__nv_bfloat16 *>(base + pp.q_bytes);
    po.kh = reinterpret_cast<__nv_bfloat16 *>(base + 2 * pp.q_bytes);
    po.kl = reinterpret_cast<__nv_bfloat16 *>(base + 2 * pp.q_bytes + pp.k_bytes);
    po.vt = reinterpret_cast<__half *>(base + 2 * pp.q_bytes + 2 * pp.k_bytes);
    po.Rp = pp.Rp;
    po.Wp = pp.Wp;
    const unsigned BH = unsigned(geo.B * geo.Hkv);
    dim3 pgrid(unsigned(pp.Wp / kPrepRows + pp.Rp / kPrepRows), BH);
    const uint16_t *q16 = static_cast<const uint16_t *>(q);
    const uint16_t *k16 = static_cast<const uint16_t *>(kc), *v16 = static_cast<const uint16_t *>(vc);
    const uint16_t *kq = static_cast<const uint16_t *>(kcur), *vq = static_cast<const uint16_t *>(vcur);
    cudaError_t e;
    if (geo.d == 128)
        e = launch_pdl(prefill_prep_kernel<128>, pgrid, dim3(256), 0, st, geo, q16, k16, v16, kq, vq,
                       sel, tab, po);
    else
        e = launch_pdl(prefill_prep_kernel<64>, pgrid, dim3(256), 0, st, geo, q16, k16, v16, kq, vq,
                       sel, tab, po);
    if (e != cudaSuccess) return e;
    const uint64_t BHu = BH;
    CUtensorMap kh, kl, vt;
    if (!map2d(&kh, po.kh, BHu * pp.Wp, geo.d, kKeyTile) || !map2d(&kl, po.kl, BHu * pp.Wp, geo.d, kKeyTile) ||
        !map2d(&vt, po.vt, BHu * geo.d, pp.Wp, uint32_t(geo.d)))
        return cudaErrorInvalidValue;
    FaArgs fa;
    fa.out = out;
    fa.sel = sel;
    fa.qh = po.qh;
    fa.ql = po.ql;
    fa.Rp = pp.Rp;
    fa.Wp = pp.Wp;
    dim3 grid(unsigned(pp.Rp / kQRows), BH);
    if (geo.d == 128) {
        auto kern = attend_prefill_tc_kernel<128>;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(FaSmem<128>::kBytes));
        if (e != cudaSuccess) return e;
        e = launch_pdl(kern, grid, dim3(kFaThreads), FaSmem<128>::kBytes, st, kh, kl, vt, geo, fa, ws);
    } else {
        auto kern = attend_prefill_tc_kernel<64>;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(FaSmem<64>::kBytes));
        if (e != cudaSuccess) return e;
        e = launch_pdl(kern, grid, dim3(kFaThreads), FaSmem<64>::kBytes, st, kh, kl, vt, geo, fa, ws);
    }
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace reatt
