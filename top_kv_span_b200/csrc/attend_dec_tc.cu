// Decode attention of the fused step on the tensor cores (tcgen05 + TMEM):
// bf16 caches, d = 128, up to 8 query rows per KV head (ReAttention
// OpenReview discussion, "Decoding Phase" pseudocode: attention over global
// ++ recalled ++ local; research-map summary "Approach": RoPE after the
// concatenation, window row p at position p, query c at W-C+c).
//
// The keys sit on the MMA's M dimension, so a 128-key tile is one M=128 MMA
// chain whatever the (small) number of queries:
//   S^T (128 keys x 16)  = [Kh | Kl] . [Qh ; Ql]^T   columns r: Kh.Qh + Kl.Qh,
//                                                    columns 8+r: Kh.Ql + Kl.Ql
//   O^T (128 dims x 16) += V^T . [Ph ; Pl]^T         column r + column 8+r = O_r
// Every rotated operand is split into bf16 hi + lo, so products keep fp32-level
// accuracy (V is exact: bf16 input).  Roles of the 14 warps:
//   warp 0      TMA: the tile's K and V rows in boxes of 32 or 8 rows x 64
//               columns, 128B-swizzled, each inside one run of the window (the
//               global part, a chosen span, the local part, the current tokens)
//               and one 32-row quarter of the tile; lane q issues quarter q, so
//               the four quarters' loads go out together.  K quarters have a
//               barrier each, V one per stage; a tile's K goes out when its
//               raw stage is free and its V when its V stage is free, so the
//               chosen rows' keys load as soon as the selection is in.  V lands
//               directly in the MN-major operand layout
//   warp 1      TMEM allocation; one thread issues S(j) and then P(j-1).V(j-1)
//   warps 2-9   rotate the raw keys of each quarter as it lands (RoPE with
//               the step's cos/sin table) and split them into the hi/lo
//               K-major operands
//   warps 10-13 the rotated query operand first; then softmax: thread t owns
//               key t of the tile (TMEM lane t): online
//               softmax with a lazily moved reference max (rescales O in TMEM
//               only when the max grows by more than 2^8), P^T as bf16 hi/lo
// The CTA walks its slice of the rows that do not depend on the selection
// first (when the window length is known up front), then its slice of the
// global and chosen rows; split CTAs merge through the workspace as the other
// decode kernels do.
#include <cuda_bf16.h>
#include <math.h>

#include "attend_common.cuh"
#include "common.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"

namespace reatt {

namespace {

using namespace tc;

constexpr int kDtD = 128;
constexpr int kDtKeys = 128;                          // keys per tile (M of S^T)
constexpr int kDtN = 16;                              // 8 hi + 8 lo query columns
constexpr int kDtConvWarps = 8;
constexpr int kDtSoftWarps = 4;
constexpr int kDtConvBase = 2;                        // first converter warp
constexpr int kDtSoftBase = kDtConvBase + kDtConvWarps;
constexpr int kDtThreads = (kDtSoftBase + kDtSoftWarps) * 32;
constexpr int kDtHalf = kDtKeys * 128;                // 64-column half of a tile: 16 KB
constexpr int kDtTile = 2 * kDtHalf;                  // 128 rows x 128 bf16
constexpr int kDtOpHalf = kDtN * 128;                 // half of the 16-row Q / P operands
constexpr uint32_t kDtTmemCols = 64;                  // S buffers at 0 and 16, O at 32
constexpr float kDtRescaleLog2 = 8.f;
constexpr int kDtSelCache = 256;                      // chosen span ids of a CTA's rows
static_assert(kDtSoftWarps * 32 == kDtKeys, "one softmax thread per key");

// Shared memory (1024-byte aligned): raw K stages | V stages | Kh | Kl | Q | P |
// barriers.
struct DtSmem {
    static constexpr int oRaw = 0;
    static constexpr int oV = oRaw + 2 * kDtTile;
    static constexpr int oKh = oV + 2 * kDtTile;
    static constexpr int oKl = oKh + kDtTile;
    static constexpr int oQ = oKl + kDtTile;
    static constexpr int oP = oQ + 2 * kDtOpHalf;
    static constexpr int oBar = oP + 2 * kDtOpHalf;
    static constexpr size_t kBytes = size_t(oBar) + 32 * 8 + 1024;
};

// Byte offset of 16-byte chunk ch (elements 8ch..8ch+7 of 128) of row r in a
// buffer of two 64-element halves, `half` bytes each, 128-byte rows,
// 128B-swizzled.  Read by tcgen05 as a K-major operand when rows are M/N and
// as an MN-major operand (64-element blocks `half` apart) when rows are K.
__device__ __forceinline__ int sw_off(int r, int ch, int half)
{
    return (ch >> 3) * half + r * 128 + (((ch & 7) ^ (r & 7)) << 4);
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b)
{
    const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t *>(&v);
}
// hi = bf16(a, b); lo = bf16 of the remainders (exact in fp32)
__device__ __forceinline__ void split_pack(float a, float b, uint32_t &hi, uint32_t &lo)
{
    hi = pack_bf16(a, b);
    const float ha = __uint_as_float(hi << 16), hb = __uint_as_float(hi & 0xffff0000u);
    lo = pack_bf16(a - ha, b - hb);
}

// Tensor maps of the caches (boxes of 32 and 8 rows) and of the current
// tokens (8 rows); every box is 64 columns wide.
struct DtMaps {
    CUtensorMap k[2], v[2], kq, vq;
};
__host__ __device__ constexpr int dt_box_rows(int i) { return i == 0 ? 32 : 8; }
constexpr int kDtQuarter = 32;                        // rows per load barrier

template <int RP>
__global__ void __launch_bounds__(kDtThreads, 1)
attend_decode_tc_kernel(const __grid_constant__ DtMaps maps, Geom geo, AttnArgs a, void *ws)
{
    constexpr int D = kDtD;
    using Sm = DtSmem;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Sm::oBar);
    uint64_t *rawempty = bars + 2, *vempty = bars + 4, *kopfull = bars + 6,
             *kopempty = bars + 7, *sfull = bars + 8, *sempty = bars + 10, *pfull = bars + 12,
             *pvdone = bars + 13, *done = bars + 14, *qready = bars + 15;
    // K rows [32q, 32q + 32) of stage s: tq[4s + q]
    uint64_t *tq = bars + 16;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 24);
    // V rows of stage s: tv[s]
    uint64_t *tv = bars + 26;
    __shared__ float red[2][kDtSoftWarps][RP], lred[kDtSoftWarps][RP];
    __shared__ float f_m[RP], f_l[RP];
    __shared__ __align__(16) float s_acc[RP * D];
    __shared__ float2 freq[D / 2];
    __shared__ int32_t sel_s[kDtSelCache];
    __shared__ int is_last, abort_flag;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        abort_flag = 0;
        for (int s = 0; s < 2; ++s) {
            mbar_init(&rawempty[s], kDtConvWarps);
            mbar_init(&vempty[s], 1);
            mbar_init(&sfull[s], 1);
            mbar_init(&sempty[s], kDtSoftWarps);
        }
        mbar_init(kopfull, kDtConvWarps);
        mbar_init(kopempty, 1);
        mbar_init(pfull, kDtSoftWarps);
        mbar_init(pvdone, 1);
        mbar_init(done, 1);
        mbar_init(qready, kDtSoftWarps);
        for (int q = 0; q < 8; ++q) mbar_init(&tq[q], 1);
        for (int q = 0; q < 2; ++q) mbar_init(&tv[q], 1);
        mbar_init_fence();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kDtTmemCols);
        tmem_relinquish();
    }
    if (tid < D / 2) freq[tid] = make_float2(geo.rope_hi[tid], geo.rope_lo[tid]);
    const bool early = a.w_known >= 0;
    if (!early) pdl_wait();   // selection and RoPE table from the preceding kernels

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
    // Rows of this CTA: a slice of [r_mid, W) (rows that do not depend on the
    // selection; empty without early mode), then a slice of [0, r_mid).
    const int r_mid = early ? g_end + nsel : int(W);
    int eb, ee, lb, le;
    {
        const int last_row = nrows - 1;
        const int c_max = (last_row / geo.C == 0) ? last_row % geo.C : geo.C - 1;
        const int lim = int(W) - geo.C + c_max + 1;
        auto part = [&](int r0, int r1, int &pb, int &pe) {
            int len = (r1 - r0 + a.nsplit - 1) / a.nsplit;
            len = (len + 15) / 16 * 16;
            pb = r0 + split * len;
            pe = pb + len;
            if (pe > r1) pe = r1;
            if (pe > lim) pe = lim;
            if (pb > pe) pb = pe;
        };
        part(r_mid, int(W), eb, ee);
        part(0, r_mid, lb, le);
    }
    const int nE = (ee - eb + kDtKeys - 1) / kDtKeys;
    const int nt = nE + (le - lb + kDtKeys - 1) / kDtKeys;
    auto tile_at = [&](int j, int &p0, int &n) {
        const int pend = j < nE ? ee : le;
        p0 = j < nE ? eb + j * kDtKeys : lb + (j - nE) * kDtKeys;
        n = pend - p0 < kDtKeys ? pend - p0 : kDtKeys;
    };
    // span ids of the chosen rows inside the late slice
    int j0 = 0, jn = 0;
    {
        const int lo = lb > g_end ? lb : g_end;
        const int hi = le < g_end + nsel ? le : g_end + nsel;
        if (lo < hi) {
            j0 = (lo - g_end) / geo.S;
            jn = (hi - 1 - g_end) / geo.S - j0 + 1;
        }
    }
    const bool sel_cached = jn <= kDtSelCache;
    auto fail = [&]() {
        report_status(ws, REATT_ETIMEOUT);
        *(volatile int *)&abort_flag = 1;
    };
    auto aborted = [&]() { return *(volatile int *)&abort_flag != 0; };

    // P starts at zero (its rows past the query rows are never written).  V
    // needs no clearing: P.V reads only the 16-key steps that hold keys of the
    // tile, and the loads fill every row of those steps.
    for (int x = tid; x < 2 * kDtOpHalf / 16; x += kDtThreads)
        reinterpret_cast<uint4 *>(smem + Sm::oP)[x] = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------ loads (TMA)
        if (lane == 0)
            for (int i = 0; i < 2; ++i) {
                prefetch_tensormap(&maps.k[i]);
                prefetch_tensormap(&maps.v[i]);
            }
        if (lane == 1) {
            prefetch_tensormap(&maps.kq);
            prefetch_tensormap(&maps.vq);
        }
        // Lane q (< 4) issues the boxes of quarter q (rows [32q, 32q + 32)) of
        // tile j: its K rows (want_v false) or its V rows, each box inside one
        // run of the window.  V gets 8 more rows past an odd number of 8-row
        // groups so P.V runs whole 16-key steps.
        auto issue_quarter = [&](int j, int q, bool want_v) {
            const int s = j & 1;
            int p0, n;
            tile_at(j, p0, n);
            uint8_t *dst = smem + (want_v ? Sm::oV : Sm::oRaw) + s * kDtTile;
            uint64_t *bar = want_v ? &tv[s] : &tq[4 * s + q];
            const int r_end = kDtQuarter * q + kDtQuarter < n ? kDtQuarter * q + kDtQuarter : n;
            for (int r = kDtQuarter * q; r < r_end;) {
                const int p = p0 + r;
                int run_end;
                bool cur = false;
                int64_t y;
                if (p < g_end) {
                    run_end = g_end;
                    y = bh * geo.Ts + p;
                } else if (p - g_end < nsel) {
                    const int qq = p - g_end, jj = qq / geo.S, off = qq - jj * geo.S;
                    int sp = sel_cached ? sel_s[jj - j0] : sel_bh[jj];
                    sp = sp < 0 ? 0 : (sp >= int(geo.NS) ? int(geo.NS) - 1 : sp);
                    run_end = g_end + (jj + 1) * geo.S;
                    y = bh * geo.Ts + geo.G + int64_t(sp) * geo.S + off;
                } else if (p - g_end - nsel < nloc) {
                    run_end = g_end + nsel + nloc;
                    y = bh * geo.Ts + m.loc_begin + (p - g_end - nsel);
                } else {
                    run_end = int(W);
                    cur = true;
                    y = bh * geo.C + (p - g_end - nsel - nloc);
                }
                int len = (run_end < p0 + r_end ? run_end : p0 + r_end) - p;
                while (len > 0) {
                    const int hs = (!cur && len >= 32 && (r & 31) == 0) ? 0 : 1;
                    const CUtensorMap *mp = want_v ? (cur ? &maps.vq : &maps.v[hs])
                                                   : (cur ? &maps.kq : &maps.k[hs]);
                    tma_load_2d(dst + r * 128, mp, 0, int(y), bar);
                    tma_load_2d(dst + kDtHalf + r * 128, mp, 64, int(y), bar);
                    r += dt_box_rows(hs);
                    if (want_v && r >= n && (r & 8)) {
                        tma_load_2d(dst + r * 128, mp, 0, int(y), bar);
                        tma_load_2d(dst + kDtHalf + r * 128, mp, 64, int(y), bar);
                    }
                    y += dt_box_rows(hs);
                    len -= dt_box_rows(hs);
                }
            }
        };
        // K of tile jk once its raw stage is free (tile jk - 2 converted) and,
        // from tile nE on, the selection is in; V of tile jv (jv < jk) once
        // its V stage is free (P.V of tile jv - 2 done).  Neither waits for
        // the other, so the chosen rows' keys load as soon as the selection
        // lands, not after the second-last tile's P.V.
        bool ok = true, sel_in = nE >= nt;
        int jk = 0, jv = 0;
        IdleWatch watch;
        while (jv < nt) {
            bool progressed = false;
            if (jv < jk) {
                bool ready = jv < 2 || mbar_test(&vempty[jv & 1], uint32_t((jv >> 1) - 1) & 1u);
                ready = __shfl_sync(0xffffffffu, ready, 0);
                if (ready) {
                    int p0, n;
                    tile_at(jv, p0, n);
                    const int ng = (n + 7) / 8;
                    if (lane == 0)
                        mbar_arrive_expect_tx(&tv[jv & 1], uint32_t(8 * (ng + (ng & 1))) * 256u);
                    __syncwarp();
                    if (lane < 4) issue_quarter(jv, lane, true);
                    __syncwarp();
                    ++jv;
                    progressed = true;
                }
            }
            if (jk < nt) {
                bool ready = true;
                if (jk == nE && !sel_in) {   // the global and chosen rows need the selection
                    __syncwarp();
                    pdl_wait();
                    sel_in = true;
                    if (sel_cached)
                        for (int x = lane; x < jn; x += 32) sel_s[x] = sel_bh[j0 + x];
                    __syncwarp();
                }
                if (jk >= 2)
                    ready = mbar_test(&rawempty[jk & 1], uint32_t((jk >> 1) - 1) & 1u);
                ready = __shfl_sync(0xffffffffu, ready, 0);
                if (ready) {
                    if (lane < 4) {
                        int p0, n;
                        tile_at(jk, p0, n);
                        const int ng = (n + 7) / 8;
                        int rows = 8 * ng - kDtQuarter * lane;
                        rows = rows < 0 ? 0 : (rows > kDtQuarter ? kDtQuarter : rows);
                        uint64_t *bar = &tq[4 * (jk & 1) + lane];
                        if (rows)
                            mbar_arrive_expect_tx(bar, uint32_t(rows) * 256u);
                        else
                            mbar_arrive(bar);
                        issue_quarter(jk, lane, false);
                    }
                    __syncwarp();
                    ++jk;
                    progressed = true;
                }
            }
            if (progressed) {
                watch.progress();
            } else {
                if (__any_sync(0xffffffffu, aborted() || watch.expired(kWaitLimitNs))) {
                    ok = false;
                    break;
                }
                __nanosleep(32);
            }
        }
        if (!ok && lane == 0) fail();
        // drain: the last loads of each stage have landed
        for (int j = nt - 2 < 0 ? 0 : nt - 2; ok && j < nt; ++j) {
            const uint32_t par = uint32_t(j >> 1) & 1u;
            bool got = mbar_wait_bounded(&tv[j & 1], par, kWaitLimitNs);
            for (int q = 0; q < 4; ++q)
                got = mbar_wait_bounded(&tq[4 * (j & 1) + q], par, kWaitLimitNs) && got;
            if (!got && lane == 0) fail();
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t id_s = idesc_bf16(kDtKeys, kDtN), id_o = idesc_bf16_amn(D, kDtN);
            const uint8_t *kh = smem + Sm::oKh, *kl = smem + Sm::oKl, *qo = smem + Sm::oQ,
                          *po = smem + Sm::oP;
            // operand descriptors at their k = 0 step
            const uint64_t dKh[2] = {sw128_desc(kh), sw128_desc(kh + kDtHalf)};
            const uint64_t dKl[2] = {sw128_desc(kl), sw128_desc(kl + kDtHalf)};
            const uint64_t dQ[2] = {sw128_desc(qo), sw128_desc(qo + kDtOpHalf)};
            const uint64_t dP0 = sw128_desc(po), dP1 = sw128_desc(po + kDtOpHalf);
            const uint64_t dV0 = sw128_mn_desc(smem + Sm::oV, kDtHalf);
            const uint64_t dV1 = sw128_mn_desc(smem + Sm::oV + kDtTile, kDtHalf);
            const bool qok = nt == 0 || (!aborted() && mbar_wait_bounded(qready, 0, kWaitLimitNs));
            if (!qok) fail();
            // S(js) as soon as tile js is converted (and its S buffer read),
            // P(jp).V(jp) as soon as P(jp) is written: whichever is ready.
            int js = 0, jp = 0;
            IdleWatch watch;
            while (qok && jp < nt) {
                bool progressed = false;
                if (js < nt && mbar_test(kopfull, uint32_t(js) & 1u) &&
                    (js < 2 || mbar_test(&sempty[js & 1], uint32_t((js >> 1) - 1) & 1u))) {
                    const int s = js & 1;
                    tc_fence_after();
                    const uint32_t d_s = tmem + uint32_t(s * kDtN);
#pragma unroll
                    for (int ks = 0; ks < D / 16; ++ks) {
                        const int bx = ks / 4, kin = ks % 4;
                        tc_mma(d_s, dKh[bx] + uint64_t(kin * 2), dQ[bx] + uint64_t(kin * 2), id_s,
                               ks > 0 ? 1u : 0u);
                        tc_mma(d_s, dKl[bx] + uint64_t(kin * 2), dQ[bx] + uint64_t(kin * 2), id_s, 1u);
                    }
                    tc_commit(&sfull[s]);
                    tc_commit(kopempty);
                    ++js;
                    progressed = true;
                }
                if (jp < js && mbar_test(pfull, uint32_t(jp) & 1u) &&
                    mbar_test(&tv[jp & 1], uint32_t(jp >> 1) & 1u)) {
                    const int s = jp & 1;
                    int p0, n;
                    tile_at(jp, p0, n);
                    tc_fence_after();
                    const uint64_t av0 = s ? dV1 : dV0;
                    for (int ks = 0; ks < (n + 15) / 16; ++ks) {
                        // 16 keys = 2048 bytes of V (descriptor units of 16 B)
                        const uint64_t bp = (ks < 4 ? dP0 : dP1) + uint64_t((ks % 4) * 2);
                        tc_mma(tmem + 32u, av0 + uint64_t(ks * 128), bp, id_o, (jp > 0 || ks > 0) ? 1u : 0u);
                    }
                    tc_commit(pvdone);
                    tc_commit(&vempty[s]);
                    ++jp;
                    progressed = true;
                }
                if (progressed) {
                    watch.progress();
                } else if (aborted() || watch.expired(kWaitLimitNs)) {
                    fail();
                    break;
                } else {
                    __nanosleep(64);   // leave the issue slots to the working warps
                }
            }
            tc_commit(done);
            if (!mbar_wait_bounded(done, 0, kWaitLimitNs)) fail();
        }
        __syncwarp();   // idle lanes wait here, not in the grid-dependency wait below
    } else if (warp < kDtSoftBase) {
        // ------------------------------------------------ RoPE + hi/lo split of K
        // All converter warps take each 32-row quarter as soon as it lands:
        // thread = (key kq of the quarter, pair chunk c); the key's cos/sin
        // come from the step's table for a tile's first quarter (loaded one
        // quarter ahead) and by rotation for the others.
        const int ct = tid - kDtConvBase * 32;
        const int c = ct & 7;                    // pairs 8c..8c+7 (dims and dims + 64)
        const int kq = ct >> 3;                  // 0..31
        static_assert(kDtConvWarps * 32 == kDtQuarter * 8, "one (key, chunk) per thread and quarter");
        auto anchors = [&](int job, float2 (&cs)[8]) {
            const int j = job >> 2, r = kDtQuarter * (job & 3) + kq;
            int p0, n;
            tile_at(j, p0, n);
            if (r < n) {
                const float4 *tr =
                    reinterpret_cast<const float4 *>(a.tab + int64_t(p0 + r) * (D / 2) + 8 * c);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float4 t = __ldcg(tr + e);
                    cs[2 * e] = make_float2(t.x, t.y);
                    cs[2 * e + 1] = make_float2(t.z, t.w);
                }
            }
        };
        float2 nx[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) nx[e] = make_float2(1.f, 0.f);
        if (nt > 0) anchors(0, nx);
        // (cos, sin) of 32 positions at this thread's frequencies: the key of
        // quarter q + 1 sits 32 positions after that of quarter q, so its
        // angles are the previous ones rotated by these (angle addition in
        // fp32, three steps at most) and the table is read once per tile.
        // Row 32 of the table exists whenever a tile has more than 32 rows.
        float2 r32[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) r32[e] = make_float2(1.f, 0.f);
        if (geo.Wmax > kDtQuarter) {
            const float4 *tr =
                reinterpret_cast<const float4 *>(a.tab + int64_t(kDtQuarter) * (D / 2) + 8 * c);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float4 t = __ldcg(tr + e);
                r32[2 * e] = make_float2(t.x, t.y);
                r32[2 * e + 1] = make_float2(t.z, t.w);
            }
        }
        bool ok = true;
        uint8_t *kh = smem + Sm::oKh, *kl = smem + Sm::oKl;
        for (int j = 0; j < nt && ok; ++j) {
            const int s = j & 1;
            int p0, n;
            tile_at(j, p0, n);
            const uint8_t *raw = smem + Sm::oRaw + s * kDtTile;
            for (int qd = 0; qd < 4; ++qd) {
                float2 cs[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) cs[e] = nx[e];
                const int job = 4 * j + qd;
                if (job + 1 < 4 * nt) {
                    if (qd < 3) {
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            nx[e] = make_float2(fmaf(cs[e].x, r32[e].x, -cs[e].y * r32[e].y),
                                                fmaf(cs[e].y, r32[e].x, cs[e].x * r32[e].y));
                    } else {
                        anchors(job + 1, nx);
                    }
                }
                ok = ok && !aborted() &&
                     mbar_wait_bounded(&tq[4 * s + qd], uint32_t(j >> 1) & 1u, kWaitLimitNs) &&
                     (qd > 0 || j == 0 || mbar_wait_bounded(kopempty, uint32_t(j - 1) & 1u, kWaitLimitNs));
                if (!__all_sync(0xffffffffu, ok)) {
                    if (lane == 0) fail();
                    ok = false;
                    break;
                }
                const int r = kDtQuarter * qd + kq;
                if (r < n) {
                    const uint4 xw = *reinterpret_cast<const uint4 *>(raw + sw_off(r, c, kDtHalf));
                    const uint4 yw = *reinterpret_cast<const uint4 *>(raw + sw_off(r, c + 8, kDtHalf));
                    const uint32_t xs[4] = {xw.x, xw.y, xw.z, xw.w}, ys[4] = {yw.x, yw.y, yw.z, yw.w};
                    uint32_t xh[4], xl[4], yh[4], yl[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float x0 = bf16lo(xs[e]), x1 = bf16hi(xs[e]);
                        const float y0 = bf16lo(ys[e]), y1 = bf16hi(ys[e]);
                        const float2 c0 = cs[2 * e], c1 = cs[2 * e + 1];
                        split_pack(x0 * c0.x - y0 * c0.y, x1 * c1.x - y1 * c1.y, xh[e], xl[e]);
                        split_pack(y0 * c0.x + x0 * c0.y, y1 * c1.x + x1 * c1.y, yh[e], yl[e]);
                    }
                    *reinterpret_cast<uint4 *>(kh + sw_off(r, c, kDtHalf)) = make_uint4(xh[0], xh[1], xh[2], xh[3]);
                    *reinterpret_cast<uint4 *>(kh + sw_off(r, c + 8, kDtHalf)) = make_uint4(yh[0], yh[1], yh[2], yh[3]);
                    *reinterpret_cast<uint4 *>(kl + sw_off(r, c, kDtHalf)) = make_uint4(xl[0], xl[1], xl[2], xl[3]);
                    *reinterpret_cast<uint4 *>(kl + sw_off(r, c + 8, kDtHalf)) = make_uint4(yl[0], yl[1], yl[2], yl[3]);
                }
            }
            if (!ok) break;
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(kopfull);
                mbar_arrive(&rawempty[s]);
            }
        }
    } else {
        // ------------------------------------------------ softmax (thread = key / dim)
        const int sw = warp - kDtSoftBase;
        const int quad = warp & 3;               // TMEM lanes this warp may access
        const int row = quad * 32 + lane;
        const uint32_t lane_base = tmem + (uint32_t(quad * 32) << 16);
        // rotated, scaled query rows: hi in operand rows 0..7, lo in rows 8..15
        for (int x = tid - kDtSoftBase * 32; x < 8 * (D / 2); x += kDtSoftWarps * 32) {
            // row r, pair i: dims i and i + 64
            const int r = x / (D / 2), i = x % (D / 2);
            float lo = 0.f, hi = 0.f;
            if (r < nrows) query_pair<uint16_t, D>(geo, freq, a.q, b, h, r, qpos0, i, lo, hi);
            const __nv_bfloat16 lh = __float2bfloat16_rn(lo), hh = __float2bfloat16_rn(hi);
            const __nv_bfloat16 ll = __float2bfloat16_rn(lo - __bfloat162float(lh));
            const __nv_bfloat16 hl = __float2bfloat16_rn(hi - __bfloat162float(hh));
            uint8_t *q = smem + Sm::oQ;
            const int cb = (i & 7) * 2;
            *reinterpret_cast<__nv_bfloat16 *>(q + sw_off(r, i >> 3, kDtOpHalf) + cb) = lh;
            *reinterpret_cast<__nv_bfloat16 *>(q + sw_off(r, 8 + (i >> 3), kDtOpHalf) + cb) = hh;
            *reinterpret_cast<__nv_bfloat16 *>(q + sw_off(8 + r, i >> 3, kDtOpHalf) + cb) = ll;
            *reinterpret_cast<__nv_bfloat16 *>(q + sw_off(8 + r, 8 + (i >> 3), kDtOpHalf) + cb) = hl;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(qready);
        uint8_t *po = smem + Sm::oP;
        float m_ref[RP], lp[RP];
#pragma unroll
        for (int r = 0; r < RP; ++r) {
            m_ref[r] = -INFINITY;
            lp[r] = 0.f;
        }
        bool ok = true;
        for (int j = 0; j < nt; ++j) {
            const int s = j & 1;
            int p0, n;
            tile_at(j, p0, n);
            float sc[RP];
            ok = ok && !aborted() && mbar_wait_bounded(&sfull[s], uint32_t(j >> 1) & 1u, kWaitLimitNs);
            if (!__all_sync(0xffffffffu, ok)) {
                if (lane == 0) fail();
                ok = false;
            }
            if (ok) {
                tc_fence_after();
                float v[16];
                tmem_ld16(lane_base + uint32_t(s * kDtN), v);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sempty[s]);
                const int64_t pos = int64_t(p0) + row;
#pragma unroll
                for (int r = 0; r < RP; ++r) {
                    const bool valid = row < n && r < nrows && pos <= qpos0 + r % geo.C;
                    sc[r] = valid ? v[r] + v[8 + r] : -INFINITY;
                    float wm = sc[r];
#pragma unroll
                    for (int o = 16; o >= 1; o >>= 1) wm = fmaxf(wm, __shfl_xor_sync(0xffffffffu, wm, o));
                    if (lane == 0) red[j & 1][sw][r] = wm;
                }
            }
            named_sync(1, kDtSoftWarps * 32);   // every softmax warp, every tile
            if (!ok) continue;
            // the P buffer and O are free once P(j-1).V(j-1) has completed
            if (j >= 1) {
                ok = !aborted() && mbar_wait_bounded(pvdone, uint32_t(j - 1) & 1u, kWaitLimitNs);
                if (!__all_sync(0xffffffffu, ok)) {
                    if (lane == 0) fail();
                    ok = false;
                    continue;
                }
                tc_fence_after();
            }
            float fac[RP];
            bool any = false;
#pragma unroll
            for (int r = 0; r < RP; ++r) {
                float tm = red[j & 1][0][r];
#pragma unroll
                for (int w2 = 1; w2 < kDtSoftWarps; ++w2) tm = fmaxf(tm, red[j & 1][w2][r]);
                const float m_new = fmaxf(m_ref[r], tm);
                fac[r] = 1.f;
                if (m_new != -INFINITY && (m_ref[r] == -INFINITY || m_new > m_ref[r] + kDtRescaleLog2)) {
                    fac[r] = m_ref[r] == -INFINITY ? 0.f : exp2f(m_ref[r] - m_new);
                    m_ref[r] = m_new;
                    lp[r] *= fac[r];
                    any = any || fac[r] != 1.f;
                }
            }
            if (j >= 1 && any) {   // rescale O^T (lane = dim) in TMEM; uniform decision
                float o[16];
                tmem_ld16(lane_base + 32u, o);
#pragma unroll
                for (int r = 0; r < RP; ++r) {
                    o[r] *= fac[r];
                    o[8 + r] *= fac[r];
                }
                tmem_st16(lane_base + 32u, o);
            }
            // column `row` of P^T: rows r (hi) and 8 + r (lo)
#pragma unroll
            for (int r = 0; r < RP; ++r) {
                const float p = sc[r] == -INFINITY ? 0.f : exp2f(sc[r] - m_ref[r]);
                lp[r] += p;
                const __nv_bfloat16 ph = __float2bfloat16_rn(p);
                const __nv_bfloat16 pl = __float2bfloat16_rn(p - __bfloat162float(ph));
                const int cb = (row & 7) * 2;
                *reinterpret_cast<__nv_bfloat16 *>(po + sw_off(r, row >> 3, kDtOpHalf) + cb) = ph;
                *reinterpret_cast<__nv_bfloat16 *>(po + sw_off(8 + r, row >> 3, kDtOpHalf) + cb) = pl;
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(pfull);
        }
        // this CTA's (reference max, sum, acc) per query row
        bool have_o = ok && nt > 0;
        if (have_o) {
            have_o = !aborted() && mbar_wait_bounded(pvdone, uint32_t(nt - 1) & 1u, kWaitLimitNs);
            if (!__all_sync(0xffffffffu, have_o)) {
                if (lane == 0) fail();
                have_o = false;
            }
        }
        float o[16];
        if (have_o) {
            tc_fence_after();
            tmem_ld16(lane_base + 32u, o);
        }
#pragma unroll
        for (int r = 0; r < RP; ++r) {
            s_acc[r * D + row] = have_o ? o[r] + o[8 + r] : 0.f;
            float x = lp[r];
#pragma unroll
            for (int o2 = 16; o2 >= 1; o2 >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o2);
            if (lane == 0) lred[sw][r] = x;
        }
        named_sync(1, kDtSoftWarps * 32);
        if (sw == 0 && lane == 0) {
#pragma unroll
            for (int r = 0; r < RP; ++r) {
                float l = 0.f;
                for (int w2 = 0; w2 < kDtSoftWarps; ++w2) l += lred[w2][r];
                f_m[r] = have_o ? m_ref[r] : -INFINITY;
                f_l[r] = have_o ? l : 0.f;
            }
        }
    }
    pdl_wait();   // split partials and tickets: after the preceding grid (it clears the tickets)
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, kDtTmemCols);
    // the raw K stages are idle now: scratch of the split merge
    split_finish<D, RP>(geo, a, bh, 0, split, nrows, f_m, f_l, s_acc,
                        reinterpret_cast<float *>(smem + Sm::oRaw), &is_last);
}

}  // namespace

bool decode_tc_eligible(const Geom &geo)
{
    // every 8-row box must lie inside one run of the window: global part,
    // chosen spans (all full), local part and the current tokens start at
    // multiples of 8 rows
    const int64_t BH = int64_t(geo.B) * geo.Hkv;
    return geo.dtype == REATT_BF16 && geo.d == kDtD && int64_t(geo.g) * geo.C <= 8 &&
           geo.g_end % 8 == 0 && geo.S % 8 == 0 && geo.n_loc % 8 == 0 &&
           (geo.NS == 0 || geo.M % geo.S == 0) && BH * geo.Ts + 8 < (int64_t(1) << 31) &&
           BH * geo.C + 8 < (int64_t(1) << 31);
}

cudaError_t launch_attend_decode_tc(const Geom &geo, const AttnArgs &a, int RP, const void *kc,
                                    const void *vc, const void *kcur, const void *vcur, void *ws,
                                    cudaStream_t st)
{
    dim3 grid(unsigned(a.nsplit), 1u, unsigned(geo.B * geo.Hkv));
    const uint64_t BH = uint64_t(geo.B) * geo.Hkv;
    DtMaps mp;
    // an empty cache still needs valid maps: point them at the current tokens
    const bool has_cache = geo.T > 0;
    const void *kb = has_cache ? kc : kcur, *vb = has_cache ? vc : vcur;
    const uint64_t rows = has_cache ? BH * geo.Ts : BH * geo.C;
    for (int i = 0; i < 2; ++i)
        if (!encode_bf16_map(&mp.k[i], kb, rows, kDtD, uint32_t(dt_box_rows(i))) ||
            !encode_bf16_map(&mp.v[i], vb, rows, kDtD, uint32_t(dt_box_rows(i))))
            return cudaErrorInvalidValue;
    if (!encode_bf16_map(&mp.kq, kcur, BH * geo.C, kDtD, 8) ||
        !encode_bf16_map(&mp.vq, vcur, BH * geo.C, kDtD, 8))
        return cudaErrorInvalidValue;
#define REATT_DTC(RPV)                                                                         \
    do {                                                                                       \
        auto kern = attend_decode_tc_kernel<RPV>;                                              \
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                                             int(DtSmem::kBytes));                             \
        if (e != cudaSuccess) return e;                                                        \
        e = launch_pdl(kern, grid, dim3(kDtThreads), DtSmem::kBytes, st, mp, geo, a, ws);     \
        if (e != cudaSuccess) return e;                                                        \
    } while (0)
    switch (RP) {
    case 1: REATT_DTC(1); break;
    case 2: REATT_DTC(2); break;
    case 4: REATT_DTC(4); break;
    default: REATT_DTC(8); break;
    }
#undef REATT_DTC
    return cudaGetLastError();
}

}  // namespace reatt
