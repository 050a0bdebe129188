// Prefill span scoring on the 5th-generation tensor cores (tcgen05 + TMEM).
//
// For a chunk of C > 1 queries (chunked prefill) the span score of the
// decoding pseudocode becomes a contraction (ReAttention OpenReview
// discussion, "Prefilling Phase": score = query . key[global:-local]^T over
// the whole chunk):
//   s[t] = max_c sum_{j in group(h)} q[b,j,c,:] . k[b,h,t,:],
//   span_score = max over the span's tokens.
// The group's query vectors are summed in fp32 (linearity), and the fp32 sum
// is split into bf16 hi + lo terms (hi = bf16(s), lo = bf16(s - hi)); both
// terms accumulate into the same fp32 TMEM tile, so the product is exact to
// ~2^-17 relative -- one bf16 rounding of the sum would not be.  With g <= 2
// query heads per KV head the raw bf16 heads are the terms instead (exact).
//
// Kernel: one CTA per SM, persistent over (head, 256-token) items: two K tiles
// of 128 tokens share every query stage, halving the L2 bytes per MMA.
//   warp 0  : TMA producer (cp.async.bulk.tensor, 128B swizzle, no multicast);
//             two K stages, so the next item's tiles load while this one runs
//   warp 1  : TMEM allocation; one thread issues tcgen05.mma (M=128 tokens,
//             N=128 queries, K=16) per K tile into two accumulator sets in turn
//   warps 2-9: epilogue, two warps per TMEM lane group (one per K tile) --
//             tcgen05.ld of the accumulator rows (one token row per thread),
//             max over valid queries, then a segmented warp max over the
//             span's tokens; only span scores reach global memory.
// Every wait is bounded; a timeout records REATT_ETIMEOUT in the workspace.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "select.cuh"
#include "tc_ptx.cuh"

namespace reatt {

namespace {

using namespace tc;

constexpr int kTcEpiWarps = 8;       // two per TMEM lane group: one per K tile
constexpr int kTcThreads = (2 + kTcEpiWarps) * 32;   // warp 0 TMA, warp 1 MMA, epilogue
constexpr int kTileM = 128;          // tokens per tile = TMEM lanes
constexpr int kTiles = 2;            // token tiles per item: each query stage feeds both
constexpr int kTileN = 128;          // queries per MMA tile = TMEM columns
constexpr int kQStages = 3;          // query-tile ring
constexpr int kKStages = 2;          // K items: the next item's tiles load during this one
constexpr uint32_t kTmemCols = 512;  // two accumulator sets of kTiles x 128 columns

struct TcArgs {
    int64_t items;   // BH * ntiles
    int ntiles;      // items (kTiles x 128 tokens) per head
    int nqt;         // 128-query tiles
    int nterms;      // bf16 terms per query
    int cpad;        // nqt * 128
};

template <int D>
__global__ void __launch_bounds__(kTcThreads, 1)
scan_prefill_tc_kernel(const __grid_constant__ CUtensorMap kmap,
                       const __grid_constant__ CUtensorMap qmap, Geom geo, TcArgs ta,
                       float *__restrict__ scores, void *ws)
{
    constexpr int KS = D / 16;             // MMA k-steps over the head width
    constexpr int NBOX = D / 64;           // 64-element swizzle boxes per row
    constexpr uint32_t kKBytes = kTiles * NBOX * kBoxBytes;
    constexpr uint32_t kQBytes = NBOX * kBoxBytes;
    extern __shared__ uint8_t smem_raw[];
    // 128B-swizzled operand tiles want 1024-byte alignment
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    uint8_t *ksm = smem;
    uint8_t *qsm = smem + kKStages * kKBytes;
    uint64_t *bars = reinterpret_cast<uint64_t *>(qsm + kQStages * kQBytes);
    uint64_t *kfull = bars, *kempty = bars + kKStages;
    uint64_t *qfull = kempty + kKStages, *qempty = qfull + kQStages;
    uint64_t *accfull = qempty + kQStages, *accempty = accfull + 2, *done = accempty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(done + 1);
    __shared__ int abort_flag;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        abort_flag = 0;
        for (int s = 0; s < kKStages; ++s) {
            mbar_init(&kfull[s], 1);
            mbar_init(&kempty[s], 1);
        }
        for (int s = 0; s < kQStages; ++s) {
            mbar_init(&qfull[s], 1);
            mbar_init(&qempty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&accfull[s], 1);
            mbar_init(&accempty[s], kTcEpiWarps);   // one arrival per epilogue warp
        }
        mbar_init(done, 1);
        mbar_init_fence();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    auto fail = [&]() {
        report_status(ws, REATT_ETIMEOUT);
        *(volatile int *)&abort_flag = 1;
    };
    auto aborted = [&]() { return *(volatile int *)&abort_flag != 0; };

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t kuse = 0, qn = 0;
            bool ok = true;
            for (int64_t it = blockIdx.x; ok && it < ta.items; it += gridDim.x) {
                const int64_t bh = it / ta.ntiles;
                const int tile = int(it % ta.ntiles);
                const int y = int(bh * geo.Ts + geo.G + int64_t(tile) * kTiles * kTileM);
                const int ks_ = int(kuse % kKStages);
                const uint32_t kround = kuse / kKStages;
                if (kround > 0 && (aborted() || !mbar_wait_bounded(&kempty[ks_], (kround - 1) & 1, kWaitLimitNs))) {
                    fail();
                    ok = false;
                    break;
                }
                mbar_arrive_expect_tx(&kfull[ks_], kKBytes);
                for (int t = 0; t < kTiles; ++t)
                    for (int bx = 0; bx < NBOX; ++bx)
                        tma_load_2d(ksm + ks_ * kKBytes + (t * NBOX + bx) * kBoxBytes, &kmap,
                                    64 * bx, y + t * kTileM, &kfull[ks_]);
                ++kuse;
                for (int qt = 0; ok && qt < ta.nqt; ++qt)
                    for (int term = 0; term < ta.nterms; ++term, ++qn) {
                        const int st = int(qn % kQStages);
                        const uint32_t use = qn / kQStages;
                        if (use > 0 && (aborted() || !mbar_wait_bounded(&qempty[st], (use - 1) & 1, kWaitLimitNs))) {
                            fail();
                            ok = false;
                            break;
                        }
                        const int qy = int((bh * ta.nterms + term) * ta.cpad + int64_t(qt) * kTileN);
                        mbar_arrive_expect_tx(&qfull[st], kQBytes);
                        for (int bx = 0; bx < NBOX; ++bx)
                            tma_load_2d(qsm + st * kQBytes + bx * kBoxBytes, &qmap, 64 * bx, qy,
                                        &qfull[st]);
                    }
            }
            // drain: the last K loads and the last query loads have landed
            for (uint32_t m = kuse > kKStages ? kuse - kKStages : 0; m < kuse; ++m)
                if (!mbar_wait_bounded(&kfull[m % kKStages], (m / kKStages) & 1, kWaitLimitNs)) fail();
            for (uint32_t m = qn > kQStages ? qn - kQStages : 0; m < qn; ++m)
                if (!mbar_wait_bounded(&qfull[m % kQStages], (m / kQStages) & 1, kWaitLimitNs)) fail();
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            uint32_t kuse = 0, qn = 0, an = 0;
            bool ok = true;
            for (int64_t it = blockIdx.x; ok && it < ta.items; it += gridDim.x) {
                const int ks_ = int(kuse % kKStages);
                if (aborted() || !mbar_wait_bounded(&kfull[ks_], (kuse / kKStages) & 1, kWaitLimitNs)) {
                    fail();
                    break;
                }
                ++kuse;
                const uint8_t *kst = ksm + ks_ * kKBytes;
                tc_fence_after();
                for (int qt = 0; ok && qt < ta.nqt; ++qt, ++an) {
                    const int acc = int(an & 1);
                    const uint32_t ause = an >> 1;
                    if (ause > 0 && (aborted() || !mbar_wait_bounded(&accempty[acc], (ause - 1) & 1, kWaitLimitNs))) {
                        fail();
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t d_tmem = tmem_base + uint32_t(acc * kTiles * kTileN);
                    for (int term = 0; term < ta.nterms; ++term, ++qn) {
                        const int st = int(qn % kQStages);
                        if (aborted() || !mbar_wait_bounded(&qfull[st], (qn / kQStages) & 1, kWaitLimitNs)) {
                            fail();
                            ok = false;
                            break;
                        }
                        tc_fence_after();
#pragma unroll
                        for (int t = 0; t < kTiles; ++t)
#pragma unroll
                            for (int ks = 0; ks < KS; ++ks) {
                                const int bx = ks / 4, kin = ks % 4;   // box, 32-byte step inside it
                                const uint64_t adesc =
                                    sw128_desc(kst + (t * NBOX + bx) * kBoxBytes) + uint64_t(kin * 2);
                                const uint64_t bdesc =
                                    sw128_desc(qsm + st * kQBytes + bx * kBoxBytes) + uint64_t(kin * 2);
                                tc_mma(d_tmem + uint32_t(t * kTileN), adesc, bdesc,
                                       idesc_bf16(kTileM, kTileN), (term | ks) != 0 ? 1u : 0u);
                            }
                        tc_commit(&qempty[st]);   // stage free once these MMAs are done
                    }
                    if (ok) tc_commit(&accfull[acc]);
                }
                if (ok) tc_commit(&kempty[ks_]);
            }
            // every MMA issued so far has completed before TMEM is released
            tc_commit(done);
            if (!mbar_wait_bounded(done, 0, kWaitLimitNs)) fail();
        }
    } else {
        // ------------------------------------------------ epilogue (256 threads)
        static_assert(kTcEpiWarps == 4 * kTiles, "one warp per lane group and K tile");
        const int quad = warp & 3;              // TMEM lane quadrant of this warp
        const int t = (warp - 2) >> 2;          // K tile of this warp
        const int row = quad * 32 + lane;       // token row in the tile
        uint32_t an = 0;
        for (int64_t it = blockIdx.x; it < ta.items; it += gridDim.x) {
            const int64_t bh = it / ta.ntiles;
            const int tile = int(it % ta.ntiles);
            float tokmax = -INFINITY;
            bool ok = true;
            for (int qt = 0; qt < ta.nqt; ++qt, ++an) {
                const int acc = int(an & 1);
                const bool got = !aborted() &&
                                 mbar_wait_bounded(&accfull[acc], (an >> 1) & 1, kWaitLimitNs);
                if (!__all_sync(0xffffffffu, got)) {
                    if (lane == 0) fail();
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t taddr = tmem_base + (uint32_t(quad * 32) << 16) +
                                       uint32_t((acc * kTiles + t) * kTileN);
                if ((qt + 1) * kTileN <= geo.C) {   // every query of the tile is real
#pragma unroll
                    for (int ch = 0; ch < kTileN / 32; ++ch) {
                        float v[32];
                        tmem_ld32(taddr + uint32_t(ch * 32), v);
#pragma unroll
                        for (int j = 0; j < 32; ++j) tokmax = fmaxf(tokmax, v[j]);
                    }
                } else {
#pragma unroll
                    for (int ch = 0; ch < kTileN / 32; ++ch) {
                        float v[32];
                        tmem_ld32(taddr + uint32_t(ch * 32), v);
                        const int c0 = qt * kTileN + ch * 32;
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            if (c0 + j < geo.C) tokmax = fmaxf(tokmax, v[j]);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&accempty[acc]);
            }
            if (!ok) break;
            // span max: S divides 32, tiles start on span boundaries
            const int64_t moff = (int64_t(tile) * kTiles + t) * kTileM + row;
            float val = moff < geo.M ? tokmax : -INFINITY;
            for (int o = 1; o < geo.S; o <<= 1) val = fmaxf(val, __shfl_xor_sync(0xffffffffu, val, o));
            if (moff < geo.M && (lane % geo.S) == 0) scores[bh * geo.NS + moff / geo.S] = val;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, kTmemCols);
}

// ---------------------------------------------------------------- query-resident form
// The same contraction with the roles of the operands swapped: two 128-query
// tiles' terms sit in TMEM as A operands (M = 128 queries each, loaded once
// per item) and the keys stream through a deep shared-memory ring as the B
// operand (N = 128 tokens), so every 32 KB key tile feeds the products of
// 256 queries: half the bytes per product that reach shared memory in the
// key-resident form above, which the transfers from L2 bound.  An item is
// (chunk of key tiles, KV head, pair of query tiles), pair fastest;
// CTAs take items round-robin, so the query tiles of one head stream the same
// key chunk from L2 at about the same time.  Span maxima over the item's
// queries are folded into global order codes with atomicMax (the codes start
// at 0, below every float's code), max over all query tiles.  Used for S = 32.
// The chunk is sized for about six items per CTA (32 to 128 key tiles): larger
// items reload the query terms less often, smaller ones balance the last wave.
//   warp 0  : TMA producer, one 128-token key tile per ring stage
//   warps 1, 10: one thread each issues the products of one query slot
//             (M128 x N128 x K16, A from TMEM) per key tile into that slot's
//             accumulator.  The tensor pipe queues only an MMA or two and an
//             mbarrier wait stalls the issuing thread for ~140 cycles, so each
//             slot has its own thread (while one waits, the other's products
//             keep the pipe busy).  Each first reads a shared-memory counter
//             (one acquire load): `landed` (key tiles in shared memory) or
//             `released` (accumulator reads done); only when the count is not
//             there yet does it wait on the matching mbarrier, which suspends
//             the thread instead of spinning.  Warp 1 also allocates TMEM.
//   warp 11 : waits on each key stage's TMA barrier in order and publishes
//             the landed count
//   warps 2-9: warp (lane group q, slot s) stores its rows' query terms of
//             slot s into TMEM at each item, then per key tile reduces its 32
//             rows x 128 tokens of slot s to four span maxima (max over the
//             tokens, then over the warp's queries) and folds them in.
constexpr int kQrThreads = (4 + 8) * 32;   // TMA, issuer 0, 8 epilogue warps, issuer 1, watcher
constexpr int kQrIssuer1 = 10;
constexpr int kQrWatcher = 11;
constexpr int kQrStages = 6;            // key tiles in flight
constexpr int kQrChunkMin = 32, kQrChunkMax = 128;   // key tiles per item
constexpr int kQrFilterChunk = 16;                    // listed key tiles per item (exact pass)
constexpr uint32_t kQrQ = 0;            // query terms of slot s at columns 128*s
constexpr uint32_t kQrAcc = 256;        // accumulator of slot s at columns 256 + 128*s

struct QrArgs {
    int64_t items;   // nkc * BH * npair
    int chunk;       // key tiles per item
    int nkt;         // 128-token key tiles per head
    int nqt;         // 128-query tiles
    int npair;       // pairs of query tiles
    int nterms;      // bf16 terms per query used by the products
    int tstride;     // terms per query in the terms buffer (>= nterms)
    int cpad;        // nqt * 128
    // Optional tile list: key tile kt of head bh is tile tiles[bh*nkt + kt],
    // for kt < ntile[bh] only (null: kt itself, for every kt < nkt).
    const int32_t *tiles;
    const int32_t *ntile;
};

template <int D>
__global__ void __launch_bounds__(kQrThreads, 1)
scan_prefill_tcq_kernel(const __grid_constant__ CUtensorMap kmap, Geom geo, QrArgs qa,
                        const __nv_bfloat16 *__restrict__ terms, uint32_t *__restrict__ codes,
                        void *ws)
{
    constexpr int KS = D / 16;
    constexpr int NBOX = D / 64;
    constexpr uint32_t kKBytes = NBOX * kBoxBytes;   // one 128-token key tile
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kQrStages * kKBytes);
    uint64_t *kfull = bars, *kempty = kfull + kQrStages, *qfull = kempty + kQrStages,
             *qempty = qfull + 2, *accfull = qempty + 2, *accempty = accfull + 2,
             *done = accempty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(done + 2);
    __shared__ int abort_flag;
    __shared__ int landed, released[2];   // key tiles landed; accumulator reads done (per slot)

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        abort_flag = 0;
        landed = 0;
        released[0] = released[1] = 0;
        for (int s = 0; s < kQrStages; ++s) {
            mbar_init(&kfull[s], 1);
            mbar_init(&kempty[s], 2);     // both issuing threads commit
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&qfull[s], 4);      // slot s's query terms stored (its four warps)
            mbar_init(&qempty[s], 1);     // the products that read slot s's terms are complete
            mbar_init(&accfull[s], 1);
            mbar_init(&accempty[s], 4);   // slot s's accumulator read by its four warps
        }
        mbar_init(&done[0], 1);
        mbar_init(&done[1], 1);
        mbar_init_fence();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    pdl_wait();   // the query terms and the zeroed codes come from the preceding launch
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    auto fail = [&]() {
        report_status(ws, REATT_ETIMEOUT);
        *(volatile int *)&abort_flag = 1;
    };
    auto aborted = [&]() { return *(volatile int *)&abort_flag != 0; };
    const int BH = geo.B * geo.Hkv;
    // item -> (key chunk, KV head, query pair) and its key tiles [k0, k1)
    auto decode = [&](int64_t it, int64_t &bh, int &pair, int &k0, int &k1) {
        const int64_t per_chunk = int64_t(BH) * qa.npair;
        const int kc = int(it / per_chunk);
        const int64_t r = it % per_chunk;
        bh = r / qa.npair;
        pair = int(r % qa.npair);
        k0 = kc * qa.chunk;
        const int kend = qa.ntile ? __ldg(qa.ntile + bh) : qa.nkt;
        k1 = k0 + qa.chunk < kend ? k0 + qa.chunk : kend;
    };
    // key tile kt of head bh
    auto tile_of = [&](int64_t bh, int kt) {
        return qa.tiles ? __ldg(qa.tiles + bh * qa.nkt + kt) : kt;
    };

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t kn = 0;
            bool ok = true;
            for (int64_t it = blockIdx.x; ok && it < qa.items; it += gridDim.x) {
                int64_t bh;
                int pair, k0, k1;
                decode(it, bh, pair, k0, k1);
                for (int kt = k0; kt < k1; ++kt, ++kn) {   // (an empty item issues nothing)
                    const int st = int(kn % kQrStages);
                    const uint32_t use = kn / kQrStages;
                    if (use > 0 && (aborted() || !mbar_wait_bounded(&kempty[st], (use - 1) & 1, kWaitLimitNs))) {
                        fail();
                        ok = false;
                        break;
                    }
                    const int y = int(bh * geo.Ts + geo.G + int64_t(tile_of(bh, kt)) * kTileM);
                    mbar_arrive_expect_tx(&kfull[st], kKBytes);
                    for (int bx = 0; bx < NBOX; ++bx)
                        tma_load_2d(smem + st * kKBytes + bx * kBoxBytes, &kmap, 64 * bx, y, &kfull[st]);
                }
            }
            for (uint32_t m = kn > kQrStages ? kn - kQrStages : 0; m < kn; ++m)
                if (!mbar_wait_bounded(&kfull[m % kQrStages], (m / kQrStages) & 1, kWaitLimitNs)) fail();
        }
    } else if (warp == 1 || warp == kQrIssuer1) {
        // ------------------------------------------------ MMA issuer of one query slot
        if (lane == 0) {
            const int sl = warp == 1 ? 0 : 1;
            const uint32_t id = idesc_bf16(kTileM, kTileN);
            const uint32_t d = tmem_base + kQrAcc + uint32_t(sl * kTileN);
            const uint32_t tq = tmem_base + kQrQ + uint32_t(sl * 128);
            uint32_t kn = 0, nt = 0, nq = 0;
            bool ok = true;
            for (int64_t it = blockIdx.x; ok && it < qa.items; it += gridDim.x) {
                int64_t bh;
                int pair, k0, k1;
                decode(it, bh, pair, k0, k1);
                if (k0 >= k1) continue;   // empty item (tile list): skipped by every role
                // without a second query tile, slot 1 only releases the key stages
                const bool mine = 2 * pair + sl < qa.nqt;
                if (mine) {
                    if (aborted() || !mbar_wait_bounded(&qfull[sl], nq & 1, kWaitLimitNs)) {
                        fail();
                        break;
                    }
                    tc_fence_after();
                }
                for (int kt = k0; kt < k1; ++kt, ++kn) {
                    const int st = int(kn % kQrStages);
                    // key tile kn landed; slot's previous accumulator read by its four warps
                    if (aborted() ||
                        (ld_acquire_shared(&landed) < int(kn) + 1 &&
                         !mbar_wait_bounded(&kfull[st], (kn / kQrStages) & 1, kWaitLimitNs)) ||
                        (mine && nt > 0 && ld_acquire_shared(&released[sl]) < 4 * int(nt) &&
                         !mbar_wait_bounded(&accempty[sl], (nt - 1) & 1, kWaitLimitNs))) {
                        fail();
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    if (mine) {
                        const uint8_t *kst = smem + st * kKBytes;
                        for (int term = 0; term < qa.nterms; ++term)
#pragma unroll
                            for (int ks = 0; ks < KS; ++ks) {
                                const int bx = ks / 4, kin = ks % 4;
                                const uint64_t kd = sw128_desc(kst + bx * kBoxBytes) + uint64_t(kin * 2);
                                tc_mma_ts(d, tq + uint32_t(term * (D / 2) + ks * 8), kd, id,
                                          (term | ks) != 0 ? 1u : 0u);
                            }
                        tc_commit(&accfull[sl]);
                        ++nt;
                    }
                    tc_commit(&kempty[st]);   // this thread's products of the stage are done
                }
                if (!ok) break;
                if (mine) {
                    tc_commit(&qempty[sl]);   // the slot's terms free once this item's products are done
                    ++nq;
                }
            }
            tc_commit(&done[sl]);
            if (!mbar_wait_bounded(&done[sl], 0, kWaitLimitNs)) fail();
        }
    } else if (warp == kQrWatcher) {
        // ------------------------------------------------ landed count of the key ring
        if (lane == 0) {
            uint32_t kn = 0;
            bool ok = true;
            for (int64_t it = blockIdx.x; ok && it < qa.items; it += gridDim.x) {
                int64_t bh;
                int pair, k0, k1;
                decode(it, bh, pair, k0, k1);
                for (int kt = k0; kt < k1; ++kt, ++kn) {
                    if (aborted() ||
                        !mbar_wait_bounded(&kfull[kn % kQrStages], (kn / kQrStages) & 1, kWaitLimitNs)) {
                        fail();
                        ok = false;
                        break;
                    }
                    st_release_shared(&landed, int(kn) + 1);
                }
            }
        }
    } else {
        // ------------------------------------------------ query terms + span maxima (256 threads)
        const int quad = warp & 3;               // TMEM lane group: query rows [32*quad, +32)
        const int sl = (warp - 2) >> 2;          // query slot of this warp
        const int row = quad * 32 + lane;
        const uint32_t lane_base = tmem_base + (uint32_t(quad * 32) << 16);
        uint32_t nt = 0, nq = 0;
        bool ok = true;
        for (int64_t it = blockIdx.x; ok && it < qa.items; it += gridDim.x) {
            int64_t bh;
            int pair, k0, k1;
            decode(it, bh, pair, k0, k1);
            if (k0 >= k1) continue;              // empty item (tile list)
            const int qt = 2 * pair + sl;
            if (qt >= qa.nqt) continue;          // no second query tile in this pair
            // this row's query terms into slot sl, once the previous item's
            // products that read the slot are complete (rows >= C are 0)
            if (nq > 0) {
                const bool got = !aborted() &&
                                 mbar_wait_bounded(&qempty[sl], (nq - 1) & 1, kWaitLimitNs);
                if (!__all_sync(0xffffffffu, got)) {
                    if (lane == 0) fail();
                    break;
                }
                tc_fence_after();
            }
            for (int term = 0; term < qa.nterms; ++term) {
                const __nv_bfloat16 *src =
                    terms + ((bh * qa.tstride + term) * qa.cpad + int64_t(qt) * kTileN + row) * D;
                const uint32_t tq = lane_base + kQrQ + uint32_t(sl * 128 + term * (D / 2));
#pragma unroll
                for (int c = 0; c < D / 64; ++c) {
                    float w[32];
                    const uint4 *s4 = reinterpret_cast<const uint4 *>(src + c * 64);
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const uint4 v = s4[e];
                        w[4 * e] = __uint_as_float(v.x);
                        w[4 * e + 1] = __uint_as_float(v.y);
                        w[4 * e + 2] = __uint_as_float(v.z);
                        w[4 * e + 3] = __uint_as_float(v.w);
                    }
                    tmem_st32(tq + uint32_t(c * 32), w);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&qfull[sl]);
            ++nq;
            const bool valid_q = qt * kTileN + row < geo.C;
            for (int kt = k0; kt < k1; ++kt, ++nt) {
                const bool got = !aborted() &&
                                 mbar_wait_bounded(&accfull[sl], nt & 1, kWaitLimitNs);
                if (!__all_sync(0xffffffffu, got)) {
                    if (lane == 0) fail();
                    ok = false;
                    break;
                }
                tc_fence_after();
                uint32_t r[4][32];
                const uint32_t ta = lane_base + kQrAcc + uint32_t(sl * kTileN);
#pragma unroll
                for (int c = 0; c < 4; ++c) tmem_ld32_nowait(ta + uint32_t(c * 32), r[c]);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 4; ++c) tmem_regs_after_wait(r[c]);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {   // the scores are in registers
                    red_release_add_shared(&released[sl], 1);
                    mbar_arrive(&accempty[sl]);
                }
                // four spans of 32 tokens: middle offsets t0 .. t0 + 127; this
                // row's max over each span's tokens
                const int64_t t0 = int64_t(tile_of(bh, kt)) * kTileM;
                float m[4];
#pragma unroll
                for (int sp = 0; sp < 4; ++sp) {
                    const int64_t ts = t0 + sp * 32;
                    float pm[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
                    if (ts + 32 <= geo.M) {
#pragma unroll
                        for (int e = 0; e < 32; ++e) pm[e & 3] = fmaxf(pm[e & 3], __uint_as_float(r[sp][e]));
                    } else {
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            if (ts + e < geo.M) pm[e & 3] = fmaxf(pm[e & 3], __uint_as_float(r[sp][e]));
                    }
                    m[sp] = valid_q ? fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])) : -INFINITY;
                }
                // max over the warp's 32 rows for all four spans at once: two
                // halving exchanges leave each lane one span (2*bit4 + bit3 of
                // its lane id), three more finish the max over all rows
                const bool u16 = (lane & 16) != 0, u8 = (lane & 8) != 0;
                float a0 = u16 ? m[2] : m[0], a1 = u16 ? m[3] : m[1];
                a0 = fmaxf(a0, __shfl_xor_sync(0xffffffffu, u16 ? m[0] : m[2], 16));
                a1 = fmaxf(a1, __shfl_xor_sync(0xffffffffu, u16 ? m[1] : m[3], 16));
                float mx = fmaxf(u8 ? a1 : a0, __shfl_xor_sync(0xffffffffu, u8 ? a0 : a1, 8));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
                if ((lane & 7) == 0) {
                    const int64_t ts = t0 + (2 * int(u16) + int(u8)) * 32;
                    if (ts < geo.M && mx != -INFINITY)
                        atomicMax(&codes[bh * geo.NS + ts / 32], order_code(mx));
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, 512);
}

// bf16 terms of the summed group query: [BH][NT][cpad][D]; rows c >= C are 0.
// One thread per (KV head, query, 4 consecutive dims): the group sum is formed
// once for both terms (grid.y = KV head; 32-bit index arithmetic).
template <int D>
__global__ void qterms_kernel(Geom geo, const uint16_t *__restrict__ q,
                              __nv_bfloat16 *__restrict__ out, int nterms, int cpad,
                              uint32_t *__restrict__ zero_codes, uint32_t *__restrict__ qnorm)
{
    constexpr int D4 = D / 4;
    const int x = blockIdx.x * blockDim.x + threadIdx.x;
    const int bh = blockIdx.y;
    if (zero_codes)   // span codes of the query-resident scan start below every score
        for (int64_t s2 = x; s2 < geo.NS; s2 += int64_t(gridDim.x) * blockDim.x)
            zero_codes[bh * geo.NS + s2] = 0u;
    if (x >= cpad * D4) return;
    const int c = x / D4, i0 = (x % D4) * 4;
    const int b = bh / geo.Hkv, h = bh % geo.Hkv;
    float v[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    if (c < geo.C) {
        if (nterms == geo.g) {   // the group's raw heads: exact products
            for (int term = 0; term < nterms; ++term) {
                const uint2 w = *reinterpret_cast<const uint2 *>(
                    q + ((int64_t(b) * geo.Hq + h * geo.g + term) * geo.C + c) * D + i0);
                v[term][0] = bf16lo(w.x);
                v[term][1] = bf16hi(w.x);
                v[term][2] = bf16lo(w.y);
                v[term][3] = bf16hi(w.y);
            }
        } else {                 // fp32 sum split into hi + lo
            float sum[4] = {0.f, 0.f, 0.f, 0.f};
            for (int j = 0; j < geo.g; ++j) {
                const uint2 w = *reinterpret_cast<const uint2 *>(
                    q + ((int64_t(b) * geo.Hq + h * geo.g + j) * geo.C + c) * D + i0);
                sum[0] += bf16lo(w.x);
                sum[1] += bf16hi(w.x);
                sum[2] += bf16lo(w.y);
                sum[3] += bf16hi(w.y);
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float hi = __bfloat162float(__float2bfloat16_rn(sum[e]));
                v[0][e] = hi;
                v[1][e] = sum[e] - hi;
            }
        }
    }
    float ss[2] = {0.f, 0.f};   // squares of the stored hi and lo terms
    for (int term = 0; term < nterms; ++term) {
        __nv_bfloat162 lo2 = __floats2bfloat162_rn(v[term][0], v[term][1]);
        __nv_bfloat162 hi2 = __floats2bfloat162_rn(v[term][2], v[term][3]);
        uint2 w;
        w.x = *reinterpret_cast<const uint32_t *>(&lo2);
        w.y = *reinterpret_cast<const uint32_t *>(&hi2);
        *reinterpret_cast<uint2 *>(out + ((int64_t(bh) * nterms + term) * cpad + c) * D + i0) = w;
        const float e0 = bf16lo(w.x), e1 = bf16hi(w.x), e2 = bf16lo(w.y), e3 = bf16hi(w.y);
        ss[term & 1] += e0 * e0 + e1 * e1 + e2 * e2 + e3 * e3;
    }
    if (qnorm) {   // max over the chunk's queries of ||q_hi|| and ||q_lo|| (D4 lanes per query)
        __shared__ float wmax[2][32];
#pragma unroll
        for (int o = D4 / 2; o >= 1; o >>= 1) {
            ss[0] += __shfl_xor_sync(0xffffffffu, ss[0], o);
            ss[1] += __shfl_xor_sync(0xffffffffu, ss[1], o);
        }
        float n0 = sqrtf(ss[0]), n1 = sqrtf(ss[1]);
#pragma unroll
        for (int o = D4; o < 32; o <<= 1) {   // the warp's other queries
            n0 = fmaxf(n0, __shfl_xor_sync(0xffffffffu, n0, o));
            n1 = fmaxf(n1, __shfl_xor_sync(0xffffffffu, n1, o));
        }
        const int warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
        if ((threadIdx.x & 31) == 0) {
            wmax[0][warp] = n0;
            wmax[1][warp] = n1;
        }
        __syncthreads();   // whole blocks reach here (cpad * D4 is a multiple of 256)
        if (threadIdx.x == 0) {   // non-negative floats order like their bit patterns
            for (int w2 = 1; w2 < nw; ++w2) {
                n0 = fmaxf(n0, wmax[0][w2]);
                n1 = fmaxf(n1, wmax[1][w2]);
            }
            atomicMax(qnorm + 2 * bh, __float_as_uint(n0));
            atomicMax(qnorm + 2 * bh + 1, __float_as_uint(n1));
        }
    }
}

// ---------------------------------------------------------------- two-pass filter
// The fused step needs only the selection, so with hi/lo query terms the
// scan runs twice: once with the hi terms alone over every key tile, and
// once with hi + lo over the key tiles that hold a span the first pass
// cannot rule out.  For a query c and key t the two passes' products differ
// by q_lo[c].k_t plus the rounding of two fp32 accumulations, so a span's
// exact maximum lies within E_sp = (max_c ||q_lo[c]|| + a 2^-14 max_c
// ||q_hi[c]|| rounding allowance) * max_{t in sp} ||k_t|| of its hi-only
// maximum.  A span whose upper bound stays below the k-th largest lower
// bound cannot be among the k largest exact maxima (each of the k spans with
// the largest lower bounds has an exact maximum at least that large), so
// only the other spans' tiles are scanned again, with the same products as
// the one-pass scan.

// kn[bh][sp] = max over the span's tokens of ||k_t||_2 (fp32); block 0 also
// clears the per-head query norms that qterms_kernel raises.  One warp per
// span of 32 tokens, each load a contiguous 512 (D = 128) or 256 bytes.
template <int D>
__global__ void __launch_bounds__(256)
span_knorm_kernel(Geom geo, const uint16_t *__restrict__ kc, float *__restrict__ kn,
                  uint32_t *__restrict__ qnorm)
{
    constexpr int CPT = D * 2 / 16;   // 16-byte chunks per token
    constexpr int TPL = 32 / CPT;     // tokens per warp load
    const int lane = threadIdx.x & 31;
    const int64_t BH = int64_t(geo.B) * geo.Hkv;
    if (blockIdx.x == 0)
        for (int i = threadIdx.x; i < 2 * BH; i += blockDim.x) qnorm[i] = 0u;
    const int64_t wid = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    if (wid >= BH * geo.NS) return;   // whole warps
    const int64_t bh = wid / geo.NS, sp = wid % geo.NS;
    const int64_t t0 = sp * 32;       // middle offset of the span's first token
    const uint4 *src = reinterpret_cast<const uint4 *>(kc + (bh * geo.Ts + geo.G + t0) * D);
    float mx = 0.f;
#pragma unroll 4
    for (int j = 0; j < CPT; ++j) {
        const int tok = j * TPL + lane / CPT;
        float ss = 0.f;
        if (t0 + tok < geo.M) {
            const uint4 w = __ldg(src + j * 32 + lane);
            const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float a0 = bf16lo(ws[e]), a1 = bf16hi(ws[e]);
                ss = fmaf(a0, a0, fmaf(a1, a1, ss));
            }
        }
#pragma unroll
        for (int o = CPT / 2; o >= 1; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        mx = fmaxf(mx, ss);
    }
#pragma unroll
    for (int o = 16; o >= CPT; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0) kn[bh * geo.NS + sp] = sqrtf(mx);
}

constexpr int kCandThreads = 1024;
constexpr int kCandE = 8;             // spans per thread: NS <= 8192, key tiles <= 2048

// One CTA per (b, KV head): from the hi-only span codes, the span key norms
// and the query norms, the list of key tiles (ascending) that hold a span
// whose upper bound reaches the k-th largest lower bound; every span code is
// then reset to 0 for the exact pass.
__global__ void __launch_bounds__(kCandThreads)
prefill_candidates_kernel(Geom geo, uint32_t *__restrict__ codes, const float *__restrict__ kn,
                          const uint32_t *__restrict__ qnorm, int32_t *__restrict__ tiles,
                          int32_t *__restrict__ ntile, int nkt)
{
    __shared__ sel::Scratch rs;
    __shared__ uint32_t tmask[kCandThreads * kCandE / 4 / 32];
    auto bsync = [] { __syncthreads(); };
    const int t = threadIdx.x;
    const int64_t bh = blockIdx.x;
    const int NS = int(geo.NS);
    for (int i = t; i < kCandThreads * kCandE / 4 / 32; i += kCandThreads) tmask[i] = 0u;
    const float qh = __uint_as_float(qnorm[2 * bh]), ql = __uint_as_float(qnorm[2 * bh + 1]);
    // bound per unit key norm; the 2^-10 factors cover the norms' own fp32 rounding
    const float unit = (ql * 1.0009765625f + qh * 6.103515625e-05f) * 1.0009765625f;
    const int i0 = t * kCandE;
    const int mine = NS - i0 < 0 ? 0 : (NS - i0 > kCandE ? kCandE : NS - i0);
    uint32_t *hc = codes + bh * NS;
    uint32_t lbc[kCandE];
    float ub[kCandE];
#pragma unroll
    for (int e = 0; e < kCandE; ++e) {
        lbc[e] = 0u;
        ub[e] = -INFINITY;
        if (e < mine) {
            const uint32_t c = hc[i0 + e];
            const float ap = c ? order_decode(c) : -INFINITY;
            const float E = __fmul_ru(unit, kn[bh * NS + i0 + e]);
            lbc[e] = order_code(__fsub_rd(ap, E));
            ub[e] = __fadd_ru(ap, E);
        }
    }
    __syncthreads();   // the tile mask is clear
    uint32_t tau, take;
    const uint32_t kk = uint32_t(geo.k < NS ? geo.k : NS);
    sel::select_regs<kCandThreads, kCandE>(t, lbc, mine, kk, rs, tau, take, bsync);
    const float tauf = order_decode(tau);
#pragma unroll
    for (int e = 0; e < kCandE; ++e)
        if (e < mine && ub[e] >= tauf) {
            const int tl = (i0 + e) >> 2;   // 4 spans of 32 tokens per 128-token tile
            atomicOr(&tmask[tl >> 5], 1u << (tl & 31));
        }
#pragma unroll
    for (int e = 0; e < kCandE; ++e)
        if (e < mine) hc[i0 + e] = 0u;
    __syncthreads();
    const int ta = 2 * t, tb = 2 * t + 1;
    const int ma = ta < nkt && ((tmask[ta >> 5] >> (ta & 31)) & 1u);
    const int mb = tb < nkt && ((tmask[tb >> 5] >> (tb & 31)) & 1u);
    int total;
    const int pos = sel::exclusive_sum<kCandThreads>(t, ma + mb, rs, &total, bsync);
    int32_t *tl = tiles + bh * nkt;
    if (ma) tl[pos] = ta;
    if (mb) tl[pos + ma] = tb;
    if (t == 0) ntile[bh] = total;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder()
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

// 2-D bf16 map over `rows` rows of D elements, boxes of 128 rows x 64 elements.
bool make_map(CUtensorMap *m, const void *base, uint64_t rows, int D)
{
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {cuuint64_t(D), cuuint64_t(rows)};
    cuuint64_t strides[1] = {cuuint64_t(D) * 2};
    cuuint32_t box[2] = {64, 128};
    cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides,
               box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// span scores from order codes, in place
__global__ void decode_codes_kernel(float *__restrict__ scores, int64_t n)
{
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += int64_t(gridDim.x) * blockDim.x)
        scores[i] = order_decode(reinterpret_cast<const uint32_t *>(scores)[i]);
}

}  // namespace

bool prefill_tc_eligible(const Geom &geo)
{
    // bf16 inputs, a chunk of queries, spans that tile a 32-token warp
    return geo.dtype == REATT_BF16 && geo.C > 1 && (32 % geo.S) == 0 &&
           int64_t(geo.B) * geo.Hkv * geo.Ts < (int64_t(1) << 31);
}

static int tc_terms(const Geom &geo) { return geo.g <= 2 ? geo.g : 2; }

static size_t up256(size_t x) { return (x + 255) / 256 * 256; }

// The two-pass filter serves the fused step's query-resident scan with hi/lo
// query terms when one CTA can rank a head's spans and it pays.  Fitted to
// the step at 8 KV heads (costs scale with the heads): the hi-only pass saves
// ~22 us per query tile per 2,016 key tiles; the key-norm pass costs ~77 us
// per 2,016 key tiles; the exact pass ~40 + 0.9 k us per 16 query tiles
// (it scales with the listed tiles, ~1.5 k per head, not with the context);
// the candidate selection ~13 us.  Measured on a 2048-query chunk over 256K
// (filter on vs off): k = 64 +198 us, 128 +147, 256 +21, 512 -177, 1024 -486;
// over 64K with k = 64 -24 us; a 512-query chunk over 128K 260 vs 234 us.
static bool filter_eligible(const Geom &geo)
{
    if (!(geo.S == 32 && geo.g > 2 && tc_terms(geo) == 2 && geo.NS <= kCandThreads * kCandE &&
          geo.k > 0 && geo.k < geo.NS))
        return false;
    const double nqt = double((geo.C + kTileN - 1) / kTileN);
    const double nkt = double((geo.M + kTileM - 1) / kTileM);
    const double heads = double(geo.B) * geo.Hkv / 8.0;
    const double gain_us = heads * (22.0 * nqt * nkt / 2016.0 - 77.0 * nkt / 2016.0 -
                                    nqt / 16.0 * (40.0 + 0.9 * double(geo.k))) -
                           13.0;
    return gain_us > 20.0;
}

static size_t terms_bytes(const Geom &geo)
{
    const int cpad = (geo.C + kTileN - 1) / kTileN * kTileN;
    return size_t(geo.B) * geo.Hkv * tc_terms(geo) * cpad * geo.d * sizeof(__nv_bfloat16);
}

// Filter workspace after the terms: span key norms [BH][NS], query norms
// [BH][2], key tile lists [BH][nkt], list lengths [BH].
struct FilterWs {
    float *kn;
    uint32_t *qnorm;
    int32_t *tiles, *ntile;
};
static size_t filter_ws(const Geom &geo, void *scratch, FilterWs *f)
{
    const size_t BH = size_t(geo.B) * geo.Hkv;
    const size_t nkt = size_t((geo.M + kTileM - 1) / kTileM);
    size_t off = up256(terms_bytes(geo));
    uint8_t *base = static_cast<uint8_t *>(scratch);
    if (f) f->kn = reinterpret_cast<float *>(base + off);
    off = up256(off + BH * geo.NS * sizeof(float));
    if (f) f->qnorm = reinterpret_cast<uint32_t *>(base + off);
    off = up256(off + 2 * BH * sizeof(uint32_t));
    if (f) f->tiles = reinterpret_cast<int32_t *>(base + off);
    off = up256(off + BH * nkt * sizeof(int32_t));
    if (f) f->ntile = reinterpret_cast<int32_t *>(base + off);
    return off + BH * sizeof(int32_t);
}

size_t prefill_tc_ws_bytes(const Geom &geo)
{
    if (!prefill_tc_eligible(geo)) return 0;
    return filter_eligible(geo) ? filter_ws(geo, nullptr, nullptr) : terms_bytes(geo);
}

cudaError_t launch_prefill_tc(const Geom &geo, const void *q, const void *kc, float *scores,
                              void *ws, void *scratch, cudaStream_t st, bool *codes_left)
{
    const int nqt = (geo.C + kTileN - 1) / kTileN;
    const int cpad = nqt * kTileN;
    const int nterms = tc_terms(geo);
    const int BH = geo.B * geo.Hkv;
    if (int64_t(BH) * geo.NS == 0) return cudaSuccess;
    // the query-resident form serves 32-token spans (one span per 32 key columns)
    const bool qres = geo.S == 32;
    __nv_bfloat16 *terms = static_cast<__nv_bfloat16 *>(scratch);
    uint32_t *codes = reinterpret_cast<uint32_t *>(scores);
    // the fused step (which reads only the selection) takes the two-pass filter
    const bool two = qres && codes_left && filter_eligible(geo);
    FilterWs fw{};
    if (two) {
        filter_ws(geo, scratch, &fw);
        const int64_t threads = int64_t(BH) * geo.NS * 32;
        const unsigned blocks = unsigned((threads + 255) / 256);
        if (geo.d == 128)
            span_knorm_kernel<128><<<blocks, 256, 0, st>>>(geo, static_cast<const uint16_t *>(kc),
                                                           fw.kn, fw.qnorm);
        else
            span_knorm_kernel<64><<<blocks, 256, 0, st>>>(geo, static_cast<const uint16_t *>(kc),
                                                          fw.kn, fw.qnorm);
    }
    const dim3 qgrid(unsigned((cpad * (geo.d / 4) + 255) / 256), unsigned(BH));
    if (geo.d == 128)
        qterms_kernel<128><<<qgrid, 256, 0, st>>>(geo, static_cast<const uint16_t *>(q), terms,
                                                  nterms, cpad, qres ? codes : nullptr,
                                                  two ? fw.qnorm : nullptr);
    else
        qterms_kernel<64><<<qgrid, 256, 0, st>>>(geo, static_cast<const uint16_t *>(q), terms,
                                                 nterms, cpad, qres ? codes : nullptr,
                                                 two ? fw.qnorm : nullptr);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    CUtensorMap kmap;
    if (!make_map(&kmap, kc, uint64_t(geo.B) * geo.Hkv * geo.Ts, geo.d)) return cudaErrorInvalidValue;
    if (qres) {
        QrArgs qa;
        qa.nkt = int((geo.M + kTileM - 1) / kTileM);
        qa.nqt = nqt;
        qa.nterms = two ? 1 : nterms;   // the filter's first pass: hi terms only
        qa.tstride = nterms;
        qa.cpad = cpad;
        qa.npair = (nqt + 1) / 2;
        qa.tiles = nullptr;
        qa.ntile = nullptr;
        const int64_t per_tile = int64_t(BH) * qa.npair;   // items per key chunk
        {
            int64_t c = int64_t(qa.nkt) * per_tile / (int64_t(num_sms()) * 6);
            qa.chunk = int(c < kQrChunkMin ? kQrChunkMin : (c > kQrChunkMax ? kQrChunkMax : c));
            qa.items = int64_t((qa.nkt + qa.chunk - 1) / qa.chunk) * per_tile;
        }
        const size_t smem = 1024 + size_t(kQrStages) * (geo.d / 64) * kBoxBytes +
                            (2 * kQrStages + 10) * 8 + 16;
        auto run = [&](const QrArgs &a) {
            int grid = num_sms();
            if (a.items < grid) grid = int(a.items);
            cudaError_t r;
            if (geo.d == 128) {
                auto kern = scan_prefill_tcq_kernel<128>;
                r = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
                if (r == cudaSuccess)
                    r = launch_pdl(kern, dim3(grid), dim3(kQrThreads), smem, st, kmap, geo, a,
                                   static_cast<const __nv_bfloat16 *>(terms), codes, ws);
            } else {
                auto kern = scan_prefill_tcq_kernel<64>;
                r = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
                if (r == cudaSuccess)
                    r = launch_pdl(kern, dim3(grid), dim3(kQrThreads), smem, st, kmap, geo, a,
                                   static_cast<const __nv_bfloat16 *>(terms), codes, ws);
            }
            return r;
        };
        e = run(qa);
        if (e != cudaSuccess) return e;
        if (two) {
            // candidate key tiles, then the exact products over them only
            prefill_candidates_kernel<<<unsigned(BH), kCandThreads, 0, st>>>(
                geo, codes, fw.kn, fw.qnorm, fw.tiles, fw.ntile, qa.nkt);
            e = cudaGetLastError();
            if (e != cudaSuccess) return e;
            QrArgs q2 = qa;
            q2.nterms = nterms;
            q2.tiles = fw.tiles;
            q2.ntile = fw.ntile;
            q2.chunk = kQrFilterChunk;
            q2.items = int64_t((qa.nkt + q2.chunk - 1) / q2.chunk) * per_tile;
            e = run(q2);
            if (e != cudaSuccess) return e;
        }
        if (codes_left) {
            *codes_left = true;   // the caller reads order codes
        } else {
            const int64_t n = int64_t(BH) * geo.NS;
            decode_codes_kernel<<<unsigned((n + 255) / 256 < 1184 ? (n + 255) / 256 : 1184), 256, 0, st>>>(scores, n);
        }
        return cudaGetLastError();
    }
    TcArgs ta;
    ta.ntiles = int((geo.M + kTiles * kTileM - 1) / (kTiles * kTileM));
    ta.items = int64_t(BH) * ta.ntiles;
    ta.nqt = nqt;
    ta.cpad = cpad;
    ta.nterms = nterms;
    CUtensorMap qmap;
    if (!make_map(&qmap, terms, uint64_t(BH) * ta.nterms * ta.cpad, geo.d)) return cudaErrorInvalidValue;
    int grid = num_sms();
    if (ta.items < grid) grid = int(ta.items);
    const size_t box = kBoxBytes;
    const size_t smem = 1024 + (geo.d / 64) * box * (kKStages * kTiles + kQStages) +
                        (2 * kKStages + 2 * kQStages + 5) * 8 + 16;
    if (geo.d == 128) {
        auto kern = scan_prefill_tc_kernel<128>;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
        if (e != cudaSuccess) return e;
        kern<<<grid, kTcThreads, smem, st>>>(kmap, qmap, geo, ta, scores, ws);
    } else {
        auto kern = scan_prefill_tc_kernel<64>;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
        if (e != cudaSuccess) return e;
        kern<<<grid, kTcThreads, smem, st>>>(kmap, qmap, geo, ta, scores, ws);
    }
    return cudaGetLastError();
}

}  // namespace reatt
