// Block-wide k-th-largest selection on order codes, shared by the top-k
// kernels and the prefill scan's candidate filter.
//
// Every helper runs on NT participating threads with thread index t in
// [0, NT) and a barrier functor `sync` that synchronises exactly those
// threads (__syncthreads for a whole block, a named barrier for the consumer
// warps of a warp-specialised block).  Codes are the order-preserving uint32
// images of the scores (larger score -> larger code; 0 is below every real
// score and marks padding).
//
// Ties: the k_eff largest codes under the order (code desc, index asc) are
// chosen; the k-th code tau and how many codes equal to tau are taken
// (take_eq) define the set, and a stable compaction in index order emits the
// chosen indices ascending.
#pragma once

#include "common.cuh"

namespace reatt {
namespace sel {

constexpr int kBins = 2048;        // 11-bit digits
constexpr int kWarpResolve = 32;   // candidates one warp ranks directly

struct Scratch {
    uint32_t hist[kBins];
    uint32_t red[2][32];
    int wsum[33];
    uint32_t bcast[3];
    uint32_t cand[kWarpResolve];
    int ncand;
};

// Exclusive prefix sum of v over the NT threads; *total receives the sum.
template <int NT, class Sync>
__device__ __forceinline__ int exclusive_sum(int t, int v, Scratch &sc, int *total, Sync sync)
{
    constexpr int NW = NT / 32;
    const int lane = t & 31, warp = t >> 5;
    int inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int x = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += x;
    }
    if (lane == 31) sc.wsum[warp] = inc;
    sync();
    if (warp == 0) {
        const int w = lane < NW ? sc.wsum[lane] : 0;
        int winc = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int x = __shfl_up_sync(0xffffffffu, winc, o);
            if (lane >= o) winc += x;
        }
        if (lane < NW) sc.wsum[lane] = winc - w;
        if (lane == 31) sc.wsum[32] = winc;
    }
    sync();
    const int res = sc.wsum[warp] + inc - v;
    *total = sc.wsum[32];
    sync();
    return res;
}

template <int NT, class Sync>
__device__ __forceinline__ void minmax(int t, uint32_t mx, uint32_t mn, Scratch &sc,
                                       uint32_t &omax, uint32_t &omin, Sync sync)
{
    constexpr int NW = NT / 32;
    const int lane = t & 31, warp = t >> 5;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
        mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    }
    if (lane == 0) {
        sc.red[0][warp] = mx;
        sc.red[1][warp] = mn;
    }
    sync();
    mx = lane < NW ? sc.red[0][lane] : 0u;
    mn = lane < NW ? sc.red[1][lane] : 0xffffffffu;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
        mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    }
    omax = mx;
    omin = mn;
    sync();
}

// kk-th largest among the valid codes held in registers (thread t holds
// u[0..nvalid_mine)); 1 <= kk <= number of valid codes.  The high bits the
// largest and smallest code share are skipped; the rest is resolved with
// 11-bit digits, and once at most kWarpResolve codes share the digit prefix,
// one warp ranks them directly.
template <int NT, int E, class Sync>
__device__ void select_regs(int t, const uint32_t (&u)[E], int nvalid_mine, uint32_t kk,
                            Scratch &sc, uint32_t &tau, uint32_t &take_eq, Sync sync)
{
    uint32_t lmax = 0u, lmin = 0xffffffffu;
#pragma unroll
    for (int e = 0; e < E; ++e)
        if (e < nvalid_mine) {
            lmax = max(lmax, u[e]);
            lmin = min(lmin, u[e]);
        }
    uint32_t gmax, gmin;
    minmax<NT>(t, lmax, lmin, sc, gmax, gmin, sync);
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
    while (hb >= 0) {
        const int lo = hb >= 10 ? hb - 10 : 0;
        const int nb = hb - lo + 1;
        const uint32_t dmask = (1u << nb) - 1u;
        for (int i = t; i < (1 << nb); i += NT) sc.hist[i] = 0u;
        sync();
#pragma unroll
        for (int e = 0; e < E; ++e)
            if (e < nvalid_mine && (u[e] & mask) == prefix)
                atomicAdd(&sc.hist[(u[e] >> lo) & dmask], 1u);
        sync();
        // thread t owns bins in descending order: [(NT-1-t)*per, +per)
        const int per = ((1 << nb) + NT - 1) / NT;
        const int top = (NT - 1 - t) * per;   // lowest bin of this thread
        uint32_t local = 0;
        for (int j = 0; j < per; ++j) {
            const int bin = top + j;
            if (bin < (1 << nb)) local += sc.hist[bin];
        }
        int tot;
        const uint32_t above = uint32_t(exclusive_sum<NT>(t, int(local), sc, &tot, sync));
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
        sync();
        remaining -= sc.bcast[1];
        prefix |= sc.bcast[0] << lo;
        mask |= dmask << lo;
        hb = lo - 1;
        const uint32_t left = sc.bcast[2];
        sync();
        if (hb >= 0 && left <= uint32_t(kWarpResolve)) {
            // few codes share the prefix: one warp ranks them (the
            // remaining-th largest is tau)
#pragma unroll
            for (int e = 0; e < E; ++e)
                if (e < nvalid_mine && (u[e] & mask) == prefix)
                    sc.cand[atomicAdd(&sc.ncand, 1)] = u[e];
            sync();
            if (t < 32) {
                const int lane = t, n = sc.ncand;
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
            sync();
            tau = sc.bcast[0];
            take_eq = sc.bcast[1];
            sync();
            return;
        }
    }
    tau = prefix;
    take_eq = remaining;
}

// Stable compaction of register-held codes: thread t's codes have the
// indices i0 + e (contiguous, ascending with t); emit(pos, i0 + e) is called
// for every chosen code with pos ascending in the index.
template <int NT, int E, class Sync, class Emit>
__device__ void compact_regs(int t, const uint32_t (&u)[E], int nvalid_mine, uint32_t tau,
                             uint32_t take_eq, int i0, Scratch &sc, Emit emit, Sync sync)
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
    const int before = exclusive_sum<NT>(t, (n_eq << 16) | n_gt, sc, &tot, sync);
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

// ---- selection straight from memory (any n): 4 passes of 8 bits ----
struct MemScratch {
    uint32_t hist[256];
    uint32_t bcast[2];
    int wsum[33];
};

template <int NT, class Get, class Sync>
__device__ void select_mem(int t, Get get, int n, uint32_t kk, MemScratch &sc, uint32_t &tau,
                           uint32_t &take_eq, Sync sync)
{
    const int lane = t & 31;
    uint32_t prefix = 0, mask = 0, remaining = kk;
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int i = t; i < 256; i += NT) sc.hist[i] = 0u;
        sync();
        for (int base = 0; base < n; base += NT) {
            const int i = base + t;
            const uint32_t u = i < n ? get(i) : 0u;
            const bool hit = i < n && (u & mask) == prefix;
            const uint32_t bin = (u >> shift) & 255u;
            const unsigned peers = __match_any_sync(0xffffffffu, hit ? bin : 0x100u);
            if (hit && lane == __ffs(peers) - 1) atomicAdd(&sc.hist[bin], __popc(peers));
        }
        sync();
        if (t < 32) {
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
        sync();
        const uint32_t bin = sc.bcast[0], above = sc.bcast[1];
        remaining -= above;
        prefix |= bin << shift;
        mask |= 0xffu << shift;
        sync();
    }
    tau = prefix;
    take_eq = remaining;
}

// Prefix sum over NT threads for the memory path (its own scratch).
template <int NT, class Sync>
__device__ __forceinline__ int exclusive_sum_mem(int t, int v, int *wsum, int *total, Sync sync)
{
    constexpr int NW = NT / 32;
    const int lane = t & 31, warp = t >> 5;
    int inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int x = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += x;
    }
    if (lane == 31) wsum[warp] = inc;
    sync();
    if (warp == 0) {
        const int w = lane < NW ? wsum[lane] : 0;
        int winc = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int x = __shfl_up_sync(0xffffffffu, winc, o);
            if (lane >= o) winc += x;
        }
        if (lane < NW) wsum[lane] = winc - w;
        if (lane == 31) wsum[32] = winc;
    }
    sync();
    const int res = wsum[warp] + inc - v;
    *total = wsum[32];
    sync();
    return res;
}

// Stable compaction in index order over memory: every thread owns a
// contiguous run of elements; emit(pos, i) for every chosen i, pos ascending.
template <int NT, class Get, class Emit, class Sync>
__device__ void compact_mem(int t, Get get, int n, uint32_t tau, uint32_t take_eq,
                            MemScratch &sc, Emit emit, Sync sync)
{
    const int per = (n + NT - 1) / NT;
    const int i0 = t * per;
    const int i1 = i0 + per < n ? i0 + per : n;
    int n_gt = 0, n_eq = 0;
    for (int i = i0; i < i1; ++i) {
        const uint32_t u = get(i);
        n_gt += u > tau;
        n_eq += u == tau;
    }
    int tot;
    const int eq_before = exclusive_sum_mem<NT>(t, n_eq, sc.wsum, &tot, sync);
    int take = int(take_eq) - eq_before;
    take = take < 0 ? 0 : (take > n_eq ? n_eq : take);
    int pos = exclusive_sum_mem<NT>(t, n_gt + take, sc.wsum, &tot, sync);
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

}  // namespace sel
}  // namespace reatt
