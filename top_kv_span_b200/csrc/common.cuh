// Device helpers shared by the sm_100a kernels of the top-k span attention path.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "reatt.h"

namespace reatt {

// ----------------------------------------------------------------- geometry
// Derived sizes of one call (host-computed, passed by value to kernels).
struct Geom {
    int B, Hq, Hkv, g, d, C, G, L, S, k;
    int64_t T;
    int64_t Ts;         // cache rows per (b, KV head): T_cap, or T for dense caches
    int64_t g_end;      // min(G, T)
    int64_t loc_begin;  // max(G, T - L)
    int64_t n_loc;      // T - loc_begin if T > loc_begin else 0
    int64_t M;          // middle tokens
    int64_t NS;         // spans
    int64_t Wmax;       // G + k*S + L + C
    double base;        // RoPE base
    int dtype;          // reatt_dtype of q, caches, current tokens
    // RoPE frequency of pair i in half-turns, base^(-2i/d) / pi, computed on
    // the host in fp64 and split into fp32 hi + lo (hi + lo == value to ~2^-48)
    float rope_hi[64];
    float rope_lo[64];
};

// Workspace header: a status word kept at offset 0 of every workspace.
constexpr size_t kWsHeader = 256;

__device__ __forceinline__ void report_status(void *ws, uint32_t code)
{
    if (ws)
        atomicMax(reinterpret_cast<unsigned int *>(ws), code);
}

// ----------------------------------------------------------------- numbers
// bf16 pair (low half = lower address) -> two floats, exactly.
__device__ __forceinline__ float bf16lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

// Order-preserving map float -> uint32 (larger float -> larger code; every
// finite float and -inf maps above 0).
__device__ __forceinline__ uint32_t order_code(float f)
{
    uint32_t u = __float_as_uint(f + 0.0f);   // -0 -> +0: equal floats, equal codes
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float order_decode(uint32_t c)
{
    return __uint_as_float((c & 0x80000000u) ? (c & 0x7fffffffu) : ~c);
}

// Element type tag: float (fp32) or bf16 stored as uint16_t.
template <typename T> struct Elem;
template <> struct Elem<float> {
    static constexpr int kBytes = 4;
    static constexpr int kVec = 4;   // elements per 16-byte vector
    __device__ __forceinline__ static void unpack(const uint4 &v, float (&o)[4])
    {
        o[0] = __uint_as_float(v.x);
        o[1] = __uint_as_float(v.y);
        o[2] = __uint_as_float(v.z);
        o[3] = __uint_as_float(v.w);
    }
    __device__ __forceinline__ static float one(const float *p, int64_t i) { return p[i]; }
};
template <> struct Elem<uint16_t> {
    static constexpr int kBytes = 2;
    static constexpr int kVec = 8;
    __device__ __forceinline__ static void unpack(const uint4 &v, float (&o)[8])
    {
        o[0] = bf16lo(v.x); o[1] = bf16hi(v.x);
        o[2] = bf16lo(v.y); o[3] = bf16hi(v.y);
        o[4] = bf16lo(v.z); o[5] = bf16hi(v.z);
        o[6] = bf16lo(v.w); o[7] = bf16hi(v.w);
    }
    __device__ __forceinline__ static float one(const uint16_t *p, int64_t i)
    {
        return __uint_as_float(static_cast<uint32_t>(p[i]) << 16);
    }
};

// 16-byte global load through the read-only path, not kept in L1.
__device__ __forceinline__ uint4 ldg_stream(const void *p)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// ----------------------------------------------------------------- RoPE
// cos/sin of pos * base^(-2i/d) in fp32 only.  The frequency comes as an
// unevaluated sum hi + lo (half-turns).  pos*hi is split exactly into its
// rounded value and the rounding error (fma), the rounded value is reduced
// modulo 2 exactly (even-integer subtraction of a nearby float), and the small
// terms are added back, so the reduced argument carries ~1 ulp error on
// [-1, 1] for positions below 2^24; sincospif then evaluates it.
__device__ __forceinline__ void rope_cs(int64_t pos, float hi, float lo, float &c, float &s)
{
    const float p = static_cast<float>(pos);          // exact for pos < 2^24
    const float ph = p * hi;
    const float pe = fmaf(p, hi, -ph);                 // exact error of p*hi
    const float r = ph - 2.0f * rintf(0.5f * ph);      // exact, |r| <= 1
    sincospif(r + fmaf(p, lo, pe), &s, &c);
}

// ----------------------------------------------------------------- mbarrier / bulk copy
__device__ __forceinline__ uint32_t smem_addr(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint64_t global_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
                 : "memory");
}
__device__ __forceinline__ void mbar_init_fence()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// Non-blocking test: has the phase with the given parity completed?
__device__ __forceinline__ bool mbar_test(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// Wait for the phase with the given parity to complete; gives up after
// limit_ns of wall time and returns false.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity, uint64_t limit_ns)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const uint64_t t0 = global_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_ns() - t0 > limit_ns)
            return false;
    }
    return true;
}
// L2 policy: data read once (streamed K) is the first to be evicted.
__device__ __forceinline__ uint64_t l2_evict_first_policy()
{
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}
// Bulk (non-tensor) async copy global -> shared; completion is signalled on
// the mbarrier as transaction bytes.  dst, src 16-byte aligned, bytes % 16 == 0.
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar,
                                          uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1], %2, [%3], %4;" ::"r"(smem_addr(dst)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar)), "l"(policy)
        : "memory");
}

// Same without an L2 policy (data that may be read again stays cacheable).
__device__ __forceinline__ void bulk_load_plain(void *dst, const void *src, uint32_t bytes,
                                                uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(smem_addr(dst)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

// Programmatic dependent launch: a kernel launched with programmatic stream
// serialization may start before its predecessor ends; pdl_wait() blocks
// until the predecessor grid has completed and its writes are visible (a
// no-op for an ordinary launch); pdl_trigger() lets the successor launch.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Named barrier over `count` threads (ids 1..15; 0 is __syncthreads).
__device__ __forceinline__ void named_sync(int id, int count)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Watchdog of a polling loop: the global timer is read only while the loop
// is idle (on its first idle pass, then every 16th), so a loop that keeps
// making progress pays nothing for it.
struct IdleWatch {
    uint64_t t0 = 0;
    uint32_t n = 0;
    __device__ __forceinline__ void progress() { n = 0; }
    // one idle pass; true once the loop has been idle for more than limit_ns
    __device__ __forceinline__ bool expired(uint64_t limit_ns)
    {
        if (n++ == 0) {
            t0 = global_ns();
            return false;
        }
        return (n & 15) == 0 && global_ns() - t0 > limit_ns;
    }
};

// Counters in shared memory published with release and read with acquire:
// a thread that issues tensor-core work polls one of these instead of
// waiting on an mbarrier (an mbarrier wait stalls the issuing thread for
// ~140 cycles even on a completed phase; this load costs a third of that).
__device__ __forceinline__ int ld_acquire_shared(const int *p)
{
    int v;
    asm volatile("ld.acquire.cta.shared::cta.b32 %0, [%1];" : "=r"(v) : "r"(smem_addr(p)) : "memory");
    return v;
}
__device__ __forceinline__ void st_release_shared(int *p, int v)
{
    asm volatile("st.release.cta.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(p)), "r"(v) : "memory");
}
__device__ __forceinline__ void red_release_add_shared(int *p, int v)
{
    asm volatile("red.release.cta.shared::cta.add.s32 [%0], %1;" ::"r"(smem_addr(p)), "r"(v) : "memory");
}

// Bounded waits give up after this long (far above any legitimate wait).
constexpr uint64_t kWaitLimitNs = 2000000000ull;

}  // namespace reatt
