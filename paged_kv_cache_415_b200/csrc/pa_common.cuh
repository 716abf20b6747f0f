// pa_common.cuh -- device helpers shared by the library's kernels (sm_100a).
//
// Inline PTX wrappers for the tensor-copy engine (TMA: cp.async.bulk.tensor
// tiles, and the untiled cp.async.bulk, global -> shared, completion counted
// on an mbarrier), mbarrier waits that give up after a bounded time,
// programmatic dependent launch, ldmatrix and warp-level mma.sync, and
// fp16 / bf16 <-> fp32 conversions.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "pa.h"

namespace pa {

constexpr unsigned kFullMask = 0xffffffffu;

// A wait for an asynchronous copy gives up after this long (the copy of a
// few KB normally lands within microseconds).
constexpr uint64_t kWaitTimeoutNs = 1000ull * 1000ull * 1000ull;   // 1 s
constexpr uint32_t kWaitMaxPolls = 1u << 30;

// Programmatic dependent launch: a kernel launched with the programmatic
// stream-serialisation attribute may start while the previous kernel in the
// stream is still running; it must call grid_dependency_wait() before it
// touches any global memory that earlier work produces or reads.  A kernel
// that calls allow_dependents() lets the next one start launching early.
// Both are no-ops when the launch carries no such dependency.
__device__ __forceinline__ void grid_dependency_wait()
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

__device__ __forceinline__ void allow_dependents()
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ uint32_t smem_u32(const void* p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}

// Makes barrier initialisation visible to the asynchronous proxy.
__device__ __forceinline__ void fence_barrier_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Orders this thread's earlier shared-memory accesses before later
// asynchronous-proxy (bulk copy) accesses to shared memory.
__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Orders this thread's earlier generic global-memory accesses before its
// later asynchronous-proxy (TMA) accesses to global memory.
__device__ __forceinline__ void fence_proxy_async_global()
{
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

// One arrival that also announces `bytes` of copies still to land.
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity)
{
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

// Waits for the barrier phase with the given parity.  Returns false if it
// has not completed after limit_ns (or kWaitMaxPolls polls).
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  uint64_t limit_ns = kWaitTimeoutNs)
{
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t i = 0; i < kWaitMaxPolls; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 63u) == 63u && global_timer_ns() - t0 > limit_ns) return false;
    }
    return false;
}

// The same wait for a whole warp, with one answer for every lane: true only
// if every lane saw the phase complete.  A lane that gives up at the limit
// while another saw the phase complete makes the warp give up, so the warp
// never diverges on it.
__device__ __forceinline__ bool mbar_wait_warp(uint64_t* bar, uint32_t parity,
                                               uint64_t limit_ns = kWaitTimeoutNs)
{
    return __all_sync(kFullMask, mbar_wait_bounded(bar, parity, limit_ns)) != 0;
}

// A warp's ring of copy stages gave up waiting at stage `first_pending`
// (copies first_pending .. issued - 1 may still be in flight into its shared
// memory).  Records PA_STATUS_TIMEOUT and waits again, bounded, for each of
// those copies.  Returns whether all of them landed.  Whatever it returns,
// the caller must not read or reuse that shared memory: the CTA writes its
// "no result" through global memory only and returns (store_aborted_rows).
template <int NSTAGE>
__device__ __forceinline__ bool drain_after_timeout(uint64_t* wbar, int first_pending, int issued,
                                                    int32_t* d_status)
{
    if ((threadIdx.x & 31) == 0 && d_status != nullptr) atomicOr(d_status, PA_STATUS_TIMEOUT);
    bool landed = true;
    for (int k = first_pending; k < issued; ++k)
        landed &= mbar_wait_warp(&wbar[k % NSTAGE], (k / NSTAGE) & 1);
    return landed;
}

// Test hook of the bounded waits (pa_selftest_decode_abort): with a nonzero
// probe, a warp waits first on `never` -- an mbarrier that nothing arrives
// on -- with a limit of probe_us microseconds, and gives up there before its
// first block, so the timeout, the drain of the copies already issued and
// the abort store all run for real.  With probe_us == 0 (every library
// call) it returns false at once.  Warp-uniform.
__device__ __forceinline__ bool probe_gives_up(uint64_t* never, uint32_t probe_us)
{
    return probe_us != 0u && !mbar_wait_warp(never, 0u, 1000ull * probe_us);
}

// Asynchronous bulk copy global -> shared of `bytes` (multiple of 16, both
// addresses 16-byte aligned); its completion is counted on `bar`.
__device__ __forceinline__ void bulk_copy_g2s(void* dst_smem, const void* src_gmem, uint32_t bytes,
                                              uint64_t* bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(smem_u32(dst_smem)),
        "l"(src_gmem), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// Same, with an L2 eviction-priority policy (a createpolicy value).
__device__ __forceinline__ void bulk_copy_g2s_hint(void* dst_smem, const void* src_gmem,
                                                   uint32_t bytes, uint64_t* bar, uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], "
        "%2, [%3], %4;" ::"r"(smem_u32(dst_smem)),
        "l"(src_gmem), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

// Tiled tensor copy global -> shared of one box of a 4-D tensor map at
// coordinates (x, y, z, w) (innermost first); completion counted on `bar`.
// x * element size must be a multiple of 16 bytes (x is 0 here).
__device__ __forceinline__ void tma_load_4d(void* dst_smem, const void* tensor_map, int x, int y,
                                            int z, int w, uint64_t* bar)
{
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(smem_u32(dst_smem)),
        "l"(reinterpret_cast<uint64_t>(tensor_map)), "r"(x), "r"(y), "r"(z), "r"(w),
        "r"(smem_u32(bar))
        : "memory");
}

// Same for a 5-D tensor map.
__device__ __forceinline__ void tma_load_5d(void* dst_smem, const void* tensor_map, int c0, int c1,
                                            int c2, int c3, int c4, uint64_t* bar)
{
    asm volatile(
        "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%2, %3, %4, %5, %6}], [%7];" ::"r"(smem_u32(dst_smem)),
        "l"(reinterpret_cast<uint64_t>(tensor_map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4),
        "r"(smem_u32(bar))
        : "memory");
}

// Four 8x8 matrices of 16-bit elements from shared memory; lane l gives the
// address of row (l % 8) of matrix (l / 8).  Lane l receives, for matrix i,
// row l / 4, elements 2 (l % 4) and 2 (l % 4) + 1 (with .trans: column l / 4,
// rows 2 (l % 4) and 2 (l % 4) + 1).
__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], uint32_t smem_addr)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_addr));
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t (&r)[4], uint32_t smem_addr)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_addr));
}

__device__ __forceinline__ uint64_t policy_evict_first()
{
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ uint4 ld_nc_v4(const void* p)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// ---------------------------------------------------------------------------
// Element types.  Both are 16-bit; a 16-byte vector holds 8 elements.
// ---------------------------------------------------------------------------
template <typename T>
struct Elem;

template <>
struct Elem<__half> {
    // Two packed binary16 values -> two floats (exact).
    static __device__ __forceinline__ float2 to_float2(uint32_t w)
    {
        __half2 h = *reinterpret_cast<const __half2*>(&w);
        return __half22float2(h);
    }
    // Two floats -> packed binary16, each rounded to nearest even.
    static __device__ __forceinline__ uint32_t from_float2(float a, float b)
    {
        __half2 h = __floats2half2_rn(a, b);
        return *reinterpret_cast<const uint32_t*>(&h);
    }
};

template <>
struct Elem<__nv_bfloat16> {
    // bfloat16 is the upper half of a binary32, so widening is a shift.
    static __device__ __forceinline__ float2 to_float2(uint32_t w)
    {
        return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
    }
    static __device__ __forceinline__ uint32_t from_float2(float a, float b)
    {
        __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
        return *reinterpret_cast<const uint32_t*>(&h);
    }
};

// acc + a.lo * b.lo + a.hi * b.hi for two packed 16-bit pairs, with fp32
// accumulation (mixed-precision fma: the 16-bit operands are widened
// exactly, each product-sum rounds once in fp32).
template <typename T>
__device__ __forceinline__ float fma_pair(uint32_t a, uint32_t b, float acc);

template <>
__device__ __forceinline__ float fma_pair<__half>(uint32_t a, uint32_t b, float acc)
{
    asm("{\n\t.reg .b16 al, ah, bl, bh;\n\t"
        "mov.b32 {al, ah}, %1;\n\t"
        "mov.b32 {bl, bh}, %2;\n\t"
        "fma.rn.f32.f16 %0, al, bl, %0;\n\t"
        "fma.rn.f32.f16 %0, ah, bh, %0;\n\t}"
        : "+f"(acc)
        : "r"(a), "r"(b));
    return acc;
}

template <>
__device__ __forceinline__ float fma_pair<__nv_bfloat16>(uint32_t a, uint32_t b, float acc)
{
    asm("{\n\t.reg .b16 al, ah, bl, bh;\n\t"
        "mov.b32 {al, ah}, %1;\n\t"
        "mov.b32 {bl, bh}, %2;\n\t"
        "fma.rn.f32.bf16 %0, al, bl, %0;\n\t"
        "fma.rn.f32.bf16 %0, ah, bh, %0;\n\t}"
        : "+f"(acc)
        : "r"(a), "r"(b));
    return acc;
}

// Warp-level D = A * B + D with A 16x16 (row-major), B 16x8 (column-major)
// of 16-bit elements and D 16x8 in fp32 (mma.sync m16n8k16).
template <typename T>
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1);

template <>
__device__ __forceinline__ void mma_16816<__nv_bfloat16>(float (&d)[4], uint32_t a0, uint32_t a1,
                                                         uint32_t a2, uint32_t a3, uint32_t b0,
                                                         uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

template <>
__device__ __forceinline__ void mma_16816<__half>(float (&d)[4], uint32_t a0, uint32_t a1,
                                                  uint32_t a2, uint32_t a3, uint32_t b0,
                                                  uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// 8 packed elements -> 8 floats.
template <typename T>
__device__ __forceinline__ void unpack8(const uint4& v, float (&f)[8])
{
    float2 a = Elem<T>::to_float2(v.x), b = Elem<T>::to_float2(v.y);
    float2 c = Elem<T>::to_float2(v.z), d = Elem<T>::to_float2(v.w);
    f[0] = a.x; f[1] = a.y; f[2] = b.x; f[3] = b.y;
    f[4] = c.x; f[5] = c.y; f[6] = d.x; f[7] = d.y;
}

template <typename T>
__device__ __forceinline__ uint4 pack8(const float (&f)[8])
{
    uint4 v;
    v.x = Elem<T>::from_float2(f[0], f[1]);
    v.y = Elem<T>::from_float2(f[2], f[3]);
    v.z = Elem<T>::from_float2(f[4], f[5]);
    v.w = Elem<T>::from_float2(f[6], f[7]);
    return v;
}

__device__ __forceinline__ void status_or(int32_t* d_status, int32_t bits)
{
    if (d_status != nullptr) atomicOr(d_status, bits);
}

}  // namespace pa
