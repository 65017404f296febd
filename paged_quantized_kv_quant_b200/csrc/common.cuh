// Device helpers shared by the pkvq kernels (sm_100a).
//
// Thin wrappers over PTX: mbarrier, TMA (bulk and tiled tensor copies, no
// cluster multicast anywhere), legacy warp-level mma.sync and the matrix
// move/load instructions used to feed it.  No arithmetic of the method lives
// here.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace pkvq {

// Status bits written to the device status word.
constexpr uint32_t kStatusWaitTimeout = 1u;   // an mbarrier wait hit its limit
constexpr uint32_t kStatusBadBlock = 2u;      // a block id outside the pool was skipped

// Every mbarrier wait gives up after this many nanoseconds of %globaltimer
// (far above any legitimate latency), records kStatusWaitTimeout and returns.
constexpr uint64_t kWaitLimitNs = 1000000000ull;

__device__ __forceinline__ uint64_t global_timer_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// True once any wait on this device has timed out (until the status word is
// cleared): kernels then skip their work instead of waiting again.
__device__ __forceinline__ bool device_wait_failed(const uint32_t *status)
{
    return status && (*(volatile const uint32_t *)status & kStatusWaitTimeout);
}

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ------------------------------------------------------------ mbarrier --

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for a phase for at most about `ns` nanoseconds, suspended (the thread
// takes no issue slots while it sleeps and wakes as soon as the phase
// completes); returns whether the phase completed.
__device__ __forceinline__ bool mbar_try_wait_for(uint64_t *bar, uint32_t parity, uint32_t ns)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(ns)
        : "memory");
    return ok != 0;
}

// Non-blocking probe of a phase (test_wait never suspends the thread, unlike
// try_wait): for a thread that polls several barriers in turn.
__device__ __forceinline__ bool mbar_test_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait: returns false (and records it) if the phase does not
// complete within kWaitLimitNs.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, uint32_t *status)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const uint64_t t0 = global_timer_ns();
    for (;;) {
        if (mbar_try_wait(bar, parity))
            return true;
        if (global_timer_ns() - t0 > kWaitLimitNs)
            break;
    }
    if (status)
        atomicOr(status, kStatusWaitTimeout);
    return false;
}

// ----------------------------------------------------------------- TMA --

// 1-D bulk copy global -> shared, completion counted on `bar` (bytes).
// src and dst 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void tma_bulk_g2s(void *dst, const void *src, uint32_t bytes,
                                             uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// 2-D tiled tensor copy global -> shared (no multicast).  x is the inner
// (byte) coordinate and must be a multiple of 16 bytes; callers pass 0.
__device__ __forceinline__ void tma_tile_2d_g2s(void *dst, const CUtensorMap *map, int32_t x,
                                                int32_t y, uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, "
        "%3}], [%4];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

// 16-byte asynchronous copy global -> shared (L2 only, no L1 allocation);
// both addresses 16-byte aligned.
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void *src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

// One arrival on `bar` once every cp.async this thread issued before has
// landed (the barrier's expected count includes this arrival).
__device__ __forceinline__ void cp_async_mbar_arrive(uint64_t *bar)
{
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void cp_async_wait_all()
{
    asm volatile("cp.async.wait_all;" ::: "memory");
}

// 4-byte copy (both addresses 4-byte aligned).
__device__ __forceinline__ void cp_async_4(uint32_t dst, const void *src)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}

// Closes this thread's current group of cp.async copies.
__device__ __forceinline__ void cp_async_commit()
{
    asm volatile("cp.async.commit_group;" ::: "memory");
}

// Waits until at most N of this thread's committed groups are still in flight.
template <int N>
__device__ __forceinline__ void cp_async_wait_group()
{
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Brings the 128-byte line holding `ptr` into L2.
__device__ __forceinline__ void prefetch_l2(const void *ptr)
{
    asm volatile("prefetch.global.L2 [%0];" ::"l"(ptr));
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap *map)
{
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ------------------------------------------------------- warp-level MMA --

// D = A * B + D, m16n8k16, fp16 inputs, fp32 accumulate (legacy tensor path).
__device__ __forceinline__ void mma_f16_16816(float (&d)[4], const uint32_t (&a)[4],
                                              const uint32_t (&b)[2])
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// Transpose an 8x8 b16 matrix held one row-pair per thread in mma layout.
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x)
{
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], uint32_t addr)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t (&r)[4], uint32_t addr)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

// ------------------------------------------------------ code -> fp16 --

// Two E4M3 codes (low 16 bits of `pair`, first code in the low byte) ->
// half2 with the first code in the low half.  Exact: every E4M3 value is an
// fp16 value.
__device__ __forceinline__ uint32_t e4m3x2_to_half2(uint32_t pair)
{
    uint32_t out;
    asm("{\n\t.reg .b16 lo;\n\t"
        "cvt.u16.u32 lo, %1;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, lo;\n\t}"
        : "=r"(out)
        : "r"(pair));
    return out;
}

// Four E4M3 codes (bytes b0..b3 of x) -> half2 (b0, b1) and half2 (b2, b3).
__device__ __forceinline__ void e4m3x4_to_half2x2(uint32_t x, uint32_t &lo, uint32_t &hi)
{
    asm("{\n\t.reg .b16 a, b;\n\t"
        "mov.b32 {a, b}, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, a;\n\t"
        "cvt.rn.f16x2.e4m3x2 %1, b;\n\t}"
        : "=r"(lo), "=r"(hi)
        : "r"(x));
}

// Four E5M2 codes (bytes b0..b3 of x) -> half2 (b0, b1) and half2 (b2, b3).
// Exact: an E5M2 code is the high byte of the fp16 with the same value.
__device__ __forceinline__ void e5m2x4_to_half2x2(uint32_t x, uint32_t &lo, uint32_t &hi)
{
    asm("{\n\t.reg .b16 a, b;\n\t"
        "mov.b32 {a, b}, %2;\n\t"
        "cvt.rn.f16x2.e5m2x2 %0, a;\n\t"
        "cvt.rn.f16x2.e5m2x2 %1, b;\n\t}"
        : "=r"(lo), "=r"(hi)
        : "r"(x));
}

// Four int8 codes (bytes b0..b3 of x) -> half2 (b0, b1) and half2 (b2, b3),
// exact (see s8x2_to_half2).
__device__ __forceinline__ void s8x4_to_half2x2(uint32_t x, uint32_t &lo, uint32_t &hi)
{
    const uint32_t biased = x ^ 0x80808080u;
    uint32_t l = __byte_perm(biased, 0x64646464u, 0x5140);
    uint32_t h = __byte_perm(biased, 0x64646464u, 0x7362);
    const __half2 k = __half2half2(__ushort_as_half(0x6480));   // 1152
    __half2 lh = __hsub2(*reinterpret_cast<__half2 *>(&l), k);
    __half2 hh = __hsub2(*reinterpret_cast<__half2 *>(&h), k);
    lo = *reinterpret_cast<uint32_t *>(&lh);
    hi = *reinterpret_cast<uint32_t *>(&hh);
}

// Four int8 codes -> half2 (b0, b1) and (b2, b3) of code * 2^e, with
// p2 = 2^e and nb2 = -1152 * 2^e (both exact in fp16): the magic-number form
// (1152 + code) times 2^e minus 1152 * 2^e in one fused multiply-add, whose
// exact result code * 2^e is representable, so it is exact whenever
// |code * 2^e| stays below 65504.
__device__ __forceinline__ void s8x4_to_half2x2_scaled(uint32_t x, __half2 p2, __half2 nb2,
                                                       uint32_t &lo, uint32_t &hi)
{
    const uint32_t biased = x ^ 0x80808080u;
    uint32_t l = __byte_perm(biased, 0x64646464u, 0x5140);
    uint32_t h = __byte_perm(biased, 0x64646464u, 0x7362);
    __half2 lh = __hfma2(*reinterpret_cast<__half2 *>(&l), p2, nb2);
    __half2 hh = __hfma2(*reinterpret_cast<__half2 *>(&h), p2, nb2);
    lo = *reinterpret_cast<uint32_t *>(&lh);
    hi = *reinterpret_cast<uint32_t *>(&hh);
}

// Two signed int8 codes (bytes b0, b1 of `pair`) -> exact half2 values.
// 0x6400 | (c ^ 0x80) is the fp16 number 1024 + 128 + c; subtracting 1152
// is exact for |c| <= 128.
__device__ __forceinline__ uint32_t s8x2_to_half2(uint32_t pair)
{
    uint32_t biased = __byte_perm(pair ^ 0x8080u, 0x6464u, 0x5140);  // [c0', 0x64, c1', 0x64]
    __half2 h = *reinterpret_cast<__half2 *>(&biased);
    h = __hsub2(h, __half2half2(__ushort_as_half(0x6480)));          // 1152
    return *reinterpret_cast<uint32_t *>(&h);
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi)
{
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

// Read-only global loads that bypass L1 allocation (streamed cache rows; the
// data was written before this kernel started).
__device__ __forceinline__ uint4 ldg_nc_v4(const uint4 *p)
{
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ uint16_t ldg_nc_u16(const uint16_t *p)
{
    uint16_t r;
    asm volatile("ld.global.nc.L1::no_allocate.u16 %0, [%1];" : "=h"(r) : "l"(p));
    return r;
}

__device__ __forceinline__ float fast_exp2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

}  // namespace pkvq
