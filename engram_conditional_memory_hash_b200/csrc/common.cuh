// Device helpers shared by the Engram kernels (sm_100a): bf16 packing, warp
// reductions, and the mbarrier + bulk-copy (TMA, non-tensor) primitives the
// gate kernels use to stream token rows into shared memory.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace engram {

// Device error word: kernels OR a code into it instead of trapping.
__device__ unsigned int g_device_error;

constexpr unsigned kErrPipelineTimeout = 1u;       // ENGRAM_DEVICE_ERR_PIPELINE_TIMEOUT
constexpr uint64_t kWaitLimitNs = 2000000000ull;   // 2 s per pipeline wait

// ---------------------------------------------------------------- bf16 ----

// Two bf16 values packed in a 32-bit word -> two floats (exact).
__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

// Two floats -> packed bf16 pair, round to nearest even.
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi)
{
    __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&p);
}

// 8 bf16 values of a 16-byte vector -> 4 float pairs (element 2i in .x).
__device__ __forceinline__ void unpack4x2(const uint4 &q, float2 f[4])
{
    f[0] = make_float2(bf16_lo(q.x), bf16_hi(q.x));
    f[1] = make_float2(bf16_lo(q.y), bf16_hi(q.y));
    f[2] = make_float2(bf16_lo(q.z), bf16_hi(q.z));
    f[3] = make_float2(bf16_lo(q.w), bf16_hi(q.w));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float2 f) { return pack_bf16(f.x, f.y); }

__device__ __forceinline__ uint4 pack4x2(const float2 f[4])
{
    uint4 q;
    q.x = pack_bf16x2(f[0]);
    q.y = pack_bf16x2(f[1]);
    q.z = pack_bf16x2(f[2]);
    q.w = pack_bf16x2(f[3]);
    return q;
}

// ------------------------------------------------------------ reductions ----

__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// ------------------------------------------------- mbarrier / bulk copy ----

__device__ __forceinline__ uint32_t smem_addr(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

// Make barrier initialisation visible to the async (bulk-copy) proxy.
__device__ __forceinline__ void fence_barrier_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

// One-dimensional bulk copy global -> this CTA's shared memory, completing
// `bytes` of transaction count on `bar`.  dst, src and bytes: multiples of 16.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes,
                                          uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(dst), "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t globaltimer_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Wait for phase `parity` of `bar` to complete; false once kWaitLimitNs have
// passed without it (the caller then records the error and stops).
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity)
{
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
    }
    return true;
}

// Programmatic dependent launch (sm_90 and later).  Wait until the kernel
// that precedes this one in the stream has completed and its writes are
// visible (a no-op when the launch carries no programmatic dependency), then
// let the next kernel of the stream be scheduled: it in turn waits here for
// this whole grid to complete before it reads anything, so the early release
// only overlaps launch latency with this kernel's tail.
__device__ __forceinline__ void pdl_wait_and_release()
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void record_device_error(unsigned code)
{
    atomicOr(&g_device_error, code);
}

}  // namespace engram
