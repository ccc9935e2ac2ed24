// bl_common.cuh -- device helpers shared by the sm_100a kernels of
// libbitlinear.so: cache-hinted loads, integer dot products, reductions,
// named barriers and the bounded-wait clock.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "bl_internal.h"

namespace bl {

constexpr float kEps = 1e-5f;      // floor of both absmax and absmean scales
constexpr float kQb = 127.0f;      // int8 activation range used by the scale

// Streamed, read-once data: bypass L1 allocation (weights are touched once).
__device__ __forceinline__ uint4 ld_stream_v4(const void *p)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ uint2 ld_stream_v2(const void *p)
{
    uint2 v;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];"
                 : "=r"(v.x), "=r"(v.y)
                 : "l"(p));
    return v;
}

// Read-only data that many threads re-read (activations): keep in L1.
__device__ __forceinline__ uint4 ld_ro_v4(const void *p)
{
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// Data that the preceding launch may have written and that a kernel reads
// only after griddepcontrol.wait (its activations under programmatic
// dependent launch): an L2-coherent load, never the non-coherent read-only
// path, which may serve a value fetched or scheduled before the wait.  The
// memory clobber keeps the load after the wait in the compiler's order.
__device__ __forceinline__ uint4 ld_dep_v4(const void *p)
{
    uint4 v;
    asm volatile("ld.global.cg.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p)
                 : "memory");
    return v;
}

__device__ __forceinline__ uint32_t ld_dep_u32(const void *p)
{
    uint32_t v;
    asm volatile("ld.global.cg.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ unsigned long long ld_dep_u64(const void *p)
{
    unsigned long long v;
    asm volatile("ld.global.cg.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ uint32_t ld_dep_u16(const void *p)
{
    unsigned short v;
    asm volatile("ld.global.cg.u16 %0, [%1];" : "=h"(v) : "l"(p) : "memory");
    return v;
}

// 4-way byte dot product, unsigned bytes of a times signed bytes of b.
__device__ __forceinline__ int dp4a_us(uint32_t a, uint32_t b, int c)
{
    int d;
    asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

__device__ __forceinline__ void named_barrier(int id, int nthreads)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ uint64_t global_timer_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

template <typename T>
__device__ __forceinline__ T warp_sum(T v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float warp_max(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

template <bool DEP>
__device__ __forceinline__ uint4 ld_in_v4(const void *p)
{
    if constexpr (DEP)
        return ld_dep_v4(p);
    else
        return ld_ro_v4(p);
}

// Eight input elements (one 16-byte bf16 vector or two fp32 vectors) as fp32.
// DEP: the elements may have been written by the preceding launch (read with
// the coherent load, see ld_dep_v4).
template <int XT, bool DEP = false>
__device__ __forceinline__ void load8(const void *base, int64_t idx, float f[8])
{
    if constexpr (XT == BL_BF16) {
        const uint4 v = ld_in_v4<DEP>(static_cast<const __nv_bfloat16 *>(base) + idx);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    } else {
        const float *p = static_cast<const float *>(base) + idx;
        const uint4 a = ld_in_v4<DEP>(p);
        const uint4 b = ld_in_v4<DEP>(p + 4);
        f[0] = __uint_as_float(a.x); f[1] = __uint_as_float(a.y);
        f[2] = __uint_as_float(a.z); f[3] = __uint_as_float(a.w);
        f[4] = __uint_as_float(b.x); f[5] = __uint_as_float(b.y);
        f[6] = __uint_as_float(b.z); f[7] = __uint_as_float(b.w);
    }
}

// int8 quantisation of one value with the per-token scale s: rint(x * s)
// (fp32 product, ties to even) clamped to [-128, 127].
__device__ __forceinline__ int quant1(float x, float s)
{
    int t = __float2int_rn(__fmul_rn(x, s));
    return max(-128, min(127, t));
}

// Final rescale: ((float)acc * d) * gamma, two round-to-nearest products.
__device__ __forceinline__ float rescale1(int acc, float d, float gamma)
{
    return __fmul_rn(__fmul_rn(static_cast<float>(acc), d), gamma);
}

// ---- mbarrier helpers (shared memory barriers tracking TMA / tcgen05 work)

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
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

constexpr uint64_t kWaitLimitNs = 2000000000ull;  // bounded waits give up after 2 s

// Bounded wait on an mbarrier phase.  Returns false (and raises *abort_flag
// and the device status word) if the phase did not complete in time, or if
// another part of the CTA has already aborted.
static __device__ __noinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                       int *status, uint64_t limit_ns = kWaitLimitNs)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity))
            return true;
        if ((it & 31) == 0) {
            if (*abort_flag)
                return false;
            if (global_timer_ns() - t0 > limit_ns) {
                *abort_flag = 1;
                atomicExch(status, BL_ERR_TIMEOUT);
                return false;
            }
        }
    }
}

// mbar_wait with its first test inline: when the phase has already completed
// (the common case in a warp-specialised pipeline that runs ahead) no call is
// made.  A function call in the issuing warp of tcgen05.mma was measured to
// stall it for hundreds of cycles per stage.
__device__ __forceinline__ bool mbar_wait_fast(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                               int *status)
{
    if (mbar_try_wait(bar, parity))
        return true;
    return mbar_wait(bar, parity, abort_flag, status);
}

// Bulk (non-tensor) TMA copy global -> shared, completion counted on `bar`.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void store_y(void *y, int yt, int64_t idx, float v)
{
    if (yt == BL_BF16)
        static_cast<__nv_bfloat16 *>(y)[idx] = __float2bfloat16_rn(v);
    else
        static_cast<float *>(y)[idx] = v;
}

}  // namespace bl
