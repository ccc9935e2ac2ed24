// tcgen05_common.cuh -- tensor-memory and tcgen05.mma wrappers shared by the
// tensor-core kernels (prefill GEMM, small-batch GEMV): allocation, the
// eight-MMA stage of k = 256 (int8, A in tensor memory, B a K-major
// 128-byte-swizzled shared-memory operand), commits, and register <-> tensor
// memory moves written together with their waits.
#pragma once

#include "bl_common.cuh"

namespace bl {
namespace {

constexpr int kTcStageK = 256;   // k per eight-MMA stage
constexpr int kTcBoxK = 128;     // k per 128-byte swizzle span of B
constexpr int kTcMmaK = 32;      // k per tcgen05.mma.kind::i8

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

// The MMA role runs on a whole warp in warp-uniform control flow; each
// tcgen05.mma and tcgen05.commit is an instruction predicated on lane 0 inside
// that uniform code.  Two points matter:
//   - issued from a single-lane divergent region instead, back-to-back
//     128x128x32 MMAs measured ~120 cycles apiece once the loop also waited on
//     an mbarrier, against 64 in warp-uniform code;
//   - the issuing lane is fixed, not chosen by elect.sync: tcgen05.commit
//     tracks only the MMAs of the thread that executes it, and leaders elected
//     separately for the MMAs and for the commit were seen to differ, which let
//     a ring slot be released while its MMAs still read it.

// One pipeline stage: eight MMAs (k = 0..255) issued by lane 0.
// b_desc0 describes the stage's first 32 k of activations; the start address
// field advances by 32 B (2 units) per MMA within a 128-k box and by one box
// (BOX16 units of 16 B) after four MMAs.  A advances 8 TMEM columns per MMA.
// accumulate_first = 0 makes the first MMA overwrite D (first stage of a tile).
template <uint32_t BOX16>
__device__ __forceinline__ void mma_stage8(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc0, uint32_t idesc,
                                           uint32_t accumulate_first)
{
    static_assert(kTcStageK / kTcMmaK == 8 && kTcBoxK / kTcMmaK == 4, "stage shape");
    asm volatile(
        "{\n\t.reg .pred e, p, t;\n\t.reg .b32 r;\n\t"
        "mov.u32 r, %%laneid;\n\t"
        "setp.eq.u32 e, r, 0;\n\t"
        "setp.ne.b32 p, %12, 0;\n\t"
        "setp.ne.b32 t, %19, 0;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %3, %11, p;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::i8 [%0], [%2], %4, %11, t;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::i8 [%0], [%13], %5, %11, t;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::i8 [%0], [%14], %6, %11, t;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::i8 [%0], [%15], %7, %11, t;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::i8 [%0], [%16], %8, %11, t;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::i8 [%0], [%17], %9, %11, t;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::i8 [%0], [%18], %10, %11, t;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "r"(a_tmem + 8), "l"(b_desc0), "l"(b_desc0 + 2), "l"(b_desc0 + 4), "l"(b_desc0 + 6),
        "l"(b_desc0 + BOX16), "l"(b_desc0 + BOX16 + 2), "l"(b_desc0 + BOX16 + 4), "l"(b_desc0 + BOX16 + 6), "r"(idesc),
        "r"(accumulate_first), "r"(a_tmem + 16), "r"(a_tmem + 24), "r"(a_tmem + 32), "r"(a_tmem + 40),
        "r"(a_tmem + 48), "r"(a_tmem + 56), "r"(1u)
        : "memory");
}

__device__ __forceinline__ void mma_commit(uint32_t bar)
{
    asm volatile(
        "{\n\t.reg .pred e;\n\t.reg .b32 r;\n\t"
        "mov.u32 r, %%laneid;\n\t"
        "setp.eq.u32 e, r, 0;\n\t"
        "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(bar)
        : "memory");
}

// tcgen05.ld and tcgen05.st move registers asynchronously: the destination
// registers of a load are valid only after tcgen05.wait::ld, and the source
// registers of a store must stay unchanged until tcgen05.wait::st.  Each
// access is therefore written together with its wait in one asm statement,
// so that the compiler neither reads a loaded register early nor reuses a
// stored one while the store is in flight.

// Sixty-four consecutive 32-bit TMEM columns of this thread's lane, stored.
__device__ __forceinline__ void tmem_st64_wait(uint32_t taddr, const uint32_t (&v)[64])
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x64.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63, %64};\n\t"
        "tcgen05.wait::st.sync.aligned;" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31]), "r"(v[32]), "r"(v[33]), "r"(v[34]), "r"(v[35]), "r"(v[36]), "r"(v[37]), "r"(v[38]), "r"(v[39]), "r"(v[40]), "r"(v[41]), "r"(v[42]), "r"(v[43]), "r"(v[44]), "r"(v[45]), "r"(v[46]), "r"(v[47]), "r"(v[48]), "r"(v[49]), "r"(v[50]), "r"(v[51]), "r"(v[52]), "r"(v[53]), "r"(v[54]), "r"(v[55]), "r"(v[56]), "r"(v[57]), "r"(v[58]), "r"(v[59]), "r"(v[60]), "r"(v[61]), "r"(v[62]), "r"(v[63])
        : "memory");
}

// Thirty-two consecutive 32-bit TMEM columns of this thread's lane, loaded.
__device__ __forceinline__ void tmem_ld32_wait(uint32_t taddr, uint32_t (&v)[32])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
        : "r"(taddr)
        : "memory");
}

// Thirty-two consecutive 32-bit TMEM columns of this thread's lane, stored.
__device__ __forceinline__ void tmem_st32_wait(uint32_t taddr, const uint32_t (&v)[32])
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};\n\t"
        "tcgen05.wait::st.sync.aligned;" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
        "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]),
        "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]),
        "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
        : "memory");
}

// Sixteen consecutive 32-bit TMEM columns of this thread's lane, loaded.
__device__ __forceinline__ void tmem_ld16_wait(uint32_t taddr, uint32_t (&v)[16])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15}, [%16];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr)
        : "memory");
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row atoms of
// 1024 bytes stacked along the token dimension (stride byte offset 1024).
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr)
{
    uint64_t d = 0;
    d |= uint64_t((addr >> 4) & 0x3fffu);        // start address
    d |= uint64_t(1) << 16;                      // leading byte offset (unused for SW128 K-major)
    d |= uint64_t(1024 >> 4) << 32;              // stride byte offset
    d |= uint64_t(1) << 46;                      // descriptor version (sm_100)
    d |= uint64_t(2) << 61;                      // layout: 128-byte swizzle
    return d;
}

}  // namespace
}  // namespace bl
