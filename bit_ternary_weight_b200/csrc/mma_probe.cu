// mma_probe.cu -- measurements of the int8 tensor-core rate: back-to-back
// tcgen05.mma.kind::i8 with A = unsigned codes in tensor memory, B = signed
// activations in 128-byte-swizzled shared memory and int32 accumulators in
// tensor memory, issued as the library's kernels issue them (eight per stage
// by lane 0 of a warp in warp-uniform code), with no operand traffic.  One CTA
// per SM; each issuing warp times its own stream of MMAs with clock64 and
// %globaltimer.
//   * 128 x 128 x 32 from one warp: the prefill GEMM's form; its rate is the
//     denominator "of the probe" of the GEMM's tensor-pipe fraction ("of 2 x
//     bf16" is the measured bf16 cuBLAS rate times the nominal int8/bf16
//     ratio).
//   * 128 x 32 x 32 from one, two or four warps, each into its own
//     accumulator: the small-batch GEMV's form, which shows how many issuing
//     threads narrow MMAs need to reach the tensor rate.
#include "bl_common.cuh"

namespace bl {
namespace {

constexpr int kProbeThreads = 160;       // warp 0 allocates; warps 0-3 fill A; warps 1 .. W issue
constexpr uint32_t kProbeBox = 128 * 128;  // shared-memory B box: up to 128 tokens x 128 k

template <int N>
__host__ __device__ constexpr uint32_t probe_idesc()
{
    return (2u << 4) | (0u << 7) | (1u << 10) | (uint32_t(N >> 3) << 17) | ((128u >> 4) << 24);
}

__device__ __forceinline__ uint64_t probe_desc(uint32_t addr)
{
    uint64_t d = 0;
    d |= uint64_t((addr >> 4) & 0x3fffu);   // start address
    d |= uint64_t(1) << 16;                 // leading byte offset (unused for this layout)
    d |= uint64_t(1024 >> 4) << 32;         // stride byte offset: 8-row atoms of 1024 bytes
    d |= uint64_t(1) << 46;                 // descriptor version
    d |= uint64_t(2) << 61;                 // 128-byte swizzle
    return d;
}

// W warps each issue `reps` stages of eight 128 x N x 32 MMAs into their own
// accumulator columns (issuer w at columns w N), all reading the same A
// (columns 256 .. 319) and B; the CTA holds all 512 tensor-memory columns.
template <int N, int W>
__global__ void __launch_bounds__(kProbeThreads, 1) mma_probe_kernel(int reps, long long *out, int *status)
{
    static_assert(N * W <= 256, "accumulators below the A columns");
    extern __shared__ __align__(1024) unsigned char probe_raw[];
    const uint32_t raw = smem_u32(probe_raw);
    unsigned char *bsm = probe_raw + (((raw + 1023u) & ~1023u) - raw);     // 1024-byte aligned box
    __shared__ __align__(8) uint64_t done[4];
    __shared__ uint32_t tslot;
    __shared__ int abort_flag;
    const int tid = threadIdx.x, warp = tid >> 5;
    for (int i = tid; i < int(kProbeBox / 16); i += kProbeThreads)
        reinterpret_cast<uint4 *>(bsm)[i] = make_uint4(0x01020304u, 0x7f00ff01u, 0x02020202u, 0u);
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    if (tid == 0) {
        abort_flag = 0;
        for (int w = 0; w < 4; ++w)
            mbar_init(smem_u32(&done[w]), 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tslot)),
                     "r"(512u)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t a_tmem = tslot + 256;        // columns 256 .. 319: one stage of A (8 MMAs x 8 columns)
    if (warp < 4) {
        // A: codes {0, 1, 2} in every byte (lane quarter = warp)
        uint32_t v[32];
#pragma unroll
        for (int i = 0; i < 32; ++i)
            v[i] = 0x00010201u + uint32_t(i & 1);
        const uint32_t lane_addr = uint32_t(warp * 32) << 16;
#pragma unroll
        for (int c = 0; c < 64; c += 32)
            asm volatile(
                "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
                "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, "
                "%31, %32};\n\ttcgen05.wait::st.sync.aligned;" ::"r"(a_tmem + lane_addr + c),
                "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
                "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]),
                "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]),
                "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
                : "memory");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    if (warp >= 1 && warp <= W) {
        const int w = warp - 1;
        const uint32_t d_tmem = tslot + uint32_t(w * N);
        const uint64_t b0 = probe_desc(smem_u32(bsm));
        const long long c0 = clock64();
        const uint64_t g0 = global_timer_ns();
        for (int r = 0; r < reps; ++r) {
            // eight MMAs: k advances 32 B (2 descriptor units) per MMA within
            // the 128-byte swizzle span, A eight columns per MMA
            asm volatile(
                "{\n\t.reg .pred e, p, t;\n\t.reg .b32 l;\n\t"
                "mov.u32 l, %%laneid;\n\t"
                "setp.eq.u32 e, l, 0;\n\t"
                "setp.ne.b32 p, %3, 0;\n\t"
                "setp.eq.u32 t, l, l;\n\t"
                "@e tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %4, p;\n\t"
                "@e tcgen05.mma.cta_group::1.kind::i8 [%0], [%5], %6, %4, t;\n\t"
                "@e tcgen05.mma.cta_group::1.kind::i8 [%0], [%7], %8, %4, t;\n\t"
                "@e tcgen05.mma.cta_group::1.kind::i8 [%0], [%9], %10, %4, t;\n\t"
                "@e tcgen05.mma.cta_group::1.kind::i8 [%0], [%11], %2, %4, t;\n\t"
                "@e tcgen05.mma.cta_group::1.kind::i8 [%0], [%12], %6, %4, t;\n\t"
                "@e tcgen05.mma.cta_group::1.kind::i8 [%0], [%13], %8, %4, t;\n\t"
                "@e tcgen05.mma.cta_group::1.kind::i8 [%0], [%14], %10, %4, t;\n\t}" ::"r"(d_tmem),
                "r"(a_tmem), "l"(b0), "r"(r > 0 ? 1u : 0u), "r"(probe_idesc<N>()), "r"(a_tmem + 8), "l"(b0 + 2),
                "r"(a_tmem + 16), "l"(b0 + 4), "r"(a_tmem + 24), "l"(b0 + 6), "r"(a_tmem + 32), "r"(a_tmem + 40),
                "r"(a_tmem + 48), "r"(a_tmem + 56)
                : "memory");
        }
        asm volatile(
            "{\n\t.reg .pred e;\n\t.reg .b32 l;\n\t"
            "mov.u32 l, %%laneid;\n\t"
            "setp.eq.u32 e, l, 0;\n\t"
            "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(
                smem_u32(&done[w]))
            : "memory");
        bool ok = mbar_wait(smem_u32(&done[w]), 0, &abort_flag, status);
        if (!ok) {
            // the MMAs must retire before their tensor memory is freed
            volatile int no_abort = 0;
            mbar_wait(smem_u32(&done[w]), 0, &no_abort, status);
        }
        const long long c1 = clock64();
        const uint64_t g1 = global_timer_ns();
        if ((tid & 31) == 0) {
            out[2 * (blockIdx.x * W + w)] = ok ? c1 - c0 : -1;
            out[2 * (blockIdx.x * W + w) + 1] = ok ? (long long)(g1 - g0) : -1;
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tslot), "r"(512u) : "memory");
}

template <int N, int W>
int launch_probe_t(int reps, long long *out, int grid, cudaStream_t s)
{
    const DeviceInfo *di = device_info();
    if (!di)
        return BL_ERR_CUDA;
    // enough shared memory that only one CTA fits on an SM: one MMA stream per SM
    const size_t smem = 120 * 1024;
    int per_sm = 0;
    int st = occupancy(reinterpret_cast<const void *>(mma_probe_kernel<N, W>), kProbeThreads, smem, &per_sm);
    if (st)
        return st;
    if (per_sm < 1)
        return BL_ERR_SHAPE;
    mma_probe_kernel<N, W><<<unsigned(grid), kProbeThreads, smem, s>>>(reps, out, di->status);
    return launch_status();
}

}  // namespace

int launch_mma_probe(int n, int issuers, int reps, long long *out, int grid, cudaStream_t s)
{
    if (n == 128 && issuers == 1)
        return launch_probe_t<128, 1>(reps, out, grid, s);
    if (n == 128 && issuers == 2)
        return launch_probe_t<128, 2>(reps, out, grid, s);
    if (n == 32 && issuers == 1)
        return launch_probe_t<32, 1>(reps, out, grid, s);
    if (n == 32 && issuers == 2)
        return launch_probe_t<32, 2>(reps, out, grid, s);
    if (n == 32 && issuers == 4)
        return launch_probe_t<32, 4>(reps, out, grid, s);
    return BL_ERR_SHAPE;
}

}  // namespace bl
