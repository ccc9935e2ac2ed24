// gemm.cu -- ternary prefill GEMM on the sm_100a tensor cores (tcgen05, int8).
//
// "How to Run BitNet Inference on GPU Using CUDA Kernels: A Complete Guide",
// FAQ: the kernel is a generic INT8 x INT2 GEMM; "BitCompute: 1.58-bit LLM
// Execution Engine", section "Future Roadmap": move the ternary add/subtract
// loops onto the tensor cores.
//
// acc[m][n] = sum_k code[n][k] q[m][k] = sum_k s[n][k] q[m][k] - rowsum[m],
// with s = code + 1 in {0,1,2} the stored 2-bit value.  The MMA multiplies the
// unsigned stored values by the signed activations; the epilogue subtracts the
// row sum and rescales.
//
// Tile: 128 weight rows (MMA M) x 128 tokens (MMA N), 128 k per stage, four
// stages.  Operands:
//   A (weights)  TL bytes of the tile arrive in shared memory by TMA (a 2-D
//                view [row groups][K/64 * 128 B], box 16 groups x 256 B); four
//                expansion warps turn each thread's row (one TMEM lane) into
//                int8 {0,1,2} -- (word >> 2i) & 0x03030303 gives four
//                consecutive k -- and write them straight into tensor memory
//                with tcgen05.st, so expanded weights never touch shared memory.
//   B (tokens)   int8 activations [M][K], TMA with 128-byte swizzle into the
//                canonical K-major layout the MMA descriptor describes.
//   D            int32 accumulators in tensor memory, 128 lanes x 128 columns.
// Warp roles (192 threads): warp 0 issues TMA, warp 1 allocates tensor memory
// and issues tcgen05.mma.kind::i8 (one thread), warps 2-5 expand and then run
// the epilogue (tcgen05.ld, subtract row sum, rescale, store).  Two CTAs fit
// per SM (tensor memory 2 x 256 columns, shared memory 2 x ~82 KB), so one
// CTA's epilogue overlaps the other's main loop.
//
// Every mbarrier wait is bounded (2 s of %globaltimer); on expiry the CTA
// records BL_ERR_TIMEOUT in the device status word, lets copies and MMAs in
// flight drain (bounded again), frees its tensor memory and returns.  No TMA
// multicast is used anywhere.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "bl_common.cuh"

namespace bl {
namespace {

constexpr int kBM = 128;     // weight rows per tile (MMA M)
constexpr int kBN = 128;     // tokens per tile (MMA N)
constexpr int kBK = 128;     // k per pipeline stage
constexpr int kStages = 4;
constexpr int kThreads = 192;
constexpr int kMmaK = 32;    // k per tcgen05.mma.kind::i8
constexpr uint32_t kTmemCols = 256;  // D: 128 columns; A: kStages x 32 columns
constexpr uint32_t kQStage = kBN * kBK;        // 16 KB of int8 activations
constexpr uint32_t kPStage = kBM * kBK / 4;    // 4 KB of packed weights
constexpr uint32_t kSmemQ = 0;
constexpr uint32_t kSmemP = kSmemQ + kStages * kQStage;
constexpr uint32_t kSmemBar = kSmemP + kStages * kPStage;
constexpr uint32_t kNumBars = 3 * kStages + 2;
constexpr uint32_t kSmemMisc = kSmemBar + kNumBars * 8;
constexpr uint32_t kSmemBytes = kSmemMisc + 16 + 1024;  // + alignment slack

struct GemmParams {
    const float *w_scale;
    const float *d;
    const int32_t *rowsum;
    int64_t M, N, K;
    void *y;
    int yt;
    int64_t ldy;
    int32_t *acc_dbg;
    int *status;
};

// ---------------------------------------------------------------- PTX wrappers

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, uint32_t bar,
                                            int32_t c0, int32_t c1)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1)
        : "memory");
}

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

// D[tmem] (+)= A[tmem] * B[smem]^T, int8 inputs, int32 accumulate.
__device__ __forceinline__ void mma_i8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void mma_commit(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

// Thirty-two consecutive 32-bit TMEM columns of this thread's lane.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32])
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
        "%28, %29, %30, %31, %32};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
        "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
        "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]),
        "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]),
        "r"(v[29]), "r"(v[30]), "r"(v[31])
        : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
        "%28, %29, %30, %31}, [%32];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
          "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),
          "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]),
          "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]),
          "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]),
          "=r"(v[31])
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

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

// Instruction descriptor: D int32, A unsigned 8-bit (stored codes), B signed
// 8-bit (activations), both K-major, M = 128, N = kBN.
constexpr uint32_t kIdesc = (2u << 4) | (0u << 7) | (1u << 10) | (uint32_t(kBN >> 3) << 17) |
                            (uint32_t(kBM >> 4) << 24);

// ---------------------------------------------------------------- kernel

__global__ void __launch_bounds__(kThreads, 1)
gemm_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap pmap,
            const GemmParams p)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    unsigned char *sm = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    const uint32_t sbase = smem_u32(sm);
    const uint32_t bar_full = sbase + kSmemBar;                  // TMA landed     [kStages]
    const uint32_t bar_afull = bar_full + 8 * kStages;          // A expanded     [kStages]
    const uint32_t bar_empty = bar_afull + 8 * kStages;         // MMA consumed   [kStages]
    const uint32_t bar_dfull = bar_empty + 8 * kStages;         // accumulators ready
    const uint32_t bar_drain = bar_dfull + 8;                   // teardown after an abort
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + kSmemMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + kSmemMisc + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t n0 = int64_t(blockIdx.x) * kBM;
    const int64_t m0 = int64_t(blockIdx.y) * kBN;
    const int KB = int((p.K + kBK - 1) / kBK);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(bar_full + 8 * s, 1);
            mbar_init(bar_afull + 8 * s, 128);
            mbar_init(bar_empty + 8 * s, 1);
        }
        mbar_init(bar_dfull, 1);
        mbar_init(bar_drain, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&qmap)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&pmap)) : "memory");
    }
    if (warp == 1)
        tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t d_tmem = tmem;                 // columns [0, 128)
    const uint32_t a_tmem0 = tmem + kBN;          // columns [128, 256): kStages x 32

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            int issued = 0;
            for (int kb = 0; kb < KB; ++kb) {
                const int s = kb % kStages;
                const uint32_t ph = uint32_t(kb / kStages) & 1u;
                if (!mbar_wait(bar_empty + 8 * s, ph ^ 1u, abort_flag, p.status))
                    break;
                mbar_arrive_tx(bar_full + 8 * s, kQStage + kPStage);
                tma_load_2d(sbase + kSmemQ + s * kQStage, &qmap, bar_full + 8 * s, kb * kBK,
                            int32_t(m0));
                tma_load_2d(sbase + kSmemP + s * kPStage, &pmap, bar_full + 8 * s, kb * (kBK * 2),
                            int32_t(n0 / 8));
                issued = kb + 1;
            }
            if (*abort_flag) {
                // let every copy this thread started land before the CTA exits
                for (int kb = issued > kStages ? issued - kStages : 0; kb < issued; ++kb) {
                    volatile int no_abort = 0;
                    mbar_wait(bar_full + 8 * (kb % kStages), uint32_t(kb / kStages) & 1u,
                              &no_abort, p.status, 100000000ull);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            int issued = 0;
            for (int kb = 0; kb < KB; ++kb) {
                const int s = kb % kStages;
                const uint32_t ph = uint32_t(kb / kStages) & 1u;
                if (!mbar_wait(bar_full + 8 * s, ph, abort_flag, p.status))
                    break;
                if (!mbar_wait(bar_afull + 8 * s, ph, abort_flag, p.status))
                    break;
                tc_fence_after();
                const uint32_t qaddr = sbase + kSmemQ + s * kQStage;
#pragma unroll
                for (int j = 0; j < kBK / kMmaK; ++j) {
                    const uint64_t bdesc = smem_desc_sw128(qaddr + j * kMmaK);
                    mma_i8_ts(d_tmem, a_tmem0 + s * (kBK / 4) + j * (kMmaK / 4), bdesc, kIdesc,
                              (kb > 0 || j > 0) ? 1u : 0u);
                }
                mma_commit(bar_empty + 8 * s);
                issued = kb + 1;
            }
            if (issued == KB) {
                mma_commit(bar_dfull);
            } else if (issued > 0) {
                // drain the MMAs in flight before tensor memory is released
                mma_commit(bar_drain);
                volatile int no_abort = 0;
                mbar_wait(bar_drain, 0, &no_abort, p.status, 100000000ull);
            }
        }
    } else {
        // ------------------------------------------------ expansion, then epilogue
        const int quarter = warp & 3;                 // TMEM lanes 32*quarter .. +31
        const int rl = quarter * 32 + lane;           // weight row within the tile
        const uint32_t lane_addr = uint32_t(quarter * 32) << 16;
        bool ok = true;
        for (int kb = 0; kb < KB; ++kb) {
            const int s = kb % kStages;
            const uint32_t ph = uint32_t(kb / kStages) & 1u;
            // warp-uniform outcome: the tcgen05.st below is .sync.aligned
            if (!__all_sync(0xffffffffu, mbar_wait(bar_full + 8 * s, ph, abort_flag, p.status))) {
                ok = false;
                break;
            }
            const unsigned char *ps = sm + kSmemP + s * kPStage + (rl >> 3) * 256 + (rl & 7) * 16;
            const uint4 c0 = *reinterpret_cast<const uint4 *>(ps);
            const uint4 c1 = *reinterpret_cast<const uint4 *>(ps + 128);
            const uint32_t wd[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
            uint32_t v[32];
#pragma unroll
            for (int w = 0; w < 8; ++w) {
                v[4 * w + 0] = wd[w] & 0x03030303u;
                v[4 * w + 1] = (wd[w] >> 2) & 0x03030303u;
                v[4 * w + 2] = (wd[w] >> 4) & 0x03030303u;
                v[4 * w + 3] = (wd[w] >> 6) & 0x03030303u;
            }
            tmem_st32(a_tmem0 + lane_addr + s * (kBK / 4), v);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar_afull + 8 * s);
        }
        if (ok && __all_sync(0xffffffffu, mbar_wait(bar_dfull, 0, abort_flag, p.status))) {
            tc_fence_after();
            const int64_t n = n0 + rl;
            const float gamma = p.w_scale[0];
#pragma unroll 1
            for (int c = 0; c < kBN / 32; ++c) {
                uint32_t v[32];
                tmem_ld32(d_tmem + lane_addr + c * 32, v);
                tmem_wait_ld();
                if (n < p.N) {
#pragma unroll 4
                    for (int j = 0; j < 32; ++j) {
                        const int64_t m = m0 + c * 32 + j;
                        if (m < p.M) {
                            const int a = int(v[j]) - __ldg(p.rowsum + m);
                            if (p.acc_dbg)
                                p.acc_dbg[m * p.N + n] = a;
                            store_y(p.y, p.yt, m * p.ldy + n, rescale1(a, __ldg(p.d + m), gamma));
                        }
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ---------------------------------------------------------------- host side

PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
        else
            cudaGetLastError();
    }
    return fn;
}

int make_map_2d(CUtensorMap *map, const void *base, uint64_t inner, uint64_t outer,
                uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, bool swizzle128)
{
    auto fn = encode_fn();
    if (!fn)
        return BL_ERR_CUDA;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? BL_OK : BL_ERR_CUDA;
}

}  // namespace

size_t gemm_workspace_bytes(int64_t, int64_t, int64_t) { return 0; }

int launch_gemm(const GemvArgs &a, void *, size_t, cudaStream_t s)
{
    const DeviceInfo *di = device_info();
    if (!di)
        return BL_ERR_CUDA;
    if (a.M > (int64_t(1) << 30) || a.N > (int64_t(1) << 30))
        return BL_ERR_SHAPE;
    CUtensorMap qmap, pmap;
    // activations: [M][K] int8, 128 x 128 boxes, 128-byte swizzle
    int st = make_map_2d(&qmap, a.q, uint64_t(a.K), uint64_t(a.M), uint64_t(a.K), kBK, kBN, true);
    if (st)
        return st;
    // packed weights as [row groups][K/64 * 128 B]: 16 groups x 256 B per stage
    const uint64_t rg_bytes = uint64_t(a.K / 64) * 128;
    st = make_map_2d(&pmap, a.packed, rg_bytes, uint64_t((a.N + 7) / 8), rg_bytes, 2 * kBK,
                     kBM / 8, false);
    if (st)
        return st;
    int per_sm = 0;
    if ((st = occupancy(reinterpret_cast<const void *>(gemm_kernel), kThreads, kSmemBytes, &per_sm)))
        return st;
    if (per_sm < 1)
        return BL_ERR_UNSUPPORTED;
    GemmParams p{a.w_scale, a.d, a.rowsum, a.M, a.N, a.K, a.y, a.yt, a.ldy, a.acc_dbg, di->status};
    dim3 grid(unsigned((a.N + kBM - 1) / kBM), unsigned((a.M + kBN - 1) / kBN));
    gemm_kernel<<<grid, kThreads, kSmemBytes, s>>>(qmap, pmap, p);
    return launch_status();
}

}  // namespace bl
