// gemv_tc.cu -- ternary GEMV for a small batch of tokens (2 .. 16) on the
// tensor cores, one launch with the activation quantisation fused in.
//
// "How to Run BitNet Inference on GPU Using CUDA Kernels: A Complete Guide",
// section "Understanding the Two-Phase Architecture": decode multiplies INT8
// activations by INT2 weights and is bound by the weight stream; "BitCompute:
// 1.58-bit LLM Execution Engine", section "Future Roadmap": put the ternary
// products on the tensor cores.  With a few tokens per step the dp4a form
// pays one dot-product instruction per four weights and token, while a
// tensor-core MMA pays only for expanding each weight once.
//
// acc[m][n] = sum_k code[n][k] q[m][k] = sum_k s[n][k] q[m][k] - rowsum[m]
// with s = code + 1 in {0,1,2}, the stored 2-bit value.
//
// Design (B200):
//   * Output rows are taken in blocks of 128 (sixteen 8-row groups of the
//     tile layout, one MMA M).  The k range of a block is split over the cs
//     CTAs of a thread-block cluster (cs = 1 .. 8), at most six stages of
//     256 k per CTA, so that a CTA's whole share of expanded weights sits in
//     its tensor memory at once (6 x 64 columns + 4 accumulators of 32).
//   * Right after the barriers are initialised every bulk copy of the CTA's
//     packed weights is issued, one per thread (the copies of one thread
//     complete one after another).  Eight expansion warps turn each stage
//     into int8 codes {0,1,2} in tensor memory (tcgen05.st) as it lands.
//     None of this needs the activations, so it overlaps the preceding
//     launch (programmatic dependent launch) and the activation reads.
//   * Eight prologue warps read the CTA's k range of every token (two tokens
//     a warp, all loads in flight together) and send each token's partial
//     absmax to every CTA of the cluster (st.async into its shared memory,
//     counted on its mbarrier); with the full absmax each CTA quantises its
//     k range into the MMA's B operand (32 token rows x k, K-major, 128-byte
//     swizzle; rows beyond M are zero) and keeps its partial row sums of q.
//   * Four warps issue the MMAs (128 x 32 x 32, kind::i8, A = codes in tensor
//     memory, B = q in shared memory), stage j by warp j mod 4 into its own
//     accumulator: one thread issues at most one such MMA per ~53 cycles,
//     four reach the tensor rate (16 cycles per MMA per SM, measured).
//   * Four warps read the accumulators back (tcgen05.ld, the first 16
//     columns of each), sum them, subtract the CTA's partial row sums and add
//     the result into the cluster leader's shared memory (red.async, counted
//     on the leader's mbarrier); the leader rescales and writes every (token,
//     row).  With cs = 1 the CTA rescales and writes its rows directly.
//   * Every mbarrier wait is bounded; on expiry the CTA records
//     BL_ERR_TIMEOUT, each part leaves its loop, MMAs and copies in flight
//     drain (bounded), a CTA waits (bounded) for the remote writes counted on
//     its own barriers before it exits, and tensor memory is freed.
#include <map>
#include <mutex>
#include <tuple>

#include "gemv_stream_common.cuh"
#include "tcgen05_common.cuh"

namespace bl {
namespace {

constexpr int kTcgTokens = 16;                     // tokens of a launch, at most
constexpr int kTcgN = 32;                          // MMA N: the tokens, padded with zero rows
constexpr int kTcgRows = 128;                      // MMA M: output rows of a block
constexpr int kTcgGroups = kTcgRows / 8;           // 8-row groups of a block
constexpr int kTcgMaxStages = 6;                   // 256-k stages of one CTA
constexpr int kTcgMaxCluster = 8;
constexpr int kTcgIssuers = 4;                     // MMA-issuing warps, one accumulator each
constexpr int kTcgExpWarp0 = kTcgIssuers;
constexpr int kTcgExpWarps = 8;                    // two per tensor-memory lane quarter
constexpr int kTcgProWarp0 = kTcgExpWarp0 + kTcgExpWarps;
constexpr int kTcgProWarps = 8;                    // prologue; the first four also drain D
constexpr int kTcgThreads = 32 * (kTcgProWarp0 + kTcgProWarps);
constexpr uint32_t kTcgTmemCols = 512;
constexpr uint32_t kTcgDCols = 32;                 // one accumulator: 128 lanes x N columns
constexpr uint32_t kTcgACol0 = kTcgIssuers * kTcgDCols;   // A stage j at columns 128 + 64 j
constexpr uint32_t kTcgBBox = kTcgN * 128;         // bytes of one 128-k box of B
// D int32, A unsigned 8-bit (stored codes), B signed 8-bit, both K-major,
// M = 128, N = 32 (the shape of the prefill GEMM's small-batch tiles).
constexpr uint32_t kTcgIdesc = (2u << 4) | (0u << 7) | (1u << 10) | (uint32_t(kTcgN >> 3) << 17) |
                               (uint32_t(kTcgRows >> 4) << 24);
static_assert(kTcgACol0 + kTcgMaxStages * 64 <= kTcgTmemCols, "tensor memory budget");
static_assert(kTcgN <= int(kTcgDCols), "accumulator columns");
static_assert(kTcgProWarps * 2 == kTcgTokens, "two tokens per prologue warp");

enum { TCG_Q = 0, TCG_X_BF16 = 1 };

struct TcgParams {
    GemvProblem prob[kGemvMaxProblems];
    int rbstart[kGemvMaxProblems + 1];   // prefix sums of the products' 128-row blocks
    int count;
    int64_t K;
    int M;
    int cs;                              // CTAs per cluster: the k split of a block
    const int8_t *q;                     // TCG_Q: [M][K] and d [M]
    const float *d;
    const void *x;                       // TCG_X_BF16: [M][ldx] bf16
    int64_t ldx;
    int yt;
    int *status;
};

struct TcgSmem {
    unsigned char b[kTcgMaxStages][2][kTcgBBox];        // B operand (1024-byte aligned boxes)
    unsigned char pk[kTcgMaxStages][kTcgGroups][512];   // packed weights: stage, group
    uint4 xs[kTcgTokens][kTcgMaxStages * 32];           // raw bf16 activations of the k range
    int acc[kTcgTokens][kTcgRows];                      // leader: the cluster's summed partials
    float amx[kTcgMaxCluster][kTcgTokens];              // partial absmax of each rank, per token
    int rsum[kTcgTokens];                               // this CTA's partial row sums of q
    float dq[kTcgTokens];                               // per-token d
    uint64_t full[kTcgMaxStages];                       // packed bytes of stage j landed
    uint64_t afull[kTcgMaxStages];                      // stage j expanded into tensor memory
    uint64_t bready;                                    // B quantised (one arrival per prologue warp)
    uint64_t xmax;                                      // every rank's partial absmax arrived
    uint64_t dsum;                                      // leader: every rank's partial sums arrived
    uint64_t dfull;                                     // every issuer's MMAs complete
    uint64_t drain[kTcgIssuers];                        // teardown, per issuer
    uint32_t tmem_base;
    int abort_flag;
};
static_assert(offsetof(TcgSmem, pk) % 16 == 0, "bulk copy destinations");
// One CTA per SM, always: a second CTA of the same cluster on an SM would
// wait in tcgen05.alloc for the first one's 512 columns while the first waits
// for it.  The dynamic shared memory asked for is kept above half of the SM's.
constexpr size_t kTcgSmemNeed = sizeof(TcgSmem) + 1024;   // + alignment slack
constexpr size_t kTcgSmemBytes = kTcgSmemNeed > 120 * 1024 ? kTcgSmemNeed : 120 * 1024;
static_assert(kTcgSmemBytes <= 227 * 1024, "shared memory per CTA");

// ---- cluster helpers (distributed shared memory)

__device__ __forceinline__ uint32_t cluster_rank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_arrive() { asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory"); }
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory"); }

// The address of this CTA's shared variable at `saddr` in the CTA of rank `rank`.
__device__ __forceinline__ uint32_t map_rank(uint32_t saddr, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}

// Asynchronous store / add into another CTA's shared memory, its four bytes
// counted on that CTA's mbarrier (both addresses from map_rank).
__device__ __forceinline__ void st_async_f32(uint32_t addr, float v, uint32_t bar)
{
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.f32 [%0], %1, [%2];" ::"r"(addr), "f"(v),
                 "r"(bar)
                 : "memory");
}

__device__ __forceinline__ void red_async_add(uint32_t addr, int v, uint32_t bar)
{
    asm volatile("red.async.relaxed.cluster.shared::cluster.mbarrier::complete_tx::bytes.add.s32 [%0], %1, [%2];" ::"r"(
                     addr),
                 "r"(v), "r"(bar)
                 : "memory");
}

// Byte offset in B of token t's 8 activations k_local = 8 c .. 8 c + 7 of the
// CTA's range, c = lane + 32 i: stage i, box lane / 16, 16-byte chunk
// (lane % 16) / 2 of the token's 128-byte row, swizzled by the row (t % 8)
// as the 128-byte swizzle mode expects, half lane % 2 of the chunk.
__device__ __forceinline__ uint32_t b_offset(int t, int i, int lane)
{
    return uint32_t(i * 2 + (lane >> 4)) * kTcgBBox + uint32_t(t >> 3) * 1024 + uint32_t(t & 7) * 128 +
           uint32_t((((lane & 15) >> 1) ^ (t & 7)) * 16) + uint32_t(lane & 1) * 8;
}

__device__ __forceinline__ void bar_arrive(int id, int nthreads)
{
    asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Named barriers: warp 0 initialises the mbarriers and warp 1 allocates the
// tensor memory, side by side; each arrives on the barriers of the warps that
// need its work, which wait there as late as they can.
constexpr int kBarInit = 1;     // mbarriers initialised: the expansion warps (copies) and issuers 1 .. 3
constexpr int kBarAlloc = 2;    // tensor memory allocated: the expansion warps and issuers 0, 2, 3
constexpr int kBarPro = 3;      // both, for the prologue warps (after their activation loads)
constexpr int kBarProAll = 4;   // the prologue warps among themselves
constexpr int kBarInitN = 32 * (kTcgIssuers + kTcgExpWarps);
constexpr int kBarAllocN = 32 * (kTcgIssuers + kTcgExpWarps);
constexpr int kBarProN = 32 * (2 + kTcgProWarps);

template <int MODE>
__global__ void __launch_bounds__(kTcgThreads, 1) gemv_tc_kernel(const TcgParams p)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    TcgSmem &sm = *reinterpret_cast<TcgSmem *>(smem_raw + (((raw + 1023u) & ~1023u) - raw));
    volatile int *abort_flag = &sm.abort_flag;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int cs = p.cs;
    const uint32_t rank = cluster_rank();
    const int rb = int(blockIdx.x) / cs;
    int pi = 0;
#pragma unroll
    for (int i = 1; i < kGemvMaxProblems; ++i)
        if (i < p.count && rb >= p.rbstart[i])
            pi = i;
    const GemvProblem &pr = p.prob[pi];
    const int64_t g0 = int64_t(rb - p.rbstart[pi]) * kTcgGroups;       // first row group of the block
    const int64_t ng_all = (pr.N + 7) / 8;
    const int ngr = int(ng_all - g0 < kTcgGroups ? ng_all - g0 : kTcgGroups);
    const int S = int(p.K / 256);
    const int st0 = int(rank) * S / cs;
    const int ns = (int(rank) + 1) * S / cs - st0;                      // 1 .. kTcgMaxStages
    const bool fold = cs > 1;                                           // partial sums go to the leader
    // bytes each rank's partial maxima / partial sums bring to a CTA's barrier
    const uint32_t xmax_bytes = MODE == TCG_X_BF16 ? uint32_t(cs * p.M) * 4u : 0u;
    const uint32_t dsum_bytes = uint32_t(cs * p.M * kTcgRows) * 4u;
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    if (warp < kTcgIssuers) {
        // ------------------------------------------------ barriers, tensor memory (warp 0), then the MMAs
        // issuer w takes the stages j = w (mod kTcgIssuers) into accumulator
        // w: one thread cannot issue tcgen05.mma of N = 32 faster than about
        // one per 53 cycles, four threads together reach the tensor rate
        const int nd = ns < kTcgIssuers ? ns : kTcgIssuers;     // accumulators in use
        if (warp == 0) {
            if (lane == 0) {
                for (int j = 0; j < kTcgMaxStages; ++j) {
                    mbar_init(smem_u32(&sm.full[j]), 1);
                    mbar_init(smem_u32(&sm.afull[j]), kTcgRows);
                }
                for (int w = 0; w < kTcgIssuers; ++w)
                    mbar_init(smem_u32(&sm.drain[w]), 1);
                mbar_init(smem_u32(&sm.bready), kTcgProWarps);
                mbar_init(smem_u32(&sm.xmax), 1);
                mbar_init(smem_u32(&sm.dsum), 1);
                mbar_init(smem_u32(&sm.dfull), uint32_t(nd));
                sm.abort_flag = 0;
                asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
            }
            __syncwarp();
            bar_arrive(kBarInit, kBarInitN);
            bar_arrive(kBarPro, kBarProN);
            // phase 0 of the cluster barrier: this CTA runs and its mbarriers
            // are initialised.  A thread waits on it only before its first
            // access to another CTA's shared memory.
            cluster_arrive();
            named_barrier(kBarAlloc, kBarAllocN);
        } else if (warp == 1) {
            cluster_arrive();
            tmem_alloc(smem_u32(&sm.tmem_base), kTcgTmemCols);
            tc_fence_before();
            bar_arrive(kBarAlloc, kBarAllocN);
            bar_arrive(kBarPro, kBarProN);
            named_barrier(kBarInit, kBarInitN);
        } else {
            cluster_arrive();
            named_barrier(kBarInit, kBarInitN);
            named_barrier(kBarAlloc, kBarAllocN);
        }
        tc_fence_after();
        const uint32_t tmem = sm.tmem_base;
        bool ok = __all_sync(0xffffffffu, mbar_wait_fast(smem_u32(&sm.bready), 0, abort_flag, p.status));
        bool issued = false;
        const uint64_t b_desc0 = smem_desc_sw128(smem_u32(sm.b[0][0]));
        for (int j = warp; j < ns && ok; j += kTcgIssuers) {
            if (!__all_sync(0xffffffffu, mbar_wait_fast(smem_u32(&sm.afull[j]), 0, abort_flag, p.status))) {
                ok = false;
                break;
            }
            tc_fence_after();
            mma_stage8<(kTcgBBox >> 4)>(tmem + kTcgDCols * uint32_t(warp), tmem + kTcgACol0 + 64u * uint32_t(j),
                                        b_desc0 + uint64_t(j) * (2 * kTcgBBox >> 4), kTcgIdesc,
                                        j >= kTcgIssuers ? 1u : 0u);
            issued = true;
        }
        if (ok && issued)
            mma_commit(smem_u32(&sm.dfull));
        if (issued) {
            // this warp's MMAs have completed before tensor memory is released
            mma_commit(smem_u32(&sm.drain[warp]));
            volatile int no_abort = 0;
            mbar_wait(smem_u32(&sm.drain[warp]), 0, &no_abort, p.status, 100000000ull);
        }
    } else if (warp < kTcgProWarp0) {
        // ------------------------------------------------ copies, then expansion into tensor memory
        cluster_arrive();
        named_barrier(kBarInit, kBarInitN);
        // one bulk copy per thread (a thread's copies complete one after
        // another): thread u copies group u % 16 of stage u / 16
        const int u = tid - 32 * kTcgExpWarp0;
        {
            const int j = u >> 4, g = u & 15;
            if (j < ns && g < ngr) {
                if (g == 0)
                    mbar_arrive_tx(smem_u32(&sm.full[j]), uint32_t(ngr) * 512u);
                bulk_load(smem_u32(sm.pk[j][g]), pr.packed + (g0 + g) * (2 * p.K) + int64_t(st0 + j) * 512, 512u,
                          smem_u32(&sm.full[j]));
            }
        }
        named_barrier(kBarAlloc, kBarAllocN);
        tc_fence_after();
        const uint32_t tmem = sm.tmem_base;
        const int e = (warp - kTcgExpWarp0) >> 2;     // expands the stages j = e (mod 2)
        const int quarter = warp & 3;                 // tensor-memory lanes 32 quarter .. + 31
        const int row = quarter * 32 + lane;          // output row within the block
        const uint32_t lane_addr = uint32_t(quarter * 32) << 16;
        const int grp = row >> 3;
        for (int j = e; j < ns; j += 2) {
            if (!__all_sync(0xffffffffu, mbar_wait_fast(smem_u32(&sm.full[j]), 0, abort_flag, p.status)))
                break;
            uint4 c4[4];
#pragma unroll
            for (int c = 0; c < 4; ++c)
                c4[c] = grp < ngr ? *reinterpret_cast<const uint4 *>(sm.pk[j][grp] + c * 128 + (row & 7) * 16)
                                  : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint32_t v[32];
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    const uint4 w4 = c4[2 * h + cc];
                    const uint32_t wd[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
                    for (int w = 0; w < 4; ++w)
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            v[16 * cc + 4 * w + i] = (wd[w] >> (2 * i)) & 0x03030303u;
                }
                tmem_st32_wait(tmem + lane_addr + kTcgACol0 + 64u * uint32_t(j) + 32u * uint32_t(h), v);
            }
            tc_fence_before();
            mbar_arrive(smem_u32(&sm.afull[j]));
        }
        // the copies have landed before the CTA exits (at once unless an
        // expansion warp gave up before consuming them)
        if (u < 16 * ns) {
            volatile int no_abort = 0;
            mbar_wait(smem_u32(&sm.full[u >> 4]), 0, &no_abort, p.status, 100000000ull);
        }
    } else {
        // ------------------------------------------------ prologue (activations), then D
        const int pw = warp - kTcgProWarp0;
        const int ptid = tid - 32 * kTcgProWarp0;
        // the activations first: every other step of the prologue runs
        // while their loads are in flight
        asm volatile("griddepcontrol.wait;" ::: "memory");
        const int64_t k0 = int64_t(st0) * 256;
        uint4 raw4[2][kTcgMaxStages];
        if constexpr (MODE == TCG_X_BF16) {
#pragma unroll
            for (int tt = 0; tt < 2; ++tt) {
                const int t = pw + 8 * tt;
                const __nv_bfloat16 *xr = static_cast<const __nv_bfloat16 *>(p.x) + int64_t(t) * p.ldx + k0;
#pragma unroll
                for (int i = 0; i < kTcgMaxStages; ++i)
                    raw4[tt][i] = (t < p.M && i < ns) ? ld_dep_v4(xr + (lane + 32 * i) * 8) : make_uint4(0, 0, 0, 0);
            }
        }
        if (fold && rank == 0)      // the leader's sums start from zero before any rank adds to them
            for (int i = ptid; i < kTcgTokens * kTcgRows; i += 32 * kTcgProWarps)
                (&sm.acc[0][0])[i] = 0;
        cluster_arrive();           // (after the zeroing: every rank waits on phase 0 before adding)
        // rows of B for tokens beyond M (and the padding rows 16 .. 31) are zero
#pragma unroll
        for (int tt = 0; tt < 4; ++tt) {
            const int t = pw + 8 * tt;
            if (t >= p.M)
                for (int i = lane; i < ns * 2 * 8; i += 32)
                    *reinterpret_cast<uint4 *>(&sm.b[0][0][0] + uint32_t(i >> 3) * kTcgBBox + uint32_t(t >> 3) * 1024 +
                                               uint32_t(t & 7) * 128 + uint32_t(i & 7) * 16) = make_uint4(0, 0, 0, 0);
        }
        bool ok = true;
        if constexpr (MODE == TCG_X_BF16) {
            // the loaded activations are kept in shared memory (each thread
            // reads back only what it stored) until the full absmax is known
            float am[2];
#pragma unroll
            for (int tt = 0; tt < 2; ++tt) {
                const int t = pw + 8 * tt;
                float a = 0.0f;
#pragma unroll
                for (int i = 0; i < kTcgMaxStages; ++i) {
                    float f[8];
                    bf16x8_f32(raw4[tt][i], f);
#pragma unroll
                    for (int e2 = 0; e2 < 8; ++e2)
                        a = fmaxf(a, fabsf(f[e2]));
                    if (t < p.M && i < ns)
                        sm.xs[t][lane + 32 * i] = raw4[tt][i];
                }
                // maxima are >= 0 and finite: bit patterns order like the values
                am[tt] = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(a)));
            }
            named_barrier(kBarPro, kBarProN);   // barriers initialised
            if (ptid == 0) {
                mbar_arrive_tx(smem_u32(&sm.xmax), xmax_bytes);
                if (fold && rank == 0)
                    mbar_arrive_tx(smem_u32(&sm.dsum), dsum_bytes);
            }
            cluster_wait();     // phase 0: every CTA of the cluster runs
            if (lane == 0) {
#pragma unroll
                for (int tt = 0; tt < 2; ++tt) {
                    const int t = pw + 8 * tt;
                    if (t < p.M)
                        for (int r = 0; r < cs; ++r)
                            st_async_f32(map_rank(smem_u32(&sm.amx[rank][t]), uint32_t(r)), am[tt],
                                         map_rank(smem_u32(&sm.xmax), uint32_t(r)));
                }
            }
            ok = __all_sync(0xffffffffu, mbar_wait_fast(smem_u32(&sm.xmax), 0, abort_flag, p.status));
            int sum[2] = {0, 0};
#pragma unroll
            for (int tt = 0; tt < 2; ++tt) {
                const int t = pw + 8 * tt;
                if (t < p.M) {
                    float a = 0.0f;
                    for (int r = 0; r < cs; ++r)
                        a = fmaxf(a, sm.amx[r][t]);
                    const float a_eff = fmaxf(a, kEps);
                    const float sc = __fdiv_rn(kQb, a_eff);
#pragma unroll
                    for (int i = 0; i < kTcgMaxStages; ++i) {
                        if (i < ns) {
                            float f[8];
                            bf16x8_f32(sm.xs[t][lane + 32 * i], f);
                            *reinterpret_cast<uint2 *>(&sm.b[0][0][0] + b_offset(t, i, lane)) = quant8(f, sc, sum[tt]);
                        }
                    }
                    if (lane == 0)
                        sm.dq[t] = __fdiv_rn(a_eff, kQb);
                }
            }
            // B is read by the tensor cores (async proxy)
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0)
                mbar_arrive(smem_u32(&sm.bready));
#pragma unroll
            for (int tt = 0; tt < 2; ++tt) {
                const int t = pw + 8 * tt;
                const int s2 = __reduce_add_sync(0xffffffffu, sum[tt]);
                if (t < p.M && lane == 0)
                    sm.rsum[t] = s2;
            }
        } else {
            // pre-quantised: copy the CTA's k range of q, partial row sums from it
            int sum[2] = {0, 0};
#pragma unroll
            for (int tt = 0; tt < 2; ++tt) {
                const int t = pw + 8 * tt;
                if (t < p.M) {
#pragma unroll
                    for (int i = 0; i < kTcgMaxStages; ++i) {
                        if (i < ns) {
                            const unsigned long long w =
                                ld_dep_u64(p.q + int64_t(t) * p.K + k0 + (lane + 32 * i) * 8);
                            const uint32_t lo = uint32_t(w), hi = uint32_t(w >> 32);
                            sum[tt] = dp4a_us(0x01010101u, lo, sum[tt]);
                            sum[tt] = dp4a_us(0x01010101u, hi, sum[tt]);
                            *reinterpret_cast<uint2 *>(&sm.b[0][0][0] + b_offset(t, i, lane)) = make_uint2(lo, hi);
                        }
                    }
                    if (lane == 0)
                        sm.dq[t] = __uint_as_float(ld_dep_u32(p.d + t));
                }
            }
            named_barrier(kBarPro, kBarProN);   // barriers initialised
            if (ptid == 0 && fold && rank == 0)
                mbar_arrive_tx(smem_u32(&sm.dsum), dsum_bytes);
            cluster_wait();     // phase 0 (the epilogue's remote additions follow)
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0)
                mbar_arrive(smem_u32(&sm.bready));
#pragma unroll
            for (int tt = 0; tt < 2; ++tt) {
                const int t = pw + 8 * tt;
                const int s2 = __reduce_add_sync(0xffffffffu, sum[tt]);
                if (t < p.M && lane == 0)
                    sm.rsum[t] = s2;
            }
        }
        named_barrier(kBarProAll, 32 * kTcgProWarps);    // rsum and dq of every token
        tc_fence_after();
        const uint32_t tmem = sm.tmem_base;
        if (pw < 4) {
            // D: 128 rows x 32 columns, the first 16 the tokens; this warp's lane quarter
            const int quarter = warp & 3;
            const int row = quarter * 32 + lane;
            const uint32_t lane_addr = uint32_t(quarter * 32) << 16;
            const float gamma = __ldg(pr.w_scale);
            const int64_t n = g0 * 8 + row;
            if (ok && __all_sync(0xffffffffu, mbar_wait_fast(smem_u32(&sm.dfull), 0, abort_flag, p.status))) {
                tc_fence_after();
                uint32_t v[16];
                tmem_ld16_wait(tmem + lane_addr, v);
                const int nd = ns < kTcgIssuers ? ns : kTcgIssuers;
                for (int w = 1; w < nd; ++w) {
                    uint32_t v2[16];
                    tmem_ld16_wait(tmem + lane_addr + kTcgDCols * uint32_t(w), v2);
#pragma unroll
                    for (int m = 0; m < 16; ++m)
                        v[m] += v2[m];
                }
                if (!fold) {
                    if (n < pr.N) {
#pragma unroll
                        for (int m = 0; m < kTcgTokens; ++m) {
                            if (m < p.M) {
                                const int a = int(v[m]) - sm.rsum[m];
                                if (pr.acc_dbg)
                                    pr.acc_dbg[int64_t(m) * pr.N + n] = a;
                                store_y(pr.y, p.yt, int64_t(m) * pr.ldy + n, rescale1(a, sm.dq[m], gamma));
                            }
                        }
                    }
                } else {
                    const uint32_t bar0 = map_rank(smem_u32(&sm.dsum), 0u);
#pragma unroll
                    for (int m = 0; m < kTcgTokens; ++m)
                        if (m < p.M)
                            red_async_add(map_rank(smem_u32(&sm.acc[m][row]), 0u), int(v[m]) - sm.rsum[m], bar0);
                }
            }
            if (fold && rank == 0 &&
                __all_sync(0xffffffffu, mbar_wait_fast(smem_u32(&sm.dsum), 0, abort_flag, p.status)) && n < pr.N) {
                // the leader: every rank's partial sums have arrived
#pragma unroll
                for (int m = 0; m < kTcgTokens; ++m) {
                    if (m < p.M) {
                        const int a = sm.acc[m][row];
                        if (pr.acc_dbg)
                            pr.acc_dbg[int64_t(m) * pr.N + n] = a;
                        store_y(pr.y, p.yt, int64_t(m) * pr.ldy + n, rescale1(a, sm.dq[m], gamma));
                    }
                }
            }
        }
        // remote writes into this CTA have landed before it exits (at once
        // unless some part gave up)
        if (ptid == 0) {
            volatile int no_abort = 0;
            if (xmax_bytes)
                mbar_wait(smem_u32(&sm.xmax), 0, &no_abort, p.status, 100000000ull);
            if (fold && rank == 0)
                mbar_wait(smem_u32(&sm.dsum), 0, &no_abort, p.status, 100000000ull);
        }
    }

    // ---------------------------------------------------- teardown
    if (warp < kTcgProWarp0)
        cluster_wait();     // phase 0 (the prologue warps waited already)
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(sm.tmem_base, kTcgTmemCols);
    }
}

// Clusters of `cs` CTAs of this kernel that can be resident at once.
template <int MODE>
int tc_capacity(int cs, int *clusters)
{
    static std::mutex mu;
    static std::map<std::tuple<int, int, int>, int> cache;
    const DeviceInfo *di = device_info();
    if (!di)
        return BL_ERR_CUDA;
    std::lock_guard<std::mutex> lock(mu);
    const auto key = std::make_tuple(di->device, MODE, cs);
    auto it = cache.find(key);
    if (it != cache.end()) {
        *clusters = it->second;
        return BL_OK;
    }
    auto kern = gemv_tc_kernel<MODE>;
    int per_sm = 0;
    int st = occupancy(reinterpret_cast<const void *>(kern), kTcgThreads, kTcgSmemBytes, &per_sm);
    if (st)
        return st;
    int n = 0;
    if (per_sm == 1) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(unsigned(cs));
        cfg.blockDim = dim3(kTcgThreads);
        cfg.dynamicSmemBytes = kTcgSmemBytes;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = unsigned(cs);
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if ((st = cuda_status(cudaOccupancyMaxActiveClusters(&n, kern, &cfg))))
            return st;
    }
    cache[key] = n;
    *clusters = n;
    return BL_OK;
}

// The cluster size for a launch of rb blocks over S stages of 256 k: the
// largest of 1 .. 8 that leaves every CTA at most kTcgMaxStages stages
// and at least one, and whose grid is resident at once; 0 if none.
template <int MODE>
int tc_pick_cs(int64_t rb, int S, int *cs_out)
{
    *cs_out = 0;
    for (int cs = kTcgMaxCluster; cs >= 1; --cs) {
        if (cs > S || (S + cs - 1) / cs > kTcgMaxStages)
            continue;
        int clusters = 0;
        int st = tc_capacity<MODE>(cs, &clusters);
        if (st)
            return st;
        if (rb <= clusters) {
            *cs_out = cs;
            return BL_OK;
        }
    }
    return BL_OK;
}

int64_t tc_blocks(const GemvBatch &b)
{
    int64_t rb = 0;
    for (int i = 0; i < b.count; ++i)
        rb += (b.prob[i].N + kTcgRows - 1) / kTcgRows;
    return rb;
}

}  // namespace

// 2 .. 16 tokens, K a multiple of 256, bf16 activations (fused) or
// pre-quantised q, and a cluster split whose grid is resident at once: the
// cluster size, 0 if the kernel does not take the batch.
int gemv_tc_cluster(const GemvBatch &b, bool fused)
{
    if (b.M < 2 || b.M > kTcgTokens || b.K % 256 != 0 || b.K < 256 || b.count < 1)
        return 0;
    if (fused && b.xt != BL_BF16)
        return 0;
    int cs = 0;
    const int S = int(b.K / 256);
    const int st = fused ? tc_pick_cs<TCG_X_BF16>(tc_blocks(b), S, &cs) : tc_pick_cs<TCG_Q>(tc_blocks(b), S, &cs);
    if (st) {
        cudaGetLastError();
        return 0;
    }
    return cs;
}

bool gemv_tc_applies(const GemvBatch &b, bool fused) { return gemv_tc_cluster(b, fused) > 0; }

int launch_gemv_tc(const GemvBatch &b, bool fused, cudaStream_t s)
{
    const DeviceInfo *di = device_info();
    if (!di)
        return BL_ERR_CUDA;
    TcgParams p{};
    p.count = b.count;
    p.rbstart[0] = 0;
    for (int i = 0; i < b.count; ++i) {
        p.prob[i] = b.prob[i];
        p.rbstart[i + 1] = p.rbstart[i] + int((b.prob[i].N + kTcgRows - 1) / kTcgRows);
    }
    for (int i = b.count; i < kGemvMaxProblems; ++i)
        p.rbstart[i + 1] = p.rbstart[b.count];
    p.K = b.K;
    p.M = int(b.M);
    p.q = b.q;
    p.d = b.d;
    p.x = b.x;
    p.ldx = b.ldx;
    p.yt = b.yt;
    p.status = di->status;
    const int S = int(b.K / 256);
    const int64_t rb = p.rbstart[b.count];
    int cs = 0;
    int st = fused ? tc_pick_cs<TCG_X_BF16>(rb, S, &cs) : tc_pick_cs<TCG_Q>(rb, S, &cs);
    if (st)
        return st;
    if (cs < 1)
        return BL_ERR_SHAPE;
    p.cs = cs;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(rb * cs));
    cfg.blockDim = dim3(kTcgThreads);
    cfg.dynamicSmemBytes = kTcgSmemBytes;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = unsigned(cs);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (b.flags & BL_FLAG_PDL) {
        attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[1].val.programmaticStreamSerializationAllowed = 1;
        cfg.numAttrs = 2;
    }
    if (fused)
        return cuda_status(cudaLaunchKernelEx(&cfg, gemv_tc_kernel<TCG_X_BF16>, p));
    return cuda_status(cudaLaunchKernelEx(&cfg, gemv_tc_kernel<TCG_Q>, p));
}

}  // namespace bl
