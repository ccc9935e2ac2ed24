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
// Persistent kernel, one CTA per SM, walking output tiles of 128 weight rows
// (MMA M) x 128 tokens (MMA N); k advances 256 per pipeline stage.  A stage is
// eight MMAs (128x128x32, 64 tensor cycles each): an issuing thread that waits
// on a barrier once per stage cannot issue faster than about one stage per
// 480 cycles, so a stage carries at least that much tensor work.  Operands:
//   B (tokens)   int8 activations [M][K]: two TMA boxes of 128 tokens x 128 k
//                per stage with 128-byte swizzle (the canonical K-major layout
//                of the MMA descriptor), in a five-slot shared-memory ring.
//   A (weights)  TL bytes of the tile arrive in the same ring slot by TMA (a
//                2-D view [row groups][K/64 * 128 B], two boxes of 16 groups x
//                256 B); each expansion thread owns one weight row (one TMEM
//                lane) and turns its bytes into int8 {0,1,2} -- (word >> 2i) &
//                0x03030303 gives four consecutive k -- written straight into a
//                four-stage ring in tensor memory with tcgen05.st.
//   D            int32 accumulators in tensor memory, two buffers of 128 lanes
//                x 128 columns: the epilogue drains one tile while the MMAs of
//                the next accumulate into the other.
// Tensor memory: D 2 x 128 columns + A 4 stages x 64 columns = 512 columns.
//
// Warp roles (608 threads):
//   warps 0-1    TMA producers.  Warp w copies the stages g = w (mod 2): lanes
//                0-1 the two activation boxes, lanes 2-3 the two packed weight
//                boxes, side by side.  TMA copies issued
//                by one thread complete one after another, so the ring is
//                spread over several threads, and over warps rather than lanes
//                of one warp, because lanes that wait on different barriers
//                move in lockstep.
//   warp 2       tensor memory allocation; lane 0 issues tcgen05.mma.kind::i8
//                after the stage's expansion barrier and its TMA barrier, the
//                whole warp running the loop.
//   warps 3-10   expansion of the packed weights into tensor memory, two groups
//                of four warps (one per TMEM lane quarter) taking alternate
//                stages: an mbarrier check costs a couple of hundred cycles
//                even when the phase has completed, and one stage's expansion
//                with its checks takes longer than the stage's MMAs.
//   warps 11-18  epilogue: tcgen05.ld, subtract the row sum, rescale, store;
//                two warps per TMEM lane quarter, each draining 64 token
//                columns, so a tile's epilogue fits in the next tile's main
//                loop even at K = 2560.  Per-token d and row sums are staged
//                in shared memory per warp.
//
// Every mbarrier wait is bounded (2 s of %globaltimer); on expiry the CTA
// records BL_ERR_TIMEOUT in the device status word, every role leaves its
// loop, copies and MMAs in flight drain (bounded again), tensor memory is
// freed and the CTA returns.  No TMA multicast is used anywhere.
#include <algorithm>

#include <cuda.h>
#include <cudaTypedefs.h>

#include "tcgen05_common.cuh"

namespace bl {
namespace {

constexpr int kBM = 128;     // weight rows per tile (MMA M)
constexpr int kBK = kTcStageK;   // k per pipeline stage: eight MMAs between barrier waits
constexpr int kBoxK = kTcBoxK;  // k per TMA box (one 128-byte swizzle span of activations)
constexpr int kBoxes = kBK / kBoxK;
constexpr int kQStages = 5;  // operand ring (shared memory): activations and packed weights
constexpr int kAStages = 4;  // expanded weight ring (tensor memory)
constexpr int kExpGroups = 2;  // expansion groups, taking alternate stages
constexpr int kProducerWarps = 2;
constexpr int kMmaWarp = kProducerWarps;
constexpr int kExpWarp0 = kMmaWarp + 1;
constexpr int kEpiWarp0 = kExpWarp0 + 4 * kExpGroups;
constexpr uint32_t kTmemCols = 512;  // D: 2 x BN columns in [0, 256); A: kAStages x 64 columns in [256, 512)
constexpr uint32_t kDCols = 256;
constexpr uint32_t kPBox = kBM * kBoxK / 4;    // 4 KB of packed weights per box
constexpr uint32_t kACols = kBK / 4;           // TMEM columns of one expanded A stage
static_assert(kDCols + kAStages * kACols == kTmemCols, "tensor memory budget");

// Shapes that depend on the token tile BN (MMA N): 128 for prefill, 32 for
// small batches (M <= 32), where a 128-token tile would be mostly padding.
template <int BN>
struct TileCfg {
    static_assert(BN == 32 || BN == 128, "token tile");
    static constexpr int kEpiSplit = BN >= 64 ? 2 : 1;      // epilogue warps per TMEM lane quarter
    static constexpr int kEpiCols = BN / kEpiSplit;         // token columns one epilogue warp drains
    static constexpr int kThreads = 32 * (kEpiWarp0 + 4 * kEpiSplit);
    static constexpr uint32_t kQBox = uint32_t(BN) * kBoxK; // int8 activations per box
    // Instruction descriptor: D int32, A unsigned 8-bit (stored codes), B
    // signed 8-bit (activations), both K-major, M = 128, N = BN.
    static constexpr uint32_t kIdesc = (2u << 4) | (0u << 7) | (1u << 10) | (uint32_t(BN >> 3) << 17) |
                                       (uint32_t(kBM >> 4) << 24);
    static_assert(2 * BN <= int(kDCols), "two accumulator buffers");
    static_assert(kEpiCols % 32 == 0, "epilogue drains 32-column chunks");
};

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
    // split-K (tm.splits > 1): int32 partial sums and arrival counters, zero
    // on entry and left zero
    int32_t *ws;
    int *counters;
};

// ---------------------------------------------------------------- PTX wrappers

// TMA load issued by lane `who` of a warp that runs in warp-uniform control
// flow, together with that lane's expect-tx arrival on the stage barrier.
__device__ __forceinline__ void tma_load_2d_lane(uint32_t who, uint32_t dst, const CUtensorMap *map, uint32_t bar,
                                                 uint32_t bytes, int32_t c0, int32_t c1)
{
    asm volatile(
        "{\n\t.reg .pred e;\n\t.reg .b32 l;\n\t"
        "mov.u32 l, %%laneid;\n\t"
        "setp.eq.u32 e, l, %0;\n\t"
        "@e mbarrier.arrive.expect_tx.shared::cta.b64 _, [%3], %4;\n\t"
        "@e cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes "
        "[%1], [%2, {%5, %6}], [%3];\n\t}" ::"r"(who),
        "r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(bytes), "r"(c0), "r"(c1)
        : "memory");
}

// ---------------------------------------------------------------- kernel

template <int BN>
struct Smem {
    using C = TileCfg<BN>;
    // activation ring (1024-byte aligned for the 128-byte swizzle)
    unsigned char q[kQStages][kBoxes][C::kQBox];
    unsigned char p[kQStages][kBoxes][kPBox];
    // per epilogue warp: d and row sums of the current tile's 128 tokens
    float ep_d[4 * C::kEpiSplit][C::kEpiCols];
    int32_t ep_r[4 * C::kEpiSplit][C::kEpiCols];
    uint64_t full[kQStages];     // activation and packed boxes landed
    uint64_t empty[kQStages];    // the slot's bytes are no longer needed (MMAs completed)
    uint64_t afull[kAStages];    // A expanded into tensor memory (and its activations landed)
    uint64_t aempty[kAStages];   // MMAs reading the A stage completed
    uint64_t tfull[2];           // accumulator buffer complete
    uint64_t tempty[2];          // accumulator buffer drained
    uint64_t drain;              // teardown after an abort
    uint32_t tmem_base;
    int abort_flag;
};
// One CTA per SM: its 512 tensor-memory columns are the whole SM's, so the
// dynamic shared memory asked for is kept above half of the SM's.
template <int BN>
constexpr uint32_t smem_bytes()
{
    constexpr uint32_t need = uint32_t(sizeof(Smem<BN>)) + 1024;  // + alignment slack
    return need > 120 * 1024 ? need : 120 * 1024;
}
static_assert(smem_bytes<128>() <= 227 * 1024 && smem_bytes<32>() <= 227 * 1024, "shared memory per CTA");

// Work units: output tile t = u / splits, k blocks [kb0, kb1) of split u % splits.
struct TileMap {
    int tiles_m;                 // token tiles
    int num_tiles;
    int bn;                      // tokens per tile
    int splits;                  // k splits per tile (1: the whole K)
    int kb_total;                // k blocks of the whole K
    int num_units;               // num_tiles * splits
    __device__ void unit(int u, int &t, int64_t &n0, int64_t &m0, int &kb0, int &kb1) const
    {
        t = u / splits;
        const int sp = u - t * splits;
        n0 = int64_t(t / tiles_m) * kBM;
        m0 = int64_t(t % tiles_m) * bn;
        kb0 = int(int64_t(sp) * kb_total / splits);
        kb1 = int(int64_t(sp + 1) * kb_total / splits);
    }
};

template <typename T>
__device__ __forceinline__ void store_out(T *y, int64_t idx, float v);
template <>
__device__ __forceinline__ void store_out<__nv_bfloat16>(__nv_bfloat16 *y, int64_t idx, float v)
{
    y[idx] = __float2bfloat16_rn(v);
}
template <>
__device__ __forceinline__ void store_out<float>(float *y, int64_t idx, float v)
{
    y[idx] = v;
}

// One 32-token chunk of the epilogue for this thread's weight row n.
template <typename T, bool FULL, bool DBG>
__device__ __forceinline__ void epilogue_chunk(const uint32_t (&v)[32], const float *sd, const int32_t *sr,
                                               int64_t n, int64_t m0, const GemmParams &p, float gamma)
{
    T *y = static_cast<T *>(p.y) + m0 * p.ldy + n;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        if (FULL || m0 + j < p.M) {
            const int a = int(v[j]) - sr[j];
            if (DBG)
                p.acc_dbg[(m0 + j) * p.N + n] = a;
            store_out<T>(y, int64_t(j) * p.ldy, rescale1(a, sd[j], gamma));
        }
    }
}

template <typename T, bool DBG>
__device__ __forceinline__ void epilogue_chunk_any(const uint32_t (&v)[32], const float *sd, const int32_t *sr,
                                                   int64_t n, int64_t m0, const GemmParams &p, float gamma)
{
    if (m0 + 32 <= p.M)
        epilogue_chunk<T, true, DBG>(v, sd, sr, n, m0, p, gamma);
    else
        epilogue_chunk<T, false, DBG>(v, sd, sr, n, m0, p, gamma);
}

template <int BN>
__global__ void __launch_bounds__(TileCfg<BN>::kThreads, 1)
gemm_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap pmap,
            const GemmParams p, const TileMap tm)
{
    using C = TileCfg<BN>;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    Smem<BN> &sm = *reinterpret_cast<Smem<BN> *>(smem_raw + (((raw + 1023u) & ~1023u) - raw));
    volatile int *abort_flag = &sm.abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kQStages; ++s) {
            mbar_init(smem_u32(&sm.full[s]), 2 * kBoxes);
            mbar_init(smem_u32(&sm.empty[s]), 1);
        }
        for (int a = 0; a < kAStages; ++a) {
            mbar_init(smem_u32(&sm.afull[a]), 128);
            mbar_init(smem_u32(&sm.aempty[a]), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&sm.tfull[b]), 1);
            mbar_init(smem_u32(&sm.tempty[b]), 128 * C::kEpiSplit);
        }
        mbar_init(smem_u32(&sm.drain), 1);
        sm.abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&qmap)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&pmap)) : "memory");
    }
    if (warp == kMmaWarp)
        tmem_alloc(smem_u32(&sm.tmem_base), kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    const uint32_t a_tmem0 = tmem + kDCols;     // columns [256, 512): kAStages x 64

    if (warp < kProducerWarps) {
        // ------------------------------------------------ TMA producers
        // lanes 0..kBoxes-1 copy the activation boxes of a stage, the next
        // kBoxes lanes its packed weight boxes; the warp waits as a whole
        int last = -1;   // global stage index of this warp's last issued stage
        int base = 0;    // global stage index of the current unit's first k block
        bool ok = true;
        for (int u = blockIdx.x; u < tm.num_units && ok; u += gridDim.x) {
            int t, kb0, kb1;
            int64_t n0, m0;
            tm.unit(u, t, n0, m0, kb0, kb1);
            const int nk = kb1 - kb0;
            for (int i = ((warp - base) % kProducerWarps + kProducerWarps) % kProducerWarps; i < nk;
                 i += kProducerWarps) {
                const int g = base + i, kb = kb0 + i;
                const int s = g % kQStages;
                const uint32_t full = smem_u32(&sm.full[s]);
                if (!__all_sync(0xffffffffu, mbar_wait_fast(smem_u32(&sm.empty[s]), (uint32_t(g / kQStages) & 1u) ^ 1u,
                                                            abort_flag, p.status))) {
                    ok = false;
                    break;
                }
#pragma unroll
                for (int box = 0; box < kBoxes; ++box) {
                    const int k0 = kb * kBK + box * kBoxK;
                    tma_load_2d_lane(box, smem_u32(sm.q[s][box]), &qmap, full, C::kQBox, k0, int32_t(m0));
                    tma_load_2d_lane(kBoxes + box, smem_u32(sm.p[s][box]), &pmap, full, kPBox, k0 * 2,
                                     int32_t(n0 / 8));
                }
                last = g;
            }
            base += nk;
        }
        if (last >= 0) {
            // the last stage's copies have landed before the CTA exits (at
            // once unless another role gave up before consuming them)
            volatile int no_abort = 0;
            mbar_wait(smem_u32(&sm.full[last % kQStages]), uint32_t(last / kQStages) & 1u, &no_abort, p.status,
                      100000000ull);
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------ MMA issuer (whole warp, lane 0 issues)
        const uint64_t q_desc0 = smem_desc_sw128(smem_u32(sm.q[0][0]));   // slot s adds its offset >> 4
        int g = 0, it = 0;
        bool ok = true, issued_any = false;
        for (int u = blockIdx.x; u < tm.num_units && ok; u += gridDim.x, ++it) {
            int t, kb0, kb1;
            int64_t n0, m0;
            tm.unit(u, t, n0, m0, kb0, kb1);
            const int b = it & 1;
            if (it >= 2 &&
                !__all_sync(0xffffffffu, mbar_wait_fast(smem_u32(&sm.tempty[b]), (uint32_t(it >> 1) & 1u) ^ 1u,
                                                        abort_flag, p.status))) {
                ok = false;
                break;
            }
            const uint32_t d_tmem = tmem + uint32_t(b * BN);
            for (int kb = kb0; kb < kb1; ++kb, ++g) {
                const int s = g % kQStages, a = g % kAStages;
                // the tensor core reads the activation tile through the async
                // proxy: wait on the barrier its TMA completes, not only on the
                // expansion barrier that follows it
                if (!__all_sync(0xffffffffu, mbar_wait_fast(smem_u32(&sm.afull[a]), uint32_t(g / kAStages) & 1u,
                                                            abort_flag, p.status) &&
                                                 mbar_wait_fast(smem_u32(&sm.full[s]), uint32_t(g / kQStages) & 1u,
                                                                abort_flag, p.status))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                mma_stage8<(C::kQBox >> 4)>(d_tmem, a_tmem0 + a * kACols,
                                            q_desc0 + uint64_t(s) * (kBoxes * C::kQBox >> 4), C::kIdesc,
                           kb > kb0 ? 1u : 0u);
                mma_commit(smem_u32(&sm.empty[s]));
                mma_commit(smem_u32(&sm.aempty[a]));
                issued_any = true;
            }
            if (ok)
                mma_commit(smem_u32(&sm.tfull[b]));
        }
        if (issued_any) {
            // every MMA has completed before tensor memory is released (at
            // once unless the epilogue gave up before draining them)
            mma_commit(smem_u32(&sm.drain));
            volatile int no_abort = 0;
            mbar_wait(smem_u32(&sm.drain), 0, &no_abort, p.status, 100000000ull);
        }
    } else if (warp < kEpiWarp0) {
        // ------------------------------------------------ expansion into tensor memory
        const int grp = (warp - kExpWarp0) / 4;       // takes the stages g = grp (mod 2)
        const int quarter = warp & 3;                 // TMEM lanes 32*quarter .. +31
        const int rl = quarter * 32 + lane;           // weight row within the tile
        const uint32_t lane_addr = uint32_t(quarter * 32) << 16;
        int g = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < tm.num_units && ok; u += gridDim.x) {
            int t, kb0, kb1;
            int64_t n0, m0;
            tm.unit(u, t, n0, m0, kb0, kb1);
            for (int kb = kb0; kb < kb1; ++kb, ++g) {
                if ((g & 1) != grp)
                    continue;
                const int s = g % kQStages, a = g % kAStages;
                // warp-uniform outcomes: the tcgen05.st below is .sync.aligned
                if (!__all_sync(0xffffffffu, mbar_wait_fast(smem_u32(&sm.full[s]), uint32_t(g / kQStages) & 1u,
                                                            abort_flag, p.status))) {
                    ok = false;
                    break;
                }
                uint4 c4[2 * kBoxes];
#pragma unroll
                for (int box = 0; box < kBoxes; ++box) {
                    const unsigned char *ps = sm.p[s][box] + (rl >> 3) * 256 + (rl & 7) * 16;
                    c4[2 * box] = *reinterpret_cast<const uint4 *>(ps);
                    c4[2 * box + 1] = *reinterpret_cast<const uint4 *>(ps + 128);
                }
                if (!__all_sync(0xffffffffu, mbar_wait_fast(smem_u32(&sm.aempty[a]), (uint32_t(g / kAStages) & 1u) ^ 1u,
                                                            abort_flag, p.status))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                uint32_t v[64];
#pragma unroll
                for (int c = 0; c < 2 * kBoxes; ++c) {
                    const uint32_t wd[4] = {c4[c].x, c4[c].y, c4[c].z, c4[c].w};
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        v[16 * c + 4 * w + 0] = wd[w] & 0x03030303u;
                        v[16 * c + 4 * w + 1] = (wd[w] >> 2) & 0x03030303u;
                        v[16 * c + 4 * w + 2] = (wd[w] >> 4) & 0x03030303u;
                        v[16 * c + 4 * w + 3] = (wd[w] >> 6) & 0x03030303u;
                    }
                }
                tmem_st64_wait(a_tmem0 + lane_addr + a * kACols, v);
                tc_fence_before();
                mbar_arrive(smem_u32(&sm.afull[a]));
            }
        }
    } else {
        // ------------------------------------------------ epilogue
        const int ew = warp - kEpiWarp0;              // this warp's staging slice
        const int quarter = warp & 3;                 // TMEM lanes 32*quarter .. +31
        const int c0 = (ew / 4) * C::kEpiCols;        // first token column this warp drains
        const int rl = quarter * 32 + lane;
        const uint32_t lane_addr = uint32_t(quarter * 32) << 16;
        const float gamma = p.w_scale[0];
        float *sd = sm.ep_d[ew];
        int32_t *sr = sm.ep_r[ew];
        int it = 0;
        for (int u = blockIdx.x; u < tm.num_units; u += gridDim.x, ++it) {
            const int b = it & 1;
            int t, kb0, kb1;
            int64_t n0, m0;
            tm.unit(u, t, n0, m0, kb0, kb1);
            __syncwarp();
#pragma unroll
            for (int c = 0; c < C::kEpiCols / 32; ++c) {
                const int64_t m = m0 + c0 + c * 32 + lane;
                sd[c * 32 + lane] = m < p.M ? __ldg(p.d + m) : 0.0f;
                sr[c * 32 + lane] = m < p.M ? __ldg(p.rowsum + m) : 0;
            }
            __syncwarp();
            if (!__all_sync(0xffffffffu,
                            mbar_wait_fast(smem_u32(&sm.tfull[b]), uint32_t(it >> 1) & 1u, abort_flag, p.status)))
                break;
            tc_fence_after();
            const int64_t n = n0 + rl;
            auto finish = [&](const uint32_t (&v)[32], int c) {
                if (n < p.N) {
                    const int64_t mc = m0 + c0 + c * 32;
                    const float *d32 = sd + c * 32;
                    const int32_t *r32 = sr + c * 32;
                    if (p.yt == BL_BF16) {
                        if (p.acc_dbg)
                            epilogue_chunk_any<__nv_bfloat16, true>(v, d32, r32, n, mc, p, gamma);
                        else
                            epilogue_chunk_any<__nv_bfloat16, false>(v, d32, r32, n, mc, p, gamma);
                    } else {
                        if (p.acc_dbg)
                            epilogue_chunk_any<float, true>(v, d32, r32, n, mc, p, gamma);
                        else
                            epilogue_chunk_any<float, false>(v, d32, r32, n, mc, p, gamma);
                    }
                }
            };
            if (tm.splits == 1) {
#pragma unroll 1
                for (int c = 0; c < C::kEpiCols / 32; ++c) {
                    uint32_t v[32];
                    tmem_ld32_wait(tmem + lane_addr + uint32_t(b * BN + c0 + c * 32), v);
                    finish(v, c);
                }
                tc_fence_before();
                mbar_arrive(smem_u32(&sm.tempty[b]));
            } else {
                // split-K: add this warp's partial sums (32 weight rows x its
                // token columns) into the workspace, laid out [tile][token][row]
                // so that a warp's adds for one token cover 128 contiguous bytes
                int32_t *wsw = p.ws + (int64_t(t) * BN + c0) * kBM + rl;
#pragma unroll 1
                for (int c = 0; c < C::kEpiCols / 32; ++c) {
                    uint32_t v[32];
                    tmem_ld32_wait(tmem + lane_addr + uint32_t(b * BN + c0 + c * 32), v);
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        atomicAdd(wsw + int64_t(c * 32 + j) * kBM, int(v[j]));
                }
                tc_fence_before();
                mbar_arrive(smem_u32(&sm.tempty[b]));
                // the warp of the last split to arrive finishes the tile's block
                __threadfence();
                __syncwarp();
                int *cnt = p.counters + int64_t(t) * (4 * C::kEpiSplit) + ew;
                int old = 0;
                if (lane == 0)
                    old = atomicAdd(cnt, 1);
                old = __shfl_sync(0xffffffffu, old, 0);
                if (old == tm.splits - 1) {
                    __threadfence();
#pragma unroll 1
                    for (int c = 0; c < C::kEpiCols / 32; ++c) {
                        uint32_t v[32];
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            int32_t *w = wsw + int64_t(c * 32 + j) * kBM;
                            v[j] = uint32_t(__ldcg(w));
                            __stcg(w, 0);   // left zero for the next call
                        }
                        finish(v, c);
                    }
                    if (lane == 0)
                        *cnt = 0;
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
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

namespace {

// Split-K plan: only small batches (32-token tiles) split K, and only while
// their output tiles alone would leave SMs idle.  Workspace: int32 partial
// sums [tile][32 tokens][128 rows], then one arrival counter per tile and
// epilogue warp.
struct SplitPlan {
    int splits = 1;
    size_t counters_offset = 0;
    size_t bytes = 0;
};

SplitPlan split_plan(int64_t M, int64_t N, int64_t K, int sms)
{
    SplitPlan sp;
    if (M > 32)
        return sp;
    const int64_t tiles = ((M + 31) / 32) * ((N + kBM - 1) / kBM);
    const int64_t kb = (K + kBK - 1) / kBK;
    if (tiles >= sms || kb < 2)
        return sp;
    // all units in one wave: a CTA that takes two units doubles the latency
    const int64_t splits = std::min<int64_t>(sms / tiles, kb);
    if (splits < 2)
        return sp;
    sp.splits = int(splits);
    sp.counters_offset = size_t(tiles) * 32 * kBM * sizeof(int32_t);
    sp.bytes = sp.counters_offset + size_t(tiles) * 4 * TileCfg<32>::kEpiSplit * sizeof(int);
    return sp;
}

}  // namespace

size_t gemm_workspace_bytes(int64_t M, int64_t N, int64_t K)
{
    const DeviceInfo *di = device_info();
    return di ? split_plan(M, N, K, di->sm_count).bytes : 0;
}

namespace {

template <int BN>
int launch_tiles(const GemvArgs &a, const DeviceInfo *di, const SplitPlan &sp, void *ws, cudaStream_t s)
{
    using C = TileCfg<BN>;
    CUtensorMap qmap, pmap;
    // activations: [M][K] int8, boxes of 128 k x BN tokens, 128-byte swizzle
    int st = make_map_2d(&qmap, a.q, uint64_t(a.K), uint64_t(a.M), uint64_t(a.K), kBoxK, BN, true);
    if (st)
        return st;
    // packed weights as [row groups][K/64 * 128 B]: boxes of 16 groups x 256 B (128 k)
    const uint64_t rg_bytes = uint64_t(a.K / 64) * 128;
    st = make_map_2d(&pmap, a.packed, rg_bytes, uint64_t((a.N + 7) / 8), rg_bytes, 2 * kBoxK,
                     kBM / 8, false);
    if (st)
        return st;
    int per_sm = 0;
    if ((st = occupancy(reinterpret_cast<const void *>(gemm_kernel<BN>), C::kThreads, smem_bytes<BN>(), &per_sm)))
        return st;
    if (per_sm < 1)
        return BL_ERR_UNSUPPORTED;
    GemmParams p{a.w_scale, a.d, a.rowsum, a.M, a.N, a.K, a.y, a.yt, a.ldy, a.acc_dbg, di->status,
                 static_cast<int32_t *>(ws),
                 ws ? reinterpret_cast<int *>(static_cast<char *>(ws) + sp.counters_offset) : nullptr};
    TileMap tm;
    tm.tiles_m = int((a.M + BN - 1) / BN);
    tm.bn = BN;
    const int64_t tiles = int64_t(tm.tiles_m) * ((a.N + kBM - 1) / kBM);
    if (tiles * sp.splits > (int64_t(1) << 30))
        return BL_ERR_SHAPE;
    tm.num_tiles = int(tiles);
    tm.splits = ws ? sp.splits : 1;
    tm.kb_total = int((a.K + kBK - 1) / kBK);
    tm.num_units = tm.num_tiles * tm.splits;
    const int grid = int(std::min<int64_t>(tm.num_units, di->sm_count));
    gemm_kernel<BN><<<grid, C::kThreads, smem_bytes<BN>(), s>>>(qmap, pmap, p, tm);
    return launch_status();
}

}  // namespace

int launch_gemm(const GemvArgs &a, void *ws, size_t ws_bytes, cudaStream_t s)
{
    const DeviceInfo *di = device_info();
    if (!di)
        return BL_ERR_CUDA;
    if (a.M > (int64_t(1) << 30) || a.N > (int64_t(1) << 30))
        return BL_ERR_SHAPE;
    // split K only with the workspace it needs (callers without one, such as
    // bitlinear_gemv's small batches, run unsplit)
    const SplitPlan sp = split_plan(a.M, a.N, a.K, di->sm_count);
    void *w = sp.splits > 1 && ws && ws_bytes >= sp.bytes ? ws : nullptr;
    // small batches: 32-token tiles (a 128-token tile would be mostly padding)
    return a.M <= 32 ? launch_tiles<32>(a, di, sp, w, s) : launch_tiles<128>(a, di, sp, nullptr, s);
}

}  // namespace bl
