// gemv_stream_mt.cu -- ternary decode GEMV for a small batch of tokens
// (2 .. 16), streaming the packed weights once for all of them.
//
// "How to Run BitNet Inference on GPU Using CUDA Kernels: A Complete Guide",
// section "Understanding the Two-Phase Architecture": decode is a
// memory-bound INT8-activation x INT2-weight product; with a few tokens per
// step the weight stream is still the whole cost, so every token must use the
// same pass over the weights.
//
// Design (the one-token streaming kernel's ring, generalised to M tokens):
//   * A producer warp fills a four-stage shared-memory ring with bulk copies
//     of the CTA's row groups (at most four groups per stage), exactly as in
//     gemv_stream.cu; eight consumer warps take piece w (and w + 8) of every
//     group of a stage.
//   * The prologue quantises the M tokens into int8 rows in shared memory
//     (or copies pre-quantised q): one warp per token, the whole row loaded
//     into registers at once (raw 16-byte vectors; rows above 4096 bf16
//     elements in two halves), a warp reduction for its absmax (K <= 8192;
//     fp32 input K <= 4096).
//   * Per stage a consumer lane expands each group's 16-byte piece once into
//     sixteen code words c = (word >> 2i) & 0x03030303 (stored codes s =
//     code + 1 of four consecutive k), then, token by token, loads the
//     token's 64 activation bytes and accumulates sixteen dp4a per group into
//     one accumulator per (group, token): the shifts and masks are paid once
//     per weight word, not once per token.  sum(code q) = sum(s q) - rowsum.
//   * At the end of a set each (group, token) accumulator is reduced over the
//     four lanes of its row and added into the CTA's row sums in shared
//     memory; the epilogue rescales every (token, row).
//   * Every mbarrier wait is bounded; on expiry the CTA records
//     BL_ERR_TIMEOUT, the consumers stop and the producer waits (bounded) for
//     its copies in flight before the CTA exits.
#include "gemv_stream_common.cuh"

namespace bl {
namespace {

constexpr int kMtKC = 8;                         // consumer warps
constexpr int kMtThreads = 32 * (kMtKC + 1);
constexpr int kMtMaxTokens = 16;
constexpr int kMtMaxSet = 4;                     // groups per stage
constexpr int kMtMaxGroupsPerCta = 32;
constexpr int64_t kMtMaxK = 8192;                // a token's row in one warp's registers

enum { MT_Q = 0, MT_X_BF16 = 1, MT_X_F32 = 2 };

struct MtParams {
    GemvProblem prob[kGemvMaxProblems];
    int64_t gstart[kGemvMaxProblems + 1];
    int count;
    int64_t K;
    int M;
    const int8_t *q;          // [M][K] (MT_Q)
    const float *d;
    const int32_t *rowsum;
    const void *x;            // [M][ldx] (MT_X_*)
    int64_t ldx;
    int yt;
    int64_t gpc_base;
    int gpc_rem;
    int set_cap;
    int *status;
};

struct MtSmem {
    uint64_t full[kStages];
    uint64_t empty[kStages];
    int abort_flag;
    int bsum[kMtMaxTokens][1];     // each token's row sum
    float d[kMtMaxTokens];
    float wscale[kGemvMaxProblems];
    int sacc[kMtMaxTokens][kMtMaxGroupsPerCta][8];
};

constexpr size_t kMtHeader = (sizeof(MtSmem) + 127) / 128 * 128;

__device__ __forceinline__ int mt_locate(const MtParams &p, int64_t G)
{
    int pi = 0;
#pragma unroll
    for (int i = 1; i < kGemvMaxProblems; ++i)
        if (i < p.count && G >= p.gstart[i])
            pi = i;
    return pi;
}

__device__ __forceinline__ void mt_sync() { named_barrier(1, 32 * kMtKC); }

// Quantise the M tokens into qs [M][K]: warp w takes tokens w, w + 8, ...,
// each a whole row: the row's 16-byte chunks are all loaded before any is
// used (CHM per lane, so one round trip to L2 per token), the absmax is a
// warp reduction, and the warp quantises from its registers.  Other warps
// read these activations after the block barrier that follows.
template <int XT, int CHM>
struct MtRow {
    static constexpr int V = XT == BL_BF16 ? 1 : 2;   // 16-byte vectors per chunk of 8 elements
    uint4 raw[CHM * V];

    // chunks lane + 32 (i0 + i), i < CHM, of token m's row
    __device__ __forceinline__ void load(const MtParams &p, int m, int i0, int lane, int chunks)
    {
#pragma unroll
        for (int i = 0; i < CHM; ++i) {
            const int c = lane + 32 * (i0 + i);
#pragma unroll
            for (int v = 0; v < V; ++v)
                raw[V * i + v] = c < chunks
                    ? ld_dep_v4(static_cast<const unsigned char *>(p.x) +
                                (int64_t(m) * p.ldx + int64_t(c) * 8) * (XT == BL_BF16 ? 2 : 4) + 16 * v)
                    : make_uint4(0, 0, 0, 0);
        }
    }
    __device__ __forceinline__ void f32(int i, float (&f)[8]) const
    {
        if constexpr (XT == BL_BF16) {
            bf16x8_f32(raw[i], f);
        } else {
            const uint4 a = raw[2 * i], b = raw[2 * i + 1];
            f[0] = __uint_as_float(a.x); f[1] = __uint_as_float(a.y);
            f[2] = __uint_as_float(a.z); f[3] = __uint_as_float(a.w);
            f[4] = __uint_as_float(b.x); f[5] = __uint_as_float(b.y);
            f[6] = __uint_as_float(b.z); f[7] = __uint_as_float(b.w);
        }
    }
    __device__ __forceinline__ float amax() const
    {
        float a = 0.0f;
#pragma unroll
        for (int i = 0; i < CHM; ++i) {
            float f[8];
            f32(i, f);
#pragma unroll
            for (int e = 0; e < 8; ++e)
                a = fmaxf(a, fabsf(f[e]));
        }
        return a;
    }
    __device__ __forceinline__ void quantise(int8_t *qrow, int i0, int lane, int chunks, float s, int &sum) const
    {
#pragma unroll
        for (int i = 0; i < CHM; ++i) {
            const int c = lane + 32 * (i0 + i);
            if (c < chunks) {
                float f[8];
                f32(i, f);
                *reinterpret_cast<uint2 *>(qrow + int64_t(c) * 8) = quant8(f, s, sum);
            }
        }
    }
};

// Quantise the M tokens into qs [M][K]: warp w takes tokens w, w + 8, ...,
// each a whole row: CHM 16-byte chunks per lane loaded before any is used
// (one round trip to L2 per token), the absmax a warp reduction, the
// quantisation from the registers.  HALVES = 2 (rows longer than 16 chunks
// per lane): the two halves in turn -- load the first, load the second
// (absmax of both), quantise the second, load the first again and quantise
// it -- so that only half a row is live.  Other warps read these activations
// after the block barrier at the end.
template <int XT, int CHM, int HALVES>
__device__ __forceinline__ void mt_quantize(const MtParams &p, MtSmem &sm, int8_t *qs)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int chunks = int(p.K / 8);
    for (int m = warp; m < p.M; m += kMtKC) {
        int8_t *qrow = qs + int64_t(m) * p.K;
        MtRow<XT, CHM> row;
        float a;
        if constexpr (HALVES == 1) {
            row.load(p, m, 0, lane, chunks);
            a = row.amax();
        } else {
            row.load(p, m, 0, lane, chunks);
            a = row.amax();
            row.load(p, m, CHM, lane, chunks);
            a = fmaxf(a, row.amax());
        }
        // maxima are >= 0 and finite: bit patterns order like the values
        a = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(a)));
        const float a_eff = fmaxf(a, kEps);
        const float s = __fdiv_rn(kQb, a_eff);
        int sum = 0;
        if constexpr (HALVES == 1) {
            row.quantise(qrow, 0, lane, chunks, s, sum);
        } else {
            row.quantise(qrow, CHM, lane, chunks, s, sum);
            row.load(p, m, 0, lane, chunks);
            row.quantise(qrow, 0, lane, chunks, s, sum);
        }
        sum = __reduce_add_sync(0xffffffffu, sum);
        if (lane == 0) {
            sm.bsum[m][0] = sum;
            sm.d[m] = __fdiv_rn(a_eff, kQb);
        }
    }
    mt_sync();
}

__device__ __forceinline__ void mt_copy_q(const MtParams &p, MtSmem &sm, int8_t *qs)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int P = int(p.K / 256);
    for (int m = 0; m < p.M; ++m) {
        for (int j = warp; j < P; j += kMtKC)
            if (lane < 16)
                *reinterpret_cast<uint4 *>(qs + int64_t(m) * p.K + j * 256 + lane * 16) =
                    ld_dep_v4(p.q + int64_t(m) * p.K + int64_t(j) * 256 + lane * 16);
        if (lane == 0 && warp == 0) {
            sm.bsum[m][0] = int(ld_dep_u32(p.rowsum + m));
            sm.d[m] = __uint_as_float(ld_dep_u32(p.d + m));
        }
    }
    __syncwarp();
}

// One piece of RG groups (their 16-byte pieces RG slots apart from `base`)
// against MT tokens' activations (token m at qbase + m * K).
template <int RG, int MT>
__device__ __forceinline__ void mt_piece(uint32_t base, uint32_t slot, uint32_t qbase, uint32_t K, int M,
                                         int (&acc)[kMtMaxSet][MT])
{
    uint32_t c[RG][16];
#pragma unroll
    for (int r = 0; r < RG; ++r) {
        const uint4 wv = lds128(base + r * slot);
        const uint32_t wd[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
        for (int w = 0; w < 4; ++w)
#pragma unroll
            for (int i = 0; i < 4; ++i)
                c[r][4 * w + i] = (wd[w] >> (2 * i)) & 0x03030303u;
    }
#pragma unroll
    for (int m = 0; m < MT; ++m) {
        if (m < M) {
            uint4 q[4];
#pragma unroll
            for (int j = 0; j < 4; ++j)
                q[j] = lds128(qbase + m * K + 16 * j);
#pragma unroll
            for (int r = 0; r < RG; ++r)
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    acc[r][m] = dp4a_us(c[r][4 * w + 0], q[w].x, acc[r][m]);
                    acc[r][m] = dp4a_us(c[r][4 * w + 1], q[w].y, acc[r][m]);
                    acc[r][m] = dp4a_us(c[r][4 * w + 2], q[w].z, acc[r][m]);
                    acc[r][m] = dp4a_us(c[r][4 * w + 3], q[w].w, acc[r][m]);
                }
        }
    }
}

template <int MT>
__device__ __forceinline__ void mt_piece_n(int rg, uint32_t base, uint32_t slot, uint32_t qbase, uint32_t K, int M,
                                           int (&acc)[kMtMaxSet][MT])
{
    switch (rg) {
    case 1: mt_piece<1, MT>(base, slot, qbase, K, M, acc); break;
    case 2: mt_piece<2, MT>(base, slot, qbase, K, M, acc); break;
    case 3: mt_piece<3, MT>(base, slot, qbase, K, M, acc); break;
    default: mt_piece<4, MT>(base, slot, qbase, K, M, acc); break;
    }
}
static_assert(kMtMaxSet == 4, "mt_piece_n covers 1..4 groups");

// End of a set: each (group, token) sum over the four lanes of its row, into
// the CTA's row sums.
template <int MT>
__device__ __forceinline__ void mt_flush(int rg, int M, int (&acc)[kMtMaxSet][MT], MtSmem &sm, int g0, int lane)
{
#pragma unroll
    for (int r = 0; r < kMtMaxSet; ++r) {
        if (r < rg) {
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                if (m < M) {
                    int v = acc[r][m];
                    v += __shfl_xor_sync(0xffffffffu, v, 8);
                    v += __shfl_xor_sync(0xffffffffu, v, 16);
                    if (lane < 8)
                        atomicAdd(&sm.sacc[m][g0 + r][lane], v);
                }
                acc[r][m] = 0;
            }
        }
    }
}

template <int MT, int MODE, int CHM>
__global__ void __launch_bounds__(kMtThreads, 1) gemv_stream_mt_kernel(const MtParams p)
{
    extern __shared__ __align__(128) unsigned char smem_raw[];
    MtSmem &sm = *reinterpret_cast<MtSmem *>(smem_raw);
    const uint32_t ring = smem_u32(smem_raw + kMtHeader);
    const int R = p.set_cap;
    const int P = int(p.K / 256);
    const int PS = stage_pieces(P, kMtKC);
    const uint32_t slot = uint32_t(PS) * 512;
    const uint32_t stage_bytes = uint32_t(R) * slot;
    int8_t *qs = reinterpret_cast<int8_t *>(smem_raw + kMtHeader + size_t(kStages) * stage_bytes);
    volatile int *abort_flag = &sm.abort_flag;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bx = blockIdx.x;
    const int64_t g_begin = bx * p.gpc_base + (bx < p.gpc_rem ? bx : p.gpc_rem);
    const int ng = int(p.gpc_base) + (bx < p.gpc_rem ? 1 : 0);
    const int subs = (P + PS - 1) / PS;
    const int64_t slab = 2 * p.K;
    const SetSplit split(ng, R);

    if (tid == 0) {
        for (int b = 0; b < kStages; ++b) {
            mbar_init(smem_u32(&sm.full[b]), 1);
            mbar_init(smem_u32(&sm.empty[b]), kMtKC);
        }
        sm.abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    for (int i = tid; i < kMtMaxTokens * kMtMaxGroupsPerCta * 8; i += kMtThreads)
        (&sm.sacc[0][0][0])[i] = 0;
    __syncthreads();
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    if (warp == kMtKC) {
        // ------------------------------------------------ producer warp
        int t = 0, sb = 0, g0 = 0;
        uint32_t ph = 0;
        bool ok = true;
        for (int i = 0; i < split.nsets && ok; ++i) {
            const int rg = split.size(i);
            const uint8_t *src = nullptr;
            if (lane < rg) {
                const int64_t G = g_begin + g0 + lane;
                const int pi = mt_locate(p, G);
                src = p.prob[pi].packed + (G - p.gstart[pi]) * slab;
            }
            for (int kb = 0; kb < subs; ++kb) {
                const int np = min(PS, P - kb * PS);
                const uint32_t bytes = uint32_t(np) * 512;
                if (!__all_sync(0xffffffffu, mbar_wait_fast(smem_u32(&sm.empty[sb]), ph ^ 1u, abort_flag, p.status))) {
                    ok = false;
                    break;
                }
                const uint32_t full = smem_u32(&sm.full[sb]);
                if (lane == 0)
                    mbar_arrive_tx(full, uint32_t(rg) * bytes);
                __syncwarp();
                const int r = (lane - t * kMtMaxSet) & 31;
                const uint8_t *src_r = reinterpret_cast<const uint8_t *>(
                    __shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(src), r & 31));
                if (r < rg)
                    bulk_load(ring + uint32_t(sb) * stage_bytes + uint32_t(r) * slot, src_r + int64_t(kb) * slot,
                              bytes, full);
                ++t;
                if (++sb == kStages) {
                    sb = 0;
                    ph ^= 1u;
                }
            }
            g0 += rg;
        }
        volatile int no_abort = 0;
        for (int u = t - kStages > 0 ? t - kStages : 0; u < t; ++u)
            mbar_wait(smem_u32(&sm.full[u % kStages]), uint32_t(u / kStages) & 1u, &no_abort, p.status,
                      100000000ull);
        return;
    }

    // ---------------------------------------------------- consumer warps
    if (tid < p.count)
        sm.wscale[tid] = __ldg(p.prob[tid].w_scale);
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if constexpr (MODE == MT_Q)
        mt_copy_q(p, sm, qs);
    else
        mt_quantize<MODE == MT_X_BF16 ? BL_BF16 : BL_F32, (CHM > 16 ? 16 : CHM), (CHM > 16 ? 2 : 1)>(p, sm, qs);
    // (pre-quantised: each warp reads only the activations it copied itself;
    // quantised here: the barrier at the end of mt_quantize)

    const uint32_t ring_lane = ring + uint32_t(warp) * 512 + uint32_t(lane) * 16;
    const uint32_t q_lane = smem_u32(qs) + uint32_t(warp) * 256 + uint32_t(lane >> 3) * 64;
    const uint32_t K32 = uint32_t(p.K);
    int acc[kMtMaxSet][MT];
#pragma unroll
    for (int r = 0; r < kMtMaxSet; ++r)
#pragma unroll
        for (int m = 0; m < MT; ++m)
            acc[r][m] = 0;
    int sb = 0, g0 = 0;
    uint32_t ph = 0;
    bool ok = true;
    for (int i = 0; i < split.nsets && ok; ++i) {
        const int rg = split.size(i);
        for (int kb = 0; kb < subs; ++kb) {
            if (!__all_sync(0xffffffffu, mbar_wait_fast(smem_u32(&sm.full[sb]), ph, abort_flag, p.status))) {
                ok = false;
                break;
            }
            const int np = min(PS, P - kb * PS);
            const uint32_t stage = ring_lane + uint32_t(sb) * stage_bytes;
            if (PS == kMtKC) {
                if (warp < np)
                    mt_piece_n<MT>(rg, stage, slot, q_lane + uint32_t(kb * kMtKC) * 256, K32, p.M, acc);
            } else {
#pragma unroll
                for (int m2 = 0; m2 < 2; ++m2)
                    if (warp + m2 * kMtKC < np)
                        mt_piece_n<MT>(rg, stage + uint32_t(m2 * kMtKC) * 512, slot,
                                       q_lane + uint32_t(m2 * kMtKC) * 256, K32, p.M, acc);
            }
            __syncwarp();
            if (lane == 0)
                mbar_arrive(smem_u32(&sm.empty[sb]));
            if (++sb == kStages) {
                sb = 0;
                ph ^= 1u;
            }
        }
        mt_flush<MT>(rg, p.M, acc, sm, g0, lane);
        g0 += rg;
    }
    mt_sync();
    // rescale and write every (token, row) of this CTA
    const int rows = ng * 8;
    for (int idx = tid; idx < rows * p.M; idx += 32 * kMtKC) {
        const int m = idx / rows, rr = idx - m * rows;
        const int64_t Gr = g_begin + (rr >> 3);
        const int pi = mt_locate(p, Gr);
        const GemvProblem &pr = p.prob[pi];
        const int64_t row = (Gr - p.gstart[pi]) * 8 + (rr & 7);
        if (row < pr.N) {
            const int a = sm.sacc[m][rr >> 3][rr & 7] - sm.bsum[m][0];
            if (pr.acc_dbg)
                pr.acc_dbg[int64_t(m) * pr.N + row] = a;
            store_y(pr.y, p.yt, int64_t(m) * pr.ldy + row, rescale1(a, sm.d[m], sm.wscale[pi]));
        }
    }
}

size_t mt_smem(int64_t K, int M, int R)
{
    const int P = int(K / 256);
    const size_t slot = size_t(stage_pieces(P, kMtKC)) * 512;
    return kMtHeader + size_t(kStages) * R * slot + size_t(M) * K;
}

template <int MT, int MODE, int CHM>
int launch_mt_t(const MtParams &base, cudaStream_t s, unsigned flags)
{
    const DeviceInfo *di = device_info();
    if (!di)
        return BL_ERR_CUDA;
    const int64_t ng_total = base.gstart[base.count];
    const int64_t grid = ng_total < di->sm_count ? ng_total : di->sm_count;
    // R: the smallest set capacity (2 .. 4) that gives every CTA the same
    // number of sets and fits in shared memory
    const int64_t lo = ng_total / grid, hi = lo + (ng_total % grid ? 1 : 0);
    int R = 0;
    for (int c = 2; c <= kMtMaxSet && !R; ++c)
        if (mt_smem(base.K, base.M, c) <= size_t(di->max_smem_optin) && (lo + c - 1) / c == (hi + c - 1) / c)
            R = c;
    if (!R)
        R = mt_smem(base.K, base.M, kMtMaxSet) <= size_t(di->max_smem_optin) ? kMtMaxSet : 2;
    const size_t smem = mt_smem(base.K, base.M, R);
    auto kern = gemv_stream_mt_kernel<MT, MODE, CHM>;
    int per_sm = 0;
    int st = occupancy(reinterpret_cast<const void *>(kern), kMtThreads, smem, &per_sm);
    if (st)
        return st;
    if (per_sm < 1)
        return BL_ERR_SHAPE;
    MtParams p = base;
    p.gpc_base = ng_total / grid;
    p.gpc_rem = int(ng_total % grid);
    p.set_cap = R;
    p.status = di->status;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(grid));
    cfg.blockDim = dim3(kMtThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    if (flags & BL_FLAG_PDL) {
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
    return cuda_status(cudaLaunchKernelEx(&cfg, kern, p));
}

// Chunks of 8 elements per lane that hold a whole row: 8, 16 or 32 (K up to
// 2048, 4096 or 8192); longer rows are not taken by this kernel.
template <int MT, int MODE>
int launch_mt_k(const MtParams &p, cudaStream_t s, unsigned flags)
{
    if (p.K <= 2048)
        return launch_mt_t<MT, MODE, 8>(p, s, flags);
    if constexpr (MODE == MT_X_F32)
        return launch_mt_t<MT, MODE, 16>(p, s, flags);
    else
        return p.K <= 4096 ? launch_mt_t<MT, MODE, 16>(p, s, flags) : launch_mt_t<MT, MODE, 32>(p, s, flags);
}

template <int MT>
int launch_mt_mode(const MtParams &p, bool fused, int xt, cudaStream_t s, unsigned flags)
{
    if (!fused)
        return launch_mt_t<MT, MT_Q, 0>(p, s, flags);
    if (xt == BL_BF16)
        return launch_mt_k<MT, MT_X_BF16>(p, s, flags);
    return launch_mt_k<MT, MT_X_F32>(p, s, flags);
}

}  // namespace

// 2 .. 16 tokens, K a multiple of 256 up to 8192 (4096 for fp32 input), at
// most 32 row groups per CTA (one CTA per SM) and the activations plus the
// ring within shared memory.
bool gemv_stream_mt_applies(const GemvBatch &b, bool fused, int sm_count, int max_smem)
{
    if (b.M < 2 || b.M > kMtMaxTokens || b.K % 256 != 0 || b.K > kMtMaxK || b.count < 1 || sm_count <= 0)
        return false;
    if (fused && b.xt != BL_BF16 && b.K > kMtMaxK / 2)     // fp32 rows: 16 chunks per lane at most
        return false;
    int64_t ng = 0;
    for (int i = 0; i < b.count; ++i)
        ng += (b.prob[i].N + 7) / 8;
    if (ng > int64_t(kMtMaxGroupsPerCta) * sm_count)
        return false;
    return mt_smem(b.K, int(b.M), 2) <= size_t(max_smem);
}

int launch_gemv_stream_mt(const GemvBatch &b, bool fused, cudaStream_t s)
{
    MtParams p{};
    p.count = b.count;
    p.gstart[0] = 0;
    for (int i = 0; i < b.count; ++i) {
        p.prob[i] = b.prob[i];
        p.gstart[i + 1] = p.gstart[i] + (b.prob[i].N + 7) / 8;
    }
    for (int i = b.count; i < kGemvMaxProblems; ++i)
        p.gstart[i + 1] = p.gstart[b.count];
    p.K = b.K;
    p.M = int(b.M);
    p.q = b.q;
    p.d = b.d;
    p.rowsum = b.rowsum;
    p.x = b.x;
    p.ldx = b.ldx;
    p.yt = b.yt;
    if (b.M <= 2)
        return launch_mt_mode<2>(p, fused, b.xt, s, b.flags);
    if (b.M <= 4)
        return launch_mt_mode<4>(p, fused, b.xt, s, b.flags);
    if (b.M <= 8)
        return launch_mt_mode<8>(p, fused, b.xt, s, b.flags);
    return launch_mt_mode<16>(p, fused, b.xt, s, b.flags);
}

}  // namespace bl
