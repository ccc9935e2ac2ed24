// gemv_stream.cu -- ternary decode GEMV for one token (K a multiple of 256),
// one or several products sharing the token (q/k/v, gate/up).
//
// "How to Run BitNet Inference on GPU Using CUDA Kernels: A Complete Guide",
// section "Understanding the Two-Phase Architecture": decode is a
// memory-bound INT8-activation x INT2-weight product, so the weight stream
// N*K/4 bytes is the whole cost and every instruction spent per weight byte
// beyond the dot product itself lowers the bandwidth an SM can sustain.
//
// Design (B200, persistent CTAs):
//   * A CTA is KC consumer warps plus one producer warp: KC = 8 up to
//     K = 8192 (10 for a launch of at most one CTA per SM whose k range has
//     more than eight pieces of 256 k), else KC = 16.  Large launches (at least 16 row groups per
//     SM) run two 8-warp CTAs per SM, so that a CTA of the next launch
//     (programmatic dependent launch) can take the place of one that has
//     finished, or one 16-warp CTA per SM, which halves the per-SM cost of
//     quantising a long token.  Smaller launches run at most one CTA per SM,
//     leaving room beside it for the next launch's CTA, which then fetches
//     its weights while this launch computes.
//   * The products' 8-row groups are concatenated into one list; each CTA
//     owns a contiguous range of it (a group's packed slab, 2*K bytes, is
//     contiguous in the tile layout).  It takes them in sets of at most R
//     groups, sized evenly, with R (4..8) chosen per launch so that every CTA
//     has the same number of sets; a set is streamed in stages, a stage
//     holding the same k range of each of the set's groups (512 bytes per
//     256 k): the whole range when it is at most 512*KC k, else 256*KC k.
//   * The producer warp fills a four-stage ring with bulk asynchronous
//     copies (one copy per group, each from a different lane, since the
//     copies of one thread complete one after another), completion counted
//     on the stage's mbarrier.
//   * Consumer warp w always takes 512-byte pieces w (and w + KC) of each
//     group in a stage (lane l: row l%8, 64 k; in a stage that ends the k
//     range short, only the warps with a piece compute), so the activations
//     it needs, 64 bytes per
//     lane, are loaded once per stage and used for all of the stage's groups
//     (whose loads are issued together, by a body specialised on the group
//     count).  Multiply with the stored codes s = code + 1: (word &
//     0x03030303), (word & 0x0c0c0c0c), ... hold s, 4s, 16s, 64s per byte;
//     one LOP3 and one dp4a per four weights into four accumulators per
//     group, folded with shifts when the group's last stage is done;
//     sum(code q) = sum(s q) - rowsum(q).
//   * The ring is filled from the start; the consumers wait on the preceding
//     launch only before they read the activations, which they quantise (or
//     copy) into shared memory.
//   * Every mbarrier wait is bounded; on expiry the CTA records
//     BL_ERR_TIMEOUT, the consumers stop and the producer waits (bounded) for
//     its copies in flight before the CTA exits.
#include "gemv_stream_common.cuh"

namespace bl {

int launch_gemv_stream(const GemvBatch &b, bool fused, cudaStream_t s);
bool gemv_stream_applies(const GemvBatch &b, int sm_count);

namespace {

// Ring protocol.  Stage t (set i, k-range kb) occupies ring slot
// t % kStages, room for R groups, of which it fills |set i|; full[slot]
// counts its bytes, empty[slot] the KC consumer warps that have read it
// (phase parity (t / kStages) & 1, kept as a running bit).
template <int KC, int MODE, int CH>
__global__ void __launch_bounds__(Geo<KC>::kThreads, Geo<KC>::kCtasPerSm)
    gemv_stream_kernel(const StreamParams p)
{
    using G = Geo<KC>;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    StreamSmem &sm = *reinterpret_cast<StreamSmem *>(smem_raw);
    const uint32_t ring = smem_u32(smem_raw + kHeader);
    const int R = p.set_cap;
    const int P = int(p.K / 256);              // 512-byte pieces per group
    const int PS = stage_pieces(P, KC);        // pieces of each group per stage
    const uint32_t slot = uint32_t(PS) * 512;  // ring bytes of one group per stage
    const uint32_t stage_bytes = uint32_t(R) * slot;
    int8_t *qs = reinterpret_cast<int8_t *>(smem_raw + kHeader + size_t(kStages) * stage_bytes);
    volatile int *abort_flag = &sm.abort_flag;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bx = blockIdx.x;
    const int64_t g_begin = bx * p.gpc_base + (bx < p.gpc_rem ? bx : p.gpc_rem);
    const int ng = int(p.gpc_base) + (bx < p.gpc_rem ? 1 : 0);
    const int subs = (P + PS - 1) / PS;        // stages per set
    const int64_t slab = 2 * p.K;              // packed bytes of one row group
    const SetSplit split(ng, R);

    if (tid == 0) {
        for (int b = 0; b < kStages; ++b) {
            mbar_init(smem_u32(&sm.full[b]), 1);
            mbar_init(smem_u32(&sm.empty[b]), KC);
        }
        sm.abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    for (int i = tid; i < ng * 8; i += G::kThreads)
        (&sm.sacc[0][0])[i] = 0;
    __syncthreads();
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    if (warp == KC) {
        // ------------------------------------------------ producer warp
        int t = 0, sb = 0, g0 = 0;
        uint32_t ph = 0;
        bool ok = true;
        for (int i = 0; i < split.nsets && ok; ++i) {
            const int rg = split.size(i);
            // lane r < rg: the packed slab of the set's group r
            const uint8_t *src = nullptr;
            if (lane < rg) {
                const int64_t G = g_begin + g0 + lane;
                const int pi = locate(p, G);
                src = p.prob[pi].packed + (G - p.gstart[pi]) * slab;
            }
            for (int kb = 0; kb < subs; ++kb) {
                const int np = min(PS, P - kb * PS);          // pieces of each group in this stage
                const uint32_t bytes = uint32_t(np) * 512;
                if (!__all_sync(0xffffffffu, mbar_wait_fast(smem_u32(&sm.empty[sb]), ph ^ 1u, abort_flag, p.status))) {
                    ok = false;
                    break;
                }
                const uint32_t full = smem_u32(&sm.full[sb]);
                if (lane == 0)
                    mbar_arrive_tx(full, uint32_t(rg) * bytes);
                __syncwarp();
                // lanes (t*kMaxSet + r) mod 32 each copy one group's part
                const int r = (lane - t * kMaxSet) & 31;
                const uint8_t *src_r = reinterpret_cast<const uint8_t *>(
                    __shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(src), r & 31));
                if (r < rg)
                    bulk_load(ring + uint32_t(sb) * stage_bytes + uint32_t(r) * slot,
                              src_r + int64_t(kb) * slot, bytes, full);
                ++t;
                if (++sb == kStages) {
                    sb = 0;
                    ph ^= 1u;
                }
            }
            g0 += rg;
        }
        // the copies still in flight land before the CTA exits (at once,
        // unless the consumers gave up before taking them)
        volatile int no_abort = 0;
        for (int u = t - kStages > 0 ? t - kStages : 0; u < t; ++u)
            mbar_wait(smem_u32(&sm.full[u % kStages]), uint32_t(u / kStages) & 1u, &no_abort, p.status,
                      100000000ull);
        return;
    }

    // ---------------------------------------------------- consumer warps
    // (nothing above waits on global memory, so the producer starts at once;
    // the weight scale's latency hides under the prologue)
    if (tid < p.count)
        sm.wscale[tid] = __ldg(p.prob[tid].w_scale);
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if constexpr (MODE == SMODE_Q)
        stream_copy_q<KC>(p, sm, qs);
    else if constexpr (MODE == SMODE_NORM_BF16)
        stream_rmsnorm_quantize<KC, BL_BF16, CH>(p, sm, qs);
    else if constexpr (MODE == SMODE_NORM_F32)
        stream_rmsnorm_quantize<KC, BL_F32, 0>(p, sm, qs);
    else if constexpr (MODE == SMODE_RELU2)
        stream_relu2_quantize<KC>(p, sm, qs);
    else if constexpr (MODE == SMODE_X_BF16 && CH > 0)
        stream_quantize_bf16<KC, CH>(p, sm, qs);
    else
        stream_quantize_2pass<KC, MODE == SMODE_X_BF16 ? BL_BF16 : BL_F32>(p, sm, qs);
    // (each warp reads only the activations it wrote itself: no barrier)

    const uint32_t ring_lane = ring + uint32_t(warp) * 512 + uint32_t(lane) * 16;
    const uint32_t q_lane = smem_u32(qs) + uint32_t(warp) * 256 + uint32_t(lane >> 3) * 64;
    int acc[kMaxSet][4];
#pragma unroll
    for (int r = 0; r < kMaxSet; ++r)
#pragma unroll
        for (int a = 0; a < 4; ++a)
            acc[r][a] = 0;
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
            // this warp's pieces of the stage: w and (one stage per set) w + KC
            const int np = min(PS, P - kb * PS);
            if (PS == KC) {
                if (warp < np) {
                    uint4 q[4];
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        q[j] = lds128(q_lane + uint32_t(kb * KC) * 256 + 16 * j);
                    stage_mac_n<KC * 512>(rg, ring_lane + uint32_t(sb) * stage_bytes, slot, q, acc);
                }
            } else {
#pragma unroll
                for (int m = 0; m < 2; ++m) {
                    if (warp + m * KC < np) {
                        uint4 q[4];
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            q[j] = lds128(q_lane + uint32_t(m * KC) * 256 + 16 * j);
                        stage_mac_n<0>(rg, ring_lane + uint32_t(sb) * stage_bytes + uint32_t(m * KC) * 512, slot, q,
                                       acc);
                    }
                }
            }
            __syncwarp();
            if (lane == 0)
                mbar_arrive(smem_u32(&sm.empty[sb]));
            if (++sb == kStages) {
                sb = 0;
                ph ^= 1u;
            }
        }
        // the set's groups are complete: add their partial row sums
        set_flush_n(rg, acc, &sm.sacc[g0], lane);
        g0 += rg;
    }
    consumers_sync<KC>();
    // rescale and write this CTA's rows
    const float dd = sm.d;
    int rs = 0;
#pragma unroll
    for (int w = 0; w < KC; ++w)
        rs += sm.bsum[w];
    for (int idx = tid; idx < ng * 8; idx += G::kConsumerThreads) {
        const int64_t Gr = g_begin + (idx >> 3);
        const int pi = locate(p, Gr);
        const GemvProblem &pr = p.prob[pi];
        const int64_t row = (Gr - p.gstart[pi]) * 8 + (idx & 7);
        if (row < pr.N) {
            const int a = (&sm.sacc[0][0])[idx] - rs;
            if (pr.acc_dbg)
                pr.acc_dbg[row] = a;
            float v = rescale1(a, dd, sm.wscale[pi]);
            if (pr.resid) {
                // residual stream: one fp32 addition before the bf16 rounding
                // (read coherently: the preceding launch may have written it)
                const uint32_t hb = ld_dep_u16(static_cast<const uint16_t *>(pr.resid) + row);
                v = __fadd_rn(__uint_as_float(hb << 16), v);
            }
            store_y(pr.y, p.yt, row, v);
        }
    }
}

template <int KC, int MODE, int CH>
int launch_mode(const StreamParams &base, cudaStream_t s, unsigned flags)
{
    const int64_t ng_total = base.gstart[base.count];
    using G = Geo<KC>;
    const DeviceInfo *di = device_info();
    if (!di)
        return BL_ERR_CUDA;
    auto kern = gemv_stream_kernel<KC, MODE, CH>;
    const int ps = stage_pieces(int(base.K / 256), KC);
    auto smem_of = [&](int c) { return kHeader + size_t(kStages) * c * ps * 512 + size_t(base.K); };
    // R: the smallest stage capacity (>= 4 groups) that fits in shared memory
    // and gives every CTA of a grid of `ctas` the same number of sets, so that
    // no CTA streams an extra set of leftovers; 4 (which always fits: K <=
    // 32768) otherwise
    auto pick_r = [&](int64_t ctas) {
        const int64_t lo = ng_total / ctas, hi = lo + (ng_total % ctas ? 1 : 0);
        for (int c = 4; c <= kMaxSet; ++c)
            if (smem_of(c) <= size_t(di->max_smem_optin) && (lo + c - 1) / c == (hi + c - 1) / c)
                return c;
        return 4;
    };
    // large launches (>= kLargeGroupsPerSm row groups per SM): G::kCtasPerSm
    // CTAs per SM (one if they do not fit); the others at most one per SM,
    // which leaves room beside each CTA for one of the next launch
    const int top = ng_total >= kLargeGroupsPerSm * int64_t(di->sm_count) ? G::kCtasPerSm : 1;
    int per_sm = 0, R = 4;
    int64_t grid_n = 0;
    for (int want = top; want >= 1; --want) {
        const int64_t cap = int64_t(want) * di->sm_count;
        grid_n = ng_total < cap ? ng_total : cap;
        R = pick_r(grid_n);
        int st = occupancy(reinterpret_cast<const void *>(kern), G::kThreads, smem_of(R), &per_sm);
        if (st)
            return st;
        if (per_sm >= want)
            break;
    }
    if (per_sm < 1)
        return BL_ERR_SHAPE;
    const size_t smem = smem_of(R);
    StreamParams pp = base;
    pp.gpc_base = ng_total / grid_n;
    pp.gpc_rem = int(ng_total % grid_n);
    pp.set_cap = R;
    pp.status = di->status;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(grid_n));
    cfg.blockDim = dim3(G::kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    if (flags & BL_FLAG_PDL) {
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
    return cuda_status(cudaLaunchKernelEx(&cfg, kern, pp));
}

template <int KC>
int launch_kc(const StreamParams &p, bool fused, int xt, cudaStream_t s, unsigned flags, bool norm)
{
    if (norm) {
        if (xt != BL_BF16)
            return launch_mode<KC, SMODE_NORM_F32, 0>(p, s, flags);
        constexpr int kNormChunks = 8 * Geo<KC>::kConsumerThreads;
        if (p.K <= int64_t(4) * kNormChunks)
            return launch_mode<KC, SMODE_NORM_BF16, 4>(p, s, flags);
        return launch_mode<KC, SMODE_NORM_BF16, 0>(p, s, flags);
    }
    if (!fused)
        return launch_mode<KC, SMODE_Q, 0>(p, s, flags);
    if (xt != BL_BF16)
        return launch_mode<KC, SMODE_X_F32, 0>(p, s, flags);
    // raw bf16 held in registers: at most 8 chunks of 8 values per consumer
    // thread (32 registers), else two passes over x
    constexpr int kChunks = 8 * Geo<KC>::kConsumerThreads;
    if (p.K <= int64_t(4) * kChunks)
        return launch_mode<KC, SMODE_X_BF16, 4>(p, s, flags);
    if (p.K <= int64_t(8) * kChunks)
        return launch_mode<KC, SMODE_X_BF16, 8>(p, s, flags);
    return launch_mode<KC, SMODE_X_BF16, 0>(p, s, flags);
}

// Ten consumer warps instead of eight for a launch of at most one CTA per SM
// (fewer than kLargeGroupsPerSm row groups per SM) whose k range has more
// than eight pieces: at K = 2560 (ten pieces) every warp takes one piece of a
// group instead of two warps taking two, and at K = 6912 (27 pieces) a group
// takes three stage rounds instead of four.  The stage work is bound by the
// latency of each warp's dp4a chains, so the busiest warp sets its length.
// Two such CTAs (352 threads) still fit on an SM beside each other, so the
// next launch's CTA keeps fetching its weights early.
bool ten_warps(const StreamParams &p)
{
    const DeviceInfo *di = device_info();
    const int64_t ng_total = p.gstart[p.count];
    return di && p.K / 256 > 8 && ng_total < kLargeGroupsPerSm * int64_t(di->sm_count);
}

}  // namespace

// One token, K a multiple of 256 (at most 32768), at most kMaxGroupsPerCta
// row groups per CTA (one CTA per SM).
bool gemv_stream_applies(const GemvBatch &b, int sm_count)
{
    if (b.M != 1 || b.K % 256 != 0 || b.K > 32768 || b.count < 1 || sm_count <= 0)
        return false;
    int64_t ng = 0;
    for (int i = 0; i < b.count; ++i)
        ng += (b.prob[i].N + 7) / 8;
    return ng <= int64_t(kMaxGroupsPerCta) * sm_count;
}

int launch_gemv_stream(const GemvBatch &b, bool fused, cudaStream_t s, const void *gain, int gt,
                       float eps, bool norm)
{
    StreamParams p{};
    p.count = b.count;
    p.gstart[0] = 0;
    for (int i = 0; i < b.count; ++i) {
        p.prob[i] = b.prob[i];
        p.gstart[i + 1] = p.gstart[i] + (b.prob[i].N + 7) / 8;
    }
    for (int i = b.count; i < kGemvMaxProblems; ++i)
        p.gstart[i + 1] = p.gstart[b.count];
    p.K = b.K;
    p.q = b.q;
    p.d = b.d;
    p.rowsum = b.rowsum;
    p.x = b.x;
    p.gain = gain;
    p.gt = gt;
    p.eps = eps;
    p.yt = b.yt;
    if (b.K <= kSmallK)
        return ten_warps(p) ? launch_kc<10>(p, fused, b.xt, s, b.flags, norm)
                            : launch_kc<8>(p, fused, b.xt, s, b.flags, norm);
    return launch_kc<16>(p, fused, b.xt, s, b.flags, norm);
}

int launch_gemv_stream(const GemvBatch &b, bool fused, cudaStream_t s)
{
    return launch_gemv_stream(b, fused, s, nullptr, BL_F32, 0.0f, false);
}

int launch_gemv_stream_relu2(const GemvBatch &b, const void *x2, cudaStream_t s)
{
    StreamParams p{};
    p.count = b.count;
    p.gstart[0] = 0;
    for (int i = 0; i < b.count; ++i) {
        p.prob[i] = b.prob[i];
        p.gstart[i + 1] = p.gstart[i] + (b.prob[i].N + 7) / 8;
    }
    for (int i = b.count; i < kGemvMaxProblems; ++i)
        p.gstart[i + 1] = p.gstart[b.count];
    p.K = b.K;
    p.x = b.x;
    p.x2 = x2;
    p.yt = b.yt;
    if (b.K <= kSmallK)
        return ten_warps(p) ? launch_mode<10, SMODE_RELU2, 0>(p, s, b.flags)
                            : launch_mode<8, SMODE_RELU2, 0>(p, s, b.flags);
    return launch_mode<16, SMODE_RELU2, 0>(p, s, b.flags);
}

}  // namespace bl
