// gemv_chain.cu -- a token's whole chain of dependent decode BitLinears in one
// persistent launch.
//
// "How to Run BitNet Inference on GPU Using CUDA Kernels: A Complete Guide",
// sections "Understanding the Two-Phase Architecture" (decode: one token at a
// time through memory-bound INT8 x INT2 linears) and "Key Components and
// Source Code Architecture" (CUDA graphs to remove launch overhead).  A
// decode step is a chain of GEMVs in which each reads the output of the one
// before (q/k/v -> o -> gate/up -> down -> next layer), so launched one by one
// every product pays a launch's ramp, the wait for the previous grid to
// drain, and the re-fetch of its activations; the weights themselves never
// depend on the activations.
//
// Design (one cooperative launch, one CTA per SM, all resident):
//   * The chain is a list of steps in device memory (the plan); a step is
//     one to eight products sharing their input x (as in
//     bitlinear_gemv_fused_multi), optionally normalised (RMSNorm) first.
//     Each CTA owns a contiguous run of every step's 8-row groups.
//   * The producer warp streams the CTA's weights for all steps, in order,
//     through a six-stage ring of 32 KiB with bulk copies (one per group per
//     stage, from different lanes), never waiting on activations: it runs
//     as far ahead of the consumers, across step boundaries, as the ring
//     allows.
//   * The sixteen consumer warps take one step at a time: wait until every CTA
//     has finished the previous step (a per-step arrival counter in the
//     plan, polled by one thread, then an acquire fence), read x from L2,
//     quantise it (the prologues of the one-token streaming kernel), consume
//     the step's stages, fold the partial row sums, rescale and store their
//     rows of y, and arrive on the step's counter (block barrier, then one
//     release reduction).
//   * Every wait -- mbarriers and counters -- is bounded (2 s of
//     %globaltimer); a CTA that gives up records BL_ERR_TIMEOUT in the device
//     status word and raises the plan's abort word, which every other wait
//     checks, so the whole grid leaves promptly; the producer waits (bounded)
//     for its copies in flight before its CTA exits.
// The host zeroes the counters and the abort word before every launch.
//
// Measured on B200 (2.4B decode stream, 120 steps, %globaltimer stamps per
// CTA and step): a step costs ~0.9 us from the last arrival to the release of
// the waiting CTAs, ~1.1 us of prologue (x from L2, absmax, quantise), the
// stage work, ~0.35 us of stores and ~0.55 us for the release reduction to
// retire behind them: 4.0-6.5 us per step, against ~3.1 us per launch when
// every step is its own launch chained with programmatic dependent launch,
// whose hand-off the hardware does faster than this software grid barrier.
// The chain is exact and needs one launch per token; the per-launch chain is
// the faster way to run a decode step here.
#include <vector>

#include "gemv_stream_common.cuh"

namespace bl {
namespace {

constexpr int kChainKC = 16;                      // consumer warps
constexpr int kChainThreads = 32 * (kChainKC + 1);
constexpr int kChainStages = 6;
constexpr uint32_t kChainStageBytes = 32 * 1024;
constexpr int64_t kChainMaxK = 16384;             // int8 activations staged in shared memory
constexpr int kChainMaxStepsLimit = 4096;

// One step of the chain (device memory; the consumers work from a copy in
// shared memory).  The field names the activation prologues read (x, K, q,
// d, rowsum, gain, gt, eps) are those of StreamParams.
struct alignas(16) ChainStep {
    GemvProblem prob[kGemvMaxProblems];
    int64_t gstart[kGemvMaxProblems + 1];   // prefix sums of the products' row groups
    int count;
    int64_t K;
    const void *x;
    int xt;
    int yt;
    int set_cap;                            // R: groups a stage holds at most
    int norm;                               // RMSNorm before quantisation
    const void *gain;
    int gt;
    float eps;
    const int8_t *q;                        // unused (always quantised in the kernel)
    const float *d;
    const int32_t *rowsum;
};

struct ChainHeader {
    int nsteps;
    int pad[3];
};

// plan = header | steps[nsteps] | counters[nsteps] (uint32) | abort word
size_t steps_offset() { return (sizeof(ChainHeader) + 127) / 128 * 128; }
size_t counters_offset(int n) { return (steps_offset() + size_t(n) * sizeof(ChainStep) + 127) / 128 * 128; }
size_t plan_bytes(int n) { return counters_offset(n) + (size_t(n) + 1) * 4; }

struct ChainSmem {
    uint64_t full[kChainStages];
    uint64_t empty[kChainStages];
    int abort_flag;
    alignas(16) float bmax[kMaxConsumers];
    int bsum[kMaxConsumers];
    double bss[kMaxConsumers];
    float d;
    float wscale[kGemvMaxProblems];
    int go;          // the step's counter wait succeeded (written by thread 0)
    int step_fail;   // a consumer warp gave up during the step
    ChainStep cur;   // the consumers' current step
    int sacc[kMaxGroupsPerCta][8];
};

constexpr size_t kChainHeader = (sizeof(ChainSmem) + 127) / 128 * 128;
constexpr size_t kChainSmem = kChainHeader + size_t(kChainStages) * kChainStageBytes + size_t(kChainMaxK);

__device__ __forceinline__ uint32_t ld_relaxed_u32(const unsigned *p)
{
    uint32_t v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void fence_acq_rel_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }

// Arrival on a step counter: release (orders this CTA's earlier stores, made
// visible to this thread by the block barrier before it) and add.
__device__ __forceinline__ void red_release_add(unsigned *p, unsigned v)
{
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ int locate_step(const ChainStep &p, int64_t G)
{
    int pi = 0;
#pragma unroll
    for (int i = 1; i < kGemvMaxProblems; ++i)
        if (i < p.count && G >= p.gstart[i])
            pi = i;
    return pi;
}

// Raise the grid-wide abort word (and this CTA's flag).
__device__ __forceinline__ void chain_abort(unsigned *g_abort, volatile int *abort_flag)
{
    *abort_flag = 1;
    atomicExch(g_abort, 1u);
}

// Wait until counter >= target, bounded; false on timeout or abort.  Relaxed
// polling, one acquire fence once the count is reached.
__device__ __noinline__ bool wait_counter(const unsigned *counter, unsigned target, unsigned *g_abort,
                                          volatile int *abort_flag, int *status, uint64_t limit_ns)
{
    if (ld_relaxed_u32(counter) >= target) {
        fence_acq_rel_gpu();
        return true;
    }
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 1;; ++it) {
        if (ld_relaxed_u32(counter) >= target) {
            fence_acq_rel_gpu();
            return true;
        }
        if ((it & 15) == 0) {
            if (*abort_flag || ld_relaxed_u32(g_abort)) {
                *abort_flag = 1;
                return false;
            }
            if (global_timer_ns() - t0 > limit_ns) {
                atomicExch(status, BL_ERR_TIMEOUT);
                chain_abort(g_abort, abort_flag);
                return false;
            }
        }
    }
}

// The step's activation prologue: quantise x (RMSNorm first when asked) into
// qs; per-warp row sums to sm.bsum, d to sm.d.
__device__ __forceinline__ void chain_prologue(const ChainStep &p, ChainSmem &sm, int8_t *qs)
{
    constexpr int KC = kChainKC;
    const bool regs = p.K <= int64_t(4) * 8 * 32 * KC;    // raw bf16 x fits 4 chunks per lane
    if (p.norm) {
        if (p.xt == BL_BF16 && regs)
            stream_rmsnorm_quantize<KC, BL_BF16, 4>(p, sm, qs);
        else if (p.xt == BL_BF16)
            stream_rmsnorm_quantize<KC, BL_BF16, 0>(p, sm, qs);
        else
            stream_rmsnorm_quantize<KC, BL_F32, 0>(p, sm, qs);
    } else {
        if (p.xt == BL_BF16 && regs)
            stream_quantize_bf16<KC, 4>(p, sm, qs);
        else if (p.xt == BL_BF16)
            stream_quantize_2pass<KC, BL_BF16>(p, sm, qs);
        else
            stream_quantize_2pass<KC, BL_F32>(p, sm, qs);
    }
}

// Row groups of step p owned by CTA b of G: [begin, begin + n).
__device__ __forceinline__ void cta_groups(const ChainStep &p, int b, int G, int64_t &begin, int &n)
{
    const int64_t total = p.gstart[p.count];
    const int64_t base = total / G;
    const int rem = int(total % G);
    begin = b * base + (b < rem ? b : rem);
    n = int(base) + (b < rem ? 1 : 0);
}

// Test hook: with test_step >= 0 the wait before step test_step expects one
// arrival more than there are CTAs -- a count nothing reaches -- so it runs
// out after limit_ns and the grid takes its abort path.
__global__ void __launch_bounds__(kChainThreads, 1) gemv_chain_kernel(const ChainStep *steps, int nsteps,
                                                                      unsigned *counters, unsigned *g_abort,
                                                                      int *status, uint64_t limit_ns,
                                                                      int test_step)
{
    constexpr int KC = kChainKC;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    ChainSmem &sm = *reinterpret_cast<ChainSmem *>(smem_raw);
    const uint32_t ring = smem_u32(smem_raw + kChainHeader);
    int8_t *qs = reinterpret_cast<int8_t *>(smem_raw + kChainHeader + size_t(kChainStages) * kChainStageBytes);
    volatile int *abort_flag = &sm.abort_flag;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bx = blockIdx.x, G = gridDim.x;

    if (tid == 0) {
        for (int b = 0; b < kChainStages; ++b) {
            mbar_init(smem_u32(&sm.full[b]), 1);
            mbar_init(smem_u32(&sm.empty[b]), KC);
        }
        sm.abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    for (int i = tid; i < kMaxGroupsPerCta * 8; i += kChainThreads)
        (&sm.sacc[0][0])[i] = 0;
    __syncthreads();

    if (warp == KC) {
        // ------------------------------------------------ producer warp
        int t = 0, sb = 0;
        uint32_t ph = 0;
        bool ok = true;
        for (int s = 0; s < nsteps && ok; ++s) {
            const ChainStep &p = steps[s];
            int64_t g_begin;
            int ng;
            cta_groups(p, bx, G, g_begin, ng);
            if (ng == 0)
                continue;
            const int P = int(p.K / 256);
            const int PS = stage_pieces(P, KC);
            const uint32_t slot = uint32_t(PS) * 512;
            const int subs = (P + PS - 1) / PS;
            const int64_t slab = 2 * p.K;
            const SetSplit split(ng, p.set_cap);
            int g0 = 0;
            for (int i = 0; i < split.nsets && ok; ++i) {
                const int rg = split.size(i);
                const uint8_t *src = nullptr;
                if (lane < rg) {
                    const int64_t Gr = g_begin + g0 + lane;
                    const int pi = locate_step(p, Gr);
                    src = p.prob[pi].packed + (Gr - p.gstart[pi]) * slab;
                }
                for (int kb = 0; kb < subs; ++kb) {
                    const int np = min(PS, P - kb * PS);
                    const uint32_t bytes = uint32_t(np) * 512;
                    if (!__all_sync(0xffffffffu,
                                    mbar_wait_fast(smem_u32(&sm.empty[sb]), ph ^ 1u, abort_flag, status))) {
                        ok = false;
                        break;
                    }
                    const uint32_t full = smem_u32(&sm.full[sb]);
                    if (lane == 0)
                        mbar_arrive_tx(full, uint32_t(rg) * bytes);
                    __syncwarp();
                    const int r = (lane - t * kMaxSet) & 31;
                    const uint8_t *src_r = reinterpret_cast<const uint8_t *>(
                        __shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(src), r & 31));
                    if (r < rg)
                        bulk_load(ring + uint32_t(sb) * kChainStageBytes + uint32_t(r) * slot,
                                  src_r + int64_t(kb) * slot, bytes, full);
                    ++t;
                    if (++sb == kChainStages) {
                        sb = 0;
                        ph ^= 1u;
                    }
                }
                g0 += rg;
            }
        }
        if (!ok)
            chain_abort(g_abort, abort_flag);
        volatile int no_abort = 0;
        for (int u = t - kChainStages > 0 ? t - kChainStages : 0; u < t; ++u)
            mbar_wait(smem_u32(&sm.full[u % kChainStages]), uint32_t(u / kChainStages) & 1u, &no_abort, status,
                      100000000ull);
        return;
    }

    // ---------------------------------------------------- consumer warps
    int acc[kMaxSet][4];
#pragma unroll
    for (int r = 0; r < kMaxSet; ++r)
#pragma unroll
        for (int a = 0; a < 4; ++a)
            acc[r][a] = 0;
    int sb = 0;
    uint32_t ph = 0;
    bool ok = true;
    const ChainStep &p = sm.cur;
    for (int s = 0; s < nsteps && ok; ++s) {
        const ChainStep &pg = steps[s];
        int64_t g_begin;
        int ng;
        cta_groups(pg, bx, G, g_begin, ng);
        if (ng > 0) {
            // every CTA has finished the previous step: its outputs (this
            // step's x, or an earlier step's) are in memory.  One thread
            // waits and the decision is read by all consumer warps after a
            // barrier, so that they all leave (or stay) together; meanwhile
            // warp 1 copies the step's descriptor into shared memory.
            if (tid == 0) {
                sm.step_fail = 0;
                const unsigned target = unsigned(G) + (s == test_step ? 1u : 0u);
                sm.go = s == 0 ? 1 : int(wait_counter(&counters[s - 1], target, g_abort, abort_flag, status, limit_ns));
            } else if (warp == 1) {
                constexpr int kVecs = int(sizeof(ChainStep) / 16);
                for (int i = lane; i < kVecs; i += 32)
                    reinterpret_cast<uint4 *>(&sm.cur)[i] = reinterpret_cast<const uint4 *>(&pg)[i];
            }
            consumers_sync<KC>();
            if (!sm.go) {
                ok = false;
                break;
            }
            if (tid < p.count)
                sm.wscale[tid] = __ldg(p.prob[tid].w_scale);
            chain_prologue(p, sm, qs);

            const int P = int(p.K / 256);
            const int PS = stage_pieces(P, KC);
            const uint32_t slot = uint32_t(PS) * 512;
            const int subs = (P + PS - 1) / PS;
            const SetSplit split(ng, p.set_cap);
            const uint32_t ring_lane = ring + uint32_t(warp) * 512 + uint32_t(lane) * 16;
            const uint32_t q_lane = smem_u32(qs) + uint32_t(warp) * 256 + uint32_t(lane >> 3) * 64;
            int g0 = 0;
            for (int i = 0; i < split.nsets && ok; ++i) {
                const int rg = split.size(i);
                for (int kb = 0; kb < subs; ++kb) {
                    if (!__all_sync(0xffffffffu, mbar_wait_fast(smem_u32(&sm.full[sb]), ph, abort_flag, status))) {
                        ok = false;
                        break;
                    }
                    const int np = min(PS, P - kb * PS);
                    if (PS == KC) {
                        if (warp < np) {
                            uint4 q[4];
#pragma unroll
                            for (int j = 0; j < 4; ++j)
                                q[j] = lds128(q_lane + uint32_t(kb * KC) * 256 + 16 * j);
                            stage_mac_n<KC * 512>(rg, ring_lane + uint32_t(sb) * kChainStageBytes, slot, q, acc);
                        }
                    } else {
#pragma unroll
                        for (int m = 0; m < 2; ++m) {
                            if (warp + m * KC < np) {
                                uint4 q[4];
#pragma unroll
                                for (int j = 0; j < 4; ++j)
                                    q[j] = lds128(q_lane + uint32_t(m * KC) * 256 + 16 * j);
                                stage_mac_n<0>(rg, ring_lane + uint32_t(sb) * kChainStageBytes + uint32_t(m * KC) * 512,
                                               slot, q, acc);
                            }
                        }
                    }
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive(smem_u32(&sm.empty[sb]));
                    if (++sb == kChainStages) {
                        sb = 0;
                        ph ^= 1u;
                    }
                }
                if (!ok)
                    break;
                set_flush_n(rg, acc, &sm.sacc[g0], lane);
                g0 += rg;
            }
            // the step's outcome, decided uniformly: step_fail is written only
            // by consumer warps, only before this barrier
            if (!ok && lane == 0)
                sm.step_fail = 1;
            consumers_sync<KC>();
            if (sm.step_fail) {
                ok = false;
                break;
            }
            // rescale and store this CTA's rows; clear the row sums behind
            const float dd = sm.d;
            int rs = 0;
#pragma unroll
            for (int w = 0; w < KC; ++w)
                rs += sm.bsum[w];
            for (int idx = tid; idx < ng * 8; idx += 32 * KC) {
                const int64_t Gr = g_begin + (idx >> 3);
                const int pi = locate_step(p, Gr);
                const GemvProblem &pr = p.prob[pi];
                const int64_t row = (Gr - p.gstart[pi]) * 8 + (idx & 7);
                const int a = (&sm.sacc[0][0])[idx] - rs;
                (&sm.sacc[0][0])[idx] = 0;
                if (row < pr.N) {
                    if (pr.acc_dbg)
                        pr.acc_dbg[row] = a;
                    store_y(pr.y, p.yt, row, rescale1(a, dd, sm.wscale[pi]));
                }
            }
            consumers_sync<KC>();
        }
        // this CTA is done with step s (its outputs are stored; the barrier
        // above ordered them before this release)
        if (tid == 0)
            red_release_add(&counters[s], 1u);
    }
    if (!ok)
        chain_abort(g_abort, abort_flag);
}

// Occupancy-checked grid: one CTA per SM, all resident (cooperative launch).
int chain_grid(int *grid)
{
    const DeviceInfo *di = device_info();
    if (!di)
        return BL_ERR_CUDA;
    int per_sm = 0;
    int st = occupancy(reinterpret_cast<const void *>(gemv_chain_kernel), kChainThreads, kChainSmem, &per_sm);
    if (st)
        return st;
    if (per_sm < 1)
        return BL_ERR_SHAPE;
    *grid = di->sm_count;
    return BL_OK;
}

}  // namespace

size_t chain_plan_bytes(int nsteps)
{
    if (nsteps < 1 || nsteps > kChainMaxStepsLimit)
        return 0;
    return plan_bytes(nsteps);
}

bool chain_step_fits(int64_t K) { return K % 256 == 0 && K >= 256 && K <= kChainMaxK; }

int build_chain_plan(int nsteps, const bitlinear_chain_step *desc, void *plan, cudaStream_t s)
{
    int G = 0;
    int st = chain_grid(&G);
    if (st)
        return st;
    std::vector<unsigned char> host(plan_bytes(nsteps), 0);
    auto *hdr = reinterpret_cast<ChainHeader *>(host.data());
    hdr->nsteps = nsteps;
    auto *steps = reinterpret_cast<ChainStep *>(host.data() + steps_offset());
    for (int i = 0; i < nsteps; ++i) {
        const bitlinear_chain_step &d = desc[i];
        ChainStep c{};
        c.count = d.count;
        c.gstart[0] = 0;
        for (int j = 0; j < d.count; ++j) {
            c.prob[j] = GemvProblem{d.packed[j], d.w_scale[j], d.N[j], d.y[j], d.N[j], d.acc_dbg[j]};
            c.gstart[j + 1] = c.gstart[j] + (d.N[j] + 7) / 8;
        }
        for (int j = d.count; j < kGemvMaxProblems; ++j)
            c.gstart[j + 1] = c.gstart[d.count];
        c.K = d.K;
        c.x = d.x;
        c.xt = d.xt;
        c.yt = d.yt;
        c.norm = d.gain != nullptr || d.norm != 0;
        c.gain = d.gain;
        c.gt = d.gt;
        c.eps = d.eps;
        // R: the smallest stage capacity (>= 4 groups when the stage has
        // room) that gives every CTA the same number of sets
        const int P = int(d.K / 256);
        const uint32_t slot = uint32_t(stage_pieces(P, kChainKC)) * 512;
        const int cap = int(kChainStageBytes / slot) < kMaxSet ? int(kChainStageBytes / slot) : kMaxSet;
        const int64_t total = c.gstart[d.count];
        if (total > int64_t(kMaxGroupsPerCta) * G)
            return BL_ERR_SHAPE;
        const int64_t lo = total / G, hi = lo + (total % G ? 1 : 0);
        int R = cap;
        for (int r = (cap < 4 ? cap : 4); r <= cap; ++r)
            if ((lo + r - 1) / r == (hi + r - 1) / r) {
                R = r;
                break;
            }
        c.set_cap = R;
        steps[i] = c;
    }
    // pageable source: the copy is staged before the call returns
    st = cuda_status(cudaMemcpyAsync(plan, host.data(), host.size(), cudaMemcpyHostToDevice, s));
    return st;
}

int launch_chain(const void *plan, int nsteps, cudaStream_t s, uint64_t limit_ns, int test_step)
{
    int G = 0;
    int st = chain_grid(&G);
    if (st)
        return st;
    auto *base = static_cast<unsigned char *>(const_cast<void *>(plan));
    auto *counters = reinterpret_cast<unsigned *>(base + counters_offset(nsteps));
    if ((st = cuda_status(cudaMemsetAsync(counters, 0, (size_t(nsteps) + 1) * 4, s))))
        return st;
    const DeviceInfo *di = device_info();
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(G));
    cfg.blockDim = dim3(kChainThreads);
    cfg.dynamicSmemBytes = kChainSmem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const ChainStep *steps = reinterpret_cast<const ChainStep *>(base + steps_offset());
    return cuda_status(cudaLaunchKernelEx(&cfg, gemv_chain_kernel, steps, nsteps, counters,
                                          counters + nsteps, di->status, limit_ns, test_step));
}

}  // namespace bl
