// gemv.cu -- ternary decode GEMV for 1 <= M <= 16 tokens with a per-warp
// weight ring.  One token with K a multiple of 256 runs the streaming kernel
// of gemv_stream.cu instead (launch_gemv_batch routes it there); this kernel
// takes the fused entry points' small batches (2..16 tokens) and single
// tokens whose K is not a multiple of 256.
//
// "How to Run BitNet Inference on GPU Using CUDA Kernels: A Complete Guide",
// sections "Understanding the Two-Phase Architecture" and "Key Components and
// Source Code Architecture": decode runs an INT8-activation x INT2-weight
// linear and is memory-bound.  "bit-floor" README, section "The core math":
// integer inner loop, floating point only in the final scale multiply.
//
// Design (B200): the weight stream N*K/4 bytes is the whole cost.
//   * One launch may carry up to kGemvMaxProblems GEMVs that share the same
//     activations x (the q/k/v or gate/up products of a decoder layer).  Their
//     8-row groups are concatenated into one list.
//   * Persistent grid of 512-thread CTAs: one per SM for small problems (so
//     that the next launch's CTA fits beside it and can start its weight
//     fetch early), two per SM for large ones.  Each CTA owns a contiguous
//     range of row groups (host-computed), taken in phases of at most
//     256 / M groups.  In a phase the 16 warps split the phase's 512-byte
//     pieces into 16 contiguous runs that cross row-group boundaries; lane l
//     of a warp always reads bytes 16l..16l+15 of a piece (row l%8, chunk
//     4p + l/8 of the TL layout).
//   * Weights stream through a per-warp ring of STAGES 512-byte slots in
//     shared memory filled by cp.async (16 bytes per lane, L1 bypassed); each
//     lane reads back only the bytes it copied, so no intra-warp sync is
//     needed.  The ring is primed before the kernel waits on the preceding
//     launch (programmatic dependent launch), so with BL_FLAG_PDL the weight
//     fetch of one BitLinear overlaps the tail of the previous one.
//   * The activations (int8, M*K bytes) sit in shared memory.  The fused
//     entry points quantise x in the prologue (absmax, scale, rint, row sum;
//     one register-resident pass for a single token).  Everything the
//     preceding launch may have written (x, or q, d and the row sums) is read
//     after the dependency wait with L2-coherent loads.
//   * Inner loop, stored codes s = code + 1 in {0,1,2}: for four consecutive
//     k, (word & 0x03030303), (word & 0x0c0c0c0c), (word & 0x30303030) and
//     (word & 0xc0c0c0c0) hold s, 4s, 16s, 64s per byte; dp4a (unsigned x
//     signed bytes) against four int8 activations into four accumulators
//     (two interleaved sets for one token) costs one LOP3 + one dp4a per four
//     weights.  For M >= 8 the codes are shifted down once and shared by all
//     tokens.  sum(code q) = sum(s q) - rowsum(q).
//   * At each row-group boundary a warp folds its partial sums into shared
//     accumulators (warp shuffles + shared atomics); after the phase barrier
//     y = ((float)acc * d_m) * gamma_eff is written, bf16 or fp32.
#include "bl_common.cuh"

namespace bl {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;

// Bytes of the weight ring: STAGES 512-byte slots per warp.
template <int STAGES>
constexpr int ring_bytes() { return kWarps * STAGES * 512; }

enum { MODE_Q = 0, MODE_X_BF16 = 1, MODE_X_F32 = 2 };

struct Params {
    GemvProblem prob[kGemvMaxProblems];
    int64_t gstart[kGemvMaxProblems + 1];  // prefix sums of the problems' row groups
    int count;
    int64_t K;
    int M;
    const int8_t *q;
    const float *d;
    const int32_t *rowsum;
    const void *x;
    int64_t ldx;
    int yt;
    // CTA b owns row groups [b*gpc_base + min(b, gpc_rem), ...), gpc_base (+1) of them
    int64_t gpc_base;
    int gpc_rem;
};

// Row groups whose partial sums a CTA holds at once (8 KB of int32 sums).
template <int MT>
constexpr int groups_per_phase() { return 256 / MT; }

template <int MT>
struct Smem {
    float bmax[kWarps][MT];
    int bsum[kWarps][MT];
    float scale[MT];
    float d[MT];
    int r[MT];
    float wscale[kGemvMaxProblems];   // each problem's gamma_eff, read before the dependency wait
    int sacc[groups_per_phase<MT>()][MT][8];
    // followed by the weight ring and the int8 activations (M*K)
};

template <int MT>
constexpr size_t smem_header()
{
    return (sizeof(Smem<MT>) + 127) / 128 * 128;
}

__device__ __forceinline__ void cp_async16(uint32_t saddr, const void *g)
{
    asm volatile("cp.async.cg.shared.global.L2::256B [%0], [%1], 16;" ::"r"(saddr), "l"(g)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }


__device__ __forceinline__ void pdl_launch_dependents()
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Problem and local row group of concatenated row group G.
__device__ __forceinline__ int locate(const Params &p, int64_t G, int64_t &g_local)
{
    int pi = 0;
#pragma unroll
    for (int i = 1; i < kGemvMaxProblems; ++i)
        if (i < p.count && G >= p.gstart[i])
            pi = i;
    g_local = G - p.gstart[pi];
    return pi;
}

// Quantise the M tokens of x into shared memory (block-cooperative).
// One token whose K/8 eight-element chunks fit two per thread: x is read once
// into registers, one block reduction gives the absmax, the quantised values
// go to shared memory and each warp leaves its partial row sum in bsum (the
// epilogue adds them up), so the prologue needs a single barrier.
template <int MT, int XT>
__device__ __forceinline__ void quantize_prologue_1(const Params &p, Smem<MT> &sm, int8_t *qs)
{
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int chunks = int(p.K / 8);
    float f[2][8];
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int c = tid + i * kThreads;
        if (c < chunks) {
            load8<XT, true>(p.x, int64_t(c) * 8, f[i]);
#pragma unroll
            for (int j = 0; j < 8; ++j)
                amax = fmaxf(amax, fabsf(f[i][j]));
        }
    }
    // per-thread maxima are finite and >= 0 (fmaxf from 0 drops NaN), so
    // their bit patterns order like the values: one redux per warp
    const uint32_t wmax = __reduce_max_sync(0xffffffffu, __float_as_uint(amax));
    if (lane == 0)
        sm.bmax[warp][0] = __uint_as_float(wmax);
    __syncthreads();
    static_assert(MT == 1 && kWarps % 4 == 0, "bmax of one token is kWarps contiguous floats");
    float a = 0.0f;
#pragma unroll
    for (int w = 0; w < kWarps; w += 4) {
        const float4 b4 = *reinterpret_cast<const float4 *>(&sm.bmax[w][0]);
        a = fmaxf(fmaxf(a, b4.x), fmaxf(b4.y, fmaxf(b4.z, b4.w)));
    }
    const float a_eff = fmaxf(a, kEps);
    const float s = __fdiv_rn(kQb, a_eff);
    if (tid == 0)
        sm.d[0] = __fdiv_rn(a_eff, kQb);
    int sum = 0;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int c = tid + i * kThreads;
        if (c < chunks) {
            uint32_t lo = 0, hi = 0;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int t0 = quant1(f[i][j], s), t1 = quant1(f[i][j + 4], s);
                sum += t0 + t1;
                lo |= (uint32_t(t0) & 0xffu) << (8 * j);
                hi |= (uint32_t(t1) & 0xffu) << (8 * j);
            }
            *reinterpret_cast<uint2 *>(qs + int64_t(c) * 8) = make_uint2(lo, hi);
        }
    }
    sum = __reduce_add_sync(0xffffffffu, sum);
    if (lane == 0)
        sm.bsum[warp][0] = sum;
    // the barrier before the main loop publishes qs, d and bsum
}

template <int MT, int XT>
__device__ __forceinline__ void quantize_prologue(const Params &p, Smem<MT> &sm, int8_t *qs)
{
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t chunks = p.K / 8;
    float pmax[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) {
        pmax[m] = 0.0f;
        if (m < p.M)
            for (int64_t c = tid; c < chunks; c += kThreads) {
                float f[8];
                load8<XT, true>(p.x, m * p.ldx + c * 8, f);
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    pmax[m] = fmaxf(pmax[m], fabsf(f[j]));
            }
    }
#pragma unroll
    for (int m = 0; m < MT; ++m) {
        float v = warp_max(pmax[m]);
        if (lane == 0)
            sm.bmax[warp][m] = v;
    }
    __syncthreads();
    if (tid < p.M) {
        float a = 0.0f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w)
            a = fmaxf(a, sm.bmax[w][tid]);
        const float a_eff = fmaxf(a, kEps);
        sm.scale[tid] = __fdiv_rn(kQb, a_eff);
        sm.d[tid] = __fdiv_rn(a_eff, kQb);
    }
    __syncthreads();
    int psum[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) {
        psum[m] = 0;
        if (m < p.M) {
            const float s = sm.scale[m];
            for (int64_t c = tid; c < chunks; c += kThreads) {
                float f[8];
                load8<XT, true>(p.x, m * p.ldx + c * 8, f);
                uint32_t lo = 0, hi = 0;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int t0 = quant1(f[j], s), t1 = quant1(f[j + 4], s);
                    psum[m] += t0 + t1;
                    lo |= (uint32_t(t0) & 0xffu) << (8 * j);
                    hi |= (uint32_t(t1) & 0xffu) << (8 * j);
                }
                *reinterpret_cast<uint2 *>(qs + m * p.K + c * 8) = make_uint2(lo, hi);
            }
        }
    }
#pragma unroll
    for (int m = 0; m < MT; ++m) {
        int v = warp_sum(psum[m]);
        if (lane == 0)
            sm.bsum[warp][m] = v;
    }
    __syncthreads();
    if (tid < p.M) {
        int r = 0;
#pragma unroll
        for (int w = 0; w < kWarps; ++w)
            r += sm.bsum[w][tid];
        sm.r[tid] = r;
    }
    __syncthreads();
}

template <int MT>
__device__ __forceinline__ void copy_prologue(const Params &p, Smem<MT> &sm, int8_t *qs)
{
    const int64_t vecs = int64_t(p.M) * p.K / 16;
    for (int64_t i = threadIdx.x; i < vecs; i += kThreads)
        reinterpret_cast<uint4 *>(qs)[i] = ld_dep_v4(p.q + i * 16);
    if (threadIdx.x < p.M) {
        sm.d[threadIdx.x] = __uint_as_float(ld_dep_u32(p.d + threadIdx.x));
        sm.r[threadIdx.x] = int(ld_dep_u32(p.rowsum + threadIdx.x));
    }
    // the epilogue reads row sums as the sum over warps of bsum
    for (int i = threadIdx.x; i < kWarps * MT; i += kThreads) {
        const int w = i / MT, m = i % MT;
        sm.bsum[w][m] = (w == 0 && m < p.M) ? int(ld_dep_u32(p.rowsum + m)) : 0;
    }
    __syncthreads();
}

// Work of one CTA: the row groups [g_begin, g_end), taken in phases of at
// most groups_per_phase<MT>() groups.  In a phase the 16 warps split the
// phase's 512-byte pieces into 16 contiguous runs; a warp streams its run
// through its cp.async ring, crossing row-group boundaries, and at each
// boundary (and at the end of its run) adds its partial row sums into the
// phase's shared accumulators.  After a barrier the phase's rows are rescaled
// and written.  The first ring fill is issued before the kernel waits on the
// preceding launch, so the weight stream starts at once.
template <int MT, int MODE, bool FULL, int STAGES>
__global__ void __launch_bounds__(kThreads, 2) gemv_kernel(const Params p)
{
    extern __shared__ __align__(128) unsigned char smem_raw[];
    Smem<MT> &sm = *reinterpret_cast<Smem<MT> *>(smem_raw);
    const uint32_t ring0 = static_cast<uint32_t>(__cvta_generic_to_shared(smem_raw + smem_header<MT>()));
    int8_t *qs = reinterpret_cast<int8_t *>(smem_raw + smem_header<MT>() + ring_bytes<STAGES>());
    const uint32_t qs_addr = static_cast<uint32_t>(__cvta_generic_to_shared(qs));
    constexpr bool kMask = MT <= 4;
    // two interleaved accumulator sets (even / odd words) halve the dp4a
    // dependency chains when there are few tokens
    constexpr int kSets = MT == 1 ? 2 : 1;
    constexpr int kAcc = kMask ? 4 * kSets : 1;
    constexpr int GP = groups_per_phase<MT>();

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int Ki = int(p.K);
    const int C = Ki / 64, P = (C + 3) / 4;
    const int64_t slab = int64_t(C) * 128;
    const int csub = lane >> 3;
    const int bx = blockIdx.x;
    const int64_t g_begin = bx * p.gpc_base + (bx < p.gpc_rem ? bx : p.gpc_rem);
    const int64_t g_end = g_begin + p.gpc_base + (bx < p.gpc_rem ? 1 : 0);
    const uint32_t ring = ring0 + uint32_t(warp) * (STAGES * 512) + lane * 16;

    auto group_ptr = [&](int64_t G) -> const uint8_t * {
        int64_t gl;
        const int pi = locate(p, G, gl);
        return p.prob[pi].packed + gl * slab + lane * 16;
    };

    // this lane's slot 0 of its warp's ring, as a generic pointer for the
    // loads (slot offsets then become immediates) and as a shared address for
    // cp.async
    const unsigned char *ring_g = smem_raw + smem_header<MT>() + warp * (STAGES * 512) + lane * 16;

    // issue cursor (runs STAGES pieces ahead of the math)
    int64_t i_group = 0;
    int i_j = 0, i_left = 0, i_rem = 0;
    const uint8_t *i_ptr = nullptr;
    // With K % 256 == 0 (FULL) a problem's pieces are one contiguous byte
    // stream, so the cursor only jumps when it moves on to the next problem.
    int i_prob = 0;
    int64_t i_to_jump = 0;
    auto issue = [&](int slot) {
        if (i_rem > 0) {
            if constexpr (FULL) {
                cp_async16(ring + slot * 512, i_ptr);
                i_ptr += 512;
                --i_rem;
                if (--i_to_jump == 0 && i_rem > 0) {
                    ++i_prob;
                    i_ptr = p.prob[i_prob].packed + lane * 16;
                    i_to_jump = (p.gstart[i_prob + 1] - p.gstart[i_prob]) * P;
                }
            } else {
                if (4 * i_j + csub < C)
                    cp_async16(ring + slot * 512, i_ptr);
                --i_rem;
                ++i_j;
                i_ptr += 512;
                if (--i_left == 0) {
                    ++i_group;
                    i_left = P;
                    i_j = 0;
                    if (i_rem > 0)
                        i_ptr = group_ptr(i_group);
                }
            }
        }
        cp_async_commit();
    };
    int acc[MT][kAcc];
    // end of a row group, or of this warp's run: fold into the shared sums
    auto flush = [&](int gi) {
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            int t;
            if constexpr (kMask) {
                t = 0;
#pragma unroll
                for (int b = 0; b < 4 * kSets; b += 4)
                    t += acc[m][b] + (acc[m][b + 1] >> 2) + (acc[m][b + 2] >> 4) +
                         (acc[m][b + 3] >> 6);
            } else {
                t = acc[m][0];
            }
#pragma unroll
            for (int a = 0; a < kAcc; ++a)
                acc[m][a] = 0;
            t += __shfl_xor_sync(0xffffffffu, t, 8);
            t += __shfl_xor_sync(0xffffffffu, t, 16);
            if (lane < 8 && m < p.M)
                atomicAdd(&sm.sacc[gi][m][lane], t);
        }
    };

    bool first = true;
    for (int64_t ph0 = g_begin; ph0 < g_end; ph0 += GP) {
        const int64_t ph1 = ph0 + GP < g_end ? ph0 + GP : g_end;
        const int nG = int(ph1 - ph0);
        const int64_t TP = int64_t(nG) * P;
        // kWarps is a power of two: the split needs no division
        const int wb = int((int64_t(warp) * TP) >> 4);
        const int n = int((int64_t(warp + 1) * TP) >> 4) - wb;
        const int gi0 = wb / P, j0 = wb - gi0 * P;
        static_assert(kWarps == 16, "the run split above assumes 16 warps");

        i_group = ph0 + gi0;
        i_j = j0;
        i_left = P - j0;
        i_rem = n;
        i_ptr = n > 0 ? group_ptr(i_group) + int64_t(j0) * 512 : nullptr;
        if constexpr (FULL) {
            int64_t gl;
            i_prob = locate(p, i_group, gl);
            i_to_jump = (p.gstart[i_prob + 1] - i_group) * P - j0;
        }
        if (first) {
            pdl_launch_dependents();
            // independent of the preceding launch: weight scales, accumulators
#pragma unroll
            for (int i = 0; i < kGemvMaxProblems; ++i)
                if (tid == i && i < p.count)
                    sm.wscale[i] = __ldg(p.prob[i].w_scale);
            for (int i = tid; i < nG * MT * 8; i += kThreads)
                (&sm.sacc[0][0][0])[i] = 0;
        }
#pragma unroll
        for (int s = 0; s < STAGES; ++s)
            issue(s);
        if (first) {
            // everything below may read what the preceding launch wrote
            pdl_wait();
            if constexpr (MODE == MODE_Q)
                copy_prologue<MT>(p, sm, qs);
            else if constexpr (MT == 1) {
                if (p.K <= int64_t(16) * kThreads)
                    quantize_prologue_1<MT, MODE == MODE_X_BF16 ? BL_BF16 : BL_F32>(p, sm, qs);
                else
                    quantize_prologue<MT, MODE == MODE_X_BF16 ? BL_BF16 : BL_F32>(p, sm, qs);
            } else {
                quantize_prologue<MT, MODE == MODE_X_BF16 ? BL_BF16 : BL_F32>(p, sm, qs);
            }
        } else {
            for (int i = tid; i < nG * MT * 8; i += kThreads)
                (&sm.sacc[0][0][0])[i] = 0;
        }
        __syncthreads();
        if (first) {
            // the activations' row sums, folded once for the epilogues
            if (tid < MT) {
                int r = 0;
#pragma unroll
                for (int w = 0; w < kWarps; ++w)
                    r += sm.bsum[w][tid];
                sm.r[tid] = r;
            }
            first = false;
        }

#pragma unroll
        for (int m = 0; m < MT; ++m)
#pragma unroll
            for (int a = 0; a < kAcc; ++a)
                acc[m][a] = 0;
        // multiply one 16-byte piece (wv, this lane's 64 k of one row) into
        // the accumulators against the activations at qp
        auto mac = [&](const uint4 wv, const int8_t *qp) {
                const uint32_t wd[4] = {wv.x, wv.y, wv.z, wv.w};
                if constexpr (kMask) {
#pragma unroll
                    for (int m = 0; m < MT; ++m) {
                        if (m >= p.M)
                            break;
                        const uint4 *q4p = reinterpret_cast<const uint4 *>(qp + m * Ki);
#pragma unroll
                        for (int w = 0; w < 4; ++w) {
                            const uint4 q4 = q4p[w];
                            const int b = 4 * (w % kSets);
                            acc[m][b + 0] = dp4a_us(wd[w] & 0x03030303u, q4.x, acc[m][b + 0]);
                            acc[m][b + 1] = dp4a_us(wd[w] & 0x0c0c0c0cu, q4.y, acc[m][b + 1]);
                            acc[m][b + 2] = dp4a_us(wd[w] & 0x30303030u, q4.z, acc[m][b + 2]);
                            acc[m][b + 3] = dp4a_us(wd[w] & 0xc0c0c0c0u, q4.w, acc[m][b + 3]);
                        }
                    }
                } else {
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        const uint32_t c0 = wd[w] & 0x03030303u;
                        const uint32_t c1 = (wd[w] >> 2) & 0x03030303u;
                        const uint32_t c2 = (wd[w] >> 4) & 0x03030303u;
                        const uint32_t c3 = (wd[w] >> 6) & 0x03030303u;
#pragma unroll
                        for (int m = 0; m < MT; ++m) {
                            if (m >= p.M)
                                break;
                            const uint4 q4 = reinterpret_cast<const uint4 *>(qp + m * Ki)[w];
                            int a = acc[m][0];
                            a = dp4a_us(c0, q4.x, a);
                            a = dp4a_us(c1, q4.y, a);
                            a = dp4a_us(c2, q4.z, a);
                            a = dp4a_us(c3, q4.w, a);
                            acc[m][0] = a;
                        }
                    }
                }
                    };

        int c_gi = gi0, c_j = j0, c_left = P - j0;
        const int8_t *qp = qs + j0 * 256 + csub * 64;
        for (int k0 = 0; k0 < n; k0 += STAGES) {
#pragma unroll
            for (int u = 0; u < STAGES; ++u) {
                if (k0 + u >= n)
                    break;
                cp_async_wait<STAGES - 1>();
                const uint4 wv = *reinterpret_cast<const uint4 *>(ring_g + u * 512);
                if (FULL || 4 * c_j + csub < C)
                    mac(wv, qp);
                // the slot's data has been consumed: refill it
                issue(u);
                qp += 256;
                if constexpr (!FULL)
                    ++c_j;
                if (--c_left == 0) {
                    flush(c_gi);
                    ++c_gi;
                    c_left = P;
                    c_j = 0;
                    qp = qs + csub * 64;
                }
            }
        }
        if (n > 0 && c_left != P)
            flush(c_gi);  // the run ended inside a group
        cp_async_wait<0>();
        __syncthreads();
        // rescale and write the phase's rows
        for (int idx = tid; idx < nG * 8 * p.M; idx += kThreads) {
            int gi, m, rr;
            if constexpr (MT == 1) {
                gi = idx >> 3;
                m = 0;
                rr = idx & 7;
            } else {
                gi = idx / (8 * p.M);
                const int rem = idx % (8 * p.M);
                m = rem >> 3;
                rr = rem & 7;
            }
            int64_t gl;
            const int pi = locate(p, ph0 + gi, gl);
            const GemvProblem &pr = p.prob[pi];
            const int64_t row = gl * 8 + rr;
            if (row < pr.N) {
                const int a = sm.sacc[gi][m][rr] - sm.r[m];
                if (pr.acc_dbg)
                    pr.acc_dbg[int64_t(m) * pr.N + row] = a;
                store_y(pr.y, p.yt, int64_t(m) * pr.ldy + row, rescale1(a, sm.d[m], sm.wscale[pi]));
            }
        }
        __syncthreads();
    }
    if (first) {
        // a CTA with no rows still honours the launch order
        pdl_launch_dependents();
        pdl_wait();
    }
}


template <int MT, int MODE>
int launch_one(const Params &base, unsigned flags, cudaStream_t s)
{
    const DeviceInfo *di = device_info();
    if (!di)
        return BL_ERR_CUDA;
    const bool full = (base.K / 64) % 4 == 0;
    const size_t act = size_t(base.M) * size_t(base.K);
    // a deep ring while two CTAs (this launch and the next one) still fit on
    // an SM, a shallow one for large activation tiles
    const bool deep = smem_header<MT>() + ring_bytes<8>() + act <= 100 * 1024;
    const size_t smem = smem_header<MT>() + (deep ? ring_bytes<8>() : ring_bytes<4>()) + act;
    if (smem > size_t(di->max_smem_optin))
        return BL_ERR_SHAPE;
    auto kern = deep ? (full ? gemv_kernel<MT, MODE, true, 8> : gemv_kernel<MT, MODE, false, 8>)
                     : (full ? gemv_kernel<MT, MODE, true, 4> : gemv_kernel<MT, MODE, false, 4>);
    int per_sm = 0;
    int st = occupancy(reinterpret_cast<const void *>(kern), kThreads, smem, &per_sm);
    if (st)
        return st;
    if (per_sm < 1)
        return BL_ERR_SHAPE;
    // one persistent CTA per SM (a second slot stays free for the next launch)
    const int64_t NGt = base.gstart[base.count];
    // large problems: up to two CTAs per SM for more warps in flight; small
    // ones keep one so that the next launch's CTA fits beside it
    const int64_t per = NGt >= 4 * int64_t(di->sm_count) && per_sm >= 2 ? 2 : 1;
    const int64_t cap = int64_t(di->sm_count) * per;
    const unsigned grid = unsigned(NGt < cap ? NGt : cap);
    Params pp = base;
    pp.gpc_base = NGt / grid;
    pp.gpc_rem = int(NGt % grid);

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
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

template <int MODE>
int dispatch_m(const Params &p, unsigned flags, cudaStream_t s)
{
    if (p.M <= 1)
        return launch_one<1, MODE>(p, flags, s);
    if (p.M <= 2)
        return launch_one<2, MODE>(p, flags, s);
    if (p.M <= 4)
        return launch_one<4, MODE>(p, flags, s);
    if (p.M <= 8)
        return launch_one<8, MODE>(p, flags, s);
    return launch_one<16, MODE>(p, flags, s);
}

}  // namespace

int launch_gemv_stream(const GemvBatch &b, bool fused, cudaStream_t s);
bool gemv_stream_applies(const GemvBatch &b, int sm_count);

// 2 .. 16 tokens: the tensor-core kernel or the dp4a multi-token kernel.
// The dp4a kernel's cost grows with the tokens x weights it multiplies and
// with K (each warp quantises whole token rows); the tensor-core kernel's is
// nearly flat in M but carries ~2 us more fixed latency (cluster exchange,
// MMA commit, tensor memory).  Measured crossover on the 2.4B shapes: the
// tensor cores from M N K >= 48 Mi, or for K above 4096.
bool small_batch_prefers_tensor(const GemvBatch &b)
{
    int64_t nk = 0;
    for (int i = 0; i < b.count; ++i)
        nk += b.prob[i].N * b.K;
    return b.M * nk >= (int64_t(48) << 20) || b.K > 4096;
}

bool small_batch_tensor(const GemvBatch &b, bool fused, int *cluster)
{
    *cluster = 0;
    if (b.flags & BL_FLAG_SMALL_BATCH_DP4A)
        return false;
    if (!(b.flags & BL_FLAG_SMALL_BATCH_TENSOR) && !small_batch_prefers_tensor(b))
        return false;
    *cluster = gemv_tc_cluster(b, fused);
    return *cluster > 0;
}

int plan_gemv_batch(const GemvBatch &b, bool fused, int *cluster)
{
    *cluster = 0;
    const DeviceInfo *di = device_info();
    if (!di)
        return -1;
    if (gemv_stream_applies(b, di->sm_count))
        return BL_GEMV_KERNEL_STREAM;
    if (small_batch_tensor(b, fused, cluster))
        return BL_GEMV_KERNEL_TENSOR;
    if (gemv_stream_mt_applies(b, fused, di->sm_count, di->max_smem_optin))
        return BL_GEMV_KERNEL_STREAM_MT;
    return BL_GEMV_KERNEL_DP4A;
}

int launch_gemv_batch(const GemvBatch &b, bool fused, cudaStream_t s)
{
    const DeviceInfo *di = device_info();
    if (!di)
        return BL_ERR_CUDA;
    // one token on a large layer: the producer/consumer streaming kernel;
    // 2 .. 16 tokens: the tensor-core kernel or the multi-token streaming
    // kernel (one weight pass for all tokens), as small_batch_tensor picks
    if (gemv_stream_applies(b, di->sm_count))
        return launch_gemv_stream(b, fused, s);
    int cluster = 0;
    if (small_batch_tensor(b, fused, &cluster))
        return launch_gemv_tc(b, fused, s);
    if (gemv_stream_mt_applies(b, fused, di->sm_count, di->max_smem_optin))
        return launch_gemv_stream_mt(b, fused, s);
    Params p{};
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
    if (!fused)
        return dispatch_m<MODE_Q>(p, b.flags, s);
    if (b.xt == BL_BF16)
        return dispatch_m<MODE_X_BF16>(p, b.flags, s);
    return dispatch_m<MODE_X_F32>(p, b.flags, s);
}

int launch_gemv(const GemvArgs &a, bool fused, cudaStream_t s)
{
    GemvBatch b{};
    b.count = 1;
    b.prob[0] = GemvProblem{a.packed, a.w_scale, a.N, a.y, a.ldy, a.acc_dbg};
    b.K = a.K;
    b.M = a.M;
    b.q = a.q;
    b.d = a.d;
    b.rowsum = a.rowsum;
    b.x = a.x;
    b.xt = a.xt;
    b.ldx = a.ldx;
    b.yt = a.yt;
    b.flags = 0;
    return launch_gemv_batch(b, fused, s);
}

}  // namespace bl
