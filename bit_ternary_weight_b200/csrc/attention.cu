// attention.cu -- decode attention of one token over a bf16 KV cache, for the
// synthetic decoder-layer stack around the BitLinear products.
//
// "How to Run BitNet Inference on GPU Using CUDA Kernels: A Complete Guide",
// section "Understanding the Two-Phase Architecture" (the decode phase runs
// Attention with a KV cache of shape (1, seq_len, kv_heads, 1, head_dim));
// "bit-floor" README, section "What's inside" (rope.rs: RoPE on queries and
// keys before attention; attention.cu: attention with a softmax over the
// cached positions).  Readings (identical on the CPU oracle):
//   RoPE       pairs (2i, 2i + 1) of a head turned by pos * base^(-2i / D):
//              the angle, its cosine and sine in fp64, rounded to fp32; the
//              rotation (a c - b s, a s + b c) in fp32 operations in that
//              order; rotated q and k rounded to bf16 (k goes to the cache).
//   scores     s_j = (float)(sum_d q[d] K[j][d]) * (float)(1 / sqrt(D)), the
//              dot product of bf16 values in fp64 (every product exact).
//   softmax    m = max_j s_j; weights e_j = exp(s_j - m), their sum S and
//              out[d] = bf16((float)((sum_j e_j V[j][d]) / S)) all in fp64.
// The kernel evaluates the softmax per block of positions against the
// block's own maximum m_b and combines the blocks with the factors
// exp(m_b - m); with every softmax quantity in fp64 this grouping, the fp64
// sums' order, and the difference between CUDA's fp64 exp, cos, sin and pow
// and the C library's, change the fp32 results only when a value lies within
// about 1e-15 (relative) of an fp32 rounding boundary.
//
// RoPE's cosines and sines come from a table of every (position, pair) that
// bitlinear_rope_table computes once (same definition), or are computed in
// the kernel when no table is given.
//
// Design: one launch of CTAs (kv head, block of 64 cached positions), so that
// one token's attention spreads over many SMs; the position pos is a device
// scalar read after the dependency wait, so a CUDA graph can replay the call
// for successive tokens (the grid covers the whole cache; blocks beyond pos
// return at once).  A CTA:
//   * brings its block's cached keys and values (positions below pos) into
//     shared memory with two bulk copies as soon as pos is known;
//   * meanwhile rotates the queries of the kv head's query heads and, in the
//     block holding pos, the new key, which it appends with the new value;
//   * scores its positions (eight lanes per position, sixteen dimensions each,
//     fp64 partial dot products for every query head, in four independent
//     partial sums), takes the block maximum, the fp64 weights, their sum and
//     the fp64 weighted values (lanes over dimensions, eight position groups),
//     and writes them to the workspace;
//   * arrives on the kv head's ticket (fence, atomic add); the last CTA to
//     arrive combines the blocks in block order (the blocks' partial values
//     of its outputs loaded first, overlapping the round trip for the block
//     maxima and sums), divides, rounds and stores, and resets the ticket.
// 256 threads: the fp64 phases are bound by latency (fp64 runs at half the
// fp32 rate here), so each SM sub-partition needs two warps; the queries are
// kept as fp64 in shared memory (one conversion each, not one per position).
// A position outside the cache records BL_ERR_SHAPE in the device status word
// and writes nothing; a bulk copy that does not land in 2 s records
// BL_ERR_TIMEOUT and that CTA leaves without output (the workspace's ticket
// must then be zeroed again).
#include "bl_common.cuh"

namespace bl {
namespace {

constexpr int kHeadDim = 128;
constexpr int kPosBlock = 64;             // cached positions per CTA
constexpr int kAttnThreads = 256;
constexpr int kAttnWarps = kAttnThreads / 32;
constexpr int kMaxGroup = 8;              // query heads per kv head
constexpr uint32_t kRowBytes = kHeadDim * 2;

struct AttnParams {
    const __nv_bfloat16 *q, *k, *v;       // [H*D], [Hkv*D], [Hkv*D]
    __nv_bfloat16 *cache_k, *cache_v;     // [Hkv][T_max][D]
    const int32_t *pos;
    int H, Hkv, T_max, nblk;
    double rope_base;
    const float2 *rope;                   // NULL, or (cos, sin) [T_max][D/2]
    __nv_bfloat16 *out;                   // [H*D]
    // workspace
    float *bmax;                          // [H][nblk] block maxima
    double *bsum;                         // [H][nblk] block sums of exp(s - m_b)
    double *bnum;                         // [H][nblk][D] block sums of exp(s - m_b) V
    unsigned *ticket;                     // [Hkv], zero between calls
    int *status;
};

struct AttnSmem {
    uint64_t bar;
    int abort_flag;
    int last;
    float2 cs[kHeadDim / 2];               // (cos, sin) of the token's angles
    // rotated queries of the group (bf16 values, as fp64): dimension 16 c + e
    // at [17 c + e], so the eight lanes of a position (one chunk c each) read
    // different banks
    double qs[kMaxGroup][kHeadDim / 16 * 17];
    float ks[kHeadDim];                    // rotated new key (block holding pos)
    float vs[kHeadDim];                    // new value
    float sc[kMaxGroup][kPosBlock];        // scores
    float mb[kMaxGroup];                   // block maxima
    double ew[kMaxGroup][kPosBlock];       // weights exp(s - m_b)
    double part[kAttnWarps][kMaxGroup][kHeadDim];   // per position group weighted values
    alignas(128) __nv_bfloat16 kb[kPosBlock][kHeadDim];   // the block's cached keys
    alignas(128) __nv_bfloat16 vb[kPosBlock][kHeadDim];   // ... and values
};

__device__ __forceinline__ float bf16_bits_f32(uint32_t b) { return __uint_as_float(b << 16); }

__device__ __forceinline__ uint32_t f32_bf16_bits(float v)
{
    return __bfloat16_as_ushort(__float2bfloat16_rn(v));
}

// cos and sin of the angle pos * base^(-2i / D), each computed in fp64 and
// rounded to fp32.
__device__ __forceinline__ float2 rope_angle(int pos, int i, double base)
{
    const double ang = double(pos) * pow(base, -double(2 * i) / double(kHeadDim));
    return make_float2(__double2float_rn(cos(ang)), __double2float_rn(sin(ang)));
}

// Rotate the pair (a, b) (one 32-bit word of two bf16 values, a in the low
// half) by (cos, sin) cs; the two rotated values rounded to bf16 (as fp32).
__device__ __forceinline__ void rope_pair(uint32_t ab, float2 cs, float &o0, float &o1)
{
    const float c = cs.x, s = cs.y;
    const float a = __uint_as_float(ab << 16), b = __uint_as_float(ab & 0xffff0000u);
    const float r0 = __fsub_rn(__fmul_rn(a, c), __fmul_rn(b, s));
    const float r1 = __fadd_rn(__fmul_rn(a, s), __fmul_rn(b, c));
    o0 = bf16_bits_f32(f32_bf16_bits(r0));
    o1 = bf16_bits_f32(f32_bf16_bits(r1));
}

__device__ __forceinline__ void bf16x8(const uint4 v, float *f)
{
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        f[2 * e] = __uint_as_float(w[e] << 16);
        f[2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
    }
}

// GT: the query heads per kv head when known at compile time (1, 2, 4, 8),
// so that the per-head loops unroll without a runtime bound; 0: any.
template <int GT>
__global__ void __launch_bounds__(kAttnThreads) attention_decode_kernel(const AttnParams p)
{
    extern __shared__ __align__(128) unsigned char attn_raw[];
    AttnSmem &sm = *reinterpret_cast<AttnSmem *>(attn_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int kv = blockIdx.x, blk = blockIdx.y;
    const int G = GT > 0 ? GT : p.H / p.Hkv;
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int pos = int(ld_dep_u32(p.pos));
    if (pos < 0 || pos >= p.T_max) {
        if (tid == 0 && kv == 0 && blk == 0)
            atomicExch(p.status, BL_ERR_SHAPE);
        return;
    }
    const int j0 = blk * kPosBlock;
    if (j0 > pos)
        return;
    const int j1 = min(j0 + kPosBlock, pos + 1);
    const int n = j1 - j0;                            // positions of this block
    const int nk = min(j1, pos) - j0;                 // of them in the cache already
    const size_t head_base = size_t(kv) * p.T_max * kHeadDim;
    if (tid == 0) {
        sm.abort_flag = 0;
        mbar_init(smem_u32(&sm.bar), 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        if (nk > 0) {
            const uint32_t bytes = uint32_t(nk) * kRowBytes;
            mbar_arrive_tx(smem_u32(&sm.bar), 2 * bytes);
            bulk_load(smem_u32(&sm.kb[0][0]), p.cache_k + head_base + size_t(j0) * kHeadDim, bytes, smem_u32(&sm.bar));
            bulk_load(smem_u32(&sm.vb[0][0]), p.cache_v + head_base + size_t(j0) * kHeadDim, bytes, smem_u32(&sm.bar));
        } else {
            mbar_arrive(smem_u32(&sm.bar));
        }
    }
    // this thread's query pairs (and the new key and value pair), loaded
    // together before any is used (they come from the preceding launch: L2)
    constexpr int kPairsPerThread = kMaxGroup * (kHeadDim / 2) / kAttnThreads;
    uint32_t qw[kPairsPerThread];
#pragma unroll
    for (int u = 0; u < kPairsPerThread; ++u) {
        const int t = tid + u * kAttnThreads;
        qw[u] = t < G * (kHeadDim / 2)
                    ? __ldcg(reinterpret_cast<const unsigned *>(p.q + (kv * G) * kHeadDim) + t)
                    : 0u;
    }
    const bool has_new = nk < n;
    uint32_t kw = 0, vw = 0;
    if (has_new && tid < kHeadDim / 2) {
        kw = __ldcg(reinterpret_cast<const unsigned *>(p.k + kv * kHeadDim) + tid);
        vw = __ldcg(reinterpret_cast<const unsigned *>(p.v + kv * kHeadDim) + tid);
    }
    if (tid < kHeadDim / 2)
        sm.cs[tid] = p.rope ? __ldg(p.rope + size_t(pos) * (kHeadDim / 2) + tid) : rope_angle(pos, tid, p.rope_base);
    __syncthreads();
#pragma unroll
    for (int u = 0; u < kPairsPerThread; ++u) {
        const int t = tid + u * kAttnThreads;
        if (t < G * (kHeadDim / 2)) {
            const int g = t / (kHeadDim / 2), i = t % (kHeadDim / 2);
            float a, b;
            rope_pair(qw[u], sm.cs[i], a, b);
            sm.qs[g][(2 * i) / 16 * 17 + (2 * i) % 16] = double(a);
            sm.qs[g][(2 * i) / 16 * 17 + (2 * i) % 16 + 1] = double(b);
        }
    }
    if (has_new && tid < kHeadDim / 2) {
        // the block holding pos: rotate the new key, append key and value
        float a, b;
        rope_pair(kw, sm.cs[tid], a, b);
        sm.ks[2 * tid] = a;
        sm.ks[2 * tid + 1] = b;
        const float v0 = __uint_as_float(vw << 16);
        const float v1 = __uint_as_float(vw & 0xffff0000u);
        sm.vs[2 * tid] = v0;
        sm.vs[2 * tid + 1] = v1;
        p.cache_k[head_base + size_t(pos) * kHeadDim + 2 * tid] = __float2bfloat16_rn(a);
        p.cache_k[head_base + size_t(pos) * kHeadDim + 2 * tid + 1] = __float2bfloat16_rn(b);
        p.cache_v[head_base + size_t(pos) * kHeadDim + 2 * tid] = __float2bfloat16_rn(v0);
        p.cache_v[head_base + size_t(pos) * kHeadDim + 2 * tid + 1] = __float2bfloat16_rn(v1);
    }
    __syncthreads();
    if (!mbar_wait(smem_u32(&sm.bar), 0, &sm.abort_flag, p.status))
        return;     // BL_ERR_TIMEOUT recorded; no output from this CTA

    // ---- scores: eight lanes per position, sixteen dims each
    const float scale = __double2float_rn(1.0 / sqrt(double(kHeadDim)));
    const int sub = lane & 7, r = lane >> 3;
    for (int jb = warp * 4; jb < n; jb += 4 * kAttnWarps) {
        const int jj = jb + r;
        float kf[16];
        if (jj < nk) {
            const uint4 *kr = reinterpret_cast<const uint4 *>(&sm.kb[jj][sub * 16]);
            bf16x8(kr[0], kf);
            bf16x8(kr[1], kf + 8);
        } else {
#pragma unroll
            for (int e = 0; e < 16; ++e)
                kf[e] = jj < n ? sm.ks[sub * 16 + e] : 0.0f;
        }
        double kd[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
            kd[e] = double(kf[e]);
#pragma unroll
        for (int g = 0; g < kMaxGroup; ++g) {
            if (g >= G)
                break;
            // four independent partial sums (every product exact; the order
            // of the fp64 sums is free, see above)
            double d4[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll
            for (int e = 0; e < 16; ++e)
                d4[e & 3] = __fma_rn(sm.qs[g][sub * 17 + e], kd[e], d4[e & 3]);
            double dot = __dadd_rn(__dadd_rn(d4[0], d4[1]), __dadd_rn(d4[2], d4[3]));
            dot = __dadd_rn(dot, __shfl_xor_sync(0xffffffffu, dot, 1));
            dot = __dadd_rn(dot, __shfl_xor_sync(0xffffffffu, dot, 2));
            dot = __dadd_rn(dot, __shfl_xor_sync(0xffffffffu, dot, 4));
            if (jj < n && sub == 0)
                sm.sc[g][jj] = __fmul_rn(__double2float_rn(dot), scale);
        }
    }
    __syncthreads();
    // ---- block maxima, fp64 weights and their sums (warp g per head)
    for (int g = warp; g < G; g += kAttnWarps) {
        float m = -INFINITY;
        for (int jj = lane; jj < n; jj += 32)
            m = fmaxf(m, sm.sc[g][jj]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        double S = 0.0;
        for (int jj = lane; jj < kPosBlock; jj += 32) {
            const double e = jj < n ? exp(double(sm.sc[g][jj]) - double(m)) : 0.0;
            sm.ew[g][jj] = e;
            S = __dadd_rn(S, e);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            S = __dadd_rn(S, __shfl_xor_sync(0xffffffffu, S, o));
        if (lane == 0) {
            sm.mb[g] = m;
            p.bmax[size_t(kv * G + g) * p.nblk + blk] = m;
            p.bsum[size_t(kv * G + g) * p.nblk + blk] = S;
        }
    }
    __syncthreads();
    // ---- weighted values: thread (pg, c) dims 4c .. 4c+3, positions pg, pg + kAttnWarps, ...
    const int pg = tid >> 5, c = tid & 31;
    double acc[kMaxGroup][4];
#pragma unroll
    for (int g = 0; g < kMaxGroup; ++g)
#pragma unroll
        for (int x = 0; x < 4; ++x)
            acc[g][x] = 0.0;
    for (int jj = pg; jj < n; jj += kAttnWarps) {
        float vf[4];
        if (jj < nk) {
            const uint2 ab = *reinterpret_cast<const uint2 *>(&sm.vb[jj][4 * c]);
            vf[0] = __uint_as_float(ab.x << 16);
            vf[1] = __uint_as_float(ab.x & 0xffff0000u);
            vf[2] = __uint_as_float(ab.y << 16);
            vf[3] = __uint_as_float(ab.y & 0xffff0000u);
        } else {
#pragma unroll
            for (int x = 0; x < 4; ++x)
                vf[x] = sm.vs[4 * c + x];
        }
#pragma unroll
        for (int g = 0; g < kMaxGroup; ++g) {
            if (g >= G)
                break;
            const double e = sm.ew[g][jj];
#pragma unroll
            for (int x = 0; x < 4; ++x)
                acc[g][x] = __fma_rn(e, double(vf[x]), acc[g][x]);
        }
    }
#pragma unroll
    for (int g = 0; g < kMaxGroup; ++g) {
        if (g >= G)
            break;
#pragma unroll
        for (int x = 0; x < 4; ++x)
            sm.part[pg][g][4 * c + x] = acc[g][x];
    }
    __syncthreads();
    for (int t = tid; t < G * kHeadDim; t += kAttnThreads) {
        const int g = t / kHeadDim, d = t % kHeadDim;
        double num = 0.0;
#pragma unroll
        for (int q4 = 0; q4 < kAttnWarps; ++q4)
            num = __dadd_rn(num, sm.part[q4][g][d]);
        p.bnum[(size_t(kv * G + g) * p.nblk + blk) * kHeadDim + d] = num;
    }
    // ---- the last block of this kv head to finish combines the blocks
    const int nact = pos / kPosBlock + 1;
    __threadfence();
    __syncthreads();
    if (tid == 0)
        sm.last = atomicAdd(&p.ticket[kv], 1u) == unsigned(nact - 1);
    __syncthreads();
    if (!sm.last)
        return;
    __threadfence();
    // factors exp(m_b - m) per head and block (reusing ew), and the sums
    double *fac = &sm.ew[0][0];               // [G][nact] when nact <= 64, else recomputed
    const bool fit = nact <= kPosBlock;
    // up to 16 blocks and two outputs per thread: the blocks' partial values
    // are loaded first, so that their round trip overlaps the factors'
    const bool pre = fit && nact <= 16 && G * kHeadDim <= 2 * kAttnThreads;
    const int pt1 = tid + kAttnThreads;
    const bool has0 = tid < G * kHeadDim, has1 = pt1 < G * kHeadDim;
    const int pg0 = tid / kHeadDim, pd0 = tid % kHeadDim, pg1 = pt1 / kHeadDim, pd1 = pt1 % kHeadDim;
    double pv0[16], pv1[16];
    if (pre) {
        const size_t hb0 = size_t(kv * G + pg0) * p.nblk, hb1 = size_t(kv * G + pg1) * p.nblk;
#pragma unroll
        for (int u = 0; u < 16; ++u) {
            pv0[u] = has0 && u < nact ? __ldcg(p.bnum + (hb0 + u) * kHeadDim + pd0) : 0.0;
            pv1[u] = has1 && u < nact ? __ldcg(p.bnum + (hb1 + u) * kHeadDim + pd1) : 0.0;
        }
    }
    __shared__ float gm[kMaxGroup];
    __shared__ double gs[kMaxGroup];
    for (int g = warp; g < G; g += kAttnWarps) {
        const size_t hb = size_t(kv * G + g) * p.nblk;
        float m = -INFINITY;
        for (int b = lane; b < nact; b += 32)
            m = fmaxf(m, __ldcg(p.bmax + hb + b));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        double S = 0.0;
        for (int b = lane; b < nact; b += 32) {
            const double f = exp(double(__ldcg(p.bmax + hb + b)) - double(m));
            if (fit)
                fac[g * kPosBlock + b] = f;
            S = __fma_rn(__ldcg(p.bsum + hb + b), f, S);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            S = __dadd_rn(S, __shfl_xor_sync(0xffffffffu, S, o));
        if (lane == 0) {
            gm[g] = m;
            gs[g] = S;
        }
    }
    __syncthreads();
    if (pre) {
        double num0 = 0.0, num1 = 0.0;
#pragma unroll
        for (int u = 0; u < 16; ++u) {
            if (u < nact) {
                num0 = __fma_rn(pv0[u], fac[(has0 ? pg0 : 0) * kPosBlock + u], num0);
                num1 = __fma_rn(pv1[u], fac[(has1 ? pg1 : 0) * kPosBlock + u], num1);
            }
        }
        if (has0)
            p.out[(kv * G + pg0) * kHeadDim + pd0] = __float2bfloat16_rn(__double2float_rn(__ddiv_rn(num0, gs[pg0])));
        if (has1)
            p.out[(kv * G + pg1) * kHeadDim + pd1] = __float2bfloat16_rn(__double2float_rn(__ddiv_rn(num1, gs[pg1])));
    } else if (fit) {
        // each thread's outputs (g, d) for t = tid, tid + kAttnThreads, ...;
        // sixteen blocks' partial values of both of a thread's first two
        // outputs loaded together, then added
        for (int t0 = tid; t0 < G * kHeadDim; t0 += 2 * kAttnThreads) {
            const int t1 = t0 + kAttnThreads;
            const bool two = t1 < G * kHeadDim;
            const int g0 = t0 / kHeadDim, d0 = t0 % kHeadDim;
            const int g1 = two ? t1 / kHeadDim : g0, d1 = two ? t1 % kHeadDim : d0;
            const size_t hb0 = size_t(kv * G + g0) * p.nblk, hb1 = size_t(kv * G + g1) * p.nblk;
            double num0 = 0.0, num1 = 0.0;
            for (int b0 = 0; b0 < nact; b0 += 16) {
                double v0[16], v1[16];
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    const bool in = b0 + u < nact;
                    v0[u] = in ? __ldcg(p.bnum + (hb0 + b0 + u) * kHeadDim + d0) : 0.0;
                    v1[u] = in && two ? __ldcg(p.bnum + (hb1 + b0 + u) * kHeadDim + d1) : 0.0;
                }
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    if (b0 + u < nact) {
                        num0 = __fma_rn(v0[u], fac[g0 * kPosBlock + b0 + u], num0);
                        num1 = __fma_rn(v1[u], fac[g1 * kPosBlock + b0 + u], num1);
                    }
                }
            }
            p.out[(kv * G + g0) * kHeadDim + d0] = __float2bfloat16_rn(__double2float_rn(__ddiv_rn(num0, gs[g0])));
            if (two)
                p.out[(kv * G + g1) * kHeadDim + d1] =
                    __float2bfloat16_rn(__double2float_rn(__ddiv_rn(num1, gs[g1])));
        }
    } else {
        for (int t = tid; t < G * kHeadDim; t += kAttnThreads) {
            const int g = t / kHeadDim, d = t % kHeadDim;
            const size_t hb = size_t(kv * G + g) * p.nblk;
            double num = 0.0;
            for (int b = 0; b < nact; ++b) {
                const double f = exp(double(__ldcg(p.bmax + hb + b)) - double(gm[g]));
                num = __fma_rn(__ldcg(p.bnum + (hb + b) * kHeadDim + d), f, num);
            }
            p.out[(kv * G + g) * kHeadDim + d] = __float2bfloat16_rn(__double2float_rn(__ddiv_rn(num, gs[g])));
        }
    }
    if (tid == 0)
        p.ticket[kv] = 0u;
}

// (cos, sin) of pos * base^(-2i / D) for every position and pair, fp64 then
// fp32 (the same values the attention kernel computes without a table).
__global__ void rope_table_kernel(float2 *tab, int T_max, double base)
{
    const int64_t idx = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
    if (idx >= int64_t(T_max) * (kHeadDim / 2))
        return;
    tab[idx] = rope_angle(int(idx / (kHeadDim / 2)), int(idx % (kHeadDim / 2)), base);
}

__global__ void position_advance_kernel(int32_t *pos)
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (threadIdx.x == 0)
        pos[0] += 1;
}

// Workspace carve-up (16-byte aligned pieces).
struct AttnWs {
    size_t bmax, bsum, bnum, ticket, total;
};

AttnWs ws_layout(int H, int Hkv, int T_max)
{
    const int nblk = (T_max + kPosBlock - 1) / kPosBlock;
    auto up = [](size_t v) { return (v + 15) / 16 * 16; };
    AttnWs w{};
    w.bmax = 0;
    w.bsum = up(w.bmax + size_t(H) * nblk * 4);
    w.bnum = up(w.bsum + size_t(H) * nblk * 8);
    w.ticket = up(w.bnum + size_t(H) * nblk * kHeadDim * 8);
    w.total = up(w.ticket + size_t(Hkv) * 4);
    return w;
}

}  // namespace

size_t attention_workspace_bytes(int H, int Hkv, int T_max) { return ws_layout(H, Hkv, T_max).total; }

int attention_max_group() { return kMaxGroup; }

int launch_rope_table(float *tab, int D, int T_max, double base, cudaStream_t s)
{
    if (D != kHeadDim)
        return BL_ERR_SHAPE;
    const int64_t n = int64_t(T_max) * (kHeadDim / 2);
    rope_table_kernel<<<unsigned((n + 255) / 256), 256, 0, s>>>(reinterpret_cast<float2 *>(tab), T_max, base);
    return launch_status();
}

namespace {

template <int GT>
int launch_attn_t(const AttnParams &p, unsigned flags, cudaStream_t s)
{
    const size_t smem = sizeof(AttnSmem);
    int per_sm = 0;
    int st = occupancy(reinterpret_cast<const void *>(attention_decode_kernel<GT>), kAttnThreads, smem, &per_sm);
    if (st)
        return st;
    if (per_sm < 1)
        return BL_ERR_SHAPE;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(p.Hkv), unsigned(p.nblk));
    cfg.blockDim = dim3(kAttnThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    if (flags & BL_FLAG_PDL) {
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
    return cuda_status(cudaLaunchKernelEx(&cfg, attention_decode_kernel<GT>, p));
}

}  // namespace

int launch_attention_decode(const void *q, const void *k, const void *v, void *cache_k, void *cache_v,
                            const int32_t *pos, int H, int Hkv, int D, int T_max, double rope_base,
                            const float *rope, void *out, void *ws, unsigned flags, cudaStream_t s)
{
    const DeviceInfo *di = device_info();
    if (!di)
        return BL_ERR_CUDA;
    if (D != kHeadDim || H / Hkv > kMaxGroup)
        return BL_ERR_SHAPE;
    const AttnWs w = ws_layout(H, Hkv, T_max);
    auto *base = static_cast<unsigned char *>(ws);
    AttnParams p{};
    p.q = static_cast<const __nv_bfloat16 *>(q);
    p.k = static_cast<const __nv_bfloat16 *>(k);
    p.v = static_cast<const __nv_bfloat16 *>(v);
    p.cache_k = static_cast<__nv_bfloat16 *>(cache_k);
    p.cache_v = static_cast<__nv_bfloat16 *>(cache_v);
    p.pos = pos;
    p.H = H;
    p.Hkv = Hkv;
    p.T_max = T_max;
    p.nblk = (T_max + kPosBlock - 1) / kPosBlock;
    p.rope_base = rope_base;
    p.rope = reinterpret_cast<const float2 *>(rope);
    p.out = static_cast<__nv_bfloat16 *>(out);
    p.bmax = reinterpret_cast<float *>(base + w.bmax);
    p.bsum = reinterpret_cast<double *>(base + w.bsum);
    p.bnum = reinterpret_cast<double *>(base + w.bnum);
    p.ticket = reinterpret_cast<unsigned *>(base + w.ticket);
    p.status = di->status;
    const int g = H / Hkv;
    switch (g) {
    case 1: return launch_attn_t<1>(p, flags, s);
    case 2: return launch_attn_t<2>(p, flags, s);
    case 4: return launch_attn_t<4>(p, flags, s);
    case 8: return launch_attn_t<8>(p, flags, s);
    default: return launch_attn_t<0>(p, flags, s);
    }
}

int launch_position_advance(int32_t *pos, cudaStream_t s)
{
    position_advance_kernel<<<1, 32, 0, s>>>(pos);
    return launch_status();
}

}  // namespace bl
