// gemv_stream_common.cuh -- device pieces shared by the one-token streaming
// GEMV (gemv_stream.cu) and the persistent decode chain (gemv_chain.cu): CTA
// geometry, the activation prologues (quantisation, RMSNorm + quantisation,
// pre-quantised copy), the dp4a stage bodies over the TL bytes, and the
// per-set fold of partial row sums.  The prologues take any params / shared
// memory types that carry the fields they use (x, K, q, d, rowsum, gain, gt,
// eps; bmax, bsum, bss, d).
#pragma once

#include "bl_common.cuh"

namespace bl {
namespace {

constexpr int kMaxConsumers = 16;
constexpr int kStages = 4;                           // ring stages
constexpr int kMaxSet = 8;                           // groups per set (stage), at most
constexpr int kMaxGroupsPerCta = 64;
constexpr int kSmallK = 8192;                        // up to here: KC = 8
constexpr int kLargeGroupsPerSm = 16;                // from here on: two 8-warp CTAs per SM

// Geometry of a CTA with KC consumer warps.
template <int KC>
struct Geo {
    static constexpr int kConsumerThreads = 32 * KC;
    static constexpr int kThreads = kConsumerThreads + 32;   // + the producer warp
    // two CTAs of up to ten consumer warps fit on an SM (at <= 93 registers)
    static constexpr int kCtasPerSm = KC <= 10 ? 2 : 1;
};

// Activations: pre-quantised q; raw bf16 / fp32 x quantised in the prologue;
// or x normalised (RMSNorm) and then quantised in the prologue.
enum { SMODE_Q = 0, SMODE_X_BF16 = 1, SMODE_X_F32 = 2, SMODE_NORM_BF16 = 3, SMODE_NORM_F32 = 4,
       SMODE_RELU2 = 5 };

// 512-byte pieces (256 k) of one group per stage: the whole k range when it
// is at most two pieces per consumer warp (one stage per set), else one per
// warp.  Either way warp w only ever takes pieces w, w + KC, w + 2 KC, ...
__host__ __device__ __forceinline__ int stage_pieces(int P, int KC) { return P <= 2 * KC ? P : KC; }

struct StreamParams {
    GemvProblem prob[kGemvMaxProblems];
    int64_t gstart[kGemvMaxProblems + 1];  // prefix sums of the products' row groups
    int count;
    int64_t K;
    const int8_t *q;
    const float *d;
    const int32_t *rowsum;
    const void *x;
    const void *x2;      // SMODE_RELU2: the up projection [K] (x is the gate), bf16
    const void *gain;    // RMSNorm gain [K] (SMODE_NORM_*), NULL for none
    int gt;              // its dtype
    float eps;           // RMSNorm epsilon
    int yt;
    // CTA b owns row groups [b*gpc_base + min(b, gpc_rem), ...), gpc_base (+1) of them
    int64_t gpc_base;
    int gpc_rem;
    int set_cap;         // R: groups a stage holds at most (4 .. kMaxSet)
    int *status;
};

struct StreamSmem {
    uint64_t full[kStages];
    uint64_t empty[kStages];
    int abort_flag;
    alignas(16) float bmax[kMaxConsumers];   // read back as float4
    int bsum[kMaxConsumers];
    double bss[kMaxConsumers];               // RMSNorm: per-warp sums of squares
    float d;
    float wscale[kGemvMaxProblems];   // each product's gamma_eff
    int sacc[kMaxGroupsPerCta][8];
    // followed by the ring (kStages x set_cap slots) and the int8 activations (K bytes)
};

constexpr size_t kHeader = (sizeof(StreamSmem) + 127) / 128 * 128;
static_assert(offsetof(StreamSmem, bmax) % 16 == 0, "bmax is read as float4");

// The CTA's ng groups in the fewest sets of at most R groups, sized evenly
// (base or base + 1 groups; the first `extra` sets take one more).
struct SetSplit {
    int nsets, base, extra;
    __device__ __forceinline__ SetSplit(int ng, int R)
    {
        nsets = (ng + R - 1) / R;
        base = ng / nsets;
        extra = ng - base * nsets;
    }
    __device__ __forceinline__ int size(int i) const { return base + (i < extra ? 1 : 0); }
};

// Product of concatenated row group G.
__device__ __forceinline__ int locate(const StreamParams &p, int64_t G)
{
    int pi = 0;
#pragma unroll
    for (int i = 1; i < kGemvMaxProblems; ++i)
        if (i < p.count && G >= p.gstart[i])
            pi = i;
    return pi;
}

__device__ __forceinline__ uint4 lds128(uint32_t saddr)
{
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(saddr));
    return v;
}

template <int KC>
__device__ __forceinline__ void consumers_sync() { named_barrier(1, Geo<KC>::kConsumerThreads); }

// Four int32 values, each already within [-128, 127], as one little-endian
// word of int8 (q0 in the low byte); the saturating pack equals the clamp.
__device__ __forceinline__ uint32_t pack4_s8(int q0, int q1, int q2, int q3)
{
    uint32_t hi, d;
    asm("cvt.pack.sat.s8.s32.b32 %0, %1, %2, 0;" : "=r"(hi) : "r"(q3), "r"(q2));
    asm("cvt.pack.sat.s8.s32.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(q1), "r"(q0), "r"(hi));
    return d;
}

// rint(x * s) for eight values (fp32 product, ties to even), packed as int8;
// the sum of the eight added to *sum.
__device__ __forceinline__ uint2 quant8(const float (&f)[8], float s, int &sum)
{
    int t[8];
#pragma unroll
    for (int j = 0; j < 8; ++j)
        t[j] = __float2int_rn(__fmul_rn(f[j], s));
    const uint32_t lo = pack4_s8(t[0], t[1], t[2], t[3]);
    const uint32_t hi = pack4_s8(t[4], t[5], t[6], t[7]);
    sum = dp4a_us(0x01010101u, lo, sum);
    sum = dp4a_us(0x01010101u, hi, sum);
    return make_uint2(lo, hi);
}

__device__ __forceinline__ void bf16x8_f32(const uint4 v, float (&f)[8])
{
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

// Block-wide absmax of the consumer threads' maxima, then the scale
// s = 127 / max(amax, eps); d = max(amax, eps) / 127 goes to sm.d.
template <int KC, class Smem>
__device__ __forceinline__ float stream_scale(Smem &sm, float amax)
{
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // maxima are >= 0 and finite (fmaxf from 0 drops NaN): their bit
    // patterns order like the values
    const uint32_t wmax = __reduce_max_sync(0xffffffffu, __float_as_uint(amax));
    if (lane == 0)
        sm.bmax[warp] = __uint_as_float(wmax);
    consumers_sync<KC>();
    float a = 0.0f;
#pragma unroll
    for (int w = 0; w + 4 <= KC; w += 4) {
        const float4 b4 = *reinterpret_cast<const float4 *>(&sm.bmax[w]);
        a = fmaxf(fmaxf(a, b4.x), fmaxf(b4.y, fmaxf(b4.z, b4.w)));
    }
#pragma unroll
    for (int w = KC & ~3; w < KC; ++w)
        a = fmaxf(a, sm.bmax[w]);
    const float a_eff = fmaxf(a, kEps);
    if (tid == 0)
        sm.d = __fdiv_rn(a_eff, kQb);
    return __fdiv_rn(kQb, a_eff);
}

// Quantise the token x into qs.  Consumer warp w only ever reads the
// activations of its own pieces (256 k each: pieces w, w + KC, w + 2 KC, ...),
// so it quantises exactly those and needs no block barrier afterwards; only
// the absmax is block-wide.  s = 127 / max(amax, eps), q = clamp(rint(x *
// s)); each warp's partial row sum goes to bsum.  Lane l takes elements
// 8l .. 8l + 7 of each piece; x stays in registers as raw bf16, CH pieces.
template <int KC, int CH, class Prm, class Smem>
__device__ __forceinline__ void stream_quantize_bf16(const Prm &p, Smem &sm, int8_t *qs)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int P = int(p.K / 256);
    uint4 raw[CH];
#pragma unroll
    for (int i = 0; i < CH; ++i) {
        const int j = i * KC + warp;
        raw[i] = j < P ? ld_dep_v4(static_cast<const __nv_bfloat16 *>(p.x) + (int64_t(j) * 32 + lane) * 8)
                       : make_uint4(0, 0, 0, 0);
    }
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < CH; ++i) {
        float f[8];
        bf16x8_f32(raw[i], f);
#pragma unroll
        for (int e = 0; e < 8; ++e)
            amax = fmaxf(amax, fabsf(f[e]));
    }
    const float s = stream_scale<KC>(sm, amax);
    int sum = 0;
#pragma unroll
    for (int i = 0; i < CH; ++i) {
        const int j = i * KC + warp;
        if (j < P) {
            float f[8];
            bf16x8_f32(raw[i], f);
            *reinterpret_cast<uint2 *>(qs + (j * 32 + lane) * 8) = quant8(f, s, sum);
        }
    }
    sum = __reduce_add_sync(0xffffffffu, sum);
    if (lane == 0)
        sm.bsum[warp] = sum;
    __syncwarp();
}

// The same for any K and either input type: one pass over the warp's pieces
// for the absmax, a second one that reads them again (from L2) to quantise.
template <int KC, int XT, class Prm, class Smem>
__device__ __forceinline__ void stream_quantize_2pass(const Prm &p, Smem &sm, int8_t *qs)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int P = int(p.K / 256);
    float amax = 0.0f;
#pragma unroll 4
    for (int j = warp; j < P; j += KC) {
        float f[8];
        load8<XT, true>(p.x, (int64_t(j) * 32 + lane) * 8, f);
#pragma unroll
        for (int e = 0; e < 8; ++e)
            amax = fmaxf(amax, fabsf(f[e]));
    }
    const float s = stream_scale<KC>(sm, amax);
    int sum = 0;
#pragma unroll 4
    for (int j = warp; j < P; j += KC) {
        float f[8];
        load8<XT, true>(p.x, (int64_t(j) * 32 + lane) * 8, f);
        *reinterpret_cast<uint2 *>(qs + (j * 32 + lane) * 8) = quant8(f, s, sum);
    }
    sum = __reduce_add_sync(0xffffffffu, sum);
    if (lane == 0)
        sm.bsum[warp] = sum;
    __syncwarp();
}

// Pre-quantised activations: each warp copies the q of its own pieces (no
// block barrier); warp 0 takes d and the row sum.
template <int KC, class Prm, class Smem>
__device__ __forceinline__ void stream_copy_q(const Prm &p, Smem &sm, int8_t *qs)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int P = int(p.K / 256);
    for (int j = warp; j < P; j += KC)
        if (lane < 16)
            *reinterpret_cast<uint4 *>(qs + j * 256 + lane * 16) = ld_dep_v4(p.q + int64_t(j) * 256 + lane * 16);
    if (lane == 0) {
        sm.bsum[warp] = warp == 0 ? int(ld_dep_u32(p.rowsum)) : 0;
        if (warp == 0)
            sm.d = __uint_as_float(ld_dep_u32(p.d));
    }
    __syncwarp();
}

// Eight gain values (k .. k + 7) as fp32; 1.0 without a gain (an exact
// identity for the product that applies it).
template <class Prm>
__device__ __forceinline__ void stream_gain8(const Prm &p, int64_t k, float (&g)[8])
{
    if (!p.gain) {
#pragma unroll
        for (int j = 0; j < 8; ++j)
            g[j] = 1.0f;
    } else if (p.gt == BL_BF16) {
        bf16x8_f32(ld_ro_v4(static_cast<const __nv_bfloat16 *>(p.gain) + k), g);
    } else {
        const float *gp = static_cast<const float *>(p.gain) + k;
        const uint4 a = ld_ro_v4(gp), b = ld_ro_v4(gp + 4);
        g[0] = __uint_as_float(a.x); g[1] = __uint_as_float(a.y);
        g[2] = __uint_as_float(a.z); g[3] = __uint_as_float(a.w);
        g[4] = __uint_as_float(b.x); g[5] = __uint_as_float(b.y);
        g[6] = __uint_as_float(b.z); g[7] = __uint_as_float(b.w);
    }
}

// Block-wide sum of the consumer threads' fp64 partial sums of squares, then
// the RMSNorm factor r = 1 / sqrt((float)(S / K) + eps) (fp32, correctly
// rounded square root and division).
template <int KC, class Prm, class Smem>
__device__ __forceinline__ float stream_rms_factor(const Prm &p, Smem &sm, double ss)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        ss = __dadd_rn(ss, __shfl_xor_sync(0xffffffffu, ss, o));
    if (lane == 0)
        sm.bss[warp] = ss;
    consumers_sync<KC>();
    double S = 0.0;
#pragma unroll
    for (int w = 0; w < KC; ++w)
        S = __dadd_rn(S, sm.bss[w]);
    const float ms = __double2float_rn(__ddiv_rn(S, double(p.K)));
    return __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, p.eps)));
}

// RMSNorm, then quantisation, of the token x: h = (x * r) * gain, each warp
// for the activations of its own pieces (as in stream_quantize_bf16); two
// block-wide reductions (the sum of squares, then the absmax of h).  CH > 0
// (bf16 x only): the warp's raw x stays in registers, CH pieces; CH = 0: x
// is read again from L2 for each pass.
template <int KC, int XT, int CH, class Prm, class Smem>
__device__ __forceinline__ void stream_rmsnorm_quantize(const Prm &p, Smem &sm, int8_t *qs)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int P = int(p.K / 256);
    constexpr int RC = CH > 0 ? CH : 1;
    uint4 raw[RC];
    if constexpr (CH == 0)
        raw[0] = make_uint4(0, 0, 0, 0);   // unused: x is re-read from L2
    auto load_x = [&](int i, int j, float (&f)[8]) {
        if constexpr (CH > 0)
            bf16x8_f32(raw[i], f);
        else
            load8<XT, true>(p.x, (int64_t(j) * 32 + lane) * 8, f);
    };
    if constexpr (CH > 0) {
#pragma unroll
        for (int i = 0; i < CH; ++i) {
            const int j = i * KC + warp;
            raw[i] = j < P ? ld_dep_v4(static_cast<const __nv_bfloat16 *>(p.x) + (int64_t(j) * 32 + lane) * 8)
                           : make_uint4(0, 0, 0, 0);
        }
    }
    constexpr int kUnroll = CH > 0 ? CH : 4;
    double ss = 0.0;
#pragma unroll kUnroll
    for (int i = 0; i < (CH > 0 ? CH : (P + KC - 1) / KC); ++i) {
        const int j = i * KC + warp;
        if (j < P) {
            float f[8];
            load_x(i, j, f);
#pragma unroll
            for (int e = 0; e < 8; ++e)
                ss = __dadd_rn(ss, __dmul_rn(double(f[e]), double(f[e])));
        }
    }
    const float r = stream_rms_factor<KC>(p, sm, ss);
    auto h8 = [&](int i, int j, float (&h)[8]) {
        float g[8];
        load_x(i, j, h);
        stream_gain8(p, (int64_t(j) * 32 + lane) * 8, g);
#pragma unroll
        for (int e = 0; e < 8; ++e)
            h[e] = __fmul_rn(__fmul_rn(h[e], r), g[e]);
    };
    float amax = 0.0f;
#pragma unroll kUnroll
    for (int i = 0; i < (CH > 0 ? CH : (P + KC - 1) / KC); ++i) {
        const int j = i * KC + warp;
        if (j < P) {
            float h[8];
            h8(i, j, h);
#pragma unroll
            for (int e = 0; e < 8; ++e)
                amax = fmaxf(amax, fabsf(h[e]));
        }
    }
    const float s = stream_scale<KC>(sm, amax);
    int sum = 0;
#pragma unroll kUnroll
    for (int i = 0; i < (CH > 0 ? CH : (P + KC - 1) / KC); ++i) {
        const int j = i * KC + warp;
        if (j < P) {
            float h[8];
            h8(i, j, h);
            *reinterpret_cast<uint2 *>(qs + (j * 32 + lane) * 8) = quant8(h, s, sum);
        }
    }
    sum = __reduce_add_sync(0xffffffffu, sum);
    if (lane == 0)
        sm.bsum[warp] = sum;
    __syncwarp();
}

// Squared-ReLU gate, then quantisation: h = (r * r) * u with r = max(g, 0),
// g = x and u = x2 (bf16), two fp32 products; read twice from L2 (absmax
// pass, quantise pass), each warp for the activations of its own pieces.
template <int KC, class Prm, class Smem>
__device__ __forceinline__ void stream_relu2_quantize(const Prm &p, Smem &sm, int8_t *qs)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int P = int(p.K / 256);
    auto h8 = [&](int j, float (&h)[8]) {
        float u[8];
        load8<BL_BF16, true>(p.x, (int64_t(j) * 32 + lane) * 8, h);
        load8<BL_BF16, true>(p.x2, (int64_t(j) * 32 + lane) * 8, u);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const float r = fmaxf(h[e], 0.0f);
            h[e] = __fmul_rn(__fmul_rn(r, r), u[e]);
        }
    };
    float amax = 0.0f;
#pragma unroll 4
    for (int j = warp; j < P; j += KC) {
        float h[8];
        h8(j, h);
#pragma unroll
        for (int e = 0; e < 8; ++e)
            amax = fmaxf(amax, fabsf(h[e]));
    }
    const float s = stream_scale<KC>(sm, amax);
    int sum = 0;
#pragma unroll 4
    for (int j = warp; j < P; j += KC) {
        float h[8];
        h8(j, h);
        *reinterpret_cast<uint2 *>(qs + (j * 32 + lane) * 8) = quant8(h, s, sum);
    }
    sum = __reduce_add_sync(0xffffffffu, sum);
    if (lane == 0)
        sm.bsum[warp] = sum;
    __syncwarp();
}

// One 16-byte piece of stored codes (64 k of one row) against the 64
// activations q[0..3] into four accumulators (s, 4s, 16s, 64s weighted).
__device__ __forceinline__ void mac4(const uint4 wv, const uint4 (&q)[4], int (&acc)[4])
{
    const uint32_t wd[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        acc[0] = dp4a_us(wd[w] & 0x03030303u, q[w].x, acc[0]);
        acc[1] = dp4a_us(wd[w] & 0x0c0c0c0cu, q[w].y, acc[1]);
        acc[2] = dp4a_us(wd[w] & 0x30303030u, q[w].z, acc[2]);
        acc[3] = dp4a_us(wd[w] & 0xc0c0c0c0u, q[w].w, acc[3]);
    }
}

// One stage of RG groups for this lane: the RG slots lie SLOT bytes apart
// (a compile-time stride when SLOT > 0, so the loads take immediate offsets;
// else slot_rt), and all loads are issued before the arithmetic.
template <int SLOT, int RG>
__device__ __forceinline__ void stage_mac(uint32_t base, uint32_t slot_rt, const uint4 (&q)[4],
                                          int (&acc)[kMaxSet][4])
{
    const uint32_t slot = SLOT > 0 ? uint32_t(SLOT) : slot_rt;
    uint4 wv[RG];
#pragma unroll
    for (int r = 0; r < RG; ++r)
        wv[r] = lds128(base + r * slot);
#pragma unroll
    for (int r = 0; r < RG; ++r)
        mac4(wv[r], q, acc[r]);
}

template <int SLOT>
__device__ __forceinline__ void stage_mac_n(int rg, uint32_t base, uint32_t slot, const uint4 (&q)[4],
                                            int (&acc)[kMaxSet][4])
{
    switch (rg) {
    case 1: stage_mac<SLOT, 1>(base, slot, q, acc); break;
    case 2: stage_mac<SLOT, 2>(base, slot, q, acc); break;
    case 3: stage_mac<SLOT, 3>(base, slot, q, acc); break;
    case 4: stage_mac<SLOT, 4>(base, slot, q, acc); break;
    case 5: stage_mac<SLOT, 5>(base, slot, q, acc); break;
    case 6: stage_mac<SLOT, 6>(base, slot, q, acc); break;
    case 7: stage_mac<SLOT, 7>(base, slot, q, acc); break;
    default: stage_mac<SLOT, 8>(base, slot, q, acc); break;
    }
}
static_assert(kMaxSet == 8, "stage_mac_n covers 1..8 groups");

// End of a set of RG groups for this warp: fold each group's four
// accumulators, sum the four lanes of a row (lanes l, l^8, l^16, l^24) and
// add the row's partial into the CTA's row sums; the groups' shuffle chains
// are independent and interleave.
template <int RG>
__device__ __forceinline__ void set_flush(int (&acc)[kMaxSet][4], int (*sacc)[8], int lane)
{
    int v[RG];
#pragma unroll
    for (int r = 0; r < RG; ++r) {
        v[r] = acc[r][0] + (acc[r][1] >> 2) + (acc[r][2] >> 4) + (acc[r][3] >> 6);
#pragma unroll
        for (int a = 0; a < 4; ++a)
            acc[r][a] = 0;
    }
#pragma unroll
    for (int r = 0; r < RG; ++r)
        v[r] += __shfl_xor_sync(0xffffffffu, v[r], 8);
#pragma unroll
    for (int r = 0; r < RG; ++r)
        v[r] += __shfl_xor_sync(0xffffffffu, v[r], 16);
    if (lane < 8) {
#pragma unroll
        for (int r = 0; r < RG; ++r)
            atomicAdd(&sacc[r][lane], v[r]);
    }
}

__device__ __forceinline__ void set_flush_n(int rg, int (&acc)[kMaxSet][4], int (*sacc)[8], int lane)
{
    switch (rg) {
    case 1: set_flush<1>(acc, sacc, lane); break;
    case 2: set_flush<2>(acc, sacc, lane); break;
    case 3: set_flush<3>(acc, sacc, lane); break;
    case 4: set_flush<4>(acc, sacc, lane); break;
    case 5: set_flush<5>(acc, sacc, lane); break;
    case 6: set_flush<6>(acc, sacc, lane); break;
    case 7: set_flush<7>(acc, sacc, lane); break;
    default: set_flush<8>(acc, sacc, lane); break;
    }
}

}  // namespace
}  // namespace bl
