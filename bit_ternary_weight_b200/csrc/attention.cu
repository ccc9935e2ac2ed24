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
//   softmax    m = max_j s_j; e_j = (float)exp((double)(s_j - m)) with the
//              difference in fp32; S = (float)(sum_j e_j) in fp64.
//   output     out[d] = bf16((float)(sum_j e_j V[j][d]) / S), the sum in fp64
//              (products exact), the division in fp32.
// The fp64 sums run in another order than the oracle's; each is exact or
// within an fp64 rounding of it, so the fp32 values agree unless one lies
// within about 1e-15 (relative) of an fp32 rounding boundary.  exp, cos, sin
// and pow are CUDA's fp64 functions on the GPU and the C library's on the CPU;
// they may differ in the last fp64 bit, which moves an fp32 result only on
// such a boundary too.
//
// RoPE's cosines and sines come from a table of every (position, pair) that
// bitlinear_rope_table computes once (same definition), or are computed in
// the scores kernel when no table is given.
//
// Design: two launches over blocks of 64 cached positions, so that the work
// of one token spreads over (kv heads x position blocks) CTAs instead of one
// CTA per head walking every position.  The position pos is a device scalar
// read after the dependency wait, so a CUDA graph can replay the calls for
// successive tokens; the grids cover the whole cache and the blocks beyond
// pos return at once.
//   scores   CTA (kv head, block): the rotated queries of the kv head's query
//            heads (all of them share its keys); the block holding pos also
//            rotates the new key and appends key and value at pos.  Eight
//            lanes per position (16 dimensions each, fp64 partial dot
//            products for every query head, three shuffle rounds), four
//            positions per warp step.  Scores and the block's maxima go to
//            the workspace.
//   values   CTA (kv head, block): the global maximum of each query head from
//            the blocks' maxima, the block's e_j in shared memory, the fp64
//            partial sums of e_j and of e_j V[j] (lanes over dimensions, four
//            position groups per CTA), written to the workspace; the CTA that
//            arrives last on the kv head's ticket (fence, atomic add) adds the
//            blocks' partial sums in block order, divides, rounds and stores,
//            and resets the ticket.
// A position outside the cache records BL_ERR_SHAPE in the device status word
// and writes nothing.
#include "bl_common.cuh"

namespace bl {
namespace {

constexpr int kHeadDim = 128;
constexpr int kPosBlock = 64;             // cached positions per CTA
constexpr int kScoreThreads = 128;
constexpr int kValueThreads = 128;
constexpr int kMaxGroup = 8;              // query heads per kv head

struct AttnParams {
    const __nv_bfloat16 *q, *k, *v;       // [H*D], [Hkv*D], [Hkv*D]
    __nv_bfloat16 *cache_k, *cache_v;     // [Hkv][T_max][D]
    const int32_t *pos;
    int H, Hkv, T_max, nblk;
    double rope_base;
    const float2 *rope;                   // NULL, or (cos, sin) [T_max][D/2] of every angle
    __nv_bfloat16 *out;                   // [H*D]
    // workspace
    float *sc;                            // [H][T_max] scores, then weights
    float *bmax;                          // [H][nblk]
    double *bsum;                         // [H][nblk]
    double *bnum;                         // [H][nblk][D]
    unsigned *ticket;                     // [Hkv], zero between calls
    int *status;
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

// Rotate pair i of a head vector x (bf16) by (cos, sin) cs; the two rotated
// values rounded to bf16 (as fp32).
__device__ __forceinline__ void rope_pair(const __nv_bfloat16 *x, int i, float2 cs, float &o0, float &o1)
{
    const float c = cs.x, s = cs.y;
    const float a = bf16_bits_f32(ld_dep_u16(x + 2 * i)), b = bf16_bits_f32(ld_dep_u16(x + 2 * i + 1));
    const float r0 = __fsub_rn(__fmul_rn(a, c), __fmul_rn(b, s));
    const float r1 = __fadd_rn(__fmul_rn(a, s), __fmul_rn(b, c));
    o0 = bf16_bits_f32(f32_bf16_bits(r0));
    o1 = bf16_bits_f32(f32_bf16_bits(r1));
}

// The token's position, checked against the cache; -1 (and BL_ERR_SHAPE in
// the status word, once per grid) when outside.
__device__ __forceinline__ int read_pos(const AttnParams &p)
{
    const int pos = int(ld_dep_u32(p.pos));
    if (pos < 0 || pos >= p.T_max) {
        if (threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.y == 0)
            atomicExch(p.status, BL_ERR_SHAPE);
        return -1;
    }
    return pos;
}

__global__ void __launch_bounds__(kScoreThreads) attn_scores_kernel(const AttnParams p)
{
    __shared__ float qs[kMaxGroup][kHeadDim];     // rotated queries of the group
    __shared__ float ks[kHeadDim];                // rotated new key (block holding pos)
    __shared__ float2 cs[kHeadDim / 2];           // (cos, sin) of the token's angles
    __shared__ float wmax[kScoreThreads / 32][kMaxGroup];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int kv = blockIdx.x, blk = blockIdx.y;
    const int G = p.H / p.Hkv;
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int pos = read_pos(p);
    if (pos < 0)
        return;
    const int j0 = blk * kPosBlock;
    if (j0 > pos)
        return;
    const int j1 = min(j0 + kPosBlock, pos + 1);
    const bool has_new = pos < j0 + kPosBlock;
    if (tid < kHeadDim / 2)
        cs[tid] = p.rope ? __ldg(p.rope + size_t(pos) * (kHeadDim / 2) + tid) : rope_angle(pos, tid, p.rope_base);
    __syncthreads();
    for (int t = tid; t < G * (kHeadDim / 2); t += kScoreThreads) {
        const int g = t / (kHeadDim / 2), i = t % (kHeadDim / 2);
        float a, b;
        rope_pair(p.q + (kv * G + g) * kHeadDim, i, cs[i], a, b);
        qs[g][2 * i] = a;
        qs[g][2 * i + 1] = b;
    }
    const size_t head_base = size_t(kv) * p.T_max * kHeadDim;
    if (has_new && tid < kHeadDim / 2) {
        float a, b;
        rope_pair(p.k + kv * kHeadDim, tid, cs[tid], a, b);
        ks[2 * tid] = a;
        ks[2 * tid + 1] = b;
        p.cache_k[head_base + size_t(pos) * kHeadDim + 2 * tid] = __float2bfloat16_rn(a);
        p.cache_k[head_base + size_t(pos) * kHeadDim + 2 * tid + 1] = __float2bfloat16_rn(b);
        p.cache_v[head_base + size_t(pos) * kHeadDim + 2 * tid] =
            __ushort_as_bfloat16(static_cast<unsigned short>(ld_dep_u16(p.v + kv * kHeadDim + 2 * tid)));
        p.cache_v[head_base + size_t(pos) * kHeadDim + 2 * tid + 1] =
            __ushort_as_bfloat16(static_cast<unsigned short>(ld_dep_u16(p.v + kv * kHeadDim + 2 * tid + 1)));
    }
    __syncthreads();
    // eight lanes per position (lane group r = lane / 8), sixteen dims each
    const float scale = __double2float_rn(1.0 / sqrt(double(kHeadDim)));
    const int sub = lane & 7, r = lane >> 3;
    float lmax[kMaxGroup];
#pragma unroll
    for (int g = 0; g < kMaxGroup; ++g)
        lmax[g] = -INFINITY;
    for (int jb = j0 + warp * 4; jb < j1; jb += 4 * (kScoreThreads / 32)) {
        const int j = jb + r;
        float kf[16];
        if (j < j1) {
            if (j == pos) {
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    kf[e] = ks[sub * 16 + e];
            } else {
                const uint4 *kr = reinterpret_cast<const uint4 *>(p.cache_k + head_base + size_t(j) * kHeadDim +
                                                                  sub * 16);
                const uint4 a = __ldcg(kr), b = __ldcg(kr + 1);
                const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    kf[2 * e] = __uint_as_float(w[e] << 16);
                    kf[2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
                }
            }
        } else {
#pragma unroll
            for (int e = 0; e < 16; ++e)
                kf[e] = 0.0f;
        }
#pragma unroll
        for (int g = 0; g < kMaxGroup; ++g) {
            if (g >= G)
                break;
            double dot = 0.0;
#pragma unroll
            for (int e = 0; e < 16; ++e)
                dot = __fma_rn(double(qs[g][sub * 16 + e]), double(kf[e]), dot);   // exact products
            dot = __dadd_rn(dot, __shfl_xor_sync(0xffffffffu, dot, 1));
            dot = __dadd_rn(dot, __shfl_xor_sync(0xffffffffu, dot, 2));
            dot = __dadd_rn(dot, __shfl_xor_sync(0xffffffffu, dot, 4));
            if (j < j1) {
                const float sv = __fmul_rn(__double2float_rn(dot), scale);
                if (sub == 0)
                    p.sc[size_t(kv * G + g) * p.T_max + j] = sv;
                lmax[g] = fmaxf(lmax[g], sv);
            }
        }
    }
#pragma unroll
    for (int g = 0; g < kMaxGroup; ++g) {
        if (g >= G)
            break;
        float m = lmax[g];
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 8));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
        if (lane == 0)
            wmax[warp][g] = m;
    }
    __syncthreads();
    if (tid < G) {
        float m = wmax[0][tid];
#pragma unroll
        for (int w = 1; w < kScoreThreads / 32; ++w)
            m = fmaxf(m, wmax[w][tid]);
        p.bmax[size_t(kv * G + tid) * p.nblk + blk] = m;
    }
}

__global__ void __launch_bounds__(kValueThreads) attn_values_kernel(const AttnParams p)
{
    __shared__ float ew[kMaxGroup][kPosBlock];              // weights e_j of the block
    __shared__ double part[4][kMaxGroup][kHeadDim / 4 * 4];  // per position group partial sums
    __shared__ float gmax[kMaxGroup];
    __shared__ int last;
    const int tid = threadIdx.x;
    const int kv = blockIdx.x, blk = blockIdx.y;
    const int G = p.H / p.Hkv;
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int pos = read_pos(p);
    if (pos < 0)
        return;
    const int nact = pos / kPosBlock + 1;       // blocks holding positions 0 .. pos
    const int j0 = blk * kPosBlock;
    if (blk >= nact)
        return;
    const int j1 = min(j0 + kPosBlock, pos + 1);
    // the global maximum of each query head (exact: a max is order free)
    if (tid < 32 * G) {
        const int g = tid >> 5, lane = tid & 31;
        float m = -INFINITY;
        for (int b = lane; b < nact; b += 32)
            m = fmaxf(m, __ldcg(p.bmax + size_t(kv * G + g) * p.nblk + b));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0)
            gmax[g] = m;
    }
    __syncthreads();
    // the block's weights e_j = (float)exp((double)(s_j - m))
    for (int t = tid; t < G * kPosBlock; t += kValueThreads) {
        const int g = t / kPosBlock, jj = t % kPosBlock, j = j0 + jj;
        float e = 0.0f;
        if (j < j1) {
            const float sv = __ldcg(p.sc + size_t(kv * G + g) * p.T_max + j);
            e = __double2float_rn(exp(double(__fsub_rn(sv, gmax[g]))));
        }
        ew[g][jj] = e;
    }
    __syncthreads();
    // fp64 partial sums: thread (pg, c) takes dims 4c .. 4c + 3 of the
    // positions jj = pg, pg + 4, ... of the block (pg = tid / 32, c = tid % 32)
    const int pg = tid >> 5, c = tid & 31;
    const size_t head_base = size_t(kv) * p.T_max * kHeadDim;
    double acc[kMaxGroup][4];
#pragma unroll
    for (int g = 0; g < kMaxGroup; ++g)
#pragma unroll
        for (int x = 0; x < 4; ++x)
            acc[g][x] = 0.0;
#pragma unroll 4
    for (int jj = pg; jj < j1 - j0; jj += 4) {
        const uint2 ab = __ldcg(reinterpret_cast<const uint2 *>(p.cache_v + head_base + size_t(j0 + jj) * kHeadDim +
                                                                4 * c));
        const uint32_t a = ab.x, b = ab.y;
        const double vf[4] = {double(__uint_as_float(a << 16)), double(__uint_as_float(a & 0xffff0000u)),
                              double(__uint_as_float(b << 16)), double(__uint_as_float(b & 0xffff0000u))};
#pragma unroll
        for (int g = 0; g < kMaxGroup; ++g) {
            if (g >= G)
                break;
            const double e = double(ew[g][jj]);
#pragma unroll
            for (int x = 0; x < 4; ++x)
                acc[g][x] = __fma_rn(e, vf[x], acc[g][x]);     // exact products (fp32 x bf16)
        }
    }
#pragma unroll
    for (int g = 0; g < kMaxGroup; ++g) {
        if (g >= G)
            break;
#pragma unroll
        for (int x = 0; x < 4; ++x)
            part[pg][g][4 * c + x] = acc[g][x];
    }
    __syncthreads();
    for (int t = tid; t < G * kHeadDim; t += kValueThreads) {
        const int g = t / kHeadDim, d = t % kHeadDim;
        double num = 0.0;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4)
            num = __dadd_rn(num, part[q4][g][d]);
        p.bnum[(size_t(kv * G + g) * p.nblk + blk) * kHeadDim + d] = num;
    }
    for (int g = tid >> 5; g < G; g += kValueThreads / 32) {
        const int lane = tid & 31;
        double S = __dadd_rn(double(ew[g][lane]), double(ew[g][lane + 32]));   // e_j = 0 beyond j1
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            S = __dadd_rn(S, __shfl_xor_sync(0xffffffffu, S, o));
        if (lane == 0)
            p.bsum[size_t(kv * G + g) * p.nblk + blk] = S;
    }
    // the last block of this kv head to finish combines the blocks
    __threadfence();
    __syncthreads();
    if (tid == 0)
        last = atomicAdd(&p.ticket[kv], 1u) == unsigned(nact - 1);
    __syncthreads();
    if (!last)
        return;
    __threadfence();
    for (int t = tid; t < G * kHeadDim; t += kValueThreads) {
        const int g = t / kHeadDim, d = t % kHeadDim;
        const size_t hb = size_t(kv * G + g) * p.nblk;
        double num = 0.0, S = 0.0;
#pragma unroll 8
        for (int b = 0; b < nact; ++b) {
            num = __dadd_rn(num, __ldcg(p.bnum + (hb + b) * kHeadDim + d));
            S = __dadd_rn(S, __ldcg(p.bsum + hb + b));
        }
        const float o = __fdiv_rn(__double2float_rn(num), __double2float_rn(S));
        p.out[(kv * G + g) * kHeadDim + d] = __float2bfloat16_rn(o);
    }
    if (tid == 0)
        p.ticket[kv] = 0u;
}

// (cos, sin) of pos * base^(-2i / D) for every position and pair, fp64 then
// fp32 (the same values the attention kernels compute without a table).
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
    size_t sc, bmax, bsum, bnum, ticket, total;
};

AttnWs ws_layout(int H, int Hkv, int T_max)
{
    const int nblk = (T_max + kPosBlock - 1) / kPosBlock;
    auto up = [](size_t v) { return (v + 15) / 16 * 16; };
    AttnWs w{};
    w.sc = 0;
    w.bmax = up(w.sc + size_t(H) * T_max * 4);
    w.bsum = up(w.bmax + size_t(H) * nblk * 4);
    w.bnum = up(w.bsum + size_t(H) * nblk * 8);
    w.ticket = up(w.bnum + size_t(H) * nblk * kHeadDim * 8);
    w.total = up(w.ticket + size_t(Hkv) * 4);
    return w;
}

template <class K>
int launch_pdl(K kern, dim3 grid, int threads, cudaStream_t s, unsigned flags, const AttnParams &p)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(threads);
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
    p.sc = reinterpret_cast<float *>(base + w.sc);
    p.bmax = reinterpret_cast<float *>(base + w.bmax);
    p.bsum = reinterpret_cast<double *>(base + w.bsum);
    p.bnum = reinterpret_cast<double *>(base + w.bnum);
    p.ticket = reinterpret_cast<unsigned *>(base + w.ticket);
    p.status = di->status;
    const dim3 grid(unsigned(Hkv), unsigned(p.nblk));
    int st = launch_pdl(attn_scores_kernel, grid, kScoreThreads, s, flags, p);
    if (st)
        return st;
    // the values launch always follows the scores launch programmatically
    return launch_pdl(attn_values_kernel, grid, kValueThreads, s, BL_FLAG_PDL, p);
}

int launch_position_advance(int32_t *pos, cudaStream_t s)
{
    position_advance_kernel<<<1, 32, 0, s>>>(pos);
    return launch_status();
}

}  // namespace bl
