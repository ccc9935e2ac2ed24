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
// Design: one CTA per query head (grouped heads: kv head h / (H / Hkv)),
// 256 threads.  The CTA rotates its query and its kv head's new key, and the
// first CTA of each group appends the key and value at position pos (a device
// scalar, read after the dependency wait, so that a CUDA graph can replay the
// step for successive tokens).  Eight warps split the positions for the
// scores (lane l: dimensions 4l .. 4l + 3, fp64 partial sums reduced with
// shuffles) and again for the weighted sum of values (per-warp fp64 sums of
// all 128 dimensions, combined in shared memory).  A position outside the
// cache records BL_ERR_SHAPE in the device status word and writes nothing.
#include "bl_common.cuh"

namespace bl {
namespace {

constexpr int kAttnThreads = 256;
constexpr int kAttnWarps = kAttnThreads / 32;
constexpr int kHeadDim = 128;

struct AttnParams {
    const __nv_bfloat16 *q, *k, *v;       // [H*D], [Hkv*D], [Hkv*D]
    __nv_bfloat16 *cache_k, *cache_v;     // [Hkv][T_max][D]
    const int32_t *pos;
    int H, Hkv, T_max;
    double rope_base;
    __nv_bfloat16 *out;                   // [H*D]
    int *status;
};

__device__ __forceinline__ float bf16_bits_f32(uint32_t b) { return __uint_as_float(b << 16); }

__device__ __forceinline__ uint32_t f32_bf16_bits(float v)
{
    return __bfloat16_as_ushort(__float2bfloat16_rn(v));
}

// Four consecutive bf16 values (8 bytes) as fp32.
__device__ __forceinline__ void ld4_bf16(const __nv_bfloat16 *p, float (&f)[4])
{
    uint32_t a, b;
    asm volatile("ld.global.cg.v2.u32 {%0,%1}, [%2];" : "=r"(a), "=r"(b) : "l"(p) : "memory");
    f[0] = __uint_as_float(a << 16);
    f[1] = __uint_as_float(a & 0xffff0000u);
    f[2] = __uint_as_float(b << 16);
    f[3] = __uint_as_float(b & 0xffff0000u);
}

// Rotate pair i of a head vector x (bf16) at position pos; returns the two
// rotated values rounded to bf16 (as fp32).
__device__ __forceinline__ void rope_pair(const __nv_bfloat16 *x, int i, int pos, double base, float &o0, float &o1)
{
    const double ang = double(pos) * pow(base, -double(2 * i) / double(kHeadDim));
    const float c = __double2float_rn(cos(ang)), s = __double2float_rn(sin(ang));
    const float a = bf16_bits_f32(ld_dep_u16(x + 2 * i)), b = bf16_bits_f32(ld_dep_u16(x + 2 * i + 1));
    const float r0 = __fsub_rn(__fmul_rn(a, c), __fmul_rn(b, s));
    const float r1 = __fadd_rn(__fmul_rn(a, s), __fmul_rn(b, c));
    o0 = bf16_bits_f32(f32_bf16_bits(r0));
    o1 = bf16_bits_f32(f32_bf16_bits(r1));
}

__device__ __forceinline__ double warp_sum_f64(double v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v = __dadd_rn(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__global__ void __launch_bounds__(kAttnThreads) attention_decode_kernel(const AttnParams p)
{
    extern __shared__ __align__(16) float attn_smem[];
    float *qs = attn_smem;                    // rotated query [D]
    float *ks = qs + kHeadDim;                // rotated new key [D]
    float *vs = ks + kHeadDim;                // new value [D]
    double *red = reinterpret_cast<double *>(vs + kHeadDim);   // [warps][D] partial sums
    float *wred = reinterpret_cast<float *>(red + kAttnWarps * kHeadDim);  // [warps]
    double *dred = reinterpret_cast<double *>(wred + 2 * kAttnWarps);      // [warps]
    float *sc = reinterpret_cast<float *>(dred + kAttnWarps);             // scores [T]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int h = blockIdx.x;
    const int group = p.H / p.Hkv;
    const int kv = h / group;

    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int pos = int(ld_dep_u32(p.pos));
    if (pos < 0 || pos >= p.T_max) {
        if (tid == 0)
            atomicExch(p.status, BL_ERR_SHAPE);
        return;
    }
    const int T = pos + 1;

    // ---- RoPE on the query and the new key; the new value as it is
    if (tid < kHeadDim / 2) {
        float a, b;
        rope_pair(p.q + h * kHeadDim, tid, pos, p.rope_base, a, b);
        qs[2 * tid] = a;
        qs[2 * tid + 1] = b;
        rope_pair(p.k + kv * kHeadDim, tid, pos, p.rope_base, a, b);
        ks[2 * tid] = a;
        ks[2 * tid + 1] = b;
    } else if (tid < kHeadDim / 2 + kHeadDim) {
        const int d = tid - kHeadDim / 2;
        vs[d] = bf16_bits_f32(ld_dep_u16(p.v + kv * kHeadDim + d));
    }
    __syncthreads();
    const size_t head_base = size_t(kv) * p.T_max * kHeadDim;
    if (h % group == 0 && tid < kHeadDim) {
        // the group's first CTA appends the key and value at pos
        p.cache_k[head_base + size_t(pos) * kHeadDim + tid] = __float2bfloat16_rn(ks[tid]);
        p.cache_v[head_base + size_t(pos) * kHeadDim + tid] = __float2bfloat16_rn(vs[tid]);
    }

    // ---- scores: warp w takes positions w, w + 8, ...; lane l dims 4l .. 4l+3
    const float scale = __double2float_rn(1.0 / sqrt(double(kHeadDim)));
    double qd[4];
#pragma unroll
    for (int e = 0; e < 4; ++e)
        qd[e] = double(qs[4 * lane + e]);
    float mloc = -INFINITY;
    for (int j = warp; j < T; j += kAttnWarps) {
        float kf[4];
        if (j == pos) {
#pragma unroll
            for (int e = 0; e < 4; ++e)
                kf[e] = ks[4 * lane + e];
        } else {
            ld4_bf16(p.cache_k + head_base + size_t(j) * kHeadDim + 4 * lane, kf);
        }
        double dot = 0.0;
#pragma unroll
        for (int e = 0; e < 4; ++e)
            dot = __fma_rn(qd[e], double(kf[e]), dot);     // exact products of bf16 values
        dot = warp_sum_f64(dot);
        const float s = __fmul_rn(__double2float_rn(dot), scale);
        if (lane == 0)
            sc[j] = s;
        mloc = fmaxf(mloc, s);
    }
    if (lane == 0)
        wred[warp] = mloc;
    __syncthreads();
    float m = wred[0];
#pragma unroll
    for (int w = 1; w < kAttnWarps; ++w)
        m = fmaxf(m, wred[w]);

    // ---- softmax weights and their fp64 sum
    double sloc = 0.0;
    for (int j = tid; j < T; j += kAttnThreads) {
        const float e = __double2float_rn(exp(double(__fsub_rn(sc[j], m))));
        sc[j] = e;
        sloc = __dadd_rn(sloc, double(e));
    }
    sloc = warp_sum_f64(sloc);
    if (lane == 0)
        dred[warp] = sloc;
    __syncthreads();
    double S = 0.0;
#pragma unroll
    for (int w = 0; w < kAttnWarps; ++w)
        S = __dadd_rn(S, dred[w]);
    const float Sf = __double2float_rn(S);

    // ---- weighted sum of values: warp w positions w, w + 8, ...; lane l dims 4l .. 4l+3
    double acc[4] = {0.0, 0.0, 0.0, 0.0};
    for (int j = warp; j < T; j += kAttnWarps) {
        float vf[4];
        if (j == pos) {
#pragma unroll
            for (int e = 0; e < 4; ++e)
                vf[e] = vs[4 * lane + e];
        } else {
            ld4_bf16(p.cache_v + head_base + size_t(j) * kHeadDim + 4 * lane, vf);
        }
        const double e = double(sc[j]);
#pragma unroll
        for (int x = 0; x < 4; ++x)
            acc[x] = __fma_rn(e, double(vf[x]), acc[x]);     // exact products (fp32 x bf16)
    }
#pragma unroll
    for (int x = 0; x < 4; ++x)
        red[warp * kHeadDim + 4 * lane + x] = acc[x];
    __syncthreads();
    if (tid < kHeadDim) {
        double num = 0.0;
#pragma unroll
        for (int w = 0; w < kAttnWarps; ++w)
            num = __dadd_rn(num, red[w * kHeadDim + tid]);
        const float o = __fdiv_rn(__double2float_rn(num), Sf);
        p.out[h * kHeadDim + tid] = __float2bfloat16_rn(o);
    }
}

__global__ void position_advance_kernel(int32_t *pos)
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (threadIdx.x == 0)
        pos[0] += 1;
}

}  // namespace

size_t attention_smem_bytes(int T_max)
{
    return size_t(3 * kHeadDim) * 4 + size_t(kAttnWarps) * kHeadDim * 8 + size_t(2 * kAttnWarps) * 4 +
           size_t(kAttnWarps) * 8 + size_t(T_max) * 4;
}

int launch_attention_decode(const void *q, const void *k, const void *v, void *cache_k, void *cache_v,
                            const int32_t *pos, int H, int Hkv, int D, int T_max, double rope_base,
                            void *out, unsigned flags, cudaStream_t s)
{
    const DeviceInfo *di = device_info();
    if (!di)
        return BL_ERR_CUDA;
    if (D != kHeadDim)
        return BL_ERR_SHAPE;
    const size_t smem = attention_smem_bytes(T_max);
    int per_sm = 0;
    int st = occupancy(reinterpret_cast<const void *>(attention_decode_kernel), kAttnThreads, smem, &per_sm);
    if (st)
        return st;
    if (per_sm < 1)
        return BL_ERR_SHAPE;
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
    p.rope_base = rope_base;
    p.out = static_cast<__nv_bfloat16 *>(out);
    p.status = di->status;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(H));
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
    return cuda_status(cudaLaunchKernelEx(&cfg, attention_decode_kernel, p));
}

int launch_position_advance(int32_t *pos, cudaStream_t s)
{
    position_advance_kernel<<<1, 32, 0, s>>>(pos);
    return launch_status();
}

}  // namespace bl
