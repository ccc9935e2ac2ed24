// quant.cu -- per-token absmax int8 activation quantisation.
//
// "How to Run BitNet Inference on GPU Using CUDA Kernels: A Complete Guide",
// section "Understanding the Two-Phase Architecture": the decode linear
// quantises its inputs to INT8 with scaling factors.  Per token m:
//   a_m = max(max_k |x|, 1e-5);  s_m = 127 / a_m;  q = clamp(rint(x s_m))
//   d_m = a_m / 127;  rowsum_m = sum_k q.
//
// One CTA per token.  The token's row is read once into registers (16-byte
// vectors: raw bf16, eight elements each, or fp32 as floats), reduced for the
// absmax, quantised from the registers and written as 8-byte int8 vectors; a
// second block reduction gives the row sum.  Rows longer than the register
// budget are read a second time (from L1/L2).  HBM-bound: M*K*(2 + 1) bytes
// for bf16 input.  Keeping bf16 rows raw halves their registers, so more CTAs
// (and more bytes of x) are in flight per SM: the kernel's time per token is
// mostly load latency.
#include "bl_common.cuh"

namespace bl {
namespace {

constexpr int kQuantThreads = 128;
constexpr int kQuantRegChunks = 8;  // 8-element chunks kept in registers per thread (K <= 8192)

__device__ __forceinline__ void bf16x8_to_f32(const uint4 v, float f[8])
{
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

template <int XT>
__global__ void __launch_bounds__(kQuantThreads)
quantize_act_kernel(const void *__restrict__ x, int64_t K, int64_t ldx,
                    int8_t *__restrict__ q, float *__restrict__ d,
                    int32_t *__restrict__ rowsum)
{
    __shared__ float s_red[kQuantThreads / 32];
    __shared__ int s_sum[kQuantThreads / 32];
    const int64_t m = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t chunks = K / 8;
    const int64_t xrow = m * ldx;
    const bool in_regs = chunks <= int64_t(kQuantThreads) * kQuantRegChunks;
    // register copy of the row: raw bf16 vectors, or eight floats per chunk
    constexpr int kRegF = XT == BL_BF16 ? 1 : 8;
    uint4 raw[XT == BL_BF16 ? kQuantRegChunks : 1];
    float v[XT == BL_BF16 ? 1 : kQuantRegChunks][kRegF];
    auto chunk_f32 = [&](int i, float f[8]) {
        if constexpr (XT == BL_BF16) {
            bf16x8_to_f32(raw[i], f);
        } else {
#pragma unroll
            for (int j = 0; j < 8; ++j)
                f[j] = v[i][j];
        }
    };

    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < kQuantRegChunks; ++i) {
        const int64_t c = tid + int64_t(i) * kQuantThreads;
        if (in_regs && c < chunks) {
            float f[8];
            if constexpr (XT == BL_BF16) {
                raw[i] = ld_ro_v4(static_cast<const __nv_bfloat16 *>(x) + xrow + c * 8);
                bf16x8_to_f32(raw[i], f);
            } else {
                load8<XT>(x, xrow + c * 8, f);
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    v[i][j] = f[j];
            }
#pragma unroll
            for (int j = 0; j < 8; ++j)
                amax = fmaxf(amax, fabsf(f[j]));
        }
    }
    if (!in_regs) {
        for (int64_t c = tid; c < chunks; c += kQuantThreads) {
            float f[8];
            load8<XT>(x, xrow + c * 8, f);
#pragma unroll
            for (int j = 0; j < 8; ++j)
                amax = fmaxf(amax, fabsf(f[j]));
        }
    }
    // per-thread maxima are finite and >= 0 (fmaxf from 0 drops NaN), so
    // their bit patterns order like the values
    amax = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(amax)));
    if (lane == 0)
        s_red[warp] = amax;
    __syncthreads();
    float a = s_red[0];
#pragma unroll
    for (int w = 1; w < kQuantThreads / 32; ++w)
        a = fmaxf(a, s_red[w]);
    const float a_eff = fmaxf(a, kEps);
    const float s = __fdiv_rn(kQb, a_eff);

    int sum = 0;
    int8_t *qrow = q + m * K;
    auto emit = [&](int64_t c, const float f[8]) {
        uint32_t lo = 0, hi = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            int t0 = quant1(f[j], s), t1 = quant1(f[j + 4], s);
            sum += t0 + t1;
            lo |= (uint32_t(t0) & 0xffu) << (8 * j);
            hi |= (uint32_t(t1) & 0xffu) << (8 * j);
        }
        *reinterpret_cast<uint2 *>(qrow + c * 8) = make_uint2(lo, hi);
    };
    if (in_regs) {
#pragma unroll
        for (int i = 0; i < kQuantRegChunks; ++i) {
            const int64_t c = tid + int64_t(i) * kQuantThreads;
            if (c < chunks) {
                float f[8];
                chunk_f32(i, f);
                emit(c, f);
            }
        }
    } else {
        for (int64_t c = tid; c < chunks; c += kQuantThreads) {
            float f[8];
            load8<XT>(x, xrow + c * 8, f);
            emit(c, f);
        }
    }
    sum = __reduce_add_sync(0xffffffffu, sum);
    if (lane == 0)
        s_sum[warp] = sum;
    __syncthreads();
    if (tid == 0) {
        int r = 0;
#pragma unroll
        for (int w = 0; w < kQuantThreads / 32; ++w)
            r += s_sum[w];
        rowsum[m] = r;
        d[m] = __fdiv_rn(a_eff, kQb);
    }
}

}  // namespace

int launch_quantize_act(const void *x, int xt, int64_t M, int64_t K, int64_t ldx,
                        int8_t *q, float *d, int32_t *rowsum, cudaStream_t s)
{
    dim3 grid(static_cast<unsigned>(M));
    if (xt == BL_BF16)
        quantize_act_kernel<BL_BF16><<<grid, kQuantThreads, 0, s>>>(x, K, ldx, q, d, rowsum);
    else
        quantize_act_kernel<BL_F32><<<grid, kQuantThreads, 0, s>>>(x, K, ldx, q, d, rowsum);
    return launch_status();
}

}  // namespace bl
