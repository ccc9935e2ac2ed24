// quant.cu -- per-token absmax int8 activation quantisation.
//
// "How to Run BitNet Inference on GPU Using CUDA Kernels: A Complete Guide",
// section "Understanding the Two-Phase Architecture": the decode linear
// quantises its inputs to INT8 with scaling factors.  Per token m:
//   a_m = max(max_k |x|, 1e-5);  s_m = 127 / a_m;  q = clamp(rint(x s_m))
//   d_m = a_m / 127;  rowsum_m = sum_k q.
//
// One CTA per token.  The token's row is read once into registers (16-byte
// vectors, eight elements each), reduced for the absmax, quantised from the
// registers and written as 8-byte int8 vectors; a second block reduction gives
// the row sum.  Rows longer than the register budget are read a second time
// (from L1/L2).  HBM-bound: M*K*(2 + 1) bytes for bf16 input.
#include "bl_common.cuh"

namespace bl {
namespace {

constexpr int kQuantThreads = 256;
constexpr int kQuantRegChunks = 4;  // 8-element chunks kept in registers per thread

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

    float v[kQuantRegChunks][8];
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < kQuantRegChunks; ++i) {
        const int64_t c = tid + int64_t(i) * kQuantThreads;
        if (in_regs && c < chunks) {
            load8<XT>(x, xrow + c * 8, v[i]);
#pragma unroll
            for (int j = 0; j < 8; ++j)
                amax = fmaxf(amax, fabsf(v[i][j]));
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
    amax = warp_max(amax);
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
            if (c < chunks)
                emit(c, v[i]);
        }
    } else {
        for (int64_t c = tid; c < chunks; c += kQuantThreads) {
            float f[8];
            load8<XT>(x, xrow + c * 8, f);
            emit(c, f);
        }
    }
    sum = warp_sum(sum);
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
