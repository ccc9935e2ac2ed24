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
//
// RMSNorm in front of the quantiser runs a second kernel, row_quant_kernel
// (RMSNorm; the "bit-floor" README, section "What's
// inside": rmsnorm.cu reduces the mean square and applies an rsqrt scale per
// element).  One warp per token, with no block-wide barrier on the token's
// path: lane 0 brings the whole row into a shared-memory slot of the warp
// with one bulk asynchronous copy, two slots per warp so the next token's
// row lands while this one is processed, and the warp makes its passes over
// the slot -- sum of squares (fp64, RMSNorm only), absmax of the normalised
// values, quantisation -- with warp shuffles for the reductions.  RMSNorm
// reading (identical on the CPU oracle): S = sum x^2 in fp64, ms =
// (float)(S / K), r = 1 / sqrt(ms + eps) (fp32, correctly rounded square root
// and division), h = (x * r) * g (two fp32 products); h then goes through
// the absmax quantiser above.  The fp64 sum's order differs from the
// oracle's, which can change ms only when S / K lies within about 1e-15
// (relative) of an fp32 rounding boundary.
#include <algorithm>

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
    uint4 raw[XT == BL_BF16 ? kQuantRegChunks : 1] = {};
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

// ---------------------------------------------------------------------------
// row_quant_kernel: one warp per token, rows staged in shared memory.

constexpr int kRowMaxWarps = 8;
constexpr int kRowSlots = 2;                 // row slots per warp (double buffering)
constexpr size_t kRowSmemBudget = 200 * 1024;  // dynamic shared memory per CTA, at most

struct RowQuantParams {
    const void *x;
    int64_t M, K, ldx;     // ldx in elements
    const void *gain;      // RMSNorm gain [K] (dtype gt), or NULL
    float eps;             // RMSNorm epsilon
    int8_t *q;
    float *d;
    int32_t *rowsum;
    int *status;
    int slots;             // row slots per warp (1 or 2)
};

// Eight consecutive gain values as fp32 (1.0 everywhere without a gain, which
// leaves (x * r) * 1 = x * r exact).
template <int GT>
__device__ __forceinline__ void gain8(const float *gs, int64_t k, float g[8])
{
    if constexpr (GT < 0) {
#pragma unroll
        for (int j = 0; j < 8; ++j)
            g[j] = 1.0f;
    } else {
        const float4 a = *reinterpret_cast<const float4 *>(gs + k);
        const float4 b = *reinterpret_cast<const float4 *>(gs + k + 4);
        g[0] = a.x; g[1] = a.y; g[2] = a.z; g[3] = a.w;
        g[4] = b.x; g[5] = b.y; g[6] = b.z; g[7] = b.w;
    }
}

// Eight elements of a row in shared memory as fp32.
template <int XT>
__device__ __forceinline__ void smem8(const unsigned char *row, int64_t k, float f[8])
{
    if constexpr (XT == BL_BF16) {
        bf16x8_to_f32(*reinterpret_cast<const uint4 *>(row + k * 2), f);
    } else {
        const float4 a = *reinterpret_cast<const float4 *>(row + k * 4);
        const float4 b = *reinterpret_cast<const float4 *>(row + k * 4 + 16);
        f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
        f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
    }
}

// XT: activation dtype; NORM: RMSNorm first; GT: gain dtype (-1: none).
// Dynamic shared memory: [gain as fp32, K floats, NORM with a gain only]
// [warps x slots row buffers of K * esz bytes] ; mbarriers are static.
template <int XT, bool NORM, int GT>
__global__ void __launch_bounds__(32 * kRowMaxWarps)
row_quant_kernel(const RowQuantParams p)
{
    extern __shared__ __align__(128) unsigned char smem_raw[];
    __shared__ __align__(8) uint64_t full[kRowMaxWarps][kRowSlots];
    __shared__ int abort_flag;
    constexpr int esz = XT == BL_BF16 ? 2 : 4;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int wpb = blockDim.x >> 5;
    const int64_t K = p.K;
    const uint32_t row_bytes = uint32_t(K * esz);
    const size_t gain_bytes = (NORM && GT >= 0) ? size_t(K) * 4 : 0;
    float *gs = reinterpret_cast<float *>(smem_raw);
    unsigned char *rows = smem_raw + gain_bytes;

    if (threadIdx.x == 0) {
        for (int w = 0; w < wpb; ++w)
            for (int b = 0; b < p.slots; ++b)
                mbar_init(smem_u32(&full[w][b]), 1);
        abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if constexpr (NORM && GT >= 0) {
        // the gain, once per CTA, as fp32
        for (int64_t k = threadIdx.x; k < K; k += blockDim.x)
            gs[k] = GT == BL_BF16 ? __bfloat162float(static_cast<const __nv_bfloat16 *>(p.gain)[k])
                                  : static_cast<const float *>(p.gain)[k];
    }
    __syncthreads();

    const int64_t stride = int64_t(gridDim.x) * wpb;
    const int64_t first = int64_t(blockIdx.x) * wpb + warp;
    const unsigned char *xb = static_cast<const unsigned char *>(p.x);
    const int64_t row_pitch = p.ldx * esz;
    auto slot_ptr = [&](int b) { return rows + (size_t(warp) * p.slots + b) * row_bytes; };
    auto issue = [&](int64_t m, int b) {
        // lane 0: the whole row of token m into slot b
        const uint32_t bar = smem_u32(&full[warp][b]);
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        mbar_arrive_tx(bar, row_bytes);
        bulk_load(smem_u32(slot_ptr(b)), xb + m * row_pitch, row_bytes, bar);
    };
    if (lane == 0)
        for (int b = 0; b < p.slots; ++b)
            if (first + b * stride < p.M)
                issue(first + b * stride, b);

    const int64_t chunks = K / 8;       // 8 elements per lane and step
    uint32_t phase = 0;                 // bit b: parity of slot b's next completion
    int b = 0;
    for (int64_t m = first; m < p.M; m += stride) {
        if (!__all_sync(0xffffffffu, mbar_wait_fast(smem_u32(&full[warp][b]), (phase >> b) & 1u,
                                                    &abort_flag, p.status)))
            break;
        phase ^= 1u << b;
        const unsigned char *row = slot_ptr(b);

        float r = 1.0f;
        if constexpr (NORM) {
            double S = 0.0;
            for (int64_t c = lane; c < chunks; c += 32) {
                float f[8];
                smem8<XT>(row, c * 8, f);
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    S = __dadd_rn(S, __dmul_rn(double(f[j]), double(f[j])));
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
                S = __dadd_rn(S, __shfl_xor_sync(0xffffffffu, S, o));
            const float ms = __double2float_rn(__ddiv_rn(S, double(K)));
            r = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, p.eps)));
        }
        auto h8 = [&](int64_t c, float h[8]) {
            smem8<XT>(row, c * 8, h);
            if constexpr (NORM) {
                float g[8];
                gain8<GT>(gs, c * 8, g);
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    h[j] = __fmul_rn(__fmul_rn(h[j], r), g[j]);
            }
        };
        float amax = 0.0f;
        for (int64_t c = lane; c < chunks; c += 32) {
            float h[8];
            h8(c, h);
#pragma unroll
            for (int j = 0; j < 8; ++j)
                amax = fmaxf(amax, fabsf(h[j]));
        }
        // maxima are >= 0 and finite (fmaxf from 0 drops NaN): their bit
        // patterns order like the values
        amax = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(amax)));
        const float a_eff = fmaxf(amax, kEps);
        const float s = __fdiv_rn(kQb, a_eff);
        int sum = 0;
        int8_t *qrow = p.q + m * K;
        for (int64_t c = lane; c < chunks; c += 32) {
            float h[8];
            h8(c, h);
            uint32_t lo = 0, hi = 0;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int t0 = quant1(h[j], s), t1 = quant1(h[j + 4], s);
                sum += t0 + t1;
                lo |= (uint32_t(t0) & 0xffu) << (8 * j);
                hi |= (uint32_t(t1) & 0xffu) << (8 * j);
            }
            *reinterpret_cast<uint2 *>(qrow + c * 8) = make_uint2(lo, hi);
        }
        sum = __reduce_add_sync(0xffffffffu, sum);
        if (lane == 0) {
            p.rowsum[m] = sum;
            p.d[m] = __fdiv_rn(a_eff, kQb);
        }
        // every lane is done with the slot: refill it with a later token
        __syncwarp();
        const int64_t next = m + int64_t(p.slots) * stride;
        if (lane == 0 && next < p.M)
            issue(next, b);
        b = (b + 1 == p.slots) ? 0 : b + 1;
    }
    // a warp that gave up waits (bounded) for the copies it still has in flight
    __syncwarp();
    if (lane == 0 && abort_flag) {
        volatile int no_abort = 0;
        for (int bb = 0; bb < p.slots; ++bb)
            mbar_wait(smem_u32(&full[warp][bb]), (phase >> bb) & 1u, &no_abort, p.status, 100000000ull);
    }
}

// Warps per CTA and row slots per warp for a row of row_bytes, within the
// shared-memory budget; false if even one slot does not fit.
bool row_geometry(size_t row_bytes, size_t gain_bytes, int *warps, int *slots)
{
    if (gain_bytes + row_bytes > kRowSmemBudget)
        return false;
    const size_t room = kRowSmemBudget - gain_bytes;
    *slots = room >= kRowSlots * row_bytes ? kRowSlots : 1;
    size_t w = room / (size_t(*slots) * row_bytes);
    *warps = int(w > size_t(kRowMaxWarps) ? kRowMaxWarps : w);
    return *warps >= 1;
}

template <int XT, bool NORM, int GT>
int launch_row_quant_t(const RowQuantParams &base, cudaStream_t s)
{
    const DeviceInfo *di = device_info();
    if (!di)
        return BL_ERR_CUDA;
    constexpr int esz = XT == BL_BF16 ? 2 : 4;
    const size_t row_bytes = size_t(base.K) * esz;
    const size_t gain_bytes = (NORM && GT >= 0) ? size_t(base.K) * 4 : 0;
    int warps = 0, slots = 0;
    if (!row_geometry(row_bytes, gain_bytes, &warps, &slots))
        return BL_ERR_SHAPE;
    RowQuantParams p = base;
    p.slots = slots;
    p.status = di->status;
    const size_t smem = gain_bytes + size_t(warps) * slots * row_bytes;
    auto kern = row_quant_kernel<XT, NORM, GT>;
    int per_sm = 0;
    int st = occupancy(reinterpret_cast<const void *>(kern), 32 * warps, smem, &per_sm);
    if (st)
        return st;
    if (per_sm < 1)
        return BL_ERR_SHAPE;
    const int64_t need = (base.M + warps - 1) / warps;
    const int64_t cap = int64_t(per_sm) * di->sm_count;
    const unsigned grid = unsigned(need < cap ? need : cap);
    kern<<<grid, 32 * warps, smem, s>>>(p);
    return launch_status();
}

template <int XT>
int launch_row_quant_x(const RowQuantParams &p, bool norm, int gt, cudaStream_t s)
{
    if (!norm)
        return launch_row_quant_t<XT, false, -1>(p, s);
    if (!p.gain)
        return launch_row_quant_t<XT, true, -1>(p, s);
    if (gt == BL_BF16)
        return launch_row_quant_t<XT, true, BL_BF16>(p, s);
    return launch_row_quant_t<XT, true, BL_F32>(p, s);
}

int launch_row_quant(const void *x, int xt, int64_t M, int64_t K, int64_t ldx, const void *gain,
                     int gt, float eps, bool norm, int8_t *q, float *d, int32_t *rowsum,
                     cudaStream_t s)
{
    RowQuantParams p{};
    p.x = x;
    p.M = M;
    p.K = K;
    p.ldx = ldx;
    p.gain = gain;
    p.eps = eps;
    p.q = q;
    p.d = d;
    p.rowsum = rowsum;
    if (xt == BL_BF16)
        return launch_row_quant_x<BL_BF16>(p, norm, gt, s);
    return launch_row_quant_x<BL_F32>(p, norm, gt, s);
}

// Many short rows (bf16, K <= 3072): one warp per token over a grid of a
// few CTAs per SM, each warp walking tokens gw, gw + warps, ...  The whole
// row sits in the lanes' registers (CH 16-byte vectors per lane), both
// reductions are warp shuffles, and there is no block barrier: a CTA per
// token (above) is bound by how fast the GPU starts CTAs when a row is only
// a few KB.  Same arithmetic as quantize_act_kernel.
constexpr int kRowsThreads = 256;

template <int CH>
__global__ void __launch_bounds__(kRowsThreads, 2)
quantize_rows_bf16_kernel(const __nv_bfloat16 *__restrict__ x, int64_t M, int64_t K, int64_t ldx,
                          int8_t *__restrict__ q, float *__restrict__ d, int32_t *__restrict__ rowsum)
{
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = int64_t(gridDim.x) * (kRowsThreads / 32);
    const int chunks = int(K / 8);
    for (int64_t m = (int64_t(blockIdx.x) * kRowsThreads + threadIdx.x) >> 5; m < M; m += nwarps) {
        const __nv_bfloat16 *xr = x + m * ldx;
        uint4 raw[CH];
#pragma unroll
        for (int i = 0; i < CH; ++i) {
            const int c = lane + 32 * i;
            raw[i] = c < chunks ? ld_ro_v4(xr + int64_t(c) * 8) : make_uint4(0, 0, 0, 0);
        }
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < CH; ++i) {
            float f[8];
            bf16x8_to_f32(raw[i], f);
#pragma unroll
            for (int j = 0; j < 8; ++j)
                amax = fmaxf(amax, fabsf(f[j]));
        }
        // per-lane maxima are finite and >= 0: their bit patterns order like the values
        amax = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(amax)));
        const float a_eff = fmaxf(amax, kEps);
        const float s = __fdiv_rn(kQb, a_eff);
        int sum = 0;
        int8_t *qrow = q + m * K;
#pragma unroll
        for (int i = 0; i < CH; ++i) {
            const int c = lane + 32 * i;
            if (c < chunks) {
                float f[8];
                bf16x8_to_f32(raw[i], f);
                uint32_t lo = 0, hi = 0;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int t0 = quant1(f[j], s), t1 = quant1(f[j + 4], s);
                    sum += t0 + t1;
                    lo |= (uint32_t(t0) & 0xffu) << (8 * j);
                    hi |= (uint32_t(t1) & 0xffu) << (8 * j);
                }
                *reinterpret_cast<uint2 *>(qrow + int64_t(c) * 8) = make_uint2(lo, hi);
            }
        }
        sum = __reduce_add_sync(0xffffffffu, sum);
        if (lane == 0) {
            rowsum[m] = sum;
            d[m] = __fdiv_rn(a_eff, kQb);
        }
    }
}

template <int CH>
int launch_rows(const void *x, int64_t M, int64_t K, int64_t ldx, int8_t *q, float *d, int32_t *rowsum,
                cudaStream_t s)
{
    const DeviceInfo *di = device_info();
    if (!di)
        return BL_ERR_CUDA;
    const int64_t warps_needed = M;
    const int64_t cap = int64_t(di->sm_count) * 2;   // two CTAs of eight warps per SM
    const int64_t grid = std::min<int64_t>(cap, (warps_needed + 7) / 8);
    quantize_rows_bf16_kernel<CH><<<unsigned(grid), kRowsThreads, 0, s>>>(
        static_cast<const __nv_bfloat16 *>(x), M, K, ldx, q, d, rowsum);
    return launch_status();
}

}  // namespace

// Plain quantisation runs the CTA-per-token kernel: measured against the
// warp-per-token kernel at 8192 tokens it was as fast at K = 2560 and faster
// at K = 6912 (more warps per SM with the row in registers).
int launch_quantize_act(const void *x, int xt, int64_t M, int64_t K, int64_t ldx,
                        int8_t *q, float *d, int32_t *rowsum, cudaStream_t s)
{
    // many tokens of short bf16 rows: a warp per token
    if (xt == BL_BF16 && M >= 1024 && K <= 2048)
        return launch_rows<8>(x, M, K, ldx, q, d, rowsum, s);
    if (xt == BL_BF16 && M >= 1024 && K <= 3072)
        return launch_rows<12>(x, M, K, ldx, q, d, rowsum, s);
    dim3 grid(static_cast<unsigned>(M));
    if (xt == BL_BF16)
        quantize_act_kernel<BL_BF16><<<grid, kQuantThreads, 0, s>>>(x, K, ldx, q, d, rowsum);
    else
        quantize_act_kernel<BL_F32><<<grid, kQuantThreads, 0, s>>>(x, K, ldx, q, d, rowsum);
    return launch_status();
}

int launch_rmsnorm_quantize_act(const void *x, int xt, int64_t M, int64_t K, int64_t ldx,
                                const void *gain, int gt, float eps, int8_t *q, float *d,
                                int32_t *rowsum, cudaStream_t s)
{
    return launch_row_quant(x, xt, M, K, ldx, gain, gt, eps, true, q, d, rowsum, s);
}

bool rmsnorm_quantize_fits(int xt, int64_t K, bool has_gain)
{
    int w = 0, sl = 0;
    return row_geometry(size_t(K) * (xt == BL_BF16 ? 2 : 4), has_gain ? size_t(K) * 4 : 0, &w, &sl);
}

}  // namespace bl
