// binary.cu -- binary (1-bit) weight packer and XNOR / popcount GEMV.
//
// "bit-floor" README, section "The core math": each weight row is packed into
// ceil(K/64) 64-bit words and y[i] = scale_w * scale_x *
// (2 * POPCNT(XNOR(W_i, x)) - K), with no floating point before the final
// scale multiply; section "What's inside": absmax scale for binary weights.
// Bit j of word w holds k = 64 w + j and is set for negative values.
//
// The GEMV streams N*K/8 bytes.  Persistent CTAs of 256 threads; each CTA
// packs the sign bits of x into shared memory in its prologue (warp ballots)
// and takes max |x| with a block reduction.  One warp handles one row at a
// time: lane l reads 64-bit words l, l+32, ... of the row (coalesced 256-byte
// segments) kRowsInFlight rows ahead, XNORs against its own words of x held
// in registers, popcounts, and the warp reduces with shuffles.
#include "bl_common.cuh"

namespace bl {
namespace {

constexpr int kPackThreads = 256;

// One warp per (row, 64-bit word pair): two ballots of 32 consecutive k make
// one 64-bit word.  max |W| is folded with an atomic max on the float's bit
// pattern (monotone for non-negative floats, order-independent, exact).
template <int WT>
__global__ void __launch_bounds__(kPackThreads)
binary_pack_kernel(const void *__restrict__ W, int64_t N, int64_t K,
                   unsigned long long *__restrict__ Wb, unsigned int *__restrict__ s_w_bits)
{
    const int lane = threadIdx.x & 31;
    const int64_t words = K / 64;
    const int64_t total = N * words;
    const int64_t warp_global = (int64_t(blockIdx.x) * kPackThreads + threadIdx.x) >> 5;
    const int64_t warps = (int64_t(gridDim.x) * kPackThreads) >> 5;
    float amax = 0.0f;
    for (int64_t i = warp_global; i < total; i += warps) {
        const int64_t n = i / words, w = i % words;
        const int64_t base = n * K + w * 64;
        float v0, v1;
        if (WT == BL_BF16) {
            v0 = __bfloat162float(static_cast<const __nv_bfloat16 *>(W)[base + lane]);
            v1 = __bfloat162float(static_cast<const __nv_bfloat16 *>(W)[base + 32 + lane]);
        } else {
            v0 = static_cast<const float *>(W)[base + lane];
            v1 = static_cast<const float *>(W)[base + 32 + lane];
        }
        amax = fmaxf(amax, fmaxf(fabsf(v0), fabsf(v1)));
        const unsigned lo = __ballot_sync(0xffffffffu, v0 < 0.0f);
        const unsigned hi = __ballot_sync(0xffffffffu, v1 < 0.0f);
        if (lane == 0)
            Wb[i] = (static_cast<unsigned long long>(hi) << 32) | lo;
    }
    amax = warp_max(amax);
    if (lane == 0)
        atomicMax(s_w_bits, __float_as_uint(amax));
}

constexpr int kGemvThreads = 256;
constexpr int kMaxWordsPerLane = 32;  // K <= 32 * 64 * 32 = 65536
// Rows whose loads are in flight per warp: fewer for long rows (registers).
template <int WPL>
constexpr int rows_in_flight() { return WPL <= 4 ? 4 : (WPL <= 8 ? 2 : 1); }

template <int XT, int WPL>
__global__ void __launch_bounds__(kGemvThreads)
binary_gemv_kernel(const unsigned long long *__restrict__ Wb, const float *__restrict__ s_w,
                   int64_t N, int64_t K, const void *__restrict__ x, void *__restrict__ y,
                   int yt, int32_t *__restrict__ acc_dbg)
{
    __shared__ unsigned long long xb_s[kMaxWordsPerLane * 32];
    __shared__ float red[kGemvThreads / 32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int words = int(K / 64);

    // prologue: sign bits of x (two ballots per word) and max |x|
    float amax = 0.0f;
    for (int w = warp; w < words; w += kGemvThreads / 32) {
        float v0, v1;
        if (XT == BL_BF16) {
            v0 = __bfloat162float(static_cast<const __nv_bfloat16 *>(x)[w * 64 + lane]);
            v1 = __bfloat162float(static_cast<const __nv_bfloat16 *>(x)[w * 64 + 32 + lane]);
        } else {
            v0 = static_cast<const float *>(x)[w * 64 + lane];
            v1 = static_cast<const float *>(x)[w * 64 + 32 + lane];
        }
        amax = fmaxf(amax, fmaxf(fabsf(v0), fabsf(v1)));
        const unsigned lo = __ballot_sync(0xffffffffu, v0 < 0.0f);
        const unsigned hi = __ballot_sync(0xffffffffu, v1 < 0.0f);
        if (lane == 0)
            xb_s[w] = (static_cast<unsigned long long>(hi) << 32) | lo;
    }
    amax = warp_max(amax);
    if (lane == 0)
        red[warp] = amax;
    __syncthreads();
    float s_x = red[0];
#pragma unroll
    for (int w = 1; w < kGemvThreads / 32; ++w)
        s_x = fmaxf(s_x, red[w]);
    const float scale = __fmul_rn(s_w[0], s_x);

    unsigned long long xr[WPL];
#pragma unroll
    for (int j = 0; j < WPL; ++j) {
        const int w = lane + 32 * j;
        xr[j] = w < words ? xb_s[w] : 0ull;
    }

    constexpr int kRowsInFlight = rows_in_flight<WPL>();
    const int64_t warp_global = int64_t(blockIdx.x) * (kGemvThreads / 32) + warp;
    const int64_t nwarps = int64_t(gridDim.x) * (kGemvThreads / 32);
    for (int64_t n0 = warp_global * kRowsInFlight; n0 < N; n0 += nwarps * kRowsInFlight) {
        unsigned long long wv[kRowsInFlight][WPL];
#pragma unroll
        for (int r = 0; r < kRowsInFlight; ++r)
#pragma unroll
            for (int j = 0; j < WPL; ++j) {
                const int w = lane + 32 * j;
                const int64_t n = n0 + r;
                if (n < N && w < words) {
                    const uint2 v = ld_stream_v2(Wb + n * words + w);
                    wv[r][j] = (static_cast<unsigned long long>(v.y) << 32) | v.x;
                } else {
                    wv[r][j] = 0ull;
                }
            }
#pragma unroll
        for (int r = 0; r < kRowsInFlight; ++r) {
            int pc = 0;
#pragma unroll
            for (int j = 0; j < WPL; ++j) {
                const int w = lane + 32 * j;
                if (w < words)
                    pc += __popcll(~(wv[r][j] ^ xr[j]));
            }
            pc = warp_sum(pc);
            const int64_t n = n0 + r;
            if (lane == 0 && n < N) {
                const int acc = 2 * pc - int(K);
                if (acc_dbg)
                    acc_dbg[n] = acc;
                store_y(y, yt, n, __fmul_rn(static_cast<float>(acc), scale));
            }
        }
    }
}

template <int XT, int WPL>
int launch_binary_gemv_t(const uint64_t *Wb, const float *s_w, int64_t N, int64_t K,
                         const void *x, void *y, int yt, int32_t *acc_dbg, cudaStream_t s)
{
    auto kern = binary_gemv_kernel<XT, WPL>;
    const DeviceInfo *di = device_info();
    if (!di)
        return BL_ERR_CUDA;
    int per_sm = 0;
    int st = occupancy(reinterpret_cast<const void *>(kern), kGemvThreads, 0, &per_sm);
    if (st)
        return st;
    const int64_t rows_per_cta = int64_t(kGemvThreads / 32) * rows_in_flight<WPL>();
    int64_t grid = (N + rows_per_cta - 1) / rows_per_cta;
    const int64_t cap = int64_t(di->sm_count) * (per_sm > 0 ? per_sm : 1);
    if (grid > cap)
        grid = cap;
    kern<<<unsigned(grid), kGemvThreads, 0, s>>>(
        reinterpret_cast<const unsigned long long *>(Wb), s_w, N, K, x, y, yt, acc_dbg);
    return launch_status();
}

template <int XT>
int dispatch_wpl(const uint64_t *Wb, const float *s_w, int64_t N, int64_t K, const void *x,
                 void *y, int yt, int32_t *acc_dbg, cudaStream_t s)
{
    const int64_t words = K / 64;
    if (words <= 32)
        return launch_binary_gemv_t<XT, 1>(Wb, s_w, N, K, x, y, yt, acc_dbg, s);
    if (words <= 64)
        return launch_binary_gemv_t<XT, 2>(Wb, s_w, N, K, x, y, yt, acc_dbg, s);
    if (words <= 128)
        return launch_binary_gemv_t<XT, 4>(Wb, s_w, N, K, x, y, yt, acc_dbg, s);
    if (words <= 256)
        return launch_binary_gemv_t<XT, 8>(Wb, s_w, N, K, x, y, yt, acc_dbg, s);
    if (words <= 512)
        return launch_binary_gemv_t<XT, 16>(Wb, s_w, N, K, x, y, yt, acc_dbg, s);
    return launch_binary_gemv_t<XT, 32>(Wb, s_w, N, K, x, y, yt, acc_dbg, s);
}

}  // namespace

int launch_binary_pack(const void *W, int wt, int64_t N, int64_t K, uint64_t *Wb,
                       float *s_w, cudaStream_t s)
{
    int st = cuda_status(cudaMemsetAsync(s_w, 0, sizeof(float), s));
    if (st)
        return st;
    const DeviceInfo *di = device_info();
    if (!di)
        return BL_ERR_CUDA;
    const int64_t warps_needed = N * (K / 64);
    int64_t blocks = (warps_needed + kPackThreads / 32 - 1) / (kPackThreads / 32);
    const int64_t cap = int64_t(di->sm_count) * 8;
    if (blocks > cap)
        blocks = cap;
    auto *bits = reinterpret_cast<unsigned int *>(s_w);
    auto *out = reinterpret_cast<unsigned long long *>(Wb);
    if (wt == BL_BF16)
        binary_pack_kernel<BL_BF16><<<unsigned(blocks), kPackThreads, 0, s>>>(W, N, K, out, bits);
    else
        binary_pack_kernel<BL_F32><<<unsigned(blocks), kPackThreads, 0, s>>>(W, N, K, out, bits);
    return launch_status();
}

int launch_binary_gemv(const uint64_t *Wb, const float *s_w, int64_t N, int64_t K,
                       const void *x, int xt, void *y, int yt, int32_t *acc_dbg,
                       cudaStream_t s)
{
    if (xt == BL_BF16)
        return dispatch_wpl<BL_BF16>(Wb, s_w, N, K, x, y, yt, acc_dbg, s);
    return dispatch_wpl<BL_F32>(Wb, s_w, N, K, x, y, yt, acc_dbg, s);
}

}  // namespace bl
