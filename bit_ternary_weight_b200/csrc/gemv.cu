// gemv.cu -- ternary decode GEMV for 1 <= M <= 16 tokens (M = 1 is decode).
//
// "How to Run BitNet Inference on GPU Using CUDA Kernels: A Complete Guide",
// sections "Understanding the Two-Phase Architecture" and "Key Components and
// Source Code Architecture": decode runs an INT8-activation x INT2-weight
// linear and is memory-bound.  "bit-floor" README, section "The core math":
// integer inner loop, floating point only in the final scale multiply.
//
// Design (B200): the weight stream N*K/4 bytes is the whole cost.
//   * Persistent grid, one or two 512-thread CTAs per SM.  Each CTA owns a
//     contiguous range of 8-row groups, i.e. one contiguous byte range of the
//     TL array, so the per-SM byte counts differ by at most one row group.
//   * A row group's slab (K/64 chunks x 8 rows x 16 B) is split into 512-byte
//     pieces; one warp-wide 16-byte load per lane reads one piece: lane l gets
//     row l%8, chunk 4p + l/8.  Loads bypass L1 (read once) and are issued
//     kUnroll pieces ahead of the math.
//   * Teams of T warps share a row group (T chosen so that every warp of the
//     grid has work); partial sums meet in shared memory behind a named
//     barrier per team, double-buffered so there is one barrier per group.
//   * The activations (int8, M*K bytes) sit in shared memory.  With the fused
//     entry point the CTA quantises x itself in its prologue (absmax, scale,
//     rint, row sum), so decode is one launch per BitLinear.
//   * Inner loop: the stored codes s = code + 1 in {0,1,2} of four consecutive
//     k are (word & (3 << 2i)) per byte; dp4a (unsigned x signed bytes) against
//     four int8 activations gives 4^i * sum(s q).  For M <= 4 each of the four
//     shifts keeps its own accumulator (one LOP3 + one dp4a per 4 weights per
//     token), for M >= 8 the codes are shifted down once and shared by all
//     tokens.  sum(code q) = sum(s q) - rowsum(q).
//   * Epilogue: y = ((float)acc * d_m) * gamma_eff, bf16 or fp32.
#include "bl_common.cuh"

namespace bl {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kUnroll = 4;

enum { MODE_Q = 0, MODE_X_BF16 = 1, MODE_X_F32 = 2 };

struct Params {
    const uint8_t *packed;
    const float *w_scale;
    int64_t N, K, NG;
    int M;
    int T;  // warps per team: 1, 2, 4, 8 or 16
    const int8_t *q;
    const float *d;
    const int32_t *rowsum;
    const void *x;
    int64_t ldx;
    void *y;
    int yt;
    int64_t ldy;
    int32_t *acc_dbg;
};

template <int MT>
struct Smem {
    float bmax[kWarps][MT];
    int bsum[kWarps][MT];
    float scale[MT];
    float d[MT];
    int r[MT];
    int red[2][kWarps][MT][8];
    // followed by the int8 activations, M*K bytes, 16-byte aligned
};

template <int MT>
constexpr size_t smem_header()
{
    return (sizeof(Smem<MT>) + 15) / 16 * 16;
}

// Quantise the M tokens of x into shared memory (block-cooperative).
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
                load8<XT>(p.x, m * p.ldx + c * 8, f);
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
                load8<XT>(p.x, m * p.ldx + c * 8, f);
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
        reinterpret_cast<uint4 *>(qs)[i] = ld_ro_v4(p.q + i * 16);
    if (threadIdx.x < p.M) {
        sm.d[threadIdx.x] = p.d[threadIdx.x];
        sm.r[threadIdx.x] = p.rowsum[threadIdx.x];
    }
    __syncthreads();
}

template <int MT>
__device__ __forceinline__ void epilogue(const Params &p, const Smem<MT> &sm, float gamma,
                                         int64_t g, int rr, int m, int total)
{
    const int64_t n = g * 8 + rr;
    if (n >= p.N)
        return;
    const int a = total - sm.r[m];
    if (p.acc_dbg)
        p.acc_dbg[int64_t(m) * p.N + n] = a;
    store_y(p.y, p.yt, int64_t(m) * p.ldy + n, rescale1(a, sm.d[m], gamma));
}

template <int MT, int MODE, int MINB>
__global__ void __launch_bounds__(kThreads, MINB) gemv_kernel(const Params p)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    Smem<MT> &sm = *reinterpret_cast<Smem<MT> *>(smem_raw);
    int8_t *qs = reinterpret_cast<int8_t *>(smem_raw + smem_header<MT>());

    if constexpr (MODE == MODE_Q)
        copy_prologue<MT>(p, sm, qs);
    else if constexpr (MODE == MODE_X_BF16)
        quantize_prologue<MT, BL_BF16>(p, sm, qs);
    else
        quantize_prologue<MT, BL_F32>(p, sm, qs);

    constexpr bool kMaskVariant = MT <= 4;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int T = p.T, nteams = kWarps / T, team = warp / T, wt = warp % T;
    const int64_t C = p.K / 64, P = (C + 3) / 4, slab = C * 128;
    const int csub = lane >> 3;
    const float gamma = p.w_scale[0];
    const int64_t g_begin = int64_t(blockIdx.x) * p.NG / gridDim.x;
    const int64_t g_end = int64_t(blockIdx.x + 1) * p.NG / gridDim.x;
    int parity = 0;

    for (int64_t g = g_begin + team; g < g_end; g += nteams) {
        int acc[MT][kMaskVariant ? 4 : 1];
#pragma unroll
        for (int m = 0; m < MT; ++m)
#pragma unroll
            for (int i = 0; i < (kMaskVariant ? 4 : 1); ++i)
                acc[m][i] = 0;
        const uint8_t *sp = p.packed + g * slab + lane * 16;

        for (int64_t p0 = wt; p0 < P; p0 += int64_t(T) * kUnroll) {
            uint4 wv[kUnroll];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int64_t pp = p0 + int64_t(u) * T;
                const int64_t c = 4 * pp + csub;
                wv[u] = (pp < P && c < C) ? ld_stream_v4(sp + pp * 512) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int64_t pp = p0 + int64_t(u) * T;
                const int64_t c = 4 * pp + csub;
                if (!(pp < P && c < C))
                    continue;
                const uint32_t wd[4] = {wv[u].x, wv[u].y, wv[u].z, wv[u].w};
                if constexpr (kMaskVariant) {
#pragma unroll
                    for (int m = 0; m < MT; ++m) {
                        if (m >= p.M)
                            break;
                        const uint4 *qp = reinterpret_cast<const uint4 *>(qs + m * p.K + c * 64);
#pragma unroll
                        for (int w = 0; w < 4; ++w) {
                            const uint4 q4 = qp[w];
                            acc[m][0] = dp4a_us(wd[w] & 0x03030303u, q4.x, acc[m][0]);
                            acc[m][1] = dp4a_us(wd[w] & 0x0c0c0c0cu, q4.y, acc[m][1]);
                            acc[m][2] = dp4a_us(wd[w] & 0x30303030u, q4.z, acc[m][2]);
                            acc[m][3] = dp4a_us(wd[w] & 0xc0c0c0c0u, q4.w, acc[m][3]);
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
                            const uint4 q4 =
                                reinterpret_cast<const uint4 *>(qs + m * p.K + c * 64)[w];
                            int a = acc[m][0];
                            a = dp4a_us(c0, q4.x, a);
                            a = dp4a_us(c1, q4.y, a);
                            a = dp4a_us(c2, q4.z, a);
                            a = dp4a_us(c3, q4.w, a);
                            acc[m][0] = a;
                        }
                    }
                }
            }
        }

        int tot[MT];
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            if constexpr (kMaskVariant)
                tot[m] = acc[m][0] + (acc[m][1] >> 2) + (acc[m][2] >> 4) + (acc[m][3] >> 6);
            else
                tot[m] = acc[m][0];
            tot[m] += __shfl_xor_sync(0xffffffffu, tot[m], 8);
            tot[m] += __shfl_xor_sync(0xffffffffu, tot[m], 16);
        }
        if (T == 1) {
            if (lane < 8) {
#pragma unroll
                for (int m = 0; m < MT; ++m)
                    if (m < p.M)
                        epilogue<MT>(p, sm, gamma, g, lane, m, tot[m]);
            }
        } else {
            if (lane < 8) {
#pragma unroll
                for (int m = 0; m < MT; ++m)
                    if (m < p.M)
                        sm.red[parity][warp][m][lane] = tot[m];
            }
            named_barrier(1 + team, T * 32);
            if (wt == 0) {
                for (int idx = lane; idx < p.M * 8; idx += 32) {
                    const int m = idx >> 3, rr = idx & 7;
                    int s = 0;
                    for (int t = 0; t < T; ++t)
                        s += sm.red[parity][team * T + t][m][rr];
                    epilogue<MT>(p, sm, gamma, g, rr, m, s);
                }
            }
            parity ^= 1;
        }
    }
}

template <int MT, int MODE>
int launch_one(const Params &base, cudaStream_t s)
{
    constexpr int kMinBlocks = MT <= 4 ? 2 : 1;
    auto kern = gemv_kernel<MT, MODE, kMinBlocks>;
    const DeviceInfo *di = device_info();
    if (!di)
        return BL_ERR_CUDA;
    const size_t smem = smem_header<MT>() + size_t(base.M) * size_t(base.K);
    if (smem > size_t(di->max_smem_optin))
        return BL_ERR_SHAPE;
    int per_sm = 0;
    int st = occupancy(reinterpret_cast<const void *>(kern), kThreads, smem, &per_sm);
    if (st)
        return st;
    if (per_sm < 1)
        return BL_ERR_SHAPE;
    Params p = base;
    const int64_t warps_total = int64_t(di->sm_count) * per_sm * kWarps;
    const int64_t P = (p.K / 64 + 3) / 4;
    int tmax = 1;
    while (tmax * 2 <= kWarps && tmax * 2 <= P)
        tmax *= 2;
    int T = 1;
    while (T < tmax && p.NG * T < warps_total)
        T *= 2;
    p.T = T;
    const int nteams = kWarps / T;
    const int64_t want = (p.NG + nteams - 1) / nteams;
    const int64_t grid = want < int64_t(di->sm_count) * per_sm ? want : int64_t(di->sm_count) * per_sm;
    kern<<<unsigned(grid), kThreads, smem, s>>>(p);
    return launch_status();
}

template <int MODE>
int dispatch_m(const Params &p, cudaStream_t s)
{
    if (p.M <= 1)
        return launch_one<1, MODE>(p, s);
    if (p.M <= 2)
        return launch_one<2, MODE>(p, s);
    if (p.M <= 4)
        return launch_one<4, MODE>(p, s);
    if (p.M <= 8)
        return launch_one<8, MODE>(p, s);
    return launch_one<16, MODE>(p, s);
}

}  // namespace

int launch_gemv(const GemvArgs &a, bool fused, cudaStream_t s)
{
    Params p{};
    p.packed = a.packed;
    p.w_scale = a.w_scale;
    p.N = a.N;
    p.K = a.K;
    p.NG = (a.N + 7) / 8;
    p.M = int(a.M);
    p.T = 1;
    p.q = a.q;
    p.d = a.d;
    p.rowsum = a.rowsum;
    p.x = a.x;
    p.ldx = a.ldx;
    p.y = a.y;
    p.yt = a.yt;
    p.ldy = a.ldy;
    p.acc_dbg = a.acc_dbg;
    if (!fused)
        return dispatch_m<MODE_Q>(p, s);
    if (a.xt == BL_BF16)
        return dispatch_m<MODE_X_BF16>(p, s);
    return dispatch_m<MODE_X_F32>(p, s);
}

}  // namespace bl
