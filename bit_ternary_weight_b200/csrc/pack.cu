// pack.cu -- offline ternary packer: absmean weight scale, round-clip to
// {-1, 0, +1} and 2-bit packing into layout TL.
//
// "bit-floor" README, section "What's inside": f32 weights packed with a
// mean-abs scale for ternary zero-suppression.  "BitCompute: 1.58-bit LLM
// Execution Engine", section "Future Roadmap": four weights per byte.
//
// Three launches on the caller's stream:
//   1. row_abs_sum_kernel  fp64 sum of |W[n][k]| over k, ascending k, one thread
//                          per row; tiles of 256 rows x 32 k are staged through
//                          shared memory so that global reads stay coalesced.
//   2. scale_kernel        one thread adds the N row sums in ascending n (fp64),
//                          divides by N*K, rounds to fp32 and floors at 1e-5.
//   3. pack_kernel         one thread per 32-bit output word (16 codes).
// The order of the fp64 additions is part of the definition of gamma, so the
// result is bit-identical to a sequential CPU evaluation.
#include <mutex>

#include "bl_common.cuh"

namespace bl {
namespace {

constexpr int kRowsPerBlock = 256;
constexpr int kTileK = 32;

template <int WT>
__device__ __forceinline__ float load_w(const void *W, int64_t i)
{
    if (WT == BL_BF16)
        return __bfloat162float(static_cast<const __nv_bfloat16 *>(W)[i]);
    return static_cast<const float *>(W)[i];
}

template <int WT>
__global__ void __launch_bounds__(kRowsPerBlock)
row_abs_sum_kernel(const void *__restrict__ W, int64_t N, int64_t K,
                   double *__restrict__ row_sums)
{
    __shared__ float tile[kRowsPerBlock][kTileK + 1];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t n0 = int64_t(blockIdx.x) * kRowsPerBlock;
    double acc = 0.0;
    for (int64_t k0 = 0; k0 < K; k0 += kTileK) {
        // warp w loads rows w, w+8, ...: 32 consecutive k per row (coalesced)
        for (int r = warp; r < kRowsPerBlock; r += kRowsPerBlock / 32) {
            const int64_t n = n0 + r;
            tile[r][lane] = n < N ? fabsf(load_w<WT>(W, n * K + k0 + lane)) : 0.0f;
        }
        __syncthreads();
#pragma unroll
        for (int j = 0; j < kTileK; ++j)
            acc = __dadd_rn(acc, static_cast<double>(tile[tid][j]));
        __syncthreads();
    }
    const int64_t n = n0 + tid;
    if (n < N)
        row_sums[n] = acc;
}

__global__ void scale_kernel(const double *__restrict__ row_sums, int64_t N, int64_t K,
                             float *__restrict__ w_scale)
{
    if (threadIdx.x != 0 || blockIdx.x != 0)
        return;
    double S = 0.0;
#pragma unroll 8
    for (int64_t n = 0; n < N; ++n)
        S = __dadd_rn(S, row_sums[n]);
    const double mean = __ddiv_rn(S, static_cast<double>(N * K));
    w_scale[0] = fmaxf(__double2float_rn(mean), kEps);
}

// Word o of the packed array: o = ((g * (K/64) + c) * 8 + r) * 4 + w.
// Its 16 codes are k = 64c + 16w + 4i + j for i, j in 0..3, code at bit 8j+2i.
template <int WT>
__global__ void __launch_bounds__(256)
pack_kernel(const void *__restrict__ W, int64_t N, int64_t K, int64_t words,
            const float *__restrict__ w_scale, uint32_t *__restrict__ packed)
{
    const int64_t o = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
    if (o >= words)
        return;
    const int64_t C = K / 64;
    const int w = int(o & 3);
    const int r = int((o >> 2) & 7);
    const int64_t gc = o >> 5;
    const int64_t c = gc % C, g = gc / C;
    const int64_t n = g * 8 + r;
    uint32_t word = 0x55555555u;  // code 0 (stored 1) everywhere: padding rows
    if (n < N) {
        const float gamma = w_scale[0];
        const int64_t base = n * K + c * 64 + w * 16;
        word = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float t = rintf(__fdiv_rn(load_w<WT>(W, base + 4 * i + j), gamma));
                const int code = t >= 1.0f ? 1 : (t <= -1.0f ? -1 : 0);
                word |= uint32_t(code + 1) << (8 * j + 2 * i);
            }
    }
    packed[o] = word;
}

}  // namespace

int launch_pack(const void *W, int wt, int64_t N, int64_t K, uint8_t *packed,
                float *w_scale, double *row_sums, cudaStream_t s)
{
    const unsigned blocks = static_cast<unsigned>((N + kRowsPerBlock - 1) / kRowsPerBlock);
    if (wt == BL_BF16)
        row_abs_sum_kernel<BL_BF16><<<blocks, kRowsPerBlock, 0, s>>>(W, N, K, row_sums);
    else
        row_abs_sum_kernel<BL_F32><<<blocks, kRowsPerBlock, 0, s>>>(W, N, K, row_sums);
    int st = launch_status();
    if (st)
        return st;
    scale_kernel<<<1, 32, 0, s>>>(row_sums, N, K, w_scale);
    if ((st = launch_status()))
        return st;
    const int64_t words = (N + 7) / 8 * 8 * (K / 16);
    const unsigned pblocks = static_cast<unsigned>((words + 255) / 256);
    if (wt == BL_BF16)
        pack_kernel<BL_BF16><<<pblocks, 256, 0, s>>>(W, N, K, words, w_scale,
                                                     reinterpret_cast<uint32_t *>(packed));
    else
        pack_kernel<BL_F32><<<pblocks, 256, 0, s>>>(W, N, K, words, w_scale,
                                                    reinterpret_cast<uint32_t *>(packed));
    return launch_status();
}

// ---------------------------------------------------------------------------
// Packing with no caller-provided workspace (bitlinear_pack_noalloc).
//
// The per-row fp64 sums live in this file-scope device array instead of a
// workspace the caller allocates.  Every GPU that loads the library holds it
// (512 KiB) until the process exits.  In host code the symbol is only a
// host-side stand-in, so its device address is looked up once per device with
// cudaGetSymbolAddress, with that device current, and passed to the kernels.
constexpr int64_t kNoAllocMaxRows = BITLINEAR_PACK_NOALLOC_MAX_ROWS;
static __device__ __align__(256) double g_pack_scratch[kNoAllocMaxRows];

namespace {

constexpr int kMaxScratchDevices = 64;
std::mutex g_scratch_mutex;
double *g_scratch_addr[kMaxScratchDevices] = {};

// Device address of g_pack_scratch on the current device (set up on first use).
int scratch_address(double **out)
{
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return cuda_status(e);
    if (dev < 0 || dev >= kMaxScratchDevices)
        return BL_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_pack_scratch);
        if (e != cudaSuccess)
            return cuda_status(e);
        g_scratch_addr[dev] = static_cast<double *>(p);
    }
    *out = g_scratch_addr[dev];
    return BL_OK;
}

}  // namespace

}  // namespace bl

extern "C" int bitlinear_pack_noalloc(const void *W, int wt, int64_t N, int64_t K,
                                      uint8_t *packed, float *w_scale, void *stream)
{
    using namespace bl;
    if (!W || !packed || !w_scale)
        return BL_ERR_NULL;
    if (wt != BL_F32 && wt != BL_BF16)
        return BL_ERR_DTYPE;
    if (!valid_nk(N, K) || N > kNoAllocMaxRows)
        return BL_ERR_SHAPE;
    if ((reinterpret_cast<uintptr_t>(W) & 15u) || (reinterpret_cast<uintptr_t>(packed) & 15u) ||
        (reinterpret_cast<uintptr_t>(w_scale) & 3u))
        return BL_ERR_ALIGN;
    const DeviceInfo *di;
    int st = need_device(&di);
    if (st)
        return st;
    if ((st = check_dev_ptrs({W, packed, w_scale})))
        return st;
    double *scratch = nullptr;
    st = scratch_address(&scratch);
    if (st)
        return st;
    return launch_pack(W, wt, N, K, packed, w_scale, scratch, static_cast<cudaStream_t>(stream));
}
