// lut_gemv.cu -- ternary decode GEMV of one token by table lookup instead of
// multiplication: the lookup-table method of the CPU kernels ("Run 100B
// Models on Your Laptop CPU: Microsoft BitNet Exposed", sections "What is
// Microsoft BitNet?" and "Key Features That Make BitNet Insane": TL1 / TL2
// kernels built on the lookup-table method of T-MAC), here on the GPU over
// the same packed layout TL as the dp4a kernels, for comparison with them.
//
// In TL a 4-bit field of a byte holds the stored codes s = code + 1 of two
// weights of one row, k and k + 4 (bits [1:0] and [3:2] of the low nibble of
// byte j of a 32-bit word are k0 + j and k0 + 4 + j, the high nibble k0 + 8 +
// j and k0 + 12 + j).  For every such pair of activations (ka, kb) the kernel
// precomputes the 16-entry table
//     T[v] = (v % 4 - 1) * q[ka] + (v / 4 - 1) * q[kb]     (v = s_a + 4 s_b)
// (entries with a stored 3 never occur and hold 0), so that
//     acc[n] = sum over the row's nibbles v of T_pair[v]
// exactly -- the same integer as sum_k code q, with no rowsum correction.
// Tables are int16 (|T| <= 254), 32 bytes per pair; the 32 pairs of a 64-k
// chunk take 1 KiB, padded to 1056 bytes so that the four chunks a warp
// reads at once fall on different shared-memory banks.  K is limited by the
// tables: 16.5 bytes per k, K <= 12288.
//
// Every CTA builds the tables of the whole k range (all threads, from q in
// global memory), then its warps walk row groups: lane l takes row l % 8 and
// 64-k chunk l / 8 of every 256 k (one 512-byte coalesced warp load per
// step, the TL layout of the dp4a kernels), looks up 32 pair entries per
// 16-byte chunk (one bit-field extract, one shared load, one add each) and
// the four lanes of a row are reduced with shuffles.  Per weight that is
// about three times the instructions of the dp4a path (one LOP3 and one dp4a
// per four weights), which is what this kernel exists to measure.
#include "bl_common.cuh"

namespace bl {
namespace {

constexpr int kLutThreads = 256;
constexpr int kLutWarps = kLutThreads / 32;
constexpr int kChunkEntries = 528;          // int16 entries per 64-k chunk block (512 + 16 pad)
constexpr int64_t kLutMaxK = 12288;

struct LutParams {
    const uint8_t *packed;
    const float *w_scale;
    int64_t N, K;
    const int8_t *q;
    const float *d;
    void *y;
    int yt;
    int32_t *acc_dbg;
};

// Table slot of pair (c, i, j, h): chunk c, 16-k word i, byte j, nibble h.
__device__ __forceinline__ int lut_slot(int c, int i, int j, int h)
{
    return c * kChunkEntries + ((i * 4 + j) * 2 + h) * 16;
}

__global__ void __launch_bounds__(kLutThreads) lut_gemv_kernel(const LutParams p)
{
    extern __shared__ __align__(16) int16_t lut[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int C = int(p.K / 64);
    // ---- tables: 32 pairs x 16 entries per chunk
    const int entries = C * 512;
    for (int e = tid; e < entries; e += kLutThreads) {
        const int v = e & 15, pair = e >> 4;
        const int h = pair & 1, j = (pair >> 1) & 3, i = (pair >> 3) & 3, c = pair >> 5;
        const int sa = v & 3, sb = v >> 2;
        int t = 0;
        if (sa != 3 && sb != 3) {
            const int ka = c * 64 + i * 16 + h * 8 + j;
            t = (sa - 1) * int(p.q[ka]) + (sb - 1) * int(p.q[ka + 4]);
        }
        lut[lut_slot(c, i, j, h) + v] = int16_t(t);
    }
    __syncthreads();

    const float gamma = __ldg(p.w_scale);
    const float dd = __ldg(p.d);
    const int64_t groups = (p.N + 7) / 8;
    const int r = lane & 7, sub = lane >> 3;          // row in group, chunk within 256 k
    const uint32_t lut_base = smem_u32(lut);
    for (int64_t g = int64_t(blockIdx.x) * kLutWarps + warp; g < groups; g += int64_t(gridDim.x) * kLutWarps) {
        const uint8_t *slab = p.packed + g * 2 * p.K;    // the group's TL bytes
        int acc = 0;
        for (int c0 = 0; c0 < C; c0 += 4) {
            const int c = c0 + sub;
            if (c < C) {
                const uint4 v = ld_stream_v4(slab + (int64_t(c) * 8 + r) * 16);
                const uint32_t wd[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const uint32_t base = lut_base + uint32_t(lut_slot(c, i, 0, 0)) * 2;
#pragma unroll
                    for (int n = 0; n < 8; ++n) {               // nibble n = 2 j + h
                        const uint32_t off = (wd[i] >> (4 * n)) & 15u;
                        int16_t t;
                        asm volatile("ld.shared.s16 %0, [%1];" : "=h"(t) : "r"(base + (n * 16 + off) * 2));
                        acc += t;
                    }
                }
            }
        }
        acc += __shfl_xor_sync(0xffffffffu, acc, 8);
        acc += __shfl_xor_sync(0xffffffffu, acc, 16);
        const int64_t row = g * 8 + r;
        if (sub == 0 && row < p.N) {
            if (p.acc_dbg)
                p.acc_dbg[row] = acc;
            store_y(p.y, p.yt, row, rescale1(acc, dd, gamma));
        }
    }
}

}  // namespace

bool lut_gemv_applies(int64_t K) { return K <= kLutMaxK; }

int launch_lut_gemv(const uint8_t *packed, const float *w_scale, int64_t N, int64_t K,
                    const int8_t *q, const float *d, void *y, int yt, int32_t *acc_dbg,
                    cudaStream_t s)
{
    const DeviceInfo *di = device_info();
    if (!di)
        return BL_ERR_CUDA;
    LutParams p{packed, w_scale, N, K, q, d, y, yt, acc_dbg};
    const size_t smem = size_t(K / 64) * kChunkEntries * sizeof(int16_t);
    int per_sm = 0;
    int st = occupancy(reinterpret_cast<const void *>(lut_gemv_kernel), kLutThreads, smem, &per_sm);
    if (st)
        return st;
    if (per_sm < 1)
        return BL_ERR_SHAPE;
    const int64_t groups = (N + 7) / 8;
    int64_t grid = (groups + kLutWarps - 1) / kLutWarps;
    const int64_t cap = int64_t(per_sm) * di->sm_count;
    if (grid > cap)
        grid = cap;
    lut_gemv_kernel<<<unsigned(grid), kLutThreads, smem, s>>>(p);
    return launch_status();
}

}  // namespace bl
