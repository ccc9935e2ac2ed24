// popc_stream.cu -- XNOR / popcount decode GEMVs of one token, streamed
// through a shared-memory ring by bulk asynchronous copies:
//   * binary weights (one bit each): acc = 2 * POPCNT(XNOR(W, x)) - K,
//     y = acc * (s_w * s_x)                ("bit-floor" README, "The core math")
//   * ternary weights on two bit-planes against 1-bit activations:
//     acc = POPCNT(mag & XNOR(sign, x)) - POPCNT(mag & XOR(sign, x)),
//     y = acc * (gamma * s_x)              (same section: "Ternary GEMV")
// x enters as its sign bits (set for negative values) and s_x = max |x|.
//
// Both stream N rows of RB bytes (binary: K/8, bit-planes: K/4) exactly once,
// so they are HBM-bound.  Layouts: binary uint64 [N][K/64], bit j of word w
// <-> k = 64 w + j; bit-planes uint64 [N][K/64][2], the pair (mag, sign) of
// each 64-k word side by side, so that a row stays one contiguous span and a
// run of rows one contiguous block.
//
// Design (persistent CTAs, two per SM):
//   * Each CTA owns a contiguous run of rows and streams it in stages of
//     whole rows (up to 24 KiB), a four-stage ring filled by one producer
//     warp with bulk copies of at most 4 KiB, each from a different lane
//     (copies of one thread complete one after another), completion counted
//     on the stage's mbarrier.  The producer starts at once: the weights do
//     not depend on x.
//   * Eight consumer warps meanwhile build x's sign words in shared memory
//     (eight lanes per 64-bit word, eight elements each, combined with
//     shuffles; all loads of a batch issued first) and the block-wide
//     max |x|, then take the
//     stage's rows in turn, one row per warp at a time: each lane XORs /
//     popcounts 16-byte pieces of the row against the matching x words, and
//     one warp reduction (redux.sync) gives the row's count.
//   * Every mbarrier wait is bounded; on expiry the CTA records
//     BL_ERR_TIMEOUT, the consumers stop and the producer waits (bounded) for
//     its copies in flight before the CTA exits.
#include "bl_common.cuh"

namespace bl {
namespace {

constexpr int kPcConsumers = 8;
constexpr int kPcThreads = 32 * (kPcConsumers + 1);
constexpr int kPcStages = 4;
constexpr uint32_t kPcStageBytes = 24 * 1024;
constexpr uint32_t kPcCopyBytes = 4 * 1024;
constexpr int kPcMaxWords = 1024;           // K <= 65536

enum { PC_BINARY = 1, PC_BITPLANE = 2 };

struct PcParams {
    const unsigned char *w;      // N rows of RB bytes
    int64_t N, K;
    uint32_t RB;                 // bytes per row
    int rows_per_stage;
    const void *x;
    const float *w_scale;        // s_w (binary) or gamma_eff (bit-planes)
    void *y;
    int yt;
    int32_t *acc_dbg;
    int64_t rpc_base;            // rows per CTA: rpc_base (+1 for the first rpc_rem CTAs)
    int rpc_rem;
    int *status;
};

struct PcSmem {
    uint64_t full[kPcStages];
    uint64_t empty[kPcStages];
    int abort_flag;
    float wmax[kPcConsumers];
    // followed by the ring (kPcStages x kPcStageBytes) and the x sign words
};

constexpr size_t kPcHeader = (sizeof(PcSmem) + 127) / 128 * 128;

__device__ __forceinline__ uint4 pc_lds128(uint32_t saddr)
{
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(saddr));
    return v;
}

__device__ __forceinline__ uint64_t u64_of(uint32_t lo, uint32_t hi)
{
    return (static_cast<uint64_t>(hi) << 32) | lo;
}

template <int VAR, int XT>
__global__ void __launch_bounds__(kPcThreads, 2) popc_stream_kernel(const PcParams p)
{
    extern __shared__ __align__(128) unsigned char smem_raw[];
    PcSmem &sm = *reinterpret_cast<PcSmem *>(smem_raw);
    const uint32_t ring = smem_u32(smem_raw + kPcHeader);
    uint64_t *xw = reinterpret_cast<uint64_t *>(smem_raw + kPcHeader + size_t(kPcStages) * kPcStageBytes);
    volatile int *abort_flag = &sm.abort_flag;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bx = blockIdx.x;
    const int64_t r_begin = bx * p.rpc_base + (bx < p.rpc_rem ? bx : p.rpc_rem);
    const int nr = int(p.rpc_base) + (bx < p.rpc_rem ? 1 : 0);
    const int RS = p.rows_per_stage;
    const int nst = (nr + RS - 1) / RS;

    if (tid == 0) {
        for (int b = 0; b < kPcStages; ++b) {
            mbar_init(smem_u32(&sm.full[b]), 1);
            mbar_init(smem_u32(&sm.empty[b]), kPcConsumers);
        }
        sm.abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    if (warp == kPcConsumers) {
        // ------------------------------------------------ producer warp
        int sb = 0;
        uint32_t ph = 0;
        int t = 0;
        for (; t < nst; ++t) {
            const int rows = min(RS, nr - t * RS);
            const uint32_t bytes = uint32_t(rows) * p.RB;
            if (!__all_sync(0xffffffffu, mbar_wait_fast(smem_u32(&sm.empty[sb]), ph ^ 1u, abort_flag, p.status)))
                break;
            const uint32_t full = smem_u32(&sm.full[sb]);
            if (lane == 0)
                mbar_arrive_tx(full, bytes);
            __syncwarp();
            const uint32_t off = uint32_t(lane) * kPcCopyBytes;
            if (off < bytes) {
                const uint32_t len = min(kPcCopyBytes, bytes - off);
                bulk_load(ring + uint32_t(sb) * kPcStageBytes + off,
                          p.w + (r_begin + int64_t(t) * RS) * p.RB + off, len, full);
            }
            if (++sb == kPcStages) {
                sb = 0;
                ph ^= 1u;
            }
        }
        // copies still in flight land before the CTA exits
        volatile int no_abort = 0;
        for (int u = t - kPcStages > 0 ? t - kPcStages : 0; u < t; ++u)
            mbar_wait(smem_u32(&sm.full[u % kPcStages]), uint32_t(u / kPcStages) & 1u, &no_abort, p.status,
                      100000000ull);
        return;
    }

    // ---------------------------------------------------- consumer warps
    asm volatile("griddepcontrol.wait;" ::: "memory");
    // x's sign words: eight lanes per 64-bit word, eight elements (one or two
    // 16-byte loads) per lane, so a warp covers four words per step; the
    // loads of kXBatch steps are issued before any of them is used
    const int words = int(p.K / 64);
    constexpr int kXBatch = 4;
    float amax = 0.0f;
    const int sub = lane & 7;
    for (int w0 = warp * 4; w0 < words; w0 += kPcConsumers * 4 * kXBatch) {
        float f[kXBatch][8];
#pragma unroll
        for (int b = 0; b < kXBatch; ++b) {
            const int w = w0 + b * kPcConsumers * 4 + (lane >> 3);
            if (w < words)
                load8<XT, true>(p.x, int64_t(w) * 64 + sub * 8, f[b]);
            else
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    f[b][e] = 0.0f;
        }
#pragma unroll
        for (int b = 0; b < kXBatch; ++b) {
            const int w = w0 + b * kPcConsumers * 4 + (lane >> 3);
            uint32_t neg = 0;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                amax = fmaxf(amax, fabsf(f[b][e]));
                neg |= uint32_t(f[b][e] < 0.0f) << e;
            }
            uint64_t word = static_cast<uint64_t>(neg) << (8 * sub);
            word |= __shfl_xor_sync(0xffffffffu, word, 1);
            word |= __shfl_xor_sync(0xffffffffu, word, 2);
            word |= __shfl_xor_sync(0xffffffffu, word, 4);
            if (sub == 0 && w < words)
                xw[w] = word;
        }
    }
    // maxima are >= 0 and finite (fmaxf from 0 drops NaN): bit patterns order like the values
    amax = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(amax)));
    if (lane == 0)
        sm.wmax[warp] = amax;
    named_barrier(1, 32 * kPcConsumers);
    float s_x = sm.wmax[0];
#pragma unroll
    for (int w = 1; w < kPcConsumers; ++w)
        s_x = fmaxf(s_x, sm.wmax[w]);
    const float scale = __fmul_rn(__ldg(p.w_scale), s_x);

    const uint32_t pieces = p.RB / 16;     // 16-byte pieces per row
    int sb = 0;
    uint32_t ph = 0;
    for (int t = 0; t < nst; ++t) {
        if (!__all_sync(0xffffffffu, mbar_wait_fast(smem_u32(&sm.full[sb]), ph, abort_flag, p.status)))
            break;
        const int rows = min(RS, nr - t * RS);
        const uint32_t stage = ring + uint32_t(sb) * kPcStageBytes;
        for (int rr = warp; rr < rows; rr += kPcConsumers) {
            const uint32_t row = stage + uint32_t(rr) * p.RB;
            int cnt = 0;
            for (uint32_t c = lane; c < pieces; c += 32) {
                const uint4 v = pc_lds128(row + c * 16);
                if constexpr (VAR == PC_BINARY) {
                    const uint64_t w0 = u64_of(v.x, v.y), w1 = u64_of(v.z, v.w);
                    cnt += __popcll(~(w0 ^ xw[2 * c])) + __popcll(~(w1 ^ xw[2 * c + 1]));
                } else {
                    const uint64_t m = u64_of(v.x, v.y), s = u64_of(v.z, v.w);
                    const uint64_t diff = (s ^ xw[c]) & m;      // non-zero weights of opposite sign
                    cnt += __popcll(m) - 2 * __popcll(diff);    // agree - disagree
                }
            }
            cnt = __reduce_add_sync(0xffffffffu, cnt);
            if (lane == 0) {
                const int64_t n = r_begin + int64_t(t) * RS + rr;
                const int acc = VAR == PC_BINARY ? 2 * cnt - int(p.K) : cnt;
                if (p.acc_dbg)
                    p.acc_dbg[n] = acc;
                store_y(p.y, p.yt, n, __fmul_rn(static_cast<float>(acc), scale));
            }
        }
        __syncwarp();
        if (lane == 0)
            mbar_arrive(smem_u32(&sm.empty[sb]));
        if (++sb == kPcStages) {
            sb = 0;
            ph ^= 1u;
        }
    }
}

template <int VAR, int XT>
int launch_pc_t(PcParams p, cudaStream_t s)
{
    const DeviceInfo *di = device_info();
    if (!di)
        return BL_ERR_CUDA;
    auto kern = popc_stream_kernel<VAR, XT>;
    const size_t smem = kPcHeader + size_t(kPcStages) * kPcStageBytes + size_t(p.K / 64) * 8;
    int per_sm = 0;
    int st = occupancy(reinterpret_cast<const void *>(kern), kPcThreads, smem, &per_sm);
    if (st)
        return st;
    if (per_sm < 1)
        return BL_ERR_SHAPE;
    p.rows_per_stage = int(kPcStageBytes / p.RB);
    // enough CTAs to spread the rows, at most the resident ones, and no CTA
    // with fewer rows than a stage holds unless the rows run out
    const int64_t stages = (p.N + p.rows_per_stage - 1) / p.rows_per_stage;
    int64_t grid = int64_t(per_sm < 2 ? per_sm : 2) * di->sm_count;
    if (grid > stages)
        grid = stages;
    if (grid < 1)
        grid = 1;
    p.rpc_base = p.N / grid;
    p.rpc_rem = int(p.N % grid);
    p.status = di->status;
    kern<<<unsigned(grid), kPcThreads, smem, s>>>(p);
    return launch_status();
}

// Bit-plane packer: word pair (mag, sign) of row n and 64-k word c from the
// 16-byte TL chunk of the same row and k range (stored value s = code + 1:
// s != 1 marks a non-zero weight, s == 0 a negative one).
__global__ void __launch_bounds__(256)
bitplane_pack_kernel(const uint8_t *__restrict__ tl, int64_t N, int64_t K,
                     unsigned long long *__restrict__ planes)
{
    const int64_t C = K / 64;
    const int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= N * C)
        return;
    const int64_t n = i / C, c = i % C;
    const uint4 v = *reinterpret_cast<const uint4 *>(tl + ((n / 8 * C + c) * 8 + n % 8) * 16);
    const uint32_t wd[4] = {v.x, v.y, v.z, v.w};
    unsigned long long mag = 0, sign = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q)          // TL word q: k = 16 q + 4 a + j at bits 8 j + 2 a
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t sv = (wd[q] >> (8 * j + 2 * a)) & 3u;
                const int k = 16 * q + 4 * a + j;
                mag |= static_cast<unsigned long long>(sv != 1u) << k;
                sign |= static_cast<unsigned long long>(sv == 0u) << k;
            }
    planes[2 * i] = mag;
    planes[2 * i + 1] = sign;
}

}  // namespace

bool popc_stream_applies_binary(int64_t K) { return (K / 8) % 16 == 0 && K / 64 <= kPcMaxWords; }

int launch_binary_gemv_stream(const uint64_t *Wb, const float *s_w, int64_t N, int64_t K,
                              const void *x, int xt, void *y, int yt, int32_t *acc_dbg,
                              cudaStream_t s)
{
    PcParams p{};
    p.w = reinterpret_cast<const unsigned char *>(Wb);
    p.N = N;
    p.K = K;
    p.RB = uint32_t(K / 8);
    p.x = x;
    p.w_scale = s_w;
    p.y = y;
    p.yt = yt;
    p.acc_dbg = acc_dbg;
    if (xt == BL_BF16)
        return launch_pc_t<PC_BINARY, BL_BF16>(p, s);
    return launch_pc_t<PC_BINARY, BL_F32>(p, s);
}

int launch_bitplane_gemv(const uint64_t *planes, const float *w_scale, int64_t N, int64_t K,
                         const void *x, int xt, void *y, int yt, int32_t *acc_dbg, cudaStream_t s)
{
    PcParams p{};
    p.w = reinterpret_cast<const unsigned char *>(planes);
    p.N = N;
    p.K = K;
    p.RB = uint32_t(K / 4);
    p.x = x;
    p.w_scale = w_scale;
    p.y = y;
    p.yt = yt;
    p.acc_dbg = acc_dbg;
    if (xt == BL_BF16)
        return launch_pc_t<PC_BITPLANE, BL_BF16>(p, s);
    return launch_pc_t<PC_BITPLANE, BL_F32>(p, s);
}

int launch_bitplane_pack(const uint8_t *packed, int64_t N, int64_t K, uint64_t *planes, cudaStream_t s)
{
    const int64_t total = N * (K / 64);
    const unsigned blocks = unsigned((total + 255) / 256);
    bitplane_pack_kernel<<<blocks, 256, 0, s>>>(packed, N, K, reinterpret_cast<unsigned long long *>(planes));
    return launch_status();
}

}  // namespace bl
