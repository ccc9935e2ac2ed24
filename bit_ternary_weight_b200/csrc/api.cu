// api.cu -- the extern "C" entry points of libbitlinear.so: argument checks in
// a fixed order (null -> dtype -> shape -> alignment -> device -> device
// pointers -> workspace), then the launchers of the other translation units.
// Every check that can fail runs before any launch, so a rejected call writes
// nothing.
#include <cuda_runtime.h>
#include <map>
#include <mutex>
#include <tuple>
#include <stdio.h>
#include <string.h>

#include "bl_internal.h"

namespace bl {

// Device status word: kernels whose bounded waits run out write an error code
// here; bitlinear_last_device_status() reads and clears it.
__device__ int g_device_status;

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_info_mutex;
DeviceInfo g_info[kMaxDevices];
thread_local char g_cuda_err[256] = "";

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool valid_dtype(int t) { return t == BL_F32 || t == BL_BF16; }
int elem_bytes(int t) { return t == BL_BF16 ? 2 : 4; }

}  // namespace

// Device (or managed) memory that belongs to the current device.  Memory of
// another GPU is rejected too: the kernels launch on the current device, and a
// pointer into a peer's memory would be dereferenced there.
bool is_device_ptr(const void *p)
{
    cudaPointerAttributes attr;
    cudaError_t e = cudaPointerGetAttributes(&attr, p);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    if (attr.type == cudaMemoryTypeManaged)
        return true;
    if (attr.type != cudaMemoryTypeDevice)
        return false;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return attr.device == dev;
}

// Common shape rule: N >= 1, K >= 64, K % 64 == 0, and sizes that keep every
// index inside int32 tiles and int64 byte offsets comfortably.
bool valid_nk(int64_t N, int64_t K)
{
    return N >= 1 && K >= 64 && K % 64 == 0 && N <= (int64_t(1) << 31) &&
           K <= (int64_t(1) << 22);
}

// Device presence and architecture; returns BL_OK and the info, or an error.
// The library is built for sm_100a only, whose code runs on compute
// capability 10.0 alone.
int need_device(const DeviceInfo **out)
{
    const DeviceInfo *di = device_info();
    if (!di)
        return BL_ERR_CUDA;
    if (di->cc_major != 10 || di->cc_minor != 0)
        return BL_ERR_UNSUPPORTED;
    *out = di;
    return BL_OK;
}

int check_dev_ptrs(std::initializer_list<const void *> ptrs)
{
    for (const void *p : ptrs)
        if (p && !is_device_ptr(p))
            return BL_ERR_NOT_DEVICE_PTR;
    return BL_OK;
}

const DeviceInfo *device_info()
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(g_info_mutex);
    DeviceInfo &di = g_info[dev];
    if (di.device == dev)
        return &di;
    DeviceInfo t;
    t.device = dev;
    if (cudaDeviceGetAttribute(&t.sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&t.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&t.cc_major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&t.cc_minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
        cuda_status(cudaGetLastError());
        return nullptr;
    }
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) {
        cuda_status(cudaGetLastError());
        return nullptr;
    }
    t.status = static_cast<int *>(p);
    di = t;
    return &di;
}

int cuda_status(cudaError_t e)
{
    if (e == cudaSuccess)
        return BL_OK;
    snprintf(g_cuda_err, sizeof g_cuda_err, "%s: %s", cudaGetErrorName(e),
             cudaGetErrorString(e));
    return BL_ERR_CUDA;
}

int launch_status() { return cuda_status(cudaGetLastError()); }

int occupancy(const void *func, int threads, size_t smem, int *per_sm)
{
    static std::mutex mu;
    static std::map<std::tuple<int, const void *, int, size_t>, int> cache;
    static std::map<std::pair<int, const void *>, bool> raised;
    const DeviceInfo *di = device_info();
    if (!di)
        return BL_ERR_CUDA;
    std::lock_guard<std::mutex> lock(mu);
    auto key = std::make_tuple(di->device, func, threads, smem);
    auto it = cache.find(key);
    if (it != cache.end()) {
        *per_sm = it->second;
        return BL_OK;
    }
    auto rk = std::make_pair(di->device, func);
    if (!raised.count(rk)) {
        // the dynamic limit may take whatever the kernel's static shared memory leaves
        cudaFuncAttributes fa;
        int st = cuda_status(cudaFuncGetAttributes(&fa, func));
        if (st)
            return st;
        const int dyn_max = di->max_smem_optin - int(fa.sharedSizeBytes);
        if (smem > size_t(dyn_max > 0 ? dyn_max : 0))
            return BL_ERR_SHAPE;
        st = cuda_status(cudaFuncSetAttribute(
            func, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn_max));
        if (st)
            return st;
        raised[rk] = true;
    }
    int n = 0;
    int st = cuda_status(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, func, threads, smem));
    if (st)
        return st;
    cache[key] = n;
    *per_sm = n;
    return BL_OK;
}

}  // namespace bl

using namespace bl;

extern "C" {

const char *bitlinear_status_string(int status)
{
    switch (status) {
    case BL_OK: return "BL_OK";
    case BL_ERR_NULL: return "BL_ERR_NULL: a required pointer is NULL";
    case BL_ERR_DTYPE: return "BL_ERR_DTYPE: unsupported element type";
    case BL_ERR_SHAPE: return "BL_ERR_SHAPE: shape or stride out of range";
    case BL_ERR_ALIGN: return "BL_ERR_ALIGN: pointer or stride not 16-byte aligned";
    case BL_ERR_NOT_DEVICE_PTR: return "BL_ERR_NOT_DEVICE_PTR: host memory or another GPU's memory where memory of the current device is required";
    case BL_ERR_WORKSPACE: return "BL_ERR_WORKSPACE: workspace missing or too small";
    case BL_ERR_CUDA: return "BL_ERR_CUDA: CUDA runtime error";
    case BL_ERR_TIMEOUT: return "BL_ERR_TIMEOUT: a device-side bounded wait ran out";
    case BL_ERR_UNSUPPORTED: return "BL_ERR_UNSUPPORTED: needs a compute capability 10.0 (B200, sm_100a) device";
    default: return "unknown status";
    }
}

const char *bitlinear_last_cuda_error(void) { return g_cuda_err; }

size_t bitlinear_packed_bytes(int64_t N, int64_t K)
{
    if (!valid_nk(N, K))
        return 0;
    return static_cast<size_t>((N + 7) / 8 * 8) * static_cast<size_t>(K / 4);
}

size_t bitlinear_pack_workspace_bytes(int64_t N, int64_t K)
{
    if (!valid_nk(N, K))
        return 0;
    return static_cast<size_t>(N) * sizeof(double);
}

int bitlinear_pack(const void *W, int wt, int64_t N, int64_t K, uint8_t *packed,
                   float *w_scale, void *ws, size_t ws_bytes, void *stream)
{
    if (!W || !packed || !w_scale)
        return BL_ERR_NULL;
    if (!valid_dtype(wt))
        return BL_ERR_DTYPE;
    if (!valid_nk(N, K))
        return BL_ERR_SHAPE;
    if (!aligned16(W) || !aligned16(packed) || !aligned16(ws) || (reinterpret_cast<uintptr_t>(w_scale) & 3u))
        return BL_ERR_ALIGN;
    const DeviceInfo *di;
    int st = need_device(&di);
    if (st)
        return st;
    if ((st = check_dev_ptrs({W, packed, w_scale, ws})))
        return st;
    if (!ws || ws_bytes < bitlinear_pack_workspace_bytes(N, K))
        return BL_ERR_WORKSPACE;
    return launch_pack(W, wt, N, K, packed, w_scale, static_cast<double *>(ws),
                       static_cast<cudaStream_t>(stream));
}

int bitlinear_quantize_act(const void *x, int xt, int64_t M, int64_t K, int64_t ldx,
                           int8_t *q, float *d, int32_t *rowsum, void *stream)
{
    if (!x || !q || !d || !rowsum)
        return BL_ERR_NULL;
    if (!valid_dtype(xt))
        return BL_ERR_DTYPE;
    if (!valid_nk(1, K) || M < 1 || M > (int64_t(1) << 31) || ldx < K)
        return BL_ERR_SHAPE;
    if (!aligned16(x) || !aligned16(q) || (ldx * elem_bytes(xt)) % 16 ||
        (reinterpret_cast<uintptr_t>(d) & 3u) || (reinterpret_cast<uintptr_t>(rowsum) & 3u))
        return BL_ERR_ALIGN;
    const DeviceInfo *di;
    int st = need_device(&di);
    if (st)
        return st;
    if ((st = check_dev_ptrs({x, q, d, rowsum})))
        return st;
    return launch_quantize_act(x, xt, M, K, ldx, q, d, rowsum,
                               static_cast<cudaStream_t>(stream));
}

int bitlinear_rmsnorm_quantize_act(const void *x, int xt, int64_t M, int64_t K, int64_t ldx,
                                   const void *gain, int gt, float eps, int8_t *q, float *d,
                                   int32_t *rowsum, void *stream)
{
    if (!x || !q || !d || !rowsum)
        return BL_ERR_NULL;
    if (!valid_dtype(xt) || (gain && !valid_dtype(gt)))
        return BL_ERR_DTYPE;
    if (!valid_nk(1, K) || M < 1 || M > (int64_t(1) << 31) || ldx < K || !(eps >= 0.0f) ||
        !(eps <= 3.0e38f) || !rmsnorm_quantize_fits(xt, K, gain != nullptr))
        return BL_ERR_SHAPE;
    if (!aligned16(x) || !aligned16(q) || !aligned16(gain) || (ldx * elem_bytes(xt)) % 16 ||
        (reinterpret_cast<uintptr_t>(d) & 3u) || (reinterpret_cast<uintptr_t>(rowsum) & 3u))
        return BL_ERR_ALIGN;
    const DeviceInfo *di;
    int st = need_device(&di);
    if (st)
        return st;
    if ((st = check_dev_ptrs({x, gain, q, d, rowsum})))
        return st;
    return launch_rmsnorm_quantize_act(x, xt, M, K, ldx, gain, gt, eps, q, d, rowsum,
                                       static_cast<cudaStream_t>(stream));
}

namespace {

int check_gemv_common(const uint8_t *packed, const float *w_scale, int64_t N,
                      int64_t K, int64_t M, void *y, int yt, int64_t ldy,
                      int64_t max_m)
{
    if (!packed || !w_scale || !y)
        return BL_ERR_NULL;
    if (!valid_dtype(yt))
        return BL_ERR_DTYPE;
    if (!valid_nk(N, K) || M < 1 || M > max_m || ldy < N)
        return BL_ERR_SHAPE;
    if (!aligned16(packed) || (reinterpret_cast<uintptr_t>(w_scale) & 3u) ||
        (reinterpret_cast<uintptr_t>(y) & (yt == BL_BF16 ? 1u : 3u)))
        return BL_ERR_ALIGN;
    return BL_OK;
}

constexpr int64_t kGemvMaxM = 16;
constexpr int64_t kGemvTensorM = 8;     // above this, bitlinear_gemv may take the tcgen05 GEMM
constexpr int64_t kGemvMaxMK = 163840;

}  // namespace

int bitlinear_gemv(const uint8_t *packed, const float *w_scale, int64_t N, int64_t K,
                   const int8_t *q, const float *d, const int32_t *rowsum, int64_t M,
                   void *y, int yt, int64_t ldy, int32_t *acc_dbg, void *stream)
{
    if (!q || !d || !rowsum)
        return BL_ERR_NULL;
    int st = check_gemv_common(packed, w_scale, N, K, M, y, yt, ldy, kGemvMaxM);
    if (st)
        return st;
    if (M * K > kGemvMaxMK)
        return BL_ERR_SHAPE;
    if (!aligned16(q) || (reinterpret_cast<uintptr_t>(d) & 3u) ||
        (reinterpret_cast<uintptr_t>(rowsum) & 3u) || (reinterpret_cast<uintptr_t>(acc_dbg) & 3u))
        return BL_ERR_ALIGN;
    const DeviceInfo *di;
    if ((st = need_device(&di)))
        return st;
    if ((st = check_dev_ptrs({packed, w_scale, q, d, rowsum, y, acc_dbg})))
        return st;
    GemvArgs a{packed, w_scale, N, K, M, q, d, rowsum, nullptr, BL_F32, 0, y, yt, ldy, acc_dbg};
    // beyond kGemvTensorM tokens, where neither small-batch kernel takes the
    // shape (tensor-core or multi-token streaming), the per-warp dp4a work
    // outgrows the weight stream: the product runs on the tcgen05 GEMM
    // (same results)
    if (M > kGemvTensorM) {
        GemvBatch b{};
        b.count = 1;
        b.prob[0].N = N;
        b.K = K;
        b.M = M;
        b.xt = BL_F32;
        int cluster = 0;
        if (plan_gemv_batch(b, false, &cluster) == BL_GEMV_KERNEL_DP4A)
            return launch_gemm(a, nullptr, 0, static_cast<cudaStream_t>(stream));
    }
    return launch_gemv(a, false, static_cast<cudaStream_t>(stream));
}

int bitlinear_gemv_fused(const uint8_t *packed, const float *w_scale, int64_t N,
                         int64_t K, const void *x, int xt, int64_t ldx, int64_t M,
                         void *y, int yt, int64_t ldy, int32_t *acc_dbg, void *stream)
{
    if (!x)
        return BL_ERR_NULL;
    int st = check_gemv_common(packed, w_scale, N, K, M, y, yt, ldy, kGemvMaxM);
    if (st)
        return st;
    if (!valid_dtype(xt))
        return BL_ERR_DTYPE;
    if (M * K > kGemvMaxMK || ldx < K)
        return BL_ERR_SHAPE;
    if (!aligned16(x) || (ldx * elem_bytes(xt)) % 16 ||
        (reinterpret_cast<uintptr_t>(acc_dbg) & 3u))
        return BL_ERR_ALIGN;
    const DeviceInfo *di;
    if ((st = need_device(&di)))
        return st;
    if ((st = check_dev_ptrs({packed, w_scale, x, y, acc_dbg})))
        return st;
    GemvArgs a{packed, w_scale, N, K, M, nullptr, nullptr, nullptr, x, xt, ldx, y, yt, ldy, acc_dbg};
    return launch_gemv(a, true, static_cast<cudaStream_t>(stream));
}

int bitlinear_gemv_fused_multi(int count, const uint8_t *const *packed,
                               const float *const *w_scale, const int64_t *N, int64_t K,
                               const void *x, int xt, int64_t ldx, int64_t M, void *const *y,
                               int yt, const int64_t *ldy, int32_t *const *acc_dbg,
                               unsigned flags, void *stream)
{
    if (!packed || !w_scale || !N || !y || !ldy || !x)
        return BL_ERR_NULL;
    if (count < 1 || count > kGemvMaxProblems)
        return BL_ERR_SHAPE;
    if ((flags & ~(BL_FLAG_PDL | BL_FLAG_SMALL_BATCH_DP4A | BL_FLAG_SMALL_BATCH_TENSOR)) ||
        (flags & BL_FLAG_SMALL_BATCH_DP4A && flags & BL_FLAG_SMALL_BATCH_TENSOR))
        return BL_ERR_SHAPE;
    if (!valid_dtype(xt) || !valid_dtype(yt))
        return BL_ERR_DTYPE;
    if (M * K > kGemvMaxMK || ldx < K)
        return BL_ERR_SHAPE;
    int st;
    for (int i = 0; i < count; ++i) {
        if ((st = check_gemv_common(packed[i], w_scale[i], N[i], K, M, y[i], yt, ldy[i],
                                    kGemvMaxM)))
            return st;
        if (acc_dbg && (reinterpret_cast<uintptr_t>(acc_dbg[i]) & 3u))
            return BL_ERR_ALIGN;
    }
    if (!aligned16(x) || (ldx * elem_bytes(xt)) % 16)
        return BL_ERR_ALIGN;
    const DeviceInfo *di;
    if ((st = need_device(&di)))
        return st;
    if ((st = check_dev_ptrs({x})))
        return st;
    GemvBatch b{};
    b.count = count;
    for (int i = 0; i < count; ++i) {
        if ((st = check_dev_ptrs({packed[i], w_scale[i], y[i], acc_dbg ? acc_dbg[i] : nullptr})))
            return st;
        b.prob[i] = GemvProblem{packed[i], w_scale[i], N[i], y[i], ldy[i],
                                acc_dbg ? acc_dbg[i] : nullptr};
    }
    b.K = K;
    b.M = M;
    b.x = x;
    b.xt = xt;
    b.ldx = ldx;
    b.yt = yt;
    b.flags = flags;
    return launch_gemv_batch(b, true, static_cast<cudaStream_t>(stream));
}

int bitlinear_gemv_plan(int count, const int64_t *N, int64_t K, int64_t M, int xt,
                        int fused, unsigned flags, int *kernel, int *cluster)
{
    if (!N || !kernel || !cluster)
        return BL_ERR_NULL;
    if (count < 1 || count > kGemvMaxProblems || K < 1 || M < 1 || M > kGemvMaxM ||
        (flags & ~(BL_FLAG_PDL | BL_FLAG_SMALL_BATCH_DP4A | BL_FLAG_SMALL_BATCH_TENSOR)) ||
        (flags & BL_FLAG_SMALL_BATCH_DP4A && flags & BL_FLAG_SMALL_BATCH_TENSOR))
        return BL_ERR_SHAPE;
    if (!valid_dtype(xt))
        return BL_ERR_DTYPE;
    GemvBatch b{};
    b.count = count;
    for (int i = 0; i < count; ++i) {
        if (N[i] < 1)
            return BL_ERR_SHAPE;
        b.prob[i].N = N[i];
    }
    b.K = K;
    b.M = M;
    b.xt = xt;
    b.flags = flags;
    const DeviceInfo *di;
    int st = need_device(&di);
    if (st)
        return st;
    const int k = plan_gemv_batch(b, fused != 0, cluster);
    if (k < 0)
        return BL_ERR_CUDA;
    *kernel = k;
    return BL_OK;
}

int bitlinear_rmsnorm_gemv_fused_multi(int count, const uint8_t *const *packed,
                                       const float *const *w_scale, const int64_t *N, int64_t K,
                                       const void *x, int xt, const void *gain, int gt, float eps,
                                       void *const *y, int yt, const int64_t *ldy,
                                       int32_t *const *acc_dbg, unsigned flags, void *stream)
{
    if (!packed || !w_scale || !N || !y || !ldy || !x)
        return BL_ERR_NULL;
    if (count < 1 || count > kGemvMaxProblems)
        return BL_ERR_SHAPE;
    if (flags & ~BL_FLAG_PDL)
        return BL_ERR_SHAPE;
    if (!valid_dtype(xt) || !valid_dtype(yt) || (gain && !valid_dtype(gt)))
        return BL_ERR_DTYPE;
    if (!(eps >= 0.0f) || !(eps <= 3.0e38f))
        return BL_ERR_SHAPE;
    int st;
    for (int i = 0; i < count; ++i) {
        if ((st = check_gemv_common(packed[i], w_scale[i], N[i], K, 1, y[i], yt, ldy[i], 1)))
            return st;
        if (acc_dbg && (reinterpret_cast<uintptr_t>(acc_dbg[i]) & 3u))
            return BL_ERR_ALIGN;
    }
    if (!aligned16(x) || !aligned16(gain))
        return BL_ERR_ALIGN;
    const DeviceInfo *di;
    if ((st = need_device(&di)))
        return st;
    GemvBatch b{};
    b.count = count;
    for (int i = 0; i < count; ++i)
        b.prob[i] = GemvProblem{packed[i], w_scale[i], N[i], y[i], ldy[i],
                                acc_dbg ? acc_dbg[i] : nullptr};
    b.K = K;
    b.M = 1;
    b.x = x;
    b.xt = xt;
    b.ldx = K;
    b.yt = yt;
    b.flags = flags;
    // the streaming one-token kernel only: K a multiple of 256 up to 32768
    if (!gemv_stream_applies(b, di->sm_count))
        return BL_ERR_SHAPE;
    if ((st = check_dev_ptrs({x, gain})))
        return st;
    for (int i = 0; i < count; ++i)
        if ((st = check_dev_ptrs({packed[i], w_scale[i], y[i], acc_dbg ? acc_dbg[i] : nullptr})))
            return st;
    return launch_gemv_stream(b, true, static_cast<cudaStream_t>(stream), gain, gt, eps, true);
}

int bitlinear_decode_linear(int count, const uint8_t *const *packed, const float *const *w_scale,
                            const int64_t *N, int64_t K, int act, const void *x, int xt,
                            const void *x2, const void *gain, int gt, float eps, void *const *y,
                            int yt, const int64_t *ldy, const void *const *resid,
                            int32_t *const *acc_dbg, unsigned flags, void *stream)
{
    if (!packed || !w_scale || !N || !y || !ldy || !x)
        return BL_ERR_NULL;
    if (act == BL_ACT_RELU2_GATE && !x2)
        return BL_ERR_NULL;
    if (count < 1 || count > kGemvMaxProblems || (flags & ~BL_FLAG_PDL) ||
        (act != BL_ACT_PLAIN && act != BL_ACT_RMSNORM && act != BL_ACT_RELU2_GATE))
        return BL_ERR_SHAPE;
    if (!valid_dtype(xt) || !valid_dtype(yt) || (gain && !valid_dtype(gt)) ||
        (act == BL_ACT_RELU2_GATE && xt != BL_BF16))
        return BL_ERR_DTYPE;
    bool any_resid = false;
    if (resid)
        for (int i = 0; i < count; ++i)
            any_resid = any_resid || resid[i] != nullptr;
    if (any_resid && yt != BL_BF16)
        return BL_ERR_DTYPE;
    if (act == BL_ACT_RMSNORM && (!(eps >= 0.0f) || !(eps <= 3.0e38f)))
        return BL_ERR_SHAPE;
    int st;
    for (int i = 0; i < count; ++i) {
        if ((st = check_gemv_common(packed[i], w_scale[i], N[i], K, 1, y[i], yt, ldy[i], 1)))
            return st;
        if ((acc_dbg && (reinterpret_cast<uintptr_t>(acc_dbg[i]) & 3u)) ||
            (resid && (reinterpret_cast<uintptr_t>(resid[i]) & 1u)))
            return BL_ERR_ALIGN;
    }
    if (!aligned16(x) || !aligned16(x2) || !aligned16(gain))
        return BL_ERR_ALIGN;
    const DeviceInfo *di;
    if ((st = need_device(&di)))
        return st;
    GemvBatch b{};
    b.count = count;
    for (int i = 0; i < count; ++i) {
        b.prob[i] = GemvProblem{packed[i], w_scale[i], N[i], y[i], ldy[i], acc_dbg ? acc_dbg[i] : nullptr,
                                resid ? resid[i] : nullptr};
    }
    b.K = K;
    b.M = 1;
    b.x = x;
    b.xt = xt;
    b.ldx = K;
    b.yt = yt;
    b.flags = flags;
    if (!gemv_stream_applies(b, di->sm_count))
        return BL_ERR_SHAPE;
    if ((st = check_dev_ptrs({x, x2, gain})))
        return st;
    for (int i = 0; i < count; ++i)
        if ((st = check_dev_ptrs({packed[i], w_scale[i], y[i], acc_dbg ? acc_dbg[i] : nullptr,
                                  resid ? resid[i] : nullptr})))
            return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (act == BL_ACT_RELU2_GATE)
        return launch_gemv_stream_relu2(b, x2, s);
    return launch_gemv_stream(b, true, s, gain, gt, eps, act == BL_ACT_RMSNORM);
}

size_t bitlinear_attention_workspace_bytes(int H, int Hkv, int T_max)
{
    if (H < 1 || Hkv < 1 || H % Hkv || H / Hkv > attention_max_group() || T_max < 1 ||
        T_max > 32768)
        return 0;
    return attention_workspace_bytes(H, Hkv, T_max);
}

int bitlinear_rope_table(int D, int T_max, double rope_base, float *table, void *stream)
{
    if (!table)
        return BL_ERR_NULL;
    if (D != 128 || T_max < 1 || T_max > 32768 || !(rope_base > 1.0) || !(rope_base < 1e30))
        return BL_ERR_SHAPE;
    if (reinterpret_cast<uintptr_t>(table) & 7u)
        return BL_ERR_ALIGN;
    const DeviceInfo *di;
    int st = need_device(&di);
    if (st)
        return st;
    if ((st = check_dev_ptrs({table})))
        return st;
    return launch_rope_table(table, D, T_max, rope_base, static_cast<cudaStream_t>(stream));
}

int bitlinear_attention_decode(const void *q, const void *k, const void *v, void *cache_k,
                               void *cache_v, const int32_t *pos, int H, int Hkv, int D,
                               int T_max, double rope_base, const float *rope_table, void *out,
                               void *ws, size_t ws_bytes, unsigned flags, void *stream)
{
    if (!q || !k || !v || !cache_k || !cache_v || !pos || !out)
        return BL_ERR_NULL;
    if (H < 1 || Hkv < 1 || H % Hkv || H / Hkv > attention_max_group() || D != 128 ||
        T_max < 1 || T_max > 32768 || !(rope_base > 1.0) || !(rope_base < 1e30) ||
        (flags & ~BL_FLAG_PDL) || Hkv > 65535)
        return BL_ERR_SHAPE;
    if ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) | reinterpret_cast<uintptr_t>(v) |
         reinterpret_cast<uintptr_t>(cache_k) | reinterpret_cast<uintptr_t>(cache_v) |
         reinterpret_cast<uintptr_t>(out)) & 15u || (reinterpret_cast<uintptr_t>(pos) & 3u) ||
        !aligned16(ws) || (reinterpret_cast<uintptr_t>(rope_table) & 7u))
        return BL_ERR_ALIGN;
    const DeviceInfo *di;
    int st = need_device(&di);
    if (st)
        return st;
    if ((st = check_dev_ptrs({q, k, v, cache_k, cache_v, pos, out, ws, rope_table})))
        return st;
    if (!ws || ws_bytes < attention_workspace_bytes(H, Hkv, T_max))
        return BL_ERR_WORKSPACE;
    return launch_attention_decode(q, k, v, cache_k, cache_v, pos, H, Hkv, D, T_max, rope_base,
                                   rope_table, out, ws, flags, static_cast<cudaStream_t>(stream));
}

int bitlinear_position_advance(int32_t *pos, void *stream)
{
    if (!pos)
        return BL_ERR_NULL;
    if (reinterpret_cast<uintptr_t>(pos) & 3u)
        return BL_ERR_ALIGN;
    const DeviceInfo *di;
    int st = need_device(&di);
    if (st)
        return st;
    if ((st = check_dev_ptrs({pos})))
        return st;
    return launch_position_advance(pos, static_cast<cudaStream_t>(stream));
}

size_t bitlinear_chain_plan_bytes(int nsteps) { return chain_plan_bytes(nsteps); }

int bitlinear_chain_plan(int nsteps, const bitlinear_chain_step *steps, void *plan,
                         size_t plan_bytes, void *stream)
{
    if (!steps || !plan)
        return BL_ERR_NULL;
    if (nsteps < 1 || nsteps > BITLINEAR_CHAIN_MAX_STEPS)
        return BL_ERR_SHAPE;
    int st;
    for (int i = 0; i < nsteps; ++i) {
        const bitlinear_chain_step &d = steps[i];
        if (!d.x)
            return BL_ERR_NULL;
        if (d.count < 1 || d.count > kGemvMaxProblems)
            return BL_ERR_SHAPE;
        if (!valid_dtype(d.xt) || !valid_dtype(d.yt) || (d.gain && !valid_dtype(d.gt)))
            return BL_ERR_DTYPE;
        if (!chain_step_fits(d.K) || !(d.eps >= 0.0f) || !(d.eps <= 3.0e38f))
            return BL_ERR_SHAPE;
        for (int j = 0; j < d.count; ++j) {
            if ((st = check_gemv_common(d.packed[j], d.w_scale[j], d.N[j], d.K, 1, d.y[j], d.yt,
                                        d.N[j], 1)))
                return st;
            if (reinterpret_cast<uintptr_t>(d.acc_dbg[j]) & 3u)
                return BL_ERR_ALIGN;
        }
        if (!aligned16(d.x) || !aligned16(d.gain))
            return BL_ERR_ALIGN;
    }
    if (plan_bytes < chain_plan_bytes(nsteps))
        return BL_ERR_WORKSPACE;
    if (!aligned16(plan))
        return BL_ERR_ALIGN;
    const DeviceInfo *di;
    if ((st = need_device(&di)))
        return st;
    if ((st = check_dev_ptrs({plan})))
        return st;
    for (int i = 0; i < nsteps; ++i) {
        const bitlinear_chain_step &d = steps[i];
        if ((st = check_dev_ptrs({d.x, d.gain})))
            return st;
        for (int j = 0; j < d.count; ++j)
            if ((st = check_dev_ptrs({d.packed[j], d.w_scale[j], d.y[j], d.acc_dbg[j]})))
                return st;
    }
    return build_chain_plan(nsteps, steps, plan, static_cast<cudaStream_t>(stream));
}

int bitlinear_chain_run(const void *plan, int nsteps, void *stream)
{
    if (!plan)
        return BL_ERR_NULL;
    if (nsteps < 1 || nsteps > BITLINEAR_CHAIN_MAX_STEPS)
        return BL_ERR_SHAPE;
    if (!aligned16(plan))
        return BL_ERR_ALIGN;
    const DeviceInfo *di;
    int st = need_device(&di);
    if (st)
        return st;
    if ((st = check_dev_ptrs({plan})))
        return st;
    return launch_chain(plan, nsteps, static_cast<cudaStream_t>(stream), 2000000000ull, -1);
}

int bitlinear_chain_run_timeout_test(const void *plan, int nsteps, uint64_t wait_limit_ns,
                                     void *stream)
{
    if (!plan)
        return BL_ERR_NULL;
    if (nsteps < 2 || nsteps > BITLINEAR_CHAIN_MAX_STEPS || wait_limit_ns < 1000 ||
        wait_limit_ns > 2000000000ull)
        return BL_ERR_SHAPE;
    if (!aligned16(plan))
        return BL_ERR_ALIGN;
    const DeviceInfo *di;
    int st = need_device(&di);
    if (st)
        return st;
    if ((st = check_dev_ptrs({plan})))
        return st;
    return launch_chain(plan, nsteps, static_cast<cudaStream_t>(stream), wait_limit_ns, 1);
}

size_t bitlinear_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K)
{
    if (!valid_nk(N, K) || M < 1)
        return 0;
    return gemm_workspace_bytes(M, N, K);
}

int bitlinear_gemm(const uint8_t *packed, const float *w_scale, int64_t N, int64_t K,
                   const int8_t *q, const float *d, const int32_t *rowsum, int64_t M,
                   void *y, int yt, int64_t ldy, int32_t *acc_dbg, void *ws,
                   size_t ws_bytes, void *stream)
{
    if (!q || !d || !rowsum)
        return BL_ERR_NULL;
    int st = check_gemv_common(packed, w_scale, N, K, M, y, yt, ldy, int64_t(1) << 31);
    if (st)
        return st;
    if (!aligned16(q) || (reinterpret_cast<uintptr_t>(d) & 3u) ||
        (reinterpret_cast<uintptr_t>(rowsum) & 3u) || (reinterpret_cast<uintptr_t>(acc_dbg) & 3u) ||
        !aligned16(ws))
        return BL_ERR_ALIGN;
    const DeviceInfo *di;
    if ((st = need_device(&di)))
        return st;
    if ((st = check_dev_ptrs({packed, w_scale, q, d, rowsum, y, acc_dbg, ws})))
        return st;
    size_t need = gemm_workspace_bytes(M, N, K);
    if (need && (!ws || ws_bytes < need))
        return BL_ERR_WORKSPACE;
    GemvArgs a{packed, w_scale, N, K, M, q, d, rowsum, nullptr, BL_F32, 0, y, yt, ldy, acc_dbg};
    return launch_gemm(a, ws, ws_bytes, static_cast<cudaStream_t>(stream));
}

size_t bitlinear_binary_packed_bytes(int64_t N, int64_t K)
{
    if (!valid_nk(N, K))
        return 0;
    return static_cast<size_t>(N) * static_cast<size_t>(K / 64) * 8;
}

int bitlinear_binary_pack(const void *W, int wt, int64_t N, int64_t K, uint64_t *Wb,
                          float *s_w, void *stream)
{
    if (!W || !Wb || !s_w)
        return BL_ERR_NULL;
    if (!valid_dtype(wt))
        return BL_ERR_DTYPE;
    if (!valid_nk(N, K))
        return BL_ERR_SHAPE;
    if (!aligned16(W) || !aligned16(Wb) || (reinterpret_cast<uintptr_t>(s_w) & 3u))
        return BL_ERR_ALIGN;
    const DeviceInfo *di;
    int st = need_device(&di);
    if (st)
        return st;
    if ((st = check_dev_ptrs({W, Wb, s_w})))
        return st;
    return launch_binary_pack(W, wt, N, K, Wb, s_w, static_cast<cudaStream_t>(stream));
}

int bitlinear_binary_gemv(const uint64_t *Wb, const float *s_w, int64_t N, int64_t K,
                          const void *x, int xt, void *y, int yt, int32_t *acc_dbg,
                          void *stream)
{
    if (!Wb || !s_w || !x || !y)
        return BL_ERR_NULL;
    if (!valid_dtype(xt) || !valid_dtype(yt))
        return BL_ERR_DTYPE;
    if (!valid_nk(N, K) || K > 65536)
        return BL_ERR_SHAPE;
    if (!aligned16(Wb) || !aligned16(x) || (reinterpret_cast<uintptr_t>(s_w) & 3u) ||
        (reinterpret_cast<uintptr_t>(y) & (yt == BL_BF16 ? 1u : 3u)) ||
        (reinterpret_cast<uintptr_t>(acc_dbg) & 3u))
        return BL_ERR_ALIGN;
    const DeviceInfo *di;
    int st = need_device(&di);
    if (st)
        return st;
    if ((st = check_dev_ptrs({Wb, s_w, x, y, acc_dbg})))
        return st;
    if (popc_stream_applies_binary(K))
        return launch_binary_gemv_stream(Wb, s_w, N, K, x, xt, y, yt, acc_dbg,
                                         static_cast<cudaStream_t>(stream));
    return launch_binary_gemv(Wb, s_w, N, K, x, xt, y, yt, acc_dbg,
                              static_cast<cudaStream_t>(stream));
}

int bitlinear_lut_gemv(const uint8_t *packed, const float *w_scale, int64_t N, int64_t K,
                       const int8_t *q, const float *d, void *y, int yt, int32_t *acc_dbg,
                       void *stream)
{
    if (!q || !d)
        return BL_ERR_NULL;
    int st = check_gemv_common(packed, w_scale, N, K, 1, y, yt, N, 1);
    if (st)
        return st;
    if (!lut_gemv_applies(K))
        return BL_ERR_SHAPE;
    if ((reinterpret_cast<uintptr_t>(d) & 3u) || (reinterpret_cast<uintptr_t>(acc_dbg) & 3u))
        return BL_ERR_ALIGN;
    const DeviceInfo *di;
    if ((st = need_device(&di)))
        return st;
    if ((st = check_dev_ptrs({packed, w_scale, q, d, y, acc_dbg})))
        return st;
    return launch_lut_gemv(packed, w_scale, N, K, q, d, y, yt, acc_dbg,
                           static_cast<cudaStream_t>(stream));
}

size_t bitlinear_bitplane_bytes(int64_t N, int64_t K)
{
    if (!valid_nk(N, K))
        return 0;
    return static_cast<size_t>(N) * static_cast<size_t>(K / 64) * 16;
}

int bitlinear_bitplane_pack(const uint8_t *packed, int64_t N, int64_t K, uint64_t *planes,
                            void *stream)
{
    if (!packed || !planes)
        return BL_ERR_NULL;
    if (!valid_nk(N, K) || K > 65536)
        return BL_ERR_SHAPE;
    if (!aligned16(packed) || !aligned16(planes))
        return BL_ERR_ALIGN;
    const DeviceInfo *di;
    int st = need_device(&di);
    if (st)
        return st;
    if ((st = check_dev_ptrs({packed, planes})))
        return st;
    return launch_bitplane_pack(packed, N, K, planes, static_cast<cudaStream_t>(stream));
}

int bitlinear_bitplane_gemv(const uint64_t *planes, const float *w_scale, int64_t N, int64_t K,
                            const void *x, int xt, void *y, int yt, int32_t *acc_dbg,
                            void *stream)
{
    if (!planes || !w_scale || !x || !y)
        return BL_ERR_NULL;
    if (!valid_dtype(xt) || !valid_dtype(yt))
        return BL_ERR_DTYPE;
    if (!valid_nk(N, K) || K > 65536)
        return BL_ERR_SHAPE;
    if (!aligned16(planes) || !aligned16(x) || (reinterpret_cast<uintptr_t>(w_scale) & 3u) ||
        (reinterpret_cast<uintptr_t>(y) & (yt == BL_BF16 ? 1u : 3u)) ||
        (reinterpret_cast<uintptr_t>(acc_dbg) & 3u))
        return BL_ERR_ALIGN;
    const DeviceInfo *di;
    int st = need_device(&di);
    if (st)
        return st;
    if ((st = check_dev_ptrs({planes, w_scale, x, y, acc_dbg})))
        return st;
    return launch_bitplane_gemv(planes, w_scale, N, K, x, xt, y, yt, acc_dbg,
                                static_cast<cudaStream_t>(stream));
}

static int probe_mma(int n, int issuers, int reps, long long *out, int grid, void *stream)
{
    if (!out)
        return BL_ERR_NULL;
    if (reps < 1 || reps > (1 << 17) || grid < 1)   // (1 << 17) stages: ~35 ms, far inside the 2 s wait
        return BL_ERR_SHAPE;
    if (!((n == 128 && (issuers == 1 || issuers == 2)) || (n == 32 && (issuers == 1 || issuers == 2 || issuers == 4))))
        return BL_ERR_SHAPE;
    if (reinterpret_cast<uintptr_t>(out) & 7u)
        return BL_ERR_ALIGN;
    const DeviceInfo *di;
    int st = need_device(&di);
    if (st)
        return st;
    if (grid > di->sm_count)
        return BL_ERR_SHAPE;
    if ((st = check_dev_ptrs({out})))
        return st;
    return launch_mma_probe(n, issuers, reps, out, grid, static_cast<cudaStream_t>(stream));
}

int bitlinear_probe_mma_i8(int reps, long long *out, int grid, void *stream)
{
    return probe_mma(128, 1, reps, out, grid, stream);
}

int bitlinear_probe_mma_i8_issue(int n, int issuers, int reps, long long *out, int grid, void *stream)
{
    return probe_mma(n, issuers, reps, out, grid, stream);
}

int bitlinear_last_device_status(void *stream)
{
    const DeviceInfo *di = device_info();
    if (!di)
        return BL_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int st = cuda_status(cudaStreamSynchronize(s));
    if (st)
        return st;
    int v = 0;
    st = cuda_status(cudaMemcpy(&v, di->status, sizeof v, cudaMemcpyDeviceToHost));
    if (st)
        return st;
    if (v != 0) {
        int zero = 0;
        st = cuda_status(cudaMemcpy(di->status, &zero, sizeof zero, cudaMemcpyHostToDevice));
        if (st)
            return st;
    }
    return v;
}

int bitlinear_device_sm_count(void)
{
    const DeviceInfo *di = device_info();
    return di ? di->sm_count : 0;
}

}  // extern "C"
