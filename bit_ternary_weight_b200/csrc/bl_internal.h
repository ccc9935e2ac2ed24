// bl_internal.h -- host-side declarations shared by the translation units of
// libbitlinear.so (launchers, device properties, error bookkeeping).
#pragma once

#include <cuda_runtime.h>
#include <initializer_list>
#include <stddef.h>
#include <stdint.h>

#include "../../include/bitlinear.h"

namespace bl {

struct DeviceInfo {
    int device = -1;
    int sm_count = 0;
    int max_smem_optin = 0;     // bytes per block with opt-in
    int cc_major = 0, cc_minor = 0;
    int *status = nullptr;      // device address of the status word
};

// Properties of the current device (cached per device).  nullptr on error.
const DeviceInfo *device_info();

// --- argument checks shared by every entry point -------------------------

// Device (or managed) memory of the current device.
bool is_device_ptr(const void *p);

// N >= 1, K >= 64, K % 64 == 0, within the index ranges the kernels use.
bool valid_nk(int64_t N, int64_t K);

// A compute capability 10.0 device is current: BL_OK and its info, else
// BL_ERR_CUDA / BL_ERR_UNSUPPORTED.
int need_device(const DeviceInfo **out);

// BL_ERR_NOT_DEVICE_PTR if any non-NULL pointer is not device memory of the
// current device, else BL_OK.
int check_dev_ptrs(std::initializer_list<const void *> ptrs);

// Records `e` as the last CUDA error of this thread and returns BL_ERR_CUDA,
// or BL_OK when e == cudaSuccess.
int cuda_status(cudaError_t e);

// Launch-error check after a kernel launch.
int launch_status();

// Resident CTAs per SM of `func` at this block size and dynamic shared memory,
// with the kernel's dynamic shared memory limit raised to the device maximum
// on first use.  Cached per (device, func, threads, smem).
int occupancy(const void *func, int threads, size_t smem, int *per_sm);

// --- launchers (arguments already validated) ------------------------------

int launch_quantize_act(const void *x, int xt, int64_t M, int64_t K,
                        int64_t ldx, int8_t *q, float *d, int32_t *rowsum,
                        cudaStream_t s);

// RMSNorm, then per-token absmax quantisation of the normalised rows.
int launch_rmsnorm_quantize_act(const void *x, int xt, int64_t M, int64_t K, int64_t ldx,
                                const void *gain, int gt, float eps, int8_t *q, float *d,
                                int32_t *rowsum, cudaStream_t s);
// Whether a row of K elements (and the gain) fits the RMSNorm kernel's
// shared-memory staging.
bool rmsnorm_quantize_fits(int xt, int64_t K, bool has_gain);

int launch_pack(const void *W, int wt, int64_t N, int64_t K, uint8_t *packed,
                float *w_scale, double *row_sums, cudaStream_t s);

struct GemvArgs {
    const uint8_t *packed;
    const float *w_scale;
    int64_t N, K, M;
    // exactly one of (q, d, rowsum) or (x, xt, ldx) is used
    const int8_t *q;
    const float *d;
    const int32_t *rowsum;
    const void *x;
    int xt;
    int64_t ldx;
    void *y;
    int yt;
    int64_t ldy;
    int32_t *acc_dbg;
};

int launch_gemv(const GemvArgs &a, bool fused, cudaStream_t s);

// Several GEMVs that share their activations, in one launch.
constexpr int kGemvMaxProblems = BITLINEAR_GEMV_MAX_PROBLEMS;

struct GemvProblem {
    const uint8_t *packed;
    const float *w_scale;
    int64_t N;
    void *y;
    int64_t ldy;
    int32_t *acc_dbg;
    const void *resid = nullptr;   // bf16 [N] added before the final rounding (one token, streaming kernel)
};

struct GemvBatch {
    int count;
    GemvProblem prob[kGemvMaxProblems];
    int64_t K, M;
    const int8_t *q;        // pre-quantised activations (unfused), or
    const float *d;
    const int32_t *rowsum;
    const void *x;          // raw activations (fused)
    int xt;
    int64_t ldx;
    int yt;
    unsigned flags;
};

int launch_gemv_batch(const GemvBatch &b, bool fused, cudaStream_t s);

// Which kernel launch_gemv_batch runs for the batch (BL_GEMV_KERNEL_*), and
// for the tensor-core kernel its cluster size (else 0).
int plan_gemv_batch(const GemvBatch &b, bool fused, int *cluster);

// The tensor-core small-batch kernel (gemv_tc.cu): 2 .. 16 tokens, K a
// multiple of 256, bf16 x when fused; whether it takes the batch (a cluster
// split of the row blocks that is resident at once), and its launch.
bool gemv_tc_applies(const GemvBatch &b, bool fused);
int gemv_tc_cluster(const GemvBatch &b, bool fused);   // CTAs per cluster, 0: not taken
int launch_gemv_tc(const GemvBatch &b, bool fused, cudaStream_t s);

// The streaming one-token kernel (gemv_stream.cu): whether it takes the batch,
// and its launch with the token normalised (RMSNorm with gain / eps) before
// quantisation when `norm` is set.
bool gemv_stream_applies(const GemvBatch &b, int sm_count);
int launch_gemv_stream(const GemvBatch &b, bool fused, cudaStream_t s, const void *gain, int gt,
                       float eps, bool norm);
// Small batches (2 .. 16 tokens) on the streaming design (gemv_stream_mt.cu).
bool gemv_stream_mt_applies(const GemvBatch &b, bool fused, int sm_count, int max_smem);
int launch_gemv_stream_mt(const GemvBatch &b, bool fused, cudaStream_t s);

// The same with the squared-ReLU gate in front: the token is relu(x)^2 * x2
// (x, x2 bf16 [K]).
int launch_gemv_stream_relu2(const GemvBatch &b, const void *x2, cudaStream_t s);

// Decode attention of one token (attention.cu).
size_t attention_workspace_bytes(int H, int Hkv, int T_max);
int attention_max_group();
int launch_rope_table(float *tab, int D, int T_max, double base, cudaStream_t s);
int launch_attention_decode(const void *q, const void *k, const void *v, void *cache_k, void *cache_v,
                            const int32_t *pos, int H, int Hkv, int D, int T_max, double rope_base,
                            const float *rope, void *out, void *ws, unsigned flags, cudaStream_t s);
int launch_position_advance(int32_t *pos, cudaStream_t s);

size_t gemm_workspace_bytes(int64_t M, int64_t N, int64_t K);
int launch_gemm(const GemvArgs &a, void *ws, size_t ws_bytes, cudaStream_t s);

int launch_binary_pack(const void *W, int wt, int64_t N, int64_t K,
                       uint64_t *Wb, float *s_w, cudaStream_t s);
int launch_binary_gemv(const uint64_t *Wb, const float *s_w, int64_t N,
                       int64_t K, const void *x, int xt, void *y, int yt,
                       int32_t *acc_dbg, cudaStream_t s);

// Streaming popcount GEMVs (popc_stream.cu): binary weights (rows of K/8
// bytes, which must be a multiple of 16) and ternary bit-planes (rows of K/4
// bytes), K <= 65536.
bool popc_stream_applies_binary(int64_t K);
int launch_binary_gemv_stream(const uint64_t *Wb, const float *s_w, int64_t N, int64_t K,
                              const void *x, int xt, void *y, int yt, int32_t *acc_dbg,
                              cudaStream_t s);
int launch_bitplane_pack(const uint8_t *packed, int64_t N, int64_t K, uint64_t *planes,
                         cudaStream_t s);
int launch_bitplane_gemv(const uint64_t *planes, const float *w_scale, int64_t N, int64_t K,
                         const void *x, int xt, void *y, int yt, int32_t *acc_dbg, cudaStream_t s);

// Lookup-table ternary GEMV of one token (lut_gemv.cu), K <= 12288.
bool lut_gemv_applies(int64_t K);
int launch_lut_gemv(const uint8_t *packed, const float *w_scale, int64_t N, int64_t K,
                    const int8_t *q, const float *d, void *y, int yt, int32_t *acc_dbg,
                    cudaStream_t s);

// int8 tensor-core rate probe (mma_probe.cu): per CTA (clock cycles, ns).
int launch_mma_probe(int n, int issuers, int reps, long long *out, int grid, cudaStream_t s);

// Persistent decode chain (gemv_chain.cu).
size_t chain_plan_bytes(int nsteps);
bool chain_step_fits(int64_t K);
int build_chain_plan(int nsteps, const bitlinear_chain_step *steps, void *plan, cudaStream_t s);
int launch_chain(const void *plan, int nsteps, cudaStream_t s, uint64_t limit_ns, int test_step);

}  // namespace bl
