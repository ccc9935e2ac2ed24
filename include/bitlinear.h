/*
 * bitlinear.h -- C ABI of libbitlinear.so, the B200 (sm_100a) BitNet b1.58
 * BitLinear product.
 *
 * What the library computes (pages cited by title and section):
 *   - per-token absmax int8 activation quantisation ("How to Run BitNet
 *     Inference on GPU Using CUDA Kernels: A Complete Guide", section
 *     "Understanding the Two-Phase Architecture": BitLinearKernel quantises its
 *     inputs to INT8 with scaling factors before the INT2 kernel);
 *   - a product with ternary {-1, 0, +1} weights stored two bits each, with
 *     exact int32 accumulation (same guide, FAQ "Can I use the CUDA kernel for
 *     models other than the default BitNet architecture?": an INT8 x INT2
 *     GEMM; "BitCompute: 1.58-bit LLM Execution Engine", sections "Features"
 *     and "Future Roadmap": add / subtract / skip, four weights per byte);
 *   - the rescale by the per-tensor absmean weight scale and the per-token
 *     activation scale ("bit-floor" README, section "The core math": no
 *     floating point until the final scale multiply; section "What's inside":
 *     mean-abs scale for ternary weights, absmax scale for binary weights);
 *   - the binary 1-bit XNOR / popcount GEMV ("bit-floor" README, section "The
 *     core math": y = scale_w * scale_x * (2 * POPCNT(XNOR(W, x)) - K)).
 *
 * Numerics (identical on the CPU oracle):
 *   gamma     = (float)(sum_n sum_k |W[n][k]| / (N*K)), the sums in fp64, k
 *               ascending inside a row, then rows ascending; gamma_eff =
 *               max(gamma, 1e-5f).  Stored in *w_scale.
 *   code      = clamp(rint(W / gamma_eff), -1, 1), fp32 division, ties to even.
 *   a_m       = max(max_k |x[m][k]|, 1e-5f); s_m = 127 / a_m (fp32);
 *   q[m][k]   = clamp(rint(x * s_m), -128, 127), fp32 product, ties to even;
 *   d[m]      = a_m / 127 (fp32); rowsum[m] = sum_k q[m][k].
 *   acc[m][n] = sum_k code[n][k] * q[m][k] (exact int32, |acc| <= 128 K).
 *   y[m][n]   = ((float)acc * d[m]) * gamma_eff, two fp32 round-to-nearest
 *               products in that order; bf16 output rounds y to nearest even.
 *   Inputs must be finite (the pages define no other case): a NaN or +-Inf
 *   in token m of x leaves q[m], d[m], rowsum[m] and row m of y unspecified,
 *   and one in W leaves gamma and every output unspecified.  Such input
 *   causes no fault and no error status, and other tokens are unaffected.
 *
 * Packed ternary layout "TL" (the pages fix none; this library's choice):
 *   stored value s = code + 1 in {0, 1, 2} (3 never appears), rows padded to
 *   a multiple of 8 with code 0; byte of (n, k) =
 *     ((n/8 * (K/64) + k/64) * 8 + n%8) * 16 + ((k%64)/16) * 4 + k%4,
 *   bit offset 2 * ((k%16)/4).  A 16-byte chunk holds 64 consecutive k of one
 *   row; a 32-bit word w of a chunk gives, after (w >> 2i) & 0x03030303, the
 *   stored codes of four consecutive k in byte order.
 * Binary layout: uint64 [N][K/64], bit j of word w <-> k = 64 w + j, bit set
 *   when the value is negative (-0.0 counts as positive).
 *
 * Conventions for every entry point:
 *   - Pointers named as device pointers must be device (or managed) memory of
 *     the current device; a host pointer, or memory that belongs to another
 *     GPU, gives BL_ERR_NOT_DEVICE_PTR.  Kernels launch on the current device,
 *     so a caller with tensors on another GPU makes that GPU current first.
 *     There is no CPU fallback.
 *   - The library runs on compute capability 10.0 (B200, sm_100a) only; any
 *     other current device gives BL_ERR_UNSUPPORTED.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Every call is asynchronous on it; the caller owns all memory
 *     and keeps it alive until the stream has passed the call.
 *   - The library allocates no device memory.  It keeps a device status word
 *     and cached device properties only.
 *   - Argument errors return before any launch, with nothing written.  A
 *     failed launch returns BL_ERR_CUDA (text via bitlinear_last_cuda_error).
 *     Device-side errors (a bounded wait that ran out) are reported by the next
 *     bitlinear_last_device_status().
 *   - Shapes: N >= 1, K >= 64 and K % 64 == 0, 1 <= M.
 *   - Alignment: weight, packed, q, x and y base pointers 16-byte aligned;
 *     row strides (ldx, ldy) in elements such that each row starts 16-byte
 *     aligned.  Otherwise BL_ERR_ALIGN.
 */
#ifndef BITLINEAR_H
#define BITLINEAR_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    BL_OK = 0,
    BL_ERR_NULL = 1,            /* a required pointer is NULL */
    BL_ERR_DTYPE = 2,           /* unsupported element type */
    BL_ERR_SHAPE = 3,           /* N, K, M, strides out of range */
    BL_ERR_ALIGN = 4,           /* pointer or stride misaligned */
    BL_ERR_NOT_DEVICE_PTR = 5,  /* a device pointer is host or another GPU's memory */
    BL_ERR_WORKSPACE = 6,       /* workspace missing or too small */
    BL_ERR_CUDA = 7,            /* CUDA runtime error */
    BL_ERR_TIMEOUT = 8,         /* a device-side bounded wait ran out */
    BL_ERR_UNSUPPORTED = 9      /* the current device is not compute capability 10.0 */
} bl_status;

typedef enum { BL_F32 = 0, BL_BF16 = 1 } bl_dtype;

/* Human-readable name of a status code (static string). */
const char *bitlinear_status_string(int status);

/* Text of the last CUDA runtime error seen by this library in this thread
 * (static per-thread buffer; "" if none). */
const char *bitlinear_last_cuda_error(void);

/* Bytes of the TL packed array for an N x K weight (rows padded to 8). */
size_t bitlinear_packed_bytes(int64_t N, int64_t K);

/* Bytes of workspace bitlinear_pack needs: one fp64 partial sum per row. */
size_t bitlinear_pack_workspace_bytes(int64_t N, int64_t K);

/*
 * Offline ternary packer: absmean scale, round-clip to {-1, 0, +1}, 2-bit
 * pack into layout TL.  Source: "bit-floor" README, section "What's inside"
 * (mean-abs scale for ternary weights, packing f32 weights); "BitCompute",
 * section "Future Roadmap" (four weights per byte).
 *   W        device, [N][K] row-major, dtype wt (BL_F32 or BL_BF16)
 *   packed   device, bitlinear_packed_bytes(N, K) bytes, written
 *   w_scale  device, 1 float, written with gamma_eff
 *   ws       device workspace of at least bitlinear_pack_workspace_bytes;
 *            contents on entry are ignored, on exit unspecified
 */
int bitlinear_pack(const void *W, int wt, int64_t N, int64_t K,
                   uint8_t *packed, float *w_scale, void *ws, size_t ws_bytes,
                   void *stream);

/* Largest N that bitlinear_pack_noalloc accepts. */
#define BITLINEAR_PACK_NOALLOC_MAX_ROWS 65536

/*
 * bitlinear_pack without a workspace argument: the same result, bit for bit,
 * as bitlinear_pack, for callers that cannot allocate device memory at the
 * time they pack weights -- for example a plain C host with no device
 * allocator of its own, or a runtime whose memory pool already owns the GPU's
 * memory, where a cudaMalloc would fail, fragment the pool or synchronise the
 * device.  The pages have no counterpart of this entry point; it exists for
 * such callers only.
 *   W, wt, N, K, packed, w_scale, stream   as for bitlinear_pack
 * Scratch: the per-row fp64 sums use a device array that lives inside the
 * library, BITLINEAR_PACK_NOALLOC_MAX_ROWS doubles (512 KiB) on every GPU that
 * loads the library, kept until the process exits.  N above
 * BITLINEAR_PACK_NOALLOC_MAX_ROWS returns BL_ERR_SHAPE.  The first call on a
 * device looks up that array's device address (once per device) and should
 * come before any stream capture.  Every call on a device shares the array:
 * calls whose work overlaps on the GPU (different streams with no ordering
 * between them) race and may produce wrong scales.  Nothing in the array needs
 * to start at zero, since every call writes each value it reads.  The call
 * allocates nothing, and frees nothing.
 */
int bitlinear_pack_noalloc(const void *W, int wt, int64_t N, int64_t K,
                           uint8_t *packed, float *w_scale, void *stream);

/*
 * Per-token absmax int8 activation quantisation.  Source: "How to Run BitNet
 * Inference on GPU Using CUDA Kernels", section "Understanding the Two-Phase
 * Architecture" (inputs quantised to INT8 with scaling factors).
 *   x       device, [M][ldx] of dtype xt (BL_F32 or BL_BF16), ldx >= K
 *   q       device, [M][K] int8, written
 *   d       device, [M] float (dequantisation scale a_m / 127), written
 *   rowsum  device, [M] int32 (sum of q over k), written
 */
int bitlinear_quantize_act(const void *x, int xt, int64_t M, int64_t K,
                           int64_t ldx, int8_t *q, float *d, int32_t *rowsum,
                           void *stream);

/*
 * Ternary GEMV for 1 <= M <= 16 tokens on pre-quantised activations.
 * Source: "How to Run BitNet Inference on GPU Using CUDA Kernels", section
 * "Key Components and Source Code Architecture" (the decode-phase INT8 x INT2
 * linear); "bit-floor" README, section "The core math".
 *   packed, w_scale   from bitlinear_pack (device)
 *   q, d, rowsum      from bitlinear_quantize_act (device), q is [M][K]
 *   y                 device, [M][ldy] of dtype yt (BL_F32 or BL_BF16), ldy >= N
 *   acc_dbg           NULL, or device [M][N] int32 receiving acc (before rescale)
 * M * K must not exceed 163840 (the activations are staged on chip).  2 ..
 * 16 tokens run the tensor-core small-batch kernel or the dp4a multi-token
 * streaming kernel (the crossover of BL_FLAG_SMALL_BATCH_DP4A's note), both
 * one pass over the weights for all tokens; above 8 tokens on a shape that
 * neither takes, the product runs on the tcgen05 GEMM of bitlinear_gemm.
 * Results are identical either way.
 */
int bitlinear_gemv(const uint8_t *packed, const float *w_scale, int64_t N,
                   int64_t K, const int8_t *q, const float *d,
                   const int32_t *rowsum, int64_t M, void *y, int yt,
                   int64_t ldy, int32_t *acc_dbg, void *stream);

/*
 * Ternary GEMV with the activation quantisation fused into the kernel: the
 * whole decode BitLinear (quantise, product, rescale) in one launch.
 *   x    device, [M][ldx] of dtype xt (BL_F32 or BL_BF16)
 *   other arguments as for bitlinear_gemv.
 * One token with K a multiple of 256 (at most 32768) runs a streaming kernel
 * (a producer warp fills a shared-memory ring with bulk copies of the packed
 * weights); a chain of such launches on one stream reaches the highest weight
 * bandwidth with bitlinear_gemv_fused_multi and BL_FLAG_PDL inside a CUDA
 * graph.  Other shapes run a kernel with a per-warp weight ring.  Results are
 * identical either way.
 */
int bitlinear_gemv_fused(const uint8_t *packed, const float *w_scale,
                         int64_t N, int64_t K, const void *x, int xt,
                         int64_t ldx, int64_t M, void *y, int yt, int64_t ldy,
                         int32_t *acc_dbg, void *stream);

/* Most GEMVs one bitlinear_gemv_fused_multi call may carry. */
#define BITLINEAR_GEMV_MAX_PROBLEMS 8

/* Launch flag: the kernel may start while the work before it in the stream is
 * still running, and fetch its packed weights early (programmatic dependent
 * launch).  It still waits for that work to finish before it reads x or
 * writes anything, so a chain of dependent BitLinears stays correct.  The
 * caller promises that the packed weights and scales were not written by the
 * kernel immediately before this call in the stream. */
#define BL_FLAG_PDL 1u

/* Launch flags for 2 .. 16 tokens, which run either the tensor-core
 * small-batch kernel or the dp4a multi-token streaming kernel.  By default the
 * tensor cores take a batch when M * sum(N) * K >= 48 * 2^20 or K > 4096 (the
 * measured crossover; the dp4a kernel's cost grows with M * N * K, the tensor
 * cores' is nearly flat in M).  These flags force one or the other (where it
 * applies); both give identical results. */
#define BL_FLAG_SMALL_BATCH_DP4A 2u
#define BL_FLAG_SMALL_BATCH_TENSOR 4u

/*
 * Decode BitLinear for `count` weights that share the same activations x
 * (for instance the q, k and v products, or the gate and up products, of one
 * decoder layer), quantising x once and running all products in one launch.
 * Source: "How to Run BitNet Inference on GPU Using CUDA Kernels", sections
 * "Understanding the Two-Phase Architecture" (Attention and FeedForward use the
 * BitLinear kernel) and "Key Components and Source Code Architecture" (CUDA
 * graphs to remove launch overhead in decode).
 *   count            1 .. BITLINEAR_GEMV_MAX_PROBLEMS
 *   packed[i], w_scale[i], N[i]   the i-th packed weight (all share K)
 *   x, xt, ldx, M    as for bitlinear_gemv_fused (1 <= M <= 16)
 *   y[i], ldy[i]     device outputs [M][ldy[i]] of dtype yt
 *   acc_dbg          NULL, or a host array of `count` device pointers (each
 *                    NULL or [M][N[i]] int32)
 *   flags            0, or BL_FLAG_PDL and / or one of BL_FLAG_SMALL_BATCH_DP4A,
 *                    BL_FLAG_SMALL_BATCH_TENSOR
 * The pointer arrays are host memory, read during the call only.
 */
int bitlinear_gemv_fused_multi(int count, const uint8_t *const *packed,
                               const float *const *w_scale, const int64_t *N,
                               int64_t K, const void *x, int xt, int64_t ldx,
                               int64_t M, void *const *y, int yt,
                               const int64_t *ldy, int32_t *const *acc_dbg,
                               unsigned flags, void *stream);

/* Kernels of the decode / small-batch GEMV entry points (bitlinear_gemv_plan). */
#define BL_GEMV_KERNEL_STREAM 1      /* one token: producer-warp streaming kernel */
#define BL_GEMV_KERNEL_TENSOR 2      /* 2 .. 16 tokens: tensor-core small-batch kernel */
#define BL_GEMV_KERNEL_STREAM_MT 3   /* 2 .. 16 tokens: dp4a multi-token streaming kernel */
#define BL_GEMV_KERNEL_DP4A 4        /* any other shape: per-warp dp4a kernel */

/*
 * Which kernel bitlinear_gemv_fused_multi (fused = 1, activations of dtype
 * xt) or bitlinear_gemv (fused = 0, pre-quantised) runs for these shapes and
 * flags, without running it; for the tensor-core kernel also the number of
 * CTAs of a thread-block cluster that share one 128-row block's k range.
 * The choice depends on the device (its SM count and how many clusters of a
 * size it holds at once), so this needs the current device.  Where it
 * answers BL_GEMV_KERNEL_DP4A for more than 8 pre-quantised tokens,
 * bitlinear_gemv runs the tcgen05 GEMM instead.
 *   count, N, K, M   as for bitlinear_gemv_fused_multi (N: host array)
 *   kernel, cluster  host outputs: BL_GEMV_KERNEL_*, and the cluster size (0
 *                    unless the tensor-core kernel)
 * Returns BL_OK, or BL_ERR_NULL / BL_ERR_SHAPE / BL_ERR_DTYPE /
 * BL_ERR_NO_DEVICE / BL_ERR_UNSUPPORTED.
 */
int bitlinear_gemv_plan(int count, const int64_t *N, int64_t K, int64_t M, int xt,
                        int fused, unsigned flags, int *kernel, int *cluster);

/*
 * RMSNorm, then per-token absmax int8 quantisation of the normalised rows:
 * the step in front of a BitLinear in a decoder layer, in one launch.
 * Source: "bit-floor" README, section "What's inside" (rmsnorm.cu: a
 * mean-square reduction over the row, an rsqrt scale applied per element);
 * "How to Run BitNet Inference on GPU Using CUDA Kernels", section
 * "Understanding the Two-Phase Architecture" (Attention and FeedForward feed
 * their inputs to BitLinear).  Per token m (identical on the CPU oracle):
 *   S    = sum_k x[m][k]^2 in fp64;  ms = (float)(S / K)
 *   r    = 1 / sqrt(ms + eps)        fp32, correctly rounded sqrt and divide
 *   h[k] = (x[m][k] * r) * gain[k]   two fp32 products (gain NULL: x * r)
 *   q, d, rowsum of h as bitlinear_quantize_act defines them.
 * The fp64 sum runs in a different order than the oracle's; the two can
 * differ only when S / K lies within about 1e-15 (relative) of an fp32
 * rounding boundary.
 *   x, xt, M, K, ldx, q, d, rowsum   as for bitlinear_quantize_act
 *   gain    device [K] of dtype gt (BL_F32 or BL_BF16), 16-byte aligned, or
 *           NULL for no gain
 *   eps     >= 0, finite (1e-5 is this library's default reading)
 * A token's row (and the gain as fp32) is staged in shared memory: K * 2
 * (bf16) or K * 4 (fp32) bytes, plus K * 4 with a gain, must fit in 200 KiB,
 * else BL_ERR_SHAPE.
 */
int bitlinear_rmsnorm_quantize_act(const void *x, int xt, int64_t M, int64_t K,
                                   int64_t ldx, const void *gain, int gt,
                                   float eps, int8_t *q, float *d,
                                   int32_t *rowsum, void *stream);

/*
 * Decode BitLinears of one token with RMSNorm in front, in one launch: the
 * token x is normalised (as bitlinear_rmsnorm_quantize_act defines it),
 * quantised, multiplied by `count` packed weights that share it (for
 * instance gate and up, or q, k and v) and rescaled.  Sources as for
 * bitlinear_rmsnorm_quantize_act and bitlinear_gemv_fused_multi.
 *   x, xt        device [K] (one token), BL_F32 or BL_BF16
 *   gain, gt, eps  as for bitlinear_rmsnorm_quantize_act
 *   other arguments as for bitlinear_gemv_fused_multi (with M = 1)
 * Runs the streaming one-token kernel only: K a multiple of 256 up to 32768
 * and at most 64 row groups of 8 per SM, else BL_ERR_SHAPE (other shapes:
 * bitlinear_rmsnorm_quantize_act, then bitlinear_gemv).  Under BL_FLAG_PDL
 * the gain, like the packed weights and scales, must not have been written
 * by the kernel immediately before this call.
 */
int bitlinear_rmsnorm_gemv_fused_multi(int count, const uint8_t *const *packed,
                                       const float *const *w_scale,
                                       const int64_t *N, int64_t K,
                                       const void *x, int xt, const void *gain,
                                       int gt, float eps, void *const *y, int yt,
                                       const int64_t *ldy,
                                       int32_t *const *acc_dbg, unsigned flags,
                                       void *stream);

/* Activation modes of bitlinear_decode_linear. */
#define BL_ACT_PLAIN 0       /* quantise x */
#define BL_ACT_RMSNORM 1     /* RMSNorm x (gain, eps), then quantise */
#define BL_ACT_RELU2_GATE 2  /* quantise relu(x)^2 * x2 (x: gate, x2: up, bf16) */

/*
 * One token through the decode BitLinears of a decoder layer, in one launch:
 * the activation step in front (act), `count` products sharing it, the
 * rescale, and optionally the residual add.  Sources: "How to Run BitNet
 * Inference on GPU Using CUDA Kernels", section "Understanding the Two-Phase
 * Architecture" (Attention and FeedForward call BitLinear); "bit-floor"
 * README, section "What's inside" (rmsnorm.cu).  The gate's activation is a
 * reading of this library (the pages name none): squared ReLU,
 *   h[k] = (r * r) * x2[k],  r = max(x[k], 0),   two fp32 products,
 * quantised like any activation (the fp32 h, not rounded to bf16 first).
 *   act            BL_ACT_PLAIN, BL_ACT_RMSNORM or BL_ACT_RELU2_GATE
 *   x, xt          device [K] (one token); bf16 for BL_ACT_RELU2_GATE
 *   x2             BL_ACT_RELU2_GATE: device bf16 [K] (the up projection)
 *   gain, gt, eps  BL_ACT_RMSNORM: as for bitlinear_rmsnorm_quantize_act
 *   resid          NULL, or a host array of `count` pointers, each NULL or a
 *                  device bf16 [N[i]]: y[i] = bf16(resid[i] + y32) with one
 *                  fp32 addition (yt must be BL_BF16).  resid[i] may be y[i]
 *                  itself (an in-place residual stream); it must not overlap
 *                  x or x2.
 *   other arguments as for bitlinear_gemv_fused_multi (M = 1)
 * Runs the streaming one-token kernel only (K a multiple of 256 up to
 * 32768, at most 64 row groups per SM), else BL_ERR_SHAPE.  Under
 * BL_FLAG_PDL, x, x2 and resid may come from the kernel just before; the
 * weights, scales and gain may not.
 */
int bitlinear_decode_linear(int count, const uint8_t *const *packed,
                            const float *const *w_scale, const int64_t *N,
                            int64_t K, int act, const void *x, int xt,
                            const void *x2, const void *gain, int gt, float eps,
                            void *const *y, int yt, const int64_t *ldy,
                            const void *const *resid, int32_t *const *acc_dbg,
                            unsigned flags, void *stream);

/*
 * Decode attention of one token over a bf16 KV cache, with RoPE and the
 * append of this token's key and value.  Sources: "How to Run BitNet
 * Inference on GPU Using CUDA Kernels", section "Understanding the Two-Phase
 * Architecture" (Attention with a KV cache of shape (1, seq_len, kv_heads,
 * 1, head_dim)); "bit-floor" README, section "What's inside" (rope.rs,
 * attention.cu).  Readings (identical on the CPU oracle): interleaved RoPE
 * pairs (2i, 2i + 1) turned by pos * rope_base^(-2i / D) (angle, cos, sin in
 * fp64, rounded to fp32; rotation in fp32; rotated q and k rounded to bf16);
 * s_j = (float)(q . K[j]) * (float)(1 / sqrt(D)) with the dot product in
 * fp64; softmax weights e_j = exp(s_j - max s), S = sum_j e_j and out =
 * bf16((float)((sum_j e_j V[j]) / S)), all in fp64.  Query head h reads kv
 * head h / (H / Hkv).
 *   q, k, v          device bf16 [H*D], [Hkv*D], [Hkv*D] (this token)
 *   cache_k, cache_v device bf16 [Hkv][T_max][D]; position *pos of every kv
 *                    head is written, positions 0 .. *pos read
 *   pos              device int32 scalar: this token's position, read by
 *                    the kernel (a CUDA graph can replay the call for the
 *                    next token after bitlinear_position_advance)
 *   rope_table       NULL, or device (cos, sin) pairs from
 *                    bitlinear_rope_table(D, T_max, rope_base) (same values,
 *                    fewer fp64 evaluations per token)
 *   out              device bf16 [H*D]
 *   ws, ws_bytes     device workspace of at least
 *                    bitlinear_attention_workspace_bytes(H, Hkv, T_max) bytes,
 *                    16-byte aligned: per-block maxima and fp64 partial
 *                    sums, and one arrival ticket per kv head.  It
 *                    must be all zero before its first use; every call that
 *                    completes leaves the tickets zero.  Calls ordered on one
 *                    stream may share it; calls that can overlap may not.
 *   flags            0 or BL_FLAG_PDL (q, k, v may come from the kernel just
 *                    before; the cache and pos from earlier work)
 * One launch on `stream` over (kv head, block of 64 cached positions) CTAs;
 * each block's softmax is taken against its own maximum and the blocks are
 * combined with the factors exp(m_block - m), the whole softmax in fp64.
 * D must be 128; H a multiple of Hkv with H / Hkv <= 8; T_max <= 32768.  A
 * position outside [0, T_max) writes nothing and makes the next
 * bitlinear_last_device_status() return BL_ERR_SHAPE; a block whose bulk
 * copy does not land in 2 s makes it return BL_ERR_TIMEOUT, leaves `out`
 * unwritten and the workspace's ticket non-zero (zero it again).
 */
int bitlinear_attention_decode(const void *q, const void *k, const void *v,
                               void *cache_k, void *cache_v, const int32_t *pos,
                               int H, int Hkv, int D, int T_max, double rope_base,
                               const float *rope_table, void *out, void *ws,
                               size_t ws_bytes, unsigned flags, void *stream);

/*
 * RoPE's cosines and sines for every position and pair, so that
 * bitlinear_attention_decode need not evaluate them per token: table[t][i] =
 * (cos, sin) of t * rope_base^(-2i / D), each computed in fp64 and rounded to
 * fp32 -- the values the attention kernels compute without a table.
 *   table   device float [T_max][D/2][2], written; 8-byte aligned
 * D must be 128; T_max <= 32768.
 */
int bitlinear_rope_table(int D, int T_max, double rope_base, float *table,
                         void *stream);

/* Bytes of workspace bitlinear_attention_decode needs (0 if out of range). */
size_t bitlinear_attention_workspace_bytes(int H, int Hkv, int T_max);

/* *pos += 1 on the device (after a token's last attention call). */
int bitlinear_position_advance(int32_t *pos, void *stream);

/*
 * One step of a decode chain: `count` BitLinears sharing the token x (as in
 * bitlinear_gemv_fused_multi with M = 1), RMSNorm first when `norm` is set or
 * a gain is given.  All pointers are device pointers except the struct itself.
 */
typedef struct {
    int count;                                          /* 1 .. BITLINEAR_GEMV_MAX_PROBLEMS */
    const uint8_t *packed[BITLINEAR_GEMV_MAX_PROBLEMS]; /* from bitlinear_pack */
    const float *w_scale[BITLINEAR_GEMV_MAX_PROBLEMS];
    int64_t N[BITLINEAR_GEMV_MAX_PROBLEMS];
    void *y[BITLINEAR_GEMV_MAX_PROBLEMS];               /* [N[i]] of dtype yt */
    int32_t *acc_dbg[BITLINEAR_GEMV_MAX_PROBLEMS];      /* NULL or [N[i]] int32 */
    int64_t K;                                          /* a multiple of 256, <= 16384 */
    const void *x;                                      /* [K] of dtype xt */
    int xt, yt;                                         /* BL_F32 or BL_BF16 */
    int norm;                                           /* nonzero: RMSNorm x first */
    const void *gain;                                   /* NULL or [K] of dtype gt */
    int gt;
    float eps;                                          /* RMSNorm epsilon, >= 0 */
} bitlinear_chain_step;

/* Most steps one chain may hold. */
#define BITLINEAR_CHAIN_MAX_STEPS 4096

/* Bytes of device memory a plan of `nsteps` steps needs (0 if out of range). */
size_t bitlinear_chain_plan_bytes(int nsteps);

/*
 * Prepare a decode chain: the steps of one token, each reading the output of
 * an earlier step (or the token's input), to be run as ONE persistent launch
 * by bitlinear_chain_run.  Source: "How to Run BitNet Inference on GPU Using
 * CUDA Kernels", sections "Understanding the Two-Phase Architecture" (the
 * decode phase chains memory-bound INT8 x INT2 linears through Attention and
 * FeedForward) and "Key Components and Source Code Architecture" (CUDA graphs
 * to remove launch overhead).  Every step computes exactly what
 * bitlinear_gemv_fused_multi (or, with norm, bitlinear_rmsnorm_gemv_fused_multi)
 * computes on the same arguments.
 *   steps     host array of nsteps descriptors, read during the call only
 *   plan      device buffer of at least bitlinear_chain_plan_bytes(nsteps),
 *             16-byte aligned, owned by the caller; written here (a copy
 *             from host memory on `stream`), read and updated by every run
 * A step's outputs must not overlap its own input x.  Make the plan outside
 * stream capture; runs may be captured.  Errors: BL_ERR_SHAPE for a K that
 * is not a multiple of 256 or above 16384, more than 64 row groups of 8 per
 * SM in one step, or nsteps out of range; the usual checks otherwise.
 */
int bitlinear_chain_plan(int nsteps, const bitlinear_chain_step *steps,
                         void *plan, size_t plan_bytes, void *stream);

/*
 * Run a prepared chain: one cooperative launch (one CTA per SM, all resident)
 * after a reset of the plan's step counters, both on `stream`.  Each CTA owns
 * a slice of every step's rows; its producer warp streams the weights of all
 * steps ahead through shared memory, and its consumers start step s once all
 * CTAs have finished step s - 1.  Every wait is bounded (2 s): a timeout is
 * reported by the next bitlinear_last_device_status() as BL_ERR_TIMEOUT and
 * leaves the outputs of the unfinished steps unspecified.  Runs of one plan
 * must be ordered (one stream); the buffers the plan names must stay alive.
 * On B200 a step of the 2.4B decode stream takes 4-6.5 us this way, against
 * ~3.1 us as separate bitlinear_gemv_fused_multi launches with BL_FLAG_PDL
 * in a CUDA graph: use the chain where one launch per token matters more
 * than per-step latency.
 *   plan, nsteps   as given to bitlinear_chain_plan
 */
int bitlinear_chain_run(const void *plan, int nsteps, void *stream);

/*
 * For testing failure handling without a GPU fault: runs the chain with its
 * bounded waits limited to wait_limit_ns (1 us .. 2 s) and with the wait
 * before step 1 expecting one more arrival than there are CTAs, a count
 * nothing reaches.  That wait runs out, the grid leaves through its abort
 * path, and the next bitlinear_last_device_status() returns BL_ERR_TIMEOUT;
 * the device stays usable.  Step 0's outputs are complete, later outputs
 * unspecified.  nsteps >= 2.
 */
int bitlinear_chain_run_timeout_test(const void *plan, int nsteps,
                                     uint64_t wait_limit_ns, void *stream);

/*
 * Bytes of workspace bitlinear_gemm needs for this problem (0 if none).
 * Nonzero for small batches (M <= 32) whose output tiles alone would leave
 * SMs idle: K is then split across CTAs and the int32 partial sums meet in
 * the workspace.
 */
size_t bitlinear_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K);

/*
 * Ternary GEMM for any M >= 1 (prefill), on the tcgen05 int8 tensor cores
 * with int32 accumulators in tensor memory.  Source: "How to Run BitNet
 * Inference on GPU Using CUDA Kernels", FAQ (a generic INT8 x INT2 GEMM);
 * "BitCompute", section "Future Roadmap" (tensor-core execution of the
 * ternary product).  Arguments as for bitlinear_gemv, plus
 *   ws, ws_bytes   device workspace, at least bitlinear_gemm_workspace_bytes
 *                  (may be NULL when that is 0).  It must be all zero before
 *                  its first use, and every call that completes leaves it
 *                  zero; it may be reused by calls that are ordered on one
 *                  stream, not shared by calls that can run at the same time.
 *                  A call whose bounded wait ran out (the next
 *                  bitlinear_last_device_status() returns BL_ERR_TIMEOUT) may
 *                  leave partial sums and arrival counts in it: zero it again
 *                  before the next call that uses it.
 * q must be 16-byte aligned and K % 64 == 0.
 */
int bitlinear_gemm(const uint8_t *packed, const float *w_scale, int64_t N,
                   int64_t K, const int8_t *q, const float *d,
                   const int32_t *rowsum, int64_t M, void *y, int yt,
                   int64_t ldy, int32_t *acc_dbg, void *ws, size_t ws_bytes,
                   void *stream);

/* Bytes of the binary packed array: N * (K/64) * 8. */
size_t bitlinear_binary_packed_bytes(int64_t N, int64_t K);

/*
 * Binary (1-bit) weight packer: sign bits and the absmax scale.  Source:
 * "bit-floor" README, section "What's inside" (binary packing, absmax scale).
 *   W     device [N][K] of dtype wt
 *   Wb    device uint64 [N][K/64], written
 *   s_w   device, 1 float, written with max |W|
 */
int bitlinear_binary_pack(const void *W, int wt, int64_t N, int64_t K,
                          uint64_t *Wb, float *s_w, void *stream);

/*
 * Binary GEMV of one token: acc[n] = 2 * popcount(XNOR(Wb[n], xb)) - K,
 * y[n] = (float)acc[n] * (s_w * s_x), s_x = max |x|, xb the sign bits of x.
 * Source: "bit-floor" README, section "The core math".
 *   x        device [K] of dtype xt
 *   y        device [N] of dtype yt
 *   acc_dbg  NULL or device [N] int32
 */
int bitlinear_binary_gemv(const uint64_t *Wb, const float *s_w, int64_t N,
                          int64_t K, const void *x, int xt, void *y, int yt,
                          int32_t *acc_dbg, void *stream);

/*
 * Ternary GEMV of one token by table lookup (the lookup-table method of the
 * TL1 / TL2 CPU kernels: "Run 100B Models on Your Laptop CPU: Microsoft
 * BitNet Exposed", section "Key Features That Make BitNet Insane", T-MAC's
 * lookup tables), on the TL packed weights.  For each pair of activations
 * (k, k + 4) that one 4-bit field of a TL byte covers, a 16-entry table of
 * (s_a - 1) q[k] + (s_b - 1) q[k + 4] is built in shared memory and indexed
 * by the field; acc is the same exact integer as bitlinear_gemv's, and
 * y = ((float)acc * d) * gamma_eff.  Offered for comparison with the dp4a
 * GEMV (same inputs, same results).
 *   packed, w_scale   from bitlinear_pack (device)
 *   q, d              device, one token from bitlinear_quantize_act (q [K])
 *   y                 device [N] of dtype yt;  acc_dbg NULL or device [N]
 * K <= 12288 (the tables take 16.5 bytes of shared memory per k).
 */
int bitlinear_lut_gemv(const uint8_t *packed, const float *w_scale, int64_t N,
                       int64_t K, const int8_t *q, const float *d, void *y,
                       int yt, int32_t *acc_dbg, void *stream);

/* Bytes of the bit-plane array: N * (K/64) * 16 (a mag and a sign word per
 * 64 k of each row). */
size_t bitlinear_bitplane_bytes(int64_t N, int64_t K);

/*
 * Ternary weights as two bit-planes, from the TL packed array: for every row
 * n and 64-k word w, the pair (mag, sign) at uint64 index 2 (n (K/64) + w)
 * and 2 (n (K/64) + w) + 1, bit j <-> k = 64 w + j; mag set for a non-zero
 * weight, sign set for a negative one.  Source: "bit-floor" README, sections
 * "The core math" (ternary GEMV on two bit-planes) and "What's inside"
 * (ternary weights packed as two bit-plane u64 word arrays).  The planes
 * keep the weight scale of the packed weight (its w_scale).
 *   packed   device, from bitlinear_pack (N, K)
 *   planes   device, bitlinear_bitplane_bytes(N, K) bytes, written
 * K <= 65536.
 */
int bitlinear_bitplane_pack(const uint8_t *packed, int64_t N, int64_t K,
                            uint64_t *planes, void *stream);

/*
 * Ternary-weight x 1-bit-activation GEMV of one token on the bit-planes:
 *   acc[n] = POPCNT(mag & XNOR(sign, xb)) - POPCNT(mag & XOR(sign, xb))
 *          = sum_k code[n][k] * (x[k] < 0 ? -1 : +1)
 *   y[n]   = (float)acc[n] * (w_scale * s_x),  s_x = max |x|
 * with xb the sign bits of x (set for negative values, -0.0 counts as
 * positive).  Source: "bit-floor" README, section "The core math" (ternary
 * GEMV, "no floating point in the inner loop").
 *   planes   device, from bitlinear_bitplane_pack
 *   w_scale  device, 1 float: gamma_eff of the packed weight
 *   x        device [K] of dtype xt;  y device [N] of dtype yt
 *   acc_dbg  NULL or device [N] int32
 * K <= 65536.
 */
int bitlinear_bitplane_gemv(const uint64_t *planes, const float *w_scale,
                            int64_t N, int64_t K, const void *x, int xt,
                            void *y, int yt, int32_t *acc_dbg, void *stream);

/*
 * Measurement aid: the int8 tensor-core rate the prefill GEMM can draw on.
 * `grid` CTAs (at most one per SM) each issue `reps` stages of eight
 * back-to-back tcgen05.mma.kind::i8 of the GEMM's form (128 x 128 x 32: A =
 * unsigned codes in tensor memory, B = signed activations in 128-byte-swizzled
 * shared memory, int32 accumulators), with no operand traffic, and time them.
 *   out   device int64 [2 * grid]: per CTA, clock cycles and nanoseconds
 *         (-1 if the final wait ran out; BL_ERR_TIMEOUT in the status word)
 * MACs per CTA = reps * 8 * 128 * 128 * 32; reps <= 131072.  Asynchronous on
 * `stream`.
 */
int bitlinear_probe_mma_i8(int reps, long long *out, int grid, void *stream);

/*
 * Measurement aid: how the issue rate of narrow MMAs depends on the number of
 * issuing threads.  As bitlinear_probe_mma_i8, with MMAs of 128 x n x 32 (n =
 * 32 or 128) issued by `issuers` warps of each CTA at once (1, 2 or 4 for n =
 * 32; 1 or 2 for n = 128), each into its own accumulator columns.
 *   out   device int64 [2 * issuers * grid]: per CTA and issuer, clock cycles
 *         and nanoseconds (-1 if its final wait ran out)
 * MACs per issuer = reps * 8 * 128 * n * 32; reps <= 131072.
 */
int bitlinear_probe_mma_i8_issue(int n, int issuers, int reps, long long *out, int grid,
                                 void *stream);

/*
 * Synchronises `stream`, then reads and clears the device status word of the
 * current device: BL_OK, BL_ERR_TIMEOUT if a kernel's bounded wait ran out,
 * or BL_ERR_SHAPE if a kernel found a device-side argument out of range (a
 * position outside the KV cache), since the last call.  BL_ERR_CUDA if the
 * synchronisation failed.
 */
int bitlinear_last_device_status(void *stream);

/* Number of SMs of the current device (0 on error); for callers sizing work. */
int bitlinear_device_sm_count(void);

#ifdef __cplusplus
}
#endif

#endif /* BITLINEAR_H */
