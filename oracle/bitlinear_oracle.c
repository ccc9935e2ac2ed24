/*
 * bitlinear_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, CPU statement of the BitNet b1.58 BitLinear product, used to
 * check the CUDA library.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load it; the product path never does.  It
 * shares no code, header, table or constant generator with the CUDA sources.
 *
 * Sources (web pages, cited by title and section):
 *   [GUIDE]  "How to Run BitNet Inference on GPU Using CUDA Kernels: A Complete
 *            Guide", section "Understanding the Two-Phase Architecture"
 *            (BitLinearKernel quantises inputs to INT8 with scaling factors and
 *            calls an INT8 x INT2 linear) and FAQ "Can I use the CUDA kernel for
 *            models other than the default BitNet architecture?" (generic
 *            INT8xINT2 GEMM).
 *   [FLOOR]  "bit-floor" README, section "The core math" (binary GEMV as
 *            XNOR/popcount, "no floating point until the final scale multiply")
 *            and section "What's inside" (absmax scale for binary weights,
 *            mean-abs scale for ternary weights).
 *   [BITC]   "BitCompute: 1.58-bit LLM Execution Engine", sections "Features"
 *            (multiplying by -1, 0, +1 is add / subtract / skip) and "Future
 *            Roadmap" (four 1.58-bit weights packed into one byte).
 *   [BLOG]   "Run 100B Models on Your Laptop CPU: Microsoft BitNet Exposed",
 *            section "What is Microsoft BitNet?" (ternary {-1, 0, +1} weights).
 *
 * The pages give no formula for the scales; the readings used here are:
 *   weight scale    gamma = mean |W| over the whole tensor, summed in fp64 in a
 *                   fixed order (row by row, k ascending inside a row, rows in
 *                   ascending order), rounded once to fp32, then
 *                   gamma_eff = max(gamma, 1e-5).
 *   ternary code    code = clamp(rint(w / gamma_eff), -1, 1), fp32 division,
 *                   round half to even.
 *   activation      per token: a = max(max_k |x|, 1e-5); s = 127 / a (fp32);
 *                   q = clamp(rint(x * s), -128, 127) (fp32 product, round half
 *                   to even); d = a / 127 (fp32); r = sum_k q.
 *   product         acc[m][n] = sum_k code[n][k] * q[m][k], exact integer.
 *   rescale         y = ((float)acc * d[m]) * gamma_eff: two fp32 products in
 *                   that order, no fused multiply-add; bf16 output rounds y to
 *                   nearest even.
 *   binary          bit = (v < 0); acc = 2 * popcount(XNOR(Wb, xb)) - K;
 *                   y = (float)acc * (s_w * s_x) with s_w = max |W| over the
 *                   tensor and s_x = max |x| over the token.
 * Floating-point decisions that produce integers (codes, q) are taken in fp32,
 * the precision the kernels use, so that both sides decide identically.
 *
 * Build: gcc -O2 -ffp-contract=off -fno-fast-math -fopenmp -shared -fPIC.
 * Parity of the fp64 weight-scale sum is exact by construction because the
 * order of additions is part of the definition above.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <math.h>

#define ORACLE_EPS 1e-5f
#define ORACLE_QB 127.0f

/* ---------------------------------------------------------------------------
 * Weight scale (absmean).  [FLOOR] "What's inside": mean-abs scale for ternary
 * weights; [BLOG] "What is Microsoft BitNet?": ternary weights.
 * ------------------------------------------------------------------------- */
float oracle_weight_scale(const float *W, int64_t N, int64_t K)
{
    double S = 0.0;
    for (int64_t n = 0; n < N; ++n) {
        double row = 0.0;
        for (int64_t k = 0; k < K; ++k)
            row += fabs((double)W[n * K + k]);
        S += row;
    }
    float gamma = (float)(S / (double)(N * K));
    return gamma > ORACLE_EPS ? gamma : ORACLE_EPS;
}

/* Ternary round-clip: code = clamp(rint(w / gamma_eff), -1, 1). */
void oracle_ternary_codes(const float *W, int64_t N, int64_t K, float gamma_eff,
                          int8_t *codes)
{
    for (int64_t i = 0; i < N * K; ++i) {
        float r = W[i] / gamma_eff;
        float t = rintf(r);
        int8_t c = 0;
        if (t >= 1.0f)
            c = 1;
        else if (t <= -1.0f)
            c = -1;
        codes[i] = c;
    }
}

/* ---------------------------------------------------------------------------
 * Packed layout "TL" (the pages fix none: [BITC] "Future Roadmap" packs four
 * weights per byte; [GUIDE] names an INT2 layout without describing it).
 *
 *   stored value  s = code + 1 in {0, 1, 2}; 3 is never written
 *   rows          padded up to a multiple of 8 with code 0 (s = 1)
 *   K             a multiple of 64
 *   byte offset   of (n, k):  ((g * (K/64) + c) * 8 + r) * 16 + w * 4 + j
 *                 with g = n/8, r = n%8, c = k/64, w = (k%64)/16, j = k%4
 *   bit offset    2 * i with i = (k%16)/4
 * So a 16-byte chunk holds 64 consecutive k of one row, and the eight rows of
 * a row group are adjacent for each chunk.
 * ------------------------------------------------------------------------- */
int64_t oracle_packed_bytes(int64_t N, int64_t K)
{
    int64_t Np = (N + 7) / 8 * 8;
    return Np * (K / 4);
}

static int64_t tl_byte(int64_t n, int64_t k, int64_t K)
{
    int64_t g = n / 8, r = n % 8, c = k / 64;
    int64_t w = (k % 64) / 16, j = k % 4;
    return ((g * (K / 64) + c) * 8 + r) * 16 + w * 4 + j;
}

static int tl_shift(int64_t k)
{
    return (int)(2 * ((k % 16) / 4));
}

void oracle_pack(const int8_t *codes, int64_t N, int64_t K, uint8_t *packed)
{
    int64_t Np = (N + 7) / 8 * 8;
    memset(packed, 0, (size_t)oracle_packed_bytes(N, K));
    for (int64_t n = 0; n < Np; ++n)
        for (int64_t k = 0; k < K; ++k) {
            int code = n < N ? codes[n * K + k] : 0;
            unsigned s = (unsigned)(code + 1);
            packed[tl_byte(n, k, K)] |= (uint8_t)(s << tl_shift(k));
        }
}

void oracle_unpack(const uint8_t *packed, int64_t N, int64_t K, int8_t *codes)
{
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) {
            unsigned s = (packed[tl_byte(n, k, K)] >> tl_shift(k)) & 3u;
            codes[n * K + k] = (int8_t)((int)s - 1);
        }
}

/* ---------------------------------------------------------------------------
 * Per-token absmax int8 activation quantisation.  [GUIDE] "Understanding the
 * Two-Phase Architecture": inputs quantised to INT8 with scaling factors.  The
 * page says "per-batch"; the reading here is per token (identical at M = 1).
 * ------------------------------------------------------------------------- */
void oracle_quantize_act(const float *x, int64_t M, int64_t K, int8_t *q,
                         float *d, int32_t *rowsum)
{
    for (int64_t m = 0; m < M; ++m) {
        const float *xm = x + m * K;
        float amax = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            float a = fabsf(xm[k]);
            if (a > amax)
                amax = a;
        }
        float a_eff = amax > ORACLE_EPS ? amax : ORACLE_EPS;
        float s = ORACLE_QB / a_eff;
        int32_t r = 0;
        for (int64_t k = 0; k < K; ++k) {
            float v = xm[k] * s;
            float t = rintf(v);
            if (t > 127.0f)
                t = 127.0f;
            if (t < -128.0f)
                t = -128.0f;
            int8_t qi = (int8_t)t;
            q[m * K + k] = qi;
            r += qi;
        }
        d[m] = a_eff / ORACLE_QB;
        rowsum[m] = r;
    }
}

/* ---------------------------------------------------------------------------
 * RMSNorm in front of the activation quantiser.  [FLOOR] "What's inside"
 * (rmsnorm.cu: a mean-square reduction over the row, an rsqrt scale applied
 * element by element) and [GUIDE] "Understanding the Two-Phase Architecture"
 * (the Attention and FeedForward layers feed their inputs to BitLinear).
 * The pages give no formula; the reading here, per token m:
 *   S     = sum_k (double)x[k] * (double)x[k]     fp64, k ascending
 *   ms    = (float)(S / (double)K)                rounded once to fp32
 *   r     = 1.0f / sqrtf(ms + eps)                fp32 add, correctly rounded
 *                                                 square root and division
 *   h[k]  = (x[k] * r) * g[k]                     two fp32 products, in that
 *                                                 order (g = 1 without a gain)
 * h stays fp32 and goes straight to oracle_quantize_act.
 * ------------------------------------------------------------------------- */
void oracle_rmsnorm(const float *x, int64_t M, int64_t K, const float *gain,
                    float eps, float *h)
{
    for (int64_t m = 0; m < M; ++m) {
        const float *xm = x + m * K;
        double S = 0.0;
        for (int64_t k = 0; k < K; ++k)
            S += (double)xm[k] * (double)xm[k];
        float ms = (float)(S / (double)K);
        float den = sqrtf(ms + eps);
        float r = 1.0f / den;
        for (int64_t k = 0; k < K; ++k) {
            float t = xm[k] * r;
            h[m * K + k] = gain ? t * gain[k] : t;
        }
    }
}

/* ---------------------------------------------------------------------------
 * Ternary product with exact integer accumulation.  [BITC] "Features": a
 * product with -1 / 0 / +1 is subtract / skip / add.  [GUIDE] FAQ: an
 * INT8 x INT2 GEMM.  Accumulated in int64 and narrowed (|acc| <= 128 * K).
 * ------------------------------------------------------------------------- */
void oracle_ternary_acc(const int8_t *codes, const int8_t *q, int64_t M,
                        int64_t N, int64_t K, int32_t *acc)
{
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        const int8_t *wn = codes + n * K;
        for (int64_t m = 0; m < M; ++m) {
            const int8_t *qm = q + m * K;
            int64_t s = 0;
            for (int64_t k = 0; k < K; ++k) {
                if (wn[k] == 1)
                    s += qm[k];
                else if (wn[k] == -1)
                    s -= qm[k];
            }
            acc[m * N + n] = (int32_t)s;
        }
    }
}

/* Rescale: y = ((float)acc * d[m]) * gamma_eff.  [FLOOR] "The core math": no
 * floating point until the final scale multiply. */
void oracle_rescale(const int32_t *acc, const float *d, float gamma_eff,
                    int64_t M, int64_t N, float *y)
{
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            float a = (float)acc[m * N + n];
            float t = a * d[m];
            y[m * N + n] = t * gamma_eff;
        }
}

/* fp32 -> bf16, round to nearest even; NaN stays NaN. */
void oracle_to_bf16(const float *y, int64_t n, uint16_t *out)
{
    for (int64_t i = 0; i < n; ++i) {
        uint32_t u;
        memcpy(&u, &y[i], 4);
        if ((u & 0x7fffffffu) > 0x7f800000u) {
            out[i] = (uint16_t)((u >> 16) | 0x40u);
        } else {
            uint32_t lsb = (u >> 16) & 1u;
            u += 0x7fffu + lsb;
            out[i] = (uint16_t)(u >> 16);
        }
    }
}

/* ---------------------------------------------------------------------------
 * Binary 1-bit variant.  [FLOOR] "The core math": rows packed into ceil(K/64)
 * 64-bit words, y = scale_w * scale_x * (2 * POPCNT(XNOR(W, x)) - K);
 * [FLOOR] "What's inside": absmax scale for binary weights.
 * Bit j of word w holds k = 64 w + j; the bit is 1 when the value is negative.
 * Pad bits (K not a multiple of 64) are 0 in W and 1 in x, so XNOR is 0 there.
 * ------------------------------------------------------------------------- */
float oracle_absmax(const float *v, int64_t n)
{
    float a = 0.0f;
    for (int64_t i = 0; i < n; ++i) {
        float t = fabsf(v[i]);
        if (t > a)
            a = t;
    }
    return a;
}

void oracle_binary_signs(const float *v, int64_t R, int64_t K, int pad_bit,
                         uint64_t *out)
{
    int64_t words = (K + 63) / 64;
    for (int64_t r = 0; r < R; ++r)
        for (int64_t w = 0; w < words; ++w) {
            uint64_t word = 0;
            for (int64_t j = 0; j < 64; ++j) {
                int64_t k = 64 * w + j;
                uint64_t bit;
                if (k < K)
                    bit = v[r * K + k] < 0.0f ? 1u : 0u;
                else
                    bit = (uint64_t)pad_bit;
                word |= bit << j;
            }
            out[r * words + w] = word;
        }
}

static int64_t popcount64_plain(uint64_t v)
{
    int64_t c = 0;
    while (v) {
        c += (int64_t)(v & 1u);
        v >>= 1;
    }
    return c;
}

void oracle_binary_acc(const uint64_t *Wb, const uint64_t *xb, int64_t N,
                       int64_t K, int32_t *acc)
{
    int64_t words = (K + 63) / 64;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        int64_t pc = 0;
        for (int64_t w = 0; w < words; ++w)
            pc += popcount64_plain(~(Wb[n * words + w] ^ xb[w]));
        acc[n] = (int32_t)(2 * pc - K);
    }
}

void oracle_binary_rescale(const int32_t *acc, float s_w, float s_x, int64_t N,
                           float *y)
{
    float s = s_w * s_x;
    for (int64_t n = 0; n < N; ++n)
        y[n] = (float)acc[n] * s;
}

/* ---------------------------------------------------------------------------
 * Ternary weights x 1-bit activations on two bit-planes.  [FLOOR] "The core
 * math": a ternary row is two bit-planes, mag (bit set: the weight is
 * non-zero) and sign (bit set: the weight is negative), and
 *   dot = POPCNT(mag & XNOR(sign, x)) - POPCNT(mag & XOR(sign, x)),
 * with x the activation's sign bits; [FLOOR] "What's inside": ternary
 * weights as two bit-plane u64 word arrays.  Readings: the planes come from
 * the same absmean codes as the 2-bit path; bit j of word w holds k = 64 w + j;
 * the activation bit is set for negative values (as in the binary variant, so
 * XNOR marks a positive product); y = (float)dot * (gamma_eff * s_x) with
 * s_x = max |x| (the binary variant's activation scale).  Pad bits (K not a
 * multiple of 64) are 0 in mag, so they never count.
 * ------------------------------------------------------------------------- */
void oracle_bitplanes(const int8_t *codes, int64_t N, int64_t K, uint64_t *mag,
                      uint64_t *sign)
{
    int64_t words = (K + 63) / 64;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t w = 0; w < words; ++w) {
            uint64_t m = 0, s = 0;
            for (int64_t j = 0; j < 64; ++j) {
                int64_t k = 64 * w + j;
                if (k >= K)
                    continue;
                int c = codes[n * K + k];
                if (c != 0)
                    m |= (uint64_t)1 << j;
                if (c < 0)
                    s |= (uint64_t)1 << j;
            }
            mag[n * words + w] = m;
            sign[n * words + w] = s;
        }
}

void oracle_bitplane_acc(const uint64_t *mag, const uint64_t *sign,
                         const uint64_t *xb, int64_t N, int64_t K, int32_t *acc)
{
    int64_t words = (K + 63) / 64;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        int64_t dot = 0;
        for (int64_t w = 0; w < words; ++w) {
            uint64_t m = mag[n * words + w], s = sign[n * words + w];
            dot += popcount64_plain(m & ~(s ^ xb[w]));
            dot -= popcount64_plain(m & (s ^ xb[w]));
        }
        acc[n] = (int32_t)dot;
    }
}

/* ---------------------------------------------------------------------------
 * The rest of a decoder layer around the BitLinears, for the synthetic layer
 * stack.  [GUIDE] "Understanding the Two-Phase Architecture" (Attention and
 * FeedForward call BitLinear; a KV cache of shape (1, seq_len, kv_heads, 1,
 * head_dim)); [FLOOR] "What's inside" (rope.rs: RoPE applied to queries and
 * keys before attention; attention.cu: attention with a softmax over the
 * cached positions).  The pages fix no formula; the readings:
 *   RoPE       pairs (2i, 2i + 1) of each head rotated by the angle
 *              pos * base^(-2i / D) (fp64, then cos and sin rounded to fp32);
 *              out = (a c - b s, a s + b c), each product and the sum or
 *              difference an fp32 operation in that order.
 *   attention  per query head h (kv head h / (H / Hkv)) over positions
 *              j = 0 .. T - 1: s_j = (float)(sum_d q[d] K[j][d]) * scale with
 *              the dot product in fp64 and scale = (float)(1 / sqrt(D));
 *              m = max s_j; the softmax weights e_j = exp(s_j - m), their sum
 *              S and out[d] = (float)((sum_j e_j V[j][d]) / S) all in fp64
 *              (the weights are not rounded to fp32: any fp64 grouping of the
 *              sums, and any factoring of the exponentials, then agrees to
 *              about 1e-15, far inside one fp32 rounding).
 *   FFN gate   m = (r * r) * u with r = max(g, 0) (squared ReLU gating), fp32.
 * ------------------------------------------------------------------------- */
void oracle_rope(const float *x, int64_t heads, int64_t D, int64_t pos, double base,
                 float *out)
{
    for (int64_t h = 0; h < heads; ++h)
        for (int64_t i = 0; i < D / 2; ++i) {
            double ang = (double)pos * pow(base, -(double)(2 * i) / (double)D);
            float c = (float)cos(ang), s = (float)sin(ang);
            float a = x[h * D + 2 * i], b = x[h * D + 2 * i + 1];
            float ac = a * c, bs = b * s, as = a * s, bc = b * c;
            out[h * D + 2 * i] = ac - bs;
            out[h * D + 2 * i + 1] = as + bc;
        }
}

/* K, V: [Hkv][T_stride][D]; positions 0 .. T - 1 are used. */
void oracle_attention_decode(const float *q, const float *K, const float *V, int64_t H,
                             int64_t Hkv, int64_t D, int64_t T, int64_t T_stride,
                             float *out)
{
    float scale = (float)(1.0 / sqrt((double)D));
    float *sc = (float *)malloc((size_t)T * sizeof(float));
    double *e = (double *)malloc((size_t)T * sizeof(double));
    for (int64_t h = 0; h < H; ++h) {
        int64_t kv = h / (H / Hkv);
        const float *qh = q + h * D;
        const float *Kh = K + kv * T_stride * D;
        const float *Vh = V + kv * T_stride * D;
        float m = -INFINITY;
        for (int64_t j = 0; j < T; ++j) {
            double dot = 0.0;
            for (int64_t d = 0; d < D; ++d)
                dot += (double)qh[d] * (double)Kh[j * D + d];
            sc[j] = (float)dot * scale;
            if (sc[j] > m)
                m = sc[j];
        }
        double S = 0.0;
        for (int64_t j = 0; j < T; ++j) {
            e[j] = exp((double)sc[j] - (double)m);
            S += e[j];
        }
        for (int64_t d = 0; d < D; ++d) {
            double num = 0.0;
            for (int64_t j = 0; j < T; ++j)
                num += e[j] * (double)Vh[j * D + d];
            out[h * D + d] = (float)(num / S);
        }
    }
    free(sc);
    free(e);
}

void oracle_relu2_gate(const float *g, const float *u, int64_t n, float *out)
{
    for (int64_t i = 0; i < n; ++i) {
        float r = g[i] > 0.0f ? g[i] : 0.0f;
        float rr = r * r;
        out[i] = rr * u[i];
    }
}

/* Residual add: out = h + y, one fp32 addition (h a bf16 value as fp32). */
void oracle_residual_add(const float *h, const float *y, int64_t n, float *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = h[i] + y[i];
}

/* Threads the OpenMP loops above use (1 when built without OpenMP). */
#ifdef _OPENMP
#include <omp.h>
#endif
int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Sets the thread count of those loops (no effect without OpenMP). */
void oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0)
        omp_set_num_threads(n);
#else
    (void)n;
#endif
}
