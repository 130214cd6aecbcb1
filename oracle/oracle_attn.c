/*
 * fp64 CPU oracle for full (non-causal) multi-head joint self-attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file: only the tests, the smoke check and the CPU-baseline leg of
 * the bench use it.  It shares no code, header or constant with the CUDA path.
 *
 * What it computes (one DiT block's attention core).  The pages describe the
 * DiT denoiser whose repeated transformer passes dominate inference time
 * ("How to Scale Diffusion Inference Across AMD RDNA 4 GPUs", section
 * "Understanding the Inference Pipeline") and the attention backend those
 * passes call (same page, "Select an Attention Backend and Compile the
 * Transformer"); they cite "Attention Is All You Need" and FlashAttention-2
 * for the operation ("xDiT: an Inference Engine for Diffusion Transformers
 * (DiTs) with Massive Parallelism", reference list).  The pages never print
 * the formula, so this file writes out the textbook definition of scaled
 * dot-product attention, with no mask and no dropout:
 *
 *   s_j   = scale * sum_d q_d k_{j,d}                 j = 0..L-1
 *   m     = max_j s_j
 *   p_j   = exp(s_j - m)
 *   l     = sum_j p_j                                 (left to right)
 *   o_d   = (sum_j p_j v_{j,d}) / l
 *   lse   = m + log(l)                                (natural log)
 *
 * It is deliberately two-pass (max first, no running rescale, no tiling), so
 * it is not the GPU algorithm.  Inputs are decoded exactly to fp64:
 *   - bf16: the upper 16 bits of an IEEE-754 binary32 (shift, reinterpret);
 *   - FP8 E4M3 (OCP 8-bit floating point, "fn" variant: no infinities,
 *     S.1111.111 is NaN, exponent bias 7, subnormals at exponent field 0),
 *     multiplied by a per-(batch, head) fp32 dequantisation scale
 *     (x = s * decode(x_hat)); the FP8 attention backend is named on the
 *     pages (fosswire.org summary, "Technical implementation of xDiT on
 *     RDNA 4"; RDNA 4 guide, "Select an Attention Backend ...");
 *   - fp64: used as is (pins and closed-form tests).
 *
 * Built with plain gcc, without -ffast-math; exp/log are libm's.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORACLE_BF16 = 0, ORACLE_E4M3 = 1, ORACLE_F64 = 2 };

/* bf16 -> fp64: bf16 is the high half of a binary32, so place the 16 bits at
 * the top of a 32-bit word and read it as a float; the float widens exactly. */
double oracle_bf16_to_f64(uint16_t bits)
{
    uint32_t w = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &w, sizeof f);
    return (double)f;
}

/* OCP FP8 E4M3 -> fp64, written from the format's definition:
 *   field E = bits 6..3, field M = bits 2..0, sign = bit 7
 *   E = 15 and M = 7  -> NaN (the only non-finite code; no infinities)
 *   E = 0             -> subnormal  (-1)^S * 2^(1-7) * (M / 8)
 *   otherwise         -> normal     (-1)^S * 2^(E-7) * (1 + M / 8)      */
double oracle_e4m3_to_f64(uint8_t code)
{
    int sign = (code >> 7) & 1;
    int e = (code >> 3) & 0xF;
    int m = code & 0x7;
    double mag;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        mag = ldexp((double)m / 8.0, 1 - 7);
    else
        mag = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -mag : mag;
}

void oracle_decode_bf16(const uint16_t *in, double *out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = oracle_bf16_to_f64(in[i]);
}

void oracle_decode_e4m3(const uint8_t *in, double *out, int64_t n, double scale)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = oracle_e4m3_to_f64(in[i]) * scale;
}

/* Decode one [L, D] slice (the (b,h) head) of an input to fp64. */
static void decode_slice(int dtype, const void *base, const float *scales, int64_t bh,
                         int64_t n, double *out)
{
    int64_t off = bh * n;
    if (dtype == ORACLE_BF16) {
        oracle_decode_bf16((const uint16_t *)base + off, out, n);
    } else if (dtype == ORACLE_E4M3) {
        oracle_decode_e4m3((const uint8_t *)base + off, out, n, (double)scales[bh]);
    } else {
        memcpy(out, (const double *)base + off, (size_t)n * sizeof(double));
    }
}

/* One query row against all L keys of its head: the definition above. */
static void attend_row(const double *qrow, const double *kh, const double *vh, int L, int D,
                       double scale, double *s, double *orow, double *lse_out)
{
    double m = -INFINITY, l = 0.0;
    for (int j = 0; j < L; ++j) {
        const double *kj = kh + (int64_t)j * D;
        double dot = 0.0;
        for (int d = 0; d < D; ++d)
            dot += qrow[d] * kj[d];
        s[j] = scale * dot;
        if (s[j] > m)
            m = s[j];
    }
    for (int j = 0; j < L; ++j) {
        s[j] = exp(s[j] - m);          /* p_j */
        l += s[j];
    }
    for (int d = 0; d < D; ++d)
        orow[d] = 0.0;
    for (int j = 0; j < L; ++j) {
        const double *vj = vh + (int64_t)j * D;
        for (int d = 0; d < D; ++d)
            orow[d] += s[j] * vj[d];
    }
    for (int d = 0; d < D; ++d)
        orow[d] /= l;
    if (lse_out)
        *lse_out = m + log(l);
}

/*
 * oracle_attention — fp64 attention over [B, H, L, D] inputs.
 *
 *   dtype      ORACLE_BF16 (uint16 bit patterns), ORACLE_E4M3 (uint8 codes,
 *              with q/k/v_scale [B*H] fp32 dequant scales) or ORACLE_F64.
 *   q, k, v    contiguous [B, H, L, D], D innermost.
 *   scale      softmax scale applied to q.k (the configs use 1/sqrt(D)).
 *   rows       NULL: every query row, nrows must equal L.  Otherwise
 *              [B*H][nrows] query indices, each in [0, L).
 *   o          out: [B*H][nrows][D] fp64.
 *   lse        out: [B*H][nrows] fp64, may be NULL.
 *   nthreads   OpenMP threads (<= 0: the runtime default).
 * Returns 0, or a negative value for bad arguments / out of memory.
 */
int oracle_attention(int dtype, const void *q, const void *k, const void *v,
                     const float *q_scale, const float *k_scale, const float *v_scale,
                     int B, int H, int L, int D, double scale,
                     const int64_t *rows, int nrows, double *o, double *lse, int nthreads)
{
    if (B < 1 || H < 1 || L < 1 || D < 1 || !q || !k || !v || !o)
        return -1;
    if (dtype != ORACLE_BF16 && dtype != ORACLE_E4M3 && dtype != ORACLE_F64)
        return -2;
    if (dtype == ORACLE_E4M3 && (!q_scale || !k_scale || !v_scale))
        return -3;
    if (!rows && nrows != L)
        return -4;
    if (nrows < 1)
        return -4;
    if (rows) {
        for (int64_t i = 0; i < (int64_t)B * H * nrows; ++i)
            if (rows[i] < 0 || rows[i] >= L)
                return -5;
    }
#ifdef _OPENMP
    if (nthreads > 0)
        omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
    int64_t n = (int64_t)L * D;
    double *kh = (double *)malloc((size_t)n * sizeof(double));
    double *vh = (double *)malloc((size_t)n * sizeof(double));
    double *qh = (double *)malloc((size_t)n * sizeof(double));
    if (!kh || !vh || !qh) {
        free(kh); free(vh); free(qh);
        return -6;
    }
    int rc = 0;
    for (int64_t bh = 0; bh < (int64_t)B * H; ++bh) {
        decode_slice(dtype, k, k_scale, bh, n, kh);
        decode_slice(dtype, v, v_scale, bh, n, vh);
        decode_slice(dtype, q, q_scale, bh, n, qh);
        int fail = 0;
#pragma omp parallel
        {
            double *s = (double *)malloc((size_t)L * sizeof(double));
            if (!s) {
#pragma omp atomic write
                fail = 1;
            } else {
#pragma omp for schedule(dynamic, 4)
                for (int r = 0; r < nrows; ++r) {
                    int64_t i = rows ? rows[bh * nrows + r] : r;
                    attend_row(qh + i * D, kh, vh, L, D, scale, s,
                               o + (bh * nrows + r) * D,
                               lse ? lse + bh * nrows + r : NULL);
                }
                free(s);
            }
        }
        if (fail) {
            rc = -6;
            break;
        }
    }
    free(kh); free(vh); free(qh);
    return rc;
}

/* Threads an OpenMP region would use (the CPU baseline reports it). */
int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
