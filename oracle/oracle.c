/*
 * oracle.c -- plain, slow CPU oracle for the low-bit KV-cache hot path.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may call, link or
 * load this file; only the tests, the package smoke check and the benchmark's
 * CPU-baseline leg use it. It shares no code, header, table or constant with
 * the CUDA library.
 *
 * Build: gcc -O2 -ffp-contract=off -fno-fast-math -fPIC -shared (oracle/build.py).
 * Every float operation below is a single IEEE-754 operation rounded to the
 * type it is written in (x86-64 SSE, no contraction into FMA), so the fp32
 * recipe of the quantizer is reproduced exactly.
 *
 * Sources (titles of the pages the method comes from):
 *  [SAW]  "SAW-INT4: System-Aware 4-Bit KV-Cache Quantization for Real-World
 *         LLM Serving", Abstract: token-wise INT4 quantization with a
 *         block-diagonal Hadamard rotation, fused into paged KV layouts.
 *  [INQ]  "InnerQ: Hardware-Aware Tuning-Free Quantization of KV Cache for
 *         Large Language Models", Abstract: group-wise quantization along the
 *         inner dimension; high-precision windows of recent tokens.
 *  [XQ]   "XQuant: Breaking the Memory Wall for LLM Inference with KV Cache
 *         Rematerialization", Abstract: cache quantized layer inputs X and
 *         recompute K and V from them.
 *  [DQK]  "Dual-QK: Sharp Queries and Flat Keys for Prunable 2-bit KV Caches",
 *         Abstract: the orthogonal transform applied to keys is applied to
 *         queries as well, so query-key dot products are preserved.
 *
 * The pages give no formula for the quantizer. The fp32 recipe used here is
 * the plainest asymmetric min/max reading, fixed so that codes are unique:
 *   z = fp16 rounded toward -inf of min(x)   (a zero minimum taken as +0)
 *   s = fp16 rounded toward +inf of fp32(fp32(max(x) - z) / L),  L = 2^bits - 1
 *   s == 0 -> every code is 0
 *   else r = fp32(1 / s), q = clamp(rint_even(fp32(fp32(x - z) * r)), 0, L)
 * Directed rounding of s and z makes [z, z + L*s] cover [min, max], so every
 * element dequantizes to within s/2 (plus a few fp32 roundings) of itself.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include "oracle.h"

/* ------------------------------------------------------------------------ */
/* Number encodings                                                          */
/* ------------------------------------------------------------------------ */

/* Round the magnitude m >= 0 to a multiple of `quantum` (a power of two) in
 * the given magnitude mode: 0 nearest-even, 1 toward zero, 2 away from zero. */
static double round_to_quantum(double m, double quantum, int mag_mode)
{
    double t = m / quantum; /* exact: quantum is a power of two */
    double r;
    if (mag_mode == 0)
        r = nearbyint(t); /* default rounding mode is nearest-even */
    else if (mag_mode == 1)
        r = floor(t);
    else
        r = ceil(t);
    return r * quantum;
}

/* Map a signed rounding mode (0 nearest-even, 1 toward -inf, 2 toward +inf)
 * onto a magnitude rounding mode for a value of the given sign. */
static int magnitude_mode(int mode, int negative)
{
    if (mode == ORACLE_RN)
        return 0;
    if (mode == ORACLE_RD)
        return negative ? 2 : 1;
    return negative ? 1 : 2;
}

/* IEEE binary16: 1 sign, 5 exponent (bias 15), 10 fraction bits.
 * Normal numbers have quantum 2^(E-10) for exponent E in [-14, 15];
 * subnormals have quantum 2^-24. Largest finite value 65504. */
uint16_t oracle_f32_to_f16(float v, int mode)
{
    double a = (double)v;
    if (isnan(a))
        return 0x7E00;
    int neg = signbit(a) ? 1 : 0;
    uint16_t sign = neg ? 0x8000 : 0;
    double m = fabs(a);
    if (isinf(m))
        return sign | 0x7C00;
    if (m == 0.0)
        return sign;
    int mag = magnitude_mode(mode, neg);
    int e2;
    frexp(m, &e2); /* m = f * 2^e2, f in [0.5, 1) */
    int E = e2 - 1;
    if (E < -14)
        E = -14;
    double res = round_to_quantum(m, ldexp(1.0, E - 10), mag);
    if (res > 65504.0) {
        /* Past the largest finite half: nearest-even reaches infinity only
         * from 65520 up (handled by the rounding above giving 65536);
         * toward zero stops at 65504; away from zero goes to infinity. */
        if (mag == 1)
            res = 65504.0;
        else
            return sign | 0x7C00;
    }
    if (res == 0.0)
        return sign;
    if (res < ldexp(1.0, -14)) /* subnormal */
        return sign | (uint16_t)(res / ldexp(1.0, -24));
    int e;
    double f = frexp(res, &e); /* res = f * 2^e, f in [0.5, 1) */
    uint16_t exp_field = (uint16_t)(e - 1 + 15);
    uint16_t frac = (uint16_t)((f * 2.0 - 1.0) * 1024.0);
    return sign | (uint16_t)(exp_field << 10) | frac;
}

void oracle_f32_to_f16_array(const float *v, int64_t n, int mode, uint16_t *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = oracle_f32_to_f16(v[i], mode);
}

float oracle_f16_to_f32(uint16_t h)
{
    int neg = (h >> 15) & 1;
    int exp_field = (h >> 10) & 0x1F;
    int frac = h & 0x3FF;
    double m;
    if (exp_field == 0x1F)
        m = frac ? NAN : INFINITY;
    else if (exp_field == 0)
        m = ldexp((double)frac, -24);
    else
        m = ldexp(1.0 + frac / 1024.0, exp_field - 15);
    return (float)(neg ? -m : m);
}

/* bfloat16: 1 sign, 8 exponent (bias 127), 7 fraction bits. Normal numbers
 * have quantum 2^(E-7) for E in [-126, 127]; subnormals 2^-133. */
uint16_t oracle_f32_to_bf16_rn(float v)
{
    double a = (double)v;
    if (isnan(a))
        return 0x7FC0;
    int neg = signbit(a) ? 1 : 0;
    uint16_t sign = neg ? 0x8000 : 0;
    double m = fabs(a);
    if (isinf(m))
        return sign | 0x7F80;
    if (m == 0.0)
        return sign;
    int e2;
    frexp(m, &e2);
    int E = e2 - 1;
    if (E < -126)
        E = -126;
    double res = round_to_quantum(m, ldexp(1.0, E - 7), 0);
    double max_bf16 = ldexp(255.0 / 128.0, 127);
    if (res > max_bf16)
        return sign | 0x7F80;
    if (res == 0.0)
        return sign;
    if (res < ldexp(1.0, -126))
        return sign | (uint16_t)(res / ldexp(1.0, -133));
    int e;
    double f = frexp(res, &e);
    uint16_t exp_field = (uint16_t)(e - 1 + 127);
    uint16_t frac = (uint16_t)((f * 2.0 - 1.0) * 128.0);
    return sign | (uint16_t)(exp_field << 7) | frac;
}

void oracle_f32_to_bf16_rn_array(const float *v, int64_t n, uint16_t *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = oracle_f32_to_bf16_rn(v[i]);
}

float oracle_bf16_to_f32(uint16_t b)
{
    int neg = (b >> 15) & 1;
    int exp_field = (b >> 7) & 0xFF;
    int frac = b & 0x7F;
    double m;
    if (exp_field == 0xFF)
        m = frac ? NAN : INFINITY;
    else if (exp_field == 0)
        m = ldexp((double)frac, -133);
    else
        m = ldexp(1.0 + frac / 128.0, exp_field - 127);
    return (float)(neg ? -m : m);
}

/* ------------------------------------------------------------------------ */
/* Rotation [SAW], [DQK]                                                     */
/* ------------------------------------------------------------------------ */

/* Normalized Sylvester Walsh-Hadamard transform of n = 2^k fp32 values, in
 * place. Butterfly stages run with half-width h = 1, 2, 4, ..., n/2 in that
 * order; each butterfly maps (x[j], x[j+h]) to (x[j] + x[j+h], x[j] - x[j+h]),
 * each sum and difference rounded to fp32. Afterwards every element is
 * multiplied once by c = fp32(1/sqrt(n)). The unnormalized stages compute
 * H_n x for the Sylvester matrix H_1 = [1], H_2m = [[H_m, H_m], [H_m, -H_m]];
 * H_n H_n^T = n I, so c * H_n is orthogonal. */
void oracle_fwht_f32(float *x, int n)
{
    for (int h = 1; h < n; h <<= 1) {
        for (int i = 0; i < n; i += 2 * h) {
            for (int j = i; j < i + h; ++j) {
                float a = x[j];
                float b = x[j + h];
                x[j] = a + b;
                x[j + h] = a - b;
            }
        }
    }
    float c = (float)(1.0 / sqrt((double)n));
    for (int i = 0; i < n; ++i)
        x[i] = x[i] * c;
}

/* The same transform in float64 (butterflies and the final 1/sqrt(n) in
 * double): used to rotate queries, whose rotation need not reproduce the
 * fp32 rounding of the key path, only the transform itself [DQK]. */
void oracle_fwht_f64(double *x, int n)
{
    for (int h = 1; h < n; h <<= 1) {
        for (int i = 0; i < n; i += 2 * h) {
            for (int j = i; j < i + h; ++j) {
                double a = x[j];
                double b = x[j + h];
                x[j] = a + b;
                x[j + h] = a - b;
            }
        }
    }
    double c = 1.0 / sqrt((double)n);
    for (int i = 0; i < n; ++i)
        x[i] = x[i] * c;
}

void oracle_rotate_blocks_f64(double *x, int64_t n_vec, int D, int hb)
{
    for (int64_t v = 0; v < n_vec; ++v)
        for (int b = 0; b < D; b += hb)
            oracle_fwht_f64(x + v * D + b, hb);
}

/* Block-diagonal rotation [SAW]: each of the n_vec rows of D values is split
 * into D/hb consecutive blocks of hb values, each rotated independently. */
void oracle_rotate_blocks_f32(float *x, int64_t n_vec, int D, int hb)
{
    for (int64_t v = 0; v < n_vec; ++v)
        for (int b = 0; b < D; b += hb)
            oracle_fwht_f32(x + v * D + b, hb);
}

/* ------------------------------------------------------------------------ */
/* Group quantization [SAW] token-wise, [INQ] group-wise                     */
/* ------------------------------------------------------------------------ */

void oracle_quantize_group(const float *x, int n, int stride, int bits,
                           uint16_t *s_out, uint16_t *z_out, uint8_t *q_out,
                           int q_stride)
{
    const int L = (1 << bits) - 1;
    float mn = x[0], mx = x[0];
    for (int i = 1; i < n; ++i) {
        float v = x[(int64_t)i * stride];
        if (v < mn)
            mn = v;
        if (v > mx)
            mx = v;
    }
    /* A zero extreme is taken as +0 (adding +0 turns -0 into +0), so the
     * zero-point's bit pattern does not depend on which signed zero comes
     * first in the group. */
    mn = mn + 0.0f;
    mx = mx + 0.0f;
    uint16_t zb = oracle_f32_to_f16(mn, ORACLE_RD);
    float z = oracle_f16_to_f32(zb);
    float range = mx - z;
    float step = range / (float)L;
    uint16_t sb = oracle_f32_to_f16(step, ORACLE_RU);
    float s = oracle_f16_to_f32(sb);
    *s_out = sb;
    *z_out = zb;
    if (s == 0.0f) {
        for (int i = 0; i < n; ++i)
            q_out[(int64_t)i * q_stride] = 0;
        return;
    }
    float r = 1.0f / s;
    for (int i = 0; i < n; ++i) {
        float d = x[(int64_t)i * stride] - z;
        float t = d * r;
        float qf = rintf(t);
        if (qf < 0.0f)
            qf = 0.0f;
        if (qf > (float)L)
            qf = (float)L;
        q_out[(int64_t)i * q_stride] = (uint8_t)qf;
    }
}

/* Hybrid symmetric/asymmetric choice per group [INQ] "(i) hybrid
 * quantization ... based on local statistics". The page states no criterion;
 * this reading takes the candidate with the smaller worst-case reconstruction
 * error of the group, ties to the asymmetric one:
 *   asymmetric: the recipe of oracle_quantize_group above;
 *   symmetric:  a grid with an exact zero level. Qp = 2^(bits-1) - 1,
 *     C = 2^(bits-1), m = max(|min|, |max|) (zero extremes as +0),
 *     s = fp16 rounded toward +inf of fp32(m / Qp), z = -C * s (exact; the
 *     candidate is dropped when |z| > 65504, the largest fp16),
 *     s == 0 -> every code is C, else r = fp32(1 / s),
 *     q = clamp(rint_even(fp32(x * r)), -Qp, Qp) + C.
 *   Both candidates store (s, z) as fp16 and dequantize as q * s + z, so the
 *   choice is invisible to the readers of the cache.
 *   Error of a candidate: the largest |e| over the group with
 *   e = fp32(x - fma(q, s, z)) per element; a maximum is exact, so the choice
 *   does not depend on the order the elements are visited in. Symmetric iff
 *   its largest error is smaller. */
static float max_abs_err(const float *x, int n, int stride, const uint8_t *q,
                         int q_stride, float s, float z)
{
    float m = 0.0f;
    for (int i = 0; i < n; ++i) {
        float xh = fmaf((float)q[(int64_t)i * q_stride], s, z);
        float e = fabsf(x[(int64_t)i * stride] - xh);
        if (e > m)
            m = e;
    }
    return m;
}

void oracle_quantize_group_hybrid(const float *x, int n, int stride, int bits,
                                  uint16_t *s_out, uint16_t *z_out,
                                  uint8_t *q_out, int q_stride)
{
    uint16_t sa, za;
    oracle_quantize_group(x, n, stride, bits, &sa, &za, q_out, q_stride);
    *s_out = sa;
    *z_out = za;
    const int C = 1 << (bits - 1), Qp = C - 1;
    float mn = x[0], mx = x[0];
    for (int i = 1; i < n; ++i) {
        float v = x[(int64_t)i * stride];
        if (v < mn)
            mn = v;
        if (v > mx)
            mx = v;
    }
    mn = mn + 0.0f;
    mx = mx + 0.0f;
    float m = fabsf(mn) > fabsf(mx) ? fabsf(mn) : fabsf(mx);
    uint16_t sb = oracle_f32_to_f16(m / (float)Qp, ORACLE_RU);
    float ss = oracle_f16_to_f32(sb);
    float zs = -(float)C * ss;
    if (!(fabsf(zs) <= 65504.0f))
        return;
    uint16_t zb = oracle_f32_to_f16(zs, ORACLE_RN);
    uint8_t *qs = (uint8_t *)calloc((size_t)n, 1);
    float r = (ss == 0.0f) ? 0.0f : 1.0f / ss;
    for (int i = 0; i < n; ++i) {
        float t = rintf(x[(int64_t)i * stride] * r);
        if (t < -(float)Qp)
            t = -(float)Qp;
        if (t > (float)Qp)
            t = (float)Qp;
        qs[i] = (uint8_t)(int)(t + (float)C);
    }
    float ea = max_abs_err(x, n, stride, q_out, q_stride, oracle_f16_to_f32(sa),
                           oracle_f16_to_f32(za));
    float es = max_abs_err(x, n, stride, qs, 1, ss, zs);
    if (es < ea) {
        *s_out = sb;
        *z_out = zb;
        for (int i = 0; i < n; ++i)
            q_out[(int64_t)i * q_stride] = qs[i];
    }
    free(qs);
}

/* Packing: INT4 puts element 2i in the low nibble of byte i and 2i+1 in the
 * high nibble; INT2 puts element 4i+j in bits 2j..2j+1 of byte i. */
void oracle_pack_codes(const uint8_t *q, int n, int bits, uint8_t *out)
{
    int per_byte = 8 / bits;
    for (int i = 0; i < n / per_byte; ++i) {
        uint8_t b = 0;
        for (int j = 0; j < per_byte; ++j)
            b |= (uint8_t)(q[i * per_byte + j] << (bits * j));
        out[i] = b;
    }
}

void oracle_unpack_codes(const uint8_t *packed, int n, int bits, uint8_t *q)
{
    int per_byte = 8 / bits;
    uint8_t mask = (uint8_t)((1 << bits) - 1);
    for (int i = 0; i < n; ++i)
        q[i] = (packed[i / per_byte] >> (bits * (i % per_byte))) & mask;
}

/* Token-wise quantization of n_vec vectors of D fp32 values: optional
 * block-diagonal rotation (hb = 0: none), then groups of G consecutive
 * elements along D. codes: [n_vec][D*bits/8], sz: [n_vec][D/G][2] holding
 * the fp16 bit patterns (scale, zero). */
void oracle_quantize_tokens(const float *x, int64_t n_vec, int D, int hb,
                            int G, int bits, int hybrid, uint8_t *codes,
                            uint16_t *sz)
{
    float *tmp = (float *)malloc(sizeof(float) * D);
    uint8_t *q = (uint8_t *)malloc(D);
    int row_bytes = D * bits / 8;
    int ng = D / G;
    for (int64_t v = 0; v < n_vec; ++v) {
        memcpy(tmp, x + v * D, sizeof(float) * D);
        if (hb > 0)
            oracle_rotate_blocks_f32(tmp, 1, D, hb);
        for (int g = 0; g < ng; ++g) {
            uint16_t *p = sz + (v * ng + g) * 2;
            (hybrid ? oracle_quantize_group_hybrid : oracle_quantize_group)(
                tmp + g * G, G, 1, bits, &p[0], &p[1], q + g * G, 1);
        }
        oracle_pack_codes(q, D, bits, codes + v * row_bytes);
    }
    free(q);
    free(tmp);
}

/* Channel-wise quantization of one block of R tokens x D channels (KIVI-style
 * keys): each channel's R values form one group. codes: [R][D*bits/8] packed
 * along channels within each token; sz: [D][2]. */
void oracle_quantize_channel_block(const float *x, int R, int D, int bits,
                                   int hybrid, uint8_t *codes, uint16_t *sz)
{
    uint8_t *q = (uint8_t *)malloc((size_t)R * D);
    for (int d = 0; d < D; ++d)
        (hybrid ? oracle_quantize_group_hybrid : oracle_quantize_group)(
            x + d, R, D, bits, &sz[2 * d], &sz[2 * d + 1], q + d, D);
    int row_bytes = D * bits / 8;
    for (int t = 0; t < R; ++t)
        oracle_pack_codes(q + (int64_t)t * D, D, bits, codes + (int64_t)t * row_bytes);
    free(q);
}

/* Dequantization x_hat = q * s + z, exact in float64. */
void oracle_dequant_tokens(const uint8_t *codes, const uint16_t *sz,
                           int64_t n_vec, int D, int G, int bits, double *out)
{
    uint8_t *q = (uint8_t *)malloc(D);
    int row_bytes = D * bits / 8;
    int ng = D / G;
    for (int64_t v = 0; v < n_vec; ++v) {
        oracle_unpack_codes(codes + v * row_bytes, D, bits, q);
        for (int i = 0; i < D; ++i) {
            const uint16_t *p = sz + (v * ng + i / G) * 2;
            double s = oracle_f16_to_f32(p[0]);
            double z = oracle_f16_to_f32(p[1]);
            out[v * D + i] = (double)q[i] * s + z;
        }
    }
    free(q);
}

void oracle_dequant_channel_block(const uint8_t *codes, const uint16_t *sz,
                                  int R, int D, int bits, double *out)
{
    uint8_t *q = (uint8_t *)malloc(D);
    int row_bytes = D * bits / 8;
    for (int t = 0; t < R; ++t) {
        oracle_unpack_codes(codes + (int64_t)t * row_bytes, D, bits, q);
        for (int d = 0; d < D; ++d) {
            double s = oracle_f16_to_f32(sz[2 * d]);
            double z = oracle_f16_to_f32(sz[2 * d + 1]);
            out[(int64_t)t * D + d] = (double)q[d] * s + z;
        }
    }
    free(q);
}

/* ------------------------------------------------------------------------ */
/* Decode attention over the dequantized cache [SAW] fused attention,        */
/* [INQ] decode stage                                                        */
/* ------------------------------------------------------------------------ */

/* For each of the n_q query rows: s_t = scale * (q . k_t) for t in [0, T),
 * p_t = exp(s_t - max_t s_t), out = sum_t p_t v_t / sum_t p_t. float64. */
void oracle_attention(const double *q, int n_q, const double *k,
                      const double *v, int64_t T, int D, double scale,
                      double *out)
{
    double *s = (double *)malloc(sizeof(double) * (T > 0 ? T : 1));
    for (int h = 0; h < n_q; ++h) {
        const double *qh = q + (int64_t)h * D;
        double *oh = out + (int64_t)h * D;
        for (int d = 0; d < D; ++d)
            oh[d] = 0.0;
        if (T == 0)
            continue;
        double m = -INFINITY;
        for (int64_t t = 0; t < T; ++t) {
            double acc = 0.0;
            for (int d = 0; d < D; ++d)
                acc += qh[d] * k[t * D + d];
            s[t] = acc * scale;
            if (s[t] > m)
                m = s[t];
        }
        double l = 0.0;
        for (int64_t t = 0; t < T; ++t) {
            double p = exp(s[t] - m);
            l += p;
            for (int d = 0; d < D; ++d)
                oh[d] += p * v[t * D + d];
        }
        for (int d = 0; d < D; ++d)
            oh[d] /= l;
    }
    free(s);
}

/* ------------------------------------------------------------------------ */
/* Rematerialization [XQ]                                                    */
/* ------------------------------------------------------------------------ */

/* Dequantize token-wise quantized X to the bf16 operand of the GEMM:
 * x_hat = bf16_rn(fp32(q * s + z)). q * s + z is computed exactly in
 * float64 (q <= 15 and s, z are fp16, so it needs well under 53 bits) and
 * rounded once to fp32, then once to bf16. Output: bf16 values widened to
 * fp32, [n_tok][hidden]. */
void oracle_dequant_x_bf16(const uint8_t *codes, const uint16_t *sz,
                           int64_t n_tok, int hidden, int G, int bits,
                           float *xhat)
{
    uint8_t *q = (uint8_t *)malloc(hidden);
    int row_bytes = hidden * bits / 8;
    int ng = hidden / G;
    for (int64_t t = 0; t < n_tok; ++t) {
        oracle_unpack_codes(codes + t * row_bytes, hidden, bits, q);
        for (int i = 0; i < hidden; ++i) {
            const uint16_t *p = sz + (t * ng + i / G) * 2;
            double s = oracle_f16_to_f32(p[0]);
            double z = oracle_f16_to_f32(p[1]);
            float f = (float)((double)q[i] * s + z);
            xhat[t * hidden + i] = oracle_bf16_to_f32(oracle_f32_to_bf16_rn(f));
        }
    }
    free(q);
}

/* out[m][n] = sum_k a[m][k] * w[n][k] in float64 (w stored [N][K], the
 * layout of a linear layer's weight). */
void oracle_matmul_nt(const float *a, const float *w, int64_t M, int N, int K,
                      double *out)
{
    for (int64_t m = 0; m < M; ++m) {
        const float *am = a + m * K;
        for (int n = 0; n < N; ++n) {
            const float *wn = w + (int64_t)n * K;
            double acc = 0.0;
            for (int k = 0; k < K; ++k)
                acc += (double)am[k] * (double)wn[k];
            out[m * N + n] = acc;
        }
    }
}

/* Rotary position embedding (RoFormer) in the rotate-half pairing: for each
 * head of D values and i in [0, D/2), with angle a = pos * theta^(-2i/D):
 *   y[i]       = x[i] cos a - x[i + D/2] sin a
 *   y[i + D/2] = x[i + D/2] cos a + x[i] sin a
 * x: [M][H][D] float64, in place; pos: [M]. */
void oracle_rope(double *x, const int64_t *pos, int64_t M, int H, int D,
                 double theta)
{
    int half = D / 2;
    for (int64_t m = 0; m < M; ++m) {
        for (int h = 0; h < H; ++h) {
            double *xh = x + (m * H + h) * D;
            for (int i = 0; i < half; ++i) {
                double inv_freq = pow(theta, -2.0 * (double)i / (double)D);
                double a = (double)pos[m] * inv_freq;
                double c = cos(a), s = sin(a);
                double x0 = xh[i], x1 = xh[i + half];
                xh[i] = x0 * c - x1 * s;
                xh[i + half] = x1 * c + x0 * s;
            }
        }
    }
}
