/*
 * CPU oracle for the NF4 + double-quantization codec.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, loads or
 * calls this file; only the test-suite, the smoke check and the benchmark's
 * CPU-baseline leg do.  It shares no source, header, table or helper with the
 * CUDA library: every number here is recomputed from the definitions.
 *
 * Plain scalar C, built with -O2 -ffp-contract=off (no FMA contraction, no
 * fast-math), so every float expression below is one IEEE-754 binary32 or
 * binary64 operation rounded to nearest-even, in the order written.
 *
 * Sources (web pages the method is described on):
 *   [P1] "LoRA 与 QLoRA" (whoami-wesleyyou.top), section QLoRA
 *        "1. NF4" (Gaussian 假设与分位数 / 分位数采样与端点问题 / 归一化与匹配)
 *        and "2. Double Quantization (DQ)".
 *   [P2] "QLoRA: Efficient Finetuning of Quantized LLMs", flash-card deck
 *        "3 QLoRA Finetuning" (learn.ifs.name), cards 2, 3, 4.
 *   [P4] jjjymmm.cn 2024/03 QLoRA post, sections "4-bit NormalFloat(NF4)"
 *        (the printed quant book) and "Double Quantization" / "QLoRA"
 *        (doubleDequant: restore the constant first, then the weight).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* Standard normal CDF and its inverse.                                     */
/* ------------------------------------------------------------------------ */

/* Phi(x) = P(Z <= x), Z ~ N(0,1), written through libm's erfc. */
double oracle_normal_cdf(double x) { return 0.5 * erfc(-x / sqrt(2.0)); }

/* Q_Z(p): the quantile function of N(0,1) [P1, Gaussian 假设与分位数].
 * Found by bisection on the monotone Phi until the bracket cannot shrink
 * further in binary64; obviously correct, slow, and independent of any
 * rational approximation. */
double oracle_normal_quantile(double p) {
    double lo = -40.0, hi = 40.0;
    for (int it = 0; it < 2000; ++it) {
        double mid = 0.5 * (lo + hi);
        if (mid <= lo || mid >= hi) break; /* bracket is two adjacent doubles */
        if (oracle_normal_cdf(mid) < p) lo = mid; else hi = mid;
    }
    return 0.5 * (lo + hi);
}

/* ------------------------------------------------------------------------ */
/* O1. The NF4 codebook.                                                    */
/* ------------------------------------------------------------------------ */

static int cmp_double(const void *a, const void *b) {
    double x = *(const double *)a, y = *(const double *)b;
    return (x > y) - (x < y);
}

/*
 * Asymmetric quantile construction [P2 card 3: separate negative and positive
 * halves sharing one zero; P1 归一化与匹配: normalize by the largest quantile].
 *   positive half: 9 probabilities evenly spaced from delta down to 1/2, the
 *                  1/2 dropped -> 8 values Q_Z(p);
 *   negative half: 8 probabilities evenly spaced from delta down to 1/2, the
 *                  1/2 dropped -> 7 values -Q_Z(p);
 *   plus an exact 0 (P1: 0 -> 0); all divided by Q_Z(delta) so the ends are
 *   exactly -1 and +1; sorted ascending.
 * delta is not printed on the pages; the printed table pins it (see tests).
 * out64 receives the binary64 values, out32 their round-to-nearest binary32.
 */
void oracle_nf4_codebook(double delta, double out64[16], float out32[16]) {
    double v[16];
    int n = 0;
    double top = oracle_normal_quantile(delta);
    for (int i = 0; i < 8; ++i) {
        double p = delta + (double)i * (0.5 - delta) / 8.0;
        v[n++] = oracle_normal_quantile(p) / top;
    }
    for (int i = 0; i < 7; ++i) {
        double p = delta + (double)i * (0.5 - delta) / 7.0;
        v[n++] = -oracle_normal_quantile(p) / top;
    }
    v[n++] = 0.0;
    qsort(v, 16, sizeof(double), cmp_double);
    for (int i = 0; i < 16; ++i) {
        out64[i] = v[i];
        out32[i] = (float)v[i];
    }
}

/* ------------------------------------------------------------------------ */
/* O2. Blockwise quantization (block of 64).                                */
/* ------------------------------------------------------------------------ */

/* Nearest codebook entry to x, by brute force over all 16 entries
 * [P4 4-bit NormalFloat(NF4): divide by ABSMAX, take the closest value of the
 * quant book].  Distances are exact in binary64 (x and cb[k] are binary32).
 * Ties keep the lower index. */
int oracle_nf4_nearest(float x, const float cb[16]) {
    int best = 0;
    double bestd = fabs((double)x - (double)cb[0]);
    for (int k = 1; k < 16; ++k) {
        double d = fabs((double)x - (double)cb[k]);
        if (d < bestd) { bestd = d; best = k; }
    }
    return best;
}

/* W (numel fp32, any numel >= 1) -> codes (ceil(numel/2) bytes, element 2i
 * in the high nibble of byte i) and absmax (ceil(numel/64) fp32).
 * a_j = max |w| over block j [P1 DQ: a_j = max|W_j|]; x = w / a_j rounded to
 * binary32; code = nearest entry.  An all-zero block (a_j == 0) gets code 7
 * (the exact zero) everywhere.
 * Tails (reading; the pages only use whole blocks): the last block holds the
 * numel mod 64 remaining weights and its absmax is taken over them; when numel
 * is odd the low nibble of the last byte is code 7, the code a zero weight
 * gets -- the same bytes as quantizing W zero-padded to whole blocks. */
void oracle_nf4_quantize(const float *w, int64_t numel, const float cb[16],
                         uint8_t *codes, float *absmax) {
    int64_t nb = (numel + 63) / 64;
    for (int64_t j = 0; j < nb; ++j) {
        const float *blk = w + j * 64;
        int len = numel - j * 64 < 64 ? (int)(numel - j * 64) : 64;
        float a = 0.0f;
        for (int i = 0; i < len; ++i) {
            float m = fabsf(blk[i]);
            if (m > a) a = m;
        }
        absmax[j] = a;
        int q[64];
        for (int i = 0; i < 64; ++i) {
            if (i >= len || a == 0.0f) { q[i] = 7; continue; }
            float x = blk[i] / a;
            q[i] = oracle_nf4_nearest(x, cb);
        }
        for (int i = 0; 2 * i < len; ++i)
            codes[j * 32 + i] = (uint8_t)((q[2 * i] << 4) | q[2 * i + 1]);
    }
}

/* ------------------------------------------------------------------------ */
/* O3. Double quantization of the block constants (groups of 256).          */
/* ------------------------------------------------------------------------ */

/* mu, the mean of the a_j, is computed exactly by the Python front end
 * (oracle/codec.py, dq_mean) and passed in: the binary32 value nearest to the
 * exact mean, ties to even. */

/* [P1 DQ] r_j = (a_j - mu) / b, r_j quantized to 8 bits as rhat_j,
 * restored as ahat_j = mu + b * rhat_j; mu and b kept in 32 bits.
 * [P2 card 4, P4 Double Quantization] the constants are quantized in blocks of
 * 256, each block keeping one 32-bit scale.
 * Reading (absmax scaling onto signed 8-bit, P4's INT-N quantization):
 *   d_j   = fp32(a_j - mu)
 *   B_g   = max_{j in g} |d_j|
 *   b_g   = fp32(B_g / 127)
 *   rhat  = clamp(rint(fp32(d_j / b_g)), -127, 127), ties to even; 0 if b_g == 0.
 * The final group may be partial. */
void oracle_nf4_double_quant(const float *absmax, int64_t nb, float mu, int8_t *qabs,
                             float *scale) {
    int64_t ng = (nb + 255) / 256;
    for (int64_t g = 0; g < ng; ++g) {
        int64_t j0 = g * 256, j1 = j0 + 256 < nb ? j0 + 256 : nb;
        float B = 0.0f;
        for (int64_t j = j0; j < j1; ++j) {
            float d = fabsf(absmax[j] - mu);
            if (d > B) B = d;
        }
        float b = B / 127.0f;
        scale[g] = b;
        for (int64_t j = j0; j < j1; ++j) {
            if (b == 0.0f) { qabs[j] = 0; continue; }
            float r = (absmax[j] - mu) / b;
            float rr = rintf(r); /* default rounding mode: nearest, ties to even */
            if (rr > 127.0f) rr = 127.0f;
            if (rr < -127.0f) rr = -127.0f;
            qabs[j] = (int8_t)rr;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* O3'. Double quantization with 8-bit floats (FP8 E4M3).                   */
/* ------------------------------------------------------------------------ */

/* [P2 card 4] quantizes the constants to "8-bit floats".  The 8-bit float
 * format here is OCP FP8 E4M3 (the "fn" variant): 1 sign bit, 4 exponent bits
 * with bias 7, 3 mantissa bits, no infinities, NaN only at S.1111.111.
 *   exponent field 0:      value = (m / 8) * 2^-6      (subnormals, +-0)
 *   exponent field e > 0:  value = (1 + m / 8) * 2^(e-7)
 * so the largest finite value is 1.75 * 2^8 = 448. */
double oracle_e4m3_value(uint8_t code) {
    int s = code >> 7, e = (code >> 3) & 15, m = code & 7;
    if (e == 15 && m == 7) return NAN;
    double v = e == 0 ? ldexp((double)m / 8.0, -6) : ldexp(1.0 + (double)m / 8.0, e - 7);
    return s ? -v : v;
}

/* Round a binary32 to E4M3: the nearest finite code, ties to the code with an
 * even mantissa, and anything beyond +-448 saturated to +-448 ("satfinite").
 * Brute force over the 127 non-negative finite codes; the sign is applied
 * after (the format is sign-magnitude).  Distances are exact in binary64. */
uint8_t oracle_e4m3_encode(float x) {
    double ax = fabs((double)x);
    uint8_t best = 0;
    double bestd = INFINITY;
    for (int c = 0; c <= 0x7e; ++c) {
        double d = fabs(ax - oracle_e4m3_value((uint8_t)c));
        if (d < bestd || (d == bestd && (c & 1) == 0)) {
            bestd = d;
            best = (uint8_t)c;
        }
    }
    if (ax >= 448.0) best = 0x7e;
    return (uint8_t)(best | (signbit(x) ? 0x80 : 0x00));
}

/* [P2 card 4] "8-bit floats" reading of the DQ step, otherwise as the INT8
 * reading above (same mu, same groups of 256):
 *   d_j   = fp32(a_j - mu)
 *   b_g   = fp32(max_{j in g} |d_j| / 448)        (448: the largest E4M3 value)
 *   rhat  = E4M3(fp32(d_j / b_g)), nearest-even, saturating; code 0 if b_g == 0. */
void oracle_nf4_double_quant_e4m3(const float *absmax, int64_t nb, float mu, uint8_t *qabs,
                                  float *scale) {
    int64_t ng = (nb + 255) / 256;
    for (int64_t g = 0; g < ng; ++g) {
        int64_t j0 = g * 256, j1 = j0 + 256 < nb ? j0 + 256 : nb;
        float B = 0.0f;
        for (int64_t j = j0; j < j1; ++j) {
            float d = fabsf(absmax[j] - mu);
            if (d > B) B = d;
        }
        float b = B / 448.0f;
        scale[g] = b;
        for (int64_t j = j0; j < j1; ++j) {
            if (b == 0.0f) { qabs[j] = 0; continue; }
            float r = (absmax[j] - mu) / b;
            qabs[j] = oracle_e4m3_encode(r);
        }
    }
}

/* ahat_j = fp32(mu + fp32(b_g * rhat_j)) [P1 DQ reconstruction, in the written
 * order: the product first, then the sum]. */
float oracle_dq_restore(int8_t rhat, float b, float mu) {
    float prod = b * (float)rhat;
    return mu + prod;
}

/* The same with an E4M3 code (its value is exact in binary32). */
float oracle_dq_restore_e4m3(uint8_t code, float b, float mu) {
    float prod = b * (float)oracle_e4m3_value(code);
    return mu + prod;
}

/* ------------------------------------------------------------------------ */
/* O4. doubleDequant to BF16.                                               */
/* ------------------------------------------------------------------------ */

/* binary32 -> bfloat16 bits, round to nearest, ties to even (NaN -> quiet). */
uint16_t oracle_bf16_rn(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu))
        return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

/* [P4 QLoRA: doubleDequant restores the quantization constant first, then
 * dequantizes the weight with it; P4 NF4: dequantization takes the quant-book
 * value] [P2 card 1: weights are dequantized to BFloat16 for the matmul]
 *   w' = bf16_RN( fp32( ahat_j * cb[q] ) ),  for the numel weights (any numel)
 * With qabs == NULL the block constants are the plain fp32 absmax (no DQ). */
void oracle_nf4_dequant_fmt(const uint8_t *codes, int64_t numel, const float *absmax,
                            const uint8_t *qabs, int e4m3, const float *scale, const float *mu,
                            const float cb[16], uint16_t *out) {
    int64_t nb = (numel + 63) / 64;
    for (int64_t j = 0; j < nb; ++j) {
        float a = !qabs ? absmax[j]
                  : e4m3 ? oracle_dq_restore_e4m3(qabs[j], scale[j / 256], *mu)
                         : oracle_dq_restore((int8_t)qabs[j], scale[j / 256], *mu);
        for (int i = 0; i < 64 && j * 64 + i < numel; ++i) {
            int64_t e = j * 64 + i;
            uint8_t byte = codes[e / 2];
            int q = (e % 2 == 0) ? (byte >> 4) : (byte & 15);
            float v = a * cb[q];
            out[e] = oracle_bf16_rn(v);
        }
    }
}

void oracle_nf4_dequant(const uint8_t *codes, int64_t numel, const float *absmax,
                        const int8_t *qabs, const float *scale, const float *mu,
                        const float cb[16], uint16_t *out) {
    oracle_nf4_dequant_fmt(codes, numel, absmax, (const uint8_t *)qabs, 0, scale, mu, cb, out);
}

/* Same as above but returns the binary32 value before the BF16 rounding. */
void oracle_nf4_dequant_f32_fmt(const uint8_t *codes, int64_t numel, const float *absmax,
                                const uint8_t *qabs, int e4m3, const float *scale, const float *mu,
                                const float cb[16], float *out) {
    int64_t nb = (numel + 63) / 64;
    for (int64_t j = 0; j < nb; ++j) {
        float a = !qabs ? absmax[j]
                  : e4m3 ? oracle_dq_restore_e4m3(qabs[j], scale[j / 256], *mu)
                         : oracle_dq_restore((int8_t)qabs[j], scale[j / 256], *mu);
        for (int i = 0; i < 64 && j * 64 + i < numel; ++i) {
            int64_t e = j * 64 + i;
            uint8_t byte = codes[e / 2];
            int q = (e % 2 == 0) ? (byte >> 4) : (byte & 15);
            out[e] = a * cb[q];
        }
    }
}

void oracle_nf4_dequant_f32(const uint8_t *codes, int64_t numel, const float *absmax,
                            const int8_t *qabs, const float *scale, const float *mu,
                            const float cb[16], float *out) {
    oracle_nf4_dequant_f32_fmt(codes, numel, absmax, (const uint8_t *)qabs, 0, scale, mu, cb, out);
}
