/*
 * vox_ref.c -- plain, slow CPU oracle for the Q4_0 decode hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the bench's
 * CPU-baseline leg may load this library.  It shares no code, header, table
 * or helper with the CUDA path; every function below is written from the
 * definition it cites, accumulates in double precision, and makes no attempt
 * at speed beyond an OpenMP loop over independent output rows.
 *
 * Sources (page titles as they appear on the pages):
 *  - Q4_0 block format: "Voxtral Mini 4B Realtime (Rust)", page 5,
 *    "Arquitetura" (GGUF Q4_0 path).  Block = fp16 scale d + 16 bytes of
 *    nibbles for 32 weights, w = (q - 8) * d.  GGUF byte order: element j
 *    (j < 16) is the low nibble of byte j, element j + 16 the high nibble.
 *  - Fused dequant + matmul: "브라우저에서 도는 4B 음성인식: Voxtral Rust+WASM
 *    구현 해부", section "F32(9GB) vs Q4 GGUF(2.5GB)".
 *  - Rolling KV cache of 8192 positions and GQA 32/8: "Mistral Voxtral
 *    Realtime 4B ... 순수 C 기반 CPU 전용 추론 구현", sections "주요 기능" and
 *    "모델 아키텍처".
 *
 * Readings where the pages are silent (each listed in the design notes):
 *  R1 GGUF nibble order, R2 bf16 round-to-nearest-even with NaN -> 0x7FC0,
 *  R6 slot = pos mod W and the first min(pos+1, W) slots are valid,
 *  R7 q head h reads kv head h / (n_q / n_kv), scale given by the caller.
 *
 * Pins: every function here is checked by tests/test_oracle_pins.py against
 * hand-built blocks, numpy's fp16 and torch's bf16 casts, the block-sum
 * identity, brute-force list models and closed forms.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#include <stdlib.h>

/* IEEE-754 binary16 -> double, written out from the format definition:
 * sign(1) exponent(5, bias 15) fraction(10). */
double vr_half_to_double(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int expo = (h >> 10) & 31;
    int frac = h & 1023;
    double v;
    if (expo == 0) {
        v = ldexp((double)frac, -24);                 /* subnormal: frac * 2^-24 */
    } else if (expo == 31) {
        v = frac ? NAN : INFINITY;
    } else {
        v = ldexp((double)(1024 + frac), expo - 25);  /* (1 + frac/1024) * 2^(expo-15) */
    }
    return sign ? -v : v;
}

/* bf16 bit pattern -> double: the bf16 value is the top half of an fp32. */
double vr_bf16_to_double(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* fp32 -> bf16, round to nearest, ties to even; NaN -> 0x7FC0 (R2).
 * Written from the rounding rule: keep the top 16 bits, look at the 16
 * dropped bits, round up when they exceed half an ulp or equal it with an
 * odd kept part. */
uint16_t vr_f32_to_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return 0x7FC0;
    uint32_t kept = u >> 16;
    uint32_t dropped = u & 0xFFFFu;
    if (dropped > 0x8000u || (dropped == 0x8000u && (kept & 1u))) kept += 1; /* may carry into inf */
    return (uint16_t)kept;
}

/* The 4-bit code of element j (0..31) of one block, GGUF order (R1). */
static int q4_code(const uint8_t *qs16, int j)
{
    return j < 16 ? (qs16[j] & 0x0F) : (qs16[j - 16] >> 4);
}

/* Exact dequantised weights of one row: w[32 b + j] = (q - 8) * d_b. */
void vr_q4_row(const uint8_t *qs /* [nb][16] */, const uint16_t *d /* [nb] */,
               int64_t nb, double *w /* [32 nb] */)
{
    for (int64_t b = 0; b < nb; ++b) {
        double db = vr_half_to_double(d[b]);
        for (int j = 0; j < 32; ++j) w[32 * b + j] = (double)(q4_code(qs + 16 * b, j) - 8) * db;
    }
}

/* Dequantise rows [row0, row0+nrows) to fp32.  (q-8)*d needs at most 4 + 11
 * significant bits, so the fp32 result is exact and any correct
 * implementation gives the same bits. */
void vr_q4_dequant_f32(const uint8_t *qs, const uint16_t *d, int64_t n, int64_t k,
                       int64_t row0, int64_t nrows, float *out)
{
    (void)n;
    int64_t nb = k / 32;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < nrows; ++r) {
        double *w = (double *)malloc(sizeof(double) * (size_t)k);
        vr_q4_row(qs + (row0 + r) * nb * 16, d + (row0 + r) * nb, nb, w);
        for (int64_t c = 0; c < k; ++c) out[r * k + c] = (float)w[c];
        free(w);
    }
}

/* Dequantise to bf16: round-to-nearest-even of the exact fp32 weight (R2). */
void vr_q4_dequant_bf16(const uint8_t *qs, const uint16_t *d, int64_t n, int64_t k,
                        int64_t row0, int64_t nrows, uint16_t *out)
{
    (void)n;
    int64_t nb = k / 32;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < nrows; ++r) {
        double *w = (double *)malloc(sizeof(double) * (size_t)k);
        vr_q4_row(qs + (row0 + r) * nb * 16, d + (row0 + r) * nb, nb, w);
        for (int64_t c = 0; c < k; ++c) out[r * k + c] = vr_f32_to_bf16((float)w[c]);
        free(w);
    }
}

/* Dense route: y[m][r] = sum_k w[row0 + r][k] * x[m][k] in double, over the
 * exactly dequantised weights, for output rows [row0, row0 + nrows). */
void vr_q4_matvec(const uint8_t *qs, const uint16_t *d, int64_t n, int64_t k,
                  int64_t row0, int64_t nrows,
                  const float *x, int64_t m, int64_t ldx, double *y /* [m][nrows] */)
{
    (void)n;
    int64_t nb = k / 32;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < nrows; ++r) {
        double *w = (double *)malloc(sizeof(double) * (size_t)k);
        vr_q4_row(qs + (row0 + r) * nb * 16, d + (row0 + r) * nb, nb, w);
        for (int64_t i = 0; i < m; ++i) {
            double acc = 0.0;
            for (int64_t c = 0; c < k; ++c) acc += w[c] * (double)x[i * ldx + c];
            y[i * nrows + r] = acc;
        }
        free(w);
    }
}

/* Block-sum route of the same product, a second derivation used to pin the
 * dense route: y = sum_b d_b * (sum_j q_j x_j - 8 sum_j x_j). */
void vr_q4_matvec_blocksum(const uint8_t *qs, const uint16_t *d, int64_t n, int64_t k,
                           const float *x, int64_t m, int64_t ldx, double *y /* [m][n] */)
{
    int64_t nb = k / 32;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n; ++r) {
        for (int64_t i = 0; i < m; ++i) {
            double acc = 0.0;
            for (int64_t b = 0; b < nb; ++b) {
                const uint8_t *blk = qs + (r * nb + b) * 16;
                double sqx = 0.0, sx = 0.0;
                for (int j = 0; j < 32; ++j) {
                    double xv = (double)x[i * ldx + 32 * b + j];
                    sqx += (double)q4_code(blk, j) * xv;
                    sx += xv;
                }
                acc += vr_half_to_double(d[r * nb + b]) * (sqx - 8.0 * sx);
            }
            y[i * n + r] = acc;
        }
    }
}

/* Rolling cache slot of absolute position pos in a window of W slots (R6). */
int64_t vr_kv_slot(int64_t pos, int64_t window)
{
    return pos % window;
}

/* Append one position: k_new, v_new fp32 [n_kv][hd] are rounded to bf16 (R2)
 * and stored at slot pos mod W of caches laid out [n_kv][W][hd]. */
void vr_kv_append(uint16_t *k_cache, uint16_t *v_cache, const float *k_new, const float *v_new,
                  int n_kv, int hd, int64_t window, int64_t pos)
{
    int64_t slot = vr_kv_slot(pos, window);
    for (int h = 0; h < n_kv; ++h)
        for (int c = 0; c < hd; ++c) {
            k_cache[((int64_t)h * window + slot) * hd + c] = vr_f32_to_bf16(k_new[h * hd + c]);
            v_cache[((int64_t)h * window + slot) * hd + c] = vr_f32_to_bf16(v_new[h * hd + c]);
        }
}

/* GQA decode attention over the rolling cache after position pos was written.
 * Valid slots: 0 .. min(pos+1, W)-1 (R6).  Query head h reads kv head
 * h / (n_q / n_kv) (R7).  s_j = scale * q.k_j, p = softmax(s), o = sum p_j v_j.
 * Only o is returned; the split-KV partials are a NumPy-side reference. */
void vr_gqa_attn(const float *q /* [n_q][hd] */, const uint16_t *k_cache, const uint16_t *v_cache,
                 int n_q, int n_kv, int hd, int64_t window, int64_t pos, double scale,
                 double *out /* [n_q][hd] */)
{
    int64_t n_valid = pos + 1 < window ? pos + 1 : window;
    int group = n_q / n_kv;
#pragma omp parallel for schedule(static)
    for (int h = 0; h < n_q; ++h) {
        int kvh = h / group;
        double *s = (double *)malloc(sizeof(double) * (size_t)n_valid);
        double smax = -INFINITY;
        for (int64_t j = 0; j < n_valid; ++j) {
            double acc = 0.0;
            for (int c = 0; c < hd; ++c)
                acc += (double)q[h * hd + c] * vr_bf16_to_double(k_cache[((int64_t)kvh * window + j) * hd + c]);
            s[j] = scale * acc;
            if (s[j] > smax) smax = s[j];
        }
        double denom = 0.0;
        for (int64_t j = 0; j < n_valid; ++j) {
            s[j] = exp(s[j] - smax);
            denom += s[j];
        }
        for (int c = 0; c < hd; ++c) {
            double acc = 0.0;
            for (int64_t j = 0; j < n_valid; ++j)
                acc += s[j] * vr_bf16_to_double(v_cache[((int64_t)kvh * window + j) * hd + c]);
            out[h * hd + c] = acc / denom;
        }
        free(s);
    }
}
