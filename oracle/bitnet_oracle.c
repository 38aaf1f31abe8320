/*
 * bitnet_oracle.c -- plain CPU oracle for the I2_S ternary linear layer.
 *
 * TEST INFRASTRUCTURE ONLY (see bitnet_oracle.h for the readings R1-R4 and
 * the passages they follow).  Single-threaded, no blocking, no vectorisation
 * tricks: every output is computed straight from its definition.  Compile with
 * -ffp-contract=off so that no multiply is fused into an add.
 */
#include "bitnet_oracle.h"

#include <math.h>
#include <stddef.h>
#include <stdlib.h>

int64_t oracle_blocks(int64_t k) { return (k + 127) / 128; }
int64_t oracle_kpad(int64_t k) { return 128 * oracle_blocks(k); }

/* R1 -- per-token INT8 activation quantisation done at run time
 * (VibeVoice-ASR-BitNet Technical Report, §2.2.2), with the absmax/127 rule. */
int oracle_quant_act(const float *x, int64_t m, int64_t k, int8_t *q, float *s_act)
{
    int status = ORACLE_OK;
    const int64_t kpad = oracle_kpad(k);
    for (int64_t r = 0; r < m; ++r) {
        const float *xr = x + r * k;
        int8_t *qr = q + r * kpad;
        int finite = 1;
        float amax = 0.0f;
        for (int64_t i = 0; i < k; ++i) {
            if (!isfinite(xr[i])) finite = 0;
            else if (fabsf(xr[i]) > amax) amax = fabsf(xr[i]);
        }
        for (int64_t i = 0; i < kpad; ++i) qr[i] = 0;
        if (!finite) {
            s_act[r] = 0.0f;
            status |= ORACLE_NONFINITE;
            continue;
        }
        if (amax == 0.0f) {
            s_act[r] = 0.0f;
            continue;
        }
        const float inv = 127.0f / amax;
        for (int64_t i = 0; i < k; ++i) {
            if (xr[i] == 0.0f) { qr[i] = 0; continue; }
            float v = xr[i] * inv;           /* one rounded fp32 product */
            if (v > 127.0f) v = 127.0f;      /* clamping to integers commutes */
            if (v < -127.0f) v = -127.0f;    /* with rounding to integers     */
            qr[i] = (int8_t)(int)rintf(v);   /* default mode: half to even    */
        }
        s_act[r] = amax / 127.0f;
    }
    return status;
}

/* R5, second pass -- the ternary codes at a given scale s: fp32 divide, fp32
 * rint (half to even), clamp to [-1, 1]; s == 0 gives every code 0. */
void oracle_ternary_round(const float *W, int64_t total, float s, int8_t *w)
{
    for (int64_t i = 0; i < total; ++i) {
        if (s == 0.0f) {
            w[i] = 0;
            continue;
        }
        float v = rintf(W[i] / s);        /* one rounded fp32 quotient, half to even */
        if (v > 1.0f) v = 1.0f;
        if (v < -1.0f) v = -1.0f;
        w[i] = (int8_t)(int)v;
    }
}

/* R5 -- absmean ternary quantiser, written from its definition: one pass for
 * the mean of |W| (fp64 sum in row-major order, one rounding to fp32), one
 * pass for the codes at that scale. */
int oracle_absmean_ternary(const float *W, int64_t n, int64_t k, int8_t *w, float *scale)
{
    const int64_t total = n * k;
    double sum = 0.0;
    int finite = 1;
    for (int64_t i = 0; i < total; ++i) {
        if (!isfinite(W[i])) {
            finite = 0;
            break;
        }
        sum += fabs((double)W[i]);
    }
    if (!finite || total == 0) {
        for (int64_t i = 0; i < total; ++i) w[i] = 0;
        *scale = 0.0f;
        return finite ? ORACLE_OK : ORACLE_NONFINITE;
    }
    const float s = (float)(sum / (double)total);
    *scale = s;
    oracle_ternary_round(W, total, s, w);
    return ORACLE_OK;
}

/* Position of element k inside a packed row (R2): byte index and bit shift. */
static int64_t code_byte(int64_t k) { return 32 * (k / 128) + (k % 32); }
static int code_shift(int64_t k) { return (int)(2 * ((k % 128) / 32)); }

/* R2/R3 -- 2-bit ternary codes in 128-element groups (technical report §2.2.2;
 * blog post, second postscript: the on-disk format groups 128 elements). */
int oracle_pack(const int8_t *w, int64_t n, int64_t k, uint8_t *packed)
{
    int status = ORACLE_OK;
    const int64_t kb = oracle_blocks(k), rowb = 32 * kb, kpad = 128 * kb;
    for (int64_t r = 0; r < n; ++r) {
        uint8_t *row = packed + r * rowb;
        for (int64_t i = 0; i < rowb; ++i) row[i] = 0;
        for (int64_t i = 0; i < kpad; ++i) {
            int code = 1;                               /* tail: weight 0 */
            if (i < k) {
                int v = w[r * k + i];
                if (v == -1) code = 0;
                else if (v == 0) code = 1;
                else if (v == 1) code = 2;
                else { code = 1; status |= ORACLE_NOT_TERNARY; }
            }
            row[code_byte(i)] |= (uint8_t)(code << code_shift(i));
        }
    }
    return status;
}

static int decode_code(int code) { return code - 1; }  /* R3 */

void oracle_unpack(const uint8_t *packed, int64_t n, int64_t k, int8_t *w)
{
    const int64_t rowb = 32 * oracle_blocks(k);
    for (int64_t r = 0; r < n; ++r)
        for (int64_t i = 0; i < k; ++i) {
            int code = (packed[r * rowb + code_byte(i)] >> code_shift(i)) & 3;
            w[r * k + i] = (int8_t)decode_code(code);
        }
}

/* The misreading the blog post's fourth bug describes: same bytes, read as
 * 64-element groups of 16 bytes.  Used only to show the tests catch it. */
void oracle_unpack_misread64(const uint8_t *packed, int64_t n, int64_t k, int8_t *w)
{
    const int64_t rowb = 32 * oracle_blocks(k);
    for (int64_t r = 0; r < n; ++r)
        for (int64_t i = 0; i < k; ++i) {
            int64_t byte = 16 * (i / 64) + (i % 16);
            int shift = (int)(2 * ((i % 64) / 16));
            int code = (packed[r * rowb + byte] >> shift) & 3;
            w[r * k + i] = (int8_t)decode_code(code);
        }
}

/* R4, integer part -- each 2-bit code is expanded to an INT8 weight and
 * multiplied into an integer sum over K (technical report §2.2.2, §2.4.2,
 * Figure 4). */
int oracle_ternary_matmul(const int8_t *q, int64_t m, const uint8_t *packed,
                          int64_t n, int64_t k, int32_t *acc)
{
    int status = ORACLE_OK;
    const int64_t rowb = 32 * oracle_blocks(k), kpad = oracle_kpad(k);
    for (int64_t r = 0; r < m; ++r)
        for (int64_t c = 0; c < n; ++c) {
            int64_t s = 0;
            for (int64_t i = 0; i < k; ++i) {
                int code = (packed[c * rowb + code_byte(i)] >> code_shift(i)) & 3;
                s += (int64_t)q[r * kpad + i] * (int64_t)decode_code(code);
            }
            if (s > INT32_MAX) { s = INT32_MAX; status |= ORACLE_OVERFLOW; }
            if (s < INT32_MIN) { s = INT32_MIN; status |= ORACLE_OVERFLOW; }
            acc[r * n + c] = (int32_t)s;
        }
    return status;
}

/* R4, fp part: dequantise by the per-token activation scale and the
 * per-tensor weight scale. */
void oracle_dequant(const int32_t *acc, const float *s_act, float s_w,
                    int64_t m, int64_t n, double *y64, float *y32)
{
    for (int64_t r = 0; r < m; ++r)
        for (int64_t c = 0; c < n; ++c) {
            int32_t a = acc[r * n + c];
            if (y64) y64[r * n + c] = (double)a * (double)s_act[r] * (double)s_w;
            if (y32) {
                float t = (float)a * s_act[r];
                y32[r * n + c] = t * s_w;
            }
        }
}

int oracle_linear(const float *x, int64_t m, int64_t k, const uint8_t *packed,
                  int64_t n, float s_w, int32_t *acc, double *y64, float *y32)
{
    const int64_t kpad = oracle_kpad(k);
    int8_t *q = (int8_t *)malloc((size_t)(m * kpad));
    float *sa = (float *)malloc((size_t)m * sizeof(float));
    int32_t *a = acc ? acc : (int32_t *)malloc((size_t)(m * n) * sizeof(int32_t));
    int status = oracle_quant_act(x, m, k, q, sa);
    status |= oracle_ternary_matmul(q, m, packed, n, k, a);
    oracle_dequant(a, sa, s_w, m, n, y64, y32);
    if (!acc) free(a);
    free(q);
    free(sa);
    return status;
}

/* R7 -- I8_S: whole Q_K = 32 blocks per weight row. */
int64_t oracle_i8_row_bytes(int64_t k) { return 32 * ((k + 31) / 32); }

/* R7, integer part -- the plain int8 x int8 dot product over k < K, summed
 * in int64 and checked against the int32 range. */
int oracle_i8_matmul(const int8_t *q, int64_t m, const int8_t *w, int64_t n, int64_t k, int32_t *acc)
{
    int status = ORACLE_OK;
    const int64_t kpad = oracle_kpad(k), rowb = oracle_i8_row_bytes(k);
    for (int64_t r = 0; r < m; ++r)
        for (int64_t c = 0; c < n; ++c) {
            int64_t s = 0;
            for (int64_t i = 0; i < k; ++i) s += (int64_t)q[r * kpad + i] * (int64_t)w[c * rowb + i];
            if (s > INT32_MAX) { s = INT32_MAX; status |= ORACLE_OVERFLOW; }
            if (s < INT32_MIN) { s = INT32_MIN; status |= ORACLE_OVERFLOW; }
            acc[r * n + c] = (int32_t)s;
        }
    return status;
}

int oracle_linear_i8(const float *x, int64_t m, int64_t k, const int8_t *w, int64_t n, float s_w,
                     int32_t *acc, double *y64, float *y32)
{
    const int64_t kpad = oracle_kpad(k);
    int8_t *q = (int8_t *)malloc((size_t)(m * kpad));
    float *sa = (float *)malloc((size_t)m * sizeof(float));
    int32_t *a = acc ? acc : (int32_t *)malloc((size_t)(m * n) * sizeof(int32_t));
    int status = oracle_quant_act(x, m, k, q, sa);
    status |= oracle_i8_matmul(q, m, w, n, k, a);
    oracle_dequant(a, sa, s_w, m, n, y64, y32);
    if (!acc) free(a);
    free(q);
    free(sa);
    return status;
}

/* R6 -- the fused epilogue after the dequantisation, in the order of the
 * technical report's §2.4.1 operator fusion: matrix multiply + bias + ReLU
 * (mul_mat_add_relu), then residual addition with a layer-scale factor
 * (add_scaled):  h = relu(y + bias[c]);  out = residual[r,c] + gamma[c] * h.
 * Each operand is optional (NULL: the step is skipped; relu == 0: no ReLU).
 * The fp32 form rounds every step once (no fused multiply-add); relu(h) is
 * h when h > 0 and +0 otherwise.  The fp64 form applies the same steps to
 * y64 in double precision. */
void oracle_epilogue(const float *bias, const float *gamma, const float *residual, int relu,
                     int64_t m, int64_t n, float *y32, double *y64)
{
    for (int64_t r = 0; r < m; ++r) {
        for (int64_t c = 0; c < n; ++c) {
            const int64_t i = r * n + c;
            if (y32) {
                float h = y32[i];
                if (bias) h = h + bias[c];
                if (relu) h = h > 0.0f ? h : 0.0f;
                if (gamma) h = gamma[c] * h;
                if (residual) h = residual[i] + h;
                y32[i] = h;
            }
            if (y64) {
                double h = y64[i];
                if (bias) h = h + (double)bias[c];
                if (relu) h = h > 0.0 ? h : 0.0;
                if (gamma) h = (double)gamma[c] * h;
                if (residual) h = (double)residual[i] + h;
                y64[i] = h;
            }
        }
    }
}

int oracle_linear_rows(const float *x, int64_t m, int64_t k, const uint8_t *packed,
                       int64_t n, float s_w, const int64_t *idx, int64_t cnt,
                       int32_t *acc, double *y64)
{
    const int64_t kpad = oracle_kpad(k), rowb = 32 * oracle_blocks(k);
    int8_t *q = (int8_t *)malloc((size_t)(m * kpad));
    float *sa = (float *)malloc((size_t)m * sizeof(float));
    int status = oracle_quant_act(x, m, k, q, sa);
    for (int64_t t = 0; t < cnt; ++t) {
        int64_t c = idx[t];
        if (c < 0 || c >= n) continue;
        int32_t a1[1];
        for (int64_t r = 0; r < m; ++r) {
            status |= oracle_ternary_matmul(q + r * kpad, 1, packed + c * rowb, 1, k, a1);
            if (acc) acc[r * cnt + t] = a1[0];
            if (y64) y64[r * cnt + t] = (double)a1[0] * (double)sa[r] * (double)s_w;
        }
    }
    free(q);
    free(sa);
    return status;
}
