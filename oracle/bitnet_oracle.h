/*
 * bitnet_oracle.h -- plain, slow, single-threaded CPU oracle for the I2_S
 * ternary linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may include, link or
 * call this code: only the test suite, the smoke check and the benchmark's CPU
 * baseline leg use it.  It shares no header, helper, table or constant with the
 * CUDA library; it is written from the method's definition:
 *
 *   "VibeVoice-ASR-BitNet Technical Report", §2.2.2 (I2_S: ternary weights
 *   {-1,0,+1} stored in 2 bits, activations quantised to INT8 online per token,
 *   unpack-to-INT8 then multiply-add) and §2.4.2 (I2_S kernel block size Q_K);
 *   the ARM debugging blog post "Paper 說支援 ARM，我大概是第一個真的去編譯的人",
 *   second postscript (the file format groups 128 elements; decoding it with a
 *   64-element layout shuffles every weight matrix).
 *
 * Readings of points the pages leave open (each stated once, here):
 *  R1 activation quantiser (per token m, fp32 arithmetic, no FMA contraction):
 *       amax = max_k |x[m,k]|;  a row holding NaN/Inf is "non-finite": its codes
 *       and scale are 0 and ORACLE_NONFINITE is reported;  amax == 0 gives codes
 *       0 and scale 0;  otherwise inv = 127/amax (IEEE divide), and for each k
 *       q = 0 when x == 0, else clamp(rint(x*inv), -127, 127) with rint rounding
 *       half to even;  scale = amax/127.  -128 is never produced.
 *  R2 packed layout: row n of a weight matrix [N,K] occupies 32*ceil(K/128)
 *       bytes; element k = 128*j + 32*g + b (g in 0..3, b in 0..31) is stored in
 *       byte 32*j + b of the row at bits [2g, 2g+1].
 *  R3 code = w + 1 (0 -> -1, 1 -> 0, 2 -> +1; 3 is never written), positions
 *       k >= K of the last block hold code 1 (weight 0).
 *  R4 linear: acc[m,n] = sum_{k<K} q[m,k]*w[n,k], exact integer;
 *       y[m,n] = acc[m,n] * s_act[m] * s_w evaluated in fp64 (the oracle's
 *       reference value); the fp32 form ((float)acc*s_act)*s_w is also given.
 *  R5 absmean weight quantiser (the ternary weights of §2.2.2 come from a
 *       full-precision tensor by the BitNet b1.58 recipe the report cites but
 *       does not print; plainest reading): scale = mean over all n*k elements
 *       of |W|, summed in fp64 and rounded once to fp32; w = clamp(rint(W /
 *       scale), -1, 1) with the division and the rounding in fp32 (rounding
 *       half to even).  An all-zero tensor gives scale 0 and w = 0; a tensor
 *       holding NaN/Inf gives scale 0, w = 0 and ORACLE_NONFINITE.
 *  R6 fused epilogue (§2.4.1 operator fusion: multiply + bias + ReLU, then
 *       residual addition with a layer scale): h = relu(y + bias);
 *       out = residual + gamma * h; one fp32 rounding per step.
 *  R7 I8_S linear (§2.2.1 full-pipeline INT8; §2.4.2: the I8_S kernel works
 *       on blocks of Q_K = 32 elements and shares the maddubs multiply-add
 *       pipeline with I2_S, using the sign trick for signed x signed):
 *       weights are plain int8 [N, K] with one fp32 scale per tensor, each
 *       row stored in 32*ceil(K/32) bytes (whole Q_K blocks, pads 0);
 *       activations as R1; acc[m,n] = sum_{k<K} q[m,k]*w[n,k], exact integer
 *       (the sign trick |w| * (sign(w) x) gives the same products);
 *       y = acc * s_act * s_w as in R4, where (float)acc now rounds to
 *       nearest even when |acc| > 2^24.
 */
#ifndef BITNET_ORACLE_H
#define BITNET_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* status bits returned by the oracle functions */
#define ORACLE_OK          0
#define ORACLE_NONFINITE   1   /* a row of x held NaN or Inf (R1)          */
#define ORACLE_NOT_TERNARY 2   /* a weight outside {-1,0,+1} was given      */
#define ORACLE_OVERFLOW    4   /* an accumulator left the int32 range       */

/* ceil(K/128) and the padded width 128*ceil(K/128) */
int64_t oracle_blocks(int64_t k);
int64_t oracle_kpad(int64_t k);

/* R7: bytes of one I8_S weight row, 32*ceil(K/32) */
int64_t oracle_i8_row_bytes(int64_t k);

/* R7, integer part: acc [m,n] from quantised q [m, kpad] (R1 layout) and
 * int8 weights w [n, oracle_i8_row_bytes(k)]; only k < K is read.
 * Returns ORACLE_OVERFLOW if a sum leaves the int32 range. */
int oracle_i8_matmul(const int8_t *q, int64_t m, const int8_t *w, int64_t n, int64_t k, int32_t *acc);

/* R7, whole layer: quantise x (R1), contract with the int8 weights, and
 * dequantise (R4's two forms); acc may be NULL. */
int oracle_linear_i8(const float *x, int64_t m, int64_t k, const int8_t *w, int64_t n, float s_w,
                     int32_t *acc, double *y64, float *y32);

/* R1: x fp32 [m,k] -> q int8 [m, kpad] (pads zero), s_act fp32 [m].
 * Returns ORACLE_NONFINITE if any row was non-finite. */
int oracle_quant_act(const float *x, int64_t m, int64_t k, int8_t *q, float *s_act);

/* R2/R3: w int8 [n,k] -> packed [n, 32*blocks].  A value outside {-1,0,+1}
 * is stored as weight 0 and ORACLE_NOT_TERNARY is returned. */
int oracle_pack(const int8_t *w, int64_t n, int64_t k, uint8_t *packed);

/* R5: W fp32 [n,k] -> ternary w int8 [n,k] and the per-tensor scale.
 * Returns ORACLE_NONFINITE if W held NaN or Inf. */
/* R5, second pass: codes clamp(rint(W / s), -1, 1) for a given fp32 scale s
 * (fp32 quotient, half to even); s == 0 gives 0 everywhere. */
void oracle_ternary_round(const float *W, int64_t total, float s, int8_t *w);
int oracle_absmean_ternary(const float *W, int64_t n, int64_t k, int8_t *w, float *scale);

/* Inverse of oracle_pack: packed [n, 32*blocks] -> w int8 [n,k]. */
void oracle_unpack(const uint8_t *packed, int64_t n, int64_t k, int8_t *w);

/* PLANTED MISTAKE, for the mutation test only: decodes the same bytes as if
 * the format grouped 64 elements per 16 bytes (element k = 64*j + 16*g + b in
 * byte 16*j + b, bits 2g) -- the misreading the ARM blog post reports. */
void oracle_unpack_misread64(const uint8_t *packed, int64_t n, int64_t k, int8_t *w);

/* R4, integer part: acc [m,n] from quantised q [m, kpad] and packed weights.
 * Decodes each weight from its 2-bit code element by element.
 * Returns ORACLE_OVERFLOW if a sum does not fit int32 (then acc is clamped). */
int oracle_ternary_matmul(const int8_t *q, int64_t m, const uint8_t *packed,
                          int64_t n, int64_t k, int32_t *acc);

/* R4, fp part: y64 = acc*s_act*s_w in fp64; y32 = ((float)acc*s_act)*s_w in
 * fp32 (either pointer may be NULL). */
void oracle_dequant(const int32_t *acc, const float *s_act, float s_w,
                    int64_t m, int64_t n, double *y64, float *y32);

/* Whole layer: quantise x, multiply, dequantise.  acc/y32/y64 may be NULL. */
int oracle_linear(const float *x, int64_t m, int64_t k, const uint8_t *packed,
                  int64_t n, float s_w, int32_t *acc, double *y64, float *y32);

/* R6 -- fused epilogue applied in place to a layer's outputs (fp32 form y32
 * and/or fp64 form y64, each [m, n]; either may be NULL):
 *   h = relu(y + bias[c]);  out = residual[r, c] + gamma[c] * h
 * bias, gamma [n] and residual [m, n] may each be NULL (step skipped);
 * relu != 0 applies h > 0 ? h : +0. */
void oracle_epilogue(const float *bias, const float *gamma, const float *residual, int relu,
                     int64_t m, int64_t n, float *y32, double *y64);

/* Sampled outputs of one layer: only the rows listed in idx[0..cnt) of the
 * weight matrix are computed; acc/y64 are [m, cnt]. */
int oracle_linear_rows(const float *x, int64_t m, int64_t k, const uint8_t *packed,
                       int64_t n, float s_w, const int64_t *idx, int64_t cnt,
                       int32_t *acc, double *y64);

#ifdef __cplusplus
}
#endif
#endif
