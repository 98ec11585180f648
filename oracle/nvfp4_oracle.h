/*
 * nvfp4_oracle.h -- plain CPU reference of the grouped row-scaled NVFP4 cast.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may include, link or
 * call this file: only the tests, the smoke check and the benchmark's CPU
 * baseline use it. It shares no code with the CUDA library.
 *
 * Sources (web pages the method is taken from):
 *  - TransformerEngine #3649, "single-launch grouped row-scaled NVFP4 cast",
 *    Description: a grouped amax over the packed (sum_M, K) buffer yields
 *    rowwise [sum_M] and columnwise [num_tensors*K] amax in one pass; a
 *    grouped cast consumes both and writes packed FP4 data and scales.
 *  - TransformerEngine #2931, "Implement per-token NVFP4 fprop recipe",
 *    Changes and sequence diagram: per-token (row) amax as the FP32
 *    second-level scale, FP8 (E4M3) block scales, FP4 data; dequantize looks
 *    up the amax of the element's row; the GEMM runs with amax = 1 and its
 *    rows are multiplied back by the row amax.
 *  - TransformerEngine #3324, "Enable NVFP4 row-scaled (per-token) backward
 *    for GroupedLinear", summary: per-column amax for the columnwise operand.
 *  - TransformerEngine #3824, "What this changes", item 2: a 0-element split
 *    must not fail.
 *
 * All floating point is IEEE-754 binary32, round to nearest even, one
 * rounding per written operation (the translation unit is compiled with
 * -ffp-contract=off on SSE). Return values: 0 = ok, nonzero = error (see
 * NVO_E_* below).
 */
#ifndef NVFP4_ORACLE_H
#define NVFP4_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define NVO_OK 0
#define NVO_E_ARG 1        /* bad size, split or pointer */
#define NVO_E_NONFINITE 2  /* an input element is Inf or NaN */

/* format helpers */
float nvo_bf16_to_f32(uint16_t bits);
float nvo_e2m1_decode(uint8_t code);          /* low 4 bits used */
uint8_t nvo_e2m1_encode(float y);             /* RNE onto E2M1, saturating */
float nvo_e4m3_decode(uint8_t code);          /* E4M3 "FN": NaN for 0x7F/0xFF */
uint8_t nvo_e4m3_encode(float v);             /* RNE onto E4M3, saturating */

/* element-wise array forms of the two encoders (test helpers) */
void nvo_e2m1_encode_array(const float* y, int64_t n, uint8_t* out);
void nvo_e4m3_encode_array(const float* v, int64_t n, uint8_t* out);

/* second-level scales of one amax value a */
float nvo_s_enc(float a);
float nvo_s_dec(float a);

/* one 16-element block: block scale byte and 16 codes (one per element) */
void nvo_block_encode(const float* x16, float s_enc, uint8_t* s8, uint8_t* codes16);

/* grouped amax (both directions). row_amax [sum_M], col_amax [E*K];
 * either output may be NULL to skip that direction. */
int nvo_group_amax(const uint16_t* x, int64_t sum_M, int64_t K,
                   const int64_t* m_splits, int32_t E,
                   float* row_amax, float* col_amax);

/* grouped cast. Rowwise outputs: row_data [sum_M, K/2], row_scale
 * [sum_M, K/16], row_s2 [sum_M]. Colwise outputs: per group g a transposed
 * slice, col_data at byte K*o_g/2 of shape [K, m_g/2], col_scale at byte
 * K*o_g/16 of shape [K, m_g/16], col_s2 [E*K]. A direction whose three
 * pointers are NULL is skipped. */
int nvo_group_cast(const uint16_t* x, int64_t sum_M, int64_t K,
                   const int64_t* m_splits, int32_t E,
                   const float* row_amax, const float* col_amax,
                   uint8_t* row_data, uint8_t* row_scale, float* row_s2,
                   uint8_t* col_data, uint8_t* col_scale, float* col_s2);

/* dequantize one row-major quantized matrix [rows, cols] with one s2 per row */
int nvo_dequantize(const uint8_t* data, const uint8_t* scale, const float* s2,
                   int64_t rows, int64_t cols, float* out);

/* ------------------------------------------------ consumer side of the cast */

/* The 128x4-tiled scale layout that block-scaled grouped GEMMs read (the
 * "swizzle contract" of "[NVFP4 4over6] Add the grouped-experts four-over-six
 * converter" (torchtitan #14), Design notes, which needs 128-row-aligned
 * token groups; TransformerEngine #3649's review asks the same alignment of
 * uniform expert sizes). The pages do not print the layout. Reading: the
 * scale matrix [rows, cols] is
 * cut into tiles of 128 rows x 4 columns (zero padded at the edges), stored
 * one after another in row-major tile order, 512 bytes each; inside a tile,
 * element (r, c) sits at byte (r % 32) * 16 + (r / 32) * 4 + c. out holds
 * ceil(rows/128)*128 * ceil(cols/4)*4 bytes. */
int nvo_swizzle_scales_128x4(const uint8_t* scale, int64_t rows, int64_t cols, uint8_t* out);

/* ------------------------------------------------------------- MXFP4 */

/* MXFP4: E2M1 data in blocks of 32 elements with one E8M0 (power-of-two)
 * scale each and no second-level scale (TransformerEngine #3824, Testing and
 * item 1: the "E2M1/block-32/E8M0" pow_2_scales configuration; row-scaled
 * NVFP4 is not combined with it). The pages do not spell out the scale
 * rule; reading (the OCP Microscaling conversion): with a = max |x| of the
 * block, the shared exponent is s = floor(log2 a) - 2 (2 = exponent of
 * E2M1's largest value, 6 = 1.5 * 2^2), clamped to [-127, 127] (a = 0 gives
 * -127); the scale byte is s + 127; each element encodes as
 * E2M1_rne_satfinite(x * 2^-s) (exact multiply; values past 6 saturate). */
float nvo_e8m0_decode(uint8_t code);  /* 2^(code-127); NaN for 0xFF */
void nvo_mx_block_encode(const float* x32, uint8_t* e8m0, uint8_t* codes32);

/* grouped MXFP4 cast: rowwise row_data [sum_M, K/2], row_scale [sum_M, K/32];
 * colwise per group g col_data at byte K*o_g/2 of shape [K, m_g/2] and
 * col_scale at byte K*o_g/32 of shape [K, m_g/32]. K % 32 == 0, and for the
 * colwise direction every m_g % 32 == 0. A direction whose two pointers are
 * NULL is skipped. */
int nvo_mx_group_cast(const uint16_t* x, int64_t sum_M, int64_t K, const int64_t* m_splits, int32_t E,
                      uint8_t* row_data, uint8_t* row_scale, uint8_t* col_data, uint8_t* col_scale);

/* x_hat = e2m1(code) * 2^(scale-127), one row-major matrix [rows, cols] */
int nvo_mx_dequantize(const uint8_t* data, const uint8_t* scale, int64_t rows, int64_t cols, float* out);

/* IEEE binary32 -> bfloat16 bits, round to nearest even (NaN stays NaN). */
uint16_t nvo_f32_to_bf16(float v);

/* The FP32 post-scale after a GEMM run with the row amax replaced by ones
 * (TransformerEngine #2931, sequence diagram: the output rows are multiplied
 * by the row-wise scales, then converted to the target dtype; the bias is
 * taken out before and added back after). y[r][c] = fl(in[r][c] * amax[r]),
 * then, with a bias, fl(y + bias[c]). out_f32 and out_bf16 (RNE of y) may
 * each be NULL; bias may be NULL. */
int nvo_row_post_scale(const float* in, int64_t rows, int64_t cols, const float* amax,
                       const float* bias, float* out_f32, uint16_t* out_bf16);

#ifdef __cplusplus
}
#endif

#endif
