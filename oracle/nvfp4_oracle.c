/*
 * nvfp4_oracle.c -- plain CPU reference of the grouped row-scaled NVFP4 cast.
 *
 * TEST INFRASTRUCTURE ONLY: used by the tests, the smoke check and the
 * benchmark's CPU baseline, never by the product path. It is written for a
 * reader checking it against the method's definition, not for speed: scalar
 * loops, one rounding per written float operation, and encoders that pick the
 * nearest representable value from a sorted table of the format's values.
 *
 * Pages cited (see nvfp4_oracle.h for what each one contributes):
 *   [G]  TransformerEngine #3649 "single-launch grouped row-scaled NVFP4 cast",
 *        Description.
 *   [T]  TransformerEngine #2931 "Implement per-token NVFP4 fprop recipe",
 *        Changes; Important Files Changed (dequantize row lookup);
 *        sequence diagram (GEMM with amax = 1, rows multiplied by amax).
 *   [B]  TransformerEngine #3324 "Enable NVFP4 row-scaled (per-token)
 *        backward for GroupedLinear", summary (per-column amax).
 *   [C]  TransformerEngine #3824, "What this changes", item 2 (empty split).
 *
 * Readings where the pages say nothing (every one is a choice of this
 * implementation, pinned by the tests, not taken from the pages):
 *   - the second-level encode scale is 2688/amax with 2688 = 6 * 448 (E2M1
 *     max times E4M3 max); amax == 0 gives 1; an overflowing quotient is
 *     clamped to FLT_MAX. The decode scale is amax/2688.
 *   - the block scale is ((bmax / 6) * S_enc) rounded to E4M3 with round to
 *     nearest even and saturation at 448.
 *   - the element scale is S_enc / e4m3(s8) (0 when s8 == 0, FLT_MAX clamp);
 *     elements are x * that, rounded to E2M1 with ties to the even code,
 *     saturating at 6, sign kept (so -0 and negatives that round to 0 give
 *     code 0x8).
 *   - packing: element 2j in the low nibble of byte j; colwise blocks run
 *     along the row index within the group.
 */
#include "nvfp4_oracle.h"

#include <float.h>
#include <math.h>
#include <string.h>

/* ---------------------------------------------------------------- formats */

float nvo_bf16_to_f32(uint16_t bits) {
  /* bf16 is the upper half of a binary32 word: the conversion is exact */
  uint32_t u = ((uint32_t)bits) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return f;
}

/* E2M1: 1 sign, 2 exponent (bias 1), 1 mantissa bit; no Inf/NaN.
 * exponent field 0 is subnormal: value = m * 0.5 */
float nvo_e2m1_decode(uint8_t code) {
  int s = (code >> 3) & 1;
  int e = (code >> 1) & 3;
  int m = code & 1;
  float mag = (e == 0) ? 0.5f * (float)m : ldexpf(1.0f + 0.5f * (float)m, e - 1);
  return s ? -mag : mag;
}

/* E4M3 "FN" (as used by NVFP4 block scales): 1 sign, 4 exponent (bias 7),
 * 3 mantissa bits; no infinities; exponent 15 with mantissa 7 is NaN;
 * exponent 0 is subnormal: value = m * 2^-9 */
float nvo_e4m3_decode(uint8_t code) {
  int s = (code >> 7) & 1;
  int e = (code >> 3) & 15;
  int m = code & 7;
  float mag;
  if (e == 15 && m == 7) return NAN;
  if (e == 0)
    mag = ldexpf((float)m, -9);
  else
    mag = ldexpf(1.0f + (float)m / 8.0f, e - 7);
  return s ? -mag : mag;
}

/* Nearest entry of an increasing table of non-negative magnitudes, where the
 * table index is the magnitude code. Ties go to the even code (the code whose
 * last mantissa bit is 0); a value above the last entry saturates to it. */
static int nearest_code(const float* table, int n, float a) {
  int c = 0;
  /* largest c with table[c] <= a (table[0] == 0 <= a) */
  while (c + 1 < n && table[c + 1] <= a) c++;
  if (c + 1 == n) return c; /* at or beyond the largest value: saturate */
  double below = (double)a - (double)table[c];
  double above = (double)table[c + 1] - (double)a;
  if (below < above) return c;
  if (above < below) return c + 1;
  return (c % 2 == 0) ? c : c + 1;
}

static float e2m1_table[8];
static float e4m3_table[127]; /* codes 0x00 .. 0x7E, increasing */

/* filled once when the library is loaded, before any caller thread runs */
__attribute__((constructor)) static void make_tables(void) {
  for (int c = 0; c < 8; c++) e2m1_table[c] = nvo_e2m1_decode((uint8_t)c);
  for (int c = 0; c < 127; c++) e4m3_table[c] = nvo_e4m3_decode((uint8_t)c);
}

uint8_t nvo_e2m1_encode(float y) {
  uint8_t sign = signbit(y) ? 0x8 : 0x0;
  return (uint8_t)(sign | nearest_code(e2m1_table, 8, fabsf(y)));
}

uint8_t nvo_e4m3_encode(float v) {
  uint8_t sign = signbit(v) ? 0x80 : 0x00;
  return (uint8_t)(sign | nearest_code(e4m3_table, 127, fabsf(v)));
}

/* --------------------------------------------------------- scale formulas */

/* encode scale S_enc = 6*448 / amax (second-level, FP32) */
float nvo_s_enc(float a) {
  if (a == 0.0f) return 1.0f;
  float q = 2688.0f / a;
  return fminf(q, FLT_MAX);
}

/* decode scale S_dec = amax / (6*448): the factor the GEMM output row is
 * multiplied by once the GEMM ran with amax replaced by 1 ([T], diagram) */
float nvo_s_dec(float a) { return a / 2688.0f; }

void nvo_block_encode(const float* x16, float s_enc, uint8_t* s8, uint8_t* codes16) {
  float bmax = 0.0f;
  for (int j = 0; j < 16; j++) {
    float ax = fabsf(x16[j]);
    if (ax > bmax) bmax = ax;
  }
  float t = bmax / 6.0f;
  float s32 = t * s_enc;
  uint8_t sc = nvo_e4m3_encode(s32);
  float enc = 0.0f;
  if (sc != 0) {
    float q = s_enc / nvo_e4m3_decode(sc);
    enc = fminf(q, FLT_MAX);
  }
  for (int j = 0; j < 16; j++) {
    float y = x16[j] * enc;
    codes16[j] = nvo_e2m1_encode(y);
  }
  *s8 = sc;
}

/* ------------------------------------------------------------- validation */

static int check_splits(int64_t sum_M, int64_t K, const int64_t* m_splits, int32_t E,
                        int need_m16) {
  if (sum_M < 0 || K < 0 || E < 0 || (K % 16) != 0) return NVO_E_ARG;
  if (E > 0 && m_splits == NULL) return NVO_E_ARG;
  int64_t total = 0;
  for (int32_t g = 0; g < E; g++) {
    if (m_splits[g] < 0) return NVO_E_ARG;
    if (need_m16 && (m_splits[g] % 16) != 0) return NVO_E_ARG;
    total += m_splits[g];
  }
  if (total != sum_M) return NVO_E_ARG;
  return NVO_OK;
}

static int check_finite(const uint16_t* x, int64_t n) {
  for (int64_t i = 0; i < n; i++)
    if (!isfinite(nvo_bf16_to_f32(x[i]))) return NVO_E_NONFINITE;
  return NVO_OK;
}

/* ------------------------------------------------------------ grouped amax */

/* [G] grouped amax: row_amax[r] = max_k |x[r,k]|;
 * col_amax[g*K+k] = max over the rows r of group g of |x[r,k]|;
 * an empty group keeps 0 ([C]). */
int nvo_group_amax(const uint16_t* x, int64_t sum_M, int64_t K,
                   const int64_t* m_splits, int32_t E,
                   float* row_amax, float* col_amax) {
  int rc = check_splits(sum_M, K, m_splits, E, 0);
  if (rc) return rc;
  if (sum_M * K > 0 && x == NULL) return NVO_E_ARG;
  rc = check_finite(x, sum_M * K);
  if (rc) return rc;

  if (row_amax != NULL) {
    for (int64_t r = 0; r < sum_M; r++) {
      float m = 0.0f;
      for (int64_t k = 0; k < K; k++) {
        float a = fabsf(nvo_bf16_to_f32(x[r * K + k]));
        if (a > m) m = a;
      }
      row_amax[r] = m;
    }
  }
  if (col_amax != NULL) {
    int64_t o = 0;
    for (int32_t g = 0; g < E; g++) {
      for (int64_t k = 0; k < K; k++) {
        float m = 0.0f;
        for (int64_t r = o; r < o + m_splits[g]; r++) {
          float a = fabsf(nvo_bf16_to_f32(x[r * K + k]));
          if (a > m) m = a;
        }
        col_amax[(int64_t)g * K + k] = m;
      }
      o += m_splits[g];
    }
  }
  return NVO_OK;
}

/* ------------------------------------------------------------ grouped cast */

/* [G] grouped cast + [T] per-token scaling: rowwise blocks run along K and
 * use the row's amax; colwise blocks run along the rows of one group and use
 * that group's column amax ([B]). */
int nvo_group_cast(const uint16_t* x, int64_t sum_M, int64_t K,
                   const int64_t* m_splits, int32_t E,
                   const float* row_amax, const float* col_amax,
                   uint8_t* row_data, uint8_t* row_scale, float* row_s2,
                   uint8_t* col_data, uint8_t* col_scale, float* col_s2) {
  int do_row = (row_data != NULL || row_scale != NULL || row_s2 != NULL);
  int do_col = (col_data != NULL || col_scale != NULL || col_s2 != NULL);
  if (do_row && (row_data == NULL || row_scale == NULL || row_s2 == NULL || row_amax == NULL))
    return NVO_E_ARG;
  if (do_col && (col_data == NULL || col_scale == NULL || col_s2 == NULL || col_amax == NULL))
    return NVO_E_ARG;
  int rc = check_splits(sum_M, K, m_splits, E, do_col);
  if (rc) return rc;
  if (sum_M * K > 0 && x == NULL) return NVO_E_ARG;
  rc = check_finite(x, sum_M * K);
  if (rc) return rc;

  float blk[16];
  uint8_t codes[16];
  uint8_t s8;

  if (do_row) {
    for (int64_t r = 0; r < sum_M; r++) {
      float s_enc = nvo_s_enc(row_amax[r]);
      row_s2[r] = nvo_s_dec(row_amax[r]);
      for (int64_t b = 0; b < K / 16; b++) {
        for (int j = 0; j < 16; j++) blk[j] = nvo_bf16_to_f32(x[r * K + 16 * b + j]);
        nvo_block_encode(blk, s_enc, &s8, codes);
        row_scale[r * (K / 16) + b] = s8;
        for (int j = 0; j < 8; j++)
          row_data[r * (K / 2) + 8 * b + j] =
              (uint8_t)(codes[2 * j] | (codes[2 * j + 1] << 4));
      }
    }
  }

  if (do_col) {
    int64_t o = 0;
    for (int32_t g = 0; g < E; g++) {
      int64_t m = m_splits[g];
      uint8_t* gdata = col_data + K * o / 2;   /* [K, m/2] */
      uint8_t* gscale = col_scale + K * o / 16; /* [K, m/16] */
      for (int64_t k = 0; k < K; k++) {
        float a = col_amax[(int64_t)g * K + k];
        float s_enc = nvo_s_enc(a);
        col_s2[(int64_t)g * K + k] = nvo_s_dec(a);
        for (int64_t b = 0; b < m / 16; b++) {
          for (int j = 0; j < 16; j++) blk[j] = nvo_bf16_to_f32(x[(o + 16 * b + j) * K + k]);
          nvo_block_encode(blk, s_enc, &s8, codes);
          gscale[k * (m / 16) + b] = s8;
          for (int j = 0; j < 8; j++)
            gdata[k * (m / 2) + 8 * b + j] = (uint8_t)(codes[2 * j] | (codes[2 * j + 1] << 4));
        }
      }
      o += m;
    }
  }
  return NVO_OK;
}

/* -------------------------------------------------------------- dequantize */

/* [T] dequantize with the per-row amax lookup: x_hat = (e2m1(code) *
 * e4m3(s8)) * s2[row]. The first product is exact (at most 6 significant
 * bits), so one rounding happens, in the multiply by s2. */
int nvo_dequantize(const uint8_t* data, const uint8_t* scale, const float* s2,
                   int64_t rows, int64_t cols, float* out) {
  if (rows < 0 || cols < 0 || (cols % 16) != 0) return NVO_E_ARG;
  if (rows * cols > 0 && (data == NULL || scale == NULL || s2 == NULL || out == NULL))
    return NVO_E_ARG;
  for (int64_t r = 0; r < rows; r++) {
    for (int64_t c = 0; c < cols; c++) {
      uint8_t byte = data[r * (cols / 2) + c / 2];
      uint8_t code = (c % 2 == 0) ? (byte & 0xF) : (byte >> 4);
      float q = nvo_e2m1_decode(code) * nvo_e4m3_decode(scale[r * (cols / 16) + c / 16]);
      out[r * cols + c] = q * s2[r];
    }
  }
  return NVO_OK;
}

/* ------------------------------------------------------------------- MXFP4 */

/* [T] E8M0: an exponent byte with bias 127, no sign, no mantissa */
float nvo_e8m0_decode(uint8_t code) {
  if (code == 0xFF) return NAN;
  return ldexpf(1.0f, (int)code - 127);
}

/* [T] one block of 32: the shared exponent from the block amax (frexp gives
 * a = m * 2^k with m in [0.5, 1), so floor(log2 a) = k - 1 exactly), then
 * every element scaled by the power of two and encoded */
void nvo_mx_block_encode(const float* x32, uint8_t* e8m0, uint8_t* codes32) {
  float a = 0.0f;
  for (int i = 0; i < 32; i++) {
    const float m = fabsf(x32[i]);
    if (m > a) a = m;
  }
  int s = -127;
  if (a > 0.0f) {
    int k;
    frexpf(a, &k);
    s = (k - 1) - 2;
    if (s < -127) s = -127;
    if (s > 127) s = 127;
  }
  *e8m0 = (uint8_t)(s + 127);
  for (int i = 0; i < 32; i++) codes32[i] = nvo_e2m1_encode(ldexpf(x32[i], -s));
}

int nvo_mx_group_cast(const uint16_t* x, int64_t sum_M, int64_t K, const int64_t* m_splits, int32_t E,
                      uint8_t* row_data, uint8_t* row_scale, uint8_t* col_data, uint8_t* col_scale) {
  if (sum_M < 0 || K < 0 || E < 0 || (K % 32) != 0) return NVO_E_ARG;
  if (E > 0 && m_splits == NULL) return NVO_E_ARG;
  const int do_row = row_data != NULL || row_scale != NULL;
  const int do_col = col_data != NULL || col_scale != NULL;
  int64_t total = 0;
  for (int32_t g = 0; g < E; g++) {
    if (m_splits[g] < 0 || (do_col && (m_splits[g] % 32) != 0)) return NVO_E_ARG;
    total += m_splits[g];
  }
  if (total != sum_M) return NVO_E_ARG;
  if (sum_M * K > 0 && x == NULL) return NVO_E_ARG;
  if (do_row && sum_M * K > 0 && (row_data == NULL || row_scale == NULL)) return NVO_E_ARG;
  if (do_col && sum_M * K > 0 && (col_data == NULL || col_scale == NULL)) return NVO_E_ARG;
  for (int64_t i = 0; i < sum_M * K; i++)
    if (!isfinite(nvo_bf16_to_f32(x[i]))) return NVO_E_NONFINITE;
  float blk[32];
  uint8_t codes[32];
  if (do_row) {
    for (int64_t r = 0; r < sum_M; r++) {
      for (int64_t b = 0; b < K / 32; b++) {
        for (int i = 0; i < 32; i++) blk[i] = nvo_bf16_to_f32(x[r * K + b * 32 + i]);
        nvo_mx_block_encode(blk, &row_scale[r * (K / 32) + b], codes);
        for (int i = 0; i < 32; i += 2)
          row_data[r * (K / 2) + b * 16 + i / 2] = (uint8_t)(codes[i] | (codes[i + 1] << 4));
      }
    }
  }
  if (do_col) {
    int64_t o = 0;
    for (int32_t g = 0; g < E; g++) {
      const int64_t m = m_splits[g];
      uint8_t* cd = col_data + K * o / 2;
      uint8_t* cs = col_scale + K * o / 32;
      for (int64_t k = 0; k < K; k++) {
        for (int64_t b = 0; b < m / 32; b++) {
          for (int i = 0; i < 32; i++) blk[i] = nvo_bf16_to_f32(x[(o + b * 32 + i) * K + k]);
          nvo_mx_block_encode(blk, &cs[k * (m / 32) + b], codes);
          for (int i = 0; i < 32; i += 2) cd[k * (m / 2) + b * 16 + i / 2] = (uint8_t)(codes[i] | (codes[i + 1] << 4));
        }
      }
      o += m;
    }
  }
  return NVO_OK;
}

int nvo_mx_dequantize(const uint8_t* data, const uint8_t* scale, int64_t rows, int64_t cols, float* out) {
  if (rows < 0 || cols < 0 || (cols % 32) != 0) return NVO_E_ARG;
  if (rows * cols > 0 && (data == NULL || scale == NULL || out == NULL)) return NVO_E_ARG;
  for (int64_t r = 0; r < rows; r++) {
    for (int64_t c = 0; c < cols; c++) {
      const uint8_t byte = data[r * (cols / 2) + c / 2];
      const uint8_t code = (uint8_t)((byte >> (4 * (c % 2))) & 0xF); /* element 2j: low nibble */
      out[r * cols + c] = nvo_e2m1_decode(code) * nvo_e8m0_decode(scale[r * (cols / 32) + c / 32]);
    }
  }
  return NVO_OK;
}

/* ------------------------------------------------ consumer side of the cast */

/* [T] the 128x4-tiled scale layout, written straight from its index map */
int nvo_swizzle_scales_128x4(const uint8_t* scale, int64_t rows, int64_t cols, uint8_t* out) {
  if (rows < 0 || cols < 0) return NVO_E_ARG;
  const int64_t row_tiles = (rows + 127) / 128, col_tiles = (cols + 3) / 4;
  if (row_tiles * col_tiles > 0 && out == NULL) return NVO_E_ARG;
  if (rows * cols > 0 && scale == NULL) return NVO_E_ARG;
  for (int64_t i = 0; i < row_tiles * col_tiles * 512; i++) out[i] = 0;
  for (int64_t r = 0; r < rows; r++) {
    for (int64_t c = 0; c < cols; c++) {
      const int64_t tile = (r / 128) * col_tiles + (c / 4);
      const int64_t rr = r % 128, cc = c % 4;
      out[tile * 512 + (rr % 32) * 16 + (rr / 32) * 4 + cc] = scale[r * cols + c];
    }
  }
  return NVO_OK;
}

/* [T] round to nearest even on the 16 bits that are dropped: add half an
 * ulp of the result, less one unless the kept part is odd, and truncate */
uint16_t nvo_f32_to_bf16(float v) {
  uint32_t b;
  memcpy(&b, &v, sizeof b);
  if ((b & 0x7F800000u) == 0x7F800000u && (b & 0x007FFFFFu) != 0u)
    return (uint16_t)((b >> 16) | 0x0040u); /* NaN: keep it a (quiet) NaN */
  b += 0x7FFFu + ((b >> 16) & 1u);
  return (uint16_t)(b >> 16);
}

/* [T] post-GEMM row scaling, one rounding per operation */
int nvo_row_post_scale(const float* in, int64_t rows, int64_t cols, const float* amax,
                       const float* bias, float* out_f32, uint16_t* out_bf16) {
  if (rows < 0 || cols < 0) return NVO_E_ARG;
  if (rows * cols > 0 && (in == NULL || amax == NULL)) return NVO_E_ARG;
  for (int64_t r = 0; r < rows; r++) {
    for (int64_t c = 0; c < cols; c++) {
      float y = in[r * cols + c] * amax[r];
      if (bias != NULL) y = y + bias[c];
      if (out_f32 != NULL) out_f32[r * cols + c] = y;
      if (out_bf16 != NULL) out_bf16[r * cols + c] = nvo_f32_to_bf16(y);
    }
  }
  return NVO_OK;
}

/* --------------------------------------------- array forms for the tests */

void nvo_e2m1_encode_array(const float* y, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; i++) out[i] = nvo_e2m1_encode(y[i]);
}

void nvo_e4m3_encode_array(const float* v, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; i++) out[i] = nvo_e4m3_encode(v[i]);
}
