// codec.cuh -- device helpers of the NVFP4 encoding on sm_100a.
//
// NVFP4 as the per-token recipe uses it (TransformerEngine #2931, "Implement
// per-token NVFP4 fprop recipe", Changes): E2M1 element codes packed two per
// byte, one E4M3 scale per 16-element block, and an FP32 second-level scale
// taken from the amax of the element's row (or, for the transposed operand,
// of its column within the group). Every float operation here is a single
// IEEE binary32 operation rounded to nearest even: the translation unit is
// built with --fmad=false, and the divides and multiplies below are the _rn
// intrinsics. The conversions to E2M1 / E4M3 are the hardware's
// round-to-nearest-even, saturating converts.
#pragma once

#include <cfloat>
#include <cstdint>

namespace nvfp4rs {

// ----------------------------------------------------------------- bf16 max

// Packed |a|,|b| maximum of two bf16x2 words: the magnitude of each half is
// max(|a_i|, |b_i|); the sign bit is meaningless and is cleared by the caller.
__device__ __forceinline__ uint32_t maxabs2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Per-half unsigned maximum; for sign-cleared bf16 bit patterns this is the
// float maximum.
__device__ __forceinline__ uint32_t umax2(uint32_t a, uint32_t b) { return __vmaxu2(a, b); }

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// bf16 halves of a word as fp32 (exact)
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// ------------------------------------------------------- second-level scale

// S_enc(a) = 6*448 / a, 1 for a == 0, clamped to FLT_MAX when it overflows
__device__ __forceinline__ float s_enc_of(float a) {
  return a == 0.0f ? 1.0f : fminf(__fdiv_rn(2688.0f, a), FLT_MAX);
}
// S_dec(a) = a / (6*448)
__device__ __forceinline__ float s_dec_of(float a) { return __fdiv_rn(a, 2688.0f); }

// --------------------------------------------------------------- E4M3 scale

// two fp32 -> two E4M3 bytes (RNE, saturating); `hi` lands in bits 8..15
__device__ __forceinline__ uint32_t e4m3x2(float hi, float lo) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// two E4M3 bytes (bits 0..7 and 8..15) -> fp32 values (exact)
__device__ __forceinline__ void e4m3x2_to_f32(uint32_t pair, float& lo, float& hi) {
  uint32_t h2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(static_cast<uint16_t>(pair)));
  asm("{.reg .f16 l, h;\n\t"
      "mov.b32 {l, h}, %2;\n\t"
      "cvt.f32.f16 %0, l;\n\t"
      "cvt.f32.f16 %1, h;}"
      : "=f"(lo), "=f"(hi) : "r"(h2));
}

// Block scales of two 16-element blocks with maxima bm0 / bm1 and encode
// scales se0 / se1: returns the two E4M3 bytes (block 0 in bits 0..7) and
// the element multipliers enc = S_enc / e4m3(s8), 0 when s8 == 0.
__device__ __forceinline__ uint32_t block_scales2(float bm0, float se0, float bm1, float se1,
                                                  float& enc0, float& enc1) {
  const float s0 = __fmul_rn(__fdiv_rn(bm0, 6.0f), se0);
  const float s1 = __fmul_rn(__fdiv_rn(bm1, 6.0f), se1);
  const uint32_t p = e4m3x2(s1, s0);
  float v0, v1;
  e4m3x2_to_f32(p, v0, v1);
  const float q0 = fminf(__fdiv_rn(se0, v0), FLT_MAX);
  const float q1 = fminf(__fdiv_rn(se1, v1), FLT_MAX);
  enc0 = (p & 0xFFu) ? q0 : 0.0f;
  enc1 = (p & 0xFF00u) ? q1 : 0.0f;
  return p;
}

// ------------------------------------------------------------- E2M1 codes

// d = (a0 * b0, a1 * b1), one IEEE multiply per lane (packed on sm_100a)
__device__ __forceinline__ void mul2(float a0, float a1, float b0, float b1, float& d0, float& d1) {
  asm("{.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\t"
      "mov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\t"
      "mov.b64 {%0, %1}, rd;}"
      : "=f"(d0), "=f"(d1) : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

// Eight fp32 values -> one word of eight E2M1 codes; value 2j in the low
// nibble of byte j (RNE, saturating at 6, sign kept).
__device__ __forceinline__ uint32_t e2m1x8(float v0, float v1, float v2, float v3, float v4,
                                           float v5, float v6, float v7) {
  uint32_t r;
  asm("{.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};}"
      : "=r"(r)
      : "f"(v0), "f"(v1), "f"(v2), "f"(v3), "f"(v4), "f"(v5), "f"(v6), "f"(v7));
  return r;
}

// Four pairs (lo_i, hi_i) -> one word whose byte i holds the pair's two
// codes (lo_i in the low nibble).
__device__ __forceinline__ uint32_t e2m1x2x4(float lo0, float hi0, float lo1, float hi1,
                                             float lo2, float hi2, float lo3, float hi3) {
  return e2m1x8(lo0, hi0, lo1, hi1, lo2, hi2, lo3, hi3);
}

// Row encode of eight bf16 (one 16-byte chunk = four words) with one
// multiplier: the packed codes of the chunk.
__device__ __forceinline__ uint32_t encode_chunk(const uint4& w, float enc) {
  float y0, y1, y2, y3, y4, y5, y6, y7;
  mul2(bf16lo(w.x), bf16hi(w.x), enc, enc, y0, y1);
  mul2(bf16lo(w.y), bf16hi(w.y), enc, enc, y2, y3);
  mul2(bf16lo(w.z), bf16hi(w.z), enc, enc, y4, y5);
  mul2(bf16lo(w.w), bf16hi(w.w), enc, enc, y6, y7);
  return e2m1x8(y0, y1, y2, y3, y4, y5, y6, y7);
}

// --------------------------------------------------------------- decoding

// one word of eight E2M1 codes -> eight fp32 values (exact)
__device__ __forceinline__ void e2m1x8_to_f32(uint32_t w, float (&v)[8]) {
  uint32_t h0, h1, h2, h3;
  asm("{.reg .b8 b0, b1, b2, b3;\n\t"
      "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, b3;}"
      : "=r"(h0), "=r"(h1), "=r"(h2), "=r"(h3) : "r"(w));
  const uint32_t h[4] = {h0, h1, h2, h3};
#pragma unroll
  for (int i = 0; i < 4; i++) {
    float lo, hi;
    asm("{.reg .f16 l, h;\n\t"
        "mov.b32 {l, h}, %2;\n\t"
        "cvt.f32.f16 %0, l;\n\t"
        "cvt.f32.f16 %1, h;}"
        : "=f"(lo), "=f"(hi) : "r"(h[i]));
    v[2 * i] = lo;
    v[2 * i + 1] = hi;
  }
}

// one E4M3 byte -> fp32 (exact)
__device__ __forceinline__ float e4m3_to_f32(uint32_t byte) {
  float lo, hi;
  e4m3x2_to_f32(byte & 0xFFu, lo, hi);
  return lo;
}

}  // namespace nvfp4rs

namespace nvfp4rs {

// ------------------------------------------- exact divisions without a divide
//
// Markstein's correction (P. Markstein, IBM J. Res. Dev. 34(1), 1990): with
// y = RN(1/b), q0 = RN(a*y), r = fma(-q0, b, a) (exact), q = fma(r, y, q0)
// gives q = RN(a/b). The project's tests prove this exhaustively, by exact
// integer emulation, for every operand pair these two helpers can meet above
// the 2^-100 cut-off; below it (tiny values, where r could be subnormal) they
// fall back to the IEEE divide.

// RN(b / 6) for a block maximum b >= 0 (a bf16 value)
__device__ __forceinline__ float div6(float b) {
  if (b < 0x1p-100f) return __fdiv_rn(b, 6.0f);
  const float y = 0x1.555556p-3f;  // RN(1/6)
  const float q0 = __fmul_rn(b, y);
  const float r = __fmaf_rn(-q0, 6.0f, b);
  return __fmaf_rn(r, y, q0);
}

// Element multiplier min(RN(S / v), FLT_MAX) for S = S_enc and vy = {v,
// RN(1/v)} of the block's E4M3 scale; vy = {1, 0} for scale code 0 gives 0.
// An overflowing q0 turns into NaN, which fminf maps to FLT_MAX -- the
// clamped value of an overflowing quotient.
__device__ __forceinline__ float elem_scale(float S, float2 vy) {
  if (S < 0x1p-100f) return vy.y == 0.0f ? 0.0f : fminf(__fdiv_rn(S, vy.x), FLT_MAX);
  const float q0 = __fmul_rn(S, vy.y);
  const float r = __fmaf_rn(-q0, vy.x, S);
  return fminf(__fmaf_rn(r, vy.y, q0), FLT_MAX);
}

// Table entry for E4M3 code c (0..127): {value, RN(1/value)}; codes 0 and
// 0x7F (NaN, never produced by the saturating convert) hold {1, 0}.
__device__ __forceinline__ float2 e4m3_entry(int c) {
  if (c == 0 || c >= 0x7F) return make_float2(1.0f, 0.0f);
  const int e = c >> 3, m = c & 7;
  const float v = e == 0 ? __fmul_rn(static_cast<float>(m), 0x1p-9f)
                         : __uint_as_float((static_cast<uint32_t>(e + 120) << 23) |
                                           (static_cast<uint32_t>(m) << 20));
  return make_float2(v, __frcp_rn(v));
}

}  // namespace nvfp4rs
