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

// --------------------------------------------------------------- decoding

// one E4M3 byte -> fp32 (exact)
__device__ __forceinline__ float e4m3_to_f32(uint32_t byte) {
  float lo, hi;
  e4m3x2_to_f32(byte & 0xFFu, lo, hi);
  return lo;
}

}  // namespace nvfp4rs

namespace nvfp4rs {

// E4M3 tables used by the block-scale shortcut below, one entry per code c
// (0..127): nv = -value(c) and r = RN(1/value(c)). Code 0 and 0x7F (NaN, never
// produced by the saturating convert) hold nv = -1, r = 0, which makes the
// element multiplier of a zero scale come out 0 with no branch.
struct E4m3Table {
  float nv[128];
  float r[128];
};

// Entry c of the table, written by thread c of a block (c < 128).
__device__ __forceinline__ void e4m3_table_fill(E4m3Table& tab, int c) {
  if (c == 0 || c >= 0x7F) {
    tab.nv[c] = -1.0f;
    tab.r[c] = 0.0f;
    return;
  }
  const int e = c >> 3, m = c & 7;
  const float v = e == 0 ? __fmul_rn(static_cast<float>(m), 0x1p-9f)
                         : __uint_as_float((static_cast<uint32_t>(e + 120) << 23) |
                                           (static_cast<uint32_t>(m) << 20));
  tab.nv[c] = -v;
  tab.r[c] = __frcp_rn(v);
}

}  // namespace nvfp4rs

namespace nvfp4rs {

// --------------------------------------- packed (f32x2) element arithmetic
//
// The element path keeps each bf16 pair of a word as one 64-bit register pair
// (low element in the low half) from the unpack through the multiply to the
// E2M1 convert, so no moves are needed to form f32x2 operands.

// bf16x2 word -> f32x2 pair (exact)
__device__ __forceinline__ uint64_t unpack2(uint32_t w) {
  uint64_t r;
  asm("{.reg .b32 lo, hi;\n\t"
      "shl.b32 lo, %1, 16;\n\t"
      "and.b32 hi, %1, 0xffff0000;\n\t"
      "mov.b64 %0, {lo, hi};}"
      : "=l"(r) : "r"(w));
  return r;
}

__device__ __forceinline__ uint64_t pack2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}

// pairwise IEEE multiply
__device__ __forceinline__ uint64_t mul2x(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// pairwise a*b + c, one rounding per element
__device__ __forceinline__ uint64_t fma2x(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

// the low / high float of an f32x2 register pair
__device__ __forceinline__ float lo_of(uint64_t p) {
  float l;
  asm("{.reg .b32 t;\n\tmov.b64 {%0, t}, %1;}" : "=f"(l) : "l"(p));
  return l;
}
__device__ __forceinline__ float hi_of(uint64_t p) {
  float h;
  asm("{.reg .b32 t;\n\tmov.b64 {t, %0}, %1;}" : "=f"(h) : "l"(p));
  return h;
}

// Codes of four pairs, pair i -> byte i with its low element in the low nibble.
__device__ __forceinline__ uint32_t e2m1_pairs(uint64_t p0, uint64_t p1, uint64_t p2, uint64_t p3) {
  uint32_t r;
  asm("{.reg .b8 b0, b1, b2, b3;\n\t"
      ".reg .b32 l0, h0, l1, h1, l2, h2, l3, h3;\n\t"
      "mov.b64 {l0, h0}, %1;\n\t"
      "mov.b64 {l1, h1}, %2;\n\t"
      "mov.b64 {l2, h2}, %3;\n\t"
      "mov.b64 {l3, h3}, %4;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, h0, l0;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, h1, l1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, h2, l2;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, h3, l3;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};}"
      : "=r"(r) : "l"(p0), "l"(p1), "l"(p2), "l"(p3));
  return r;
}

// Codes across two rows: p (row i) and q (row i+1) hold the same column
// pair. Byte 0 = (p.lo, q.lo), byte 1 = (p.hi, q.hi), byte 2 = (r.lo, s.lo),
// byte 3 = (r.hi, s.hi), the row-i value in the low nibble.
__device__ __forceinline__ uint32_t e2m1_cross(uint64_t p, uint64_t q, uint64_t r, uint64_t s) {
  uint32_t d;
  asm("{.reg .b8 b0, b1, b2, b3;\n\t"
      ".reg .b32 pl, ph, ql, qh, rl, rh, sl, sh;\n\t"
      "mov.b64 {pl, ph}, %1;\n\t"
      "mov.b64 {ql, qh}, %2;\n\t"
      "mov.b64 {rl, rh}, %3;\n\t"
      "mov.b64 {sl, sh}, %4;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, ql, pl;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, qh, ph;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, sl, rl;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, sh, rh;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};}"
      : "=r"(d) : "l"(p), "l"(q), "l"(r), "l"(s));
  return d;
}

// ------------------------------------------------- branch-free block scales
//
// Markstein's correction (P. Markstein, IBM J. Res. Dev. 34(1), 1990): with
// y = RN(1/b), q0 = RN(a*y), r = fma(-q0, b, a) (exact), q = fma(r, y, q0)
// gives q = RN(a/b). The project's tests prove this exhaustively, by exact
// integer emulation, for every operand pair used below in its stated range.
//
// The common path of a block scale has no branch, so the compiler can
// interleave the independent blocks of a lane. It is exact whenever the
// governing (row or column) amax a is 0 or lies in [2^-81, 2^111]:
//  - then S_enc = 2688 / a >= 2^-100, the range over which the exhaustive
//    test proves the element-scale shortcut;
//  - block maxima b >= 2^-100 (or b == 0) are covered by the test of the
//    divide-by-6 shortcut;
//  - a block maximum 0 < b < 2^-100 under an amax a >= 2^-81 has
//    b/6 * 2688/a < 448 * 2^-19 < 2^-10, so its scale is E4M3 zero whether or
//    not b/6 was rounded exactly, and its multiplier is 0 either way.
// Tiles holding a row or column outside that range take scales2_exact.

constexpr float kFastAmaxMin = 0x1p-81f;
constexpr float kFastAmaxMax = 0x1p111f;

__device__ __forceinline__ bool fast_path_amax(float a) {
  return a == 0.0f || (a >= kFastAmaxMin && a <= kFastAmaxMax);
}

// Two block scales at once (the blocks of one lane that share an f32x2
// register pair): bm2 = {bmax0, bmax1} (block maxima), se2 = {S_enc0,
// S_enc1}. Returns the two E4M3 codes (block 0 in bits 0..7, block 1 in bits
// 8..15) and sets enc2 = {enc0, enc1}, the element multipliers:
//   s32 = fl(fl(bmax/6) * S_enc), code = E4M3_rne_satfinite(s32),
//   enc = fl(S_enc / e4m3(code)) (0 for a zero code).
// Both divides use Markstein's correction with the reciprocal taken from
// RN(1/6) or the table (tab.r), and the exact remainder fma(q0, -b, a) (the
// table stores -value, so no negation is needed).
__device__ __forceinline__ uint32_t scales2x_fast(uint64_t bm2, uint64_t se2, const E4m3Table& tab,
                                                  uint64_t& enc2) {
  const uint64_t y6 = pack2(0x1.555556p-3f, 0x1.555556p-3f);  // RN(1/6)
  const uint64_t m6 = pack2(-6.0f, -6.0f);
  const uint64_t q6 = mul2x(bm2, y6);
  const uint64_t d6 = fma2x(fma2x(q6, m6, bm2), y6, q6);
  const uint64_t s32 = mul2x(d6, se2);
  const uint32_t p = e4m3x2(hi_of(s32), lo_of(s32));
  const uint32_t c0 = p & 0xFFu, c1 = p >> 8;
  const uint64_t nv = pack2(tab.nv[c0], tab.nv[c1]);
  const uint64_t yr = pack2(tab.r[c0], tab.r[c1]);
  const uint64_t q0 = mul2x(se2, yr);
  enc2 = fma2x(fma2x(q0, nv, se2), yr, q0);
  return p;
}

// The same quantities with IEEE divides (any operand range).
__device__ __forceinline__ uint32_t scales2_exact(float bm0, float se0, float bm1, float se1,
                                                  float& enc0, float& enc1) {
  const uint32_t p = e4m3x2(__fmul_rn(__fdiv_rn(bm1, 6.0f), se1), __fmul_rn(__fdiv_rn(bm0, 6.0f), se0));
  const float v0 = e4m3_to_f32(p & 0xFFu), v1 = e4m3_to_f32(p >> 8);
  enc0 = (p & 0xFFu) ? fminf(__fdiv_rn(se0, v0), FLT_MAX) : 0.0f;
  enc1 = (p & 0xFF00u) ? fminf(__fdiv_rn(se1, v1), FLT_MAX) : 0.0f;
  return p;
}

template <bool kExact>
__device__ __forceinline__ uint32_t scales2x_any(uint64_t bm2, uint64_t se2, const E4m3Table& tab,
                                                 uint64_t& enc2) {
  if (kExact) {
    float e0, e1;
    const uint32_t p = scales2_exact(lo_of(bm2), lo_of(se2), hi_of(bm2), hi_of(se2), e0, e1);
    enc2 = pack2(e0, e1);
    return p;
  }
  return scales2x_fast(bm2, se2, tab, enc2);
}

}  // namespace nvfp4rs
