// dequant.cuh -- NVFP4 and MXFP4 to FP32.
//
// TransformerEngine #2931 ("Implement per-token NVFP4 fprop recipe",
// Important Files Changed): the dequantize kernel takes the amax of the
// element's row instead of one per-tensor amax. Here each row carries its
// decode scale S_dec = amax / (6*448) and an element decodes to
// (e2m1(code) * e4m3(block scale)) * S_dec; the first product is exact, so
// the one rounding is the multiply by S_dec. MXFP4 (TransformerEngine #3824,
// "E2M1/block-32/E8M0"): e2m1(code) * 2^(scale - 127), one rounding.
//
// Bound by the 4-byte-per-element FP32 writes. A warp takes a row at a time
// (rows dealt round robin over the grid's warps); lane l decodes elements
// 4l .. 4l+3 of each 128-element run of the row, so every store instruction
// writes 512 contiguous bytes (streaming, evict-first), from one 2-byte code
// load and one scale byte; no division.
#pragma once

#include "bounds.cuh"
#include "codec.cuh"

namespace nvfp4rs {

constexpr int kDequantThreads = 256;

// four codes (two bytes, element 4q in the low nibble) -> fp32. The code
// pair goes in as a 16-bit operand split into its two bytes (a 32-bit operand
// holding a zero-extended 16-bit load, split four ways, decoded to zeros).
__device__ __forceinline__ void e2m1x4_to_f32(uint16_t c, float (&v)[4]) {
  uint32_t h0, h1;
  asm("{.reg .b8 b0, b1;\n\t"
      "mov.b16 {b0, b1}, %2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, b1;}"
      : "=r"(h0), "=r"(h1) : "h"(c));
  asm("{.reg .f16 e0, e1, e2, e3;\n\t"
      "mov.b32 {e0, e1}, %4;\n\t"
      "mov.b32 {e2, e3}, %5;\n\t"
      "cvt.f32.f16 %0, e0;\n\t"
      "cvt.f32.f16 %1, e1;\n\t"
      "cvt.f32.f16 %2, e2;\n\t"
      "cvt.f32.f16 %3, e3;}"
      : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]) : "r"(h0), "r"(h1));
}

// kMx = false: NVFP4 (E4M3 scale per 16 elements, S_dec per row);
// kMx = true: MXFP4 (E8M0 scale per 32 elements).
template <bool kMx>
__global__ void __launch_bounds__(kDequantThreads)
dequant_kernel(const uint16_t* __restrict__ data, const uint8_t* __restrict__ scale,
               const float* __restrict__ s2, int64_t rows, int64_t cols, float4* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  const int64_t cols4 = cols >> 2;                         // 4-element pieces per row
  const int64_t spr = kMx ? (cols >> 5) : (cols >> 4);     // scales per row
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (kDequantThreads / 32);
  for (int64_t r = static_cast<int64_t>(blockIdx.x) * (kDequantThreads / 32) + (threadIdx.x >> 5); r < rows;
       r += warps) {
    const uint16_t* d = data + r * cols4;
    const uint8_t* sc = scale + r * spr;
    const float sd = kMx ? 1.0f : gload(&s2[r]);
    float4* o = out + r * cols4;
#pragma unroll 4
    for (int64_t q = lane; q < cols4; q += 32) {
      const uint16_t c = gload(&d[q]);
      const uint32_t sb = gload(&sc[kMx ? (q >> 3) : (q >> 2)]);
      float v[4];
      e2m1x4_to_f32(c, v);
      float4 y;
      if (kMx) {
        // 2^(sb - 127): sb == 0 is the subnormal 2^-127, 0xFF is NaN
        const float s = sb == 0u ? 0x1p-127f : (sb == 0xFFu ? __uint_as_float(0x7FC00000u) : __uint_as_float(sb << 23));
        y = make_float4(__fmul_rn(v[0], s), __fmul_rn(v[1], s), __fmul_rn(v[2], s), __fmul_rn(v[3], s));
      } else {
        const float sv = e4m3_to_f32(sb);
        y = make_float4(__fmul_rn(__fmul_rn(v[0], sv), sd), __fmul_rn(__fmul_rn(v[1], sv), sd),
                        __fmul_rn(__fmul_rn(v[2], sv), sd), __fmul_rn(__fmul_rn(v[3], sv), sd));
      }
      if (NVFP4_STORE_OK(o + q, 16)) __stcs(o + q, y);
    }
  }
}

}  // namespace nvfp4rs
