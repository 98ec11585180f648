// dequant.cuh -- NVFP4 to FP32 with one decode scale per row.
//
// TransformerEngine #2931 ("Implement per-token NVFP4 fprop recipe",
// Important Files Changed): the dequantize kernel takes the amax of the
// element's row instead of one per-tensor amax. Here each row carries its
// decode scale S_dec = amax / (6*448) and an element decodes to
// (e2m1(code) * e4m3(block scale)) * S_dec; the first product is exact, so
// the one rounding is the multiply by S_dec.
//
// One thread decodes one 16-element block: an 8-byte load of codes, one
// scale byte, one S_dec, and four 16-byte stores. The kernel is bound by the
// 4-byte-per-element FP32 writes.
#pragma once

#include "codec.cuh"

namespace nvfp4rs {

constexpr int kDequantThreads = 256;

__global__ void __launch_bounds__(kDequantThreads)
dequant_kernel(const uint2* __restrict__ data, const uint8_t* __restrict__ scale,
               const float* __restrict__ s2, int64_t rows, int64_t blocks_per_row,
               float4* __restrict__ out) {
  const int64_t n = rows * blocks_per_row;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kDequantThreads;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * kDequantThreads + threadIdx.x; i < n;
       i += stride) {
    const int64_t r = i / blocks_per_row;
    const uint2 d = data[i];
    const float sv = e4m3_to_f32(scale[i]);
    const float sd = s2[r];
    float v0[8], v1[8];
    e2m1x8_to_f32(d.x, v0);
    e2m1x8_to_f32(d.y, v1);
    float o[16];
#pragma unroll
    for (int k = 0; k < 8; k++) {
      o[k] = __fmul_rn(__fmul_rn(v0[k], sv), sd);
      o[8 + k] = __fmul_rn(__fmul_rn(v1[k], sv), sd);
    }
    float4* dst = out + 4 * i;
    dst[0] = make_float4(o[0], o[1], o[2], o[3]);
    dst[1] = make_float4(o[4], o[5], o[6], o[7]);
    dst[2] = make_float4(o[8], o[9], o[10], o[11]);
    dst[3] = make_float4(o[12], o[13], o[14], o[15]);
  }
}

}  // namespace nvfp4rs
