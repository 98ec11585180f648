// post_scale.cuh -- FP32 per-row scaling of a GEMM output (the consumer side
// of the row-scaled cast).
//
// TransformerEngine #2931 ("Implement per-token NVFP4 fprop recipe"), sequence
// diagram: the GEMM sees the row-scaled operand with its amax replaced by
// ones and produces an FP32 output; the output rows are then multiplied by
// the row-wise amax and converted to the target dtype (Important Files
// Changed, gemm.py: a bias is taken out before this scaling and added back
// after). Per element: y = fl(x * amax[r]), then fl(y + bias[c]) with a
// bias, then f32 or bf16 (round to nearest even).
//
// Memory-bound: 4 bytes in and 4 or 2 out per element. The output is cut
// into units of 16 rows x 128 columns, dealt round robin to the warps of the
// grid (neighbouring warps take neighbouring column chunks of the same rows).
// A lane owns 4 columns of a unit: it loads their bias once, takes the 16
// rows' amax from one load and shuffles, and keeps 16 independent 16-byte
// loads in flight.
#pragma once

#include <cstdint>

#include "bounds.cuh"

namespace nvfp4rs {

constexpr int kPostThreads = 256;

__device__ __forceinline__ float4 ld_stream_f4(const float4* p) {
  float4 v;
  if (!NVFP4_LOAD_OK(p, 16)) return make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  asm("ld.global.nc.L1::no_allocate.v4.f32 {%0, %1, %2, %3}, [%4];"
      : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
      : "l"(p));
  return v;
}

// two floats -> packed bf16x2, round to nearest even (lo in the low half)
__device__ __forceinline__ uint32_t bf16x2_rn(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

constexpr int kPostUnitRows = 16;

template <bool kBf16, bool kBias>
__global__ void __launch_bounds__(kPostThreads, 2)
row_post_scale_kernel(const float4* in, int64_t rows, int64_t cols4, const float* __restrict__ amax,
                      const float4* __restrict__ bias, void* out) {
  const int lane = threadIdx.x & 31;
  const int64_t n_cb = (cols4 + 31) / 32;                        // 128-column chunks
  const int64_t units = (rows + kPostUnitRows - 1) / kPostUnitRows * n_cb;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (kPostThreads / 32);
  for (int64_t u = static_cast<int64_t>(blockIdx.x) * (kPostThreads / 32) + (threadIdx.x >> 5); u < units;
       u += warps) {
    const int64_t rb = u / n_cb, cb = u - rb * n_cb;
    const int64_t r0 = rb * kPostUnitRows;
    const int64_t c = cb * 32 + lane;
    const int nr = rows - r0 < kPostUnitRows ? static_cast<int>(rows - r0) : kPostUnitRows;
    const float a_lane = lane < nr ? gload(&amax[r0 + lane]) : 0.0f;
    float4 b = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    if (kBias && c < cols4) b = gload(&bias[c]);
    float4 x[kPostUnitRows];
#pragma unroll
    for (int i = 0; i < kPostUnitRows; i++)
      if (i < nr && c < cols4) x[i] = ld_stream_f4(in + (r0 + i) * cols4 + c);
#pragma unroll
    for (int i = 0; i < kPostUnitRows; i++) {
      const float a = __shfl_sync(0xFFFFFFFFu, a_lane, i);
      if (i < nr && c < cols4) {
        float4 y = make_float4(__fmul_rn(x[i].x, a), __fmul_rn(x[i].y, a), __fmul_rn(x[i].z, a),
                               __fmul_rn(x[i].w, a));
        if (kBias)
          y = make_float4(__fadd_rn(y.x, b.x), __fadd_rn(y.y, b.y), __fadd_rn(y.z, b.z), __fadd_rn(y.w, b.w));
        const int64_t o = (r0 + i) * cols4 + c;
        if (kBf16)
          gstore(reinterpret_cast<uint2*>(out) + o, make_uint2(bf16x2_rn(y.x, y.y), bf16x2_rn(y.z, y.w)));
        else if (NVFP4_STORE_OK(reinterpret_cast<float4*>(out) + o, 16))
          __stcs(reinterpret_cast<float4*>(out) + o, y);
      }
    }
  }
}

}  // namespace nvfp4rs
