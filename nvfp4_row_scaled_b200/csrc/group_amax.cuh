// group_amax.cuh -- grouped amax, both directions from one read of x.
//
// TransformerEngine #3649 (grouped row-scaled NVFP4 cast), Description: a
// single launch over the packed (sum_M, K) bf16 buffer produces the per-row
// amax [sum_M] and the per-group, per-column amax [E*K]. The per-column amax
// is what the transposed operand is scaled by (TransformerEngine #3324,
// summary: columnwise per-column amax).
//
// Work split. Tiles are 128 rows of the packed buffer; group sizes are
// multiples of 16, so every 16-row block lies in one group. Most tiles lie
// in one group; a "mixed" tile, which a group boundary crosses, sends each
// lane's column maxima straight to that lane's group, and the last tile may
// hold fewer than 128 routed rows (the rest is skipped). The K/128 column
// chunks of a tile are dealt round
// robin to a thread-block cluster of CN CTAs (CN <= 8, the largest divisor of
// K/128): CTA q takes chunks q, q + CN, q + 2CN, ..., so the cluster reads each
// row left to right in CN * 256-byte runs (much kinder to DRAM than one slab
// per CTA). A CTA's work is cut into units of (128-column chunk, 32-row
// quarter); warp w takes every unit of quarter w, so the four warps stay
// balanced for any K.
//
// Inside a unit a lane owns 8 columns (one 16-byte chunk) of 16 rows (the
// 16-row block 2w + h of the tile, h = lane / 16):
//  - column maxima: packed bf16x2 |.|-max over the lane's 16 rows, merged with
//    the other half-warp by a shuffle, then into a per-CTA shared array;
//  - row maxima: the lane's 8-column maximum of each of its 16 rows is
//    reduced over the 16 lanes sharing those rows with a reduce-scatter
//    butterfly (8 shuffles), which leaves lane j holding row j's maximum.
// Row maxima of the CTA's columns meet in shared memory; the cluster's CN
// partial row maxima are then combined through distributed shared memory by
// CTA rank 0, which writes row_amax. Column maxima go to col_amax with one
// unsigned atomic max per column per CTA (non-negative floats order like
// their bit patterns, and max is order-free, so the result is deterministic).
// col_amax must be zero before the kernel's first atomic: the host enqueues
// zero_f32_kernel just before it and launches this kernel programmatically
// after it, so that the reads of x overlap the zeroing; every atomic on
// col_amax comes after grid_dependency_wait().
#pragma once

#include <cooperative_groups.h>

#include "codec.cuh"
#include "routing.cuh"

namespace nvfp4rs {

namespace cg = cooperative_groups;

constexpr int kAmaxThreads = 128;
constexpr int kCols128 = 128;  // columns per chunk

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 v;
  if (!NVFP4_LOAD_OK(p, 16)) return make_uint4(0u, 0u, 0u, 0u);
  asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
      : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
      : "l"(p));
  return v;
}

__device__ __forceinline__ void red_max_u32(float* addr, uint32_t v) {
  if (!NVFP4_STORE_OK(addr, 4)) return;
  asm volatile("red.global.max.u32 [%0], %1;" ::"l"(addr), "r"(v) : "memory");
}

// Zeroes n floats, after letting the kernel launched after it on the stream
// start at once (that kernel waits for this one before it touches p).
__global__ void __launch_bounds__(256) zero_f32_kernel(float* __restrict__ p, int64_t n) {
  launch_dependents();
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    gstore(&p[i], 0.0f);
}

template <class Routing>
__global__ void __launch_bounds__(kAmaxThreads, 6)
group_amax_kernel(const __grid_constant__ Routing routing, const uint4* __restrict__ x,
                  int32_t K, int32_t cn, float* __restrict__ row_amax,
                  float* __restrict__ col_amax) {
  __shared__ RoutingSmem rs;
  __shared__ uint32_t rmax[kRows];
  // the cast launched after this kernel may start its set-up now
  launch_dependents();
  // dynamic: column maxima of this CTA's chunks (128 per chunk), then the
  // E+1 group offsets. The ceil(K/128) chunks of 128 columns are dealt over
  // the cluster; columns of the last chunk past K are neither read nor written.
  const int cols = (((K + kCols128 - 1) / kCols128) / cn) * kCols128;
  extern __shared__ uint32_t cmax[];
  routing.load(rs, reinterpret_cast<int32_t*>(cmax + cols));

  const int t = threadIdx.x;
  const int lane = t & 31, warp = t >> 5;
  const int cc = lane & 15, h = lane >> 4;
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());
  const int tile = blockIdx.x / cn;
  const int32_t r0 = tile * kRows;
  const bool active = rs.ok && r0 < rs.total;
  // routed rows of the tile (a multiple of 16: the tail tile may be short),
  // this lane's 16-row block and its group; a tile that holds rows of more
  // than one group ("mixed") sends each lane's column maxima to its own group
  const int valid = active ? min(kRows, rs.total - r0) : 0;
  const int rb = 2 * warp + h;
  const bool lane_ok = kBlockRows * rb < valid;
  const int g_first = active ? group_of_row(rs, r0) : 0;
  const bool mixed = active && rs.off[g_first + 1] < r0 + valid;
  const int g_lane = (mixed && lane_ok) ? group_of_row(rs, r0 + kBlockRows * rb) : g_first;

  rmax[t] = 0u;
  for (int c = t; c < cols; c += kAmaxThreads) cmax[c] = 0u;
  __syncthreads();

  if (active) {
    const int nchunks = cols >> 7;
    const size_t K8 = static_cast<size_t>(K) >> 3;  // row pitch in 16-byte units
    for (int ch = 0; ch < nchunks; ch++) {
      // this lane: rows r0 + 16*rb + i (i < 16), columns c0 .. c0+7
      const int c_loc = (ch << 7) + (cc << 3);                // index into this CTA's cmax
      const int c_glb = ((ch * cn + rank) << 7) + (cc << 3);  // chunk ch of the CTA: rank + ch*cn
      const bool col_ok = c_glb < K;                          // the lane's 8 columns are inside K
      // (a lane past the routed rows reads the tile's first block instead and
      // contributes nothing; a lane past K reads nothing)
      const uint4* p = x + (static_cast<size_t>(r0 + (lane_ok ? kBlockRows * rb : 0)) * K8) + (c_glb >> 3);
      uint4 v[16];
      if (col_ok) {
#pragma unroll
        for (int i = 0; i < 16; i++) v[i] = ld_stream(p + i * K8);
      } else {
#pragma unroll
        for (int i = 0; i < 16; i++) v[i] = make_uint4(0u, 0u, 0u, 0u);
      }

      // column maxima over the lane's 16 rows
      uint32_t c0 = v[0].x, c1 = v[0].y, c2 = v[0].z, c3 = v[0].w;
#pragma unroll
      for (int i = 1; i < 16; i++) {
        c0 = maxabs2(c0, v[i].x);
        c1 = maxabs2(c1, v[i].y);
        c2 = maxabs2(c2, v[i].z);
        c3 = maxabs2(c3, v[i].w);
      }
      if (!lane_ok) c0 = c1 = c2 = c3 = 0u;
      // row partial maxima, packed two rows per word: P[k] = (row 2k, row 2k+1)
      uint32_t P[8];
#pragma unroll
      for (int k = 0; k < 8; k++) {
        const uint32_t a = maxabs2(maxabs2(v[2 * k].x, v[2 * k].y), maxabs2(v[2 * k].z, v[2 * k].w));
        const uint32_t b = maxabs2(maxabs2(v[2 * k + 1].x, v[2 * k + 1].y),
                                   maxabs2(v[2 * k + 1].z, v[2 * k + 1].w));
        // (a.lo, b.lo) vs (a.hi, b.hi)
        P[k] = maxabs2(prmt(a, b, 0x5410), prmt(a, b, 0x7632)) & 0x7FFF7FFFu;
      }
      // reduce-scatter over the 16 lanes of this half-warp: lane cc ends with row cc
      {
        const bool b3 = cc & 8, b2 = cc & 4, b1 = cc & 2, b0 = cc & 1;
        uint32_t Q[4];
#pragma unroll
        for (int k = 0; k < 4; k++) {
          const uint32_t keep = b3 ? P[4 + k] : P[k];
          const uint32_t send = b3 ? P[k] : P[4 + k];
          Q[k] = umax2(keep, __shfl_xor_sync(0xFFFFFFFFu, send, 8));
        }
        uint32_t R[2];
#pragma unroll
        for (int k = 0; k < 2; k++) {
          const uint32_t keep = b2 ? Q[2 + k] : Q[k];
          const uint32_t send = b2 ? Q[k] : Q[2 + k];
          R[k] = umax2(keep, __shfl_xor_sync(0xFFFFFFFFu, send, 4));
        }
        uint32_t S;
        {
          const uint32_t keep = b1 ? R[1] : R[0];
          const uint32_t send = b1 ? R[0] : R[1];
          S = umax2(keep, __shfl_xor_sync(0xFFFFFFFFu, send, 2));
        }
        const uint32_t keep = b0 ? (S >> 16) : (S & 0xFFFFu);
        const uint32_t send = b0 ? (S & 0xFFFFu) : (S >> 16);
        const uint32_t rowm = max(keep, __shfl_xor_sync(0xFFFFFFFFu, send, 1));
        // lane (cc, h) holds tile row 16*rb + cc
        atomicMax(&rmax[kBlockRows * rb + cc], rowm << 16);
      }
      if (mixed) {  // straight to this lane's group (a mixed tile is rare)
        if (lane_ok && col_ok && col_amax != nullptr) {
          grid_dependency_wait();  // col_amax is zero
          float* dst = col_amax + static_cast<size_t>(g_lane) * K + c_glb;
          const uint32_t w[4] = {c0 & 0x7FFF7FFFu, c1 & 0x7FFF7FFFu, c2 & 0x7FFF7FFFu, c3 & 0x7FFF7FFFu};
#pragma unroll
          for (int q = 0; q < 4; q++) {
            red_max_u32(dst + 2 * q, w[q] << 16);
            red_max_u32(dst + 2 * q + 1, w[q] & 0xFFFF0000u);
          }
        }
        continue;
      }
      // merge the two half-warps' column maxima, then into the CTA's array
      c0 = maxabs2(c0, __shfl_xor_sync(0xFFFFFFFFu, c0, 16)) & 0x7FFF7FFFu;
      c1 = maxabs2(c1, __shfl_xor_sync(0xFFFFFFFFu, c1, 16)) & 0x7FFF7FFFu;
      c2 = maxabs2(c2, __shfl_xor_sync(0xFFFFFFFFu, c2, 16)) & 0x7FFF7FFFu;
      c3 = maxabs2(c3, __shfl_xor_sync(0xFFFFFFFFu, c3, 16)) & 0x7FFF7FFFu;
      const uint32_t wa = h ? c2 : c0, wb = h ? c3 : c1;  // h=0: cols 0..3, h=1: cols 4..7
      uint32_t* cm = &cmax[c_loc + 4 * h];
      atomicMax(cm + 0, wa << 16);
      atomicMax(cm + 1, wa & 0xFFFF0000u);
      atomicMax(cm + 2, wb << 16);
      atomicMax(cm + 3, wb & 0xFFFF0000u);
    }
  }
  __syncthreads();
  if (active && !mixed && col_amax != nullptr) {
    grid_dependency_wait();  // col_amax is zero
    float* dst = col_amax + static_cast<size_t>(g_first) * K;
    for (int c = t; c < cols; c += kAmaxThreads) {
      const int gc = (((c >> 7) * cn + rank) << 7) | (c & 127);
      if (gc < K) red_max_u32(dst + gc, cmax[c]);
    }
  }
  // every CTA of the cluster reaches both barriers, active or not
  cluster.sync();
  if (active && rank == 0 && row_amax != nullptr && t < valid) {
    uint32_t m = rmax[t];
    for (int q = 1; q < cn; q++) m = max(m, *cluster.map_shared_rank(&rmax[t], q));
    gstore(&row_amax[r0 + t], __uint_as_float(m));
  }
  cluster.sync();
}

}  // namespace nvfp4rs
