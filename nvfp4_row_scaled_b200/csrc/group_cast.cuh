// group_cast.cuh -- grouped row-scaled NVFP4 cast, rowwise and colwise from
// one read of each tile.
//
// TransformerEngine #3649 (grouped row-scaled NVFP4 cast), Description: the
// second single launch takes the row and column amax vectors and writes the
// packed FP4 data and the scales of every group; TransformerEngine #2931
// ("Implement per-token NVFP4 fprop recipe", Changes) defines the per-token
// scaling; TransformerEngine #3324 (row-scaled backward for GroupedLinear,
// summary) adds the columnwise (transposed) operand with per-column amax.
//
// This file holds what the cast kernels share: TMA and mbarrier helpers, the
// lane patch, the element and block-scale encoding (encode_codes,
// encode_patch) and the scale stores. The grouped NVFP4 cast kernel is in
// group_cast_plain.cuh, the one-launch amax + cast in group_quantize.cuh and
// the MXFP4 cast in mx_cast.cuh.
//
// The lane patch (all kernels): a lane holds 16 rows x 8 columns of a
// 128 x 128 tile in registers -- 8 complete colwise blocks and 16 half
// rowwise blocks, completed with the neighbouring lane -- and encodes both
// directions from it. Block scales use exact shortcuts instead of IEEE
// divides: a per-CTA table of every E4M3 value and its correctly rounded
// reciprocal, and Markstein's correction (codec.cuh).
#pragma once

#include <cuda.h>

#include "codec.cuh"
#include "routing.cuh"

namespace nvfp4rs {

constexpr int kCastThreads = 128;
constexpr int kCols = 128;
constexpr int kStages = 2;
constexpr int kBoxCols = 64;                          // TMA box: 64 columns (128 bytes) x 128 rows
constexpr int kBoxBytes = kBoxCols * kRows * 2;       // 16 KB
constexpr int kTileBytes = 2 * kBoxBytes;             // 32 KB per 128 x 128 tile
constexpr uint32_t kSpinLimit = 1u << 22;             // bounded mbarrier waits

struct CastOut {
  uint8_t* row_data;
  uint8_t* row_scale;
  float* row_s2;
  uint8_t* col_data;
  uint8_t* col_scale;
  float* col_s2;
  int32_t tiled_scales;  // nonzero: both scale outputs in the 128x4-tiled layout
};


// ------------------------------------------------------------- TMA / mbarrier

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

// Wait for the phase with parity `phase` to complete; false after `tries` tries.
__device__ __forceinline__ bool mbar_wait_some(uint64_t* bar, uint32_t phase, uint32_t tries) {
  const uint32_t a = smem_addr(bar);
  for (uint32_t i = 0; i < tries; i++) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(a), "r"(phase)
        : "memory");
    if (done) return true;
  }
  return false;
}

// Wait for the phase with parity `phase` to complete; false after kSpinLimit tries.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t phase) {
  return mbar_wait_some(bar, phase, kSpinLimit);
}

__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ void st_global_u2_hint(void* p, uint2 v, uint64_t policy) {
  if (!NVFP4_STORE_OK(p, 8)) return;
  asm volatile("st.global.L2::cache_hint.v2.u32 [%0], {%1, %2}, %3;" ::"l"(p), "r"(v.x), "r"(v.y),
               "l"(policy) : "memory");
}
__device__ __forceinline__ void st_global_u32_hint(void* p, uint32_t v, uint64_t policy) {
  if (!NVFP4_STORE_OK(p, 4)) return;
  asm volatile("st.global.L2::cache_hint.u32 [%0], %1, %2;" ::"l"(p), "r"(v), "l"(policy) : "memory");
}
__device__ __forceinline__ void st_global_u4_hint(void* p, uint4 v, uint64_t policy) {
  if (!NVFP4_STORE_OK(p, 16)) return;
  asm volatile("st.global.L2::cache_hint.v4.u32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(p), "r"(v.x),
               "r"(v.y), "r"(v.z), "r"(v.w), "l"(policy) : "memory");
}
__device__ __forceinline__ uint64_t policy_evict_normal() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y,
                                            uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar)), "l"(policy)
      : "memory");
}

// Untiled bulk copy global -> shared (16-byte aligned, multiple of 16 bytes),
// completion counted on `bar`. No multicast.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  src = NVFP4_BULK_SRC(src, bytes);
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// A lane's patch: rows rl .. rl+15, columns 8cc .. 8cc+7 of the swizzled
// 128 x 128 tile at `tile` (two 64-column boxes).
__device__ __forceinline__ void load_patch(const uint8_t* tile, int cc, int rl, uint4 (&v)[16]) {
  const uint8_t* tb = tile + (cc >> 3) * kBoxBytes + rl * 128;
  const int j = cc & 7;
#pragma unroll
  for (int i = 0; i < 16; i++)
    v[i] = *reinterpret_cast<const uint4*>(tb + i * 128 + ((j ^ (i & 7)) << 4));
}

__device__ __forceinline__ void st_global_u32(uint8_t* p, uint32_t v) {
  gstore(reinterpret_cast<uint32_t*>(p), v);
}

// The codes of a lane's 16 x 8 patch, once the multipliers are known: renc[i]
// multiplies row i (rowwise codes, stored straight to rdst + i * row_pitch
// when row_store; with kRowHint under the L2 policy row_policy), cenc2[q] the
// column pair (2q, 2q+1) (colwise codes, handed to col_sink(half, cw): cw[q]
// holds rows 8*half .. 8*half+7 of column q, row 8*half in the low nibble).
// Shared by the NVFP4 and the MXFP4 casts.
template <bool kRowHint = false, class ColSink>
__device__ __forceinline__ void encode_codes(const uint4 (&v)[16], const float (&renc)[16],
                                             const uint64_t (&cenc2)[4], bool do_row, bool do_col,
                                             uint8_t* rdst, size_t row_pitch, bool row_store,
                                             ColSink&& col_sink, uint64_t row_policy = 0) {
#pragma unroll
  for (int half = 0; half < 2; half++) {
    uint32_t A[4], B[4];  // per row pair: codes of columns 0..3 / 4..7
#pragma unroll
    for (int pp = 0; pp < 4; pp++) {
      const int i = 8 * half + 2 * pp;
      const uint64_t x0[4] = {unpack2(v[i].x), unpack2(v[i].y), unpack2(v[i].z), unpack2(v[i].w)};
      const uint64_t x1[4] = {unpack2(v[i + 1].x), unpack2(v[i + 1].y), unpack2(v[i + 1].z),
                              unpack2(v[i + 1].w)};
      if (do_row) {
        const uint64_t e0 = pack2(renc[i], renc[i]), e1 = pack2(renc[i + 1], renc[i + 1]);
        const uint32_t w0 = e2m1_pairs(mul2x(x0[0], e0), mul2x(x0[1], e0), mul2x(x0[2], e0), mul2x(x0[3], e0));
        const uint32_t w1 = e2m1_pairs(mul2x(x1[0], e1), mul2x(x1[1], e1), mul2x(x1[2], e1), mul2x(x1[3], e1));
        if (row_store) {  // false for a 16-row block past the routed rows
          if (kRowHint) {
            st_global_u32_hint(rdst + i * row_pitch, w0, row_policy);
            st_global_u32_hint(rdst + (i + 1) * row_pitch, w1, row_policy);
          } else {
            st_global_u32(rdst + i * row_pitch, w0);
            st_global_u32(rdst + (i + 1) * row_pitch, w1);
          }
        }
      }
      if (do_col) {
        uint64_t y0[4], y1[4];
#pragma unroll
        for (int q = 0; q < 4; q++) {
          y0[q] = mul2x(x0[q], cenc2[q]);
          y1[q] = mul2x(x1[q], cenc2[q]);
        }
        // byte q of A = codes of (row i, row i+1) in column q
        A[pp] = e2m1_cross(y0[0], y1[0], y0[1], y1[1]);
        B[pp] = e2m1_cross(y0[2], y1[2], y0[3], y1[3]);
      }
    }
    if (do_col) {
      // 4x4 byte transposes: the word of column q = bytes A[0..3][q], rows
      // 8*half .. 8*half+7 of this lane's block, staged right away
      uint32_t cw[8];
      const uint32_t t0 = prmt(A[0], A[1], 0x5140), t1 = prmt(A[0], A[1], 0x7362);
      const uint32_t t2 = prmt(A[2], A[3], 0x5140), t3 = prmt(A[2], A[3], 0x7362);
      cw[0] = prmt(t0, t2, 0x5410);
      cw[1] = prmt(t0, t2, 0x7632);
      cw[2] = prmt(t1, t3, 0x5410);
      cw[3] = prmt(t1, t3, 0x7632);
      const uint32_t u0 = prmt(B[0], B[1], 0x5140), u1 = prmt(B[0], B[1], 0x7362);
      const uint32_t u2 = prmt(B[2], B[3], 0x5140), u3 = prmt(B[2], B[3], 0x7362);
      cw[4] = prmt(u0, u2, 0x5410);
      cw[5] = prmt(u0, u2, 0x7632);
      cw[6] = prmt(u1, u3, 0x5410);
      cw[7] = prmt(u1, u3, 0x7632);
      col_sink(half, cw);
    }
  }
}

// The shared tables a tile's encode reads: the E4M3 table of the block-scale
// shortcut, and S_enc of the tile's 128 rows.
struct EncodeTables {
  const E4m3Table* e4m3;
  const float* row_senc;
};

// S_enc of the lane's 8 columns as four pairs (2q, 2q+1), from a 128-entry
// table of the tile's columns.
__device__ __forceinline__ void col_senc_pairs(const float* col_senc, int cc, uint64_t (&cse)[4]) {
  const uint64_t* se = reinterpret_cast<const uint64_t*>(&col_senc[8 * cc]);
#pragma unroll
  for (int q = 0; q < 4; q++) cse[q] = se[q];
}

// Everything one lane does for one tile after its 16 x 8 patch is in
// registers: block scales of both directions, all codes, the rowwise data
// stores, the staging of the block scales (col_stg: [row block][column],
// row_stg: [column block][row], both 128 wide) and the colwise codes handed
// to col_sink. cc (0..15) is the lane's 8-column chunk of the tile, rb (0..7)
// its 16-row block; the other half of each of its rowwise blocks is on lane
// cc ^ 1 (the neighbouring lane). cse: S_enc of the lane's 8 columns in
// pairs (2q, 2q+1). kExact selects the IEEE-divide block scales (tiles with a
// row or column amax outside the shortcut's range).
template <bool kExact, bool kRowHint = false, class ColSink>
__device__ __forceinline__ void encode_patch(const uint4 (&v)[16], const EncodeTables& tab, const uint64_t (&cse)[4],
                                             uint8_t* col_stg, uint8_t* row_stg, bool do_row, bool do_col, int cc,
                                             int rb, uint8_t* rdst, size_t row_pitch, bool row_store,
                                             ColSink&& col_sink, uint64_t row_policy = 0) {
  const int rl = 16 * rb;
  const bool odd = cc & 1;

  // ------------------------------------------------------ colwise scales
  uint64_t cenc2[4];  // {enc of column 2q, enc of column 2q+1}
  if (do_col) {
    uint32_t m0 = v[0].x, m1 = v[0].y, m2 = v[0].z, m3 = v[0].w;
#pragma unroll
    for (int i = 1; i < 16; i++) {
      m0 = maxabs2(m0, v[i].x);
      m1 = maxabs2(m1, v[i].y);
      m2 = maxabs2(m2, v[i].z);
      m3 = maxabs2(m3, v[i].w);
    }
    const uint32_t mw[4] = {m0 & 0x7FFF7FFFu, m1 & 0x7FFF7FFFu, m2 & 0x7FFF7FFFu,
                            m3 & 0x7FFF7FFFu};
    uint32_t s8w[2] = {0u, 0u};
#pragma unroll
    for (int q = 0; q < 4; q++) {
      const uint32_t p2 = scales2x_any<kExact>(unpack2(mw[q]), cse[q], *tab.e4m3, cenc2[q]);
      s8w[q >> 1] |= p2 << (16 * (q & 1));
    }
    *reinterpret_cast<uint2*>(&col_stg[rb * kCols + 8 * cc]) = make_uint2(s8w[0], s8w[1]);
  } else {
#pragma unroll
    for (int q = 0; q < 4; q++) cenc2[q] = 0;
  }

  // ------------------------------------------------------ rowwise scales
  float renc[16];  // element multiplier of row i
  if (do_row) {
    uint32_t P[8];  // (row 2k, row 2k+1) maxima over the lane's 8 columns
#pragma unroll
    for (int kk = 0; kk < 8; kk++) {
      const uint32_t a = maxabs2(maxabs2(v[2 * kk].x, v[2 * kk].y), maxabs2(v[2 * kk].z, v[2 * kk].w));
      const uint32_t b = maxabs2(maxabs2(v[2 * kk + 1].x, v[2 * kk + 1].y),
                                 maxabs2(v[2 * kk + 1].z, v[2 * kk + 1].w));
      P[kk] = maxabs2(prmt(a, b, 0x5410), prmt(a, b, 0x7632)) & 0x7FFF7FFFu;
    }
    // The even lane of a pair scales rows 0..7, the odd lane rows 8..15: each
    // sends the partner the half-block maxima of the partner's rows, and
    // scales its own rows two at a time (row pairs are the f32x2 pairs).
    const uint64_t* rse = reinterpret_cast<const uint64_t*>(&tab.row_senc[rl + (odd ? 8 : 0)]);
    uint64_t mine[4];  // {enc of row 2k, of row 2k+1} of the lane's 8 rows
    uint32_t s8w[2] = {0u, 0u};
#pragma unroll
    for (int kk = 0; kk < 4; kk++) {
      const uint32_t send = odd ? P[kk] : P[kk + 4];
      const uint32_t keep = odd ? P[kk + 4] : P[kk];
      const uint32_t full = umax2(keep, __shfl_xor_sync(0xFFFFFFFFu, send, 1));
      const uint32_t p2 = scales2x_any<kExact>(unpack2(full), rse[kk], *tab.e4m3, mine[kk]);
      s8w[kk >> 1] |= p2 << (16 * (kk & 1));
    }
    *reinterpret_cast<uint2*>(&row_stg[(cc >> 1) * kRows + rl + (odd ? 8 : 0)]) = make_uint2(s8w[0], s8w[1]);
    // rows 0..7's multipliers come from the even lane, rows 8..15's from the odd one
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int kk = 0; kk < 4; kk++) {
      renc[2 * kk] = __shfl_sync(0xFFFFFFFFu, lo_of(mine[kk]), lane & ~1);
      renc[2 * kk + 1] = __shfl_sync(0xFFFFFFFFu, hi_of(mine[kk]), lane & ~1);
      renc[8 + 2 * kk] = __shfl_sync(0xFFFFFFFFu, lo_of(mine[kk]), lane | 1);
      renc[9 + 2 * kk] = __shfl_sync(0xFFFFFFFFu, hi_of(mine[kk]), lane | 1);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 16; i++) renc[i] = 0.0f;
  }

  // -------------------------------------------------------------- codes
  encode_codes<kRowHint>(v, renc, cenc2, do_row, do_col, rdst, row_pitch, row_store, col_sink, row_policy);
}

// The 128x4-tiled scale layout (the grouped GEMM's swizzle contract; see the
// oracle for the reading): in a 512-byte tile, scale (r, c) sits at byte
// (r % 32) * 16 + (r / 32) * 4 + c. A tile of this kernel fills two such
// tiles; thread t (of 128) writes 8 bytes of tile t / 64: rows q, q + 32 (t
// even) or q + 64, q + 96 (t odd) with q = (t / 2) % 32, columns 0..3 each,
// taken from staged scales stg[c * 128 + r] (c = 16-element block 0..3).
__device__ __forceinline__ uint32_t tiled_piece_offset(int t) { return 16u * ((t >> 1) & 31) + 8u * (t & 1); }

__device__ __forceinline__ uint2 tiled_piece(const uint8_t* stg, int t) {
  const int q = (t >> 1) & 31, i0 = 2 * (t & 1);
  uint32_t w[2];
#pragma unroll
  for (int ii = 0; ii < 2; ii++) {
    const int r = q + 32 * (i0 + ii);
    w[ii] = static_cast<uint32_t>(stg[r]) | (static_cast<uint32_t>(stg[kRows + r]) << 8) |
            (static_cast<uint32_t>(stg[2 * kRows + r]) << 16) | (static_cast<uint32_t>(stg[3 * kRows + r]) << 24);
  }
  return make_uint2(w[0], w[1]);
}

// The staged block scales of a tile of a 128-aligned group: colwise
// (col_stg [row block][column]) 8 bytes per column, rowwise (row_stg
// [column block][row]) 8 bytes per row, compact or as two whole 128x4 tiles
// per direction (kTiled).
template <bool kTiled>
__device__ __forceinline__ void store_scales(const uint8_t* col_stg, const uint8_t* row_stg, const CastOut& out,
                                             int K, int32_t o_g, int64_t m_g, int32_t r0, int c0, int t,
                                             bool do_row, bool do_col, uint64_t keep) {
  if (do_col) {
    if (kTiled) {
      // the tile's 128 x 8 block scales are two whole 128x4 tiles of the
      // group's [K, m_g/16] scale matrix: tile row c0/128, tile columns
      // (r0 - o_g)/64 + 0, 1 (m_g/64 tiles per tile row)
      const int j = t >> 6;
      uint8_t* blk = out.col_scale + (static_cast<size_t>(K) * o_g >> 4) +
                     ((static_cast<size_t>(c0 >> 7) * (static_cast<size_t>(m_g) >> 6)) + ((r0 - o_g) >> 6) + j) * 512;
      st_global_u2_hint(blk + tiled_piece_offset(t), tiled_piece(col_stg + 4 * j * kCols, t), keep);
    } else {
      const size_t m16 = static_cast<size_t>(m_g) >> 4;
      uint8_t* gs = out.col_scale + (static_cast<size_t>(K) * o_g >> 4) + ((r0 - o_g) >> 4);
      uint32_t s0 = 0u, s1 = 0u;
#pragma unroll
      for (int r = 0; r < 4; r++) {
        s0 |= static_cast<uint32_t>(col_stg[r * kCols + t]) << (8 * r);
        s1 |= static_cast<uint32_t>(col_stg[(r + 4) * kCols + t]) << (8 * r);
      }
      st_global_u2_hint(gs + static_cast<size_t>(c0 + t) * m16, make_uint2(s0, s1), keep);
    }
  }
  if (do_row) {
    if (kTiled) {
      // two whole 128x4 tiles of the [rows, K/16] scale matrix: tile row
      // r0/128, tile columns c0/64 + 0, 1 (K/64 tiles per tile row)
      const int j = t >> 6;
      uint8_t* blk = out.row_scale + (static_cast<size_t>(r0 >> 7) * (K >> 6) + (c0 >> 6) + j) * 512;
      st_global_u2_hint(blk + tiled_piece_offset(t), tiled_piece(row_stg + 4 * j * kRows, t), keep);
    } else {
      uint32_t s0 = 0u, s1 = 0u;
#pragma unroll
      for (int r = 0; r < 4; r++) {
        s0 |= static_cast<uint32_t>(row_stg[r * kRows + t]) << (8 * r);
        s1 |= static_cast<uint32_t>(row_stg[(r + 4) * kRows + t]) << (8 * r);
      }
      st_global_u2_hint(out.row_scale + static_cast<size_t>(r0 + t) * (K >> 4) + (c0 >> 4),
                        make_uint2(s0, s1), keep);
    }
  }
}

}  // namespace nvfp4rs
