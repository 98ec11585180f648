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
// Work split. A CTA (4 warps) owns one 128-row tile (inside one group) and up
// to kColTilesPerCta consecutive 128-column tiles of it. For each 128 x 128
// tile, lane (cc, h) of warp w loads rows 32w + 16h + i (i < 16), columns
// 8cc .. 8cc+7 with 16-byte loads -- one 16-row x 8-column patch, held in
// registers. From that patch alone it has:
//  - 8 complete colwise blocks (16 rows of one column each), and
//  - 16 half rowwise blocks (8 of 16 columns), completed with lane cc ^ 1.
// So both directions are encoded from the same registers, with no shared
// memory transpose of the input. Shared memory only stages the outputs that
// are not contiguous per lane -- colwise data and scales and rowwise scales
// -- so that every global store is a full 16- or 8-byte piece of a
// contiguous run.
//
// Extra CTAs at the front of the grid (only when the colwise direction is
// requested) write col_s2 = S_dec(col_amax) for all E*K entries, empty groups
// included.
#pragma once

#include "codec.cuh"
#include "routing.cuh"

namespace nvfp4rs {

constexpr int kCastThreads = 128;
constexpr int kColTilesPerCta = 4;
constexpr int kCols = 128;

struct CastOut {
  uint8_t* row_data;
  uint8_t* row_scale;
  float* row_s2;
  uint8_t* col_data;
  uint8_t* col_scale;
  float* col_s2;
};

// Per-tile output staging (one buffer; the kernel double-buffers it).
struct CastStage {
  uint8_t col_data[kCols * 64];     // [column][64 B]; 8-byte slot b at (b ^ (column/8 % 8))
  uint8_t col_scale[8 * kCols];     // [row block][column]
  uint8_t row_scale[8 * kRows];     // [column block][row]
};

__device__ __forceinline__ void st_global_u32(uint8_t* p, uint32_t v) {
  *reinterpret_cast<uint32_t*>(p) = v;
}

template <class Routing>
__global__ void __launch_bounds__(kCastThreads)
group_cast_kernel(const __grid_constant__ Routing routing, const uint4* __restrict__ x,
                  int32_t K, int32_t n_col_groups, int32_t n_s2_ctas,
                  const float* __restrict__ row_amax, const float* __restrict__ col_amax,
                  const CastOut out) {
  __shared__ RoutingSmem rs;
  __shared__ float row_senc[kRows];
  __shared__ float col_senc[kColTilesPerCta * kCols];
  __shared__ __align__(16) CastStage stage[2];

  routing.load(rs);
  if (!rs.ok) return;

  const int t = threadIdx.x;
  const bool do_row = out.row_data != nullptr;
  const bool do_col = out.col_data != nullptr;

  // ---- decode scales of the columns (all groups, empty ones included)
  if (static_cast<int>(blockIdx.x) < n_s2_ctas) {
    const int64_t n = static_cast<int64_t>(rs.E) * K;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * kCastThreads + t; i < n;
         i += static_cast<int64_t>(n_s2_ctas) * kCastThreads)
      out.col_s2[i] = s_dec_of(col_amax[i]);
    return;
  }

  const int b = blockIdx.x - n_s2_ctas;
  const int tile = b / n_col_groups;
  const int cgrp = b % n_col_groups;
  const int32_t r0 = tile * kRows;
  if (r0 >= rs.total) return;

  const int g = group_of_row(rs, r0);
  const int32_t o_g = rs.off[g];
  const int64_t m_g = rs.off[g + 1] - o_g;
  const int ct0 = cgrp * kColTilesPerCta;
  const int nct = min(kColTilesPerCta, (K >> 7) - ct0);

  // ---- second-level scales of this CTA's rows and columns
  if (do_row) {
    const float a = row_amax[r0 + t];
    row_senc[t] = s_enc_of(a);
    if (cgrp == 0) out.row_s2[r0 + t] = s_dec_of(a);
  }
  if (do_col) {
    const float* ca = col_amax + static_cast<size_t>(g) * K + ct0 * kCols;
    for (int j = t; j < nct * kCols; j += kCastThreads) col_senc[j] = s_enc_of(ca[j]);
  }
  __syncthreads();

  const int lane = t & 31, warp = t >> 5;
  const int cc = lane & 15, h = lane >> 4;
  const int rb = 2 * warp + h;  // 16-row block of the tile, 0..7
  const int rl = 16 * rb;       // first tile row of this lane
  const bool odd = cc & 1;
  const size_t K8 = static_cast<size_t>(K) >> 3;

  for (int j = 0; j < nct; j++) {
    const int c0 = (ct0 + j) * kCols;
    CastStage& st = stage[j & 1];

    uint4 v[16];
    {
      const uint4* p = x + static_cast<size_t>(r0 + rl) * K8 + ((c0 >> 3) + cc);
#pragma unroll
      for (int i = 0; i < 16; i++) v[i] = p[i * K8];
    }

    // ---------------------------------------------------- colwise scales
    float cenc[8];
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
      const float* se = &col_senc[j * kCols + 8 * cc];
      uint32_t s8w[2] = {0u, 0u};
#pragma unroll
      for (int q = 0; q < 4; q++) {
        const uint32_t p2 = block_scales2(bf16lo(mw[q]), se[2 * q], bf16hi(mw[q]), se[2 * q + 1],
                                          cenc[2 * q], cenc[2 * q + 1]);
        s8w[q >> 1] |= p2 << (16 * (q & 1));
      }
      // scales of column 8cc+q, row block rb -> col_scale stage [rb][column]
      *reinterpret_cast<uint2*>(&st.col_scale[rb * kCols + 8 * cc]) = make_uint2(s8w[0], s8w[1]);
    }

    // ---------------------------------------------------- rowwise scales
    float renc[16];
    if (do_row) {
      uint32_t P[8];  // (row 2k, row 2k+1) partial maxima over this lane's 8 columns
#pragma unroll
      for (int k = 0; k < 8; k++) {
        const uint32_t a = maxabs2(maxabs2(v[2 * k].x, v[2 * k].y), maxabs2(v[2 * k].z, v[2 * k].w));
        const uint32_t bb = maxabs2(maxabs2(v[2 * k + 1].x, v[2 * k + 1].y),
                                    maxabs2(v[2 * k + 1].z, v[2 * k + 1].w));
        P[k] = maxabs2(prmt(a, bb, 0x5410), prmt(a, bb, 0x7632)) & 0x7FFF7FFFu;
        P[k] = umax2(P[k], __shfl_xor_sync(0xFFFFFFFFu, P[k], 1));  // whole 16-column block
      }
      // the even lane of a pair scales rows 0..7, the odd lane rows 8..15
      float mine[8];
      uint32_t s8mine[2] = {0u, 0u};
#pragma unroll
      for (int k = 0; k < 4; k++) {
        const uint32_t w = odd ? P[4 + k] : P[k];
        const int rr = rl + (odd ? 8 : 0) + 2 * k;
        const uint32_t p2 = block_scales2(bf16lo(w), row_senc[rr], bf16hi(w), row_senc[rr + 1],
                                          mine[2 * k], mine[2 * k + 1]);
        s8mine[k >> 1] |= p2 << (16 * (k & 1));
      }
      float other[8];
#pragma unroll
      for (int k = 0; k < 8; k++) other[k] = __shfl_xor_sync(0xFFFFFFFFu, mine[k], 1);
#pragma unroll
      for (int k = 0; k < 8; k++) {
        renc[k] = odd ? other[k] : mine[k];
        renc[8 + k] = odd ? mine[k] : other[k];
      }
      const uint32_t so0 = __shfl_xor_sync(0xFFFFFFFFu, s8mine[0], 1);
      const uint32_t so1 = __shfl_xor_sync(0xFFFFFFFFu, s8mine[1], 1);
      if (!odd) {
        // 16 scale bytes of column block cc/2 for rows rl .. rl+15
        *reinterpret_cast<uint4*>(&st.row_scale[(cc >> 1) * kRows + rl]) =
            make_uint4(s8mine[0], s8mine[1], so0, so1);
      }
    }

    // ---------------------------------------------------- codes
    uint8_t* rdst = do_row ? out.row_data + static_cast<size_t>(r0 + rl) * (K >> 1) + (c0 >> 1) + 4 * cc
                           : nullptr;
    uint32_t cw[2][8];  // colwise words: [rows 0-7 | 8-15][column q]
#pragma unroll
    for (int half = 0; half < 2; half++) {
      uint32_t A[4], B[4];  // per row pair: codes of columns 0..3 / 4..7
#pragma unroll
      for (int pp = 0; pp < 4; pp++) {
        const int i = 8 * half + 2 * pp;
        const uint4 w0 = v[i], w1 = v[i + 1];
        if (do_row) {
          st_global_u32(rdst + static_cast<size_t>(i) * (K >> 1), encode_chunk(w0, renc[i]));
          st_global_u32(rdst + static_cast<size_t>(i + 1) * (K >> 1), encode_chunk(w1, renc[i + 1]));
        }
        if (do_col) {
          const uint32_t a[4] = {w0.x, w0.y, w0.z, w0.w};
          const uint32_t c[4] = {w1.x, w1.y, w1.z, w1.w};
          float y0[8], y1[8];
#pragma unroll
          for (int q = 0; q < 4; q++) {
            mul2(bf16lo(a[q]), bf16hi(a[q]), cenc[2 * q], cenc[2 * q + 1], y0[2 * q], y0[2 * q + 1]);
            mul2(bf16lo(c[q]), bf16hi(c[q]), cenc[2 * q], cenc[2 * q + 1], y1[2 * q], y1[2 * q + 1]);
          }
          // byte q of A = codes of (row i, row i+1) in column q
          A[pp] = e2m1x2x4(y0[0], y1[0], y0[1], y1[1], y0[2], y1[2], y0[3], y1[3]);
          B[pp] = e2m1x2x4(y0[4], y1[4], y0[5], y1[5], y0[6], y1[6], y0[7], y1[7]);
        }
      }
      if (do_col) {
        // 4x4 byte transposes: word for column q = bytes A[0..3][q]
        const uint32_t t0 = prmt(A[0], A[1], 0x5140), t1 = prmt(A[0], A[1], 0x7362);
        const uint32_t t2 = prmt(A[2], A[3], 0x5140), t3 = prmt(A[2], A[3], 0x7362);
        cw[half][0] = prmt(t0, t2, 0x5410);
        cw[half][1] = prmt(t0, t2, 0x7632);
        cw[half][2] = prmt(t1, t3, 0x5410);
        cw[half][3] = prmt(t1, t3, 0x7632);
        const uint32_t u0 = prmt(B[0], B[1], 0x5140), u1 = prmt(B[0], B[1], 0x7362);
        const uint32_t u2 = prmt(B[2], B[3], 0x5140), u3 = prmt(B[2], B[3], 0x7362);
        cw[half][4] = prmt(u0, u2, 0x5410);
        cw[half][5] = prmt(u0, u2, 0x7632);
        cw[half][6] = prmt(u1, u3, 0x5410);
        cw[half][7] = prmt(u1, u3, 0x7632);
      }
    }
    if (do_col) {
      const int slot = rb ^ (cc & 7);
#pragma unroll
      for (int q = 0; q < 8; q++) {
        *reinterpret_cast<uint2*>(&st.col_data[(8 * cc + q) * 64 + 8 * slot]) =
            make_uint2(cw[0][q], cw[1][q]);
      }
    }
    __syncthreads();

    // ---------------------------------------------------- staged stores
    if (do_col) {
      const size_t half_m = static_cast<size_t>(m_g) >> 1;
      uint8_t* gd = out.col_data + (static_cast<size_t>(K) * o_g >> 1) + ((r0 - o_g) >> 1);
#pragma unroll
      for (int k = 0; k < 4; k++) {
        const int u = k * kCastThreads + t;
        const int col = u >> 2, part = u & 3;
        const int s = (col >> 3) & 7;
        const uint2 lo = *reinterpret_cast<const uint2*>(&st.col_data[col * 64 + 8 * ((2 * part) ^ s)]);
        const uint2 hi = *reinterpret_cast<const uint2*>(&st.col_data[col * 64 + 8 * ((2 * part + 1) ^ s)]);
        *reinterpret_cast<uint4*>(gd + static_cast<size_t>(c0 + col) * half_m + 16 * part) =
            make_uint4(lo.x, lo.y, hi.x, hi.y);
      }
      const size_t m16 = static_cast<size_t>(m_g) >> 4;
      uint8_t* gs = out.col_scale + (static_cast<size_t>(K) * o_g >> 4) + ((r0 - o_g) >> 4);
      uint32_t s0 = 0u, s1 = 0u;
#pragma unroll
      for (int r = 0; r < 4; r++) {
        s0 |= static_cast<uint32_t>(st.col_scale[r * kCols + t]) << (8 * r);
        s1 |= static_cast<uint32_t>(st.col_scale[(r + 4) * kCols + t]) << (8 * r);
      }
      *reinterpret_cast<uint2*>(gs + static_cast<size_t>(c0 + t) * m16) = make_uint2(s0, s1);
    }
    if (do_row) {
      uint32_t s0 = 0u, s1 = 0u;
#pragma unroll
      for (int r = 0; r < 4; r++) {
        s0 |= static_cast<uint32_t>(st.row_scale[r * kRows + t]) << (8 * r);
        s1 |= static_cast<uint32_t>(st.row_scale[(r + 4) * kRows + t]) << (8 * r);
      }
      *reinterpret_cast<uint2*>(out.row_scale + static_cast<size_t>(r0 + t) * (K >> 4) + (c0 >> 4)) =
          make_uint2(s0, s1);
    }
  }
}

}  // namespace nvfp4rs
