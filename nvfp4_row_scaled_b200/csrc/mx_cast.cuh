// mx_cast.cuh -- grouped MXFP4 cast (E2M1 data, 32-element blocks, one E8M0
// power-of-two scale per block), rowwise and colwise from one read of x.
//
// TransformerEngine #3824 (custom recipes for grouped GEMMs), Testing and
// item 1: the MXFP4 configuration is E2M1 data with block-32 E8M0 scales
// (the pow_2_scales branch); row-scaled NVFP4 is not combined with it, so
// there is no second-level scale and no amax pass: a block's scale depends
// on the block alone. The scale rule (not spelled out on the pages) is read
// as the OCP Microscaling conversion: shared exponent s = floor(log2 amax)
// - 2, clamped to [-127, 127], scale byte s + 127, elements encoded as
// E2M1_rne_satfinite(x * 2^-s). From the bf16 bits of the block amax that is
// code = max(E - 2, 0) with E its biased exponent (a zero or subnormal amax
// gives 0), and 2^-s = 2^(127 - s) is the float with biased exponent
// 254 - code, always normal; x * 2^-s is exact (a bf16 times a power of two,
// below 8 in magnitude).
//
// Structure: the cast kernel's persistent CTAs, TMA ring and 16-row x
// 8-column lane patches (group_cast.cuh), with the same 128-aligned groups.
// A rowwise block (32 columns) spans four lanes (cc .. cc+3, two shuffles);
// a colwise block (32 rows) spans the two half-warps (one shuffle). Codes go
// through the shared encode_codes; rowwise scales are staged as [block][row],
// colwise scales as [block][column], and stored as 4 bytes per row / column.
#pragma once

#include "group_cast.cuh"

namespace nvfp4rs {

// E8M0 code of a block whose amax has bf16 bits `b` (sign clear)
__device__ __forceinline__ uint32_t mx_code(uint32_t b) {
  const uint32_t e = (b >> 7) & 0xFFu;
  return e > 2u ? e - 2u : 0u;
}

// the element multiplier 2^-s of a block with E8M0 code `code`
__device__ __forceinline__ float mx_mult(uint32_t code) { return __uint_as_float((254u - code) << 23); }

__device__ __forceinline__ void mx_encode_patch(const uint4 (&v)[16], CastStage& st, bool do_row, bool do_col,
                                                int cc, int rb, uint8_t* rdst, size_t row_pitch) {
  const int rl = 16 * rb;
  // ---------------------------------------- colwise: 32-row blocks (h pairs)
  uint64_t cmul2[4];
  if (do_col) {
    uint32_t m[4] = {v[0].x, v[0].y, v[0].z, v[0].w};
#pragma unroll
    for (int i = 1; i < 16; i++) {
      m[0] = maxabs2(m[0], v[i].x);
      m[1] = maxabs2(m[1], v[i].y);
      m[2] = maxabs2(m[2], v[i].z);
      m[3] = maxabs2(m[3], v[i].w);
    }
    uint32_t cw[2] = {0u, 0u};
#pragma unroll
    for (int q = 0; q < 4; q++) {
      m[q] &= 0x7FFF7FFFu;
      m[q] = umax2(m[q], __shfl_xor_sync(0xFFFFFFFFu, m[q], 16));
      const uint32_t lo = mx_code(m[q] & 0xFFFFu), hi = mx_code(m[q] >> 16);
      cmul2[q] = pack2(mx_mult(lo), mx_mult(hi));
      cw[q >> 1] |= (lo | (hi << 8)) << (16 * (q & 1));
    }
    if ((rb & 1) == 0)  // block rb / 2 of the tile, columns 8cc .. 8cc+7
      *reinterpret_cast<uint2*>(&st.col_scale[(rb >> 1) * kCols + 8 * cc]) = make_uint2(cw[0], cw[1]);
  } else {
#pragma unroll
    for (int q = 0; q < 4; q++) cmul2[q] = 0;
  }
  // ------------------------------------- rowwise: 32-column blocks (4 lanes)
  float rmul[16];
  if (do_row) {
    uint32_t cw[4] = {0u, 0u, 0u, 0u};  // row i's code in byte i
#pragma unroll
    for (int kk = 0; kk < 8; kk++) {
      const uint32_t a = maxabs2(maxabs2(v[2 * kk].x, v[2 * kk].y), maxabs2(v[2 * kk].z, v[2 * kk].w));
      const uint32_t b = maxabs2(maxabs2(v[2 * kk + 1].x, v[2 * kk + 1].y),
                                 maxabs2(v[2 * kk + 1].z, v[2 * kk + 1].w));
      uint32_t P = maxabs2(prmt(a, b, 0x5410), prmt(a, b, 0x7632)) & 0x7FFF7FFFu;  // (row 2kk, 2kk+1)
      P = umax2(P, __shfl_xor_sync(0xFFFFFFFFu, P, 1));
      P = umax2(P, __shfl_xor_sync(0xFFFFFFFFu, P, 2));
      const uint32_t c0 = mx_code(P & 0xFFFFu), c1 = mx_code(P >> 16);
      rmul[2 * kk] = mx_mult(c0);
      rmul[2 * kk + 1] = mx_mult(c1);
      cw[kk >> 1] |= (c0 | (c1 << 8)) << (16 * (kk & 1));
    }
    if ((cc & 3) == 0)  // block cc / 4 of the tile, rows rl .. rl+15
      *reinterpret_cast<uint4*>(&st.row_scale[(cc >> 2) * kRows + rl]) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
  } else {
#pragma unroll
    for (int i = 0; i < 16; i++) rmul[i] = 0.0f;
  }
  encode_codes(v, rmul, cmul2, do_row, do_col, rdst, row_pitch, true, StageColSink{st, cc, rb});
}

// Outputs of the MXFP4 cast (device pointers; a direction with both NULL is skipped).
struct MxOut {
  uint8_t* row_data;   // [rows, K/2]
  uint8_t* row_scale;  // [rows, K/32]
  uint8_t* col_data;   // per group [K, m_g/2] at byte K*o_g/2
  uint8_t* col_scale;  // per group [K, m_g/32] at byte K*o_g/32
};

template <class Routing>
__global__ void __launch_bounds__(kCastThreads, 3)
mx_cast_kernel(const __grid_constant__ Routing routing, const __grid_constant__ CUtensorMap tmap, int32_t K,
               const MxOut out) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  CastSmem& sm = *reinterpret_cast<CastSmem*>(base);
  int32_t* off = reinterpret_cast<int32_t*>(base + ((sizeof(CastSmem) + 15) & ~size_t{15}));
  __shared__ RoutingSmem rs;

  routing.load(rs, off);
  if (!rs.ok) return;

  const int t = threadIdx.x;
  const bool do_row = out.row_data != nullptr;
  const bool do_col = out.col_data != nullptr;
  const int n_ct = K >> 7;
  const int n_tiles = (rs.total >> 7) * n_ct;
  const int G = gridDim.x;
  if (t == 0) {
    for (int s = 0; s < kStages; s++) mbar_init(&sm.full[s], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (t == 0) {
    for (int s = 0; s < kStages && blockIdx.x + s * G < n_tiles; s++)
      issue_tile(sm, &tmap, s, blockIdx.x + s * G, n_ct);
  }

  const int lane = t & 31, warp = t >> 5;
  const int cc = lane & 15, h = lane >> 4;
  const int rb = 2 * warp + h;
  const int rl = 16 * rb;
  const size_t row_pitch = static_cast<size_t>(K) >> 1;
  const uint64_t keep = policy_evict_last();
  int k = 0;
  bool failed = false;
  int cur_rt = -1, g = 0;
  int32_t o_g = 0;
  int64_t m_g = 0;
  for (int tl = blockIdx.x; tl < n_tiles; tl += G, k++) {
    const int s = k % kStages;
    const uint32_t phase = (k / kStages) & 1;
    const int rt = tl / n_ct, ct = tl - rt * n_ct;
    const int32_t r0 = rt * kRows;
    const int c0 = ct * kCols;
    if (rt != cur_rt) {
      cur_rt = rt;
      g = group_of_row(rs, r0);
      o_g = rs.off[g];
      m_g = rs.off[g + 1] - o_g;
    }
    const bool ok = mbar_wait(&sm.full[s], phase);
    uint4 v[16];
    load_patch(sm.tile[s], cc, rl, v);
    if (__syncthreads_or(!ok)) {
      failed = true;
      break;
    }
    // (issued by lane 0 of warp k % 4, so that the issue work does not always
    // delay the same warp at the next barrier)
    if (t == 32 * (k & 3) && k >= 1 && tl + G < n_tiles) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      issue_tile(sm, &tmap, (k + 1) % kStages, tl + G, n_ct);
    }
    CastStage& st = *reinterpret_cast<CastStage*>(sm.tile[s]);
    uint8_t* rdst = do_row ? out.row_data + static_cast<size_t>(r0 + rl) * row_pitch + (c0 >> 1) + 4 * cc : nullptr;
    mx_encode_patch(v, st, do_row, do_col, cc, rb, rdst, row_pitch);
    __syncthreads();
    // staged outputs: colwise codes (64 bytes per column), then 4 scale bytes
    // per column (colwise) and per row (rowwise)
    if (do_col) {
      store_col_data(st, out.col_data, K, o_g, m_g, r0, c0, t, keep);
      const uint32_t w = static_cast<uint32_t>(st.col_scale[t]) | (static_cast<uint32_t>(st.col_scale[kCols + t]) << 8) |
                         (static_cast<uint32_t>(st.col_scale[2 * kCols + t]) << 16) |
                         (static_cast<uint32_t>(st.col_scale[3 * kCols + t]) << 24);
      gstore(reinterpret_cast<uint32_t*>(out.col_scale + (static_cast<size_t>(K) * o_g >> 5) +
                                         static_cast<size_t>(c0 + t) * (static_cast<size_t>(m_g) >> 5) +
                                         ((r0 - o_g) >> 5)),
             w);
    }
    if (do_row) {
      const uint32_t w = static_cast<uint32_t>(st.row_scale[t]) | (static_cast<uint32_t>(st.row_scale[kRows + t]) << 8) |
                         (static_cast<uint32_t>(st.row_scale[2 * kRows + t]) << 16) |
                         (static_cast<uint32_t>(st.row_scale[3 * kRows + t]) << 24);
      gstore(reinterpret_cast<uint32_t*>(out.row_scale + static_cast<size_t>(r0 + t) * (K >> 5) + (c0 >> 5)), w);
    }
  }
  if (failed && t == 0) {
    for (int j = k; j <= (k == 0 ? 1 : k) && blockIdx.x + j * G < n_tiles; j++)
      mbar_wait(&sm.full[j % kStages], (j / kStages) & 1);
    routing.report(NVFP4_ERR_TIMEOUT);
  }
}

}  // namespace nvfp4rs
