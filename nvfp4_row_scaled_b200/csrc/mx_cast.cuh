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
// Structure: the NVFP4 cast kernel's (group_cast_plain.cuh) -- one CTA per
// SM of three warp groups, each with its own one-stage TMA ring, 16-row x
// 8-column lane patches, rowwise and colwise codes straight from registers to
// global memory -- with the MXFP4 block rule and no amax inputs. A rowwise
// block (32 columns) spans four lanes (lanes ^1, ^2), a colwise block (32
// rows) two lanes of the same warp (lane ^ 8: the neighbouring 16-row block).
// Groups are multiples of 32 rows, so a 32-row block lies in one group, and K
// is a multiple of 32. As in the NVFP4 cast, a plain loop serves routings whose
// groups are multiples of 128 rows with K % 128 == 0, and a general loop the
// rest (the short last row tile, tiles a group boundary crosses, groups off
// the 128-row grid, a partial last column tile).
#pragma once

#include "group_cast_plain.cuh"

namespace nvfp4rs {

// E8M0 code of a block whose amax has bf16 bits `b` (sign clear)
__device__ __forceinline__ uint32_t mx_code(uint32_t b) {
  const uint32_t e = (b >> 7) & 0xFFu;
  return e > 2u ? e - 2u : 0u;
}

// the element multiplier 2^-s of a block with E8M0 code `code`
__device__ __forceinline__ float mx_mult(uint32_t code) { return __uint_as_float((254u - code) << 23); }

// One lane's 16 x 8 patch: E8M0 scales of both directions, staged as
// col_stg [32-row block][column] and row_stg [32-column block][row] (both 128
// wide), and all codes (encode_codes). cc (0..15) is the lane's 8-column
// chunk, rb (0..7) its 16-row block.
template <class ColSink>
__device__ __forceinline__ void mx_encode_patch(const uint4 (&v)[16], uint8_t* col_stg, uint8_t* row_stg, bool do_row,
                                                bool do_col, int cc, int rb, uint8_t* rdst, size_t row_pitch,
                                                bool row_store, ColSink&& col_sink) {
  const int rl = 16 * rb;
  // ----------------------------------- colwise: 32-row blocks (lanes ^ 8)
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
      m[q] = umax2(m[q], __shfl_xor_sync(0xFFFFFFFFu, m[q], 8));
      const uint32_t lo = mx_code(m[q] & 0xFFFFu), hi = mx_code(m[q] >> 16);
      cmul2[q] = pack2(mx_mult(lo), mx_mult(hi));
      cw[q >> 1] |= (lo | (hi << 8)) << (16 * (q & 1));
    }
    if ((rb & 1) == 0)  // block rb / 2 of the tile, columns 8cc .. 8cc+7
      *reinterpret_cast<uint2*>(&col_stg[(rb >> 1) * kCols + 8 * cc]) = make_uint2(cw[0], cw[1]);
  } else {
#pragma unroll
    for (int q = 0; q < 4; q++) cmul2[q] = 0;
  }
  // ------------------------------- rowwise: 32-column blocks (lanes ^1, ^2)
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
      *reinterpret_cast<uint4*>(&row_stg[(cc >> 2) * kRows + rl]) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
  } else {
#pragma unroll
    for (int i = 0; i < 16; i++) rmul[i] = 0.0f;
  }
  encode_codes(v, rmul, cmul2, do_row, do_col, rdst, row_pitch, row_store, col_sink);
}

// Outputs of the MXFP4 cast (device pointers; a direction with both NULL is skipped).
struct MxOut {
  uint8_t* row_data;   // [rows, K/2]
  uint8_t* row_scale;  // [rows, K/32]
  uint8_t* col_data;   // per group [K, m_g/2] at byte K*o_g/2
  uint8_t* col_scale;  // per group [K, m_g/32] at byte K*o_g/32
};

struct alignas(16) MxGroup {
  uint8_t col_scale[2][4 * kCols];  // staged colwise scales [32-row block][column]
  uint8_t row_scale[2][4 * kRows];  // staged rowwise scales [32-column block][row]
  TileInfo info[kPInfo];
  uint64_t full;  // the stage's mbarrier: tile k completes phase k % 2
  int32_t fail;
};

// Dynamic shared memory of the kernel; `off` (E+1 int32) follows it.
struct MxSmem {
  uint8_t tile[kPGroups][kTileBytes];  // one stage per group, at offset 0 of a 1024-byte aligned block
  MxGroup grp[kPGroups];
  RoutingSmem rs;
};

constexpr size_t mx_smem_bytes(int E) {
  return ((sizeof(MxSmem) + 15) & ~size_t{15}) + sizeof(int32_t) * (E + 1);
}

// One thread of the group: tile (rt, ct) -- the group's k-th -- into the
// stage with its tile info (as plain_info and plain_load of the NVFP4 cast
// together, without amax copies; the info is written when the tile is issued,
// one tile ahead, and read after the next barrier).
__device__ __forceinline__ void mx_issue(MxGroup& pg, uint8_t* stage, const CUtensorMap* map, int k, int rt,
                                         int ct, const RoutingSmem& rs, int K, bool k128) {
  const int32_t r0 = rt * kRows;
  const int c0 = ct * kCols;
  const int g = group_of_row(rs, r0);
  TileInfo& inf = pg.info[k % kPInfo];
  const int32_t o_g = rs.off[g], m_g = rs.off[g + 1] - o_g;
  const int32_t valid = min(kRows, rs.total - r0);
  const int32_t kcols = min(kCols, K - c0);
  const bool mixed = o_g + m_g < r0 + valid;
  inf.o_g = o_g;
  inf.m_g = m_g;
  inf.valid = valid;
  inf.kcols = kcols;
  inf.plain = !mixed && valid == kRows && k128 && ((o_g | m_g) & (kRows - 1)) == 0;
  inf.mixed = mixed;
  if (!inf.plain) {  // the group of each 16-row block (groups only move forward)
    int gb = g;
#pragma unroll
    for (int b = 0; b < 8; b++) {
      const int32_t r = r0 + kBlockRows * b;
      while (gb + 1 < rs.E && rs.off[gb + 1] <= r) gb++;
      inf.gb[b] = gb;
    }
  }
  mbar_expect_tx(&pg.full, kTileBytes);
  const uint64_t pol = policy_evict_first();
  tma_load_2d(stage, map, c0, r0, &pg.full, pol);
  tma_load_2d(stage + kBoxBytes, map, c0 + kBoxCols, r0, &pg.full, pol);
}

// The staged scales of a tile: a plain tile's as 4 bytes per column and per
// row; a general tile's byte by byte, per (column, 32-row block) to the
// block's own group and per row the blocks inside K, nothing past the routed
// rows or past K.
template <bool kGeneral>
__device__ __forceinline__ void mx_store_scales(const MxGroup& pg, int buf, const TileInfo& inf, const MxOut& out,
                                                const RoutingSmem& rs, int K, int32_t r0, int c0, int t, bool do_row,
                                                bool do_col) {
  const uint8_t* col_stg = pg.col_scale[buf];
  const uint8_t* row_stg = pg.row_scale[buf];
  if (!kGeneral || inf.plain) {
    if (do_col) {
      const uint32_t w = static_cast<uint32_t>(col_stg[t]) | (static_cast<uint32_t>(col_stg[kCols + t]) << 8) |
                         (static_cast<uint32_t>(col_stg[2 * kCols + t]) << 16) |
                         (static_cast<uint32_t>(col_stg[3 * kCols + t]) << 24);
      gstore(reinterpret_cast<uint32_t*>(out.col_scale + (static_cast<size_t>(K) * inf.o_g >> 5) +
                                         static_cast<size_t>(c0 + t) * (static_cast<size_t>(inf.m_g) >> 5) +
                                         ((r0 - inf.o_g) >> 5)),
             w);
    }
    if (do_row) {
      const uint32_t w = static_cast<uint32_t>(row_stg[t]) | (static_cast<uint32_t>(row_stg[kRows + t]) << 8) |
                         (static_cast<uint32_t>(row_stg[2 * kRows + t]) << 16) |
                         (static_cast<uint32_t>(row_stg[3 * kRows + t]) << 24);
      gstore(reinterpret_cast<uint32_t*>(out.row_scale + static_cast<size_t>(r0 + t) * (K >> 5) + (c0 >> 5)), w);
    }
    return;
  }
  if (do_col && t < inf.kcols) {
#pragma unroll
    for (int b = 0; b < 4; b++) {
      if (32 * b >= inf.valid) break;
      const int g = inf.gb[2 * b];
      const int32_t o = rs.off[g];
      const size_t m32 = static_cast<size_t>(rs.off[g + 1] - o) >> 5;
      gstore(&out.col_scale[(static_cast<size_t>(K) * o >> 5) + static_cast<size_t>(c0 + t) * m32 +
                            ((r0 + 32 * b - o) >> 5)],
             col_stg[b * kCols + t]);
    }
  }
  if (do_row && t < inf.valid) {
    uint8_t* dst = out.row_scale + static_cast<size_t>(r0 + t) * (static_cast<size_t>(K) >> 5) + (c0 >> 5);
#pragma unroll
    for (int b = 0; b < 4; b++) {
      if (32 * b >= inf.kcols) break;
      gstore(&dst[b], row_stg[b * kRows + t]);
    }
  }
}

// The tile loop of warp group j (thread gt of it); kGeneral as in cast_tiles.
template <bool kGeneral, class Routing>
__device__ __forceinline__ void mx_tiles(MxSmem& sm, MxGroup& pg, const Routing& routing, const CUtensorMap* tmap,
                                         int32_t K, const MxOut& out, int j, int gt, int first, int G, int n_ct,
                                         int n_tiles, bool k128, bool do_row, bool do_col) {
  const RoutingSmem& rs = sm.rs;
  const int lane = gt & 31, w = gt >> 5;
  const int cc = 8 * (w & 1) + (lane & 7);  // 8-column chunk of the tile, 0..15
  const int rb = 4 * (w >> 1) + (lane >> 3);  // 16-row block of the tile, 0..7
  const int rl = 16 * rb;
  const size_t row_pitch = static_cast<size_t>(K) >> 1;
  const uint64_t keep = policy_evict_last();
  const int bar_id = 1 + j;
  const int Gq = G / n_ct, Gr = G - Gq * n_ct;
  int rt = first / n_ct, ct = first - rt * n_ct;
  int k = 0;
  bool failed = false;
  int rtp = 0, ctp = 0;
  for (int tl = first; tl < n_tiles; tl += G, k++) {
    const int32_t r0 = rt * kRows;
    const int c0 = ct * kCols;
    const bool ok = mbar_wait(&pg.full, k & 1);
    if (!ok) pg.fail = 1;
    uint4 v[16];
    load_patch(sm.tile[j], cc, rl, v);
    group_bar(bar_id);
    if (pg.fail) {
      failed = true;
      break;
    }
    // every patch of tile k is in registers: the stage takes tile k+1
    if (gt == 32 * (k & 3) && tl + G < n_tiles) {
      int rt2 = rt + Gq, ct2 = ct + Gr;
      if (ct2 >= n_ct) {
        ct2 -= n_ct;
        rt2++;
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mx_issue(pg, sm.tile[j], tmap, k + 1, rt2, ct2, rs, K, k128);
    }
    if (k >= 1)  // the previous tile's staged scales (complete since the barrier)
      mx_store_scales<kGeneral>(pg, (k - 1) & 1, pg.info[(k - 1) % kPInfo], out, rs, K, rtp * kRows, ctp * kCols, gt,
                                do_row, do_col);
    const TileInfo& inf = pg.info[k % kPInfo];
    int32_t o_l = inf.o_g, m_l = inf.m_g;
    bool lane_ok = true;
    if (kGeneral) {
      lane_ok = rl < inf.valid && 8 * cc < inf.kcols;
      if (!inf.plain) {
        const int gl = inf.gb[rb];
        o_l = rs.off[gl];
        m_l = rs.off[gl + 1] - o_l;
      }
    }
    const size_t half_m = static_cast<size_t>(m_l) >> 1;
    uint8_t* rdst = do_row ? out.row_data + static_cast<size_t>(r0 + rl) * row_pitch + (c0 >> 1) + 4 * cc : nullptr;
    DirectColSink sink{do_col ? out.col_data + (static_cast<size_t>(K) * o_l >> 1) +
                                    static_cast<size_t>(c0 + 8 * cc) * half_m + ((r0 - o_l + rl) >> 1)
                              : nullptr,
                       half_m, keep, do_col && lane_ok, {}};
    mx_encode_patch(v, pg.col_scale[k & 1], pg.row_scale[k & 1], do_row, do_col, cc, rb, rdst, row_pitch, lane_ok,
                    sink);
    rtp = rt;
    ctp = ct;
    ct += Gr;
    rt += Gq;
    if (ct >= n_ct) {
      ct -= n_ct;
      rt++;
    }
  }
  if (!failed && k >= 1) {  // the last tile's staged scales
    group_bar(bar_id);
    mx_store_scales<kGeneral>(pg, (k - 1) & 1, pg.info[(k - 1) % kPInfo], out, rs, K, rtp * kRows, ctp * kCols, gt,
                              do_row, do_col);
  }
  if (failed && gt == 0) {
    // drain the load this group issued and did not consume (tile k)
    mbar_wait(&pg.full, k & 1);
    routing.report(NVFP4_ERR_TIMEOUT);
  }
}

template <class Routing>
__global__ void __launch_bounds__(kPThreads, 1)
mx_cast_kernel(const __grid_constant__ Routing routing, const __grid_constant__ CUtensorMap tmap, int32_t K,
               const MxOut out) {
  // the 128-byte swizzle wants each stage 1024-byte aligned; the host adds
  // 1024 bytes of slack for this
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  MxSmem& sm = *reinterpret_cast<MxSmem*>(base);
  int32_t* off = reinterpret_cast<int32_t*>(base + ((sizeof(MxSmem) + 15) & ~size_t{15}));

  routing.load(sm.rs, off);
  const RoutingSmem& rs = sm.rs;
  if (!rs.ok) return;

  const int t = threadIdx.x;
  const bool do_row = out.row_data != nullptr;
  const bool do_col = out.col_data != nullptr;
  const int j = t / kCastThreads;  // warp group
  const int gt = t - j * kCastThreads;
  MxGroup& pg = sm.grp[j];
  const int n_ct = (K + kCols - 1) >> 7;
  const bool k128 = (K & (kCols - 1)) == 0;
  const int n_tiles = ((rs.total + kRows - 1) >> 7) * n_ct;  // the last row tile may be short
  const int G = gridDim.x * kPGroups;
  const int first = j * gridDim.x + blockIdx.x;  // groups running together take neighbouring tiles
  if (gt == 0) {
    mbar_init(&pg.full, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    pg.fail = 0;
  }
  __syncthreads();
  if (gt == 0) {
    const int rti = first / n_ct, cti = first - rti * n_ct;
    if (first < n_tiles) mx_issue(pg, sm.tile[j], &tmap, 0, rti, cti, rs, K, k128);
  }
  // every group a multiple of 128 rows and K % 128 == 0: every tile is plain
  if (rs.all128 && k128)
    mx_tiles<false>(sm, pg, routing, &tmap, K, out, j, gt, first, G, n_ct, n_tiles, k128, do_row, do_col);
  else
    mx_tiles<true>(sm, pg, routing, &tmap, K, out, j, gt, first, G, n_ct, n_tiles, k128, do_row, do_col);
}

}  // namespace nvfp4rs
