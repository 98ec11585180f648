// group_cast_plain.cuh -- the grouped row-scaled NVFP4 cast kernel.
//
// TransformerEngine #3649 (grouped row-scaled NVFP4 cast), Description: the
// cast step takes the row and column amax vectors and writes the packed FP4
// data and scales of every group, rowwise and colwise (TransformerEngine
// #3324, summary). One kernel serves both routing front-ends and every
// routing: groups of any multiple of 16 rows, and K any multiple of 16.
//
// Tiles. x is cut into 128-row x 128-column tiles in row-major tile order.
// A "plain" tile lies inside one group whose rows start and end on the
// 128-row grid, holds 128 routed rows and 128 columns, and K is a multiple of
// 128: that is every tile of MoE routing padded to 128 rows, and it takes the
// fast path below. Every other tile is "general": the short last row tile
// (fewer than 128 routed rows), a tile that a group boundary crosses
// ("mixed"; group sizes are multiples of 16, so a lane's 16-row block always
// lies in one group), a tile of a group off the 128-row grid, and the last
// column tile when K % 128 != 0 (its columns past K are loaded as zeros by
// the TMA unit and never stored).
//
// Organisation (kept for the plain tiles, which the SM must keep issuing):
//  - One CTA per SM made of three independent warp groups of four warps
//    (named barriers 1..3), each with its own tile sequence, TMA ring and
//    mbarriers. The tables all groups read (E4M3 values and reciprocals,
//    group offsets) exist once per SM.
//  - One stage per group: the stage is refilled with the group's next tile
//    as soon as its warps hold their patches (one barrier per tile), so the
//    load of tile k+1 overlaps the encode of tile k while the SM's other two
//    groups keep their own loads in flight. (Two stages per group measured
//    slower: 1% on DeepSeek-V3 shapes at 4096 tokens, 3% at 1024 tokens, 8%
//    on an L2-resident 4096 x 7168 case.)
//    Colwise codes go from registers straight to global memory; the block
//    scales are staged in a double buffer and stored after the next tile's
//    barrier.
//  - Warp w covers rows 64*(w/2) .. +63 and columns 64*(w%2) .. +63 of the
//    tile; lane (hb, c8) holds 16 rows (block 4*(w/2) + hb) by 8 columns
//    (chunk 8*(w%2) + c8). A rowwise store instruction then writes four rows
//    x 32 contiguous bytes and a colwise one eight columns x 32 contiguous
//    bytes: whole sectors.
//  - A tile's row amax and (unless it is mixed) its group's column amax come
//    by bulk copy on the tile's mbarrier into a three-slot ring and are
//    turned into S_enc in place before the barrier. A lane of a mixed tile
//    loads the column amax of its own block's group itself.
//  - General tiles differ only at the edges: each lane finds its own block's
//    group for the colwise stores, lanes past the routed rows or past K store
//    nothing, and the staged scales are stored byte by byte
//    (store_scales_general).
// Ring invariants (tile k of a group): the stage completes phase k % 2 of
// its mbarrier, amax slot k % 3, tile info entry k % 4, scale staging k % 2.
// After tile k's barrier one thread loads tile k+1 into the stage and slot
// (k+1) % 3 (its info, entry (k+1) % 4, was written after tile k-1's
// barrier) and writes tile k+2's info into entry (k+2) % 4. Every read of
// the stage by tile k happened before that barrier; what tile k reads after
// it (slot k % 3, entry k % 4) and tile k-1's scale stores (entry
// (k-1) % 4, staging (k-1) % 2) are other entries; entry (k+2) % 4 was last
// read by tile k-2, before tile k-1's barrier.
#pragma once

#include "group_cast.cuh"

namespace nvfp4rs {

constexpr int kPGroups = 3;                         // warp groups per CTA
constexpr int kPThreads = kPGroups * kCastThreads;  // 384
constexpr int kPSlots = 3;                          // amax ring depth
constexpr int kPInfo = 4;                           // tile-info ring depth

// What the issuing thread records about a tile for the compute threads.
struct TileInfo {
  int32_t o_g;        // first row of the group of the tile's first row
  int32_t m_g;        // its rows
  int32_t valid;      // routed rows of the tile (a multiple of 16, <= 128)
  int32_t kcols;      // columns of the tile inside K (a multiple of 16, <= 128)
  int32_t plain;      // nonzero: the fast path applies (see the top of the file)
  int32_t mixed;      // nonzero: a group boundary crosses the tile's routed rows
  int32_t g;          // the group of the tile's first row
  int32_t gb[8];      // group of each 16-row block (general tiles only)
};

struct alignas(16) PlainGroup {
  float col_senc[kPSlots][kCols];   // bulk-copied column amax, then S_enc
  float row_senc[kPSlots][kRows];   // bulk-copied row amax, then S_enc
  uint8_t col_scale[2][8 * kCols];  // staged colwise block scales [row block][column]
  uint8_t row_scale[2][8 * kRows];  // staged rowwise block scales [column block][row]
  TileInfo info[kPInfo];
  uint64_t full;  // the stage's mbarrier: tile k completes phase k % 2
  int32_t fail;
};

// Dynamic shared memory of the kernel; `off` (E+1 int32) follows it.
struct PlainSmem {
  uint8_t tile[kPGroups][kTileBytes];  // one stage per group, at offset 0 of a 1024-byte aligned block
  PlainGroup grp[kPGroups];
  E4m3Table e4m3;
  RoutingSmem rs;
};

constexpr size_t plain_smem_bytes(int E) {
  return ((sizeof(PlainSmem) + 15) & ~size_t{15}) + sizeof(int32_t) * (E + 1);
}

// Named barrier of warp group `id - 1` (128 threads); returns the OR of pred.
__device__ __forceinline__ bool group_bar_or(int id, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(pred)), "r"(id), "n"(kCastThreads)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void group_bar(int id) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "n"(kCastThreads) : "memory");
}

// Colwise sink of encode_codes: the lane's 8 columns x 16 rows of codes, 8
// bytes per column, straight to its group's transposed data (half 0 is held
// until half 1 completes the column's piece). Inactive lanes (past the routed
// rows or past K) store nothing.
struct DirectColSink {
  uint8_t* dst;   // the lane's first column, at its 16-row block
  size_t pitch;   // bytes per column of the group (m_g / 2)
  uint64_t policy;
  bool active;
  uint32_t lo[8];
  __device__ __forceinline__ void operator()(int half, const uint32_t (&cw)[8]) {
    if (half == 0) {
#pragma unroll
      for (int q = 0; q < 8; q++) lo[q] = cw[q];
    } else if (active) {
#pragma unroll
      for (int q = 0; q < 8; q++) st_global_u2_hint(dst + q * pitch, make_uint2(lo[q], cw[q]), policy);
    }
  }
};

// One thread of the group: the info of tile (rt, ct), the group's k-th.
__device__ __noinline__ void plain_info(PlainGroup& pg, int k, int rt, int ct, const RoutingSmem& rs, int K,
                                           bool k128) {
  const int32_t r0 = rt * kRows;
  const int c0 = ct * kCols;
  const int g = group_of_row(rs, r0);
  TileInfo& inf = pg.info[k % kPInfo];
  const int32_t o_g = rs.off[g], m_g = rs.off[g + 1] - o_g;
  const int32_t valid = min(kRows, rs.total - r0);
  const int32_t kcols = min(kCols, K - c0);
  const bool mixed = o_g + m_g < r0 + valid;
  const bool plain = !mixed && valid == kRows && k128 && ((o_g | m_g) & (kRows - 1)) == 0;
  inf.o_g = o_g;
  inf.m_g = m_g;
  inf.valid = valid;
  inf.kcols = kcols;
  inf.plain = plain;
  inf.mixed = mixed;
  inf.g = g;
  if (!plain) {  // the group of each 16-row block (groups only move forward)
    int gb = g;
#pragma unroll
    for (int b = 0; b < 8; b++) {
      const int32_t r = r0 + kBlockRows * b;
      while (gb + 1 < rs.E && rs.off[gb + 1] <= r) gb++;
      inf.gb[b] = gb;
    }
  }
}

// The thread that wrote tile k's info (or one that met it at a barrier since):
// the tile into the stage with the row and column amax it needs (NULL:
// direction not requested), all completing on the stage's mbarrier. Only the
// routed rows' amax (valid rows) and the columns inside K are copied; the
// column amax are those of the group of the tile's first row (lanes of a
// mixed tile in another group load their own).
__device__ __forceinline__ void plain_load(PlainGroup& pg, uint8_t* stage, const CUtensorMap* map, int k, int rt,
                                           int ct, int K, const float* row_amax, const float* col_amax) {
  const int32_t r0 = rt * kRows;
  const int c0 = ct * kCols;
  const TileInfo& inf = pg.info[k % kPInfo];
  const int slot = k % kPSlots;
  const uint32_t col_bytes = col_amax != nullptr ? 4u * inf.kcols : 0u;
  const uint32_t row_bytes = row_amax != nullptr ? 4u * inf.valid : 0u;
  mbar_expect_tx(&pg.full, kTileBytes + col_bytes + row_bytes);
  const uint64_t pol = policy_evict_first();
  tma_load_2d(stage, map, c0, r0, &pg.full, pol);
  tma_load_2d(stage + kBoxBytes, map, c0 + kBoxCols, r0, &pg.full, pol);
  if (col_bytes != 0u)
    bulk_load(pg.col_senc[slot], col_amax + static_cast<size_t>(inf.g) * K + c0, col_bytes, &pg.full);
  if (row_bytes != 0u) bulk_load(pg.row_senc[slot], row_amax + r0, row_bytes, &pg.full);
}

// The staged block scales of a general tile: one byte per (column, 16-row
// block) to the block's own group, and per row the bytes of the tile's column
// blocks inside K; nothing past the routed rows or past K.
__device__ __noinline__ void store_scales_general(const uint8_t* col_stg, const uint8_t* row_stg, const CastOut& out,
                                                  const RoutingSmem& rs, const TileInfo& inf, int K, int32_t r0,
                                                  int c0, int t, bool do_row, bool do_col) {
  if (do_col && t < inf.kcols) {
#pragma unroll
    for (int b = 0; b < 8; b++) {
      if (kBlockRows * b >= inf.valid) break;
      const int g = inf.gb[b];
      const int32_t o = rs.off[g];
      const size_t m16 = static_cast<size_t>(rs.off[g + 1] - o) >> 4;
      gstore(&out.col_scale[(static_cast<size_t>(K) * o >> 4) + static_cast<size_t>(c0 + t) * m16 +
                            ((r0 + kBlockRows * b - o) >> 4)],
             col_stg[b * kCols + t]);
    }
  }
  if (do_row && t < inf.valid) {
    uint8_t* dst = out.row_scale + static_cast<size_t>(r0 + t) * (static_cast<size_t>(K) >> 4) + (c0 >> 4);
    if ((K & (kCols - 1)) == 0) {  // the row's 8 bytes are 8-byte aligned and all inside K
      uint32_t s0 = 0u, s1 = 0u;
#pragma unroll
      for (int r = 0; r < 4; r++) {
        s0 |= static_cast<uint32_t>(row_stg[r * kRows + t]) << (8 * r);
        s1 |= static_cast<uint32_t>(row_stg[(r + 4) * kRows + t]) << (8 * r);
      }
      gstore(reinterpret_cast<uint2*>(dst), make_uint2(s0, s1));
    } else {
#pragma unroll
      for (int j = 0; j < 8; j++) {
        if (kBlockRows * j >= inf.kcols) break;
        gstore(&dst[j], row_stg[j * kRows + t]);
      }
    }
  }
}

// The tile loop of warp group j (thread gt of it). kGeneral: some tile may be
// general (see the top of the file); without it every tile is plain and the
// edge handling is compiled out.
template <bool kGeneral, bool kTiled, class Routing>
__device__ __forceinline__ void cast_tiles(PlainSmem& sm, PlainGroup& pg, const Routing& routing,
                                           const CUtensorMap* tmap, int32_t K, const float* ra, const float* ca,
                                           const float* col_amax, const CastOut& out, int j, int gt, int first,
                                           int G, int n_ct, int n_tiles, bool k128, bool do_row, bool do_col) {
  const RoutingSmem& rs = sm.rs;
  const int lane = gt & 31, w = gt >> 5;
  const int cc = 8 * (w & 1) + (lane & 7);  // 8-column chunk of the tile, 0..15
  const int rb = 4 * (w >> 1) + (lane >> 3);  // 16-row block of the tile, 0..7
  const int rl = 16 * rb;
  const size_t row_pitch = static_cast<size_t>(K) >> 1;
  const uint64_t keep = policy_evict_last();
  const int bar_id = 1 + j;

  // the tile's row and column tile, advanced by G tiles per step without a
  // division; (rtp, ctp): the previous tile's
  const int Gq = G / n_ct, Gr = G - Gq * n_ct;
  int rt = first / n_ct, ct = first - rt * n_ct;
  int k = 0;
  bool failed = false;
  int rtp = 0, ctp = 0;
  // the general loop reads a tile's info before waiting for the tile; the
  // info of tiles 0 and 1 was written by the prologue, so meet once
  if (kGeneral) group_bar(bar_id);
  for (int tl = first; tl < n_tiles; tl += G, k++) {
    const int slot = k % kPSlots;
    const int32_t r0 = rt * kRows;
    const int c0 = ct * kCols;
    // the tile's info was written two tiles ahead, before the previous
    // tile's barrier, so it is readable before the tile's data lands
    const TileInfo& inf = pg.info[k % kPInfo];
    // a lane of a mixed tile whose block is not in the tile's first group
    // takes its 8 columns' S_enc from its own group's column amax (own_col);
    // the loads are issued before the wait for the tile
    bool own_col = false;
    float4 oa0, oa1;
    if (kGeneral && do_col && inf.mixed) {
      const int gl = inf.gb[rb];
      own_col = gl != inf.gb[0] && rl < inf.valid && 8 * cc < inf.kcols;
      if (own_col) {
        const float4* src = reinterpret_cast<const float4*>(col_amax + static_cast<size_t>(gl) * K + c0 + 8 * cc);
        oa0 = gload(src);
        oa1 = gload(src + 1);
      }
    }
    const bool ok = mbar_wait(&pg.full, k & 1);
    // S_enc of the tile's rows and columns, in place (thread gt: entry gt).
    // General tiles: entries past the routed rows or past K are never used
    // for a stored output and are set to 1.
    bool slow = false;
    uint64_t cse[4];  // S_enc of the lane's 8 columns, pairs (2q, 2q+1)
    if (ok) {
      int32_t valid = kRows, kcols = kCols;
      if (kGeneral) {
        valid = inf.valid;
        kcols = inf.kcols;
      }
      if (do_row) {
        if (!kGeneral || gt < valid) {
          const float a = pg.row_senc[slot][gt];
          pg.row_senc[slot][gt] = s_enc_of(a);
          slow |= !fast_path_amax(a);
          if (ct == 0) gstore(&out.row_s2[r0 + gt], s_dec_of(a));
        } else {
          pg.row_senc[slot][gt] = 1.0f;
        }
      }
      if (do_col) {
        if (!kGeneral || gt < kcols) {
          const float a = pg.col_senc[slot][gt];
          pg.col_senc[slot][gt] = s_enc_of(a);
          slow |= !fast_path_amax(a);
        } else {
          pg.col_senc[slot][gt] = 1.0f;
        }
        if (kGeneral && own_col) {
          const float a[8] = {oa0.x, oa0.y, oa0.z, oa0.w, oa1.x, oa1.y, oa1.z, oa1.w};
          float e[8];
#pragma unroll
          for (int q = 0; q < 8; q++) {
            e[q] = s_enc_of(a[q]);
            slow |= !fast_path_amax(a[q]);
          }
#pragma unroll
          for (int q = 0; q < 4; q++) cse[q] = pack2(e[2 * q], e[2 * q + 1]);
        }
      }
    } else {
      pg.fail = 1;
    }
    uint4 v[16];
    load_patch(sm.tile[j], cc, rl, v);
    const bool any_slow = group_bar_or(bar_id, slow);
    if (pg.fail) {
      failed = true;
      break;
    }
    // every patch of tile k is in registers: the stage takes tile k+1,
    // whose info was written in the previous step, and tile k+2's info is
    // written. The issuing thread is lane 0 of warp k % 4, so that the issue
    // work (group search, expect_tx, four copies) does not always delay the
    // same warp at the next barrier.
    if (gt == 32 * (k & 3) && tl + G < n_tiles) {
      int rt1 = rt + Gq, ct1 = ct + Gr;
      if (ct1 >= n_ct) {
        ct1 -= n_ct;
        rt1++;
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      plain_load(pg, sm.tile[j], tmap, k + 1, rt1, ct1, K, ra, ca);
      if (tl + 2 * G < n_tiles) {
        int rt2 = rt1 + Gq, ct2 = ct1 + Gr;
        if (ct2 >= n_ct) {
          ct2 -= n_ct;
          rt2++;
        }
        plain_info(pg, k + 2, rt2, ct2, rs, K, k128);
      }
    }
    if (k >= 1) {  // the previous tile's staged scales (complete since the barrier)
      const TileInfo& pinf = pg.info[(k - 1) % kPInfo];
      if (!kGeneral || pinf.plain)
        store_scales<kTiled>(pg.col_scale[(k - 1) & 1], pg.row_scale[(k - 1) & 1], out, K, pinf.o_g, pinf.m_g,
                             rtp * kRows, ctp * kCols, gt, do_row, do_col, keep);
      else
        store_scales_general(pg.col_scale[(k - 1) & 1], pg.row_scale[(k - 1) & 1], out, rs, pinf, K, rtp * kRows,
                             ctp * kCols, gt, do_row, do_col);
    }
    if (do_col && !own_col) col_senc_pairs(pg.col_senc[slot], cc, cse);
    // the lane's block: its group's colwise slice, and whether it is stored
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
    uint8_t* rdst = do_row ? out.row_data + static_cast<size_t>(r0 + rl) * row_pitch + (c0 >> 1) + 4 * cc : nullptr;
    const EncodeTables tab{&sm.e4m3, pg.row_senc[slot]};
    const size_t half_m = static_cast<size_t>(m_l) >> 1;
    DirectColSink sink{do_col ? out.col_data + (static_cast<size_t>(K) * o_l >> 1) +
                                    static_cast<size_t>(c0 + 8 * cc) * half_m + ((r0 - o_l + rl) >> 1)
                              : nullptr,
                       half_m, keep, do_col && lane_ok, {}};
    if (any_slow)
      encode_patch<true>(v, tab, cse, pg.col_scale[k & 1], pg.row_scale[k & 1], do_row, do_col, cc, rb, rdst,
                         row_pitch, lane_ok, sink);
    else
      encode_patch<false>(v, tab, cse, pg.col_scale[k & 1], pg.row_scale[k & 1], do_row, do_col, cc, rb, rdst,
                          row_pitch, lane_ok, sink);
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
    const TileInfo& pinf = pg.info[(k - 1) % kPInfo];
    if (!kGeneral || pinf.plain)
      store_scales<kTiled>(pg.col_scale[(k - 1) & 1], pg.row_scale[(k - 1) & 1], out, K, pinf.o_g, pinf.m_g,
                           rtp * kRows, ctp * kCols, gt, do_row, do_col, keep);
    else
      store_scales_general(pg.col_scale[(k - 1) & 1], pg.row_scale[(k - 1) & 1], out, rs, pinf, K, rtp * kRows,
                           ctp * kCols, gt, do_row, do_col);
  }
  if (failed && gt == 0) {
    // drain the load this group issued and did not consume (tile k)
    mbar_wait(&pg.full, k & 1);
    routing.report(NVFP4_ERR_TIMEOUT);
  }
}

template <class Routing, bool kTiled>
__global__ void __launch_bounds__(kPThreads, 1)
group_cast_plain_kernel(const __grid_constant__ Routing routing, const __grid_constant__ CUtensorMap tmap,
                        int32_t K, const float* __restrict__ row_amax, const float* __restrict__ col_amax,
                        const CastOut out) {
  // the 128-byte swizzle wants each stage 1024-byte aligned; the host adds
  // 1024 bytes of slack for this
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  PlainSmem& sm = *reinterpret_cast<PlainSmem*>(base);
  int32_t* off = reinterpret_cast<int32_t*>(base + ((sizeof(PlainSmem) + 15) & ~size_t{15}));

  // device routing may come from the kernel before this one: wait for it
  // first; otherwise the set-up below overlaps that kernel's tail
  if (Routing::kOnDevice) grid_dependency_wait();
  routing.load(sm.rs, off);
  const RoutingSmem& rs = sm.rs;
  if (!rs.ok) return;

  const int t = threadIdx.x;
  const bool do_row = out.row_s2 != nullptr;
  const bool do_col = out.col_s2 != nullptr;
  if (t < 128) e4m3_table_fill(sm.e4m3, t);

  const int j = t / kCastThreads;  // warp group
  const int gt = t - j * kCastThreads;
  PlainGroup& pg = sm.grp[j];
  const int n_ct = (K + kCols - 1) >> 7;
  const bool k128 = (K & (kCols - 1)) == 0;
  const int n_tiles = ((rs.total + kRows - 1) >> 7) * n_ct;  // the last row tile may be short
  const int G = gridDim.x * kPGroups;
  const int first = j * gridDim.x + blockIdx.x;  // groups running together take neighbouring tiles
  const float* ra = do_row ? row_amax : nullptr;
  const float* ca = do_col ? col_amax : nullptr;
  if (gt == 0) {
    mbar_init(&pg.full, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    pg.fail = 0;
  }
  __syncthreads();
  // from here on x and the amax vectors are read
  if (!Routing::kOnDevice) grid_dependency_wait();
  if (gt == 0) {
    // the first tile, and the info of the second
    int rti = first / n_ct, cti = first - rti * n_ct;
    if (first < n_tiles) {
      plain_info(pg, 0, rti, cti, rs, K, k128);
      plain_load(pg, sm.tile[j], &tmap, 0, rti, cti, K, ra, ca);
    }
    if (first + G < n_tiles) {
      const int Gq = G / n_ct, Gr = G - Gq * n_ct;
      cti += Gr;
      rti += Gq;
      if (cti >= n_ct) {
        cti -= n_ct;
        rti++;
      }
      plain_info(pg, 1, rti, cti, rs, K, k128);
    }
  }
  if (do_col) {  // decode scales of all columns of all groups, spread over the grid, while the first tiles load
    const int64_t n = static_cast<int64_t>(rs.E) * K;
#pragma unroll 4
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * kPThreads + t; i < n;
         i += static_cast<int64_t>(gridDim.x) * kPThreads)
      gstore(&out.col_s2[i], s_dec_of(gload(&col_amax[i])));
  }

  // every group a multiple of 128 rows and K % 128 == 0: every tile is plain
  if (rs.all128 && k128)
    cast_tiles<false, kTiled>(sm, pg, routing, &tmap, K, ra, ca, col_amax, out, j, gt, first, G, n_ct, n_tiles,
                              k128, do_row, do_col);
  else
    cast_tiles<true, kTiled>(sm, pg, routing, &tmap, K, ra, ca, col_amax, out, j, gt, first, G, n_ct, n_tiles,
                             k128, do_row, do_col);
}

}  // namespace nvfp4rs
