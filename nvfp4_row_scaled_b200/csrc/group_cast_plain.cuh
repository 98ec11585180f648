// group_cast_plain.cuh -- the grouped row-scaled NVFP4 cast when every group
// starts and ends on a 128-row boundary (MoE routing padded to 128 rows).
//
// TransformerEngine #3649 (grouped row-scaled NVFP4 cast), Description: the
// cast step takes the row and column amax vectors and writes the packed FP4
// data and scales of every group, rowwise and colwise (TransformerEngine
// #3324, summary). Same arithmetic and the same bytes as group_cast_kernel
// (both run encode_patch); this kernel is organised to keep the SM issuing:
//  - One CTA per SM made of three independent warp groups of four warps
//    (named barriers 1..3), each with its own tile sequence, TMA ring and
//    mbarriers. The tables all groups read (E4M3 values and reciprocals,
//    group offsets) exist once per SM, and what that saves pays for each
//    group's separate staging buffers.
//  - Nothing is staged in a tile's stage, so the stage is refilled with the
//    group's tile after next as soon as its warps hold their patches: two
//    tiles are in flight while one is encoded. Colwise codes go from
//    registers straight to global memory; the block scales are staged in a
//    double buffer and stored after the next tile's barrier. One barrier per
//    tile.
//  - Warp w covers rows 64*(w/2) .. +63 and columns 64*(w%2) .. +63 of the
//    128 x 128 tile; lane (hb, c8) holds 16 rows (block 4*(w/2) + hb) by 8
//    columns (chunk 8*(w%2) + c8). A rowwise store instruction then writes
//    four rows x 32 contiguous bytes and a colwise one eight columns x 32
//    contiguous bytes: whole sectors.
//  - A tile's row and column amax come by bulk copy on the tile's mbarrier
//    into a three-slot ring and are turned into S_enc in place before the
//    barrier.
// Ring invariants (tile k of a group): stage k % 2, amax slot k % 3, group
// info entry k % 4, scale staging k % 2. The refill issued after tile k's
// barrier writes stage k % 2, slot (k+2) % 3 and entry (k+2) % 4; every read
// of those by tiles k-1 and k-2 happened before that barrier.
#pragma once

#include "group_cast.cuh"

namespace nvfp4rs {

constexpr int kPGroups = 3;                         // warp groups per CTA
constexpr int kPThreads = kPGroups * kCastThreads;  // 384
constexpr int kPSlots = 3;                          // amax ring depth
constexpr int kPInfo = 4;                           // group-info ring depth

struct alignas(16) PlainGroup {
  float col_senc[kPSlots][kCols];   // bulk-copied column amax, then S_enc
  float row_senc[kPSlots][kRows];   // bulk-copied row amax, then S_enc
  uint8_t col_scale[2][8 * kCols];  // staged colwise block scales [row block][column]
  uint8_t row_scale[2][8 * kRows];  // staged rowwise block scales [column block][row]
  int32_t info[kPInfo][2];          // first row and size of the tile's group
  uint64_t full[kStages];
  int32_t fail;
};

// Dynamic shared memory of the kernel; `off` (E+1 int32) follows it.
struct PlainSmem {
  uint8_t tile[kPGroups][kStages][kTileBytes];  // at offset 0 of a 1024-byte aligned block
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
// bytes per column, straight to the group's transposed data (half 0 is held
// until half 1 completes the column's piece).
struct DirectColSink {
  uint8_t* dst;   // the lane's first column, at its 16-row block
  size_t pitch;   // bytes per column of the group (m_g / 2)
  uint64_t policy;
  uint32_t lo[8];
  __device__ __forceinline__ void operator()(int half, const uint32_t (&cw)[8]) {
    if (half == 0) {
#pragma unroll
      for (int q = 0; q < 8; q++) lo[q] = cw[q];
    } else {
#pragma unroll
      for (int q = 0; q < 8; q++) st_global_u2_hint(dst + q * pitch, make_uint2(lo[q], cw[q]), policy);
    }
  }
};

// One thread of the group: tile `tl` (the group's k-th) into stage s, with its group's
// row range and the 128 column and 128 row amax it needs (NULL: direction
// not requested), all completing on the stage's mbarrier.
__device__ __forceinline__ void plain_issue(PlainGroup& pg, uint8_t* stage, const CUtensorMap* map, int s,
                                            int k, int tl, int n_ct, const RoutingSmem& rs, int K,
                                            const float* row_amax, const float* col_amax) {
  const int rt = tl / n_ct, ct = tl - rt * n_ct;
  const int g = group_of_row(rs, rt * kRows);
  pg.info[k % kPInfo][0] = rs.off[g];
  pg.info[k % kPInfo][1] = rs.off[g + 1] - rs.off[g];
  const int slot = k % kPSlots;
  mbar_expect_tx(&pg.full[s], kTileBytes + (col_amax != nullptr ? 512u : 0u) + (row_amax != nullptr ? 512u : 0u));
  const uint64_t pol = policy_evict_first();
  tma_load_2d(stage, map, ct * kCols, rt * kRows, &pg.full[s], pol);
  tma_load_2d(stage + kBoxBytes, map, ct * kCols + kBoxCols, rt * kRows, &pg.full[s], pol);
  if (col_amax != nullptr)
    bulk_load(pg.col_senc[slot], col_amax + static_cast<size_t>(g) * K + ct * kCols, 512u, &pg.full[s]);
  if (row_amax != nullptr) bulk_load(pg.row_senc[slot], row_amax + static_cast<size_t>(rt) * kRows, 512u, &pg.full[s]);
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
  const int n_ct = K >> 7;
  const int n_tiles = (rs.total >> 7) * n_ct;
  const int G = gridDim.x * kPGroups;
  const int first = j * gridDim.x + blockIdx.x;  // groups running together take neighbouring tiles
  const float* ra = do_row ? row_amax : nullptr;
  const float* ca = do_col ? col_amax : nullptr;
  if (gt == 0) {
    for (int s = 0; s < kStages; s++) mbar_init(&pg.full[s], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    pg.fail = 0;
  }
  __syncthreads();
  if (gt == 0)
    for (int k = 0; k < kStages && first + k * G < n_tiles; k++)
      plain_issue(pg, sm.tile[j][k], &tmap, k, k, first + k * G, n_ct, rs, K, ra, ca);
  if (do_col) {  // decode scales of all columns of all groups, spread over the grid, while the first tiles load
    const int64_t n = static_cast<int64_t>(rs.E) * K;
#pragma unroll 4
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * kPThreads + t; i < n;
         i += static_cast<int64_t>(gridDim.x) * kPThreads)
      gstore(&out.col_s2[i], s_dec_of(gload(&col_amax[i])));
  }

  const int lane = gt & 31, w = gt >> 5;
  const int cc = 8 * (w & 1) + (lane & 7);  // 8-column chunk of the tile, 0..15
  const int rb = 4 * (w >> 1) + (lane >> 3);  // 16-row block of the tile, 0..7
  const int rl = 16 * rb;
  const size_t row_pitch = static_cast<size_t>(K) >> 1;
  const uint64_t keep = policy_evict_last();
  const int bar_id = 1 + j;

  int k = 0;
  bool failed = false;
  // the tile's row and column tile, advanced by G tiles per step without a
  // division; r0p, c0p: the previous tile's first row and column
  const int Gq = G / n_ct, Gr = G - Gq * n_ct;
  int rt = first / n_ct, ct = first - rt * n_ct;
  int32_t r0p = 0;
  int c0p = 0;
  for (int tl = first; tl < n_tiles; tl += G, k++) {
    const int s = k & 1;
    const int slot = k % kPSlots;
    const uint32_t phase = (k >> 1) & 1;
    const int32_t r0 = rt * kRows;
    const int c0 = ct * kCols;
    const bool ok = mbar_wait(&pg.full[s], phase);
    // S_enc of the tile's rows and columns, in place (thread gt: entry gt)
    bool slow = false;
    if (ok) {
      if (do_row) {
        const float a = pg.row_senc[slot][gt];
        pg.row_senc[slot][gt] = s_enc_of(a);
        slow |= !fast_path_amax(a);
        if (ct == 0) gstore(&out.row_s2[r0 + gt], s_dec_of(a));
      }
      if (do_col) {
        const float a = pg.col_senc[slot][gt];
        pg.col_senc[slot][gt] = s_enc_of(a);
        slow |= !fast_path_amax(a);
      }
    } else {
      pg.fail = 1;
    }
    uint4 v[16];
    load_patch(sm.tile[j][s], cc, rl, v);
    const bool any_slow = group_bar_or(bar_id, slow);
    if (pg.fail) {
      failed = true;
      break;
    }
    // every patch of tile k is in registers: its stage takes tile k+2. The
    // issuing thread is lane 0 of warp k % 4, so that the issue work (group
    // search, expect_tx, four copies) does not always delay the same warp at
    // the next barrier.
    if (gt == 32 * (k & 3) && tl + 2 * G < n_tiles) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      plain_issue(pg, sm.tile[j][s], &tmap, s, k + 2, tl + 2 * G, n_ct, rs, K, ra, ca);
    }
    if (k >= 1)  // the previous tile's staged scales (complete since the barrier)
      store_scales<kTiled>(pg.col_scale[(k - 1) & 1], pg.row_scale[(k - 1) & 1], out, K,
                           pg.info[(k - 1) % kPInfo][0], pg.info[(k - 1) % kPInfo][1], r0p, c0p, gt, do_row,
                           do_col, keep);
    const int32_t o_g = pg.info[k % kPInfo][0];
    const size_t half_m = static_cast<size_t>(pg.info[k % kPInfo][1]) >> 1;
    uint8_t* rdst = do_row ? out.row_data + static_cast<size_t>(r0 + rl) * row_pitch + (c0 >> 1) + 4 * cc : nullptr;
    DirectColSink sink{do_col ? out.col_data + (static_cast<size_t>(K) * o_g >> 1) +
                                    static_cast<size_t>(c0 + 8 * cc) * half_m + ((r0 - o_g + rl) >> 1)
                              : nullptr,
                       half_m, keep, {}};
    const EncodeTables tab{&sm.e4m3, pg.row_senc[slot], pg.col_senc[slot]};
    if (any_slow)
      encode_patch<true>(v, tab, pg.col_scale[k & 1], pg.row_scale[k & 1], do_row, do_col, cc, rb, rdst, row_pitch,
                         true, sink);
    else
      encode_patch<false>(v, tab, pg.col_scale[k & 1], pg.row_scale[k & 1], do_row, do_col, cc, rb, rdst, row_pitch,
                          true, sink);
    r0p = r0;
    c0p = c0;
    ct += Gr;
    rt += Gq;
    if (ct >= n_ct) {
      ct -= n_ct;
      rt++;
    }
  }

  if (!failed && k >= 1) {  // the last tile's staged scales
    group_bar(bar_id);
    store_scales<kTiled>(pg.col_scale[(k - 1) & 1], pg.row_scale[(k - 1) & 1], out, K,
                         pg.info[(k - 1) % kPInfo][0], pg.info[(k - 1) % kPInfo][1], r0p, c0p, gt, do_row, do_col,
                         keep);
  }
  if (failed && gt == 0) {
    // drain the loads this group issued and did not consume (tiles k, k+1)
    for (int jj = k; jj <= k + 1 && first + jj * G < n_tiles; jj++) mbar_wait(&pg.full[jj & 1], (jj >> 1) & 1);
    routing.report(NVFP4_ERR_TIMEOUT);
  }
}

}  // namespace nvfp4rs
