// group_quantize.cuh -- grouped amax and grouped cast in ONE launch.
//
// TransformerEngine #3649 (grouped row-scaled NVFP4 cast), Description: the
// grouped amax and the grouped cast are two single launches, the second
// consuming the row and column amax vectors of the first. This kernel runs
// both steps in one persistent launch so that each tile of x comes from DRAM
// once: its amax pass leaves it in L2 and its cast pass reads it back from
// there shortly after. The outputs -- row_amax, col_amax and every cast
// output -- are byte-identical to the two-launch path: maxima are exact, and
// the cast of a tile is the very code of group_cast.cuh.
//
// Work items. Every 128 x 128 tile of x is visited twice: by an A item (its
// column maxima go to col_amax, its row maxima to a row accumulator, by
// unsigned atomic max on the float bits, which orders non-negative floats)
// and by a B item (the tile's cast, from the finished amax of its group). A
// B item needs every A item of its group: the column amax spans all rows of
// the group, and a row's amax spans all column tiles, which share the group.
//
// Schedule. The 2n items form one fixed sequence that the persistent CTAs
// claim in order from a global counter: the A items in tile order, with the
// B items of group g (in tile order, as one block) inserted after the first
// P_g A items,
//     P_g = min(n, max(end_g, start_g + lag))
// (start_g, end_g: first and one-past-last tile of the group). So every B
// item comes after all A items of its group, and about 2*lag claims after
// the A item of its own tile: late enough for the group's A items to be
// finished when it is claimed, early enough for the tile to still be in L2.
// With Q_g = P_g + start_g the position of the group's first B item, the
// item at position p is found by one binary search over Q (decode_item).
//
// Roles. A CTA has four compute warps, a producer warp and a publisher warp
// (one lane each). The producer claims items, loads their tiles by TMA into a
// three-stage ring and, for a B item, waits until its group's A items are
// published, then has the TMA unit copy the finished row and column maxima
// (128 + 128 floats, from L2) beside the stage. The compute warps hold the
// same 16 x 8 patches as group_cast.cuh: an A item reduces them to column
// and row maxima, a B item turns the copied maxima into encode scales and
// encodes. The publisher follows the items in order; when the compute warps
// are done with an A item it publishes the maxima, and it hands every stage
// back to the producer. So the claim atomics, the dependency waits and the
// publishing fences all stay off the compute warps' path.
//
// No deadlock, for any number of resident CTAs: an item waits only for A
// items that precede it in the sequence; a CTA issues its items in claim
// order; its compute warps finish every issued item without waiting for
// anything else, and its publisher publishes them without waiting for
// anything else. So the earliest claimed unfinished item can always
// proceed. Every wait is bounded: a producer that gives up raises the
// workspace's abort word (which ends the other CTAs' waits at once) and
// reports NVFP4_ERR_TIMEOUT.
//
// Publishing an A item: its 128 compute threads arrive on the stage's empty
// barrier after their atomics (release, CTA scope); the publisher, having
// seen the barrier complete (acquire), fences (acq_rel, GPU scope) and adds
// one to the group's done counter. The producer waits for a group with
// acquire loads of that counter, then a proxy fence orders the TMA unit's
// reads of the maxima after them.
//
// Workspace (32-bit words, zeroed by the host before the launch):
//   [0] item counter   [1] abort word   [kWsDone + g] done counter of group g
//   then, from word quant_ws_header_words(E), the row accumulators when the
//   caller does not provide them (graph-safe call; see nvfp4rs.cu).
#pragma once

#include "group_amax.cuh"
#include "group_cast.cuh"

namespace nvfp4rs {

constexpr int kWsDone = 64;                 // first done counter (word index)
constexpr int kBItem = 1 << 30;             // item tag: B (cast); tile index below it
constexpr int kNoItem = -1;
constexpr uint32_t kDoneSpinLimit = 1u << 20;  // bounded dependency waits (~1 s)

// Words of the workspace before the row accumulators (a multiple of 64).
constexpr int64_t quant_ws_header_words(int64_t E) { return (kWsDone + E + 63) / 64 * 64; }

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ uint32_t ld_relaxed_u32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Publish the finished atomics of an A item (ordered before this thread by
// the stage's empty barrier) and count one finished A item of the group.
__device__ __forceinline__ void release_add_one(uint32_t* p) {
  asm volatile(
      "fence.acq_rel.gpu;\n\t"
      "red.relaxed.gpu.global.add.u32 [%0], 1;" ::"l"(p)
      : "memory");
}

__device__ __forceinline__ void named_bar_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// First tile of group g in the row-major tile order.
__device__ __forceinline__ uint32_t group_first_tile(const RoutingSmem& rs, int g, int n_ct) {
  return static_cast<uint32_t>(rs.off[g] >> 7) * static_cast<uint32_t>(n_ct);
}

// The item at sequence position p (n tiles; q = Q_g of every group):
// kNoItem, an A tile (its index) or a B tile (its index | kBItem).
__device__ __forceinline__ int decode_item(const RoutingSmem& rs, const uint32_t* q, int n_ct,
                                           uint32_t n, uint32_t p) {
  if (p >= 2u * n) return kNoItem;
  int lo = -1, hi = rs.E - 1;  // the last g with q[g] <= p, or -1
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (q[mid] <= p)
      lo = mid;
    else
      hi = mid - 1;
  }
  if (lo < 0) return static_cast<int>(p);  // before the first B block
  const uint32_t start = group_first_tile(rs, lo, n_ct);
  const uint32_t end = group_first_tile(rs, lo + 1, n_ct);
  const uint32_t d = p - q[lo];
  if (d < end - start) return static_cast<int>(start + d) | kBItem;
  return static_cast<int>(p - end);  // an A tile after group lo's B block
}

__device__ __forceinline__ int item_tile(int item) { return item & (kBItem - 1); }

// ----------------------------------------------------------- shared memory

constexpr int kQStages = 3;           // tile ring of the one-launch kernel
constexpr int kComputeThreads = 128;  // warps 0-3
constexpr int kProducerWarp = 4;
constexpr int kPublisherWarp = 5;
constexpr int kQThreads = 192;
constexpr int kAbortItem = -2;        // the producer gave up on this item
constexpr uint32_t kAmaxBytes = 512;  // 128 fp32 maxima: one tile's rows, or its columns

// What comes with each stage besides the tile.
struct QuantStageInfo {
  float row_amax[kRows];  // B item: amax of the tile's rows (bulk copy from L2)
  float col_amax[kCols];  // B item: amax of the tile's columns in its group (bulk copy)
  float row_senc[kRows];  // B item: S_enc of those, from the compute threads
  float col_senc[kCols];
  int item;               // kNoItem, kAbortItem, an A tile or a B tile (| kBItem)
  int group;
  int slow;               // B item: some amax outside the shortcut range
  int pad;
};

struct QuantSmem {
  uint8_t tile[kQStages][kTileBytes];  // at offset 0 of a 1024-byte aligned block
  QuantStageInfo info[kQStages];
  float2 e4m3[128];                    // {value, RN(1/value)} per E4M3 code
  uint64_t full[kQStages];     // 2 producer arrivals + the tile bytes (+ the amax bytes)
  uint64_t empty[kQStages];    // 128 arrivals: the compute threads are done with the stage
  uint64_t retired[kQStages];  // 1 arrival: the publisher has accounted for the stage's item
  int abort;                   // a compute thread gave up waiting for a stage
};

// Dynamic shared memory: QuantSmem, the E+1 group offsets, Q_g of every group.
constexpr size_t quantize_smem_bytes(int E) {
  return ((sizeof(QuantSmem) + 15) & ~size_t{15}) + sizeof(int32_t) * (E + 1) + sizeof(uint32_t) * E;
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

// mbar_wait that also gives up when *flag becomes nonzero.
__device__ __forceinline__ bool mbar_wait_flag(uint64_t* bar, uint32_t phase, const volatile int* flag) {
  for (uint32_t i = 0; i < kSpinLimit; i += 64) {
    if (mbar_wait_some(bar, phase, 64)) return true;
    if (*flag) return false;
  }
  return false;
}

// Compute warps' named barrier (warps 0-3); returns the OR of `pred` over them.
__device__ __forceinline__ bool compute_bar_or(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 1, %2, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(pred)), "n"(kComputeThreads)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void compute_bar() { named_bar_sync(1, kComputeThreads); }

__device__ __forceinline__ void raise_abort(uint32_t* abort_word) { atomicExch(abort_word, 1u); }

// Spin (bounded) until *done >= need, with acquire loads. False when the
// abort word or the CTA's abort flag is raised, or at the spin limit.
__device__ __forceinline__ bool wait_group(const uint32_t* done, uint32_t need, const uint32_t* abort_word,
                                           const volatile int* cta_abort) {
  for (uint32_t i = 0; i < kDoneSpinLimit; i++) {
    if (ld_acquire_u32(done) >= need) return true;
    if (*cta_abort || ld_relaxed_u32(abort_word) != 0u) return false;
    __nanosleep(64);
  }
  return false;
}

// ----------------------------------------------------------------- kernel

// kTiled: both scale outputs in the 128x4-tiled layout.
template <class Routing, bool kTiled>
__global__ void __launch_bounds__(kQThreads, 2)
group_quantize_kernel(const __grid_constant__ Routing routing, const __grid_constant__ CUtensorMap tmap,
                      int32_t K, int32_t lag, uint32_t* ws, float* row_acc, float* row_amax,
                      float* col_amax, const CastOut out) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  QuantSmem& sm = *reinterpret_cast<QuantSmem*>(base);
  int32_t* off = reinterpret_cast<int32_t*>(base + ((sizeof(QuantSmem) + 15) & ~size_t{15}));
  __shared__ RoutingSmem rs;

  routing.load(rs, off);
  if (!rs.ok) return;

  const int t = threadIdx.x;
  const int E = rs.E;
  const int G = gridDim.x;
  const bool do_row = out.row_s2 != nullptr;
  const bool do_col = out.col_s2 != nullptr;
  const int n_ct = K >> 7;
  const uint32_t n = static_cast<uint32_t>(rs.total >> 7) * static_cast<uint32_t>(n_ct);
  uint32_t* qpos = reinterpret_cast<uint32_t*>(off + E + 1);
  uint32_t* const counter = ws;
  uint32_t* const abort_word = ws + 1;
  uint32_t* const done = ws + kWsDone;

  for (int g = t; g < E; g += kQThreads) {
    const uint32_t start = group_first_tile(rs, g, n_ct);
    const uint32_t end = group_first_tile(rs, g + 1, n_ct);
    const uint32_t p = min(n, max(end, start + static_cast<uint32_t>(lag)));
    qpos[g] = p + start;
  }
  if (do_col) {  // empty groups own no tile: their col_s2 is S_dec(0) (col_amax stays 0)
    for (int g = blockIdx.x; g < E; g += G)
      if (off[g + 1] == off[g])
        for (int c = t; c < K; c += kQThreads) out.col_s2[static_cast<size_t>(g) * K + c] = s_dec_of(0.0f);
  }
  if (t < 128) sm.e4m3[t] = e4m3_entry(t);
  if (t == 0) {
    for (int s = 0; s < kQStages; s++) {
      mbar_init(&sm.full[s], 2);
      mbar_init(&sm.empty[s], kComputeThreads);
      mbar_init(&sm.retired[s], 1);
    }
    sm.abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();  // the last CTA-wide barrier: the roles part here

  const int lane = t & 31, warp = t >> 5;
  volatile int* cta_abort = &sm.abort;

  if (warp == kProducerWarp) {
    // ============================================================ producer
    // Claims items in sequence order and loads their tiles; for a B item it
    // waits until the group's A items are published, then has the TMA unit
    // bring the finished row and column maxima beside the stage. Runs up to
    // kQStages items ahead of the compute warps.
    if (lane != 0) return;
    uint32_t raw = atomicAdd(counter, 1u);  // position of the next item
    int j = 0;                              // items issued so far
    bool fail = false;
    for (;; j++) {
      const int s = j % kQStages;
      const int item = decode_item(rs, qpos, n_ct, n, raw);
      if (item != kNoItem) raw = atomicAdd(counter, 1u);  // read one item later
      // stage s is free once the publisher has accounted for item j - kQStages
      if (j >= kQStages && !mbar_wait_flag(&sm.retired[s], ((j / kQStages) - 1) & 1, cta_abort)) {
        fail = true;
        break;
      }
      QuantStageInfo& inf = sm.info[s];
      if (item == kNoItem) {  // the end mark: no bytes, both arrivals
        inf.item = kNoItem;
        mbar_arrive(&sm.full[s]);
        mbar_arrive(&sm.full[s]);
        j++;
        break;
      }
      const bool is_b = (item & kBItem) != 0;
      const int tl = item_tile(item);
      const int rt = tl / n_ct, ct = tl - rt * n_ct;
      const int32_t r0 = rt * kRows;
      const int c0 = ct * kCols;
      const int g = group_of_row(rs, r0);
      inf.item = item;
      inf.group = g;
      inf.slow = 0;
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      const uint32_t amax_bytes = is_b ? (do_row ? kAmaxBytes : 0u) + (do_col ? kAmaxBytes : 0u) : 0u;
      mbar_expect_tx(&sm.full[s], kTileBytes + amax_bytes);  // first arrival
      const uint64_t policy = is_b ? policy_evict_first() : policy_evict_normal();
      tma_load_2d(sm.tile[s], &tmap, c0, r0, &sm.full[s], policy);
      tma_load_2d(sm.tile[s] + kBoxBytes, &tmap, c0 + kBoxCols, r0, &sm.full[s], policy);
      bool ok = true;
      if (is_b) {
        const uint32_t need = static_cast<uint32_t>((rs.off[g + 1] - rs.off[g]) >> 7) *
                              static_cast<uint32_t>(n_ct);
        ok = wait_group(&done[g], need, abort_word, cta_abort);
        if (!ok) inf.item = kAbortItem;
        // the maxima are final once the counter is seen complete; the copies
        // read them through the async proxy (issued even after a give-up, so
        // that the stage's transaction count completes)
        asm volatile("fence.proxy.async.global;" ::: "memory");
        if (do_row) bulk_load(inf.row_amax, row_acc + r0, kAmaxBytes, &sm.full[s]);
        if (do_col) bulk_load(inf.col_amax, col_amax + static_cast<size_t>(g) * K + c0, kAmaxBytes, &sm.full[s]);
      }
      mbar_arrive(&sm.full[s]);  // second arrival: `inf` is written
      if (!ok) {
        fail = true;
        j++;
        break;
      }
    }
    if (fail) {
      raise_abort(abort_word);
      routing.report(NVFP4_ERR_TIMEOUT);
      // the last kQStages issued items may still have bytes in flight
      for (int i = j > kQStages ? j - kQStages : 0; i < j; i++)
        mbar_wait(&sm.full[i % kQStages], (i / kQStages) & 1);
    }
    return;
  }

  if (warp == kPublisherWarp) {
    // =========================================================== publisher
    // Follows the items in order: once the compute threads are done with an
    // A item, its maxima are published (fence, then one more on the group's
    // done counter); every stage is then handed back to the producer.
    if (lane != 0) return;
    for (int r = 0;; r++) {
      const int s = r % kQStages;
      const uint32_t ph = (r / kQStages) & 1;
      if (!mbar_wait_flag(&sm.full[s], ph, cta_abort)) break;
      const int item = sm.info[s].item;
      const int g = sm.info[s].group;
      if (item < 0) break;  // end mark, or the producer gave up
      if (!mbar_wait_flag(&sm.empty[s], ph, cta_abort)) break;
      mbar_arrive(&sm.retired[s]);
      if ((item & kBItem) == 0) release_add_one(&done[g]);
    }
    return;
  }

  // ========================================================= compute warps
  const int cc = lane & 15, h = lane >> 4;
  const int rb = 2 * warp + h;  // 16-row block of the tile, 0..7
  const int rl = 16 * rb;       // first tile row of this lane
  const size_t row_pitch = static_cast<size_t>(K) >> 1;
  const uint64_t keep = policy_evict_last();
  for (int k = 0;; k++) {
    const int s = k % kQStages;
    const bool ok = mbar_wait(&sm.full[s], (k / kQStages) & 1);
    QuantStageInfo& inf = sm.info[s];
    const int item = inf.item;
    const bool is_b = item >= 0 && (item & kBItem) != 0;
    uint4 v[16];
    load_patch(sm.tile[s], cc, rl, v);
    if (ok && is_b) {
      // this thread's row and column: encode scales for the whole tile, and
      // the decode scales (a row's in its first column tile, a column's in
      // its group's first row tile)
      const int tl = item_tile(item);
      const int rt = tl / n_ct, ct = tl - rt * n_ct;
      const int32_t r0 = rt * kRows;
      const int g = inf.group;
      bool slow = false;
      if (do_row) {
        const float a = inf.row_amax[t];
        inf.row_senc[t] = s_enc_of(a);
        slow |= !fast_path_amax(a);
        if (ct == 0) {
          if (row_amax != row_acc) row_amax[r0 + t] = a;
          out.row_s2[r0 + t] = s_dec_of(a);
        }
      }
      if (do_col) {
        const float a = inf.col_amax[t];
        inf.col_senc[t] = s_enc_of(a);
        slow |= !fast_path_amax(a);
        if (r0 == rs.off[g]) out.col_s2[static_cast<size_t>(g) * K + ct * kCols + t] = s_dec_of(a);
      }
      if (slow) inf.slow = 1;
    }
    // every patch is in registers (the stage may now be overwritten) and the
    // encode scales are in place; a failed wait anywhere ends every compute
    // warp here
    if (compute_bar_or(!ok)) {
      if (t == 0) {
        *cta_abort = 1;
        raise_abort(abort_word);
        routing.report(NVFP4_ERR_TIMEOUT);
      }
      break;
    }
    if (item < 0) break;  // end mark, or the producer gave up
    const int g = inf.group;
    const int tl = item_tile(item);
    const int rt = tl / n_ct, ct = tl - rt * n_ct;
    const int32_t r0 = rt * kRows;
    const int c0 = ct * kCols;

    if (!is_b) {
      // ------------------------------------------------------------ A item
      uint32_t cm[4] = {v[0].x, v[0].y, v[0].z, v[0].w};
#pragma unroll
      for (int i = 1; i < 16; i++) {
        cm[0] = maxabs2(cm[0], v[i].x);
        cm[1] = maxabs2(cm[1], v[i].y);
        cm[2] = maxabs2(cm[2], v[i].z);
        cm[3] = maxabs2(cm[3], v[i].w);
      }
#pragma unroll
      for (int q = 0; q < 4; q++)
        cm[q] = umax2(cm[q] & 0x7FFF7FFFu, __shfl_xor_sync(0xFFFFFFFFu, cm[q] & 0x7FFF7FFFu, 16));
      if (do_row) {
        // P[kk] = maxima of rows (2kk, 2kk+1) over this lane's 8 columns
        uint32_t P[8];
#pragma unroll
        for (int kk = 0; kk < 8; kk++) {
          const uint32_t a = maxabs2(maxabs2(v[2 * kk].x, v[2 * kk].y), maxabs2(v[2 * kk].z, v[2 * kk].w));
          const uint32_t b = maxabs2(maxabs2(v[2 * kk + 1].x, v[2 * kk + 1].y),
                                     maxabs2(v[2 * kk + 1].z, v[2 * kk + 1].w));
          P[kk] = maxabs2(prmt(a, b, 0x5410), prmt(a, b, 0x7632)) & 0x7FFF7FFFu;
        }
        // reduce-scatter over the 16 lanes sharing these rows: lane cc ends
        // with the maximum of row rl + cc
        const bool b3 = cc & 8, b2 = cc & 4, b1 = cc & 2, b0 = cc & 1;
        uint32_t Q4[4];
#pragma unroll
        for (int kk = 0; kk < 4; kk++) {
          const uint32_t mine = b3 ? P[4 + kk] : P[kk];
          const uint32_t send = b3 ? P[kk] : P[4 + kk];
          Q4[kk] = umax2(mine, __shfl_xor_sync(0xFFFFFFFFu, send, 8));
        }
        uint32_t R2[2];
#pragma unroll
        for (int kk = 0; kk < 2; kk++) {
          const uint32_t mine = b2 ? Q4[2 + kk] : Q4[kk];
          const uint32_t send = b2 ? Q4[kk] : Q4[2 + kk];
          R2[kk] = umax2(mine, __shfl_xor_sync(0xFFFFFFFFu, send, 4));
        }
        const uint32_t S1 = umax2(b1 ? R2[1] : R2[0], __shfl_xor_sync(0xFFFFFFFFu, b1 ? R2[0] : R2[1], 2));
        const uint32_t mine = b0 ? (S1 >> 16) : (S1 & 0xFFFFu);
        const uint32_t send = b0 ? (S1 & 0xFFFFu) : (S1 >> 16);
        const uint32_t rowm = max(mine, __shfl_xor_sync(0xFFFFFFFFu, send, 1));
        red_max_u32(&row_acc[r0 + rl + cc], rowm << 16);
      }
      // column maxima of the four warps meet in the (consumed) stage
      uint32_t* cw = reinterpret_cast<uint32_t*>(sm.tile[s]);  // [warp][64 words]
      if (h == 0) *reinterpret_cast<uint4*>(&cw[warp * 64 + 4 * cc]) = make_uint4(cm[0], cm[1], cm[2], cm[3]);
      compute_bar();
      if (do_col) {
        const int sh = (t & 1) * 16;  // column t: half t & 1 of word t / 2
        uint32_t m = 0u;
#pragma unroll
        for (int w = 0; w < 4; w++) m = max(m, (cw[w * 64 + (t >> 1)] >> sh) & 0xFFFFu);
        red_max_u32(&col_amax[static_cast<size_t>(g) * K + c0 + t], m << 16);
      }
    } else {
      // ------------------------------------------------------------ B item
      const int32_t o_g = rs.off[g];
      const int64_t m_g = rs.off[g + 1] - o_g;
      CastStage& st = *reinterpret_cast<CastStage*>(sm.tile[s]);
      uint8_t* rdst = do_row ? out.row_data + static_cast<size_t>(r0 + rl) * row_pitch + (c0 >> 1) + 4 * cc
                             : nullptr;
      const EncodeTables tab{sm.e4m3, inf.row_senc, inf.col_senc};
      if (inf.slow)
        encode_patch<true>(v, tab, st, do_row, do_col, cc, rb, rdst, row_pitch);
      else
        encode_patch<false>(v, tab, st, do_row, do_col, cc, rb, rdst, row_pitch);
      compute_bar();
      store_staged<kTiled>(st, out, K, o_g, m_g, r0, c0, t, do_row, do_col, keep);
    }
    // this thread's generic writes to the stage come before the next TMA load into it
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    mbar_arrive(&sm.empty[s]);
  }
}

}  // namespace nvfp4rs
