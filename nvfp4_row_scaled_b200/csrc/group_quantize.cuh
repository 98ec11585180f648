// group_quantize.cuh -- grouped amax and grouped cast in ONE launch.
//
// TransformerEngine #3649 (grouped row-scaled NVFP4 cast), Description: the
// grouped amax and the grouped cast are two single launches, the second
// consuming the row and column amax vectors of the first. This kernel runs
// both steps in one persistent launch so that each tile of x comes from DRAM
// once: its amax pass leaves it in L2 and its cast pass reads it back from
// there a little later. The outputs -- row_amax, col_amax and every cast
// output -- are byte-identical to the two-launch path: maxima are exact, and
// the cast of a tile is the very code of group_cast_plain.cuh.
//
// Work items. Every 128 x 128 tile of x is visited twice: by an A item (its
// column maxima go to col_amax, its row maxima to a row accumulator, by
// unsigned atomic max on the float bits, which orders non-negative floats)
// and by a B item (the tile's cast, from the finished amax of its group). A
// B item needs every A item of its group: the column amax spans all rows of
// the group, and a row's amax spans all column tiles, which share the group.
//
// Schedule. The 2n items form one fixed sequence that the CTAs claim in
// order from a global counter: the A items in tile order, with the B items
// of group g inserted as one block after the first
//     P_g = min(n, end_g + lag)
// A items (start_g, end_g: first and one-past-last tile of the group). The
// block runs over the group's tiles in REVERSE order, so the tiles whose A
// items ran last -- the ones most likely still in L2 -- are cast first, and
// a group larger than L2 loses only its oldest tiles. Every B item comes at
// least `lag` claims after the A items of its group: late enough for them to
// be finished when it is claimed. With Q_g = P_g + start_g the position of
// the group's first B item, a producer decodes its (increasing) positions
// with two forward-only cursors over Q and the group offsets (ItemCursor).
//
// Roles. One CTA per SM, four warp groups:
//  - Three compute groups of four warps, each with its own two-stage TMA
//    ring and named barrier, run the cast kernel's patch code (B items) or
//    its amax reductions (A items). They wait only for their ring.
//  - The control group: lane 0 of warp 12 + j is the producer of compute
//    group j. It claims items, loads each tile by TMA into the group's ring
//    and, for a B item, waits until its group's A items are published, then
//    has the TMA unit copy the finished row and column maxima (from L2)
//    beside the stage. Lane 0 of warp 15 is the publisher: when a compute
//    group reports an A item done (its threads' atomics issued), it fences
//    and adds one to the group's done counter.
//  - setmaxnreg hands the control group's registers to the compute groups:
//    3 x 128 threads x 160 + 128 x 32 = 65536, the block's launch total.
//
// No deadlock, for any number of resident CTAs: an item waits only for A
// items that precede it in the sequence; each producer issues its claims in
// claim order and its compute group finishes them in that order; an A item needs
// nothing but its tile, and the publisher publishes it without waiting for
// anything else. So the earliest claimed unfinished item can always
// proceed. Every wait is bounded: a thread that gives up raises the
// workspace's abort word (which ends the other CTAs' waits) and reports
// NVFP4_ERR_TIMEOUT.
//
// Publishing an A item: each compute thread arrives on the group's adone
// barrier after its atomics (release, CTA scope); the publisher, having seen
// the phase complete (acquire), fences (acq_rel, GPU scope) and adds one to
// the group's done counter (one fence for all the items a sweep finds). The producer waits for a group with acquire
// loads of that counter, then a proxy fence orders the TMA unit's reads of
// the maxima after them. adone has kPubSlots slots per compute group, and a
// slot is reused only after the publisher acknowledged its previous use (aack), so
// no phase of it can be missed.
//
// Workspace (32-bit words, zeroed by the host before the launch):
//   [0] item counter   [1] abort word   [kWsDone + g] done counter of group g
//   then, from word quant_ws_header_words(E), the row accumulators when the
//   caller does not provide them (graph-safe call; see nvfp4rs.cu).
#pragma once

#include "group_amax.cuh"
#include "group_cast_plain.cuh"

namespace nvfp4rs {

constexpr int kWsDone = 64;                 // first done counter (word index)
constexpr int kBItem = 1 << 30;             // item tag: B (cast); tile index below it
constexpr int kNoItem = -1;                 // the end of the sequence
constexpr int kAbortItem = -2;              // the producer gave up on this item
constexpr uint32_t kDoneSpinLimit = 1u << 20;  // bounded dependency waits (~1 s)
constexpr uint32_t kIdleLimit = 1u << 22;      // idle control loops (>= 100 ns each) before giving up

// Words of the workspace before the row accumulators (a multiple of 64).
constexpr int64_t quant_ws_header_words(int64_t E) { return (kWsDone + E + 63) / 64 * 64; }

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p) {
  uint32_t v;
  if (!NVFP4_LOAD_OK(p, 4)) return 0u;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ uint32_t ld_relaxed_u32(const uint32_t* p) {
  uint32_t v;
  if (!NVFP4_LOAD_OK(p, 4)) return 0u;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void raise_abort(uint32_t* abort_word) {
  if (NVFP4_STORE_OK(abort_word, 4)) atomicExch(abort_word, 1u);
}

// Claim the next sequence position (past the end of any sequence when the
// counter is out of bounds in the checked build).
__device__ __forceinline__ uint32_t claim(uint32_t* counter) {
  return NVFP4_STORE_OK(counter, 4) ? atomicAdd(counter, 1u) : 0xFFFFFFFFu;
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

// Non-blocking: has the phase with parity `phase` completed?
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t phase) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_addr(bar)), "r"(phase)
      : "memory");
  return done != 0;
}

// Spin (bounded) until *done >= need, with acquire loads. False when the
// abort word is raised, or at the spin limit.
__device__ __forceinline__ bool wait_group(const uint32_t* done, uint32_t need, const uint32_t* abort_word) {
  for (uint32_t i = 0; i < kDoneSpinLimit; i++) {
    if (ld_acquire_u32(done) >= need) return true;
    if (ld_relaxed_u32(abort_word) != 0u) return false;
    __nanosleep(128);
  }
  return false;
}

// First tile of group g in the row-major tile order.
__device__ __forceinline__ uint32_t group_first_tile(const RoutingSmem& rs, int g, int n_ct) {
  return static_cast<uint32_t>(rs.off[g] >> 7) * static_cast<uint32_t>(n_ct);
}

// Decodes sequence positions (n tiles; q = Q_g of every group) into items:
// kNoItem, an A tile (its index) or a B tile (its index | kBItem), with the
// tile's group. A group's B block visits its tiles last to first. The
// positions one producer decodes only increase, and so do the last group
// with Q_g <= p and the group of the A items' tiles, so two cursors that
// only move forward replace the binary searches over shared memory.
struct ItemCursor {
  int gq = -1;  // the last g with q[g] <= p, or -1
  int ga = 0;   // the group of the last A tile

  __device__ __forceinline__ int next(const RoutingSmem& rs, const uint32_t* q, int n_ct, uint32_t n, uint32_t p,
                                      int& group) {
    if (p >= 2u * n) return kNoItem;
    while (gq + 1 < rs.E && q[gq + 1] <= p) gq++;
    uint32_t a = p;  // the A tile, if the position is not in a B block
    if (gq >= 0) {
      const uint32_t start = group_first_tile(rs, gq, n_ct);
      const uint32_t end = group_first_tile(rs, gq + 1, n_ct);
      const uint32_t d = p - q[gq];
      if (d < end - start) {
        group = gq;
        return static_cast<int>(end - 1 - d) | kBItem;
      }
      a = p - end;  // an A tile after group gq's B block
    }
    // the last g whose first row is at or before the tile's (empty groups
    // share their start with the next group and are passed over)
    const int32_t r0 = static_cast<int32_t>(a / static_cast<uint32_t>(n_ct)) * kRows;
    while (ga + 1 < rs.E && rs.off[ga + 1] <= r0) ga++;
    group = ga;
    return static_cast<int>(a);
  }
};

__device__ __forceinline__ int item_tile(int item) { return item & (kBItem - 1); }

// ----------------------------------------------------------- shared memory

constexpr int kQGroups = 3;                                  // compute warp groups
constexpr int kQThreads = kQGroups * kCastThreads + 128;     // + the control warp group
constexpr int kProducerWarp = 4 * kQGroups;                  // warps 12..14: producer of group warp - 12
constexpr int kPublisherWarp = kProducerWarp + kQGroups;     // warp 15
constexpr int kComputeRegs = 160;
constexpr int kControlRegs = 32;
static_assert(kQGroups * kCastThreads * kComputeRegs + 128 * kControlRegs <= 65536,
              "register split above the launch total");
constexpr int kQInfo = 4;  // item info ring (item k: entry k % 4)
// A items a group may have handed to the publisher and not had acknowledged:
// enough that a run of amax items never waits for the publisher's fence
constexpr int kPubSlots = 8;

// One compute group's part of shared memory. Item k uses ring entries k % 2
// (stage, amax copies, encode scales, staged block scales) and k % 4 (info).
struct alignas(16) QuantGroup {
  float col_amax[kStages][kCols];   // B item: the tile's column amax in its group (bulk copy)
  float row_amax[kStages][kRows];   // B item: the tile's row amax (bulk copy)
  float col_senc[kStages][kCols];   // B item: S_enc of those
  float row_senc[kStages][kRows];
  uint8_t col_scale[2][8 * kCols];  // B item: staged colwise block scales
  uint8_t row_scale[2][8 * kRows];  // B item: staged rowwise block scales
  int32_t item[kQInfo];             // written by the producer before the stage's last arrival
  int32_t grp[kQInfo];
  int32_t pub_grp[kPubSlots];       // group of the group's A item a (entry a % kPubSlots), for the publisher
  uint64_t full[kStages];           // 2 producer arrivals + the tile bytes (+ the amax bytes)
  uint64_t empty[kStages];          // 1 arrival: the group holds the stage's tile in registers
  uint64_t adone[kPubSlots];        // 128 arrivals: the group's atomics of an A item are issued
  uint64_t aack[kPubSlots];         // 1 arrival: the publisher has published that A item
  int32_t fail;
  int32_t a_final;                  // the group's number of A items once it is finished, else -1
};

struct QuantSmem {
  uint8_t tile[kQGroups][kStages][kTileBytes];  // at offset 0 of a 1024-byte aligned block
  QuantGroup grp[kQGroups];
  E4m3Table e4m3;                               // the block-scale shortcut's E4M3 table
  RoutingSmem rs;
};

// Dynamic shared memory: QuantSmem, the E+1 group offsets, Q_g of every group.
constexpr size_t quantize_smem_bytes(int E) {
  return ((sizeof(QuantSmem) + 15) & ~size_t{15}) + sizeof(int32_t) * (E + 1) + sizeof(uint32_t) * E;
}

// ------------------------------------------------------------ control roles

// The producer of compute group j: claims items, loads each one's tile and,
// for a B item, the finished maxima into the group's ring. Positions are
// claimed two ahead (hiding the claim's latency) and issued strictly in
// claim order, so while it waits for a B item's group, every position it
// claimed before that item is already issued -- the waits of all producers
// then always have an earliest one that can finish. Returns after the end
// mark, or after a give-up (then the abort word is raised).
template <class Routing>
__device__ __forceinline__ void quantize_producer(QuantSmem& sm, int j, const Routing& routing, const uint32_t* qpos,
                                                  const CUtensorMap* tmap, int K, uint32_t* ws, const float* row_acc,
                                                  const float* col_amax, bool do_row, bool do_col) {
  const RoutingSmem& rs = sm.rs;
  QuantGroup& pg = sm.grp[j];
  uint32_t* const counter = ws;
  uint32_t* const abort_word = ws + 1;
  const uint32_t* const done = ws + kWsDone;
  const int n_ct = K >> 7;
  const uint32_t n = static_cast<uint32_t>(rs.total >> 7) * static_cast<uint32_t>(n_ct);
  const uint32_t amax_bytes = (do_row ? 512u : 0u) + (do_col ? 512u : 0u);
  ItemCursor cur;
  uint32_t q0 = claim(counter);  // the next position to issue
  uint32_t q1 = claim(counter);  // the one after it
  bool fail = false;
  int i = 0;  // items issued
  for (;; i++) {
    const int s = i & 1;
    // stage s is free once the group holds item i - 2 in registers
    if (i >= 2 && !mbar_wait(&pg.empty[s], ((i >> 1) - 1) & 1)) {
      fail = true;
      break;
    }
    int g = 0;
    const int item = cur.next(rs, qpos, n_ct, n, q0, g);
    if (item == kNoItem) {  // the end mark: no bytes, both arrivals
      pg.item[i & 3] = kNoItem;
      mbar_arrive(&pg.full[s]);
      mbar_arrive(&pg.full[s]);
      i++;
      break;
    }
    q0 = q1;
    q1 = claim(counter);
    const bool is_b = (item & kBItem) != 0;
    const int tl = item_tile(item);
    const int rt = tl / n_ct, ct = tl - rt * n_ct;
    const int32_t r0 = rt * kRows;
    pg.item[i & 3] = item;
    pg.grp[i & 3] = g;
    mbar_expect_tx(&pg.full[s], kTileBytes + (is_b ? amax_bytes : 0u));  // first arrival
    // A loads should stay in L2 until the tile's B item; B loads are the last use
    const uint64_t pol = is_b ? policy_evict_first() : policy_evict_last();
    uint8_t* stage = sm.tile[j][s];
    tma_load_2d(stage, tmap, ct * kCols, r0, &pg.full[s], pol);
    tma_load_2d(stage + kBoxBytes, tmap, ct * kCols + kBoxCols, r0, &pg.full[s], pol);
    if (is_b) {
      const uint32_t need = static_cast<uint32_t>((rs.off[g + 1] - rs.off[g]) >> 7) * static_cast<uint32_t>(n_ct);
      if (!wait_group(&done[g], need, abort_word)) {
        pg.item[i & 3] = kAbortItem;
        fail = true;
      }
      // the maxima are final once the counter is seen complete; the copies
      // read them through the async proxy (issued even after a give-up, so
      // that the stage's transaction count completes)
      asm volatile("fence.proxy.async.global;" ::: "memory");
      if (do_row) bulk_load(pg.row_amax[s], row_acc + r0, 512u, &pg.full[s]);
      if (do_col) bulk_load(pg.col_amax[s], col_amax + static_cast<size_t>(g) * K + ct * kCols, 512u, &pg.full[s]);
    }
    mbar_arrive(&pg.full[s]);  // second arrival: the item info is final
    if (fail) {
      i++;
      break;
    }
  }
  if (fail) {
    raise_abort(abort_word);
    routing.report(NVFP4_ERR_TIMEOUT);
  }
  // every copy this thread issued lands before the CTA can exit: the last two
  // items (earlier ones were consumed before their stage was reissued)
  for (int k = i > 2 ? i - 2 : 0; k < i; k++) mbar_wait(&pg.full[k & 1], (k >> 1) & 1);
}

// The publisher: publishes every A item of every compute group in the
// group's order, and acknowledges it so the group may reuse the slot. A
// GPU-scope fence waits for the SM's outstanding stores (about a
// microsecond while the compute groups stream their outputs), so one fence
// serves every A item found ready in a sweep over the groups.
__device__ __forceinline__ void quantize_publisher(QuantSmem& sm, uint32_t* ws) {
  uint32_t* const abort_word = ws + 1;
  uint32_t* const done = ws + kWsDone;
  int a_pub[kQGroups] = {0, 0, 0};
  uint32_t idle = 0;
  for (;;) {
    bool ready[kQGroups];
    bool any = false, all = true;
    for (int j = 0; j < kQGroups; j++) {
      const int a = a_pub[j];
      ready[j] = mbar_test(&sm.grp[j].adone[a % kPubSlots], (a / kPubSlots) & 1);
      any |= ready[j];
    }
    if (any) {
      asm volatile("fence.acq_rel.gpu;" ::: "memory");
      for (int j = 0; j < kQGroups; j++) {
        if (!ready[j]) continue;
        QuantGroup& pg = sm.grp[j];
        const int a = a_pub[j];
        const int g = reinterpret_cast<volatile int32_t*>(pg.pub_grp)[a % kPubSlots];
        if (NVFP4_STORE_OK(&done[g], 4))
          asm volatile("red.relaxed.gpu.global.add.u32 [%0], 1;" ::"l"(&done[g]) : "memory");
        mbar_arrive(&pg.aack[a % kPubSlots]);
        a_pub[j] = a + 1;
      }
    }
    for (int j = 0; j < kQGroups; j++) {
      const int af = *reinterpret_cast<volatile int32_t*>(&sm.grp[j].a_final);
      if (af < 0 || a_pub[j] < af) all = false;
    }
    if (all) return;
    if (any) {
      idle = 0;
    } else if (++idle > kIdleLimit || ld_relaxed_u32(abort_word) != 0u) {
      return;  // the compute groups stop on their own bounded waits
    } else {
      __nanosleep(256);  // leave the issue slots to the compute warps
    }
  }
}

// ----------------------------------------------------------------- kernel

// kTiled: both scale outputs in the 128x4-tiled layout.
template <class Routing, bool kTiled>
__global__ void __launch_bounds__(kQThreads, 1)
group_quantize_kernel(const __grid_constant__ Routing routing, const __grid_constant__ CUtensorMap tmap,
                      int32_t K, int32_t lag, uint32_t* ws, float* row_acc, float* row_amax,
                      float* col_amax, const CastOut out) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  QuantSmem& sm = *reinterpret_cast<QuantSmem*>(base);
  int32_t* off = reinterpret_cast<int32_t*>(base + ((sizeof(QuantSmem) + 15) & ~size_t{15}));

  routing.load(sm.rs, off);
  const RoutingSmem& rs = sm.rs;
  if (!rs.ok) return;

  const int t = threadIdx.x;
  const int E = rs.E;
  const bool do_row = out.row_s2 != nullptr;
  const bool do_col = out.col_s2 != nullptr;
  const int n_ct = K >> 7;
  const uint32_t n = static_cast<uint32_t>(rs.total >> 7) * static_cast<uint32_t>(n_ct);
  uint32_t* qpos = reinterpret_cast<uint32_t*>(off + E + 1);
  uint32_t* const abort_word = ws + 1;

  for (int g = t; g < E; g += kQThreads) {
    const uint32_t start = group_first_tile(rs, g, n_ct);
    const uint32_t end = group_first_tile(rs, g + 1, n_ct);
    qpos[g] = min(n, end + static_cast<uint32_t>(lag)) + start;
  }
  if (do_col) {  // empty groups own no tile: their col_s2 is S_dec(0) (col_amax stays 0)
    for (int g = blockIdx.x; g < E; g += gridDim.x)
      if (off[g + 1] == off[g])
        for (int c = t; c < K; c += kQThreads) gstore(&out.col_s2[static_cast<size_t>(g) * K + c], s_dec_of(0.0f));
  }
  if (t < 128) e4m3_table_fill(sm.e4m3, t);
  if (t == 0) {
    for (int j = 0; j < kQGroups; j++) {
      QuantGroup& pg = sm.grp[j];
      for (int s = 0; s < kStages; s++) {
        mbar_init(&pg.full[s], 2);
        mbar_init(&pg.empty[s], 1);
      }
      for (int s = 0; s < kPubSlots; s++) {
        mbar_init(&pg.adone[s], kCastThreads);
        mbar_init(&pg.aack[s], 1);
      }
      pg.fail = 0;
      pg.a_final = -1;
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();  // the last CTA-wide barrier: the roles part here

  const int warp = t >> 5, lane = t & 31;
  if (warp >= kProducerWarp) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kControlRegs));
    if (lane == 0 && warp < kPublisherWarp)
      quantize_producer(sm, warp - kProducerWarp, routing, qpos, &tmap, K, ws, row_acc, col_amax, do_row, do_col);
    else if (lane == 0)
      quantize_publisher(sm, ws);
    return;
  }
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kComputeRegs));

  // ========================================================= compute groups
  const int j = warp >> 2;  // compute group
  const int gt = t - j * kCastThreads;
  const int w = gt >> 5;
  QuantGroup& pg = sm.grp[j];
  const int c8 = lane & 7, hb = lane >> 3;
  const int cc = 8 * (w & 1) + c8;  // 8-column chunk of the tile, 0..15
  const int rb = 4 * (w >> 1) + hb;  // 16-row block of the tile, 0..7
  const int rl = 16 * rb;
  const size_t row_pitch = static_cast<size_t>(K) >> 1;
  // every output of a cast item (codes and scales) is stored evict-first, so
  // that the tiles still waiting in L2 for their cast item keep their place
  // (measured against the default policy for rowwise codes and evict-last
  // scales: 1.61 instead of 1.69 GB read from DRAM at the DeepSeek-V3 shape,
  // 0.517 instead of 0.524 ms; 1024 tokens: 211 instead of 221 us)
  const uint64_t once = policy_evict_first();
  const int bar_id = 1 + j;

  int a_count = 0;  // A items this group has finished
  int prev_item = kNoItem, prev_g = 0;
  bool failed = false;
  for (int k = 0;; k++) {
    const int s = k & 1;
    const bool ok = mbar_wait(&pg.full[s], (k >> 1) & 1);
    const int item = ok ? pg.item[k & 3] : kAbortItem;
    const int g = pg.grp[k & 3];
    const bool is_b = item >= 0 && (item & kBItem) != 0;
    const int tl = item_tile(item);
    const int rt = tl / n_ct, ct = tl - rt * n_ct;
    const int32_t r0 = rt * kRows;
    const int c0 = ct * kCols;
    // S_enc of the tile's rows and columns (thread gt: entry gt), and the
    // decode scales (a row's in its first column tile, a column's in its
    // group's first row tile)
    bool slow = false;
    if (is_b) {
      if (do_row) {
        const float a = pg.row_amax[s][gt];
        pg.row_senc[s][gt] = s_enc_of(a);
        slow |= !fast_path_amax(a);
        if (ct == 0) {
          if (row_amax != row_acc) gstore(&row_amax[r0 + gt], a);
          gstore(&out.row_s2[r0 + gt], s_dec_of(a));
        }
      }
      if (do_col) {
        const float a = pg.col_amax[s][gt];
        pg.col_senc[s][gt] = s_enc_of(a);
        slow |= !fast_path_amax(a);
        if (r0 == rs.off[g]) gstore(&out.col_s2[static_cast<size_t>(g) * K + c0 + gt], s_dec_of(a));
      }
    }
    if (item == kAbortItem) pg.fail = 1;
    uint4 v[16];
    if (item >= 0) load_patch(sm.tile[j][s], cc, rl, v);
    const bool any_slow = group_bar_or(bar_id, slow);
    if (pg.fail) {
      failed = true;
      break;
    }
    // every patch of this item is in registers: the stage may be refilled
    if (gt == 0 && item >= 0) mbar_arrive(&pg.empty[s]);
    if (prev_item >= 0 && (prev_item & kBItem) != 0) {
      // the previous item's staged scales (complete since the barrier)
      const int tp = item_tile(prev_item), rtp = tp / n_ct;
      store_scales<kTiled>(pg.col_scale[(k - 1) & 1], pg.row_scale[(k - 1) & 1], out, K, rs.off[prev_g],
                           rs.off[prev_g + 1] - rs.off[prev_g], rtp * kRows, (tp - rtp * n_ct) * kCols, gt,
                           do_row, do_col, once);
    }
    if (item < 0) break;  // the end mark
    prev_item = item;
    prev_g = g;

    if (is_b) {
      // ------------------------------------------------------------ B item
      const int32_t o_g = rs.off[g];
      const size_t half_m = static_cast<size_t>(rs.off[g + 1] - o_g) >> 1;
      uint8_t* rdst = do_row ? out.row_data + static_cast<size_t>(r0 + rl) * row_pitch + (c0 >> 1) + 4 * cc : nullptr;
      DirectColSink sink{do_col ? out.col_data + (static_cast<size_t>(K) * o_g >> 1) +
                                      static_cast<size_t>(c0 + 8 * cc) * half_m + ((r0 - o_g + rl) >> 1)
                                : nullptr,
                         half_m, once, do_col, {}};
      const EncodeTables tab{&sm.e4m3, pg.row_senc[s]};
      uint64_t cse[4];
      if (do_col) col_senc_pairs(pg.col_senc[s], cc, cse);
      if (any_slow)
        encode_patch<true, true>(v, tab, cse, pg.col_scale[k & 1], pg.row_scale[k & 1], do_row, do_col, cc, rb,
                                 rdst, row_pitch, true, sink, once);
      else
        encode_patch<false, true>(v, tab, cse, pg.col_scale[k & 1], pg.row_scale[k & 1], do_row, do_col, cc, rb,
                                  rdst, row_pitch, true, sink, once);
    } else {
      // ------------------------------------------------------------ A item
      // column maxima over the warp's 64 rows (lanes hb = 0..3 share the
      // lane's 8 columns; lane hb takes columns 2hb, 2hb + 1 of them) and row
      // maxima over the warp's 64 columns (lanes c8 = 0..7 share the rows;
      // lane c8 takes rows 2c8, 2c8 + 1 of its block): one atomic max per
      // value, so each row and column of the tile gets two, one per half
      if (do_col) {
        uint32_t cm[4] = {v[0].x, v[0].y, v[0].z, v[0].w};
#pragma unroll
        for (int i = 1; i < 16; i++) {
          cm[0] = maxabs2(cm[0], v[i].x);
          cm[1] = maxabs2(cm[1], v[i].y);
          cm[2] = maxabs2(cm[2], v[i].z);
          cm[3] = maxabs2(cm[3], v[i].w);
        }
#pragma unroll
        for (int q = 0; q < 4; q++) {
          cm[q] &= 0x7FFF7FFFu;
          cm[q] = umax2(cm[q], __shfl_xor_sync(0xFFFFFFFFu, cm[q], 8));
          cm[q] = umax2(cm[q], __shfl_xor_sync(0xFFFFFFFFu, cm[q], 16));
        }
        const uint32_t mine = hb == 0 ? cm[0] : hb == 1 ? cm[1] : hb == 2 ? cm[2] : cm[3];
        float* dst = &col_amax[static_cast<size_t>(g) * K + c0 + 8 * cc + 2 * hb];
        red_max_u32(dst, mine << 16);
        red_max_u32(dst + 1, mine & 0xFFFF0000u);
      }
      if (do_row) {
        // P[kk] = maxima of rows (2kk, 2kk+1) of the block over this lane's 8 columns
        uint32_t P[8];
#pragma unroll
        for (int kk = 0; kk < 8; kk++) {
          const uint32_t a = maxabs2(maxabs2(v[2 * kk].x, v[2 * kk].y), maxabs2(v[2 * kk].z, v[2 * kk].w));
          const uint32_t b = maxabs2(maxabs2(v[2 * kk + 1].x, v[2 * kk + 1].y),
                                     maxabs2(v[2 * kk + 1].z, v[2 * kk + 1].w));
          P[kk] = maxabs2(prmt(a, b, 0x5410), prmt(a, b, 0x7632)) & 0x7FFF7FFFu;
        }
        // reduce-scatter over the 8 lanes sharing these rows: lane c8 ends
        // with the maxima of rows 2*c8 and 2*c8 + 1 of the block
        const bool b2 = c8 & 4, b1 = c8 & 2, b0 = c8 & 1;
        uint32_t Q4[4];
#pragma unroll
        for (int kk = 0; kk < 4; kk++) {
          const uint32_t mine = b2 ? P[4 + kk] : P[kk];
          const uint32_t send = b2 ? P[kk] : P[4 + kk];
          Q4[kk] = umax2(mine, __shfl_xor_sync(0xFFFFFFFFu, send, 4));
        }
        uint32_t R2[2];
#pragma unroll
        for (int kk = 0; kk < 2; kk++) {
          const uint32_t mine = b1 ? Q4[2 + kk] : Q4[kk];
          const uint32_t send = b1 ? Q4[kk] : Q4[2 + kk];
          R2[kk] = umax2(mine, __shfl_xor_sync(0xFFFFFFFFu, send, 2));
        }
        const uint32_t S1 = umax2(b0 ? R2[1] : R2[0], __shfl_xor_sync(0xFFFFFFFFu, b0 ? R2[0] : R2[1], 1));
        float* dst = &row_acc[r0 + rl + 2 * c8];
        red_max_u32(dst, S1 << 16);
        red_max_u32(dst + 1, S1 & 0xFFFF0000u);
      }
      // hand the item to the publisher (slot a % kPubSlots, free once A item
      // a - kPubSlots is acknowledged)
      const int a = a_count;
      if (gt == 0) {
        if (a >= kPubSlots && !mbar_wait(&pg.aack[a % kPubSlots], ((a / kPubSlots) - 1) & 1)) {
          pg.fail = 1;  // seen by the group at its next barrier
          raise_abort(abort_word);
        }
        reinterpret_cast<volatile int32_t*>(pg.pub_grp)[a % kPubSlots] = g;
      }
      mbar_arrive(&pg.adone[a % kPubSlots]);
      a_count = a + 1;
    }
  }
  if (gt == 0) *reinterpret_cast<volatile int32_t*>(&pg.a_final) = a_count;
  if (failed && gt == 0) {
    raise_abort(abort_word);
    routing.report(NVFP4_ERR_TIMEOUT);
  }
}

}  // namespace nvfp4rs
