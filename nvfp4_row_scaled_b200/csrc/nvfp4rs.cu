// nvfp4rs.cu -- the C ABI of include/nvfp4rs.h: host-side checks, grid
// shapes and launches of the grouped amax / grouped cast / dequantize kernels.
//
// Each public call validates its arguments on the host, then only enqueues
// memsets and kernels on the caller's stream: no allocation, no
// synchronisation, no host read of device memory, so every call can be
// captured in a CUDA graph. The host-split and graph-safe calls instantiate
// the same kernel templates with a different routing front-end
// (routing.cuh), which is what makes their outputs byte-identical
// (TransformerEngine #3649, grouped row-scaled NVFP4 cast, Description).
#include <algorithm>
#include <cstdint>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include "nvfp4rs.h"
#include "codec.cuh"
#include "routing.cuh"
#include "group_amax.cuh"
#include "group_cast.cuh"
#include "group_cast_plain.cuh"
#include "group_quantize.cuh"
#include "dequant.cuh"
#include "post_scale.cuh"
#include "mx_cast.cuh"

using namespace nvfp4rs;

namespace {

constexpr int64_t kMaxRows = (int64_t{1} << 31) - kRows;
constexpr int kMxBlock = 32;  // MXFP4 block: 32 elements along K (rowwise) and along a group's rows (colwise)
constexpr int kMaxAmaxCols = 32768;  // columns per amax CTA (dynamic shared memory)

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

nvfp4_status cuda_status(cudaError_t e) { return e == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA; }

#ifdef NVFP4_CHECK_BOUNDS
// The checked debug build: the byte ranges a launch may touch, registered on
// its stream just before it (see bounds.cuh). The first range must be an
// input of at least 512 bytes (x) wherever the kernel makes bulk copies.
struct SpanList {
  Spans s{};
  bool overflow = false;
  SpanList& add(const void* p, size_t bytes, bool store) {
    if (p != nullptr && bytes > 0 && s.n == kMaxSpans) overflow = true;
    if (p != nullptr && bytes > 0 && s.n < kMaxSpans) {
      s.lo[s.n] = reinterpret_cast<uint64_t>(p);
      s.hi[s.n] = s.lo[s.n] + bytes;
      s.store[s.n] = store ? 1u : 0u;
      s.n++;
    }
    return *this;
  }
  SpanList& routing(const HostRouting&) { return *this; }
  SpanList& routing(const DeviceRouting& r) {
    if (r.uniform_rows >= 0) return add(r.status, 4, true);
    return add(r.first_dims, static_cast<size_t>(r.E) * 8, false)
        .add(r.tensor_offsets, static_cast<size_t>(r.E + 1) * 8, false)
        .add(r.status, 4, true);
  }
  SpanList& outputs(const CastOut& o, int64_t rows, int64_t K, int32_t E) {
    const size_t n = static_cast<size_t>(rows) * static_cast<size_t>(K);
    return add(o.row_data, n / 2, true).add(o.row_scale, n / 16, true).add(o.row_s2, 4 * static_cast<size_t>(rows), true)
        .add(o.col_data, n / 2, true).add(o.col_scale, n / 16, true).add(o.col_s2, 4 * static_cast<size_t>(E) * K, true);
  }
  nvfp4_status set(cudaStream_t stream) const {
    if (overflow) return NVFP4_ERR_UNSUPPORTED;  // more ranges than the table holds
    set_spans_kernel<<<1, 1, 0, stream>>>(s);
    return cuda_status(cudaGetLastError());
  }
};
#define NVFP4_SPANS(expr)                           \
  do {                                              \
    const nvfp4_status span_status = (expr);        \
    if (span_status != NVFP4_OK) return span_status; \
  } while (0)
#else
#define NVFP4_SPANS(expr) \
  do {                    \
  } while (0)
#endif

// CTAs per cluster along K for the amax kernel: the largest d <= 8 that
// divides the number of 128-column chunks (ceil(K/128)) and leaves every CTA
// at least 4 of them -- below that the per-CTA setup (routing, the cluster merge of the
// row maxima) costs more than the extra CTAs gain: at K = 2048, 4 CTAs of 4
// chunks run the amax 9-15% faster than 8 CTAs of 2. A problem that would
// then have fewer CTAs than the GPU has SMs takes the largest d <= 8 that
// divides the chunks instead.
int amax_cluster(int64_t K, int64_t tiles = INT64_MAX, int sms = 0) {
  const int64_t chunks = (K + kCols - 1) / kCols;
  int widest = 1, wide4 = 1;
  for (int d = 8; d > 1; d--)
    if (chunks % d == 0) {
      if (widest == 1) widest = d;
      if (wide4 == 1 && chunks / d >= 4) wide4 = d;
    }
  return (sms > 0 && tiles < (sms + wide4 - 1) / wide4) ? widest : wide4;
}

// Columns of the amax kernel's per-CTA table: its share of the 128-column chunks.
int64_t amax_cta_cols(int64_t K, int cn) { return ((K + kCols - 1) / kCols) / cn * kCols; }

// Shape checks shared by both steps and both routings: K any multiple of 16
// (k128: the calls that need K % 128 == 0 -- the one-launch, MXFP4 and
// tiled-scale paths -- return NVFP4_ERR_UNSUPPORTED otherwise).
nvfp4_status check_shape(const void* x, int64_t rows, int64_t K, int32_t E, bool k128 = false) {
  if (rows < 0 || K < 0 || E < 0) return NVFP4_ERR_INVALID_ARG;
  if (K % 16 != 0) return NVFP4_ERR_INVALID_ARG;
  if (rows > 0 && K > 0 && x == nullptr) return NVFP4_ERR_INVALID_ARG;
  if ((k128 && K % kCols != 0) || E > NVFP4_MAX_GROUPS || rows > kMaxRows) return NVFP4_ERR_UNSUPPORTED;
  if (amax_cta_cols(K, amax_cluster(K)) > kMaxAmaxCols) return NVFP4_ERR_UNSUPPORTED;
  if (((rows + kRows - 1) / kRows) * ((K + kCols - 1) / kCols) > (int64_t{1} << 30))
    return NVFP4_ERR_UNSUPPORTED;  // tile ids fit int32
  if (!aligned(x, 16)) return NVFP4_ERR_UNSUPPORTED;
  return NVFP4_OK;
}

// Host splits -> HostRouting (row offsets), with the split checks. Every
// group must be a multiple of `align` rows (16 for the two-step calls, 128
// for the one-launch calls), else NVFP4_ERR_UNSUPPORTED.
nvfp4_status host_routing(const int64_t* m_splits, int32_t E, int64_t sum_M, HostRouting& r,
                          int32_t align = kBlockRows, bool* all_128 = nullptr) {
  if (E > 0 && m_splits == nullptr) return NVFP4_ERR_INVALID_ARG;
  int64_t total = 0;
  bool unaligned = false;
  r.E = E;
  r.off[0] = 0;
  for (int32_t g = 0; g < E; g++) {
    if (m_splits[g] < 0) return NVFP4_ERR_INVALID_ARG;
    if (m_splits[g] % align != 0) unaligned = true;
    total += m_splits[g];
    if (total > sum_M) return NVFP4_ERR_INVALID_ARG;
    r.off[g + 1] = static_cast<int32_t>(total);
  }
  if (total != sum_M) return NVFP4_ERR_INVALID_ARG;
  if (unaligned) return NVFP4_ERR_UNSUPPORTED;
  bool a128 = true;
  for (int32_t g = 0; g < E; g++) a128 = a128 && m_splits[g] % kRows == 0;
  if (all_128 != nullptr) *all_128 = a128;
  r.all128 = a128;
  r.total = static_cast<int32_t>(total);
  return NVFP4_OK;
}

// Routing arguments of a graph-safe call -> DeviceRouting, with the host-side
// checks. Both arrays NULL selects uniform groups: num_groups groups of
// capacity_rows / num_groups rows each (which must divide exactly).
nvfp4_status device_routing(const int64_t* first_dims, const int64_t* offsets, int32_t* status,
                            int64_t K, int64_t capacity_rows, int32_t E, int32_t align,
                            DeviceRouting& r) {
  if (status == nullptr) return NVFP4_ERR_INVALID_ARG;
  const bool uniform = first_dims == nullptr && offsets == nullptr;
  int64_t m = -1;
  if (uniform) {
    m = 0;
    if (E > 0) {
      if (capacity_rows % E != 0) return NVFP4_ERR_INVALID_ARG;
      m = capacity_rows / E;
      if (m % align != 0) return NVFP4_ERR_UNSUPPORTED;
    }
  } else if (offsets == nullptr || (E > 0 && first_dims == nullptr)) {
    return NVFP4_ERR_INVALID_ARG;
  }
  if (!aligned(status, 4) || !aligned(first_dims, 8) || !aligned(offsets, 8)) return NVFP4_ERR_UNSUPPORTED;
  r = DeviceRouting{first_dims, offsets, status, K, capacity_rows, E, align, m};
  return NVFP4_OK;
}

// A direction is requested when any of its three pointers is set; then every
// one of its buffers that has a nonzero size must be set (a zero-size buffer
// may be NULL, as allocators hand out for empty tensors).
nvfp4_status check_outputs(const nvfp4_outputs* out, int64_t rows, int64_t K, int32_t E,
                           bool& do_row, bool& do_col) {
  if (out == nullptr) return NVFP4_ERR_INVALID_ARG;
  if (out->scale_layout != NVFP4_SCALE_COMPACT && out->scale_layout != NVFP4_SCALE_TILED_128X4)
    return NVFP4_ERR_INVALID_ARG;
  do_row = out->row_data != nullptr || out->row_scale != nullptr || out->row_s2 != nullptr;
  do_col = out->col_data != nullptr || out->col_scale != nullptr || out->col_s2 != nullptr;
  const bool has_rows = rows > 0 && K > 0;
  if (do_row && has_rows && (out->row_data == nullptr || out->row_scale == nullptr || out->row_s2 == nullptr))
    return NVFP4_ERR_INVALID_ARG;
  if (do_col && ((has_rows && (out->col_data == nullptr || out->col_scale == nullptr)) ||
                 (E > 0 && K > 0 && out->col_s2 == nullptr)))
    return NVFP4_ERR_INVALID_ARG;
  if (!aligned(out->row_data, 16) || !aligned(out->row_scale, 16) || !aligned(out->col_data, 16) ||
      !aligned(out->col_scale, 16) || !aligned(out->row_s2, 4) || !aligned(out->col_s2, 4))
    return NVFP4_ERR_UNSUPPORTED;
  return NVFP4_OK;
}

// cuTensorMapEncodeTiled, fetched once through the runtime (no link to libcuda)
PFN_cuTensorMapEncodeTiled_v12000 encode_tiled() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<PFN_cuTensorMapEncodeTiled_v12000>(nullptr);
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }();
  return fn;
}

// TMA descriptor of x [rows, K] bf16: boxes of 64 columns x 128 rows,
// 128-byte swizzle (the layout the cast kernel reads back).
bool x_tensor_map(CUtensorMap* map, const void* x, int64_t rows, int64_t K) {
  std::memset(map, 0, sizeof(*map));
  if (rows == 0 || K == 0) return true;  // no tile: the map is never used
  PFN_cuTensorMapEncodeTiled_v12000 fn = encode_tiled();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kBoxCols), static_cast<cuuint32_t>(kRows)};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// col_amax (when given) is zeroed here first, by a kernel after which the
// amax kernel is launched programmatically (group_amax.cuh).
template <class Routing>
nvfp4_status launch_amax(const Routing& routing, const void* x, int64_t rows, int64_t K, int32_t E,
                         float* row_amax, float* col_amax, cudaStream_t stream) {
  const int64_t tiles = (rows + kRows - 1) / kRows;
  const int64_t n_col = col_amax != nullptr ? static_cast<int64_t>(E) * K : 0;
  if (n_col == 0 && (tiles == 0 || K == 0)) return NVFP4_OK;
  NVFP4_SPANS(SpanList{}
                  .add(x, static_cast<size_t>(rows) * K * 2, false)
                  .routing(routing)
                  .add(row_amax, 4 * static_cast<size_t>(rows), true)
                  .add(col_amax, 4 * static_cast<size_t>(E) * K, true)
                  .set(stream));
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return NVFP4_ERR_CUDA;
  if (n_col > 0) {
    const int64_t blocks = std::min<int64_t>((n_col + 255) / 256, 2 * static_cast<int64_t>(sms));
    zero_f32_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(col_amax, n_col);
    const nvfp4_status z = cuda_status(cudaGetLastError());
    if (z != NVFP4_OK) return z;
  }
  if (tiles == 0 || K == 0) return NVFP4_OK;
  const int cn = amax_cluster(K, tiles, sms);
  const size_t smem = static_cast<size_t>(amax_cta_cols(K, cn)) * sizeof(uint32_t) + sizeof(int32_t) * (E + 1);
  auto kernel = group_amax_kernel<Routing>;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return NVFP4_ERR_CUDA;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(tiles * cn));
  cfg.blockDim = dim3(kAmaxThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  // programmatic after the zeroing (its reads of x overlap it; its atomics
  // wait for it); a plain launch when there is no zeroing to overlap
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(cn);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = n_col > 0 ? 2 : 1;
  return cuda_status(cudaLaunchKernelEx(&cfg, kernel, routing, static_cast<const uint4*>(x),
                                        static_cast<int32_t>(K), static_cast<int32_t>(cn),
                                        row_amax, col_amax));
}

// The cast kernel: one CTA per SM, three warp groups, for every routing
// (groups of any multiple of 16 rows; general tiles take the kernel's edge
// path, see group_cast_plain.cuh).
template <class Routing>
nvfp4_status launch_cast(const Routing& routing, const void* x, int64_t rows, int64_t K, int32_t E,
                         const float* row_amax, const float* col_amax, const nvfp4_outputs* out,
                         bool do_col, cudaStream_t stream) {
  const int64_t tiles = ((rows + kRows - 1) / kRows) * ((K + kCols - 1) / kCols);
  const bool s2_work = do_col && E > 0 && K > 0;
  if (tiles == 0 && !s2_work) return NVFP4_OK;
  CUtensorMap map;
  if (!x_tensor_map(&map, x, rows, K)) return NVFP4_ERR_CUDA;
  // tiled scales come with 128-row groups and K % 128 == 0 only (checked on
  // the host, or on the device by the routing): every tile is plain
  const bool tiled = out->scale_layout == NVFP4_SCALE_TILED_128X4;
  auto kernel = tiled ? group_cast_plain_kernel<Routing, true> : group_cast_plain_kernel<Routing, false>;
  const int64_t units = (tiles + kPGroups - 1) / kPGroups;
  static_assert(plain_smem_bytes(NVFP4_MAX_GROUPS) + 1024 <= 227 * 1024, "cast kernel shared memory");
  const size_t smem = plain_smem_bytes(E) + 1024;  // + room to align the block to 1024 bytes
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return NVFP4_ERR_CUDA;
  int dev = 0, sms = 0, per_sm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kPThreads, smem) != cudaSuccess)
    return NVFP4_ERR_CUDA;
  if (per_sm < 1) return NVFP4_ERR_UNSUPPORTED;
  int64_t grid = static_cast<int64_t>(sms) * per_sm;
  if (units > 0 && units < grid) grid = units;
  if (grid < 1) grid = 1;
  CastOut o{out->row_data, out->row_scale, out->row_s2, out->col_data, out->col_scale, out->col_s2,
            out->scale_layout == NVFP4_SCALE_TILED_128X4};
  NVFP4_SPANS(SpanList{}
                  .add(x, static_cast<size_t>(rows) * K * 2, false)
                  .routing(routing)
                  .add(row_amax, 4 * static_cast<size_t>(rows), false)
                  .add(col_amax, 4 * static_cast<size_t>(E) * K, false)
                  .outputs(o, rows, K, E)
                  .set(stream));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kPThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  // programmatic dependent launch: the kernel's set-up may overlap the tail
  // of the kernel before it (the grouped amax); it waits for that kernel
  // before reading anything (griddepcontrol.wait, group_cast_plain.cuh)
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cuda_status(cudaLaunchKernelEx(&cfg, kernel, routing, map, static_cast<int32_t>(K), row_amax,
                                        col_amax, o));
}

// Persistent grid of the one-launch kernel: one CTA per SM (three compute
// groups each), fewer for a problem with fewer items. The schedule's lag --
// claims between a group's last A item and its first B item -- is a few
// rounds of every compute group in the grid, so that the A items are
// published by the time the B items are claimed.
constexpr int kQuantLagRounds = 3;

template <class Routing>
nvfp4_status launch_quantize(const Routing& routing, const void* x, int64_t rows, int64_t K, int32_t E,
                             uint32_t* ws, float* row_acc, float* row_amax, float* col_amax,
                             const nvfp4_outputs* out, bool do_col, cudaStream_t stream) {
  const int64_t tiles = (rows / kRows) * (K / kCols);
  const bool s2_work = do_col && E > 0 && K > 0;
  if (tiles == 0 && !s2_work) return NVFP4_OK;
  CUtensorMap map;
  if (!x_tensor_map(&map, x, rows, K)) return NVFP4_ERR_CUDA;
  auto kernel = out->scale_layout == NVFP4_SCALE_TILED_128X4 ? group_quantize_kernel<Routing, true>
                                                             : group_quantize_kernel<Routing, false>;
  const size_t smem = quantize_smem_bytes(E) + 1024;  // + room to align the block to 1024 bytes
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return NVFP4_ERR_CUDA;
  int dev = 0, sms = 0, per_sm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kQThreads, smem) != cudaSuccess)
    return NVFP4_ERR_CUDA;
  if (per_sm < 1) return NVFP4_ERR_UNSUPPORTED;
  int64_t grid = static_cast<int64_t>(sms) * per_sm;
  const int64_t need = (2 * tiles + kQGroups - 1) / kQGroups;  // CTAs that get an item
  if (need < grid) grid = need;
  if (grid < 1) grid = 1;
  const int32_t lag = static_cast<int32_t>(kQuantLagRounds * kQGroups * grid);
  CastOut o{out->row_data, out->row_scale, out->row_s2, out->col_data, out->col_scale, out->col_s2,
            out->scale_layout == NVFP4_SCALE_TILED_128X4};
  NVFP4_SPANS(SpanList{}
                  .add(x, static_cast<size_t>(rows) * K * 2, false)
                  .routing(routing)
                  .add(ws, 4 * static_cast<size_t>(quant_ws_header_words(E)), true)
                  .add(row_acc, 4 * static_cast<size_t>(rows), true)
                  .add(row_amax, 4 * static_cast<size_t>(rows), true)
                  .add(col_amax, 4 * static_cast<size_t>(E) * K, true)
                  .outputs(o, rows, K, E)
                  .set(stream));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kQThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  return cuda_status(cudaLaunchKernelEx(&cfg, kernel, routing, map, static_cast<int32_t>(K), lag, ws,
                                        row_acc, row_amax, col_amax, o));
}

// Argument checks of the one-launch calls beyond check_shape / check_outputs.
nvfp4_status check_quantize(int64_t rows, int64_t K, int32_t E, bool do_row, bool do_col,
                            const float* row_amax, const float* col_amax, const void* workspace,
                            size_t workspace_bytes, int64_t ws_rows) {
  if ((do_row && rows > 0 && row_amax == nullptr) || (do_col && E > 0 && K > 0 && col_amax == nullptr))
    return NVFP4_ERR_INVALID_ARG;
  if (workspace == nullptr ||
      workspace_bytes < nvfp4_group_quantize_workspace_bytes(ws_rows, E))
    return NVFP4_ERR_INVALID_ARG;
  // the kernel copies 512-byte runs of both amax vectors with the TMA unit
  if (!aligned(row_amax, 16) || !aligned(col_amax, 16) || !aligned(workspace, 16))
    return NVFP4_ERR_UNSUPPORTED;
  return NVFP4_OK;
}

// Zero what the one-launch kernel accumulates into: the workspace header, the
// row accumulators (rows of them, when the row direction is requested) and
// col_amax (when the column direction is).
nvfp4_status zero_quantize_state(void* workspace, int32_t E, float* row_acc, int64_t rows, bool do_row,
                                 float* col_amax, int64_t K, bool do_col, cudaStream_t stream) {
  nvfp4_status s = cuda_status(cudaMemsetAsync(
      workspace, 0, static_cast<size_t>(quant_ws_header_words(E)) * sizeof(uint32_t), stream));
  if (s == NVFP4_OK && do_row && rows > 0)
    s = cuda_status(cudaMemsetAsync(row_acc, 0, static_cast<size_t>(rows) * sizeof(float), stream));
  if (s == NVFP4_OK && do_col && E > 0 && K > 0)
    s = cuda_status(cudaMemsetAsync(col_amax, 0, static_cast<size_t>(E) * K * sizeof(float), stream));
  return s;
}

#ifdef NVFP4_TEST_HOOKS
// Test builds only (libnvfp4rs_test.so): the one-launch calls start their
// item counter at this position instead of 0. The amax items before it are
// then never claimed, so a cast item's bounded wait for its group runs out:
// the test of the kernel's timeout path. The product library has no hook.
uint8_t g_test_first_position = 0;

// Sets the counter's first byte (the workspace header is zero just before).
nvfp4_status test_hook_first_position(void* workspace, cudaStream_t stream) {
  if (g_test_first_position == 0) return NVFP4_OK;
  return cuda_status(cudaMemsetAsync(workspace, g_test_first_position, 1, stream));
}
#define NVFP4_TEST_HOOK(ws, stream)                                  \
  do {                                                               \
    const nvfp4_status hs = test_hook_first_position((ws), (stream)); \
    if (hs != NVFP4_OK) return hs;                                   \
  } while (0)
#else
#define NVFP4_TEST_HOOK(ws, stream) \
  do {                              \
  } while (0)
#endif

// ------------------------------------------------ scratch without allocation
//
// nvfp4_group_quantize_noalloc runs the one-launch kernel with its scratch in
// this file-scope device array instead of a caller-provided workspace. It is
// for callers that cannot hand over device memory at the call site: a C
// caller with no device allocator of its own, or one that must not allocate
// there because cudaMalloc synchronises the device. The array holds the
// workspace header for up to NVFP4_MAX_GROUPS groups (item counter, abort
// word, one done counter per group); the row accumulators are the caller's
// row_amax, as in the host-split call.
constexpr int64_t kNoAllocScratchWords = quant_ws_header_words(NVFP4_MAX_GROUPS);  // 1088 words
static __device__ __align__(256) uint32_t g_noalloc_scratch[kNoAllocScratchWords];

constexpr int kMaxDevices = 64;

// Device address of g_noalloc_scratch for the current device, looked up once
// per device (with that device current) and cached. nullptr on failure. The
// address belongs to the device's context at lookup time; a cudaDeviceReset
// of that device makes it stale (the header says so). A bounded wait that
// gives up raises abort word 1 inside this array, which no call reads back:
// HostRouting has no status word, so the give-up goes unreported here.
uint32_t* noalloc_scratch() {
  static std::mutex mu;
  static uint32_t* addr[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
    addr[dev] = static_cast<uint32_t*>(p);
  }
  return addr[dev];
}

// MXFP4 output descriptor checks (like check_outputs: a direction is
// requested when either of its pointers is set, then both must be set).
nvfp4_status check_mx_outputs(const nvfp4_mx_outputs* out, int64_t rows, int64_t K, bool& do_row, bool& do_col) {
  if (out == nullptr) return NVFP4_ERR_INVALID_ARG;
  do_row = out->row_data != nullptr || out->row_scale != nullptr;
  do_col = out->col_data != nullptr || out->col_scale != nullptr;
  const bool has_rows = rows > 0 && K > 0;
  if (has_rows && ((do_row && (out->row_data == nullptr || out->row_scale == nullptr)) ||
                   (do_col && (out->col_data == nullptr || out->col_scale == nullptr))))
    return NVFP4_ERR_INVALID_ARG;
  if (!aligned(out->row_data, 16) || !aligned(out->row_scale, 16) || !aligned(out->col_data, 16) ||
      !aligned(out->col_scale, 16))
    return NVFP4_ERR_UNSUPPORTED;
  return NVFP4_OK;
}

template <class Routing>
nvfp4_status launch_mx_cast(const Routing& routing, const void* x, int64_t rows, int64_t K, int32_t E,
                            const nvfp4_mx_outputs* out, cudaStream_t stream) {
  const int64_t tiles = ((rows + kRows - 1) / kRows) * ((K + kCols - 1) / kCols);
  if (tiles == 0) return NVFP4_OK;
  CUtensorMap map;
  if (!x_tensor_map(&map, x, rows, K)) return NVFP4_ERR_CUDA;
  auto kernel = mx_cast_kernel<Routing>;
  const size_t smem = mx_smem_bytes(E) + 1024;  // + room to align the block to 1024 bytes
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
      cudaSuccess)
    return NVFP4_ERR_CUDA;
  int dev = 0, sms = 0, per_sm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kPThreads, smem) != cudaSuccess)
    return NVFP4_ERR_CUDA;
  if (per_sm < 1) return NVFP4_ERR_UNSUPPORTED;
  int64_t grid = static_cast<int64_t>(sms) * per_sm;
  const int64_t units = (tiles + kPGroups - 1) / kPGroups;
  if (units < grid) grid = units;
  const MxOut o{out->row_data, out->row_scale, out->col_data, out->col_scale};
#ifdef NVFP4_CHECK_BOUNDS
  {
    const size_t n = static_cast<size_t>(rows) * K;
    NVFP4_SPANS(SpanList{}
                    .add(x, n * 2, false)
                    .routing(routing)
                    .add(o.row_data, n / 2, true)
                    .add(o.row_scale, n / 32, true)
                    .add(o.col_data, n / 2, true)
                    .add(o.col_scale, n / 32, true)
                    .set(stream));
  }
#endif
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kPThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  return cuda_status(cudaLaunchKernelEx(&cfg, kernel, routing, map, static_cast<int32_t>(K), o));
}

// One warp per row at a time, every SM filled (8 CTAs of 256 threads).
template <bool kMx>
nvfp4_status launch_dequant(const uint8_t* data, const uint8_t* scale, const float* s2, int64_t rows, int64_t cols,
                            float* out_f32, cudaStream_t stream) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t rows_per_cta = kDequantThreads / 32;
  int64_t grid = (rows + rows_per_cta - 1) / rows_per_cta;
#ifdef NVFP4_CHECK_BOUNDS
  {
    const size_t n = static_cast<size_t>(rows) * static_cast<size_t>(cols);
    NVFP4_SPANS(SpanList{}
                    .add(data, n / 2, false)
                    .add(scale, kMx ? n / 32 : n / 16, false)
                    .add(s2, kMx ? 0 : 4 * static_cast<size_t>(rows), false)
                    .add(out_f32, n * 4, true)
                    .set(stream));
  }
#endif
  if (grid > static_cast<int64_t>(sms) * 8) grid = static_cast<int64_t>(sms) * 8;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kDequantThreads);
  cfg.stream = stream;
  return cuda_status(cudaLaunchKernelEx(&cfg, dequant_kernel<kMx>, reinterpret_cast<const uint16_t*>(data), scale, s2,
                                        rows, cols, reinterpret_cast<float4*>(out_f32)));
}

// The host-split one-launch calls on a routing the single-launch kernel does
// not take (a group not a multiple of 128 rows, or K % 128 != 0): the grouped
// amax and the grouped cast, the two launches of the two-step calls, with the
// same outputs. The 128x4-tiled layout needs 128-row groups either way.
nvfp4_status quantize_two_launches(const HostRouting& routing, const void* x, int64_t rows, int64_t K, int32_t E,
                                   float* row_amax, float* col_amax, const nvfp4_outputs* out, bool do_row,
                                   bool do_col, cudaStream_t stream) {
  if (out->scale_layout == NVFP4_SCALE_TILED_128X4) return NVFP4_ERR_UNSUPPORTED;
  float* ra = do_row ? row_amax : nullptr;
  float* ca = do_col ? col_amax : nullptr;
  const nvfp4_status s = launch_amax(routing, x, rows, K, E, ra, ca, stream);
  if (s != NVFP4_OK) return s;
  return launch_cast(routing, x, rows, K, E, ra, ca, out, do_col, stream);
}

}  // namespace

extern "C" {

nvfp4_status nvfp4_group_amax(const void* x_bf16, int64_t sum_M, int64_t K,
                              const int64_t* m_splits_host, int32_t num_groups, float* row_amax,
                              float* col_amax, cudaStream_t stream) {
  nvfp4_status s = check_shape(x_bf16, sum_M, K, num_groups);
  if (s != NVFP4_OK) return s;
  if (sum_M > 0 && row_amax == nullptr && col_amax == nullptr) return NVFP4_ERR_INVALID_ARG;
  if (!aligned(row_amax, 4) || !aligned(col_amax, 4)) return NVFP4_ERR_UNSUPPORTED;
  static thread_local HostRouting routing;
  s = host_routing(m_splits_host, num_groups, sum_M, routing);
  if (s != NVFP4_OK) return s;
  return launch_amax(routing, x_bf16, sum_M, K, num_groups, row_amax, col_amax, stream);
}

nvfp4_status nvfp4_group_cast(const void* x_bf16, int64_t sum_M, int64_t K,
                              const int64_t* m_splits_host, int32_t num_groups,
                              const float* row_amax, const float* col_amax,
                              const nvfp4_outputs* out, cudaStream_t stream) {
  nvfp4_status s = check_shape(x_bf16, sum_M, K, num_groups);
  if (s != NVFP4_OK) return s;
  bool do_row = false, do_col = false;
  s = check_outputs(out, sum_M, K, num_groups, do_row, do_col);
  if (s != NVFP4_OK) return s;
  if ((do_row && sum_M > 0 && row_amax == nullptr) ||
      (do_col && num_groups > 0 && K > 0 && col_amax == nullptr))
    return NVFP4_ERR_INVALID_ARG;
  // the cast copies 512-byte runs of both amax vectors with the TMA unit
  if (!aligned(row_amax, 16) || !aligned(col_amax, 16)) return NVFP4_ERR_UNSUPPORTED;
  static thread_local HostRouting routing;
  bool all_128 = true;
  s = host_routing(m_splits_host, num_groups, sum_M, routing, kBlockRows, &all_128);
  if (s != NVFP4_OK) return s;
  // the 128x4-tiled layout is made of whole 128-row, 4-block tiles
  if (out->scale_layout == NVFP4_SCALE_TILED_128X4 && (!all_128 || K % kCols != 0)) return NVFP4_ERR_UNSUPPORTED;
  return launch_cast(routing, x_bf16, sum_M, K, num_groups, row_amax, col_amax, out, do_col, stream);
}

nvfp4_status nvfp4_group_amax_graphsafe(const void* x_bf16, int64_t capacity_rows, int64_t K,
                                        const int64_t* first_dims_dev,
                                        const int64_t* tensor_offsets_dev, int32_t num_groups,
                                        float* row_amax, float* col_amax, int32_t* status_dev,
                                        cudaStream_t stream) {
  nvfp4_status s = check_shape(x_bf16, capacity_rows, K, num_groups);
  if (s != NVFP4_OK) return s;
  DeviceRouting routing;
  s = device_routing(first_dims_dev, tensor_offsets_dev, status_dev, K, capacity_rows, num_groups,
                     kBlockRows, routing);
  if (s != NVFP4_OK) return s;
  if (capacity_rows > 0 && row_amax == nullptr && col_amax == nullptr) return NVFP4_ERR_INVALID_ARG;
  if (!aligned(row_amax, 4) || !aligned(col_amax, 4)) return NVFP4_ERR_UNSUPPORTED;
  s = cuda_status(cudaMemsetAsync(status_dev, 0, sizeof(int32_t), stream));
  if (s != NVFP4_OK) return s;
  return launch_amax(routing, x_bf16, capacity_rows, K, num_groups, row_amax, col_amax, stream);
}

nvfp4_status nvfp4_group_cast_graphsafe(const void* x_bf16, int64_t capacity_rows, int64_t K,
                                        const int64_t* first_dims_dev,
                                        const int64_t* tensor_offsets_dev, int32_t num_groups,
                                        const float* row_amax, const float* col_amax,
                                        const nvfp4_outputs* out, int32_t* status_dev,
                                        cudaStream_t stream) {
  nvfp4_status s = check_shape(x_bf16, capacity_rows, K, num_groups);
  if (s != NVFP4_OK) return s;
  bool do_row = false, do_col = false;
  s = check_outputs(out, capacity_rows, K, num_groups, do_row, do_col);
  if (s != NVFP4_OK) return s;
  if ((do_row && capacity_rows > 0 && row_amax == nullptr) ||
      (do_col && num_groups > 0 && K > 0 && col_amax == nullptr))
    return NVFP4_ERR_INVALID_ARG;
  if (!aligned(row_amax, 16) || !aligned(col_amax, 16)) return NVFP4_ERR_UNSUPPORTED;
  // tiled scales need 128-row groups (checked on the device) and K % 128 == 0
  const bool tiled = out->scale_layout == NVFP4_SCALE_TILED_128X4;
  if (tiled && K % kCols != 0) return NVFP4_ERR_UNSUPPORTED;
  DeviceRouting routing;
  s = device_routing(first_dims_dev, tensor_offsets_dev, status_dev, K, capacity_rows, num_groups,
                     tiled ? kRows : kBlockRows, routing);
  if (s != NVFP4_OK) return s;
  s = cuda_status(cudaMemsetAsync(status_dev, 0, sizeof(int32_t), stream));
  if (s != NVFP4_OK) return s;
  if (K == 0) return NVFP4_OK;
  return launch_cast(routing, x_bf16, capacity_rows, K, num_groups, row_amax, col_amax, out, do_col, stream);
}

nvfp4_status nvfp4_dequantize(const uint8_t* data, const uint8_t* scale, const float* s2,
                              int64_t rows, int64_t cols, float* out_f32, cudaStream_t stream) {
  if (rows < 0 || cols < 0 || cols % 16 != 0) return NVFP4_ERR_INVALID_ARG;
  if (rows == 0 || cols == 0) return NVFP4_OK;
  if (data == nullptr || scale == nullptr || s2 == nullptr || out_f32 == nullptr)
    return NVFP4_ERR_INVALID_ARG;
  if (!aligned(data, 8) || !aligned(out_f32, 16) || !aligned(s2, 4)) return NVFP4_ERR_UNSUPPORTED;
  return launch_dequant<false>(data, scale, s2, rows, cols, out_f32, stream);
}

size_t nvfp4_group_quantize_workspace_bytes(int64_t capacity_rows, int32_t num_groups) {
  if (capacity_rows < 0 || num_groups < 0 || num_groups > NVFP4_MAX_GROUPS) return 0;
  return static_cast<size_t>(quant_ws_header_words(num_groups) + capacity_rows) * sizeof(uint32_t);
}

nvfp4_status nvfp4_group_quantize(const void* x_bf16, int64_t sum_M, int64_t K,
                                  const int64_t* m_splits_host, int32_t num_groups, float* row_amax,
                                  float* col_amax, const nvfp4_outputs* out, void* workspace,
                                  size_t workspace_bytes, cudaStream_t stream) {
  nvfp4_status s = check_shape(x_bf16, sum_M, K, num_groups);
  if (s != NVFP4_OK) return s;
  bool do_row = false, do_col = false;
  s = check_outputs(out, sum_M, K, num_groups, do_row, do_col);
  if (s != NVFP4_OK) return s;
  s = check_quantize(sum_M, K, num_groups, do_row, do_col, row_amax, col_amax, workspace,
                     workspace_bytes, 0);
  if (s != NVFP4_OK) return s;
  static thread_local HostRouting routing;
  bool all_128 = true;
  s = host_routing(m_splits_host, num_groups, sum_M, routing, kBlockRows, &all_128);
  if (s != NVFP4_OK) return s;
  if (!do_row && !do_col) return NVFP4_OK;
  if (!all_128 || K % kCols != 0) return quantize_two_launches(routing, x_bf16, sum_M, K, num_groups, row_amax,
                                                               col_amax, out, do_row, do_col, stream);
  // the rows accumulate straight into row_amax
  s = zero_quantize_state(workspace, num_groups, row_amax, sum_M, do_row, col_amax, K, do_col, stream);
  if (s != NVFP4_OK) return s;
  NVFP4_TEST_HOOK(workspace, stream);
  return launch_quantize(routing, x_bf16, sum_M, K, num_groups, static_cast<uint32_t*>(workspace),
                         row_amax, row_amax, col_amax, out, do_col, stream);
}

nvfp4_status nvfp4_group_quantize_graphsafe(const void* x_bf16, int64_t capacity_rows, int64_t K,
                                            const int64_t* first_dims_dev,
                                            const int64_t* tensor_offsets_dev, int32_t num_groups,
                                            float* row_amax, float* col_amax, const nvfp4_outputs* out,
                                            void* workspace, size_t workspace_bytes,
                                            int32_t* status_dev, cudaStream_t stream) {
  nvfp4_status s = check_shape(x_bf16, capacity_rows, K, num_groups, /*k128=*/true);
  if (s != NVFP4_OK) return s;
  bool do_row = false, do_col = false;
  s = check_outputs(out, capacity_rows, K, num_groups, do_row, do_col);
  if (s != NVFP4_OK) return s;
  s = check_quantize(capacity_rows, K, num_groups, do_row, do_col, row_amax, col_amax, workspace,
                     workspace_bytes, capacity_rows);
  if (s != NVFP4_OK) return s;
  DeviceRouting routing;
  s = device_routing(first_dims_dev, tensor_offsets_dev, status_dev, K, capacity_rows, num_groups, kRows,
                     routing);
  if (s != NVFP4_OK) return s;
  s = cuda_status(cudaMemsetAsync(status_dev, 0, sizeof(int32_t), stream));
  if (s != NVFP4_OK || K == 0 || (!do_row && !do_col)) return s;
  // rows beyond the routed total must stay untouched in row_amax, so the rows
  // accumulate in the workspace and are copied out by the cast items
  float* row_acc = reinterpret_cast<float*>(static_cast<uint32_t*>(workspace) +
                                            quant_ws_header_words(num_groups));
  s = zero_quantize_state(workspace, num_groups, row_acc, capacity_rows, do_row, col_amax, K, do_col,
                          stream);
  if (s != NVFP4_OK) return s;
  NVFP4_TEST_HOOK(workspace, stream);
  return launch_quantize(routing, x_bf16, capacity_rows, K, num_groups,
                         static_cast<uint32_t*>(workspace), row_acc, row_amax, col_amax, out, do_col,
                         stream);
}

nvfp4_status nvfp4_group_quantize_noalloc(const void* x_bf16, int64_t sum_M, int64_t K,
                                          const int64_t* m_splits_host, int32_t num_groups,
                                          float* row_amax, float* col_amax, const nvfp4_outputs* out,
                                          cudaStream_t stream) {
  nvfp4_status s = check_shape(x_bf16, sum_M, K, num_groups);
  if (s != NVFP4_OK) return s;
  bool do_row = false, do_col = false;
  s = check_outputs(out, sum_M, K, num_groups, do_row, do_col);
  if (s != NVFP4_OK) return s;
  if ((do_row && sum_M > 0 && row_amax == nullptr) || (do_col && num_groups > 0 && K > 0 && col_amax == nullptr))
    return NVFP4_ERR_INVALID_ARG;
  if (!aligned(row_amax, 16) || !aligned(col_amax, 16)) return NVFP4_ERR_UNSUPPORTED;
  // the static scratch holds the header of at most NVFP4_MAX_GROUPS groups
  if (quant_ws_header_words(num_groups) > kNoAllocScratchWords) return NVFP4_ERR_UNSUPPORTED;
  static thread_local HostRouting routing;
  bool all_128 = true;
  s = host_routing(m_splits_host, num_groups, sum_M, routing, kBlockRows, &all_128);
  if (s != NVFP4_OK) return s;
  if (!do_row && !do_col) return NVFP4_OK;
  if (!all_128 || K % kCols != 0) return quantize_two_launches(routing, x_bf16, sum_M, K, num_groups, row_amax,
                                                               col_amax, out, do_row, do_col, stream);
  uint32_t* scratch = noalloc_scratch();
  if (scratch == nullptr) return NVFP4_ERR_CUDA;
  // zeroed here on `stream`: item counter, abort word, done counters; the
  // rows accumulate straight into row_amax, which is zeroed too
  s = zero_quantize_state(scratch, num_groups, row_amax, sum_M, do_row, col_amax, K, do_col, stream);
  if (s != NVFP4_OK) return s;
  return launch_quantize(routing, x_bf16, sum_M, K, num_groups, scratch, row_amax, row_amax, col_amax, out,
                         do_col, stream);
}

nvfp4_status nvfp4_row_post_scale(const float* gemm_out, int64_t rows, int64_t cols, const float* row_amax,
                                  const float* bias, void* out, int32_t out_dtype, cudaStream_t stream) {
  if (rows < 0 || cols < 0) return NVFP4_ERR_INVALID_ARG;
  if (out_dtype != NVFP4_OUT_F32 && out_dtype != NVFP4_OUT_BF16) return NVFP4_ERR_INVALID_ARG;
  if (rows == 0 || cols == 0) return NVFP4_OK;
  if (gemm_out == nullptr || row_amax == nullptr || out == nullptr) return NVFP4_ERR_INVALID_ARG;
  if (cols % 4 != 0 || !aligned(gemm_out, 16) || !aligned(bias, 16) || !aligned(row_amax, 4) ||
      !aligned(out, out_dtype == NVFP4_OUT_BF16 ? 8 : 16))
    return NVFP4_ERR_UNSUPPORTED;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t units = (rows + kPostUnitRows - 1) / kPostUnitRows * ((cols / 4 + 31) / 32);
  int64_t grid = (units + kPostThreads / 32 - 1) / (kPostThreads / 32);
  const int64_t cap = static_cast<int64_t>(sms) * 2;  // persistent: two CTAs per SM are resident
  if (grid > cap) grid = cap;
  const bool b16 = out_dtype == NVFP4_OUT_BF16, has_bias = bias != nullptr;
#ifdef NVFP4_CHECK_BOUNDS
  {
    const size_t n = static_cast<size_t>(rows) * static_cast<size_t>(cols);
    NVFP4_SPANS(SpanList{}
                    .add(gemm_out, n * 4, false)
                    .add(row_amax, 4 * static_cast<size_t>(rows), false)
                    .add(bias, 4 * static_cast<size_t>(cols), false)
                    .add(out, n * (b16 ? 2 : 4), true)
                    .set(stream));
  }
#endif
  auto kernel = b16 ? (has_bias ? row_post_scale_kernel<true, true> : row_post_scale_kernel<true, false>)
                    : (has_bias ? row_post_scale_kernel<false, true> : row_post_scale_kernel<false, false>);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kPostThreads);
  cfg.stream = stream;
  return cuda_status(cudaLaunchKernelEx(&cfg, kernel, reinterpret_cast<const float4*>(gemm_out), rows, cols / 4,
                                        row_amax, reinterpret_cast<const float4*>(bias), out));
}

nvfp4_status nvfp4_mx_group_cast(const void* x_bf16, int64_t sum_M, int64_t K, const int64_t* m_splits_host,
                                 int32_t num_groups, const nvfp4_mx_outputs* out, cudaStream_t stream) {
  nvfp4_status s = check_shape(x_bf16, sum_M, K, num_groups);
  if (s != NVFP4_OK) return s;
  if (K % kMxBlock != 0) return NVFP4_ERR_INVALID_ARG;
  bool do_row = false, do_col = false;
  s = check_mx_outputs(out, sum_M, K, do_row, do_col);
  if (s != NVFP4_OK) return s;
  static thread_local HostRouting routing;
  s = host_routing(m_splits_host, num_groups, sum_M, routing, kMxBlock);  // a 32-row block lies in one group
  if (s != NVFP4_OK) return s;
  if (!do_row && !do_col) return NVFP4_OK;
  return launch_mx_cast(routing, x_bf16, sum_M, K, num_groups, out, stream);
}

nvfp4_status nvfp4_mx_group_cast_graphsafe(const void* x_bf16, int64_t capacity_rows, int64_t K,
                                           const int64_t* first_dims_dev, const int64_t* tensor_offsets_dev,
                                           int32_t num_groups, const nvfp4_mx_outputs* out, int32_t* status_dev,
                                           cudaStream_t stream) {
  nvfp4_status s = check_shape(x_bf16, capacity_rows, K, num_groups);
  if (s != NVFP4_OK) return s;
  if (K % kMxBlock != 0) return NVFP4_ERR_INVALID_ARG;
  bool do_row = false, do_col = false;
  s = check_mx_outputs(out, capacity_rows, K, do_row, do_col);
  if (s != NVFP4_OK) return s;
  DeviceRouting routing;
  s = device_routing(first_dims_dev, tensor_offsets_dev, status_dev, K, capacity_rows, num_groups, kMxBlock,
                     routing);
  if (s != NVFP4_OK) return s;
  s = cuda_status(cudaMemsetAsync(status_dev, 0, sizeof(int32_t), stream));
  if (s != NVFP4_OK || K == 0 || (!do_row && !do_col)) return s;
  return launch_mx_cast(routing, x_bf16, capacity_rows, K, num_groups, out, stream);
}

nvfp4_status nvfp4_mx_dequantize(const uint8_t* data, const uint8_t* scale, int64_t rows, int64_t cols,
                                 float* out_f32, cudaStream_t stream) {
  if (rows < 0 || cols < 0 || cols % 32 != 0) return NVFP4_ERR_INVALID_ARG;
  if (rows == 0 || cols == 0) return NVFP4_OK;
  if (data == nullptr || scale == nullptr || out_f32 == nullptr) return NVFP4_ERR_INVALID_ARG;
  if (!aligned(data, 16) || !aligned(out_f32, 16)) return NVFP4_ERR_UNSUPPORTED;
  return launch_dequant<true>(data, scale, nullptr, rows, cols, out_f32, stream);
}

const char* nvfp4_status_string(nvfp4_status status) {
  switch (status) {
    case NVFP4_OK: return "NVFP4_OK";
    case NVFP4_ERR_INVALID_ARG: return "NVFP4_ERR_INVALID_ARG";
    case NVFP4_ERR_UNSUPPORTED: return "NVFP4_ERR_UNSUPPORTED";
    case NVFP4_ERR_CUDA: return "NVFP4_ERR_CUDA";
    case NVFP4_ERR_ROUTING: return "NVFP4_ERR_ROUTING";
    case NVFP4_ERR_TIMEOUT: return "NVFP4_ERR_TIMEOUT";
  }
  return "NVFP4_ERR_UNKNOWN";
}

}  // extern "C"

#ifdef NVFP4_TEST_HOOKS
extern "C" NVFP4RS_API void nvfp4_test_set_first_position(uint8_t position) { g_test_first_position = position; }
#endif

#ifdef NVFP4_CHECK_BOUNDS
// The checked debug build only: accesses counted outside their launch's
// registered ranges since load (or the last reset).
extern "C" NVFP4RS_API unsigned long long nvfp4_debug_bounds_faults(void) {
  unsigned long long v = 0;
  if (cudaMemcpyFromSymbol(&v, nvfp4rs::g_bounds_faults, sizeof(v)) != cudaSuccess) return ~0ull;
  return v;
}
extern "C" NVFP4RS_API int nvfp4_debug_bounds_reset(void) {
  const unsigned long long z = 0;
  return cudaMemcpyToSymbol(nvfp4rs::g_bounds_faults, &z, sizeof(z)) == cudaSuccess ? 0 : 1;
}
#endif
