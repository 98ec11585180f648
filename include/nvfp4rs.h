/*
 * nvfp4rs.h -- C ABI of the grouped row-scaled (per-token) NVFP4 cast for
 * NVIDIA B200 (sm_100a). Library: libnvfp4rs.so.
 *
 * The method (web pages it follows):
 *  - TransformerEngine #3649, "single-launch grouped row-scaled NVFP4 cast",
 *    Description: the cast of packed MoE expert activations runs as two
 *    single-launch kernels -- a grouped amax over the packed (sum_M, K) buffer
 *    that yields rowwise [sum_M] and columnwise [num_tensors*K] amax in one
 *    pass, then a grouped cast that consumes both -- and each step has a
 *    graph-safe counterpart that reads the routing from device
 *    first_dims / tensor_offsets instead of host splits, sharing the device
 *    body so that the outputs are byte-identical.
 *  - TransformerEngine #2931, "Implement per-token NVFP4 fprop recipe",
 *    Changes and Important Files Changed: per-token (row) amax as the FP32
 *    second-level scale of NVFP4 (E2M1 data, E4M3 block scales), and a
 *    dequantize that looks up the amax of each element's row.
 *  - TransformerEngine #3324, "Enable NVFP4 row-scaled (per-token) backward
 *    for GroupedLinear", summary: per-column amax for the columnwise
 *    (transposed) operand.
 *
 * Numerics (identical, byte for byte, to the CPU oracle of this project):
 *   S_enc(a) = a == 0 ? 1 : min(fl(2688 / a), FLT_MAX)      2688 = 6 * 448
 *   S_dec(a) = fl(a / 2688)
 *   per 16-element block: s8  = E4M3_rne_satfinite(fl(fl(bmax / 6) * S_enc))
 *                         enc = s8 == 0 ? 0 : min(fl(S_enc / e4m3(s8)), FLT_MAX)
 *                         code_j = E2M1_rne_satfinite(fl(x_j * enc)), sign kept
 *   dequantize: x_hat = fl((e2m1(code) * e4m3(s8)) * S_dec)
 * All float arithmetic is IEEE binary32, round to nearest even, no FMA.
 *
 * Layouts (all row-major, all compact):
 *   x          bf16  [rows, K]
 *   row_amax   fp32  [rows]
 *   col_amax   fp32  [E * K]           group g, column k at g*K + k
 *   row_data   u8    [rows, K/2]       element 2j in the low nibble of byte j
 *   row_scale  u8    [rows, K/16]      one E4M3 byte per 16-element block
 *   row_s2     fp32  [rows]            S_dec of the row amax
 *   col_data   u8    group g at byte offset K*o_g/2, shape [K, m_g/2]
 *                    (the group's transpose; element = row within the group)
 *   col_scale  u8    group g at byte offset K*o_g/16, shape [K, m_g/16]
 *   col_s2     fp32  [E * K]           S_dec of the column amax
 * where o_g = m_0 + ... + m_{g-1} is the first row of group g.
 *
 * Conventions for every call:
 *  - Ownership: the caller allocates and owns every buffer (device memory
 *    unless stated). The library allocates nothing, never synchronises the
 *    stream and never reads device memory from the host. Every call only
 *    enqueues work (memsets and kernels) on `stream`.
 *  - Errors: argument errors are found on the host before anything is
 *    enqueued and returned synchronously; nothing is written then. A failed
 *    CUDA launch returns NVFP4_ERR_CUDA. The graph-safe calls check the device
 *    routing on the device: a violation is written to *status_dev and the
 *    kernels write no output; they never trap and never hang.
 *  - Requirements: K % 16 == 0 (the rowwise block width; else
 *    NVFP4_ERR_INVALID_ARG). Else NVFP4_ERR_UNSUPPORTED: every group size
 *    m_g % 16 == 0 (the colwise block height), num_groups <=
 *    NVFP4_MAX_GROUPS, rows < 2^31, and every pointer 16-byte aligned. The
 *    128x4-tiled scale layout and the graph-safe one-launch call also need
 *    K % 128 == 0 and m_g % 128 == 0 (the 128-row alignment of the grouped
 *    GEMM's scale layout; the host-split one-launch calls run other routings
 *    as two launches); the MXFP4 calls need K % 32 == 0 (else
 *    NVFP4_ERR_INVALID_ARG) and m_g % 32 == 0 (their block size). 128-row tiles inside one group on the
 *    128-row grid, with K % 128 == 0, take the fastest path; the rest is
 *    handled at the tile's edges in the same kernel (a 128-row tile may then
 *    hold rows of several groups, the last row tile may be short, and the
 *    last column tile partial). Inputs must be finite (a non-finite input
 *    gives unspecified codes, never a fault).
 *  - Empty groups (m_g == 0) are allowed: their col_amax and col_s2 are 0
 *    and they own no bytes of col_data / col_scale.
 */
#ifndef NVFP4RS_H
#define NVFP4RS_H

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h> /* cudaStream_t */

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  NVFP4_OK = 0,
  NVFP4_ERR_INVALID_ARG = 1, /* null pointer, negative size, splits that do not add up, K % 16 */
  NVFP4_ERR_UNSUPPORTED = 2, /* valid, but outside the fast path (see above) */
  NVFP4_ERR_CUDA = 3,        /* a CUDA call or launch failed */
  NVFP4_ERR_ROUTING = 4,     /* graph-safe only: device routing is inconsistent */
  NVFP4_ERR_TIMEOUT = 5      /* graph-safe only, device status: a kernel gave up a bounded
                                wait for its own tile loads or, in the one-launch call, for
                                another CTA's amax work (not expected to happen; the
                                affected outputs are incomplete) */
} nvfp4_status;

#define NVFP4_MAX_GROUPS 1024

/* every entry point is exported; everything else in the library is hidden */
#if defined(__GNUC__)
#define NVFP4RS_API __attribute__((visibility("default")))
#else
#define NVFP4RS_API
#endif

/* Layout of the E4M3 block-scale outputs. */
typedef enum {
  NVFP4_SCALE_COMPACT = 0,   /* row-major [rows, cols] as listed above */
  NVFP4_SCALE_TILED_128X4 = 1 /* the 128x4-tiled layout block-scaled GEMMs read: the
                                 matrix [rows, cols] in tiles of 128 rows x 4 columns,
                                 512 bytes each, in row-major tile order; scale (r, c) of
                                 a tile at byte (r % 32) * 16 + (r / 32) * 4 + c. Same
                                 sizes and per-group offsets as compact. Needs every
                                 group to be a multiple of 128 rows and K % 128 == 0
                                 (else NVFP4_ERR_UNSUPPORTED). */
} nvfp4_scale_layout;

/* Output buffers of the grouped cast (device pointers). A direction whose
 * three pointers are all NULL is skipped; a direction with some but not all
 * three set is NVFP4_ERR_INVALID_ARG. */
typedef struct {
  uint8_t* row_data;  /* [rows, K/2]   */
  uint8_t* row_scale; /* [rows, K/16]  */
  float* row_s2;      /* [rows]        */
  uint8_t* col_data;  /* per group [K, m_g/2] at byte K*o_g/2   */
  uint8_t* col_scale; /* per group [K, m_g/16] at byte K*o_g/16 */
  float* col_s2;      /* [E*K]         */
  int32_t scale_layout; /* nvfp4_scale_layout of row_scale and col_scale (0 = compact) */
} nvfp4_outputs;

/*
 * Grouped amax, host-split routing (TransformerEngine #3649, Description:
 * one launch reads the packed bf16 buffer once and yields both the per-row
 * amax and the per-group per-column amax; the per-column amax is the
 * columnwise operand's scale source, as in #3324).
 *   x_bf16         device, bf16 [sum_M, K], read once
 *   sum_M, K       rows and columns; sum_M == sum of m_splits_host
 *   m_splits_host  HOST array [num_groups] of rows per group; read during the
 *                  call only (copied into kernel parameters)
 *   row_amax       device fp32 [sum_M], or NULL to skip rows
 *   col_amax       device fp32 [num_groups*K], or NULL to skip columns; it is
 *                  zeroed on `stream` by this call first
 * Two launches when col_amax is given: a kernel that zeroes col_amax, then the
 * amax kernel, launched programmatically so that its reads of x overlap the
 * zeroing (its atomics on col_amax wait for it); else the amax kernel alone.
 */
NVFP4RS_API nvfp4_status nvfp4_group_amax(const void* x_bf16, int64_t sum_M, int64_t K,
                              const int64_t* m_splits_host, int32_t num_groups,
                              float* row_amax, float* col_amax, cudaStream_t stream);

/*
 * Grouped cast, host-split routing (TransformerEngine #3649, Description:
 * the second launch, which takes both amax vectors as its scale sources;
 * #2931, Changes: per-token NVFP4 quantization). Writes, from one read of each tile of x, the rowwise blocks
 * (16 along K, scaled by the row's amax) and the colwise blocks (16 along the
 * rows of a group, scaled by the group's column amax), plus the FP32 decode
 * scales row_s2 / col_s2.
 *   row_amax, col_amax  device, as written by nvfp4_group_amax (row_amax is
 *                       needed if the row direction is requested, col_amax
 *                       if the column direction is)
 *   out                 HOST pointer to the output descriptor (device buffers)
 * One launch.
 */
NVFP4RS_API nvfp4_status nvfp4_group_cast(const void* x_bf16, int64_t sum_M, int64_t K,
                              const int64_t* m_splits_host, int32_t num_groups,
                              const float* row_amax, const float* col_amax,
                              const nvfp4_outputs* out, cudaStream_t stream);

/*
 * Grouped amax, graph-safe routing (TransformerEngine #3649, Description:
 * the twin of the host-split call whose group boundaries come from device
 * arrays, first_dims and tensor_offsets, rather than from host splits). Nothing about
 * the routing is read on the host, so the call can be captured in a CUDA
 * graph once and replayed after the routing buffers change on the device.
 * The device body is the one nvfp4_group_amax runs, so for equal routing
 * the outputs are byte-identical.
 *   capacity_rows       rows allocated in x (the grid is sized by it); rows at
 *                       or beyond the routed total are neither read nor written
 *   first_dims_dev      device int64 [num_groups]: rows of each group
 *   tensor_offsets_dev  device int64 [num_groups+1]: ELEMENT offset of each
 *                       group (row offset * K); [0] == 0, and
 *                       first_dims[g]*K == offsets[g+1] - offsets[g];
 *                       offsets[num_groups] / K <= capacity_rows
 *   status_dev          device int32 [1]: set to 0 by this call, then to
 *                       NVFP4_ERR_ROUTING (inconsistent routing) or
 *                       NVFP4_ERR_UNSUPPORTED (a group not a multiple of 16
 *                       rows) by the kernel, which then writes no amax
 * Uniform groups: with first_dims_dev and tensor_offsets_dev both NULL every
 * group has capacity_rows / num_groups rows (which must divide exactly, else
 * NVFP4_ERR_INVALID_ARG; a multiple of 16, else NVFP4_ERR_UNSUPPORTED).
 * A memset of status, then the launches of nvfp4_group_amax.
 */
NVFP4RS_API nvfp4_status nvfp4_group_amax_graphsafe(const void* x_bf16, int64_t capacity_rows, int64_t K,
                                        const int64_t* first_dims_dev,
                                        const int64_t* tensor_offsets_dev, int32_t num_groups,
                                        float* row_amax, float* col_amax, int32_t* status_dev,
                                        cudaStream_t stream);

/*
 * Grouped cast, graph-safe routing: nvfp4_group_cast with the routing of
 * nvfp4_group_amax_graphsafe (same arguments, same status rules; status_dev
 * is reset to 0 by this call too). Byte-identical to nvfp4_group_cast for
 * equal routing (the same kernel serves both). One memset of status and one
 * launch, whatever the routing turns out to be on the device.
 */
NVFP4RS_API nvfp4_status nvfp4_group_cast_graphsafe(const void* x_bf16, int64_t capacity_rows, int64_t K,
                                        const int64_t* first_dims_dev,
                                        const int64_t* tensor_offsets_dev, int32_t num_groups,
                                        const float* row_amax, const float* col_amax,
                                        const nvfp4_outputs* out, int32_t* status_dev,
                                        cudaStream_t stream);

/*
 * Bytes of workspace the one-launch calls below need. The graph-safe call
 * needs nvfp4_group_quantize_workspace_bytes(capacity_rows, num_groups); the
 * host-split call needs only nvfp4_group_quantize_workspace_bytes(0,
 * num_groups) (at most 4352 bytes). Returns 0 for a negative size or
 * num_groups > NVFP4_MAX_GROUPS.
 */
NVFP4RS_API size_t nvfp4_group_quantize_workspace_bytes(int64_t capacity_rows, int32_t num_groups);

/*
 * Grouped amax AND grouped cast in ONE launch, host-split routing. Computes
 * exactly what nvfp4_group_amax followed by nvfp4_group_cast computes
 * (TransformerEngine #3649, Description: the amax step's row and column amax
 * vectors are the cast step's scale sources) -- row_amax, col_amax and every
 * output of `out` byte-identical to that pair -- but meant to read each tile
 * of x from DRAM once: a persistent kernel runs the amax of a tile, and the
 * cast of the same tile a little later while it is still in L2, once all
 * amax work of its group has finished. A group too large for L2 between its
 * two passes is read back in part.
 *   x_bf16, sum_M, K, m_splits_host, num_groups, out
 *                   as for nvfp4_group_cast
 *   row_amax        device fp32 [sum_M], written (needed when the row
 *                   direction is requested, else may be NULL)
 *   col_amax        device fp32 [num_groups*K], written (needed when the
 *                   column direction is requested, else may be NULL)
 *   workspace       device, >= nvfp4_group_quantize_workspace_bytes(0,
 *                   num_groups) bytes, 16-byte aligned, owned by the caller;
 *                   zeroed by this call on `stream`, so calls that share a
 *                   workspace must be ordered on one stream. After the call
 *                   word 1 is nonzero only if a bounded wait inside the kernel
 *                   gave up (not expected; the outputs are then incomplete).
 * The single launch takes routings whose groups are all multiples of 128
 * rows with K % 128 == 0. Any other routing the two-step calls accept
 * (groups of multiples of 16 rows, K % 16 == 0) runs here as those two
 * launches -- the same outputs, the workspace left untouched -- except with
 * the 128x4-tiled scale layout, which needs 128-row groups and
 * K % 128 == 0 (else NVFP4_ERR_UNSUPPORTED). With no direction requested
 * nothing is enqueued. Single launch: memsets of the workspace header,
 * row_amax and col_amax, then the kernel.
 */
NVFP4RS_API nvfp4_status nvfp4_group_quantize(const void* x_bf16, int64_t sum_M, int64_t K,
                                  const int64_t* m_splits_host, int32_t num_groups,
                                  float* row_amax, float* col_amax, const nvfp4_outputs* out,
                                  void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * nvfp4_group_quantize with the graph-safe routing of
 * nvfp4_group_amax_graphsafe (same routing arguments and status rules, plus
 * NVFP4_ERR_TIMEOUT if a bounded wait gave up; a group that is not a
 * multiple of 128 rows is NVFP4_ERR_UNSUPPORTED). Byte-identical to the
 * host-split call for equal routing, and to the graph-safe two-launch pair.
 * Rows at or beyond the routed total are neither read nor written; their row
 * amax accumulates in the workspace, which must hold
 * nvfp4_group_quantize_workspace_bytes(capacity_rows, num_groups) bytes.
 * Memsets of status, the workspace and col_amax, then one launch; capturable
 * in a CUDA graph.
 */
NVFP4RS_API nvfp4_status nvfp4_group_quantize_graphsafe(const void* x_bf16, int64_t capacity_rows, int64_t K,
                                            const int64_t* first_dims_dev,
                                            const int64_t* tensor_offsets_dev, int32_t num_groups,
                                            float* row_amax, float* col_amax,
                                            const nvfp4_outputs* out, void* workspace,
                                            size_t workspace_bytes, int32_t* status_dev,
                                            cudaStream_t stream);

/*
 * nvfp4_group_quantize without a workspace argument: the same one-launch
 * kernel, same arguments and outputs (byte-identical), with its scratch in a
 * static device array inside the library; routings the single launch does
 * not take run as the two launches, as in nvfp4_group_quantize. This call has no counterpart in
 * the pages the method follows. It is for callers that cannot hand over
 * device memory at the call site: a C caller with no device allocator of
 * its own, or one that must not allocate there (cudaMalloc synchronises the
 * device). It allocates nothing.
 *   - Limit: the static scratch is 4352 bytes, the workspace header of
 *     NVFP4_MAX_GROUPS groups; larger num_groups is NVFP4_ERR_UNSUPPORTED.
 *   - Setup: the first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current) and caches it; make
 *     that first call before any stream capture. The cached address belongs
 *     to the device's current context: after cudaDeviceReset on a device,
 *     this call must not be used on that device again in the same process.
 *   - Give-up: if a bounded wait inside the kernel gives up (not expected;
 *     it needs a stalled SM elsewhere), the outputs are incomplete and this
 *     call cannot report it -- it has returned before the kernel runs, and
 *     the word that records the give-up is private to the library. Callers
 *     that need that report use nvfp4_group_quantize (workspace word 1) or
 *     nvfp4_group_quantize_graphsafe (status word).
 *   - Zeroing: each call zeroes the scratch (and row_amax, col_amax) on
 *     `stream` before its launch; nothing needs to start at zero.
 *   - Races: every call on a device shares the one scratch array, so calls
 *     whose work overlaps (different streams, or threads) race and give
 *     wrong results. Order them on one stream.
 * row_amax and col_amax must be 16-byte aligned (else NVFP4_ERR_UNSUPPORTED).
 */
NVFP4RS_API nvfp4_status nvfp4_group_quantize_noalloc(const void* x_bf16, int64_t sum_M, int64_t K,
                                          const int64_t* m_splits_host, int32_t num_groups,
                                          float* row_amax, float* col_amax,
                                          const nvfp4_outputs* out, cudaStream_t stream);

/*
 * Dequantize one quantized matrix [rows, cols] to FP32 with one decode scale
 * per row (TransformerEngine #2931, Important Files Changed: the dequantize
 * kernel looks up the amax of the element's row, tensor_amax[y]).
 *   data   device u8 [rows, cols/2], scale device u8 [rows, cols/16],
 *   s2     device fp32 [rows], out device fp32 [rows, cols]
 * Rowwise output: pass row_data/row_scale/row_s2 with rows = sum_M, cols = K.
 * Colwise output of group g: pass its slices with rows = K, cols = m_g and
 * s2 = col_s2 + g*K. Requires cols % 16 == 0 (else NVFP4_ERR_INVALID_ARG),
 * an 8-byte aligned data pointer and a 16-byte aligned out pointer (else
 * NVFP4_ERR_UNSUPPORTED). One launch.
 */
NVFP4RS_API nvfp4_status nvfp4_dequantize(const uint8_t* data, const uint8_t* scale, const float* s2,
                              int64_t rows, int64_t cols, float* out_f32, cudaStream_t stream);

/* ------------------------------------------------------------------ MXFP4
 * MXFP4: E2M1 data, blocks of 32 elements, one E8M0 (power-of-two) scale per
 * block, no second-level scale (TransformerEngine #3824, Testing and item 1:
 * the "E2M1/block-32/E8M0" pow_2_scales configuration, which row-scaled
 * NVFP4 is not combined with). Scale rule (OCP Microscaling conversion; the
 * pages do not spell it out): with a = max |x| of the block,
 *   s = clamp(floor(log2 a) - 2, -127, 127)   (a == 0 gives -127)
 *   scale byte = s + 127;  code_j = E2M1_rne_satfinite(x_j * 2^-s), sign kept
 *   dequantize: x_hat = e2m1(code) * 2^(scale - 127)
 * Same grouped structure and kernel organisation as the NVFP4 cast; groups
 * must be multiples of 32 rows (else NVFP4_ERR_UNSUPPORTED) and K a multiple
 * of 32 (else NVFP4_ERR_INVALID_ARG). One read of x, one launch: no amax step. */
typedef struct {
  uint8_t* row_data;  /* [rows, K/2]                               */
  uint8_t* row_scale; /* [rows, K/32] E8M0                         */
  uint8_t* col_data;  /* per group [K, m_g/2] at byte K*o_g/2      */
  uint8_t* col_scale; /* per group [K, m_g/32] at byte K*o_g/32    */
} nvfp4_mx_outputs;

/* Grouped MXFP4 cast, host-split routing (arguments as nvfp4_group_cast). */
NVFP4RS_API nvfp4_status nvfp4_mx_group_cast(const void* x_bf16, int64_t sum_M, int64_t K,
                                 const int64_t* m_splits_host, int32_t num_groups,
                                 const nvfp4_mx_outputs* out, cudaStream_t stream);

/* Grouped MXFP4 cast, graph-safe routing (arguments and status as
 * nvfp4_group_cast_graphsafe; a group that is not a multiple of 32 rows is
 * NVFP4_ERR_UNSUPPORTED on the device). Byte-identical to the host-split call;
 * one launch whatever the device routing holds. */
NVFP4RS_API nvfp4_status nvfp4_mx_group_cast_graphsafe(const void* x_bf16, int64_t capacity_rows, int64_t K,
                                           const int64_t* first_dims_dev,
                                           const int64_t* tensor_offsets_dev, int32_t num_groups,
                                           const nvfp4_mx_outputs* out, int32_t* status_dev,
                                           cudaStream_t stream);

/* Decode one MXFP4 matrix [rows, cols]: data [rows, cols/2], scale
 * [rows, cols/32] -> out fp32 [rows, cols]. cols % 32 == 0 (else
 * NVFP4_ERR_INVALID_ARG); data and out 16-byte aligned (else
 * NVFP4_ERR_UNSUPPORTED). Colwise output of group g: rows = K, cols = m_g. */
NVFP4RS_API nvfp4_status nvfp4_mx_dequantize(const uint8_t* data, const uint8_t* scale, int64_t rows,
                                 int64_t cols, float* out_f32, cudaStream_t stream);

/* Output type of nvfp4_row_post_scale. */
typedef enum { NVFP4_OUT_F32 = 0, NVFP4_OUT_BF16 = 1 } nvfp4_out_dtype;

/*
 * Per-row FP32 scaling of a GEMM output (TransformerEngine #2931, sequence
 * diagram: the GEMM runs with the row-scaled operand's amax replaced by
 * ones, then its output rows are multiplied by the row-wise amax and
 * converted to the target dtype; gemm.py in Important Files Changed: the
 * bias is taken out before and added back after). For every element
 *   y = fl(gemm_out[r][c] * row_amax[r]);  with a bias y = fl(y + bias[c]);
 *   out[r][c] = y as f32, or as bf16 (round to nearest even).
 *   gemm_out   device fp32 [rows, cols], row-major
 *   row_amax   device fp32 [rows] (the row amax of the row-scaled operand,
 *              e.g. row_amax of the grouped amax for packed expert rows)
 *   bias       device fp32 [cols], or NULL
 *   out        device [rows, cols] of out_dtype; may be gemm_out itself
 *              for NVFP4_OUT_F32 (in place)
 * Requires cols % 4 == 0, gemm_out and bias 16-byte aligned, out 16-byte
 * (f32) or 8-byte (bf16) aligned (else NVFP4_ERR_UNSUPPORTED). One launch.
 */
NVFP4RS_API nvfp4_status nvfp4_row_post_scale(const float* gemm_out, int64_t rows, int64_t cols,
                                  const float* row_amax, const float* bias, void* out,
                                  int32_t out_dtype, cudaStream_t stream);

/* Human-readable name of a status code (static storage, never NULL). */
NVFP4RS_API const char* nvfp4_status_string(nvfp4_status status);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4RS_H */
