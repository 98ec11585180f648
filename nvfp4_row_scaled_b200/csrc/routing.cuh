// routing.cuh -- the two routing front-ends of the grouped kernels.
//
// TransformerEngine #3649 (grouped row-scaled NVFP4 cast), Description: each
// of the two steps exists twice, once driven by host split sizes and once by
// the grouped tensor's device arrays first_dims / tensor_offsets, so that the
// device-driven pair can be captured in a CUDA graph and replayed after the
// routing changes; both share one device body, which makes their outputs
// byte-identical.
//
// Here a front-end only fills a RoutingSmem (the first row of every group,
// the number of groups, the routed row total and a verdict) in shared memory.
// Everything after that -- which tile belongs to which group, every load,
// every store -- is the same code for both. The host-split front-end copies
// the offsets out of the kernel's parameter block; the device front-end loads
// tensor_offsets / first_dims, checks them, and on a violation records a
// status code instead of trapping.
#pragma once

#include <cstdint>

#include "nvfp4rs.h"
#include "bounds.cuh"

namespace nvfp4rs {

// ---------------------------------------------- programmatic dependent launch
//
// The cast is launched with programmatic stream serialization: its CTAs may
// start while the kernel before it on the stream (normally the grouped amax)
// is still finishing. grid_dependency_wait() blocks until that kernel has
// completed and its writes are visible; a kernel calls it before its first
// read of anything an earlier kernel may write (x, the amax vectors, device
// routing). Without a programmatic launch it returns at once.
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Lets the kernel after this one on the stream (if launched programmatically)
// be scheduled now; its own grid_dependency_wait() still waits for this
// kernel to complete.
__device__ __forceinline__ void launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

constexpr int kRows = 128;     // rows per tile
constexpr int kBlockRows = 16; // group sizes are multiples of it: a 16-row block lies in one group

// Lives in static shared memory; `off` points at E+1 int32 of dynamic shared
// memory (sized by the host from the number of groups).
struct RoutingSmem {
  int32_t* off;  // first row of group g; off[E] = routed total
  int32_t E;
  int32_t total;
  int32_t ok;      // 1 when the routing is usable
  int32_t all128;  // 1 when every group is a multiple of 128 rows
};

// Host split sizes turned into row offsets by the host, passed by value.
struct HostRouting {
  static constexpr bool kOnDevice = false;  // the routing is in the kernel parameters
  int32_t E;
  int32_t total;
  int32_t all128;  // every group a multiple of 128 rows (found by the host)
  int32_t off[NVFP4_MAX_GROUPS + 1];

  __device__ __forceinline__ void load(RoutingSmem& s, int32_t* off_smem) const {
    for (int i = threadIdx.x; i <= E; i += blockDim.x) off_smem[i] = off[i];
    if (threadIdx.x == 0) {
      s.off = off_smem;
      s.E = E;
      s.total = total;
      s.ok = 1;
      s.all128 = all128;
    }
    __syncthreads();
  }
  // host-split calls have no status word: a give-up is not reported
  __device__ __forceinline__ void report(int) const {}
};

// Device routing: first_dims [E] rows per group, tensor_offsets [E+1]
// element offsets (row offset * K). Checked on every load. `status` is where
// a violation -- or a kernel's give-up on a bounded wait -- is recorded.
// With uniform_rows >= 0 the two arrays are absent and every group has
// uniform_rows rows (the host checked E * uniform_rows <= capacity_rows).
// Groups whose size is not a multiple of `align` are NVFP4_ERR_UNSUPPORTED.
struct DeviceRouting {
  static constexpr bool kOnDevice = true;  // the routing is in device memory
  const int64_t* first_dims;
  const int64_t* tensor_offsets;
  int32_t* status;
  int64_t K;
  int64_t capacity_rows;
  int32_t E;
  int32_t align;
  int64_t uniform_rows;

  __device__ __forceinline__ void load(RoutingSmem& s, int32_t* off_smem) const {
    if (uniform_rows >= 0) {
      for (int i = threadIdx.x; i <= E; i += blockDim.x) off_smem[i] = static_cast<int32_t>(i * uniform_rows);
      if (threadIdx.x == 0) {
        s.off = off_smem;
        s.E = E;
        s.ok = 1;
        s.total = static_cast<int32_t>(E * uniform_rows);
        s.all128 = uniform_rows % kRows == 0;
      }
      __syncthreads();
      return;
    }
    int bad_routing = 0, bad_align = 0, not_128 = 0;
    for (int i = threadIdx.x; i <= E; i += blockDim.x) {
      const int64_t o = gload(&tensor_offsets[i]);
      if ((i == 0 && o != 0) || o < 0 || o % K != 0 || o / K > capacity_rows) {
        bad_routing = 1;
      } else {
        off_smem[i] = static_cast<int32_t>(o / K);
      }
      if (i < E) {
        const int64_t fd = gload(&first_dims[i]);
        const int64_t next = gload(&tensor_offsets[i + 1]);
        if (fd < 0 || fd > capacity_rows || next - o != fd * K) bad_routing = 1;
        if (fd % align != 0) bad_align = 1;
        if (fd % kRows != 0) not_128 = 1;
      }
    }
    bad_routing = __syncthreads_or(bad_routing);
    bad_align = __syncthreads_or(bad_align);
    not_128 = __syncthreads_or(not_128);
    if (threadIdx.x == 0) {
      const int code = bad_routing ? NVFP4_ERR_ROUTING : (bad_align ? NVFP4_ERR_UNSUPPORTED : 0);
      s.off = off_smem;
      s.E = E;
      s.ok = code == 0;
      s.all128 = !not_128;
      s.total = code == 0 ? off_smem[E] : 0;
      if (code != 0) gstore(status, static_cast<int32_t>(code));
    }
    __syncthreads();
  }
  __device__ __forceinline__ void report(int code) const {
    if (NVFP4_STORE_OK(status, 4)) atomicCAS(status, 0, code);
  }
};

// Group holding row r (r < total): the last g with off[g] <= r. Empty groups
// share their start with the next group and are skipped by taking the last.
__device__ __forceinline__ int group_of_row(const RoutingSmem& s, int32_t r) {
  int lo = 0, hi = s.E - 1;  // answer in [lo, hi]
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (s.off[mid] <= r)
      lo = mid;
    else
      hi = mid - 1;
  }
  return lo;
}

}  // namespace nvfp4rs
