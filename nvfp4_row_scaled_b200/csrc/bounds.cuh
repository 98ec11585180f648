// bounds.cuh -- address checks of the bounds-checked debug build.
//
// Built with -DNVFP4_CHECK_BOUNDS (libnvfp4rs_debug.so), every global store,
// atomic and explicit global load of the kernels first checks that its bytes
// lie inside one of the ranges the host registered for the launch: the
// call's outputs for stores and atomics, its inputs (and outputs) for loads.
// An access outside them is counted in a device counter and skipped (a load
// returns zeros), so a wrong index shows up as a nonzero count in the tests
// instead of as a fault. A bulk copy outside them is counted and redirected to
// the first input range, so that its mbarrier still gets its bytes. TMA tile
// loads need no check: the tensor map bounds them in hardware.
//
// The host registers a launch's ranges with a one-thread kernel on the
// launch's stream just before the launch (stream-ordered and capturable in a
// CUDA graph), so calls of the debug build must not run concurrently on
// different streams. Without NVFP4_CHECK_BOUNDS every check is the constant
// true and compiles away.
#pragma once

#include <cstdint>

namespace nvfp4rs {

#ifdef NVFP4_CHECK_BOUNDS

constexpr int kMaxSpans = 16;  // the most any launch registers is 14

struct Spans {
  uint64_t lo[kMaxSpans];
  uint64_t hi[kMaxSpans];  // one past the last byte
  uint32_t store[kMaxSpans];  // nonzero: stores and atomics may go here
  int32_t n;
};

__device__ Spans g_spans;
__device__ unsigned long long g_bounds_faults;

__global__ void set_spans_kernel(const Spans s) { g_spans = s; }

__device__ __forceinline__ bool span_ok(const void* p, uint32_t bytes, bool store) {
  const uint64_t a = reinterpret_cast<uint64_t>(p);
  for (int i = 0; i < g_spans.n; i++)
    if (a >= g_spans.lo[i] && a + bytes <= g_spans.hi[i] && (!store || g_spans.store[i])) return true;
  atomicAdd(&g_bounds_faults, 1ull);
  return false;
}

// a bulk copy source outside the inputs: counted, then read from the first
// input range instead (16-byte aligned, at least `bytes` long)
__device__ __forceinline__ const void* bulk_src(const void* p, uint32_t bytes) {
  return span_ok(p, bytes, false) ? p : reinterpret_cast<const void*>(g_spans.lo[0]);
}

#define NVFP4_STORE_OK(p, bytes) ::nvfp4rs::span_ok((p), (bytes), true)
#define NVFP4_LOAD_OK(p, bytes) ::nvfp4rs::span_ok((p), (bytes), false)
#define NVFP4_BULK_SRC(p, bytes) ::nvfp4rs::bulk_src((p), (bytes))

#else

#define NVFP4_STORE_OK(p, bytes) true
#define NVFP4_LOAD_OK(p, bytes) true
#define NVFP4_BULK_SRC(p, bytes) (p)

#endif

// Plain global store and load through the checks.
template <class T>
__device__ __forceinline__ void gstore(T* p, T v) {
  if (NVFP4_STORE_OK(p, sizeof(T))) *p = v;
}

template <class T>
__device__ __forceinline__ T gload(const T* p) {
  return NVFP4_LOAD_OK(p, sizeof(T)) ? *p : T{};
}

}  // namespace nvfp4rs
