// bounds.cuh -- device bounds checks of the RKL_DEBUG build.
//
// RKL_BOUNDS(cond) is `true` in the release build.  In the debug build
// (-DRKL_DEBUG) it evaluates cond; when cond fails it records the source line
// in this translation unit's bounds word and returns false, and the caller
// skips the access (a kernel that cannot skip a load raises its abort flag
// and returns through its bounded waits).  Nothing traps: the context stays
// usable and rkl_device_error reports the first failed check's file and line.
//
// Each translation unit that includes this header keeps its own word and
// defines its host reader with RKL_DEFINE_BOUNDS_READER(name).
#pragma once

#include <cuda_runtime.h>

namespace rkl {
namespace {
__device__ int g_bounds_line = 0;  // first failed check's __LINE__ in this file (0: none)
}  // namespace

#ifdef RKL_DEBUG
__device__ __forceinline__ bool bounds_ok(bool cond, int line) {
  if (!cond) atomicCAS(&g_bounds_line, 0, line);
  return cond;
}
#define RKL_BOUNDS(cond) (::rkl::bounds_ok(static_cast<bool>(cond), __LINE__))
constexpr bool kDebugBounds = true;
#else
#define RKL_BOUNDS(cond) true
constexpr bool kDebugBounds = false;
#endif

}  // namespace rkl

// Host reader: *line = the recorded line of this file (0 if none), cleared.
#define RKL_DEFINE_BOUNDS_READER(name)                                          \
  cudaError_t name(int* line) {                                                 \
    int v = 0;                                                                  \
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_bounds_line, sizeof(int));       \
    if (e != cudaSuccess) return e;                                             \
    *line = v;                                                                  \
    if (v != 0) {                                                               \
      const int zero = 0;                                                       \
      e = cudaMemcpyToSymbol(g_bounds_line, &zero, sizeof(int));                \
    }                                                                           \
    return e;                                                                   \
  }
