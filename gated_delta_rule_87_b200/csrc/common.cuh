// Shared device helpers for the gated delta-rule kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gated_delta.h"

namespace gdr {

// q/k/v/o element access for the two io dtypes.
template <typename T> struct io;
template <> struct io<float> {
  static __device__ __forceinline__ float load(const float *p) { return __ldg(p); }
  static __device__ __forceinline__ void store(float *p, float x) { *p = x; }
};
template <> struct io<__nv_bfloat16> {
  static __device__ __forceinline__ float load(const __nv_bfloat16 *p) {
    return __bfloat162float(__ldg(p));
  }
  static __device__ __forceinline__ void store(__nv_bfloat16 *p, float x) {
    *p = __float2bfloat16_rn(x);
  }
};

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);  // .x = lo (low half)
  return *reinterpret_cast<uint32_t *>(&h);
}

__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

// ---- bounds-checked build (compiled with -DGDR_BOUNDS_CHECK) ----
// Every index a kernel computes for a global-memory access of its own (not
// the tensor-map copies, which the TMA unit bounds itself) is checked against
// the extent of the buffer it addresses.  A failed check counts one violation
// in this translation unit's counter and the access is skipped: nothing traps
// and nothing leaves the buffer.  kda_bounds_violations() reads the counters.
// In the normal build the checks compile away.
#ifdef GDR_BOUNDS_CHECK
static __device__ unsigned int g_oob_violations;
__device__ __forceinline__ bool oob_ok(bool ok) {
  if (!ok) atomicAdd(&g_oob_violations, 1u);
  return ok;
}
#define GDR_IN_BOUNDS(cond) (::gdr::oob_ok(cond))
// host reader of this translation unit's counter (reset after reading)
#define GDR_DEFINE_OOB_COUNTER(fn)                                               \
  unsigned int fn() {                                                            \
    unsigned int v = 0, z = 0;                                                   \
    if (cudaMemcpyFromSymbol(&v, g_oob_violations, sizeof(v)) != cudaSuccess) v = ~0u; \
    cudaMemcpyToSymbol(g_oob_violations, &z, sizeof(z));                         \
    return v;                                                                    \
  }
#else
#define GDR_IN_BOUNDS(cond) true
#define GDR_DEFINE_OOB_COUNTER(fn) \
  unsigned int fn() { return 0; }
#endif

}  // namespace gdr
