// common.cuh — small device helpers shared by the gbs kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gbs.h"

#define GBS_LOG2E 1.4426950408889634f
#define GBS_LN2 0.6931471805599453f

namespace gbs {

// Device error word, the first word of every workspace. 0 = fine.
struct DevErr {
  unsigned int* word;
};

__device__ __forceinline__ void set_error(unsigned int* word, unsigned int code) {
  if (word) atomicCAS(word, 0u, code);
}

// Device-side index checks of the debug build (compiled with -DGBS_DEBUG; the
// library's stand-in for a memory checker). A value read from an index list
// (a Top-K list, a count, a per-CTA plan) that lies outside [lo, hi] is
// recorded as GBS_ERR_DEVICE_CHECK in the error word and replaced by lo, so the
// access it would drive stays in bounds. Release builds compile it away.
__device__ __forceinline__ int dcheck(int v, int lo, int hi, unsigned int* word) {
#ifdef GBS_DEBUG
  if (v < lo || v > hi) {
    set_error(word, GBS_ERR_DEVICE_CHECK);
    return lo;
  }
#endif
  (void)lo;
  (void)hi;
  (void)word;
  return v;
}

template <typename T> __device__ __forceinline__ float to_f32(T x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Order-preserving map float -> uint32 (larger float -> larger key), with -0.0
// folded onto +0.0 so that the two compare equal.
__device__ __forceinline__ uint32_t ordered_key(float f) {
  uint32_t b = __float_as_uint(f);
  if (b == 0x80000000u) b = 0u;
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

}  // namespace gbs
