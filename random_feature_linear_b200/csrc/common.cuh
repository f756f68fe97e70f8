// Device helpers shared by the kernels of the DARKformer PRF attention library.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "../../include/dark.h"

namespace dark {

// log2(e) and the base-2 constants of the projection buffer: the feature
// exponent omega^T M x~ becomes (w x) * log2(e) when w carries c_w, and the
// squared norm 1/2 |M x~|^2 becomes sum (w x)^2 when w carries c_m.
constexpr double kLog2e = 1.4426950408889634073599246810019;

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ float to_f32(__half x) { return __half2float(x); }

// Element type of the projection buffer W' for token type T: fp32 tokens use an
// fp32 W'; bf16 tokens use an fp16 W' (11 significant bits for the exponents).
template <typename T> struct WeightOf { using type = float; };
template <> struct WeightOf<__nv_bfloat16> { using type = __half; };

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}
template <> __device__ __forceinline__ __half from_f32<__half>(float x) { return __float2half_rn(x); }

// Records the first device-side error of a call; later errors are dropped.
__device__ __forceinline__ void report(int* dev_status, int code) {
  if (dev_status != nullptr) atomicCAS(dev_status, 0, code);
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

// Orders floats as signed ints so that atomicMax on the encoding is a float max.
__device__ __forceinline__ int float_to_ordered(float f) {
  int i = __float_as_int(f);
  return i >= 0 ? i : i ^ 0x7fffffff;
}
__device__ __forceinline__ float ordered_to_float(int i) {
  return __int_as_float(i >= 0 ? i : i ^ 0x7fffffff);
}

}  // namespace dark
