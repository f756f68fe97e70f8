// SIMT fp32 tile-GEMM building blocks shared by the backward and exact-attention
// kernels (256 threads, 64 x 64 output tiles).
#pragma once

#include <cuda_runtime.h>

namespace dark {

// Tile GEMM building blocks. Operand tiles are staged k-major in shared memory,
// [32 k][kLd] for 64 rows or columns (the 4 extra floats keep every row 16-byte
// aligned), so one k step reads one float4 of A and one of B for 16 FMAs.
// Thread (ty, tx) = (threadIdx / 16, threadIdx % 16) owns output rows ty*4..+3
// and columns tx*4..+3 of a 64 x 64 tile.
constexpr int kLd = 68;

__device__ __forceinline__ float4 ld4(const float* p) {
  return *reinterpret_cast<const float4*>(p);
}

// acc[i][j] += sum_kk A[kk][ty*4+i] B[kk][tx*4+j], kk < 32 (A, B k-major, stride kLd).
__device__ __forceinline__ void fma_tile(const float* A, const float* B, float (&acc)[4][4]) {
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
#pragma unroll 8
  for (int kk = 0; kk < 32; ++kk) {
    const float4 a4 = ld4(A + kk * kLd + ty * 4), b4 = ld4(B + kk * kLd + tx * 4);
    const float a[4] = {a4.x, a4.y, a4.z, a4.w}, b[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
  }
}

// Stages dst[kk][row] = get(row, kk) for 64 rows x 32 k from a source whose
// rows are contiguous in k (consecutive threads read consecutive k).
template <class Get>
__device__ __forceinline__ void stage_t(float* dst, Get get) {
  for (int e = threadIdx.x; e < 64 * 32; e += blockDim.x) {
    const int row = e >> 5, kk = e & 31;
    dst[kk * kLd + row] = get(row, kk);
  }
}

// Stages dst[kk][col] = get(kk, col) for 32 k x 64 columns from a source whose
// rows are contiguous in the column index.
template <class Get>
__device__ __forceinline__ void stage_n(float* dst, Get get) {
  for (int e = threadIdx.x; e < 32 * 64; e += blockDim.x) {
    const int kk = e >> 6, col = e & 63;
    dst[kk * kLd + col] = get(kk, col);
  }
}

__device__ __forceinline__ void zero(float (&acc)[4][4]) {
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
}

}  // namespace dark
