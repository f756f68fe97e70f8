// Projection buffer W' = [c_w * Omega_h M_h ; c_m * M_h] per head.
//
// DARKformer README, section "Kernel": the feature exponent of token x is
// omega_j^T M x~ - 1/2 x~^T Sigma x~ with x~ = d^{-1/4} x and Sigma = M^T M.
// Folding d^{-1/4} and log2(e) into W' lets every forward kernel obtain the
// base-2 exponent of feature j as (W' x)_j - sum_i (W' x)_{m+i}^2 with a single
// GEMM over the raw tokens.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace dark {

// TW: fp32 for fp32 projections, fp16 for bf16 projections.
template <typename T>
__global__ void projection_kernel(const float* __restrict__ omega, int heads_omega,
                                  const float* __restrict__ geom, int heads_geom, int heads_w,
                                  int m, int r, int d, double cw, double cm, T* __restrict__ w) {
  const int h = blockIdx.y;
  const int row = blockIdx.x;                       // 0 .. m + r - 1
  const float* om = omega + (size_t)(heads_omega == 1 ? 0 : h) * m * r;
  const float* gm = geom + (size_t)(heads_geom == 1 ? 0 : h) * r * d;
  T* dst = w + ((size_t)h * (m + r) + row) * d;
  for (int c = threadIdx.x; c < d; c += blockDim.x) {
    double val;
    if (row < m) {
      double acc = 0.0;
      for (int i = 0; i < r; ++i) acc += (double)om[(size_t)row * r + i] * (double)gm[(size_t)i * d + c];
      val = cw * acc;
    } else {
      val = cm * (double)gm[(size_t)(row - m) * d + c];
    }
    dst[c] = sizeof(T) == 2 ? T(__double2half(val)) : from_f32<T>((float)val);
  }
}

cudaError_t launch_projection(const float* omega, int heads_omega, const float* geom,
                              int heads_geom, int heads_w, int m, int r, int d,
                              dark_dtype dtype, void* w, cudaStream_t stream) {
  const double s = pow((double)d, -0.25);
  const double cw = s * kLog2e;
  const double cm = s * sqrt(0.5 * kLog2e);
  dim3 grid(m + r, heads_w);
  const int threads = d < 256 ? ((d + 31) / 32) * 32 : 256;
  if (dtype == DARK_BF16)
    projection_kernel<__half><<<grid, threads, 0, stream>>>(
        omega, heads_omega, geom, heads_geom, heads_w, m, r, d, cw, cm, (__half*)w);
  else
    projection_kernel<float><<<grid, threads, 0, stream>>>(omega, heads_omega, geom, heads_geom,
                                                           heads_w, m, r, d, cw, cm, (float*)w);
  return cudaGetLastError();
}

}  // namespace dark
