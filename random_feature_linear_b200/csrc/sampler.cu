// Projection sampler: Omega [heads][m][r] drawn on the device from a counter-based
// generator, as independent Gaussian features or as orthogonal Gaussian blocks,
// and the host-side redraw schedule of a projection.
//
// DARKformer README, section "Kernel": omega_j ~ N(0, I_r); section
// "Self-attention": orthogonal Gaussian blocks by default, independent features
// with orthogonal_features=False; section "Projection lifecycle": a projection is
// kept until it is redrawn, a redraw interval makes one fall due after that many
// training forwards (forwards outside training are not counted), a fixed
// projection refuses redraws unless one is forced, and a seed reproduces them.
//
// Generator: Philox4x64-10 (Salmon, Moraes, Dror, Shaw, "Parallel random numbers:
// as easy as 1, 2, 3", SC 2011), key (seed, draw), counter (block, head, purpose,
// 0); each block's four words give two Box-Muller pairs (u1 = 1 - u(x_a),
// u2 = u(x_b), u(x) = (x >> 11) 2^-53), so stream element e is word e % 4 of block
// e / 4. Purpose 0 holds the features (or the block matrices G), purpose 1 the
// vectors whose norms scale the orthogonal rows.
// Orthogonal block b of head h: G[i][k] = z(h, 0, b r^2 + i r + k); G = Q R with
// diag(R) > 0 by Gram-Schmidt with one re-orthogonalisation pass in fp64; row i of
// the block is ||(z(h, 1, b r^2 + i r + k))_k|| * Q[:, i]; a partial last block
// keeps its first rows.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace dark {
namespace {

// Philox4x64 multipliers and Weyl key increments (the published constants).
constexpr uint64_t kPhiloxM0 = 0xD2E7470EE14C6C93ull, kPhiloxM1 = 0xCA5A826395121157ull;
constexpr uint64_t kPhiloxW0 = 0x9E3779B97F4A7C15ull, kPhiloxW1 = 0xBB67AE8584CAA73Bull;

__device__ __forceinline__ void philox4x64_10(uint64_t (&c)[4], uint64_t k0, uint64_t k1) {
#pragma unroll
  for (int round = 0; round < 10; ++round) {
    const uint64_t hi0 = __umul64hi(kPhiloxM0, c[0]), lo0 = kPhiloxM0 * c[0];
    const uint64_t hi1 = __umul64hi(kPhiloxM1, c[2]), lo1 = kPhiloxM1 * c[2];
    const uint64_t n0 = hi1 ^ c[1] ^ k0, n2 = hi0 ^ c[3] ^ k1;
    c[0] = n0;
    c[1] = lo1;
    c[2] = n2;
    c[3] = lo0;
    k0 += kPhiloxW0;
    k1 += kPhiloxW1;
  }
}

// The four Gaussians of stream block `blk` of (seed, draw, head, purpose).
__device__ void gauss4(uint64_t seed, uint64_t draw, int head, int purpose, uint64_t blk,
                       double (&z)[4]) {
  uint64_t c[4] = {blk, (uint64_t)head, (uint64_t)purpose, 0ull};
  philox4x64_10(c, seed, draw);
#pragma unroll
  for (int p = 0; p < 2; ++p) {
    const double u1 = 1.0 - (double)(c[2 * p] >> 11) * 0x1p-53;
    const double u2 = (double)(c[2 * p + 1] >> 11) * 0x1p-53;
    const double rho = sqrt(-2.0 * log(u1));
    double sn, cs;
    sincospi(2.0 * u2, &sn, &cs);
    z[2 * p] = rho * cs;
    z[2 * p + 1] = rho * sn;
  }
}

__device__ double gauss1(uint64_t seed, uint64_t draw, int head, int purpose, uint64_t e) {
  double z[4];
  gauss4(seed, draw, head, purpose, e >> 2, z);
  return z[e & 3];
}

// Independent features: Omega_h[j][i] = z(h, 0, j r + i), four per thread.
__global__ void iid_kernel(uint64_t seed, uint64_t draw, int m, int r, float* __restrict__ omega) {
  const int h = blockIdx.y;
  const uint64_t n = (uint64_t)m * r;
  const uint64_t blk = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (blk * 4 >= n) return;
  double z[4];
  gauss4(seed, draw, h, 0, blk, z);
  float* dst = omega + (size_t)h * n;
#pragma unroll
  for (int w = 0; w < 4; ++w)
    if (blk * 4 + w < n) dst[blk * 4 + w] = (float)z[w];
}

// Orthogonal blocks, step 1: G of every block, stored by columns (gc[j][i] =
// G[i][j]), and the norm of each row's scaling vector.
__global__ void orth_draw_kernel(uint64_t seed, uint64_t draw, int nblk, int r,
                                 double* __restrict__ gc, double* __restrict__ norms) {
  const int h = blockIdx.y;
  const uint64_t rr = (uint64_t)r * r;
  const uint64_t per_head = (uint64_t)nblk * rr;
  const uint64_t blk = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (blk * 4 < per_head) {
    double z[4];
    gauss4(seed, draw, h, 0, blk, z);
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const uint64_t e = blk * 4 + w;
      if (e >= per_head) break;
      const uint64_t b = e / rr, rem = e % rr, i = rem / r, k = rem % r;
      gc[((size_t)h * nblk + b) * rr + k * r + i] = z[w];
    }
  }
  // one thread per row of every block: the norm of its purpose-1 vector
  const uint64_t row = blk;
  if (row < (uint64_t)nblk * r) {
    double s = 0.0;
    for (int k = 0; k < r; ++k) {
      const double v = gauss1(seed, draw, h, 1, row * r + k);
      s = fma(v, v, s);
    }
    norms[(size_t)h * nblk * r + row] = sqrt(s);
  }
}

// Step 2: Q of one block (one CTA of 1024 threads), fp64, columns of Q stored
// like G (qc[j][i] = Q[i][j]), by block classical Gram-Schmidt: the columns in
// panels of kPanel, each panel held in shared memory. A panel is first cleared
// of the earlier columns twice (H = Q_prev^T V, V -= Q_prev H: the
// re-orthogonalisation pass of Gram-Schmidt, in blocks), then its columns are
// orthonormalised among themselves by classical Gram-Schmidt with a second pass.
// diag(R) > 0 as in the column-by-column form, so Q is the same up to rounding.
constexpr int kQrThreads = 1024;
constexpr int kPanel = 32;
constexpr size_t kQrSmem = sizeof(double) * (kPanel * 256 + 256 * kPanel + 256 + 32);
__global__ void __launch_bounds__(kQrThreads) orth_qr_kernel(const double* __restrict__ gc, int r,
                                                             double* __restrict__ qc) {
  extern __shared__ double qsm[];
  double* vs = qsm;                        // [kPanel][r] the panel, column-major
  double* hs = vs + kPanel * 256;          // [256][kPanel] projections on the earlier columns
  double* hj = hs + 256 * kPanel;          // [256] projections inside the panel
  double* red = hj + 256;                  // [32]
  const size_t off = (size_t)blockIdx.x * r * r;
  const double* g = gc + off;
  double* q = qc + off;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int i = tid & 255, cg = tid >> 8;  // update: row i, columns 8 cg .. 8 cg + 7
  for (int c0 = 0; c0 < r; c0 += kPanel) {
    const int pc = r - c0 < kPanel ? r - c0 : kPanel;
    for (int e = tid; e < pc * r; e += kQrThreads) vs[e] = g[(size_t)c0 * r + e];
    __syncthreads();
    for (int pass = 0; pass < 2 && c0 > 0; ++pass) {
      // hs[k][c] = Q[:, k] . V[:, c] for the c0 earlier columns k
      for (int k = warp; k < c0; k += kQrThreads / 32) {
        double qk[8];
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          const int ii = lane + 32 * t;
          qk[t] = ii < r ? q[(size_t)k * r + ii] : 0.0;
        }
        for (int c = 0; c < pc; ++c) {
          double s = 0.0;
#pragma unroll
          for (int t = 0; t < 8; ++t) {
            const int ii = lane + 32 * t;
            if (ii < r) s = fma(qk[t], vs[c * r + ii], s);
          }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
          if (lane == 0) hs[k * kPanel + c] = s;
        }
      }
      __syncthreads();
      // V[:, c] -= sum_k Q[:, k] hs[k][c]
      if (i < r) {
        double acc[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) acc[u] = 0.0;
        for (int k = 0; k < c0; ++k) {
          const double qik = q[(size_t)k * r + i];
#pragma unroll
          for (int u = 0; u < 8; ++u) acc[u] = fma(qik, hs[k * kPanel + 8 * cg + u], acc[u]);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u)
          if (8 * cg + u < pc) vs[(8 * cg + u) * r + i] -= acc[u];
      }
      __syncthreads();
    }
    // the panel's columns among themselves: Gram-Schmidt with a second pass
    for (int j = 0; j < pc; ++j) {
      for (int pass = 0; pass < 2 && j > 0; ++pass) {
        if (warp < j) {                    // hj[k] = V[:, k] . V[:, j], k < j
          double s = 0.0;
          for (int ii = lane; ii < r; ii += 32) s = fma(vs[warp * r + ii], vs[j * r + ii], s);
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
          if (lane == 0) hj[warp] = s;
        }
        __syncthreads();
        if (tid < r) {
          double v = vs[j * r + tid];
          for (int k = 0; k < j; ++k) v = fma(-vs[k * r + tid], hj[k], v);
          vs[j * r + tid] = v;
        }
        __syncthreads();
      }
      if (warp < 8) {
        const double v = tid < r ? vs[j * r + tid] : 0.0;
        double s = v * v;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (lane == 0) red[warp] = s;
      }
      __syncthreads();
      double nrm = 0.0;
#pragma unroll
      for (int w = 0; w < 8; ++w) nrm += red[w];
      nrm = sqrt(nrm);
      if (tid < r) vs[j * r + tid] = nrm > 0.0 ? vs[j * r + tid] / nrm : 0.0;
      __syncthreads();
    }
    for (int e = tid; e < pc * r; e += kQrThreads) q[(size_t)c0 * r + e] = vs[e];
    __syncthreads();                       // the panel is in Q before the next panel reads it
  }
}

// Step 3: Omega_h[b r + i][k] = norm_i * Q[k][i] for the first m rows.
__global__ void orth_write_kernel(const double* __restrict__ qc, const double* __restrict__ norms,
                                  int nblk, int m, int r, float* __restrict__ omega) {
  const int h = blockIdx.y;
  const uint64_t n = (uint64_t)m * r;
  const uint64_t e = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= n) return;
  const uint64_t row = e / r, k = e % r, b = row / r, i = row % r;
  const size_t base = ((size_t)h * nblk + b) * r * r;
  omega[(size_t)h * n + e] = (float)(norms[(size_t)h * nblk * r + row] * qc[base + i * r + k]);
}

struct OrthLayout {
  size_t off_g, off_q, off_n, total;
};

OrthLayout orth_layout(int heads, int m, int r) {
  const size_t nblk = (m + r - 1) / r;
  OrthLayout s;
  s.off_g = 0;
  s.off_q = align_up(sizeof(double) * heads * nblk * r * r, 256);
  s.off_n = s.off_q + align_up(sizeof(double) * heads * nblk * r * r, 256);
  s.total = s.off_n + align_up(sizeof(double) * heads * nblk * r, 256);
  return s;
}

}  // namespace

size_t omega_workspace_bytes(int heads, int m, int r, int orthogonal) {
  return orthogonal ? orth_layout(heads, m, r).total : 0;
}

cudaError_t launch_sample_omega(uint64_t seed, uint64_t draw, int heads, int m, int r,
                                int orthogonal, float* omega, void* ws, cudaStream_t stream) {
  if (!orthogonal) {
    const uint64_t blocks4 = ((uint64_t)m * r + 3) / 4;
    iid_kernel<<<dim3((unsigned)((blocks4 + 255) / 256), heads), 256, 0, stream>>>(seed, draw, m, r,
                                                                                    omega);
    return cudaGetLastError();
  }
  const OrthLayout s = orth_layout(heads, m, r);
  const int nblk = (m + r - 1) / r;
  double* gc = (double*)((char*)ws + s.off_g);
  double* qc = (double*)((char*)ws + s.off_q);
  double* norms = (double*)((char*)ws + s.off_n);
  const uint64_t per_head4 = ((uint64_t)nblk * r * r + 3) / 4;
  const uint64_t work = per_head4 > (uint64_t)nblk * r ? per_head4 : (uint64_t)nblk * r;
  orth_draw_kernel<<<dim3((unsigned)((work + 255) / 256), heads), 256, 0, stream>>>(
      seed, draw, nblk, r, gc, norms);
  static int smem_set[64];
  cudaError_t e = set_smem_limit_once((const void*)orth_qr_kernel, (int)kQrSmem, smem_set);
  if (e != cudaSuccess) return e;
  orth_qr_kernel<<<heads * nblk, kQrThreads, kQrSmem, stream>>>(gc, r, qc);
  const uint64_t n = (uint64_t)m * r;
  orth_write_kernel<<<dim3((unsigned)((n + 255) / 256), heads), 256, 0, stream>>>(qc, norms, nblk,
                                                                                   m, r, omega);
  return cudaGetLastError();
}

}  // namespace dark
