// Generic SIMT forward pass of PRF attention (self-attention, and cross-attention
// of Lq queries over Lk context keys).
//
// This is the fp32-I/O path (fp32 FFMA throughout, so no TF32 rounding enters
// the exponent) and the path for any size, stride or alignment that the
// tensor-core kernels do not cover. It materialises the feature maps in the
// workspace and runs four small kernels:
//   1. features:    Phi(K) (with the key norm, the m^{-1/2} factor and the key
//                   mask) and Psi(Q) = exp2 of the query exponents (the per-query
//                   factors exp(-1/2 |M q~|^2) / sqrt(m) cancel in the ratio);
//   2. chunk_state: per chunk of keys, Phi(K_c)^T [V_c | 1];
//   3. scan:        causal: exclusive prefix over chunks; non-causal: total;
//   4. out:         Psi(Q) S_prefix (+ causal intra-chunk masked Psi(Q) Phi(K)^T [V | 1]),
//                   then num / den.
// DARKformer README, section "Kernel" (feature map, associative ratio) and
// section "Self-attention" (mask, causal constraint).
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace dark {
namespace {

constexpr int kTF = 8;          // tokens per features block (one warp per token)
constexpr int kCausalChunk = 256;
constexpr int kSms = 148;

struct SimtLayout {
  int nc, chunk_len;
  size_t off_ck, off_phiq, off_phik, off_s, total;
};

// Lq queries attend over Lk keys (Lq = Lk for self-attention; causal only then).
SimtLayout simt_layout(int B, int H, int Lq, int Lk, int m, int d, int flags) {
  SimtLayout s;
  const int bh = B * H;
  if (flags & DARK_CAUSAL) {
    s.chunk_len = kCausalChunk;
    s.nc = (Lk + kCausalChunk - 1) / kCausalChunk;
  } else {
    int ns = (2 * kSms + bh - 1) / bh;
    const int max_ns = (Lk + 63) / 64;
    if (ns > max_ns) ns = max_ns;
    if (ns < 1) ns = 1;
    s.chunk_len = (Lk + ns - 1) / ns;
    s.nc = (Lk + s.chunk_len - 1) / s.chunk_len;
  }
  s.off_ck = kWsHeader;
  s.off_phiq = align_up(s.off_ck + sizeof(int) * (size_t)bh, 256);
  s.off_phik = align_up(s.off_phiq + sizeof(float) * (size_t)bh * Lq * m, 256);
  s.off_s = align_up(s.off_phik + sizeof(float) * (size_t)bh * Lk * m, 256);
  s.total = align_up(s.off_s + sizeof(float) * (size_t)bh * s.nc * m * (d + 1), 256);
  return s;
}

__global__ void init_ck_kernel(int* ck, int n) {
  int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) ck[i] = float_to_ordered(-INFINITY);
}

template <typename T>
__global__ void __launch_bounds__(256) features_kernel(
    const T* __restrict__ xq, int64_t qb, int64_t qh, int64_t ql, int Lq,
    const T* __restrict__ xk, int64_t kb, int64_t kh, int64_t kl, int Lk,
    const typename WeightOf<T>::type* __restrict__ w, int heads_w, int m, int r, int d, int H,
    const uint8_t* __restrict__ mask, int stabilise, float* __restrict__ phiq,
    float* __restrict__ phik, int* __restrict__ ck) {
  extern __shared__ float sm[];
  float* xs = sm;                    // [kTF][d]
  float* P = sm + kTF * d;           // [kTF][m + r]
  __shared__ float cst[kTF];
  const int side = blockIdx.z;       // 0: queries, 1: keys
  const int bh = blockIdx.y, b = bh / H, h = bh % H;
  const int t0 = blockIdx.x * kTF;
  const int L = side ? Lk : Lq;
  if (t0 >= L) return;               // the grid covers the longer side
  const T* x = side ? xk : xq;
  const int64_t sb = side ? kb : qb, sh = side ? kh : qh, sl = side ? kl : ql;
  const int ncols = side ? m + r : m;
  const int ld = m + r;
  const auto* wh = w + (size_t)(heads_w == 1 ? 0 : h) * (m + r) * d;

  for (int e = threadIdx.x; e < kTF * d; e += blockDim.x) {
    const int tt = e / d, c = e % d, t = t0 + tt;
    xs[e] = t < L ? to_f32(x[(int64_t)b * sb + (int64_t)h * sh + (int64_t)t * sl + c]) : 0.f;
  }
  __syncthreads();
  for (int j = threadIdx.x; j < ncols; j += blockDim.x) {
    float acc[kTF];
#pragma unroll
    for (int tt = 0; tt < kTF; ++tt) acc[tt] = 0.f;
    const auto* wr = wh + (size_t)j * d;
    for (int c = 0; c < d; ++c) {
      const float wv = to_f32(wr[c]);
#pragma unroll
      for (int tt = 0; tt < kTF; ++tt) acc[tt] = fmaf(wv, xs[tt * d + c], acc[tt]);
    }
#pragma unroll
    for (int tt = 0; tt < kTF; ++tt) P[tt * ld + j] = acc[tt];
  }
  __syncthreads();
  {
    // One warp per token: keys get the base-2 norm term plus 1/2 log2(m); queries
    // get their row max when stabilised (else 0: per-query constants cancel).
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const float* pr = P + warp * ld;
    float val = 0.f;
    if (side) {
      for (int i = lane; i < r; i += 32) val = fmaf(pr[m + i], pr[m + i], val);
      val = warp_sum(val) + 0.5f * log2f((float)m);
    } else if (stabilise) {
      val = -INFINITY;
      for (int j = lane; j < m; j += 32) val = fmaxf(val, pr[j]);
      val = warp_max(val);
    }
    if (lane == 0) cst[warp] = val;
  }
  __syncthreads();
  float* dst = side ? phik : phiq;
  float kmax = -INFINITY;
  for (int e = threadIdx.x; e < kTF * m; e += blockDim.x) {
    const int tt = e / m, j = e % m, t = t0 + tt;
    if (t >= L) continue;
    const float ex = P[tt * ld + j] - cst[tt];
    float val;
    if (side) {
      const bool ok = mask == nullptr || mask[(size_t)b * L + t] != 0;
      if (!ok) {
        val = stabilise ? -INFINITY : 0.f;
      } else if (stabilise) {
        val = ex;
        kmax = fmaxf(kmax, ex);
      } else {
        val = exp2f(ex);
      }
    } else {
      val = exp2f(ex);
    }
    dst[((size_t)bh * L + t) * m + j] = val;
  }
  if (side && stabilise) {
    kmax = warp_max(kmax);
    if ((threadIdx.x & 31) == 0 && kmax > -INFINITY) atomicMax(&ck[bh], float_to_ordered(kmax));
  }
}

// Stabilised keys: phi = 2^(e - c_K) with c_K the largest valid key exponent of the head.
__global__ void expshift_kernel(float* __restrict__ phik, const int* __restrict__ ck, int L, int m,
                                size_t n) {
  const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const int bh = (int)(i / ((size_t)L * m));
  const float e = phik[i];
  float c = ordered_to_float(ck[bh]);
  if (!(c > -INFINITY)) c = 0.f;
  phik[i] = e == -INFINITY ? 0.f : exp2f(e - c);
}

// Per chunk of keys: S_c = Phi(K_c)^T [V_c | 1], fp32, [m][d + 1].
template <typename T>
__global__ void __launch_bounds__(256) chunk_state_kernel(
    const float* __restrict__ phik, const T* __restrict__ v, int64_t sb, int64_t sh, int64_t sl,
    int m, int d, int H, int L, int chunk_len, int nc, float* __restrict__ chunk_s) {
  __shared__ float As[32][65];
  __shared__ float Bs[32][65];
  const int c = blockIdx.x, bh = blockIdx.y, b = bh / H, h = bh % H;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int dd = d + 1;
  const int tb = c * chunk_len;
  const int te = min(L, tb + chunk_len);
  float* out = chunk_s + ((size_t)bh * nc + c) * m * dd;
  for (int jt = 0; jt < m; jt += 64) {
    for (int et = 0; et < dd; et += 64) {
      float acc[4][4] = {};
      for (int tk = tb; tk < te; tk += 32) {
        for (int e = threadIdx.x; e < 32 * 64; e += 256) {
          const int tok = e >> 6, f = e & 63, t = tk + tok;
          As[tok][f] = (t < te && jt + f < m) ? phik[((size_t)bh * L + t) * m + jt + f] : 0.f;
          const int col = et + f;
          float bv = 0.f;
          if (t < te) {
            if (col < d) bv = to_f32(v[(int64_t)b * sb + (int64_t)h * sh + (int64_t)t * sl + col]);
            else if (col == d) bv = 1.f;
          }
          Bs[tok][f] = bv;
        }
        __syncthreads();
#pragma unroll 8
        for (int kk = 0; kk < 32; ++kk) {
          float a[4], bb[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
          for (int j = 0; j < 4; ++j) bb[j] = Bs[kk][tx * 4 + j];
#pragma unroll
          for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], bb[j], acc[i][j]);
        }
        __syncthreads();
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int row = jt + ty * 4 + i;
        if (row >= m) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int col = et + tx * 4 + j;
          if (col < dd) out[(size_t)row * dd + col] = acc[i][j];
        }
      }
    }
  }
}

// Causal: exclusive prefix over chunks, in place. Non-causal: total into chunk 0.
// Also writes the statistics over all valid keys to the state, if requested.
__global__ void scan_kernel(float* __restrict__ chunk_s, int m, int d, int nc, int causal,
                            float* __restrict__ st_kv, float* __restrict__ st_z,
                            float* __restrict__ st_shift, const int* __restrict__ ck) {
  const int dd = d + 1;
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  const int bh = blockIdx.y;
  if (st_shift != nullptr && idx == 0) {
    float c = ordered_to_float(ck[bh]);
    st_shift[bh] = c > -INFINITY ? c : 0.f;
  }
  if (idx >= m * dd) return;
  float* base = chunk_s + (size_t)bh * nc * m * dd + idx;
  const size_t step = (size_t)m * dd;
  float run = 0.f;
  for (int c = 0; c < nc; ++c) {
    const float t = base[c * step];
    if (causal) base[c * step] = run;
    run += t;
  }
  if (!causal) base[0] = run;
  if (st_kv != nullptr) {
    const int j = idx / dd, e = idx % dd;
    if (e < d) st_kv[((size_t)bh * m + j) * d + e] = run;
    else st_z[(size_t)bh * m + j] = run;
  }
}

// out = [Psi(Q) S_x + (causal) tril(Psi(Q) Phi(K)^T) [V | 1]] / den, 64 queries per block.
template <typename T>
__global__ void __launch_bounds__(256) out_kernel(
    const float* __restrict__ phiq, const float* __restrict__ phik,
    const float* __restrict__ chunk_s, const T* __restrict__ v, int64_t vb, int64_t vh,
    int64_t vl, T* __restrict__ out, int64_t ob, int64_t oh, int64_t ol, int m, int d, int H,
    int L, int causal, int chunk_len, int nc, const uint8_t* __restrict__ qmask,
    int* dev_status) {
  extern __shared__ float sm[];
  const int dd = d + 1;
  const int ET = (dd + 63) / 64;
  const int ddp = ET * 64;
  float* Qs = sm;                 // [64][33]
  float* Ks = Qs + 64 * 33;       // [32][33]
  float* At = Ks + 32 * 33;       // [64][33]
  float* Bt = At + 64 * 33;       // [32][ddp]
  float* den = Bt + 32 * ddp;     // [64]
  const int q0 = blockIdx.x * 64;
  const int bh = blockIdx.y, b = bh / H, h = bh % H;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int c = causal ? q0 / chunk_len : 0;
  const float* sx = chunk_s + ((size_t)bh * nc + c) * m * dd;
  float acc[5][4][4];
#pragma unroll
  for (int et = 0; et < 5; ++et)
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[et][i][j] = 0.f;

  for (int j0 = 0; j0 < m; j0 += 32) {
    for (int e = threadIdx.x; e < 64 * 32; e += 256) {
      const int i = e >> 5, jj = e & 31;
      Qs[i * 33 + jj] = (q0 + i < L && j0 + jj < m) ? phiq[((size_t)bh * L + q0 + i) * m + j0 + jj] : 0.f;
    }
    for (int e = threadIdx.x; e < 32 * ddp; e += 256) {
      const int jj = e / ddp, col = e % ddp;
      Bt[e] = (j0 + jj < m && col < dd) ? sx[(size_t)(j0 + jj) * dd + col] : 0.f;
    }
    __syncthreads();
    for (int kk = 0; kk < 32; ++kk) {
      float a[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = Qs[(ty * 4 + i) * 33 + kk];
#pragma unroll
      for (int et = 0; et < 5; ++et) {
        if (et < ET) {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float bv = Bt[kk * ddp + et * 64 + tx * 4 + j];
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[et][i][j] = fmaf(a[i], bv, acc[et][i][j]);
          }
        }
      }
    }
    __syncthreads();
  }
  if (causal) {
    const int kbeg = c * chunk_len;
    const int kend = min(L, q0 + 64);
    const int ai = threadIdx.x >> 2, at = (threadIdx.x & 3) * 8;
    for (int t0 = kbeg; t0 < kend; t0 += 32) {
      float a8[8] = {};
      for (int f0 = 0; f0 < m; f0 += 32) {
        for (int e = threadIdx.x; e < 64 * 32; e += 256) {
          const int i = e >> 5, jj = e & 31;
          Qs[i * 33 + jj] = (q0 + i < L && f0 + jj < m) ? phiq[((size_t)bh * L + q0 + i) * m + f0 + jj] : 0.f;
        }
        for (int e = threadIdx.x; e < 32 * 32; e += 256) {
          const int t = e >> 5, jj = e & 31;
          Ks[t * 33 + jj] = (t0 + t < L && f0 + jj < m) ? phik[((size_t)bh * L + t0 + t) * m + f0 + jj] : 0.f;
        }
        __syncthreads();
        for (int kk = 0; kk < 32; ++kk) {
          const float qa = Qs[ai * 33 + kk];
#pragma unroll
          for (int u = 0; u < 8; ++u) a8[u] = fmaf(qa, Ks[(at + u) * 33 + kk], a8[u]);
        }
        __syncthreads();
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int t = t0 + at + u;
        At[ai * 33 + at + u] = (t <= q0 + ai && t < L) ? a8[u] : 0.f;
      }
      for (int e = threadIdx.x; e < 32 * ddp; e += 256) {
        const int t = e / ddp, col = e % ddp, tok = t0 + t;
        float bv = 0.f;
        if (tok < L) {
          if (col < d) bv = to_f32(v[(int64_t)b * vb + (int64_t)h * vh + (int64_t)tok * vl + col]);
          else if (col == d) bv = 1.f;
        }
        Bt[e] = bv;
      }
      __syncthreads();
      for (int kk = 0; kk < 32; ++kk) {
        float a[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) a[i] = At[(ty * 4 + i) * 33 + kk];
#pragma unroll
        for (int et = 0; et < 5; ++et) {
          if (et < ET) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const float bv = Bt[kk * ddp + et * 64 + tx * 4 + j];
#pragma unroll
              for (int i = 0; i < 4; ++i) acc[et][i][j] = fmaf(a[i], bv, acc[et][i][j]);
            }
          }
        }
      }
      __syncthreads();
    }
  }
  // the denominator is column d of the accumulated [num | den]
#pragma unroll
  for (int et = 0; et < 5; ++et) {
    if (et < ET) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (et * 64 + tx * 4 + j == d) {
#pragma unroll
          for (int i = 0; i < 4; ++i) den[ty * 4 + i] = acc[et][i][j];
        }
      }
    }
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int row = ty * 4 + i, t = q0 + row;
    if (t >= L) continue;
    // a masked query row (cross-attention) outputs 0
    const float dn = (qmask == nullptr || qmask[(size_t)b * L + t] != 0) ? den[row] : 0.f;
#pragma unroll
    for (int et = 0; et < 5; ++et) {
      if (et < ET) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int col = et * 64 + tx * 4 + j;
          if (col < d) {
            const float o = dn > 0.f ? acc[et][i][j] / dn : 0.f;
            if (!isfinite(o)) report(dev_status, DARK_ERR_NUMERIC);
            out[(int64_t)b * ob + (int64_t)h * oh + (int64_t)t * ol + col] = from_f32<T>(o);
          }
        }
      }
    }
  }
}

template <typename T>
cudaError_t simt_forward_t(const FwdArgs& a) {
  const SimtLayout s = simt_layout(a.B, a.H, a.L, a.Lk, a.m, a.d, a.flags);
  char* ws = (char*)a.ws;
  int* ck = (int*)(ws + s.off_ck);
  float* phiq = (float*)(ws + s.off_phiq);
  float* phik = (float*)(ws + s.off_phik);
  float* cs = (float*)(ws + s.off_s);
  const int bh = a.B * a.H;
  const int stab = (a.flags & DARK_STABILISE) ? 1 : 0;
  const int causal = (a.flags & DARK_CAUSAL) ? 1 : 0;
  cudaError_t err;

  init_ck_kernel<<<(bh + 255) / 256, 256, 0, a.stream>>>(ck, bh);
  const size_t fsm = sizeof(float) * kTF * (a.d + a.m + a.r);
  err = cudaFuncSetAttribute(features_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)fsm);
  if (err != cudaSuccess) return err;
  const int lmax = a.L > a.Lk ? a.L : a.Lk;
  features_kernel<T><<<dim3((lmax + kTF - 1) / kTF, bh, 2), 256, fsm, a.stream>>>(
      (const T*)a.q, a.qs[0], a.qs[1], a.qs[2], a.L, (const T*)a.k, a.ks[0], a.ks[1], a.ks[2],
      a.Lk, (const typename WeightOf<T>::type*)a.w, a.heads_w, a.m, a.r, a.d, a.H, a.mask, stab,
      phiq, phik, ck);
  if (stab) {
    const size_t n = (size_t)bh * a.Lk * a.m;
    expshift_kernel<<<(unsigned)((n + 255) / 256), 256, 0, a.stream>>>(phik, ck, a.Lk, a.m, n);
  }
  chunk_state_kernel<T><<<dim3(s.nc, bh), 256, 0, a.stream>>>(
      phik, (const T*)a.v, a.ks[0], a.ks[1], a.ks[2], a.m, a.d, a.H, a.Lk, s.chunk_len, s.nc, cs);
  scan_kernel<<<dim3((a.m * (a.d + 1) + 255) / 256, bh), 256, 0, a.stream>>>(
      cs, a.m, a.d, s.nc, causal, a.st_kv, a.st_z, stab ? a.st_shift : nullptr, ck);
  const int ddp = ((a.d + 1 + 63) / 64) * 64;
  const size_t osm = sizeof(float) * (64 * 33 + 32 * 33 + 64 * 33 + 32 * ddp + 64);
  err = cudaFuncSetAttribute(out_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)osm);
  if (err != cudaSuccess) return err;
  out_kernel<T><<<dim3((a.L + 63) / 64, bh), 256, osm, a.stream>>>(
      phiq, phik, cs, (const T*)a.v, a.ks[0], a.ks[1], a.ks[2], (T*)a.out, a.os[0], a.os[1],
      a.os[2], a.m, a.d, a.H, a.L, causal, s.chunk_len, s.nc, a.qmask, a.dev_status);
  return cudaGetLastError();
}

}  // namespace

size_t simt_workspace_bytes(int B, int H, int Lq, int Lk, int m, int d, int flags) {
  return simt_layout(B, H, Lq, Lk, m, d, flags).total;
}

cudaError_t simt_forward(const FwdArgs& a) {
  return a.dtype == DARK_BF16 ? simt_forward_t<__nv_bfloat16>(a) : simt_forward_t<float>(a);
}

}  // namespace dark
