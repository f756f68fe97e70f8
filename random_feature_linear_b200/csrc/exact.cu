// Exact learned-kernel attention (README, section "Attention modes": in the exact
// mode M acts on queries and keys and ordinary softmax attention with scaled
// scores follows): out_i = sum_j softmax_j(u_i . w_j) v_j with u = M q~, w = M k~,
// x~ = d^{-1/4} x, i.e. scores q^T Sigma k / sqrt(d), over the valid keys (j <= i
// when causal). A query row with no visible key, or a masked query row in
// cross-attention, outputs 0.
//
// The projection's last r rows are c_m M with c_m = d^{-1/4} sqrt(log2(e)/2), so
// with p = W'_bot x the base-2 score is 2 p_q . p_k = log2(e) u . w and the mode
// needs nothing beyond the projection. Two SIMT fp32 kernels: p for every query
// and key token into the workspace, then one CTA per 64-query tile that walks the
// 64-key tiles with an online softmax (running row maximum and sum, base 2) and
// accumulates O += P V.
#include <math.h>

#include "common.cuh"
#include "internal.h"
#include "simt_tile.cuh"

namespace dark {
namespace {

constexpr int kT = 64;

struct ExactLayout {
  size_t off_pq, off_pk, total;
};

ExactLayout exact_layout(int B, int H, int Lq, int Lk, int r) {
  ExactLayout s;
  const size_t bh = (size_t)B * H;
  s.off_pq = kWsHeader;
  s.off_pk = align_up(s.off_pq + sizeof(float) * bh * Lq * r, 256);
  s.total = align_up(s.off_pk + sizeof(float) * bh * Lk * r, 256);
  return s;
}

// p = W'_bot x for 64 tokens of one side (blockIdx.z: 0 queries, 1 keys).
template <typename T>
__global__ void __launch_bounds__(256) exact_proj_kernel(
    const T* __restrict__ xq, int64_t qb, int64_t qh, int64_t ql, int Lq,
    const T* __restrict__ xk, int64_t kb, int64_t kh, int64_t kl, int Lk,
    const typename WeightOf<T>::type* __restrict__ w, int heads_w, int m, int r, int d, int H,
    float* __restrict__ pq, float* __restrict__ pk) {
  __shared__ __align__(16) float Xs[32 * kLd];
  __shared__ __align__(16) float Ws[32 * kLd];
  const int side = blockIdx.z;
  const int L = side ? Lk : Lq;
  const int t0 = blockIdx.x * kT;
  if (t0 >= L) return;                       // the grid covers the longer side
  const int bh = blockIdx.y, b = bh / H, h = bh % H;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const T* x = side ? xk + (int64_t)b * kb + (int64_t)h * kh : xq + (int64_t)b * qb + (int64_t)h * qh;
  const int64_t sl = side ? kl : ql;
  const auto* wb = w + ((size_t)(heads_w == 1 ? 0 : h) * (m + r) + m) * d;
  float* dst = (side ? pk : pq) + (size_t)bh * L * r;
  for (int c0 = 0; c0 < r; c0 += 64) {
    float acc[4][4];
    zero(acc);
    for (int k0 = 0; k0 < d; k0 += 32) {
      stage_t(Xs, [&](int t, int kk) {
        return (t0 + t < L && k0 + kk < d) ? to_f32(x[(int64_t)(t0 + t) * sl + k0 + kk]) : 0.f;
      });
      stage_t(Ws, [&](int j, int kk) {
        return (c0 + j < r && k0 + kk < d) ? to_f32(wb[(size_t)(c0 + j) * d + k0 + kk]) : 0.f;
      });
      __syncthreads();
      fma_tile(Xs, Ws, acc);
      __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int t = t0 + ty * 4 + i;
      if (t >= L) continue;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int c = c0 + tx * 4 + j;
        if (c < r) dst[(size_t)t * r + c] = acc[i][j];
      }
    }
  }
}

// One CTA per 64 queries of one (batch, head): scores against 64 keys at a time,
// online softmax in base 2, O += P V. ET = ceil(d / 64) value blocks per thread.
template <typename T, int ET>
__global__ void __launch_bounds__(256) exact_attn_kernel(
    const float* __restrict__ pq, const float* __restrict__ pk, const T* __restrict__ v,
    int64_t vb, int64_t vh, int64_t vl, T* __restrict__ out, int64_t ob, int64_t oh, int64_t ol,
    int r, int d, int H, int Lq, int Lk, int causal, const uint8_t* __restrict__ kmask,
    const uint8_t* __restrict__ qmask, int* dev_status) {
  extern __shared__ __align__(16) float sm[];
  constexpr int ddp = ET * 64;
  const int rp = (r + 31) / 32 * 32;
  float* PqT = sm;                 // [rp][kLd]   the tile's query projections, k-major
  float* Kc = PqT + rp * kLd;      // [32][kLd]   key projections, one chunk of r
  float* PT = Kc + 32 * kLd;       // [64][kLd]   probabilities, k-major (k = key)
  float* Vt = PT + 64 * kLd;       // [32][ddp]   value rows
  const int q0 = blockIdx.x * kT, bh = blockIdx.y, b = bh / H, h = bh % H;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const float* Pq = pq + (size_t)bh * Lq * r;
  const float* Pk = pk + (size_t)bh * Lk * r;
  const T* vh_ = v + (int64_t)b * vb + (int64_t)h * vh;

  for (int k0 = 0; k0 < rp; k0 += 32)
    stage_t(PqT + k0 * kLd, [&](int i, int kk) {
      return (q0 + i < Lq && k0 + kk < r) ? Pq[(size_t)(q0 + i) * r + k0 + kk] : 0.f;
    });
  float acc[ET][4][4];
#pragma unroll
  for (int et = 0; et < ET; ++et) zero(acc[et]);
  float rmax[4], rsum[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    rmax[i] = -INFINITY;
    rsum[i] = 0.f;
  }
  const int kend = causal ? min(Lk, q0 + kT) : Lk;
  for (int j0 = 0; j0 < kend; j0 += kT) {
    float s4[4][4];
    zero(s4);
    for (int k0 = 0; k0 < rp; k0 += 32) {
      stage_t(Kc, [&](int j, int kk) {
        return (j0 + j < Lk && k0 + kk < r) ? Pk[(size_t)(j0 + j) * r + k0 + kk] : 0.f;
      });
      __syncthreads();
      fma_tile(PqT + k0 * kLd, Kc, s4);
      __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int qi = q0 + ty * 4 + i;
      float tmax = -INFINITY;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int key = j0 + tx * 4 + j;
        const bool ok = key < Lk && (kmask == nullptr || kmask[(size_t)b * Lk + key] != 0) &&
                        (!causal || key <= qi);
        s4[i][j] = ok ? 2.f * s4[i][j] : -INFINITY;
        tmax = fmaxf(tmax, s4[i][j]);
      }
      // the 16 threads of a row are 16 consecutive lanes
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, o));
      const float nmax = fmaxf(rmax[i], tmax);
      const float scale = nmax == -INFINITY ? 1.f : exp2f(rmax[i] - nmax);
      float psum = 0.f;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float p = s4[i][j] == -INFINITY ? 0.f : exp2f(s4[i][j] - nmax);
        s4[i][j] = p;
        psum += p;
      }
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) psum += __shfl_xor_sync(0xffffffffu, psum, o);
      rsum[i] = rsum[i] * scale + psum;
      rmax[i] = nmax;
#pragma unroll
      for (int et = 0; et < ET; ++et)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[et][i][j] *= scale;
    }
#pragma unroll
    for (int j = 0; j < 4; ++j)
      *reinterpret_cast<float4*>(PT + (tx * 4 + j) * kLd + ty * 4) =
          make_float4(s4[0][j], s4[1][j], s4[2][j], s4[3][j]);
    for (int k0 = 0; k0 < kT; k0 += 32) {
      for (int e = threadIdx.x; e < 32 * ddp; e += blockDim.x) {
        const int kk = e / ddp, col = e % ddp, key = j0 + k0 + kk;
        Vt[e] = (key < Lk && col < d) ? to_f32(vh_[(int64_t)key * vl + col]) : 0.f;
      }
      __syncthreads();
#pragma unroll 4
      for (int kk = 0; kk < 32; ++kk) {
        const float4 a4 = ld4(PT + (k0 + kk) * kLd + ty * 4);
        const float a[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
        for (int et = 0; et < ET; ++et) {
          const float4 b4 = ld4(Vt + kk * ddp + et * 64 + tx * 4);
          const float bb[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
          for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[et][i][j] = fmaf(a[i], bb[j], acc[et][i][j]);
        }
      }
      __syncthreads();
    }
  }
  T* oh_ = out + (int64_t)b * ob + (int64_t)h * oh;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int qi = q0 + ty * 4 + i;
    if (qi >= Lq) continue;
    const bool live = qmask == nullptr || qmask[(size_t)b * Lq + qi] != 0;
    const float inv = (live && rsum[i] > 0.f) ? 1.f / rsum[i] : 0.f;
#pragma unroll
    for (int et = 0; et < ET; ++et)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int col = et * 64 + tx * 4 + j;
        if (col >= d) continue;
        const float o = acc[et][i][j] * inv;
        if (!isfinite(o)) report(dev_status, DARK_ERR_NUMERIC);
        oh_[(int64_t)qi * ol + col] = from_f32<T>(o);
      }
  }
}

size_t attn_smem_bytes(int r, int et) {
  const int rp = (r + 31) / 32 * 32;
  return sizeof(float) * ((size_t)rp * kLd + 32 * kLd + 64 * kLd + 32 * et * 64);
}

template <typename T, int ET>
cudaError_t launch_attn(const FwdArgs& a, const float* pq, const float* pk) {
  static int smem_set[64];
  const size_t bytes = attn_smem_bytes(256, ET);        // opt-in once, for the largest r
  cudaError_t err =
      set_smem_limit_once((const void*)exact_attn_kernel<T, ET>, (int)bytes, smem_set);
  if (err != cudaSuccess) return err;
  exact_attn_kernel<T, ET><<<dim3((a.L + kT - 1) / kT, a.B * a.H), 256,
                             attn_smem_bytes(a.r, ET), a.stream>>>(
      pq, pk, (const T*)a.v, a.ks[0], a.ks[1], a.ks[2], (T*)a.out, a.os[0], a.os[1], a.os[2], a.r,
      a.d, a.H, a.L, a.Lk, (a.flags & DARK_CAUSAL) ? 1 : 0, a.mask, a.qmask, a.dev_status);
  return cudaGetLastError();
}

template <typename T>
cudaError_t exact_forward_t(const FwdArgs& a) {
  const ExactLayout s = exact_layout(a.B, a.H, a.L, a.Lk, a.r);
  float* pq = (float*)((char*)a.ws + s.off_pq);
  float* pk = (float*)((char*)a.ws + s.off_pk);
  const int lmax = a.L > a.Lk ? a.L : a.Lk;
  exact_proj_kernel<T><<<dim3((lmax + kT - 1) / kT, a.B * a.H, 2), 256, 0, a.stream>>>(
      (const T*)a.q, a.qs[0], a.qs[1], a.qs[2], a.L, (const T*)a.k, a.ks[0], a.ks[1], a.ks[2],
      a.Lk, (const typename WeightOf<T>::type*)a.w, a.heads_w, a.m, a.r, a.d, a.H, pq, pk);
  switch ((a.d + 63) / 64) {
    case 1: return launch_attn<T, 1>(a, pq, pk);
    case 2: return launch_attn<T, 2>(a, pq, pk);
    case 3: return launch_attn<T, 3>(a, pq, pk);
    case 4: return launch_attn<T, 4>(a, pq, pk);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

size_t exact_workspace_bytes(int B, int H, int Lq, int Lk, int r) {
  return exact_layout(B, H, Lq, Lk, r).total;
}

cudaError_t exact_forward(const FwdArgs& a) {
  return a.dtype == DARK_BF16 ? exact_forward_t<__nv_bfloat16>(a) : exact_forward_t<float>(a);
}

}  // namespace dark
