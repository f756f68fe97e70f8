// Streaming decode step of PRF attention (DARKformer README, section
// "Encoder-decoder model and generation": in linear mode the recurrent
// statistics Phi(K)^T V and Phi(K)^T 1 are updated per appended token).
//
// One block per (batch, head). The step is bound by reading and writing the
// fp32 state (m x d + m floats per head), so the block first computes both
// feature vectors (a GEMV with W' from L2), then streams its state rows with
// coalesced 16-byte accesses, several rows in flight per thread, and folds the
// output contraction into the same pass: out = phi(q)^T kv' / phi(q)^T z'.
#include <math.h>

#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace dark {
namespace {

constexpr int kThreads = 256;
constexpr int kBatchRows = 16;  // state rows held in registers per thread and pass

__device__ __forceinline__ void row_dot2(const float* __restrict__ w, int d, const float* xk,
                                         const float* xq, bool both, float& ak, float& aq) {
  float sk = 0.f, sq = 0.f;
  if ((d & 3) == 0) {
    const float4* w4 = reinterpret_cast<const float4*>(w);
    for (int c = 0; c < d / 4; ++c) {
      const float4 u = __ldg(w4 + c);
      sk = fmaf(u.x, xk[4 * c], sk); sk = fmaf(u.y, xk[4 * c + 1], sk);
      sk = fmaf(u.z, xk[4 * c + 2], sk); sk = fmaf(u.w, xk[4 * c + 3], sk);
      if (both) {
        sq = fmaf(u.x, xq[4 * c], sq); sq = fmaf(u.y, xq[4 * c + 1], sq);
        sq = fmaf(u.z, xq[4 * c + 2], sq); sq = fmaf(u.w, xq[4 * c + 3], sq);
      }
    }
  } else {
    for (int c = 0; c < d; ++c) {
      sk = fmaf(w[c], xk[c], sk);
      if (both) sq = fmaf(w[c], xq[c], sq);
    }
  }
  ak = sk;
  aq = sq;
}

// fp16 projection rows (the weight type of bf16 tokens).
__device__ __forceinline__ void row_dot2(const __half* __restrict__ w, int d, const float* xk,
                                         const float* xq, bool both, float& ak, float& aq) {
  float sk = 0.f, sq = 0.f;
  if ((d & 7) == 0) {
    const uint4* w8 = reinterpret_cast<const uint4*>(w);
    for (int c = 0; c < d / 8; ++c) {
      const uint4 u = __ldg(w8 + c);
      const __half2* p = reinterpret_cast<const __half2*>(&u);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __half22float2(p[e]);
        sk = fmaf(f.x, xk[8 * c + 2 * e], sk);
        sk = fmaf(f.y, xk[8 * c + 2 * e + 1], sk);
        if (both) {
          sq = fmaf(f.x, xq[8 * c + 2 * e], sq);
          sq = fmaf(f.y, xq[8 * c + 2 * e + 1], sq);
        }
      }
    }
  } else {
    for (int c = 0; c < d; ++c) {
      const float f = __half2float(w[c]);
      sk = fmaf(f, xk[c], sk);
      if (both) sq = fmaf(f, xq[c], sq);
    }
  }
  ak = sk;
  aq = sq;
}

__device__ __forceinline__ float block_sum(float v, float* scratch) {
  v = warp_sum(v);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) scratch[warp] = v;
  __syncthreads();
  float t = lane < kThreads / 32 ? scratch[lane] : 0.f;
  return warp_sum(t);
}


// W' of one head is copied to shared memory (one bulk copy at the start,
// overlapping the state prefetch) when it is at most this large; the feature
// GEMV then reads it there instead of paying L2 latency per batch of rows.
constexpr size_t kStageW = 64 * 1024;

// 8 consecutive weights of a W' row as fp32 (fp16 or fp32 storage; the row is
// in global memory or, when staged, in shared memory: a generic load).
__device__ __forceinline__ void load_w8(const __half* __restrict__ w, float (&f)[8]) {
  const uint4 u = *reinterpret_cast<const uint4*>(w);
  const __half2* h = reinterpret_cast<const __half2*>(&u);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 t = __half22float2(h[e]);
    f[2 * e] = t.x;
    f[2 * e + 1] = t.y;
  }
}
__device__ __forceinline__ void load_w8(const float* __restrict__ w, float (&f)[8]) {
  const float4 a = *reinterpret_cast<const float4*>(w);
  const float4 b = *(reinterpret_cast<const float4*>(w) + 1);
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
  f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}

// Feature exponents W' k and W' q for one head into pk[0, m + r) and pq[0, m).
// Groups of 8 lanes own one W' row at a time, each lane 8 consecutive columns;
// every group first issues the loads of up to 8 of its rows, then reduces
// them with shuffles, so the L2 latency of W' is paid once per batch.
template <int kBatch, typename TW>
__device__ __forceinline__ void feature_gemv(const TW* __restrict__ wh, int m, int r, int d,
                                             const float* xk, const float* xq, float* pk,
                                             float* pq) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 3, cl = lane & 7;
  const int rows = m + r;
  constexpr int kGroups = kThreads / 8;
  for (int c0 = 0; c0 < d; c0 += 64) {
    float fk[8], fq[8];
    const int col = c0 + cl * 8;
    const bool cok = col < d;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      fk[e] = cok ? xk[col + e] : 0.f;
      fq[e] = cok ? xq[col + e] : 0.f;
    }
    for (int jb = warp * 4 + g; jb < rows; jb += kBatch * kGroups) {
      float wv[kBatch][8];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int j = jb + u * kGroups;
        if (cok && j < rows) load_w8(wh + (size_t)j * d + col, wv[u]);
        else {
#pragma unroll
          for (int e = 0; e < 8; ++e) wv[u][e] = 0.f;
        }
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int j = jb + u * kGroups;
        float ak = 0.f, aq = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          ak = fmaf(wv[u][e], fk[e], ak);
          aq = fmaf(wv[u][e], fq[e], aq);
        }
#pragma unroll
        for (int o = 4; o > 0; o >>= 1) {
          ak += __shfl_xor_sync(0xffffffffu, ak, o);
          aq += __shfl_xor_sync(0xffffffffu, aq, o);
        }
        if (cl == 0 && j < rows) {
          pk[j] = (c0 == 0 ? 0.f : pk[j]) + ak;
          if (j < m) pq[j] = (c0 == 0 ? 0.f : pq[j]) + aq;
        }
      }
    }
  }
}

// 8 consecutive weights of a staged W' row (shared memory) as fp32.
__device__ __forceinline__ void load_w8_shared(uint32_t saddr, const __half*, float (&f)[8]) {
  const uint4 u = tc::ld_shared_v4(saddr);
  const __half2* h = reinterpret_cast<const __half2*>(&u);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 t = __half22float2(h[e]);
    f[2 * e] = t.x;
    f[2 * e + 1] = t.y;
  }
}
__device__ __forceinline__ void load_w8_shared(uint32_t saddr, const float*, float (&f)[8]) {
  const uint4 a = tc::ld_shared_v4(saddr), b = tc::ld_shared_v4(saddr + 16);
  f[0] = __uint_as_float(a.x); f[1] = __uint_as_float(a.y);
  f[2] = __uint_as_float(a.z); f[3] = __uint_as_float(a.w);
  f[4] = __uint_as_float(b.x); f[5] = __uint_as_float(b.y);
  f[6] = __uint_as_float(b.z); f[7] = __uint_as_float(b.w);
}

// The feature GEMV on staged W' rows (d a multiple of 8): 8-lane groups, one
// row at a time per group, all rows of a group in flight together; also
// returns this thread's share of sum_i (W'_{m+i} k)^2 (the key norm), which
// lanes 0 of the groups hold and the caller reduces.
template <typename TW>
__device__ __forceinline__ float feature_gemv_shared(const TW* w_sm, int m, int r, int d,
                                                     const float* xk, const float* xq, float* pk,
                                                     float* pq) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 3, cl = lane & 7;
  const int rows = m + r;
  constexpr int kGroups = kThreads / 8;
  const uint32_t wbase = tc::smem_u32(w_sm);
  float nrm = 0.f;
  for (int c0 = 0; c0 < d; c0 += 64) {
    const int col = c0 + cl * 8;
    const bool cok = col < d;
    float fk[8], fq[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      fk[e] = cok ? xk[col + e] : 0.f;
      fq[e] = cok ? xq[col + e] : 0.f;
    }
#pragma unroll 4
    for (int j = warp * 4 + g; j < rows; j += kGroups) {
      float wv[8];
      if (cok) {
        load_w8_shared(wbase + (uint32_t)(((size_t)j * d + col) * sizeof(TW)), (const TW*)nullptr, wv);
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) wv[e] = 0.f;
      }
      float ak = 0.f, aq = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        ak = fmaf(wv[e], fk[e], ak);
        aq = fmaf(wv[e], fq[e], aq);
      }
#pragma unroll
      for (int o = 4; o > 0; o >>= 1) {
        ak += __shfl_xor_sync(0xffffffffu, ak, o);
        aq += __shfl_xor_sync(0xffffffffu, aq, o);
      }
      if (cl == 0) {
        const float tk = (c0 == 0 ? 0.f : pk[j]) + ak;
        pk[j] = tk;
        if (j < m) pq[j] = (c0 == 0 ? 0.f : pq[j]) + aq;
        else if (c0 + 64 >= d) nrm = fmaf(tk, tk, nrm);   // norm row, all columns summed
      }
    }
  }
  return nrm;
}

// The feature GEMV on staged fp16 W' rows (d a multiple of 8): one thread per
// row, the row's chunks of 8 columns visited from a per-row rotation so that
// the threads of a warp read different banks; no shuffles. Returns this
// thread's share of sum_i (W'_{m+i} k)^2 (the key norm).
__device__ __forceinline__ float feature_gemv_rows(const __half* w_sm, int m, int r, int d,
                                                   const float* xk, const float* xq, float* pk,
                                                   float* pq, int nthreads) {
  const int nch = d / 8;
  float nrm = 0.f;
  for (int j = threadIdx.x; j < m + r; j += nthreads) {
    const uint4* wr = reinterpret_cast<const uint4*>(w_sm + (size_t)j * d);
    float ak = 0.f, aq = 0.f;
    const bool want_q = j < m;
#pragma unroll 4
    for (int cc = 0; cc < nch; ++cc) {
      int c = cc + j;
      c -= (c / nch) * nch;
      const uint4 u = wr[c];
      const __half2* hp = reinterpret_cast<const __half2*>(&u);
      const float4 k0 = *reinterpret_cast<const float4*>(xk + 8 * c);
      const float4 k1 = *reinterpret_cast<const float4*>(xk + 8 * c + 4);
      const float2 w0 = __half22float2(hp[0]), w1 = __half22float2(hp[1]);
      const float2 w2 = __half22float2(hp[2]), w3 = __half22float2(hp[3]);
      ak = fmaf(w0.x, k0.x, ak); ak = fmaf(w0.y, k0.y, ak); ak = fmaf(w1.x, k0.z, ak);
      ak = fmaf(w1.y, k0.w, ak); ak = fmaf(w2.x, k1.x, ak); ak = fmaf(w2.y, k1.y, ak);
      ak = fmaf(w3.x, k1.z, ak); ak = fmaf(w3.y, k1.w, ak);
      if (want_q) {
        const float4 q0 = *reinterpret_cast<const float4*>(xq + 8 * c);
        const float4 q1 = *reinterpret_cast<const float4*>(xq + 8 * c + 4);
        aq = fmaf(w0.x, q0.x, aq); aq = fmaf(w0.y, q0.y, aq); aq = fmaf(w1.x, q0.z, aq);
        aq = fmaf(w1.y, q0.w, aq); aq = fmaf(w2.x, q1.x, aq); aq = fmaf(w2.y, q1.y, aq);
        aq = fmaf(w3.x, q1.z, aq); aq = fmaf(w3.y, q1.w, aq);
      }
    }
    pk[j] = ak;
    if (want_q) pq[j] = aq;
    else nrm = fmaf(ak, ak, nrm);
  }
  return nrm;
}

template <typename T>
__global__ void __launch_bounds__(kThreads, 2) decode_kernel(
    const typename WeightOf<T>::type* __restrict__ w, int heads_w, int m, int r, int d,
    float* __restrict__ kv, float* __restrict__ z, const float* __restrict__ shift, int H,
    const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v, T* __restrict__ out,
    const uint8_t* __restrict__ valid, int* dev_status, int stage_w, int update) {
  using TW = typename WeightOf<T>::type;
  extern __shared__ __align__(16) float sm[];
  const int tpr = d / 4;                  // threads per state row (one float4 each)
  const int rpp = kThreads / tpr;         // rows per pass
  float* xq = sm;                         // [d]
  float* xk = xq + d;                     // [d]
  float* xv = xk + d;                     // [d]
  float* pk = xv + d;                     // [m + r]
  float* pq = pk + m + r;                 // [m]
  float* red = pq + m;                    // [rpp][d]
  float* scratch = red + rpp * d;         // [32]
  // 16-byte aligned tail: the copy barrier, then the staged W' rows [m + r][d]
  const size_t tail = ((size_t)(3 * d + (m + r) + m + rpp * d + 32) * 4 + 15) / 16 * 16;
  uint64_t* bar_w = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(sm) + tail);
  TW* w_sm = reinterpret_cast<TW*>(reinterpret_cast<uint8_t*>(sm) + tail + 16);
  const int bh = blockIdx.x, b = bh / H, h = bh % H;
  const TW* wg = w + (size_t)(heads_w == 1 ? 0 : h) * (m + r) * d;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t w_bytes = (uint32_t)((size_t)(m + r) * d * sizeof(TW));
  if (stage_w && tid == 0) {
    tc::mbar_init(bar_w, 1);
    tc::fence_mbar_init();
    tc::mbar_arrive_expect_tx(bar_w, w_bytes);
    for (uint32_t o = 0; o < w_bytes; o += 16384)
      tc::bulk_load(reinterpret_cast<uint8_t*>(w_sm) + o, reinterpret_cast<const uint8_t*>(wg) + o,
                    w_bytes - o < 16384 ? w_bytes - o : 16384, bar_w);
  }
  const TW* wh = stage_w ? w_sm : wg;
  const int c4 = tid % tpr, r0 = tid / tpr;
  const bool rows_active = r0 < rpp;
  float4* base = reinterpret_cast<float4*>(kv + (size_t)bh * m * d) + c4;
  const int stride = d / 4;

  // The step's tokens first (they gate the feature GEMV), then the state rows
  // of the first pass, whose HBM latency overlaps the feature computation.
  // (update == 0: cross-attention against a fixed context; k and v are unused)
  const bool has_c = tid < d;             // d <= kThreads: one element per thread
  const T q_e = has_c ? q[(size_t)bh * d + tid] : T(0.f);
  const T k_e = has_c && update ? k[(size_t)bh * d + tid] : T(0.f);
  const T v_e = has_c && update ? v[(size_t)bh * d + tid] : T(0.f);
  float4 s[kBatchRows];
  if (rows_active) {
#pragma unroll
    for (int u = 0; u < kBatchRows; ++u) {
      const int j = r0 + u * rpp;
      if (j < m) s[u] = __ldcs(base + (size_t)j * stride);
    }
  }
  float zpre[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int j = tid + u * kThreads;
    zpre[u] = j < m ? __ldcs(z + (size_t)bh * m + j) : 0.f;
  }

  if (has_c) {
    xq[tid] = to_f32(q_e);
    xk[tid] = to_f32(k_e);
    xv[tid] = to_f32(v_e);
  }
  __syncthreads();
  if (stage_w) {
    // W' in shared memory (bounded wait; on a time-out nothing is written)
    const bool arrived = tc::mbar_wait(bar_w, 0);
    if (__syncthreads_or(arrived ? 0 : 1)) {
      if (tid == 0) {
        report(dev_status, DARK_ERR_TIMEOUT);
        tc::mbar_wait(bar_w, 0);   // the copy must not land after the block is gone
      }
      __syncthreads();
      return;
    }
  }
  // Feature exponents W' k and W' q: groups of 8 lanes own one row at a time,
  // each lane 8 consecutive columns (held in registers), reduced by shuffles.
  // Rows whose length is not a multiple of 8 take one thread per row instead.
  const bool stab = shift != nullptr;
  float ks, qs;
  if (stage_w && !stab) {
    // GEMV on the staged rows; the key norm from per-warp partial sums
    float part;
    if constexpr (sizeof(TW) == 2)
      part = warp_sum(feature_gemv_rows(reinterpret_cast<const __half*>(w_sm), m, r, d, xk, xq, pk,
                                        pq, kThreads));
    else
      part = warp_sum(feature_gemv_shared(w_sm, m, r, d, xk, xq, pk, pq));
    if (lane == 0) scratch[2 + warp] = part;
    __syncthreads();
    float nrm = 0.f;
#pragma unroll
    for (int i = 0; i < kThreads / 32; ++i) nrm += scratch[2 + i];
    ks = nrm + 0.5f * log2f((float)m);
    qs = 0.f;
  } else {
    if (d % 8 != 0) {
      for (int j = tid; j < m + r; j += kThreads) {
        float ak, aq;
        row_dot2(wh + (size_t)j * d, d, xk, xq, j < m, ak, aq);
        pk[j] = ak;
        if (j < m) pq[j] = aq;
      }
    } else {
      feature_gemv<2>(wh, m, r, d, xk, xq, pk, pq);
    }
    __syncthreads();
    // warp 0: key norm (base 2, with 1/2 log2 m) and, when stabilised, the query max
    if (warp == 0) {
      float nrm = 0.f, qmax = -INFINITY;
      for (int i = lane; i < r; i += 32) nrm = fmaf(pk[m + i], pk[m + i], nrm);
      if (stab)
        for (int j = lane; j < m; j += 32) qmax = fmaxf(qmax, pq[j]);
      nrm = warp_sum(nrm);
      qmax = warp_max(qmax);
      if (lane == 0) {
        scratch[0] = nrm + 0.5f * log2f((float)m) + (stab ? shift[bh] : 0.f);
        scratch[1] = stab ? qmax : 0.f;
      }
    }
    __syncthreads();
    ks = scratch[0];
    qs = scratch[1];
  }
  const bool ok = update && (valid == nullptr || valid[b] != 0);
  for (int j = tid; j < m; j += kThreads) {
    pk[j] = ok ? exp2f(pk[j] - ks) : 0.f;
    pq[j] = exp2f(pq[j] - qs);
  }
  __syncthreads();

  // kv' = kv + phi(k) v^T and num = phi(q)^T kv', one float4 column group per thread.
  float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
  if (rows_active) {
    const float4 vv = make_float4(xv[4 * c4], xv[4 * c4 + 1], xv[4 * c4 + 2], xv[4 * c4 + 3]);
    for (int j0 = r0; j0 < m; j0 += rpp * kBatchRows) {
      if (j0 != r0) {
#pragma unroll
        for (int u = 0; u < kBatchRows; ++u) {
          const int j = j0 + u * rpp;
          if (j < m) s[u] = __ldcs(base + (size_t)j * stride);
        }
      }
#pragma unroll
      for (int u = 0; u < kBatchRows; ++u) {
        const int j = j0 + u * rpp;
        if (j < m) {
          const float fk = pk[j], fq = pq[j];
          s[u].x = fmaf(fk, vv.x, s[u].x); s[u].y = fmaf(fk, vv.y, s[u].y);
          s[u].z = fmaf(fk, vv.z, s[u].z); s[u].w = fmaf(fk, vv.w, s[u].w);
          if (update) __stcs(base + (size_t)j * stride, s[u]);
          num.x = fmaf(fq, s[u].x, num.x); num.y = fmaf(fq, s[u].y, num.y);
          num.z = fmaf(fq, s[u].z, num.z); num.w = fmaf(fq, s[u].w, num.w);
        }
      }
    }
    float* rr = red + r0 * d + 4 * c4;
    rr[0] = num.x; rr[1] = num.y; rr[2] = num.z; rr[3] = num.w;
  }
  float den = 0.f;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int j = tid + u * kThreads;
    if (j < m) {
      const float zj = zpre[u] + pk[j];
      if (update) __stcs(z + (size_t)bh * m + j, zj);
      den = fmaf(pq[j], zj, den);
    }
  }
  den = block_sum(den, scratch + 2);   // contains the barrier that publishes `red`
  for (int c = tid; c < d; c += kThreads) {
    float acc = 0.f;
    for (int g = 0; g < rpp; ++g) acc += red[g * d + c];
    const float o = den > 0.f ? acc / den : 0.f;
    if (!isfinite(o)) report(dev_status, DARK_ERR_NUMERIC);
    out[(size_t)bh * d + c] = from_f32<T>(o);
  }
}


// ---------------------------------------------------------------------------
// Streaming decode step for many heads (the common case: bf16 tokens, fp16
// W', no stabiliser). The step reads and writes every head's fp32 state once,
// so it is bound by HBM bandwidth if enough state is in flight. One persistent
// block per SM walks a contiguous range of heads in projection order (item
// i -> head i / B, batch i % B, so that consecutive items share W'); each
// head's state [kv | z] is copied into one of two shared-memory buffers with a
// single bulk copy (the next head's copy is in flight while this one is
// updated), updated in place, and copied back with a bulk store. W' of the
// current projection head is staged once, with the next one prefetched into a
// second buffer when the head changes.
constexpr int kStreamThreads = 256;

struct StreamLayout {
  uint32_t state, wbytes, oS, oW, oV, total;
};
__host__ __device__ inline StreamLayout stream_layout(int m, int r, int d) {
  StreamLayout L;
  L.state = (uint32_t)m * (d + 1) * 4;                       // [kv (m x d) | z (m)] fp32
  L.wbytes = (uint32_t)(m + r) * d * 2;                      // fp16 W' of one head
  L.oS = 0;
  L.oW = (2 * L.state + 127) / 128 * 128;
  L.oV = L.oW + (2 * L.wbytes + 127) / 128 * 128;
  const int rpp = kStreamThreads / (d / 4);
  // xq, xk, xv [d]; pk [m + r]; pq [m]; red [rpp][d]; scratch [40]; 4 barriers
  L.total = L.oV + (uint32_t)(3 * d + (m + r) + m + rpp * d + 40) * 4 + 64;
  return L;
}

__global__ void __launch_bounds__(kStreamThreads, 1) decode_stream_kernel(
    const __half* __restrict__ w, int heads_w, int m, int r, int d, float* __restrict__ kv,
    float* __restrict__ z, int B, int H, const __nv_bfloat16* __restrict__ q,
    const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
    __nv_bfloat16* __restrict__ out, const uint8_t* __restrict__ valid, int* dev_status, int nitems) {
  extern __shared__ __align__(128) uint8_t smem[];
  const StreamLayout L = stream_layout(m, r, d);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tpr = d / 4, rpp = kStreamThreads / tpr;
  float* xq = reinterpret_cast<float*>(smem + L.oV);
  float* xk = xq + d;
  float* xv = xk + d;
  float* pk = xv + d;                     // [m + r]
  float* pq = pk + m + r;                 // [m]
  float* red = pq + m;                    // [rpp][d]
  float* scratch = red + rpp * d;         // [40]
  uint64_t* bars = reinterpret_cast<uint64_t*>(
      smem + ((L.oV + (uint32_t)(3 * d + (m + r) + m + rpp * d + 40) * 4 + 15) / 16 * 16));
  uint64_t* bar_s = bars;                 // [2] state buffer loaded
  uint64_t* bar_w = bars + 2;             // [2] W' buffer loaded
  const int per = nitems / gridDim.x, extra = nitems % gridDim.x;
  const int it0 = blockIdx.x * per + (blockIdx.x < extra ? blockIdx.x : extra);
  const int nit = per + (blockIdx.x < extra ? 1 : 0);
  auto head_of = [&](int i) { return i / B; };
  auto bh_of = [&](int i) { return (i % B) * H + i / B; };
  auto whead = [&](int h) -> const __half* {
    return w + (size_t)(heads_w == 1 ? 0 : h) * (m + r) * d;
  };
  // bulk copy of item j's state into buffer j & 1 / of W' for head h into buffer sel
  auto load_state = [&](int j) {
    const int bh = bh_of(it0 + j);
    uint64_t* bar = bar_s + (j & 1);
    uint8_t* dst = smem + L.oS + (j & 1) * L.state;
    const uint32_t kvb = (uint32_t)m * d * 4;
    tc::mbar_arrive_expect_tx(bar, L.state);
    for (uint32_t o = 0; o < kvb; o += 32768)
      tc::bulk_load(dst + o, reinterpret_cast<const uint8_t*>(kv + (size_t)bh * m * d) + o,
                    kvb - o < 32768 ? kvb - o : 32768, bar);
    tc::bulk_load(dst + kvb, z + (size_t)bh * m, (uint32_t)m * 4, bar);
  };
  auto load_w = [&](int h, int sel) {
    const uint8_t* src = reinterpret_cast<const uint8_t*>(whead(h));
    tc::mbar_arrive_expect_tx(bar_w + sel, L.wbytes);
    for (uint32_t o = 0; o < L.wbytes; o += 32768)
      tc::bulk_load(smem + L.oW + sel * L.wbytes + o, src + o,
                    L.wbytes - o < 32768 ? L.wbytes - o : 32768, bar_w + sel);
  };
  if (tid == 0) {
    for (int i = 0; i < 4; ++i) tc::mbar_init(bars + i, 1);
    tc::fence_mbar_init();
    if (nit > 0) {
      load_w(head_of(it0), 0);
      load_state(0);
      if (nit > 1) load_state(1);
    }
  }
  __syncthreads();
  int wsel = 0, wphase[2] = {0, 0};
  int s_last[2] = {nit > 0 ? 0 : -1, nit > 1 ? 1 : -1};   // last item loaded into each buffer
  int w_loads[2] = {nit > 0 ? 1 : 0, 0};                    // W' loads issued per buffer
  bool ok = true;
  for (int j = 0; j < nit && ok; ++j) {
    const int i = it0 + j, h = head_of(i), bh = bh_of(i), b = i % B;
    float* st = reinterpret_cast<float*>(smem + L.oS + (j & 1) * L.state);
    float* zs = st + (size_t)m * d;
    if (j > 0 && h != head_of(i - 1)) wsel ^= 1;
    const __half* w_sm = reinterpret_cast<const __half*>(smem + L.oW + wsel * L.wbytes);
    if (tid < d) {
      xq[tid] = __bfloat162float(q[(size_t)bh * d + tid]);
      xk[tid] = __bfloat162float(k[(size_t)bh * d + tid]);
      xv[tid] = __bfloat162float(v[(size_t)bh * d + tid]);
    }
    // W' of this head: wait for its load when the head changes
    const bool new_w = j == 0 || h != head_of(i - 1);
    bool w_ok = true;
    if (new_w) {
      w_ok = tc::mbar_wait(bar_w + wsel, wphase[wsel] & 1);
      wphase[wsel] ^= 1;            // the next load into this buffer completes the next phase
    }
    if (__syncthreads_or(w_ok ? 0 : 1)) {
      ok = false;
      break;
    }
    // feature exponents and the key norm (one thread per W' row)
    const float part = warp_sum(feature_gemv_rows(w_sm, m, r, d, xk, xq, pk, pq, kStreamThreads));
    if (lane == 0) scratch[8 + warp] = part;
    // the buffers of item j - 1 (state) and of the next head's W' are free now:
    // prefetch item j + 1's state once the store of item j - 1 has read it
    if (tid == 0) {
      if (j + 1 < nit && j >= 1) {
        asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
        load_state(j + 1);
        s_last[(j + 1) & 1] = j + 1;
      }
      if (j + 1 < nit && head_of(i + 1) != h) {
        load_w(head_of(i + 1), wsel ^ 1);
        ++w_loads[wsel ^ 1];
      }
    }
    __syncthreads();
    float nrm = 0.f;
#pragma unroll
    for (int u = 0; u < kStreamThreads / 32; ++u) nrm += scratch[8 + u];
    const float ks = nrm + 0.5f * log2f((float)m);
    const bool upd = valid == nullptr || valid[b] != 0;
    for (int jj = tid; jj < m; jj += kStreamThreads) {
      pk[jj] = upd ? exp2f(pk[jj] - ks) : 0.f;
      pq[jj] = exp2f(pq[jj]);
    }
    // this item's state
    const bool s_ok = tc::mbar_wait(bar_s + (j & 1), (j >> 1) & 1);
    if (__syncthreads_or(s_ok ? 0 : 1)) {
      ok = false;
      break;
    }
    // kv' = kv + phi(k) v^T and num = phi(q)^T kv', in place, one float4 column
    // group per thread
    const int c4 = tid % tpr, r0 = tid / tpr;
    float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
    if (r0 < rpp) {
      const float4 vv = make_float4(xv[4 * c4], xv[4 * c4 + 1], xv[4 * c4 + 2], xv[4 * c4 + 3]);
      float4* s4 = reinterpret_cast<float4*>(st) + c4;
#pragma unroll 4
      for (int row = r0; row < m; row += rpp) {
        float4 x = s4[(size_t)row * tpr];
        const float fk = pk[row], fq = pq[row];
        x.x = fmaf(fk, vv.x, x.x); x.y = fmaf(fk, vv.y, x.y);
        x.z = fmaf(fk, vv.z, x.z); x.w = fmaf(fk, vv.w, x.w);
        s4[(size_t)row * tpr] = x;
        num.x = fmaf(fq, x.x, num.x); num.y = fmaf(fq, x.y, num.y);
        num.z = fmaf(fq, x.z, num.z); num.w = fmaf(fq, x.w, num.w);
      }
      float* rr = red + r0 * d + 4 * c4;
      rr[0] = num.x; rr[1] = num.y; rr[2] = num.z; rr[3] = num.w;
    }
    float den = 0.f;
    for (int jj = tid; jj < m; jj += kStreamThreads) {
      const float zj = zs[jj] + pk[jj];
      zs[jj] = zj;
      den = fmaf(pq[jj], zj, den);
    }
    den = warp_sum(den);
    if (lane == 0) scratch[warp] = den;
    tc::fence_async_smem();           // the state writes above, for the bulk store
    __syncthreads();
    if (tid == 0) {
      const uint32_t kvb = (uint32_t)m * d * 4;
      const uint32_t src = tc::smem_u32(st);
      for (uint32_t o = 0; o < kvb; o += 32768)
        asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(
                         reinterpret_cast<uint8_t*>(kv + (size_t)bh * m * d) + o),
                     "r"(src + o), "r"(kvb - o < 32768 ? kvb - o : 32768)
                     : "memory");
      asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(
                       z + (size_t)bh * m),
                   "r"(src + kvb), "r"((uint32_t)m * 4)
                   : "memory");
      asm volatile("cp.async.bulk.commit_group;" ::: "memory");
    }
    float dtot = 0.f;
#pragma unroll
    for (int u = 0; u < kStreamThreads / 32; ++u) dtot += scratch[u];
    for (int c = tid; c < d; c += kStreamThreads) {
      float acc = 0.f;
      for (int g = 0; g < rpp; ++g) acc += red[g * d + c];
      const float o = dtot > 0.f ? acc / dtot : 0.f;
      if (!isfinite(o)) report(dev_status, DARK_ERR_NUMERIC);
      out[(size_t)bh * d + c] = __float2bfloat16_rn(o);
    }
    __syncthreads();                   // red, scratch and pk/pq are reused by the next item
  }
  if (!ok && tid == 0) {
    report(dev_status, DARK_ERR_TIMEOUT);
    // no copy may land after the block is gone (a completed phase passes at once)
    for (int bb = 0; bb < 2; ++bb) {
      if (s_last[bb] >= 0) tc::mbar_wait(bar_s + bb, (s_last[bb] >> 1) & 1);
      if (w_loads[bb] > 0) tc::mbar_wait(bar_w + bb, (w_loads[bb] - 1) & 1);
    }
  }
  if (tid == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}
}  // namespace

cudaError_t launch_decode(const DecodeArgs& a) {
  // the streaming kernel when the heads outnumber the SMs and two states and
  // two W' copies fit in shared memory
  if (a.dtype == DARK_BF16 && a.shift == nullptr && a.update == 1 && a.d % 8 == 0 && a.d <= 256 &&
      a.m % 4 == 0 && a.B * a.H >= 2 * num_sms() && ((uintptr_t)a.w & 15) == 0 &&
      ((uintptr_t)a.kv & 15) == 0 && ((uintptr_t)a.z & 15) == 0) {
    const StreamLayout L = stream_layout(a.m, a.r, a.d);
    if (L.total <= 227 * 1024 && L.wbytes % 16 == 0 && (a.m * 4) % 16 == 0) {
      static int done[64];
      cudaError_t err = set_smem_limit_once((const void*)decode_stream_kernel, (int)L.total, done);
      if (err != cudaSuccess) return err;
      const int n = a.B * a.H, grid = n < num_sms() ? n : num_sms();
      decode_stream_kernel<<<grid, kStreamThreads, L.total, a.stream>>>(
          (const __half*)a.w, a.heads_w, a.m, a.r, a.d, a.kv, a.z, a.B, a.H,
          (const __nv_bfloat16*)a.q, (const __nv_bfloat16*)a.k, (const __nv_bfloat16*)a.v,
          (__nv_bfloat16*)a.out, a.valid, a.dev_status, n);
      return cudaGetLastError();
    }
  }
  const int tpr = a.d / 4;
  const int rpp = kThreads / tpr;
  const size_t welt = a.dtype == DARK_BF16 ? sizeof(__half) : sizeof(float);
  const size_t w_bytes = (size_t)(a.m + a.r) * a.d * welt;
  // staged W': each head's rows 16-byte aligned for the bulk copy, and rows of
  // a multiple of 8 elements (the 8-lane GEMV, the only one reading it there)
  const int stage_w = w_bytes <= kStageW && w_bytes % 16 == 0 && a.d % 8 == 0 &&
                      ((uintptr_t)a.w & 15) == 0;
  const size_t tail = (sizeof(float) * (3 * a.d + (a.m + a.r) + a.m + rpp * a.d + 32) + 15) / 16 * 16;
  const size_t smem = tail + (stage_w ? 16 + w_bytes : 0);
  // one opt-in per device that covers every size: at most 4128 floats of
  // vectors and partial sums (d <= 256, m <= 1024, r <= 256) plus staged W'
  constexpr int kSmemOptIn = 96 * 1024;
  cudaError_t err;
  if (a.dtype == DARK_BF16) {
    static int done[64];
    err = set_smem_limit_once((const void*)decode_kernel<__nv_bfloat16>, kSmemOptIn, done);
    if (err != cudaSuccess) return err;
    decode_kernel<__nv_bfloat16><<<a.B * a.H, kThreads, smem, a.stream>>>(
        (const __half*)a.w, a.heads_w, a.m, a.r, a.d, a.kv, a.z, a.shift, a.H,
        (const __nv_bfloat16*)a.q, (const __nv_bfloat16*)a.k, (const __nv_bfloat16*)a.v,
        (__nv_bfloat16*)a.out, a.valid, a.dev_status, stage_w, a.update);
  } else {
    static int done[64];
    err = set_smem_limit_once((const void*)decode_kernel<float>, kSmemOptIn, done);
    if (err != cudaSuccess) return err;
    decode_kernel<float><<<a.B * a.H, kThreads, smem, a.stream>>>(
        (const float*)a.w, a.heads_w, a.m, a.r, a.d, a.kv, a.z, a.shift, a.H, (const float*)a.q,
        (const float*)a.k, (const float*)a.v, (float*)a.out, a.valid, a.dev_status, stage_w,
        a.update);
  }
  return cudaGetLastError();
}

}  // namespace dark
