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
    const float part = warp_sum(feature_gemv_shared(w_sm, m, r, d, xk, xq, pk, pq));
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



// Two batch rows of one projection head per CTA, for bf16 tokens without the
// stabiliser: the rows b = 2i and 2i + 1 share the staged W' (one bulk copy)
// and the block's two feature GEMVs. The tokens load first and alone (queued
// behind the step's 34 MB of state they took several microseconds); once the
// GEMVs are done the first row's state streams into registers and the second
// row's into shared memory by bulk copies (B * H / 2 CTAs, two per SM: one wave
// for 512 heads).
struct PairLayout {
  uint32_t vec, w, st, total;     // byte offsets: vectors, W', second state; total
};
__host__ __device__ inline PairLayout pair_layout(int m, int r, int d) {
  PairLayout L;
  const int rpp = kThreads / (d / 4);
  // xq, xk, xv (2 rows), pk (2 x (m + r)), pq (2 x m), scratch [32], barriers
  L.vec = 0;
  const uint32_t vec_bytes = (uint32_t)(6 * d + 2 * (m + r) + 2 * m + 32) * 4 + 32;
  L.w = (vec_bytes + 127) / 128 * 128;
  // W' (fp16); once the GEMVs are done the same bytes hold the partial sums
  const uint32_t wb = (uint32_t)(m + r) * d * 2, red = (uint32_t)rpp * d * 4;
  L.st = L.w + ((wb > red ? wb : red) + 127) / 128 * 128;
  L.total = L.st + (uint32_t)m * d * 4;
  return L;
}

__global__ void __launch_bounds__(kThreads, 2) decode_pair_kernel(
    const __half* __restrict__ w, int heads_w, int m, int r, int d, float* __restrict__ kv,
    float* __restrict__ z, int H, const __nv_bfloat16* __restrict__ q,
    const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
    __nv_bfloat16* __restrict__ out, const uint8_t* __restrict__ valid, int* dev_status) {
  extern __shared__ __align__(128) uint8_t smp[];
  const PairLayout Lp = pair_layout(m, r, d);
  const int tpr = d / 4, rpp = kThreads / tpr, nb = m / rpp;   // nb <= kBatchRows
  float* xq = reinterpret_cast<float*>(smp + Lp.vec);           // [2][d]
  float* xk = xq + 2 * d;                                       // [2][d]
  float* xv = xk + 2 * d;                                       // [2][d]
  float* pk = xv + 2 * d;                                       // [2][m + r]
  float* pq = pk + 2 * (m + r);                                 // [2][m]
  float* scratch = pq + 2 * m;                                  // [32]
  uint64_t* bars = reinterpret_cast<uint64_t*>(scratch + 32);   // W', second state
  __half* w_sm = reinterpret_cast<__half*>(smp + Lp.w);
  float* red = reinterpret_cast<float*>(smp + Lp.w);            // after the GEMVs
  const float* st2 = reinterpret_cast<const float*>(smp + Lp.st);
  const int h = blockIdx.x % H, bp = blockIdx.x / H;
  const int bhs[2] = {(2 * bp) * H + h, (2 * bp + 1) * H + h};
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t w_bytes = (uint32_t)(m + r) * d * 2, s_bytes = (uint32_t)m * d * 4;
  if (tid == 0) {
    tc::mbar_init(bars, 1);
    tc::mbar_init(bars + 1, 1);
    tc::fence_mbar_init();
    const uint8_t* wg = reinterpret_cast<const uint8_t*>(w + (size_t)(heads_w == 1 ? 0 : h) * (m + r) * d);
    tc::mbar_arrive_expect_tx(bars, w_bytes);
    for (uint32_t o = 0; o < w_bytes; o += 16384)
      tc::bulk_load(smp + Lp.w + o, wg + o, w_bytes - o < 16384 ? w_bytes - o : 16384, bars);
  }
  const int c4 = tid % tpr, r0 = tid / tpr;
  // the tokens of both rows (they gate the feature GEMVs)
  const bool has_c = tid < d;
  if (has_c) {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      xq[i * d + tid] = __bfloat162float(q[(size_t)bhs[i] * d + tid]);
      xk[i * d + tid] = __bfloat162float(k[(size_t)bhs[i] * d + tid]);
      xv[i * d + tid] = __bfloat162float(v[(size_t)bhs[i] * d + tid]);
    }
  }
  __syncthreads();
  bool ok = tc::mbar_wait(bars, 0);
  if (__syncthreads_or(ok ? 0 : 1)) {
    if (tid == 0) {
      report(dev_status, DARK_ERR_TIMEOUT);
      tc::mbar_wait(bars, 0);        // no copy may land after the block is gone
    }
    __syncthreads();
    return;
  }
  // feature exponents of both rows from the staged W'; key norms per row
  float ks[2];
  float4 s[kBatchRows];
  float zp[2][2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const float part =
        warp_sum(feature_gemv_shared(w_sm, m, r, d, xk + i * d, xq + i * d, pk + i * (m + r),
                                     pq + i * m));
    if (lane == 0) scratch[warp] = part;
    __syncthreads();
    float nrm = 0.f;
#pragma unroll
    for (int u = 0; u < kThreads / 32; ++u) nrm += scratch[u];
    ks[i] = nrm + 0.5f * log2f((float)m);
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const bool upd = valid == nullptr || valid[bhs[i] / H] != 0;
    for (int j = tid; j < m; j += kThreads) {
      pk[i * (m + r) + j] = upd ? exp2f(pk[i * (m + r) + j] - ks[i]) : 0.f;
      pq[i * m + j] = exp2f(pq[i * m + j]);
    }
  }
  __syncthreads();                   // W' is read: its bytes now hold partial sums
  // the state, once this block's GEMVs are done: the second row's by bulk
  // copies into shared memory, the first row's into registers
  if (tid == 0) {
    const uint8_t* sg = reinterpret_cast<const uint8_t*>(kv + (size_t)bhs[1] * m * d);
    tc::mbar_arrive_expect_tx(bars + 1, s_bytes);
    for (uint32_t o = 0; o < s_bytes; o += 16384)
      tc::bulk_load(smp + Lp.st + o, sg + o, s_bytes - o < 16384 ? s_bytes - o : 16384, bars + 1);
  }
  float4* base1 = reinterpret_cast<float4*>(kv + (size_t)bhs[0] * m * d) + c4;
#pragma unroll
  for (int u = 0; u < kBatchRows; ++u)
    if (u < nb) s[u] = __ldcs(base1 + (size_t)(r0 + u * rpp) * tpr);
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int j = tid + u * kThreads;
      zp[i][u] = j < m ? __ldcs(z + (size_t)bhs[i] * m + j) : 0.f;
    }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const float* fk = pk + i * (m + r);
    const float* fq = pq + i * m;
    if (i == 1) {
      ok = tc::mbar_wait(bars + 1, 0);
      if (__syncthreads_or(ok ? 0 : 1)) {
        if (tid == 0) {
          report(dev_status, DARK_ERR_TIMEOUT);
          tc::mbar_wait(bars + 1, 0);
        }
        __syncthreads();
        return;
      }
    }
    float4* base = reinterpret_cast<float4*>(kv + (size_t)bhs[i] * m * d) + c4;
    const float4 vv = make_float4(xv[i * d + 4 * c4], xv[i * d + 4 * c4 + 1],
                                  xv[i * d + 4 * c4 + 2], xv[i * d + 4 * c4 + 3]);
    float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int u = 0; u < kBatchRows; ++u) {
      if (u >= nb) break;
      const int j = r0 + u * rpp;
      float4 x = i == 0 ? s[u] : reinterpret_cast<const float4*>(st2)[(size_t)j * tpr + c4];
      const float a = fk[j], c = fq[j];
      x.x = fmaf(a, vv.x, x.x); x.y = fmaf(a, vv.y, x.y);
      x.z = fmaf(a, vv.z, x.z); x.w = fmaf(a, vv.w, x.w);
      __stcs(base + (size_t)j * tpr, x);
      num.x = fmaf(c, x.x, num.x); num.y = fmaf(c, x.y, num.y);
      num.z = fmaf(c, x.z, num.z); num.w = fmaf(c, x.w, num.w);
    }
    float* rr = red + r0 * d + 4 * c4;
    rr[0] = num.x; rr[1] = num.y; rr[2] = num.z; rr[3] = num.w;
    float den = 0.f;
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int j = tid + u * kThreads;
      if (j < m) {
        const float zj = zp[i][u] + fk[j];
        __stcs(z + (size_t)bhs[i] * m + j, zj);
        den = fmaf(fq[j], zj, den);
      }
    }
    den = block_sum(den, scratch);   // contains the barrier that publishes `red`
    for (int c = tid; c < d; c += kThreads) {
      float acc = 0.f;
      for (int g = 0; g < rpp; ++g) acc += red[g * d + c];
      const float o = den > 0.f ? acc / den : 0.f;
      if (!isfinite(o)) report(dev_status, DARK_ERR_NUMERIC);
      out[(size_t)bhs[i] * d + c] = __float2bfloat16_rn(o);
    }
    __syncthreads();                 // red and scratch are reused by the second row
  }
}
}  // namespace

cudaError_t launch_decode(const DecodeArgs& a) {
  // two batch rows per CTA when the step's tokens are bf16 with an fp16 W' that
  // fits the staging, no stabiliser, an even batch, and every row's state in
  // one register pass
  if (a.dtype == DARK_BF16 && a.shift == nullptr && a.update == 1 && a.B % 2 == 0 &&
      a.d % 8 == 0 && a.d <= 256 && (size_t)(a.m + a.r) * a.d * 2 <= kStageW &&
      ((size_t)(a.m + a.r) * a.d * 2) % 16 == 0 && ((uintptr_t)a.w & 15) == 0 &&
      ((uintptr_t)a.kv & 15) == 0 && (a.m % (kThreads / (a.d / 4))) == 0 &&
      a.m / (kThreads / (a.d / 4)) <= kBatchRows && a.m <= 2 * kThreads) {
    const PairLayout L = pair_layout(a.m, a.r, a.d);
    if (L.total <= 227 * 1024) {
      static int done[64];
      cudaError_t err = set_smem_limit_once((const void*)decode_pair_kernel, (int)L.total, done);
      if (err != cudaSuccess) return err;
      decode_pair_kernel<<<a.B / 2 * a.H, kThreads, L.total, a.stream>>>(
          (const __half*)a.w, a.heads_w, a.m, a.r, a.d, a.kv, a.z, a.H,
          (const __nv_bfloat16*)a.q, (const __nv_bfloat16*)a.k, (const __nv_bfloat16*)a.v,
          (__nv_bfloat16*)a.out, a.valid, a.dev_status);
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
