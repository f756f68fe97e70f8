// Backward pass of PRF self-attention (non-causal or causal, key-masked):
// gradients of sum(dout * out) with respect to q, k, v and the geometry M.
//
// DARKformer README, section "Kernel": M is the learned factor of Sigma = M^T M
// and Omega is a fixed draw (it gets no gradient); phi(x)_j =
// m^{-1/2} exp(omega_j^T M x~ - 1/2 |M x~|^2), x~ = d^{-1/4} x, and
// out = Phi(Q)(Phi(K)^T V) / Phi(Q)(Phi(K)^T 1). Section "Self-attention" gives
// the key mask and the causal constraint.
//
// The chain rule in the associative order (never an L x L matrix beyond one
// 64 x 64 tile of the causal diagonal). For query i and the key statistics
// S_i, z_i it sees, with g_i = dout_i:
//   w_i = g_i / den_i,  c_i = (g_i . o_i) / den_i,
//   dphi(q_i) = S_i w_i - z_i c_i,
//   dS (key j) = sum of phi(q_i) [w_i | -c_i]^T over the queries that see j,
//   dv_j = dS_j[:, :d]^T phi(k_j),  dphi(k_j) = dS_j [v_j ; 1].
// Through the base-2 exponents E2 = (W' x)_top - |(W' x)_bot|^2 of the projection
// W' = [c_w Omega M ; c_m M] (the same W' the forward uses, built here in fp32):
//   dE2 = ln2 * phi * dphi,  coef = [dE2 ; -2 (sum_j dE2_j) (W' x)_bot],
//   dx = W'^T coef,  dW' = sum_t coef_t x_t^T,
//   dM = c_w Omega^T dW'_top + c_m dW'_bot.
// For queries sum_j dE2_j = phi(q_i) . dphi(q_i) = g_i . o_i - g_i . o_i = 0, so
// the norm term vanishes and per-query factors of phi(q) can be dropped (the
// query features are taken relative to their row maximum); a per-head key
// shift (the stabiliser) also cancels from every dE2.
//
// Kernels, all fp32 FFMA, 64-token tiles (the causal chunk is one tile):
//   features -> chunk states Phi(K_c)^T [V_c | 1] -> exclusive prefix (causal)
//   or total -> query pass (den, w, c, dphi(q)) -> chunk states
//   Phi(Q_c)^T [w | -c] -> exclusive suffix or total -> key pass (dv, dphi(k))
//   -> dx for both sides -> dW' (split over tokens, fp32 atomics) -> dM.
#include <math.h>

#include "common.cuh"
#include "internal.h"
#include "simt_tile.cuh"

namespace dark {
namespace {

constexpr int kT = 64;                          // tokens per tile (= causal chunk)
constexpr float kLn2 = 0.69314718055994530942f;
constexpr int kSms = 148;

struct BwdLayout {
  int nt;                                       // tiles per (batch, head)
  size_t off_w, off_ck, off_phiq, off_phik, off_cs, off_ds, off_wq, off_cfq, off_cfk, off_g,
      total;
};

BwdLayout bwd_layout(int B, int H, int L, int m, int r, int d, int heads_w) {
  BwdLayout s;
  const size_t bh = (size_t)B * H, dd = (size_t)d + 1, mr = (size_t)m + r;
  s.nt = (L + kT - 1) / kT;
  size_t o = kWsHeader;
  auto take = [&o](size_t bytes) {
    const size_t at = o;
    o = align_up(o + bytes, 256);
    return at;
  };
  s.off_w = take(sizeof(float) * heads_w * mr * d);
  s.off_ck = take(sizeof(int) * bh);
  s.off_phiq = take(sizeof(float) * bh * L * m);
  s.off_phik = take(sizeof(float) * bh * L * m);
  s.off_cs = take(sizeof(float) * bh * s.nt * m * dd);
  s.off_ds = take(sizeof(float) * bh * s.nt * m * dd);
  s.off_wq = take(sizeof(float) * bh * L * dd);
  s.off_cfq = take(sizeof(float) * bh * L * mr);
  s.off_cfk = take(sizeof(float) * bh * L * mr);
  s.off_g = take(sizeof(float) * heads_w * mr * d);
  s.total = o;
  return s;
}

__global__ void fill_ordered_kernel(int* p, int n, float v) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) p[i] = float_to_ordered(v);
}

// Features of one side for a tile of 64 tokens from P = x W'^T (fp32 W').
// Keys: phi = 2^(P_top - |P_bot|^2 - 1/2 log2 m), masked keys 0; with the
// stabiliser the exponent is stored (-inf when masked) and the head maximum is
// collected for a shift pass. Queries: 2^(P_top - max_j P_top).
template <typename T>
__global__ void __launch_bounds__(256) bwd_features_kernel(
    const T* __restrict__ xq, const T* __restrict__ xk, int64_t sb, int64_t sh, int64_t sl,
    const float* __restrict__ w, int heads_w, int m, int r, int d, int H, int L,
    const uint8_t* __restrict__ mask, int stabilise, float* __restrict__ phiq,
    float* __restrict__ phik, int* __restrict__ ck) {
  __shared__ __align__(16) float Xs[32 * kLd];
  __shared__ __align__(16) float Ws[32 * kLd];
  __shared__ float rowc[kT];
  __shared__ int rowmax[kT];
  const int side = blockIdx.z;
  const int bh = blockIdx.y, b = bh / H, h = bh % H;
  const int t0 = blockIdx.x * kT;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const T* x = (side ? xk : xq) + (int64_t)b * sb + (int64_t)h * sh;
  const float* wh = w + (size_t)(heads_w == 1 ? 0 : h) * (m + r) * d;
  float* dst = (side ? phik : phiq) + (size_t)bh * L * m;
  for (int i = threadIdx.x; i < kT; i += blockDim.x) {
    rowc[i] = side ? 0.5f * log2f((float)m) : 0.f;
    rowmax[i] = float_to_ordered(-INFINITY);
  }
  __syncthreads();

  auto tile = [&](int c0, float (&acc)[4][4]) {
    zero(acc);
    for (int k0 = 0; k0 < d; k0 += 32) {
      stage_t(Xs, [&](int t, int kk) {
        return (t0 + t < L && k0 + kk < d) ? to_f32(x[(int64_t)(t0 + t) * sl + k0 + kk]) : 0.f;
      });
      stage_t(Ws, [&](int j, int kk) {
        return (c0 + j < m + r && k0 + kk < d) ? wh[(size_t)(c0 + j) * d + k0 + kk] : 0.f;
      });
      __syncthreads();
      fma_tile(Xs, Ws, acc);
      __syncthreads();
    }
  };

  float acc[4][4];
  if (side) {
    for (int c0 = m; c0 < m + r; c0 += 64) {
      tile(c0, acc);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float s = 0.f;
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (c0 + tx * 4 + j < m + r) s = fmaf(acc[i][j], acc[i][j], s);
        atomicAdd(&rowc[ty * 4 + i], s);
      }
    }
    __syncthreads();
  }
  float kmax = -INFINITY;
  for (int c0 = 0; c0 < m; c0 += 64) {
    tile(c0, acc);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int row = ty * 4 + i, t = t0 + row;
      if (t >= L) continue;
      const bool ok = !side || mask == nullptr || mask[(size_t)b * L + t] != 0;
      float rmax = -INFINITY;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int f = c0 + tx * 4 + j;
        if (f >= m) continue;
        const float e = acc[i][j] - rowc[row];
        float val;
        if (!side) {
          val = e;
          rmax = fmaxf(rmax, e);
        } else if (!ok) {
          val = stabilise ? -INFINITY : 0.f;
        } else if (stabilise) {
          val = e;
          kmax = fmaxf(kmax, e);
        } else {
          val = exp2f(e);
        }
        dst[(size_t)t * m + f] = val;
      }
      if (!side && rmax > -INFINITY) atomicMax(&rowmax[row], float_to_ordered(rmax));
    }
  }
  if (side) {
    if (stabilise) {
      kmax = warp_max(kmax);
      if ((threadIdx.x & 31) == 0 && kmax > -INFINITY) atomicMax(&ck[bh], float_to_ordered(kmax));
    }
    return;
  }
  __syncthreads();                  // this block's exponents are visible to all its threads
  for (int e = threadIdx.x; e < kT * m; e += blockDim.x) {
    const int row = e / m, f = e % m, t = t0 + row;
    if (t >= L) continue;
    float* p = dst + (size_t)t * m + f;
    *p = exp2f(*p - ordered_to_float(rowmax[row]));
  }
}

// Stabilised keys: phi = 2^(e - c_K) with c_K the largest valid key exponent of the head.
__global__ void bwd_shift_keys_kernel(float* __restrict__ phik, const int* __restrict__ ck,
                                      int L, int m, size_t n) {
  const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const int bh = (int)(i / ((size_t)L * m));
  const float e = phik[i];
  float c = ordered_to_float(ck[bh]);
  if (!(c > -INFINITY)) c = 0.f;
  phik[i] = e == -INFINITY ? 0.f : exp2f(e - c);
}

// Second operand of a chunk state: [v_t | 1] of the keys, or the rows [w_t | -c_t]
// the query pass wrote.
template <typename T>
struct ValuesOnes {
  const T* v;
  int64_t sb, sh, sl;
  int H, d;
  __device__ float operator()(int bh, int t, int e) const {
    if (e < d) return to_f32(v[(int64_t)(bh / H) * sb + (int64_t)(bh % H) * sh + (int64_t)t * sl + e]);
    return e == d ? 1.f : 0.f;
  }
};
struct StoredRows {
  const float* p;
  int L, dd;
  __device__ float operator()(int bh, int t, int e) const {
    return e < dd ? p[((size_t)bh * L + t) * dd + e] : 0.f;
  }
};

// Per tile of tokens: st_c = A_c^T U_c, [m][d + 1], A = feature rows [L][m].
template <class U>
__global__ void __launch_bounds__(256) chunk_state_kernel(const float* __restrict__ A, U u, int m,
                                                          int d, int L, int nt,
                                                          float* __restrict__ st) {
  __shared__ __align__(16) float As[32 * kLd];
  __shared__ __align__(16) float Bs[32 * kLd];
  const int c = blockIdx.x, bh = blockIdx.y;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int dd = d + 1;
  const int tb = c * kT, te = min(L, tb + kT);
  const float* a = A + (size_t)bh * L * m;
  float* out = st + ((size_t)bh * nt + c) * m * dd;
  for (int f0 = 0; f0 < m; f0 += 64) {
    for (int e0 = 0; e0 < dd; e0 += 64) {
      float acc[4][4];
      zero(acc);
      for (int k0 = tb; k0 < te; k0 += 32) {
        stage_n(As, [&](int kk, int f) {
          const int t = k0 + kk;
          return (t < te && f0 + f < m) ? a[(size_t)t * m + f0 + f] : 0.f;
        });
        stage_n(Bs, [&](int kk, int col) {
          const int t = k0 + kk;
          return t < te ? u(bh, t, e0 + col) : 0.f;
        });
        __syncthreads();
        fma_tile(As, Bs, acc);
        __syncthreads();
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int f = f0 + ty * 4 + i;
        if (f >= m) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int e = e0 + tx * 4 + j;
          if (e < dd) out[(size_t)f * dd + e] = acc[i][j];
        }
      }
    }
  }
}

// mode 0: exclusive prefix over tiles (causal forward statistics); 1: exclusive
// suffix (causal gradient statistics); 2: total into tile 0 (non-causal).
// Sixteen tiles' values are loaded before any is stored, so the loads overlap.
__global__ void tile_scan_kernel(float* __restrict__ st, int n, int nt, int mode) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= n) return;
  float* base = st + (size_t)blockIdx.y * nt * n + idx;
  float run = 0.f;
  for (int s0 = 0; s0 < nt; s0 += 16) {
    float v[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int s = s0 + u, c = mode == 1 ? nt - 1 - s : s;
      v[u] = s < nt ? base[(size_t)c * n] : 0.f;
    }
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int s = s0 + u, c = mode == 1 ? nt - 1 - s : s;
      if (s < nt && mode != 2) base[(size_t)c * n] = run;
      run += v[u];
    }
  }
  if (mode == 2) base[0] = run;
}

// One tile of 64 tokens of one side. SIDE 0 (queries): X = Phi(Q), Y = Phi(K),
// state = S over earlier tiles (or all keys), U = [v | 1]; phase 1 gives
// [num | den], from which w, c and P = [w | -c] (also stored for the key side).
// SIDE 1 (keys): X = Phi(K), Y = Phi(Q), state = dS over later tiles (or all
// queries), U = [w | -c]; phase 1 gives dv; P = [v | 1]. Phase 2 on both sides:
// dphi(X) = P state^T + tri(P U^T) Y, then coef = ln2 * X * dphi.
// tri keeps key <= query within the tile (causal only). ET = ceil((d + 1) / 64)
// column blocks of [num | den] per thread.
template <typename T, int SIDE, int ET>
__global__ void __launch_bounds__(256, ET <= 3 ? 2 : 1) pass_kernel(
    const float* __restrict__ phiq, const float* __restrict__ phik,
    const float* __restrict__ state, const T* __restrict__ v, int64_t vb, int64_t vh, int64_t vl,
    const T* __restrict__ g, int64_t gb, int64_t gh, int64_t gl, float* __restrict__ wq,
    T* __restrict__ dv, int64_t ob, int64_t oh, int64_t ol, float* __restrict__ coef, int m,
    int r, int d, int H, int L, int nt, int causal, int* dev_status) {
  extern __shared__ __align__(16) float sm[];
  constexpr int ddp = ET * 64;
  const int dd = d + 1;
  float* Xk = sm;                 // [32][kLd]  A staging
  float* Yk = Xk + 32 * kLd;      // [32][kLd]  B staging
  float* ScT = Yk + 32 * kLd;     // [64 k][kLd] masked tile of X Y^T, then of P U^T (k-major)
  float* Bt = ScT + 64 * kLd;     // [32][ddp]  phase-1 B operand (state rows, U rows)
  float* PsT = Bt + 32 * ddp;     // [ddp][kLd] P, k-major
  float* rowv = PsT + ddp * kLd;  // [64]
  const int c = blockIdx.x, bh = blockIdx.y, b = bh / H, h = bh % H;
  const int t0 = c * kT;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const float* X = (SIDE == 0 ? phiq : phik) + (size_t)bh * L * m;
  const float* Y = (SIDE == 0 ? phik : phiq) + (size_t)bh * L * m;
  const float* st = state + ((size_t)bh * nt + (causal ? c : 0)) * m * dd;
  float* wrow = wq + (size_t)bh * L * dd;
  const T* vh_ = v + (int64_t)b * vb + (int64_t)h * vh;

  auto U = [&](int t, int e) -> float {
    if (t >= L || e >= dd) return 0.f;
    if (SIDE == 0) return e < d ? to_f32(vh_[(int64_t)t * vl + e]) : 1.f;
    return wrow[(size_t)t * dd + e];
  };
  auto keep = [](int row, int col) { return SIDE == 0 ? col <= row : col >= row; };
  // masked 64 x 64 tile from registers into ScT[col][row] (k-major for the next GEMM)
  auto store_masked = [&](const float (&s4)[4][4]) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int col = tx * 4 + j;
      float4 o;
      o.x = keep(ty * 4 + 0, col) ? s4[0][j] : 0.f;
      o.y = keep(ty * 4 + 1, col) ? s4[1][j] : 0.f;
      o.z = keep(ty * 4 + 2, col) ? s4[2][j] : 0.f;
      o.w = keep(ty * 4 + 3, col) ? s4[3][j] : 0.f;
      *reinterpret_cast<float4*>(ScT + col * kLd + ty * 4) = o;
    }
  };

  // ---- phase 1: acc = X state + tri(X Y^T) U ----
  float acc[ET][4][4];
#pragma unroll
  for (int et = 0; et < ET; ++et)
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[et][i][j] = 0.f;
  auto acc_from = [&](const float* A) {   // acc += A[32 k][64 rows] (k-major) Bt[32][ddp]
#pragma unroll 4
    for (int kk = 0; kk < 32; ++kk) {
      const float4 a4 = ld4(A + kk * kLd + ty * 4);
      const float a[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
      for (int et = 0; et < ET; ++et) {
        const float4 b4 = ld4(Bt + kk * ddp + et * 64 + tx * 4);
        const float bb[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[et][i][j] = fmaf(a[i], bb[j], acc[et][i][j]);
      }
    }
  };
  float s4[4][4];
  zero(s4);
  for (int f0 = 0; f0 < m; f0 += 32) {
    stage_t(Xk, [&](int i, int kk) {
      return (t0 + i < L && f0 + kk < m) ? X[(size_t)(t0 + i) * m + f0 + kk] : 0.f;
    });
    if (causal)
      stage_t(Yk, [&](int j, int kk) {
        return (t0 + j < L && f0 + kk < m) ? Y[(size_t)(t0 + j) * m + f0 + kk] : 0.f;
      });
    for (int e = threadIdx.x; e < 32 * ddp; e += blockDim.x) {
      const int kk = e / ddp, col = e % ddp;
      Bt[e] = (f0 + kk < m && col < dd) ? st[(size_t)(f0 + kk) * dd + col] : 0.f;
    }
    __syncthreads();
    acc_from(Xk);
    if (causal) fma_tile(Xk, Yk, s4);
    __syncthreads();
  }
  if (causal) {
    store_masked(s4);
    for (int k0 = 0; k0 < 64; k0 += 32) {
      for (int e = threadIdx.x; e < 32 * ddp; e += blockDim.x) {
        const int kk = e / ddp, col = e % ddp;
        Bt[e] = U(t0 + k0 + kk, col);
      }
      __syncthreads();
      acc_from(ScT + k0 * kLd);
      __syncthreads();
    }
  }

  // ---- epilogue of phase 1: P into PsT (k-major) ----
  auto put_p = [&](int row, int col, float p) { PsT[col * kLd + row] = p; };
  if (SIDE == 0) {
    // den = column d of [num | den]
#pragma unroll
    for (int et = 0; et < ET; ++et)
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (et * 64 + tx * 4 + j == d) {
#pragma unroll
          for (int i = 0; i < 4; ++i) rowv[ty * 4 + i] = acc[et][i][j];
        }
    __syncthreads();
    const T* gh_ = g + (int64_t)b * gb + (int64_t)h * gh;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int row = ty * 4 + i, t = t0 + row;
      const float den = rowv[row];
      const float inv = (t < L && den > 0.f) ? 1.f / den : 0.f;
      float gv[ET][4];
      float go = 0.f;
#pragma unroll
      for (int et = 0; et < ET; ++et)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int col = et * 64 + tx * 4 + j;
          gv[et][j] = (col < d && t < L) ? to_f32(gh_[(int64_t)t * gl + col]) : 0.f;
          go = fmaf(gv[et][j], acc[et][i][j], go);
        }
      // the 16 threads of a row are 16 consecutive lanes
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) go += __shfl_xor_sync(0xffffffffu, go, o);
      const float cc = go * inv * inv;
#pragma unroll
      for (int et = 0; et < ET; ++et)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int col = et * 64 + tx * 4 + j;
          const float p = col < d ? gv[et][j] * inv : (col == d ? -cc : 0.f);
          put_p(row, col, p);
          if (t < L && col < dd) wrow[(size_t)t * dd + col] = p;
          if (col < dd && !isfinite(p)) report(dev_status, DARK_ERR_NUMERIC);
        }
    }
  } else {
    T* dvh = dv + (int64_t)b * ob + (int64_t)h * oh;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int row = ty * 4 + i, t = t0 + row;
#pragma unroll
      for (int et = 0; et < ET; ++et)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int col = et * 64 + tx * 4 + j;
          if (t < L && col < d) {
            const float gval = acc[et][i][j];
            if (!isfinite(gval)) report(dev_status, DARK_ERR_NUMERIC);
            dvh[(int64_t)t * ol + col] = from_f32<T>(gval);
          }
          put_p(row, col, t < L ? (col < d ? to_f32(vh_[(int64_t)t * vl + col])
                                           : (col == d ? 1.f : 0.f))
                                : 0.f);
        }
    }
  }
  __syncthreads();

  // ---- phase 2: dphi(X) = P state^T + tri(P U^T) Y ----
  if (causal) {
    zero(s4);
    for (int e0 = 0; e0 < ddp; e0 += 32) {
      stage_t(Yk, [&](int j, int kk) { return U(t0 + j, e0 + kk); });
      __syncthreads();
      fma_tile(PsT + e0 * kLd, Yk, s4);
      __syncthreads();
    }
    store_masked(s4);
    __syncthreads();
  }
  const int mr = m + r;
  float* cf = coef + (size_t)bh * L * mr;
  for (int f0 = 0; f0 < m; f0 += 64) {
    float a2[4][4];
    zero(a2);
    for (int e0 = 0; e0 < ddp; e0 += 32) {
      stage_t(Yk, [&](int f, int kk) {
        return (f0 + f < m && e0 + kk < dd) ? st[(size_t)(f0 + f) * dd + e0 + kk] : 0.f;
      });
      __syncthreads();
      fma_tile(PsT + e0 * kLd, Yk, a2);
      __syncthreads();
    }
    if (causal) {
      for (int k0 = 0; k0 < 64; k0 += 32) {
        stage_n(Yk, [&](int kk, int f) {
          const int t = t0 + k0 + kk;
          return (t < L && f0 + f < m) ? Y[(size_t)t * m + f0 + f] : 0.f;
        });
        __syncthreads();
        fma_tile(ScT + k0 * kLd, Yk, a2);
        __syncthreads();
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int t = t0 + ty * 4 + i;
      if (t >= L) continue;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int f = f0 + tx * 4 + j;
        if (f < m) cf[(size_t)t * mr + f] = kLn2 * X[(size_t)t * m + f] * a2[i][j];
      }
    }
  }
}

// dx = W'^T coef for a tile of 64 tokens of one side. Keys first complete coef
// with the norm part -2 (sum_j dE2_j) (W' x)_bot; for queries that part is 0.
template <typename T>
__global__ void __launch_bounds__(256) dx_kernel(
    const T* __restrict__ xq, const T* __restrict__ xk, int64_t sb, int64_t sh, int64_t sl,
    const float* __restrict__ w, int heads_w, int m, int r, int d, int H, int L,
    float* __restrict__ cfq, float* __restrict__ cfk, T* __restrict__ dq, T* __restrict__ dk,
    int64_t ob, int64_t oh, int64_t ol, int* dev_status) {
  __shared__ __align__(16) float As[32 * kLd];
  __shared__ __align__(16) float Bs[32 * kLd];
  __shared__ float rsum[kT];
  const int side = blockIdx.z;
  const int bh = blockIdx.y, b = bh / H, h = bh % H;
  const int t0 = blockIdx.x * kT;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int mr = m + r;
  const T* x = (side ? xk : xq) + (int64_t)b * sb + (int64_t)h * sh;
  const float* wh = w + (size_t)(heads_w == 1 ? 0 : h) * mr * d;
  float* cf = (side ? cfk : cfq) + (size_t)bh * L * mr;
  float acc[4][4];
  if (side) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int row = warp; row < kT; row += 8) {
      const int t = t0 + row;
      float s = 0.f;
      if (t < L)
        for (int f = lane; f < m; f += 32) s += cf[(size_t)t * mr + f];
      s = warp_sum(s);
      if (lane == 0) rsum[row] = s;
    }
    __syncthreads();
    for (int c0 = 0; c0 < r; c0 += 64) {
      zero(acc);
      for (int k0 = 0; k0 < d; k0 += 32) {
        stage_t(As, [&](int i, int kk) {
          return (t0 + i < L && k0 + kk < d) ? to_f32(x[(int64_t)(t0 + i) * sl + k0 + kk]) : 0.f;
        });
        stage_t(Bs, [&](int i, int kk) {
          return (c0 + i < r && k0 + kk < d) ? wh[(size_t)(m + c0 + i) * d + k0 + kk] : 0.f;
        });
        __syncthreads();
        fma_tile(As, Bs, acc);
        __syncthreads();
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int row = ty * 4 + i, t = t0 + row;
        if (t >= L) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int col = c0 + tx * 4 + j;
          if (col < r) cf[(size_t)t * mr + m + col] = -2.f * rsum[row] * acc[i][j];
        }
      }
    }
  } else {
    for (int e = threadIdx.x; e < kT * r; e += blockDim.x) {
      const int row = e / r, col = e % r, t = t0 + row;
      if (t < L) cf[(size_t)t * mr + m + col] = 0.f;
    }
  }
  __syncthreads();                  // this block's coef rows are visible to all its threads
  const int kend = side ? mr : m;
  T* out = (side ? dk : dq) + (int64_t)b * ob + (int64_t)h * oh;
  for (int c0 = 0; c0 < d; c0 += 64) {
    zero(acc);
    for (int k0 = 0; k0 < kend; k0 += 32) {
      stage_t(As, [&](int i, int kk) {
        return (t0 + i < L && k0 + kk < kend) ? cf[(size_t)(t0 + i) * mr + k0 + kk] : 0.f;
      });
      stage_n(Bs, [&](int kk, int cc) {
        return (k0 + kk < kend && c0 + cc < d) ? wh[(size_t)(k0 + kk) * d + c0 + cc] : 0.f;
      });
      __syncthreads();
      fma_tile(As, Bs, acc);
      __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int t = t0 + ty * 4 + i;
      if (t >= L) continue;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int col = c0 + tx * 4 + j;
        if (col >= d) continue;
        if (!isfinite(acc[i][j])) report(dev_status, DARK_ERR_NUMERIC);
        out[(int64_t)t * ol + col] = from_f32<T>(acc[i][j]);
      }
    }
  }
}

// dW'[hw] += sum over a token range of one (batch, head), both sides, of
// coef_t x_t^T; a 64 x 64 tile of [m + r][d] per block, fp32 atomics at the end.
template <typename T>
__global__ void __launch_bounds__(256) dw_kernel(
    const T* __restrict__ xq, const T* __restrict__ xk, int64_t sb, int64_t sh, int64_t sl,
    const float* __restrict__ cfq, const float* __restrict__ cfk, int m, int r, int d, int H,
    int L, int heads_w, int nsplit, float* __restrict__ G) {
  __shared__ __align__(16) float As[32 * kLd];
  __shared__ __align__(16) float Bs[32 * kLd];
  const int mr = m + r;
  const int j0 = blockIdx.x * 64, c0 = blockIdx.y * 64;
  const int bh = blockIdx.z / nsplit, split = blockIdx.z % nsplit;
  const int b = bh / H, h = bh % H;
  const int per = ((L + nsplit - 1) / nsplit + 31) / 32 * 32;
  const int tb = split * per, te = min(L, tb + per);
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4];
  zero(acc);
  for (int side = 0; side < 2; ++side) {
    const T* x = (side ? xk : xq) + (int64_t)b * sb + (int64_t)h * sh;
    const float* cf = (side ? cfk : cfq) + (size_t)bh * L * mr;
    for (int k0 = tb; k0 < te; k0 += 32) {
      stage_n(As, [&](int kk, int f) {
        const int t = k0 + kk;
        return (t < te && j0 + f < mr) ? cf[(size_t)t * mr + j0 + f] : 0.f;
      });
      stage_n(Bs, [&](int kk, int f) {
        const int t = k0 + kk;
        return (t < te && c0 + f < d) ? to_f32(x[(int64_t)t * sl + c0 + f]) : 0.f;
      });
      __syncthreads();
      fma_tile(As, Bs, acc);
      __syncthreads();
    }
  }
  float* gh = G + (size_t)(heads_w == 1 ? 0 : h) * mr * d;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int j = j0 + ty * 4 + i;
    if (j >= mr) continue;
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      const int col = c0 + tx * 4 + jj;
      if (col < d) atomicAdd(&gh[(size_t)j * d + col], acc[i][jj]);
    }
  }
}

// dM[hm] = sum over the projection heads hw that use M_hm of
// c_w Omega_hw^T dW'_top[hw] + c_m dW'_bot[hw]: a 16 x 64 block of dM per CTA,
// Omega columns and dW' rows staged 32 features at a time.
__global__ void __launch_bounds__(256) dgeom_kernel(
    const float* __restrict__ G, const float* __restrict__ omega, int heads_omega,
    int heads_geom, int heads_w, int m, int r, int d, float cw, float cm,
    float* __restrict__ dgeom) {
  __shared__ float Os[32][17];
  __shared__ __align__(16) float Gs[32][64];
  const int c0 = blockIdx.x * 64, i0 = blockIdx.y * 16, hm = blockIdx.z;
  const int ii = threadIdx.x >> 4, cq = threadIdx.x & 15;
  const int i = i0 + ii, c = c0 + 4 * cq;
  const int mr = m + r;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int hw = 0; hw < heads_w; ++hw) {
    if (heads_geom != 1 && hw != hm) continue;
    const float* om = omega + (size_t)(heads_omega == 1 ? 0 : hw) * m * r;
    const float* g = G + (size_t)hw * mr * d;
    float s4[4] = {0.f, 0.f, 0.f, 0.f};
    for (int j0 = 0; j0 < m; j0 += 32) {
      for (int e = threadIdx.x; e < 32 * 16; e += blockDim.x) {
        const int jj = e >> 4, i2 = e & 15;
        Os[jj][i2] = (j0 + jj < m && i0 + i2 < r) ? om[(size_t)(j0 + jj) * r + i0 + i2] : 0.f;
      }
      for (int e = threadIdx.x; e < 32 * 64; e += blockDim.x) {
        const int jj = e >> 6, c2 = e & 63;
        Gs[jj][c2] = (j0 + jj < m && c0 + c2 < d) ? g[(size_t)(j0 + jj) * d + c0 + c2] : 0.f;
      }
      __syncthreads();
#pragma unroll 8
      for (int jj = 0; jj < 32; ++jj) {
        const float o = Os[jj][ii];
        const float4 g4 = *reinterpret_cast<const float4*>(&Gs[jj][4 * cq]);
        s4[0] = fmaf(o, g4.x, s4[0]);
        s4[1] = fmaf(o, g4.y, s4[1]);
        s4[2] = fmaf(o, g4.z, s4[2]);
        s4[3] = fmaf(o, g4.w, s4[3]);
      }
      __syncthreads();
    }
    if (i < r)
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (c + u < d) acc[u] += cw * s4[u] + cm * g[(size_t)(m + i) * d + c + u];
  }
  if (i < r)
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (c + u < d) dgeom[((size_t)hm * r + i) * d + c + u] = acc[u];
}

size_t pass_smem_bytes(int et) {
  const int ddp = et * 64;
  return sizeof(float) * (32 * kLd * 2 + 64 * kLd + 32 * ddp + ddp * kLd + 64);
}

struct PassArgs {
  const float *phiq, *phik, *state;
  const void* v;
  int64_t vb, vh, vl;
  const void* g;
  int64_t gb, gh, gl;
  float* wq;
  void* dv;
  int64_t ob, oh, ol;
  float* coef;
  int m, r, d, H, L, nt, causal;
  int* dev_status;
};

template <typename T, int SIDE, int ET>
cudaError_t launch_pass_et(const PassArgs& p, dim3 grid, cudaStream_t stream) {
  static int smem_set[64];
  const size_t bytes = pass_smem_bytes(ET);
  cudaError_t err = set_smem_limit_once((const void*)pass_kernel<T, SIDE, ET>, (int)bytes, smem_set);
  if (err != cudaSuccess) return err;
  pass_kernel<T, SIDE, ET><<<grid, 256, bytes, stream>>>(
      p.phiq, p.phik, p.state, (const T*)p.v, p.vb, p.vh, p.vl, (const T*)p.g, p.gb, p.gh, p.gl,
      p.wq, (T*)p.dv, p.ob, p.oh, p.ol, p.coef, p.m, p.r, p.d, p.H, p.L, p.nt, p.causal,
      p.dev_status);
  return cudaGetLastError();
}

// ET = ceil((d + 1) / 64) column blocks; d <= 256 gives at most 5.
template <typename T, int SIDE>
cudaError_t launch_pass(const PassArgs& p, dim3 grid, cudaStream_t stream) {
  switch ((p.d + 1 + 63) / 64) {
    case 1: return launch_pass_et<T, SIDE, 1>(p, grid, stream);
    case 2: return launch_pass_et<T, SIDE, 2>(p, grid, stream);
    case 3: return launch_pass_et<T, SIDE, 3>(p, grid, stream);
    case 4: return launch_pass_et<T, SIDE, 4>(p, grid, stream);
    case 5: return launch_pass_et<T, SIDE, 5>(p, grid, stream);
    default: return cudaErrorInvalidValue;
  }
}

template <typename T>
cudaError_t backward_t(const BwdArgs& a) {
  const BwdLayout s = bwd_layout(a.B, a.H, a.L, a.m, a.r, a.d, a.heads_w);
  char* ws = (char*)a.ws;
  float* wf = (float*)(ws + s.off_w);
  int* ck = (int*)(ws + s.off_ck);
  float* phiq = (float*)(ws + s.off_phiq);
  float* phik = (float*)(ws + s.off_phik);
  float* cs = (float*)(ws + s.off_cs);
  float* dsn = (float*)(ws + s.off_ds);
  float* wq = (float*)(ws + s.off_wq);
  float* cfq = (float*)(ws + s.off_cfq);
  float* cfk = (float*)(ws + s.off_cfk);
  float* G = (float*)(ws + s.off_g);
  const int bh = a.B * a.H, m = a.m, r = a.r, d = a.d, L = a.L, nt = s.nt;
  const int stab = (a.flags & DARK_STABILISE) ? 1 : 0;
  const int causal = (a.flags & DARK_CAUSAL) ? 1 : 0;
  const T* q = (const T*)a.q;
  const T* k = (const T*)a.k;
  const T* v = (const T*)a.v;
  cudaError_t err;

  err = launch_projection(a.omega, a.heads_omega, a.geom, a.heads_geom, a.heads_w, m, r, d,
                          DARK_F32, wf, a.stream);
  if (err != cudaSuccess) return err;
  if (stab) fill_ordered_kernel<<<(bh + 255) / 256, 256, 0, a.stream>>>(ck, bh, -INFINITY);
  bwd_features_kernel<T><<<dim3(nt, bh, 2), 256, 0, a.stream>>>(
      q, k, a.xs[0], a.xs[1], a.xs[2], wf, a.heads_w, m, r, d, a.H, L, a.mask, stab, phiq, phik,
      ck);
  if (stab) {
    const size_t n = (size_t)bh * L * m;
    bwd_shift_keys_kernel<<<(unsigned)((n + 255) / 256), 256, 0, a.stream>>>(phik, ck, L, m, n);
  }
  const int n_st = m * (d + 1);
  const dim3 scan_grid((n_st + 255) / 256, bh);
  chunk_state_kernel<ValuesOnes<T>><<<dim3(nt, bh), 256, 0, a.stream>>>(
      phik, ValuesOnes<T>{v, a.xs[0], a.xs[1], a.xs[2], a.H, d}, m, d, L, nt, cs);
  tile_scan_kernel<<<scan_grid, 256, 0, a.stream>>>(cs, n_st, nt, causal ? 0 : 2);

  PassArgs pa{phiq, phik, cs, v, a.xs[0], a.xs[1], a.xs[2], a.dout, a.gs[0], a.gs[1], a.gs[2],
              wq, nullptr, 0, 0, 0, cfq, m, r, d, a.H, L, nt, causal, a.dev_status};
  err = launch_pass<T, 0>(pa, dim3(nt, bh), a.stream);
  if (err != cudaSuccess) return err;
  chunk_state_kernel<StoredRows><<<dim3(nt, bh), 256, 0, a.stream>>>(
      phiq, StoredRows{wq, L, d + 1}, m, d, L, nt, dsn);
  tile_scan_kernel<<<scan_grid, 256, 0, a.stream>>>(dsn, n_st, nt, causal ? 1 : 2);
  pa.state = dsn;
  pa.g = nullptr;
  pa.gb = pa.gh = pa.gl = 0;
  pa.dv = a.dv;
  pa.ob = a.ds[0];
  pa.oh = a.ds[1];
  pa.ol = a.ds[2];
  pa.coef = cfk;
  err = launch_pass<T, 1>(pa, dim3(nt, bh), a.stream);
  if (err != cudaSuccess) return err;
  dx_kernel<T><<<dim3(nt, bh, 2), 256, 0, a.stream>>>(
      q, k, a.xs[0], a.xs[1], a.xs[2], wf, a.heads_w, m, r, d, a.H, L, cfq, cfk, (T*)a.dq,
      (T*)a.dk, a.ds[0], a.ds[1], a.ds[2], a.dev_status);
  if (a.dgeom != nullptr) {
    err = cudaMemsetAsync(G, 0, sizeof(float) * (size_t)a.heads_w * (m + r) * d, a.stream);
    if (err != cudaSuccess) return err;
    const int tiles = ((m + r + 63) / 64) * ((d + 63) / 64);
    int nsplit = (4 * kSms + tiles * bh - 1) / (tiles * bh);
    const int max_split = (L + 127) / 128;
    if (nsplit > max_split) nsplit = max_split;
    if (nsplit < 1) nsplit = 1;
    dw_kernel<T><<<dim3((m + r + 63) / 64, (d + 63) / 64, bh * nsplit), 256, 0, a.stream>>>(
        q, k, a.xs[0], a.xs[1], a.xs[2], cfq, cfk, m, r, d, a.H, L, a.heads_w, nsplit, G);
    const double sc = pow((double)d, -0.25);
    dgeom_kernel<<<dim3((d + 63) / 64, (r + 15) / 16, a.heads_geom), 256, 0, a.stream>>>(
        G, a.omega, a.heads_omega, a.heads_geom, a.heads_w, m, r, d, (float)(sc * kLog2e),
        (float)(sc * sqrt(0.5 * kLog2e)), a.dgeom);
  }
  return cudaGetLastError();
}

}  // namespace

size_t bwd_workspace_bytes(int B, int H, int L, int m, int r, int d, int heads_w) {
  const size_t simt = bwd_layout(B, H, L, m, r, d, heads_w).total;
  const size_t tc = tc_bwd_workspace_bytes(B, H, L, m, r, d, heads_w);
  return simt > tc ? simt : tc;
}

cudaError_t launch_backward(const BwdArgs& a) {
  if (tc_backward_supported(a)) return launch_backward_tc(a);
  return a.dtype == DARK_BF16 ? backward_t<__nv_bfloat16>(a) : backward_t<float>(a);
}

// Steps shared with the tensor-core backward (tc_backward.cu).
cudaError_t bwd_fill_ordered(int* p, int n, float v, cudaStream_t s) {
  fill_ordered_kernel<<<(n + 255) / 256, 256, 0, s>>>(p, n, v);
  return cudaGetLastError();
}
cudaError_t bwd_shift_keys(float* phik, const int* ck, int L, int m, size_t n, cudaStream_t s) {
  bwd_shift_keys_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(phik, ck, L, m, n);
  return cudaGetLastError();
}
cudaError_t bwd_tile_scan(float* st, int n, int nt, int bh, int mode, cudaStream_t s) {
  tile_scan_kernel<<<dim3((n + 255) / 256, bh), 256, 0, s>>>(st, n, nt, mode);
  return cudaGetLastError();
}
cudaError_t bwd_dgeom(const float* G, const BwdArgs& a) {
  const double sc = pow((double)a.d, -0.25);
  dgeom_kernel<<<dim3((a.d + 63) / 64, (a.r + 15) / 16, a.heads_geom), 256, 0, a.stream>>>(
      G, a.omega, a.heads_omega, a.heads_geom, a.heads_w, a.m, a.r, a.d, (float)(sc * kLog2e),
      (float)(sc * sqrt(0.5 * kLog2e)), a.dgeom);
  return cudaGetLastError();
}

}  // namespace dark
