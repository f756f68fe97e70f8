// Backward pass of PRF self-attention for bf16 I/O on the tensor cores:
// every contraction of the chain rule runs as tcgen05 MMAs of kind::tf32 on
// fp32 operands (tf32 keeps 10 explicit mantissa bits; bf16 operands would
// not hold the gradients' tolerance), with fp32 accumulators in TMEM.
//
// DARKformer README, section "Kernel": phi(x)_j = m^{-1/2} exp(omega_j^T M x~
// - 1/2 |M x~|^2), x~ = d^{-1/4} x, out = Phi(Q)(Phi(K)^T V) / Phi(Q)(Phi(K)^T 1);
// section "Self-attention" gives the key mask and the causal constraint; M is
// learned (Sigma = M^T M), Omega is a fixed draw.
//
// The chain rule is the one of the fp32 path (backward.cu) in the associative
// order, on 128-token tiles (the causal chunk is one tile). For query i with
// the key statistics S_i, z_i it sees and g_i = dout_i:
//   w_i = g_i / den_i, c_i = (g_i . o_i) / den_i, P_i = [w_i | -c_i],
//   dphi(q_i) = S_i w_i - z_i c_i = P_i [S_i | z_i]^T,
//   dv_j = sum_i phi(q_i)^T phi(k_j) w_i,  dphi(k_j) = dS_j [v_j ; 1],
//   coef = [ln2 phi dphi ; -2 (sum_j ln2 phi_j dphi_j) (W' x)_bot],
//   dx = W'^T coef, dW' = sum_t coef_t x_t^T, dM = c_w Omega^T dW'_top + c_m dW'_bot.
//
// Launches: features (P = X W'^T, exp2 epilogue) -> tile states
// Phi(K_c)^T [V_c | 1] -> exclusive prefix (causal) or total -> query pass
// ([num | den], P = [w | -c], dphi(q), coef) -> tile states Phi(Q_c)^T [w | -c]
// -> exclusive suffix or total -> key pass (dv, dphi(k), coef) -> dx -> dW'.
// Operands are staged into shared memory by the CTA's threads (tc_tf32.cuh
// layouts) through a two-slot ring: the threads fill one slot while the MMAs
// of the other run.
#include <math.h>

#include "common.cuh"
#include "internal.h"
#include "tc_tf32.cuh"

namespace dark {
namespace {

using tc::km_bytes;
using tc::mn_bytes;

constexpr int kTT = 128;                        // tokens per tile
constexpr int kWorkers = 256;                   // staging and epilogue threads (warps 0-7)
constexpr int kThr = kWorkers + 32;             // + warp 8, which issues the MMAs
constexpr float kLn2f = 0.69314718055994530942f;
constexpr int kFeatSlots = 3, kStateSlots = 4, kPassSlots = 3, kGemmSlots = 4;
// Shared memory past the ring: 16 barrier words (full, empty, drain), the
// TMEM slot and a [2][128] fp32 reduction buffer.
constexpr uint32_t kTailBytes = 160 + 2 * 128 * 4;

__host__ __device__ constexpr int round_up(int x, int a) { return (x + a - 1) / a * a; }

// The shared-memory ring of NS slots, between the workers (warps 0-7), which
// stage the operands, and warp 8, whose lane 0 issues the MMAs. Chunk i goes
// to slot i % NS. A worker arrives on full[slot] once its copies for the
// chunk have landed (fenced for the tensor cores); the MMA thread waits for
// all 256 arrivals, issues the chunk's MMAs and commits them to empty[slot],
// which the stagers of chunk i + NS wait for. Workers keep the copies of two
// chunks in flight before they signal. Every thread runs the same sequence
// of run() calls; a wait that runs out sets `failed`, which later waits skip
// and which is made uniform after each run().
template <int NS>
struct Ring {
  // a worker signals chunk i after staging chunk i + 2, which needs the MMAs
  // of chunk i + 2 - NS: NS must exceed 2
  static_assert(NS > 2, "the ring needs more slots than chunks in flight");
  uint8_t* base;
  uint32_t slot_bytes;
  uint64_t* bar;                  // full[NS], then empty[NS]
  int done;                       // chunks completed by both sides so far
  bool failed;

  __device__ uint8_t* slot(int i) const { return base + (i % NS) * slot_bytes; }
  __device__ uint64_t* full(int i) const { return bar + (i % NS); }
  __device__ uint64_t* empty(int i) const { return bar + NS + (i % NS); }
  __device__ void wait(uint64_t* b, int parity) {
    if (!failed && !tc::mbar_wait(b, parity)) failed = true;
  }
  // Stages and issues n chunks: stage(i, slot) fills chunk i's slot (workers),
  // mma(i, slot) issues its MMAs (warp 8, lane 0).
  template <class S, class M>
  __device__ void run(int n, S stage, M mma) {
    const int g0 = done;
    if (threadIdx.x < kWorkers) {
      constexpr int D = 2;        // chunks whose copies may still be in flight
      int arrived = 0;
      auto signal = [&](int k) {
        tc::fence_async_smem();
        tc::tc_fence_before();
        tc::mbar_arrive(full(g0 + k));
      };
      for (int i = 0; i < n; ++i) {
        const int g = g0 + i;
        if (g >= NS) wait(empty(g - NS), ((g - NS) / NS) & 1);
        stage(i, slot(g));
        tc::cp_async_commit();
        if (i - arrived >= D) {
          tc::cp_async_wait<D>();
          signal(arrived++);
        }
      }
      tc::cp_async_wait<0>();
      while (arrived < n) signal(arrived++);
    } else if (threadIdx.x == kWorkers) {
      for (int i = 0; i < n; ++i) {
        const int g = g0 + i;
        wait(full(g), (g / NS) & 1);
        tc::tc_fence_after();
        if (!failed) mma(i, slot(g));
        tc::mma_commit(empty(g));
      }
    }
    done = g0 + n;
    failed = __syncthreads_or(failed ? 1 : 0) != 0;
  }
  // Every MMA issued so far has completed (their results are readable).
  __device__ void wait_all() {
    if (done > 0) wait(empty(done - 1), ((done - 1) / NS) & 1);
    failed = __syncthreads_or(failed ? 1 : 0) != 0;
    tc::tc_fence_after();
  }
};

// Shared prologue: barriers (full[ns] for the workers' arrivals, empty[ns] and
// the drain barrier for MMA commits), TMEM allocation (warp 0). Returns the
// TMEM base.
constexpr int kDrainBar = 15;
__device__ __forceinline__ uint32_t setup(uint64_t* bars, int ns, uint32_t* tslot,
                                          uint32_t ncols) {
  if (threadIdx.x == 0) {
    for (int i = 0; i < ns; ++i) tc::mbar_init(bars + i, kWorkers);
    for (int i = ns; i < 2 * ns; ++i) tc::mbar_init(bars + i, 1);
    tc::mbar_init(bars + kDrainBar, 1);
    tc::fence_mbar_init();
  }
  if (threadIdx.x < 32) tc::tmem_alloc(tslot, ncols);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  return *tslot;
}

// Shared epilogue: on a failed wait, drain the issued MMAs before TMEM is freed.
__device__ __forceinline__ void teardown(bool failed, uint64_t* bar_drain, uint32_t tmem,
                                         uint32_t ncols, int* dev_status) {
  if (failed && threadIdx.x == kWorkers) {
    report(dev_status, DARK_ERR_TIMEOUT);
    tc::drain_mmas(bar_drain);
  }
  tc::tc_fence_before();
  __syncthreads();
  if (threadIdx.x < 32) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, ncols);
  }
}

// TMEM address of this thread's lane (row 32 * (warp % 4) + lane) at column col.
__device__ __forceinline__ uint32_t lane_addr(uint32_t tmem, int col) {
  return tmem + ((uint32_t)((threadIdx.x >> 5) & 3) * 32u << 16) + (uint32_t)col;
}

// Four consecutive bf16 values as floats; `vec`: the address is 8-byte aligned.
__device__ __forceinline__ float4 ld_bf16x4(const __nv_bfloat16* p, bool vec) {
  if (vec) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    const float2 lo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
    const float2 hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
    return make_float4(lo.x, lo.y, hi.x, hi.y);
  }
  return make_float4(__bfloat162float(p[0]), __bfloat162float(p[1]), __bfloat162float(p[2]),
                     __bfloat162float(p[3]));
}
__device__ __forceinline__ void st_f4(float* p, float a, float b, float c, float d) {
  *reinterpret_cast<float4*>(p) = make_float4(a, b, c, d);
}
__device__ __forceinline__ void st_bf16x4(__nv_bfloat16* p, float4 v, bool vec) {
  const __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y), hi = __floats2bfloat162_rn(v.z, v.w);
  if (vec) {
    uint2 u;
    u.x = *reinterpret_cast<const uint32_t*>(&lo);
    u.y = *reinterpret_cast<const uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(p) = u;
  } else {
    p[0] = lo.x;
    p[1] = lo.y;
    p[2] = hi.x;
    p[3] = hi.y;
  }
}

// Epilogue blocks of 128 rows x W fp32 values in shared memory (row stride
// W + 4 floats, so that one float4 per row and thread meets no bank conflict):
// each epilogue thread fills its own row, then all threads move the block
// row by row so that global accesses are coalesced.
constexpr int kPad = 4;
// store(row, c, v): values 4c..4c+3 of the block's row.
template <int W, class S>
__device__ __forceinline__ void block_out(const float* buf, S store) {
  constexpr int per = W / 4;
  __syncthreads();
  for (int i = threadIdx.x; i < kTT * per; i += blockDim.x) {
    const int row = i / per, c = i % per;
    store(row, c, *reinterpret_cast<const float4*>(buf + row * (W + kPad) + 4 * c));
  }
  __syncthreads();
}
// Copies rows in: src(row, c) is the 16-byte aligned source of values
// 4c..4c+3 of the row, or nullptr for zeros (then `any` stands in, unread).
template <int W, class S>
__device__ __forceinline__ void block_in(float* buf, S src, const float* any) {
  constexpr int per = W / 4;
  for (int i = threadIdx.x; i < kTT * per; i += blockDim.x) {
    const int row = i / per, c = i % per;
    const float* p = src(row, c);
    tc::cp_async16(tc::smem_u32(buf + row * (W + kPad) + 4 * c), p != nullptr ? p : any,
                   p != nullptr);
  }
  tc::cp_async_commit();
}

// ---------------------------------------------------------------------------
// Features of one side for a tile of 128 tokens: P = X W'^T on the tensor
// cores (fp32 W', rows m + r for keys, m for queries). Keys: phi = 2^(P_top -
// |P_bot|^2 - 1/2 log2 m), masked keys 0, and P_bot kept for the key
// coefficients; with the stabiliser the exponent is stored (-inf when masked)
// and the head maximum collected for a shift pass. Queries: 2^(P_top - max_j
// P_top) (a per-query factor cancels from every query gradient).
// Grid (tiles, B * H, 2 sides); TMEM columns 0 .. m + r - 1 hold P.
struct FeatArgs {
  const __nv_bfloat16 *xq, *xk;
  int64_t sb, sh, sl;
  const float* w;
  int heads_w, m, r, d, H, L;
  const uint8_t* mask;
  int stabilise;
  int xvec;                       // q, k rows 8-byte aligned (4-value loads)
  float *phiq, *phik, *pbot;
  int* ck;
  int* dev_status;
};

__host__ __device__ inline uint32_t feat_slot_bytes(int m, int r) {
  return km_bytes(kTT) + km_bytes(round_up(m + r, 32));
}

__global__ void __launch_bounds__(kThr, 1) tbf_features_kernel(FeatArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const int side = blockIdx.z, bh = blockIdx.y, b = bh / a.H, h = bh % a.H;
  const int t0 = blockIdx.x * kTT;
  const int m = a.m, r = a.r, d = a.d, L = a.L;
  const int nrow = side ? m + r : m;                          // W' rows = P columns
  const uint32_t slot = feat_slot_bytes(m, r);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kFeatSlots * slot);   // slots, drain (7)
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bars + 16);
  float* red = reinterpret_cast<float*>(bars + 20);                        // [2][128]
  const uint32_t tmem = setup(bars, kFeatSlots, tslot, 512);
  Ring<kFeatSlots> ring{smem, slot, bars, 0, false};
  const __nv_bfloat16* x = (side ? a.xk : a.xq) + (int64_t)b * a.sb + (int64_t)h * a.sh;
  const float* wh = a.w + (size_t)(a.heads_w == 1 ? 0 : h) * (m + r) * d;

  ring.run(
      d / 32,
      [&](int kc, uint8_t* s) {
        tc::stage_km_async(s + km_bytes(kTT), round_up(nrow, 32), [&](int row, int c) {
          return row < nrow ? wh + (size_t)row * d + kc * 32 + 4 * c : nullptr;
        }, wh, kWorkers);
        tc::stage_km(s, kTT, [&](int row, int c) {
          const int t = t0 + row;
          return t < L ? ld_bf16x4(x + (int64_t)t * a.sl + kc * 32 + 4 * c, a.xvec)
                       : make_float4(0.f, 0.f, 0.f, 0.f);
        }, kWorkers);
      },
      [&](int kc, uint8_t* s) {
        const uint32_t sa = tc::smem_u32(s), sw = sa + km_bytes(kTT);
        for (int c0 = 0; c0 < nrow; c0 += 256) {
          const int n = nrow - c0 < 256 ? nrow - c0 : 256;
          tc::mma_chunk(tmem + c0, sa, false, sw + (uint32_t)c0 * 128u, false, n, kc > 0);
        }
      });
  ring.wait_all();

  // epilogue: warps w and w + 4 share TMEM lanes 32 (w % 4) .. +31, each
  // taking half of a block's columns; row statistics are combined through
  // `red`, outputs leave through shared memory (the ring is idle now).
  // (warp 8 only joins the block-wide steps)
  const bool wk = threadIdx.x < kWorkers;
  const int q = (threadIdx.x >> 5) & 3, hf = (threadIdx.x >> 7) & 1;
  const int row = q * 32 + (threadIdx.x & 31), t = t0 + row;
  const bool in = t < L;
  float* buf = reinterpret_cast<float*>(smem);
  float* dst = (side ? a.phik : a.phiq) + (size_t)bh * L * m;
  auto store_rows = [&](float* base, int stride, int c0) {
    return [=](int rr, int c, float4 v) {
      if (t0 + rr < L) *reinterpret_cast<float4*>(base + (size_t)(t0 + rr) * stride + c0 + 4 * c) = v;
    };
  };
  float rowc = 0.f;
  if (side) {
    // P_bot (kept for the key coefficients) and the key norm |P_bot|^2
    float nrm = 0.f;
    float* pb = a.pbot + (size_t)bh * L * r;
    for (int c0 = 0; c0 < r; c0 += 32) {
      if (wk) {
        float v[16];
        tc::tmem_ld16(lane_addr(tmem, m + c0 + hf * 16), v);
        float* o = buf + row * (32 + kPad) + hf * 16;
#pragma unroll
        for (int j = 0; j < 16; ++j) nrm = fmaf(v[j], v[j], nrm);
#pragma unroll
        for (int j = 0; j < 16; j += 4) st_f4(o + j, v[j], v[j + 1], v[j + 2], v[j + 3]);
      }
      block_out<32>(buf, store_rows(pb, r, c0));
    }
    if (wk) red[hf * kTT + row] = nrm;
    __syncthreads();
    rowc = red[row] + red[kTT + row] + 0.5f * log2f((float)m);
  } else {
    // queries: exponents relative to the row maximum
    float mx = -INFINITY;
    if (wk)
      for (int c0 = hf * 32; c0 < m; c0 += 64) {
        float v[32];
        tc::tmem_ld32(lane_addr(tmem, c0), v);
#pragma unroll
        for (int j = 0; j < 32; ++j) mx = fmaxf(mx, v[j]);
      }
    if (wk) red[hf * kTT + row] = mx;
    __syncthreads();
    rowc = fmaxf(red[row], red[kTT + row]);
  }
  const bool ok = !side || a.mask == nullptr || (in && a.mask[(size_t)b * L + t] != 0);
  float kmax = -INFINITY;
  for (int c0 = 0; c0 < m; c0 += 64) {
    if (wk) {
      float v[32];
      tc::tmem_ld32(lane_addr(tmem, c0 + hf * 32), v);
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const float e = v[j] - rowc;
        if (side && a.stabilise) {
          v[j] = ok ? e : -INFINITY;
          kmax = fmaxf(kmax, v[j]);
        } else {
          v[j] = ok ? exp2f(e) : 0.f;
        }
      }
      float* o = buf + row * (64 + kPad) + hf * 32;
#pragma unroll
      for (int j = 0; j < 32; j += 4) st_f4(o + j, v[j], v[j + 1], v[j + 2], v[j + 3]);
    }
    block_out<64>(buf, store_rows(dst, m, c0));
  }
  if (wk && side && a.stabilise) {
    kmax = warp_max(in ? kmax : -INFINITY);
    if ((threadIdx.x & 31) == 0 && kmax > -INFINITY) atomicMax(a.ck + bh, float_to_ordered(kmax));
  }
  teardown(ring.failed, bars + kDrainBar, tmem, 512, a.dev_status);
}

// ---------------------------------------------------------------------------
// Tile states st_c = X_c^T U_c as [m][dp] fp32 (dp = d + 1 rounded up to 32,
// the padding columns zero): X the feature rows of one side, U = [v | 1] for
// keys (SIDE 1) or the rows [w | -c] the query pass stored (SIDE 0). M = m
// features in one or two 128-row accumulators (TMEM columns 0 and 256), K =
// the tile's 128 tokens, N = d + 1 rounded up to 16. Grid (tiles, B * H).
struct StateArgs {
  const float* X;                 // [B*H][L][m]
  const __nv_bfloat16* v;         // keys: values
  int64_t vb, vh, vl;
  int vvec;                       // v rows 8-byte aligned
  const float* wrow;              // queries: [B*H][L][dp]
  int m, d, dp, H, L, nt;
  float* st;                      // [B*H][nt][m][dp]
  int* dev_status;
};

template <int SIDE>
__global__ void __launch_bounds__(kThr, 1) tbf_state_kernel(StateArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const int c = blockIdx.x, bh = blockIdx.y, b = bh / a.H, h = bh % a.H;
  const int t0 = c * kTT, m = a.m, d = a.d, dp = a.dp, L = a.L;
  const int mt = (m + 127) / 128, dn = round_up(d + 1, 16);
  const uint32_t abytes = mn_bytes(mt * 128), slot = abytes + mn_bytes(dp);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStateSlots * slot);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bars + 16);
  const uint32_t tmem = setup(bars, kStateSlots, tslot, 512);
  Ring<kStateSlots> ring{smem, slot, bars, 0, false};
  const float* X = a.X + (size_t)bh * L * m;
  const __nv_bfloat16* vh = a.v + (int64_t)b * a.vb + (int64_t)h * a.vh;
  const float* wr = a.wrow + (size_t)bh * L * dp;

  ring.run(
      kTT / 32,
      [&](int kc, uint8_t* s) {
        tc::stage_mn_async(s, mt * 128, [&](int k, int cc) -> const float* {
          const int t = t0 + kc * 32 + k;
          return (t < L && 4 * cc < m) ? X + (size_t)t * m + 4 * cc : nullptr;
        }, X, kWorkers);
        if constexpr (SIDE == 0) {
          tc::stage_mn_async(s + abytes, dp, [&](int k, int cc) -> const float* {
            const int t = t0 + kc * 32 + k;
            return t < L ? wr + (size_t)t * dp + 4 * cc : nullptr;
          }, wr, kWorkers);
        } else {
          tc::stage_mn(s + abytes, dp, [&](int k, int cc) {
            const int t = t0 + kc * 32 + k, e = 4 * cc;
            if (t >= L || e > d) return make_float4(0.f, 0.f, 0.f, 0.f);
            if (e == d) return make_float4(1.f, 0.f, 0.f, 0.f);
            return ld_bf16x4(vh + (int64_t)t * a.vl + e, a.vvec);
          }, kWorkers);
        }
      },
      [&](int kc, uint8_t* s) {
        const uint32_t sa = tc::smem_u32(s), sb = sa + abytes;
        for (int i = 0; i < mt; ++i)
          tc::mma_chunk(tmem + 256 * i, sa + i * 4 * tc::kMnBlockBytes, true, sb, true, dn,
                        kc > 0);
      });
  ring.wait_all();
  // warps 0-3 read accumulator 0, warps 4-7 accumulator 1 (feature rows 128..);
  // the rows [m][dp] (contiguous in the state array) leave through shared memory
  const int q = (threadIdx.x >> 5) & 3, acc = threadIdx.x >> 7;
  const int f = acc * 128 + q * 32 + (threadIdx.x & 31);
  float* buf = reinterpret_cast<float*>(smem);           // [m][dp + 4]
  const int ld = dp + kPad;
  if (acc < mt && f < m) {
    for (int c0 = 0; c0 < dp; c0 += 16) {
      float v[16];
      if (c0 < dn) tc::tmem_ld16(lane_addr(tmem, 256 * acc + c0), v);
#pragma unroll
      for (int j = 0; j < 16; ++j)
        if (c0 + j > d) v[j] = 0.f;
#pragma unroll
      for (int j = 0; j < 16; j += 4) st_f4(buf + f * ld + c0 + j, v[j], v[j + 1], v[j + 2], v[j + 3]);
    }
  } else if (acc < mt) {
    for (int c0 = 0; c0 < dn; c0 += 16) {   // the warp's loads are collective
      float v[16];
      tc::tmem_ld16(lane_addr(tmem, 256 * acc + c0), v);
    }
  }
  __syncthreads();
  float* out = a.st + ((size_t)bh * a.nt + c) * m * dp;
  const int per = dp / 4;
  for (int i = threadIdx.x; i < m * per; i += blockDim.x) {
    const int rr = i / per, cc = i - rr * per;
    *reinterpret_cast<float4*>(out + (size_t)rr * dp + 4 * cc) =
        *reinterpret_cast<const float4*>(buf + rr * ld + 4 * cc);
  }
  teardown(ring.failed, bars + kDrainBar, tmem, 512, a.dev_status);
}

// ---------------------------------------------------------------------------
// One tile of 128 tokens of one side. SIDE 0 (queries): X = Phi(Q), Y = Phi(K),
// state = [S | z] over earlier tiles (or all keys), U = [v | 1]; phase 1 gives
// [num | den], hence P = [w | -c] (stored for the key side). SIDE 1 (keys):
// X = Phi(K), Y = Phi(Q), state = [dS] over later tiles (or all queries),
// U = [w | -c]; phase 1 gives dv, and P = [v | 1]. Phase 2 on both sides:
// dphi(X) = P state^T + tri(P U^T) Y, coef = ln2 X dphi (keys add the norm
// part). tri keeps key <= query inside the tile (causal only).
// TMEM: columns 0..255 hold [num | den] / dv, later dphi; 256..383 the
// diagonal tile's scores. Shared memory: a two-slot ring and, causal, the
// masked 128 x 128 scores as a K-major operand.
struct PassArgs {
  const float *phiq, *phik;       // [B*H][L][m]
  const float* state;             // [B*H][nt][m][dp]
  const __nv_bfloat16* v;
  int64_t vb, vh, vl;
  const __nv_bfloat16* g;
  int64_t gb, gh, gl;
  int vvec, gvec;                 // v / dout rows 8-byte aligned
  float* wrow;                    // [B*H][L][dp]
  __nv_bfloat16* dv;
  int64_t ob, oh, ol;
  int ovec;                       // dv rows 8-byte aligned
  float* coef;                    // [B*H][L][m + r]
  const float* pbot;              // [B*H][L][r]
  int m, r, d, dp, H, L, nt, causal;
  int* dev_status;
};

__host__ __device__ inline uint32_t pass_slot_bytes(int m, int dp, int causal) {
  const uint32_t p1 = km_bytes(kTT) + mn_bytes(dp) + (causal ? km_bytes(kTT) : 0);
  const uint32_t p2 = km_bytes(kTT) + km_bytes(m);      // P and the state rows
  const uint32_t p3 = mn_bytes(m);                      // feature rows (diagonal)
  uint32_t s = p1 > p2 ? p1 : p2;
  return s > p3 ? s : p3;
}
__host__ __device__ inline uint32_t pass_smem_bytes(int m, int dp, int causal) {
  return 1024 + kPassSlots * pass_slot_bytes(m, dp, causal) + (causal ? 4 * km_bytes(kTT) : 0) +
         kTailBytes;
}

template <int SIDE>
__global__ void __launch_bounds__(kThr, 1) tbf_pass_kernel(PassArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const int c = blockIdx.x, bh = blockIdx.y, b = bh / a.H, h = bh % a.H;
  const int t0 = c * kTT, m = a.m, r = a.r, d = a.d, dp = a.dp, L = a.L;
  const int causal = a.causal, dn = round_up(d + 1, 16);
  const uint32_t slot = pass_slot_bytes(m, dp, causal);
  uint8_t* scores = smem + kPassSlots * slot;                     // 4 K-major chunks
  uint64_t* bars = reinterpret_cast<uint64_t*>(scores + (causal ? 4 * km_bytes(kTT) : 0));
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bars + 16);
  float* red = reinterpret_cast<float*>(bars + 20);               // [2][128]
  const uint32_t tmem = setup(bars, kPassSlots, tslot, 512);
  const uint32_t tD = tmem, tS = tmem + 256;
  Ring<kPassSlots> ring{smem, slot, bars, 0, false};

  const size_t rowbase = (size_t)bh * L;
  const float* X = (SIDE == 0 ? a.phiq : a.phik) + rowbase * m;
  const float* Y = (SIDE == 0 ? a.phik : a.phiq) + rowbase * m;
  const float* st = a.state + ((size_t)bh * a.nt + (causal ? c : 0)) * m * dp;
  float* wr = a.wrow + rowbase * dp;
  const __nv_bfloat16* vh = a.v + (int64_t)b * a.vb + (int64_t)h * a.vh;
  // [v | 1 | 0 ...] at token t, columns e .. e + 3
  auto vone4 = [&](int t, int e) -> float4 {
    if (t >= L || e > d) return make_float4(0.f, 0.f, 0.f, 0.f);
    if (e == d) return make_float4(1.f, 0.f, 0.f, 0.f);
    return ld_bf16x4(vh + (int64_t)t * a.vl + e, a.vvec);
  };
  // Staging of the tile's operands. [v | 1] is converted through registers;
  // fp32 rows ([w | -c], features, states) are copied asynchronously.
  auto v_km = [&](uint8_t* dst, int e0) {        // rows: tile tokens, K: columns e0..
    tc::stage_km(dst, kTT, [&](int rr, int cc) { return vone4(t0 + rr, e0 + 4 * cc); }, kWorkers);
  };
  auto w_km = [&](uint8_t* dst, int e0) {
    tc::stage_km_async(dst, kTT, [&](int rr, int cc) -> const float* {
      const int tt = t0 + rr;
      return tt < L ? wr + (size_t)tt * dp + e0 + 4 * cc : nullptr;
    }, wr, kWorkers);
  };
  auto v_mn = [&](uint8_t* dst, int tk0) {       // K: tokens tk0.., MN: columns
    tc::stage_mn(dst, dp, [&](int k, int cc) { return vone4(tk0 + k, 4 * cc); }, kWorkers);
  };
  auto w_mn = [&](uint8_t* dst, int tk0) {
    tc::stage_mn_async(dst, dp, [&](int k, int cc) -> const float* {
      const int tt = tk0 + k;
      return tt < L ? wr + (size_t)tt * dp + 4 * cc : nullptr;
    }, wr, kWorkers);
  };
  auto feat_km = [&](uint8_t* dst, const float* F, int f0) {   // rows: tokens, K: features
    tc::stage_km_async(dst, kTT, [&](int rr, int cc) -> const float* {
      const int tt = t0 + rr;
      return tt < L ? F + (size_t)tt * m + f0 + 4 * cc : nullptr;
    }, F, kWorkers);
  };
  auto feat_mn = [&](uint8_t* dst, const float* F, int tk0) {  // K: tokens, MN: features
    tc::stage_mn_async(dst, m, [&](int k, int cc) -> const float* {
      const int tt = tk0 + k;
      return tt < L ? F + (size_t)tt * m + 4 * cc : nullptr;
    }, F, kWorkers);
  };
  // U = [v | 1] (queries) or [w | -c] (keys); P the other one
  auto u_mn = [&](uint8_t* dst, int tk0) {
    if constexpr (SIDE == 0) v_mn(dst, tk0); else w_mn(dst, tk0);
  };
  auto u_km = [&](uint8_t* dst, int e0) {
    if constexpr (SIDE == 0) v_km(dst, e0); else w_km(dst, e0);
  };
  auto p_km = [&](uint8_t* dst, int e0) {
    if constexpr (SIDE == 0) w_km(dst, e0); else v_km(dst, e0);
  };

  // per-row work of the epilogues on warps 0-7 (warp 8 joins the block-wide steps)
  const bool wk = threadIdx.x < kWorkers;
  const int q = (threadIdx.x >> 5) & 3, hf = (threadIdx.x >> 7) & 1;
  const int row = q * 32 + (threadIdx.x & 31), t = t0 + row;
  const bool in = t < L;
  // masked diagonal scores (TMEM columns 256..383) -> K-major operand in `scores`
  auto scores_to_smem = [&]() {
    if (!wk) return;
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int c0 = hf * 64 + u * 32;
      float v[32];
      tc::tmem_ld32(lane_addr(tS, c0), v);
      uint8_t* chunk = scores + (c0 >> 5) * km_bytes(kTT);
#pragma unroll
      for (int j4 = 0; j4 < 8; ++j4) {
        float o[4];
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const int col = c0 + 4 * j4 + jj;
          const bool keep = SIDE == 0 ? col <= row : col >= row;
          o[jj] = keep ? v[4 * j4 + jj] : 0.f;
        }
        *reinterpret_cast<float4*>(chunk + (row >> 3) * 1024 + (row & 7) * 128 +
                                   (((j4 ^ row) & 7) << 4)) = make_float4(o[0], o[1], o[2], o[3]);
      }
    }
  };

  // ---- phase 1: D = X state + tri(X Y^T) U ----
  ring.run(
      m / 32,
      [&](int fc, uint8_t* s) {
        feat_km(s, X, fc * 32);
        tc::stage_mn_async(s + km_bytes(kTT), dp, [&](int k, int cc) -> const float* {
          return st + (size_t)(fc * 32 + k) * dp + 4 * cc;
        }, st, kWorkers);
        if (causal) feat_km(s + km_bytes(kTT) + mn_bytes(dp), Y, fc * 32);
      },
      [&](int fc, uint8_t* s) {
        const uint32_t sa = tc::smem_u32(s);
        tc::mma_chunk(tD, sa, false, sa + km_bytes(kTT), true, dn, fc > 0);
        if (causal)
          tc::mma_chunk(tS, sa, false, sa + km_bytes(kTT) + mn_bytes(dp), false, kTT, fc > 0);
      });
  if (causal) {
    ring.wait_all();
    scores_to_smem();
    ring.run(
        kTT / 32, [&](int kc, uint8_t* s) { u_mn(s, t0 + kc * 32); },
        [&](int kc, uint8_t* s) {
          tc::mma_chunk(tD, tc::smem_u32(scores + kc * km_bytes(kTT)), false, tc::smem_u32(s),
                        true, dn, true);
        });
  }
  ring.wait_all();

  // ---- epilogue of phase 1 (rows through shared memory; the ring is idle) ----
  const int dh = d / 2;
  float* buf = reinterpret_cast<float*>(smem);
  if (SIDE == 0) {
    // g rows in, then P = [g / den | -(g . num) / den^2 | 0 ...] in their place
    const int ld = dp + kPad, per = d / 4;
    const __nv_bfloat16* gb = a.g + (int64_t)b * a.gb + (int64_t)h * a.gh;
    for (int i = threadIdx.x; i < kTT * per; i += blockDim.x) {
      const int rr = i / per, cc = i - rr * per, tt = t0 + rr;
      const float4 g4 = tt < L ? ld_bf16x4(gb + (int64_t)tt * a.gl + 4 * cc, a.gvec)
                               : make_float4(0.f, 0.f, 0.f, 0.f);
      *reinterpret_cast<float4*>(buf + rr * ld + 4 * cc) = g4;
    }
    __syncthreads();
    const float den = wk ? tc::tmem_ld1(lane_addr(tD, d)) : 0.f;
    float* gr = buf + row * ld;
    float go = 0.f;
    if (wk)
      for (int c0 = hf * dh; c0 < (hf + 1) * dh; c0 += 16) {
        float v[16];
        tc::tmem_ld16(lane_addr(tD, c0), v);
#pragma unroll
        for (int j = 0; j < 16; ++j) go = fmaf(gr[c0 + j], v[j], go);
      }
    if (wk) red[hf * kTT + row] = go;
    __syncthreads();
    go = red[row] + red[kTT + row];
    const float inv = (in && den > 0.f) ? 1.f / den : 0.f;
    const float cc = go * inv * inv;
    if (wk)
    for (int c0 = hf * dh; c0 < (hf + 1) * dh; c0 += 4) {
      float4 g4 = *reinterpret_cast<const float4*>(gr + c0);
      g4.x *= inv; g4.y *= inv; g4.z *= inv; g4.w *= inv;
      if (!(isfinite(g4.x) && isfinite(g4.y) && isfinite(g4.z) && isfinite(g4.w)))
        report(a.dev_status, DARK_ERR_NUMERIC);
      *reinterpret_cast<float4*>(gr + c0) = g4;
    }
    if (wk && hf == 1) {
      if (!isfinite(cc)) report(a.dev_status, DARK_ERR_NUMERIC);
      for (int e = d; e < dp; e += 4) st_f4(gr + e, e == d ? -cc : 0.f, 0.f, 0.f, 0.f);
    }
    __syncthreads();
    const int pw = dp / 4;
    for (int i = threadIdx.x; i < kTT * pw; i += blockDim.x) {
      const int rr = i / pw, c4 = i - rr * pw;
      if (t0 + rr < L)
        *reinterpret_cast<float4*>(wr + (size_t)(t0 + rr) * dp + 4 * c4) =
            *reinterpret_cast<const float4*>(buf + rr * ld + 4 * c4);
    }
  } else {
    // dv rows out as bf16
    const int ld = d + kPad, per = d / 4;
    if (wk)
    for (int c0 = hf * dh; c0 < (hf + 1) * dh; c0 += 16) {
      float v[16];
      tc::tmem_ld16(lane_addr(tD, c0), v);
#pragma unroll
      for (int j = 0; j < 16; ++j)
        if (in && !isfinite(v[j])) report(a.dev_status, DARK_ERR_NUMERIC);
#pragma unroll
      for (int j = 0; j < 16; j += 4) st_f4(buf + row * ld + c0 + j, v[j], v[j + 1], v[j + 2], v[j + 3]);
    }
    __syncthreads();
    __nv_bfloat16* dvb = a.dv + (int64_t)b * a.ob + (int64_t)h * a.oh;
    for (int i = threadIdx.x; i < kTT * per; i += blockDim.x) {
      const int rr = i / per, c4 = i - rr * per;
      if (t0 + rr < L)
        st_bf16x4(dvb + (int64_t)(t0 + rr) * a.ol + 4 * c4,
                  *reinterpret_cast<const float4*>(buf + rr * ld + 4 * c4), a.ovec);
    }
  }
  tc::tc_fence_before();
  __syncthreads();                // the P rows above are read back by the staging below

  // ---- phase 2: dphi(X) = P state^T + tri(P U^T) Y ----
  if (causal)       // the diagonal tile's scores P U^T first
    ring.run(
        dp / 32,
        [&](int pc, uint8_t* s) {
          p_km(s, pc * 32);
          u_km(s + km_bytes(kTT), pc * 32);
        },
        [&](int pc, uint8_t* s) {
          const uint32_t sa = tc::smem_u32(s);
          tc::mma_chunk(tS, sa, false, sa + km_bytes(kTT), false, kTT, pc > 0);
        });
  ring.run(
      dp / 32,
      [&](int pc, uint8_t* s) {
        p_km(s, pc * 32);
        tc::stage_km_async(s + km_bytes(kTT), m, [&](int f, int cc) -> const float* {
          return st + (size_t)f * dp + pc * 32 + 4 * cc;
        }, st, kWorkers);
      },
      [&](int pc, uint8_t* s) {
        const uint32_t sa = tc::smem_u32(s);
        tc::mma_chunk(tD, sa, false, sa + km_bytes(kTT), false, m, pc > 0);
      });
  if (causal) {
    ring.wait_all();
    scores_to_smem();
    ring.run(
        kTT / 32, [&](int kc, uint8_t* s) { feat_mn(s, Y, t0 + kc * 32); },
        [&](int kc, uint8_t* s) {
          tc::mma_chunk(tD, tc::smem_u32(scores + kc * km_bytes(kTT)), false, tc::smem_u32(s),
                        true, m, true);
        });
  }
  ring.wait_all();

  // ---- coef = ln2 X dphi; keys add -2 (sum_j coef_j) P_bot ----
  // 64-column blocks: the X rows come in by copies (double-buffered), the
  // coefficients replace them and leave row by row
  float* buf0 = reinterpret_cast<float*>(smem);
  float* buf1 = buf0 + kTT * (64 + kPad);
  float* cfb = a.coef + rowbase * (size_t)(m + r);
  auto x_in = [&](int blk, float* bb) {
    block_in<64>(bb, [&](int rr, int c) -> const float* {
      const int tt = t0 + rr;
      return tt < L ? X + (size_t)tt * m + blk * 64 + 4 * c : nullptr;
    }, X);
  };
  const int nb = m / 64;
  x_in(0, buf0);
  float rs = 0.f;
  for (int blk = 0; blk < nb; ++blk) {
    float* cur = (blk & 1) ? buf1 : buf0;
    if (blk + 1 < nb) {
      x_in(blk + 1, (blk & 1) ? buf0 : buf1);
      tc::cp_async_wait<1>();
    } else {
      tc::cp_async_wait<0>();
    }
    __syncthreads();
    if (wk) {
      float v[32];
      tc::tmem_ld32(lane_addr(tD, blk * 64 + hf * 32), v);
      float* xr = cur + row * (64 + kPad) + hf * 32;
#pragma unroll
      for (int j = 0; j < 32; j += 4) {
        const float4 x4 = *reinterpret_cast<const float4*>(xr + j);
        const float o0 = kLn2f * x4.x * v[j], o1 = kLn2f * x4.y * v[j + 1];
        const float o2 = kLn2f * x4.z * v[j + 2], o3 = kLn2f * x4.w * v[j + 3];
        rs += (o0 + o1) + (o2 + o3);
        st_f4(xr + j, o0, o1, o2, o3);
      }
    }
    block_out<64>(cur, [&](int rr, int c, float4 val) {
      if (t0 + rr < L)
        *reinterpret_cast<float4*>(cfb + (size_t)(t0 + rr) * (m + r) + blk * 64 + 4 * c) = val;
    });
  }
  if (SIDE == 1) {
    if (wk) red[hf * kTT + row] = rs;
    __syncthreads();
    rs = red[row] + red[kTT + row];
    const float* pb = a.pbot + rowbase * (size_t)r;
    for (int c0 = 0; c0 < r; c0 += 32) {
      block_in<32>(buf0, [&](int rr, int c) -> const float* {
        const int tt = t0 + rr;
        return tt < L ? pb + (size_t)tt * r + c0 + 4 * c : nullptr;
      }, pb);
      tc::cp_async_wait<0>();
      __syncthreads();
      float* pr = buf0 + row * (32 + kPad) + hf * 16;
      if (wk)
#pragma unroll
      for (int j = 0; j < 16; j += 4) {
        const float4 p4 = *reinterpret_cast<const float4*>(pr + j);
        st_f4(pr + j, -2.f * rs * p4.x, -2.f * rs * p4.y, -2.f * rs * p4.z, -2.f * rs * p4.w);
      }
      block_out<32>(buf0, [&](int rr, int c, float4 val) {
        if (t0 + rr < L)
          *reinterpret_cast<float4*>(cfb + (size_t)(t0 + rr) * (m + r) + m + c0 + 4 * c) = val;
      });
    }
  } else {
    // the norm part of the query coefficients is zero
    const int per = r / 4;
    for (int i = threadIdx.x; i < kTT * per; i += blockDim.x) {
      const int rr = i / per, c4 = i - rr * per;
      if (t0 + rr < L)
        st_f4(cfb + (size_t)(t0 + rr) * (m + r) + m + 4 * c4, 0.f, 0.f, 0.f, 0.f);
    }
  }
  teardown(ring.failed, bars + kDrainBar, tmem, 512, a.dev_status);
}

// ---------------------------------------------------------------------------
// dx = coef W' for a tile of 128 tokens of one side (queries: K = m, their norm
// part is zero; keys: K = m + r). A = coef rows (K-major), B = W' (MN-major,
// N = d). Grid (tiles, B * H, 2 sides).
struct DxArgs {
  const float *cfq, *cfk;         // [B*H][L][m + r]
  const float* w;                 // [heads_w][m + r][d]
  int heads_w, m, r, d, H, L;
  __nv_bfloat16 *dq, *dk;
  int64_t ob, oh, ol;
  int ovec;                       // dq, dk rows 8-byte aligned
  int* dev_status;
};

__global__ void __launch_bounds__(kThr) tbf_dx_kernel(DxArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const int side = blockIdx.z, bh = blockIdx.y, b = bh / a.H, h = bh % a.H;
  const int t0 = blockIdx.x * kTT, m = a.m, r = a.r, d = a.d, L = a.L, mr = m + r;
  const uint32_t slot = km_bytes(kTT) + mn_bytes(d);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kGemmSlots * slot);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bars + 16);
  const uint32_t tmem = setup(bars, kGemmSlots, tslot, 128);
  Ring<kGemmSlots> ring{smem, slot, bars, 0, false};
  const float* cf = (side ? a.cfk : a.cfq) + (size_t)bh * L * mr;
  const float* wh = a.w + (size_t)(a.heads_w == 1 ? 0 : h) * mr * d;
  const int kend = side ? mr : m;
  ring.run(
      kend / 32,
      [&](int kc, uint8_t* s) {
        tc::stage_km_async(s, kTT, [&](int rr, int cc) -> const float* {
          const int t = t0 + rr;
          return t < L ? cf + (size_t)t * mr + kc * 32 + 4 * cc : nullptr;
        }, cf, kWorkers);
        tc::stage_mn_async(s + km_bytes(kTT), d, [&](int k, int cc) -> const float* {
          return wh + (size_t)(kc * 32 + k) * d + 4 * cc;
        }, wh, kWorkers);
      },
      [&](int kc, uint8_t* s) {
        const uint32_t sa = tc::smem_u32(s);
        tc::mma_chunk(tmem, sa, false, sa + km_bytes(kTT), true, d, kc > 0);
      });
  ring.wait_all();
  const int q = (threadIdx.x >> 5) & 3, hf = (threadIdx.x >> 7) & 1;
  const int row = q * 32 + (threadIdx.x & 31), t = t0 + row;
  // rows out through shared memory (the ring is idle), as bf16
  float* buf = reinterpret_cast<float*>(smem);
  const int ld = d + kPad, per = d / 4;
  if (threadIdx.x < kWorkers)
  for (int c0 = hf * (d / 2); c0 < (hf + 1) * (d / 2); c0 += 16) {
    float v[16];
    tc::tmem_ld16(lane_addr(tmem, c0), v);
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if (t < L && !isfinite(v[j])) report(a.dev_status, DARK_ERR_NUMERIC);
#pragma unroll
    for (int j = 0; j < 16; j += 4) st_f4(buf + row * ld + c0 + j, v[j], v[j + 1], v[j + 2], v[j + 3]);
  }
  __syncthreads();
  __nv_bfloat16* out = (side ? a.dk : a.dq) + (int64_t)b * a.ob + (int64_t)h * a.oh;
  for (int i = threadIdx.x; i < kTT * per; i += blockDim.x) {
    const int rr = i / per, c4 = i - rr * per;
    if (t0 + rr < L)
      st_bf16x4(out + (int64_t)(t0 + rr) * a.ol + 4 * c4,
                *reinterpret_cast<const float4*>(buf + rr * ld + 4 * c4), a.ovec);
  }
  teardown(ring.failed, bars + kDrainBar, tmem, 128, a.dev_status);
}

// dW'[hw] += sum over a token range of one (batch, head), both sides, of
// coef_t x_t^T: a 128-row block of [m + r][d] per CTA, K = tokens, A = coef^T
// and B = x both MN-major; fp32 atomics into dW' at the end.
// Grid (row blocks, B * H, token splits).
struct DwArgs {
  const __nv_bfloat16 *xq, *xk;
  int64_t sb, sh, sl;
  const float *cfq, *cfk;
  int m, r, d, H, L, heads_w, nsplit;
  int xvec;                       // q, k rows 8-byte aligned
  float* G;                       // [heads_w][m + r][d]
  int* dev_status;
};

__global__ void __launch_bounds__(kThr) tbf_dw_kernel(DwArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const int j0 = blockIdx.x * 128, bh = blockIdx.y, split = blockIdx.z;
  const int b = bh / a.H, h = bh % a.H, d = a.d, L = a.L, mr = a.m + a.r;
  const int per = round_up((L + a.nsplit - 1) / a.nsplit, 32);
  const int tb = split * per, te = min(L, tb + per);
  const uint32_t slot = mn_bytes(128) + mn_bytes(d);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kGemmSlots * slot);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bars + 16);
  const uint32_t tmem = setup(bars, kGemmSlots, tslot, 128);
  Ring<kGemmSlots> ring{smem, slot, bars, 0, false};
  const int nc = (te - tb + 31) / 32 > 0 ? (te - tb + 31) / 32 : 0;   // chunks per side
  ring.run(
      2 * nc,
      [&](int i, uint8_t* s) {
        const int side = i / nc, k0 = tb + (i % nc) * 32;
        const __nv_bfloat16* x = (side ? a.xk : a.xq) + (int64_t)b * a.sb + (int64_t)h * a.sh;
        const float* cf = (side ? a.cfk : a.cfq) + (size_t)bh * L * mr;
        tc::stage_mn_async(s, 128, [&](int k, int cc) -> const float* {
          const int t = k0 + k, j = j0 + 4 * cc;
          return (t < te && j < mr) ? cf + (size_t)t * mr + j : nullptr;
        }, cf, kWorkers);
        tc::stage_mn(s + mn_bytes(128), d, [&](int k, int cc) {
          const int t = k0 + k;
          return t < te ? ld_bf16x4(x + (int64_t)t * a.sl + 4 * cc, a.xvec)
                        : make_float4(0.f, 0.f, 0.f, 0.f);
        }, kWorkers);
      },
      [&](int i, uint8_t* s) {
        const uint32_t sa = tc::smem_u32(s);
        tc::mma_chunk(tmem, sa, true, sa + mn_bytes(128), true, d, i > 0);
      });
  ring.wait_all();
  const int q = (threadIdx.x >> 5) & 3, hf = (threadIdx.x >> 7) & 1;
  const int j = j0 + q * 32 + (threadIdx.x & 31);
  // the block's rows through shared memory, then coalesced atomics
  float* buf = reinterpret_cast<float*>(smem);
  const int ld = d + kPad, pw = d / 4;
  if (ring.done > 0) {
    if (threadIdx.x < kWorkers)
    for (int c0 = hf * (d / 2); c0 < (hf + 1) * (d / 2); c0 += 16) {
      float v[16];
      tc::tmem_ld16(lane_addr(tmem, c0), v);
      const int rr = j - j0;
#pragma unroll
      for (int u = 0; u < 16; u += 4) st_f4(buf + rr * ld + c0 + u, v[u], v[u + 1], v[u + 2], v[u + 3]);
    }
    __syncthreads();
    float* gh = a.G + ((size_t)(a.heads_w == 1 ? 0 : h) * mr + j0) * d;
    for (int i = threadIdx.x; i < 128 * pw; i += blockDim.x) {
      const int rr = i / pw, c4 = i - rr * pw;
      if (j0 + rr < mr) {
        const float4 v4 = *reinterpret_cast<const float4*>(buf + rr * ld + 4 * c4);
        float* g = gh + (size_t)rr * d + 4 * c4;
        atomicAdd(g, v4.x);
        atomicAdd(g + 1, v4.y);
        atomicAdd(g + 2, v4.z);
        atomicAdd(g + 3, v4.w);
      }
    }
  }
  teardown(ring.failed, bars + kDrainBar, tmem, 128, a.dev_status);
}

struct TcLayout {
  int nt, dp;
  size_t off_w, off_ck, off_phiq, off_phik, off_pbot, off_cs, off_ds, off_wq, off_cfq, off_cfk,
      off_g, total;
};

TcLayout tc_layout(int B, int H, int L, int m, int r, int d, int heads_w) {
  TcLayout s;
  const size_t bh = (size_t)B * H, mr = (size_t)m + r;
  s.nt = (L + kTT - 1) / kTT;
  s.dp = round_up(d + 1, 32);
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
  s.off_pbot = take(sizeof(float) * bh * L * r);
  s.off_cs = take(sizeof(float) * bh * s.nt * m * s.dp);
  s.off_ds = take(sizeof(float) * bh * s.nt * m * s.dp);
  s.off_wq = take(sizeof(float) * bh * L * s.dp);
  s.off_cfq = take(sizeof(float) * bh * L * mr);
  s.off_cfk = take(sizeof(float) * bh * L * mr);
  s.off_g = take(sizeof(float) * heads_w * mr * d);
  s.total = o;
  return s;
}

template <class K>
cudaError_t set_smem(K kernel, size_t bytes, int* done) {
  return set_smem_limit_once((const void*)kernel, (int)bytes, done);
}

// The kernels that allocate all 512 TMEM columns ask for enough shared memory
// to keep a single CTA per SM.
constexpr size_t kOneCtaSmem = 116 * 1024;
size_t one_cta(size_t bytes) { return bytes > kOneCtaSmem ? bytes : kOneCtaSmem; }

}  // namespace

size_t tc_bwd_workspace_bytes(int B, int H, int L, int m, int r, int d, int heads_w) {
  return tc_layout(B, H, L, m, r, d, heads_w).total;
}

bool tc_backward_supported(const BwdArgs& a) {
  if (a.dtype != DARK_BF16) return false;
  if (a.d % 32 != 0 || a.d > 128 || a.m % 64 != 0 || a.m > 256 || a.r % 32 != 0 || a.r > 128)
    return false;
  const int dp = round_up(a.d + 1, 32);
  const uint32_t limit = 227 * 1024;
  if (pass_smem_bytes(a.m, dp, 1) > limit) return false;
  if (1024 + kFeatSlots * feat_slot_bytes(a.m, a.r) + kTailBytes > limit) return false;
  return true;
}

cudaError_t launch_backward_tc(const BwdArgs& a) {
  const TcLayout s = tc_layout(a.B, a.H, a.L, a.m, a.r, a.d, a.heads_w);
  char* ws = (char*)a.ws;
  float* wf = (float*)(ws + s.off_w);
  int* ck = (int*)(ws + s.off_ck);
  float* phiq = (float*)(ws + s.off_phiq);
  float* phik = (float*)(ws + s.off_phik);
  float* pbot = (float*)(ws + s.off_pbot);
  float* cs = (float*)(ws + s.off_cs);
  float* dsn = (float*)(ws + s.off_ds);
  float* wq = (float*)(ws + s.off_wq);
  float* cfq = (float*)(ws + s.off_cfq);
  float* cfk = (float*)(ws + s.off_cfk);
  float* G = (float*)(ws + s.off_g);
  const int bh = a.B * a.H, m = a.m, r = a.r, d = a.d, L = a.L, nt = s.nt, dp = s.dp;
  const int stab = (a.flags & DARK_STABILISE) ? 1 : 0;
  const int causal = (a.flags & DARK_CAUSAL) ? 1 : 0;
  const __nv_bfloat16* q = (const __nv_bfloat16*)a.q;
  const __nv_bfloat16* k = (const __nv_bfloat16*)a.k;
  const __nv_bfloat16* v = (const __nv_bfloat16*)a.v;
  cudaStream_t st = a.stream;
  cudaError_t err;
  auto rows8 = [](const void* p, const int64_t* s3) {
    return ((uintptr_t)p % 8 == 0) && s3[0] % 4 == 0 && s3[1] % 4 == 0 && s3[2] % 4 == 0;
  };
  const int xvec = rows8(a.q, a.xs) && rows8(a.k, a.xs) ? 1 : 0;
  const int vvec = rows8(a.v, a.xs) ? 1 : 0;
  const int gvec = rows8(a.dout, a.gs) ? 1 : 0;

  err = launch_projection(a.omega, a.heads_omega, a.geom, a.heads_geom, a.heads_w, m, r, d,
                          DARK_F32, wf, st);
  if (err != cudaSuccess) return err;
  if (stab && (err = bwd_fill_ordered(ck, bh, -INFINITY, st)) != cudaSuccess) return err;

  {
    static int done[64];
    const size_t bytes = one_cta(1024 + kFeatSlots * feat_slot_bytes(m, r) + kTailBytes);
    if ((err = set_smem(tbf_features_kernel, bytes, done)) != cudaSuccess) return err;
    FeatArgs fa{q, k, a.xs[0], a.xs[1], a.xs[2], wf, a.heads_w, m, r, d, a.H, L, a.mask, stab,
                xvec, phiq, phik, pbot, ck, a.dev_status};
    tbf_features_kernel<<<dim3(nt, bh, 2), kThr, bytes, st>>>(fa);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
  }
  if (stab && (err = bwd_shift_keys(phik, ck, L, m, (size_t)bh * L * m, st)) != cudaSuccess)
    return err;

  const size_t st_bytes =
      one_cta(1024 + kStateSlots * (mn_bytes(round_up(m, 128)) + mn_bytes(dp)) + kTailBytes);
  StateArgs sa{phik, v, a.xs[0], a.xs[1], a.xs[2], vvec, wq, m, d, dp, a.H, L, nt, cs,
               a.dev_status};
  {
    static int done[64];
    if ((err = set_smem(tbf_state_kernel<1>, st_bytes, done)) != cudaSuccess) return err;
    tbf_state_kernel<1><<<dim3(nt, bh), kThr, st_bytes, st>>>(sa);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
  }
  if ((err = bwd_tile_scan(cs, m * dp, nt, bh, causal ? 0 : 2, st)) != cudaSuccess) return err;

  const size_t pass_bytes = one_cta(pass_smem_bytes(m, dp, causal));
  PassArgs pa{phiq, phik, cs, v, a.xs[0], a.xs[1], a.xs[2],
              (const __nv_bfloat16*)a.dout, a.gs[0], a.gs[1], a.gs[2], vvec, gvec, wq,
              nullptr, 0, 0, 0, 0, cfq, pbot, m, r, d, dp, a.H, L, nt, causal, a.dev_status};
  {
    static int done[64];
    if ((err = set_smem(tbf_pass_kernel<0>, pass_bytes, done)) != cudaSuccess) return err;
    tbf_pass_kernel<0><<<dim3(nt, bh), kThr, pass_bytes, st>>>(pa);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
  }
  sa.X = phiq;
  sa.st = dsn;
  {
    static int done[64];
    if ((err = set_smem(tbf_state_kernel<0>, st_bytes, done)) != cudaSuccess) return err;
    tbf_state_kernel<0><<<dim3(nt, bh), kThr, st_bytes, st>>>(sa);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
  }
  if ((err = bwd_tile_scan(dsn, m * dp, nt, bh, causal ? 1 : 2, st)) != cudaSuccess) return err;
  pa.state = dsn;
  pa.g = nullptr;
  pa.gb = pa.gh = pa.gl = 0;
  pa.dv = (__nv_bfloat16*)a.dv;
  pa.ob = a.ds[0];
  pa.oh = a.ds[1];
  pa.ol = a.ds[2];
  pa.ovec = rows8(a.dv, a.ds) ? 1 : 0;
  pa.coef = cfk;
  {
    static int done[64];
    if ((err = set_smem(tbf_pass_kernel<1>, pass_bytes, done)) != cudaSuccess) return err;
    tbf_pass_kernel<1><<<dim3(nt, bh), kThr, pass_bytes, st>>>(pa);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
  }
  {
    static int done[64];
    const size_t bytes = 1024 + kGemmSlots * (km_bytes(kTT) + mn_bytes(d)) + kTailBytes;
    if ((err = set_smem(tbf_dx_kernel, bytes, done)) != cudaSuccess) return err;
    DxArgs xa{cfq, cfk, wf, a.heads_w, m, r, d, a.H, L, (__nv_bfloat16*)a.dq,
              (__nv_bfloat16*)a.dk, a.ds[0], a.ds[1], a.ds[2],
              rows8(a.dq, a.ds) && rows8(a.dk, a.ds) ? 1 : 0, a.dev_status};
    tbf_dx_kernel<<<dim3(nt, bh, 2), kThr, bytes, st>>>(xa);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
  }
  if (a.dgeom != nullptr) {
    err = cudaMemsetAsync(G, 0, sizeof(float) * (size_t)a.heads_w * (m + r) * d, st);
    if (err != cudaSuccess) return err;
    const int blocks = (m + r + 127) / 128;
    int nsplit = (2 * num_sms() + blocks * bh - 1) / (blocks * bh);
    const int max_split = (L + 127) / 128;
    if (nsplit > max_split) nsplit = max_split;
    if (nsplit < 1) nsplit = 1;
    static int done[64];
    const size_t bytes = 1024 + kGemmSlots * (mn_bytes(128) + mn_bytes(d)) + kTailBytes;
    if ((err = set_smem(tbf_dw_kernel, bytes, done)) != cudaSuccess) return err;
    DwArgs wa{q, k, a.xs[0], a.xs[1], a.xs[2], cfq, cfk, m, r, d, a.H, L, a.heads_w, nsplit, xvec,
              G, a.dev_status};
    tbf_dw_kernel<<<dim3(blocks, bh, nsplit), kThr, bytes, st>>>(wa);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    if ((err = bwd_dgeom(G, a)) != cudaSuccess) return err;
  }
  return cudaSuccess;
}

}  // namespace dark
