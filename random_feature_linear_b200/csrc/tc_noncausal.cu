// Non-causal (key-masked) PRF attention forward on sm_100a tensor cores.
//
// DARKformer README, section "Kernel": out = Phi(Q)(Phi(K)^T V) / Phi(Q)(Phi(K)^T 1),
// evaluated in the associative order so no L x L matrix exists. Three launches:
//   1. keys:   each CTA walks a contiguous range of 128-token key tiles of one
//              (batch, head): TMA K/V tiles (double-buffered) -> tcgen05 feature
//              GEMM K W'^T (fp16, fp32 in TMEM) -> epilogue: key norm, exp2,
//              mask -> bf16 Phi tile in smem -> tcgen05 GEMM Phi^T [V | 1]
//              accumulated in TMEM over the range -> fp32 partial [S | z].
//   2. reduce: sums the partials of each head in a fixed order (deterministic)
//              and writes [S | z] as the hi + lo bf16 shared-memory image of the
//              query kernel's B operands (and the state, if requested).
//   3. queries: each CTA walks a range of query tiles: TMA Q -> feature GEMM
//              Q W^T -> exp2 -> bf16 Psi tile -> tcgen05 GEMM Psi [S | z]
//              (hi and lo parts) -> out = num / den.
// Psi(Q) drops the per-query factors of phi(q), which cancel in the ratio.
#include <string.h>

#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace dark {
namespace {

using namespace tc;

constexpr int kD = 64;
constexpr int kT = 128;                     // tokens per tile
constexpr int kThreads = 256;
constexpr int kSms = 148;
constexpr int kTileBytes = kT * kD * 2;
constexpr uint32_t kTmemCols = 512;

// Byte sizes of the query kernel's B-operand image of [S | z] (per head):
// S hi, S lo (MN-major, 128 B per feature), z hi, z lo (16 identical K-major rows).
__host__ __device__ constexpr uint32_t img_s_bytes(int m) { return (uint32_t)m * 128; }
__host__ __device__ constexpr uint32_t img_z_bytes(int m) { return (uint32_t)(m / 64) * 2048; }
__host__ __device__ constexpr uint32_t img_bytes(int m) { return 2 * img_s_bytes(m) + 2 * img_z_bytes(m); }

__device__ __forceinline__ bool wait_all(uint64_t* bar, uint32_t parity, int* dev_status) {
  const bool ok = mbar_wait(bar, parity);
  const int bad = __syncthreads_or(ok ? 0 : 1);
  if (bad && threadIdx.x == 0) report(dev_status, DARK_ERR_TIMEOUT);
  return bad == 0;
}

// bf16 -> fp16 in place for `bytes` of a shared tile (feature GEMM operand).
__device__ __forceinline__ void to_fp16_inplace(uint32_t saddr, int bytes, int* dev_status) {
  bool bad = false;
  for (int i = threadIdx.x; i < bytes / 16; i += kThreads) {
    const uint32_t a = saddr + i * 16;
    uint4 u = ld_shared_v4(a);
    uint32_t* w32 = &u.x;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w32[e]));
      bad |= fabsf(f.x) > 65504.f || fabsf(f.y) > 65504.f;
      const __half2 hv = __floats2half2_rn(f.x, f.y);
      w32[e] = *reinterpret_cast<const uint32_t*>(&hv);
    }
    st_shared_v4(a, u.x, u.y, u.z, u.w);
  }
  if (bad) report(dev_status, DARK_ERR_NUMERIC);
}

struct KeyParams {
  const uint8_t* mask;
  int B, H, L, ntiles, nsplit, heads_w;
  float* partials;                 // [B*H*nsplit][65][m]
  int* dev_status;
};

template <int M_, int R_>
struct KeyCfg {
  static constexpr int NW = M_ + R_, MB = M_ / 128;
  static constexpr uint32_t kW = NW * 128;
  static constexpr uint32_t kPhi = (M_ / 64) * 16384;
  static constexpr uint32_t oW = 0;
  static constexpr uint32_t oK = (kW + 1023) / 1024 * 1024;   // 2 buffers
  static constexpr uint32_t oV = oK + 2 * kTileBytes;         // 2 buffers
  static constexpr uint32_t oPhi = oV + 2 * kTileBytes;
  static constexpr uint32_t oOnes = oPhi + kPhi;
  static constexpr uint32_t oBar = oOnes + 2048;
  static constexpr uint32_t kSmem = oBar + 64 + 1024;
  static constexpr uint32_t tP = 0, tD = 320;
};

template <int M_, int R_>
__global__ void __launch_bounds__(kThreads, 1)
    keys_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const KeyParams p) {
  using G = KeyCfg<M_, R_>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t s0 = smem_u32(sm);
  uint64_t* bar_kv = (uint64_t*)(sm + G::oBar);     // [2]
  uint64_t* bar_mma = bar_kv + 2;
  uint32_t* tmem_slot = (uint32_t*)(bar_kv + 3);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int quad = warp & 3, half = warp >> 2;
  const int row = quad * 32 + lane;
  const int split = blockIdx.x, bh = blockIdx.y, b = bh / p.H, h = bh % p.H;
  const int hw = p.heads_w == 1 ? 0 : h;
  const int tb = (int)((long long)split * p.ntiles / p.nsplit);
  const int te = (int)((long long)(split + 1) * p.ntiles / p.nsplit);

  if (tid == 0) {
    mbar_init(&bar_kv[0], 1);
    mbar_init(&bar_kv[1], 1);
    mbar_init(bar_mma, 1);
    fence_mbar_init();
    if (te > tb) {
      mbar_arrive_expect_tx(&bar_kv[0], G::kW + 2 * kTileBytes);
      for (int r0 = 0; r0 < G::NW; r0 += 16)
        tma_load_2d(sm + G::oW + r0 * 128, &tm_w, 0, hw * G::NW + r0, &bar_kv[0]);
      tma_load_4d(sm + G::oK, &tm_k, 0, tb * kT, h, b, &bar_kv[0]);
      tma_load_4d(sm + G::oV, &tm_v, 0, tb * kT, h, b, &bar_kv[0]);
    }
  }
  __syncwarp();
  if (warp == 0) tmem_alloc(tmem_slot, kTmemCols);
  for (int i = tid; i < 2048 / 4; i += kThreads) ((uint32_t*)(sm + G::oOnes))[i] = 0x3F803F80u;
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_tm = tmem + ((uint32_t)(quad * 32) << 16);

  uint32_t ph_kv[2] = {0, 0}, ph_mma = 0;
  bool abort = false;
  for (int t = tb; t < te; ++t) {
    const int i = t - tb, buf = i & 1;
    if (!wait_all(&bar_kv[buf], ph_kv[buf], p.dev_status)) { abort = true; break; }
    ph_kv[buf] ^= 1;
    to_fp16_inplace(s0 + G::oK + buf * kTileBytes, kTileBytes, p.dev_status);
    fence_async_smem();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t idn0 = idesc(128, (G::NW < 256 ? G::NW : 256), false, false, true);
      constexpr uint32_t idn1 = idesc(128, (G::NW > 256 ? G::NW - 256 : 16), false, false, true);
#pragma unroll
      for (int s = 0; s < kD / 16; ++s) {
        const uint64_t ad = sdesc(s0 + G::oK + buf * kTileBytes + s * 32, 16, 1024);
        mma(tmem + G::tP, ad, sdesc(s0 + G::oW + s * 32, 16, 1024), idn0, s > 0);
        if (G::NW > 256)
          mma(tmem + G::tP + 256, ad, sdesc(s0 + G::oW + 256 * 128 + s * 32, 16, 1024), idn1, s > 0);
      }
      mma_commit(bar_mma);
    }
    // this phase also covers the chunk-state GEMM of the previous tile
    if (!wait_all(bar_mma, ph_mma, p.dev_status)) { abort = true; break; }
    ph_mma ^= 1;
    tc_fence_after();
    // the other buffer is free now: prefetch the next tile into it
    if (tid == 0 && t + 1 < te) {
      const int nb = buf ^ 1;
      mbar_arrive_expect_tx(&bar_kv[nb], 2 * kTileBytes);
      tma_load_4d(sm + G::oK + nb * kTileBytes, &tm_k, 0, (t + 1) * kT, h, b, &bar_kv[nb]);
      tma_load_4d(sm + G::oV + nb * kTileBytes, &tm_v, 0, (t + 1) * kT, h, b, &bar_kv[nb]);
    }
    {
      float nrm = 0.f;
#pragma unroll
      for (int c0 = 0; c0 < R_; c0 += 16) {
        float v[16];
        tmem_ld16(lane_tm + G::tP + M_ + c0, v);
#pragma unroll
        for (int e = 0; e < 16; ++e) nrm = fmaf(v[e], v[e], nrm);
      }
      nrm += 0.5f * __log2f((float)M_);
      const int tok = t * kT + row;
      bool valid = tok < p.L;
      if (valid && p.mask != nullptr) valid = p.mask[(size_t)b * p.L + tok] != 0;
#pragma unroll 1
      for (int f0 = half * (M_ / 2); f0 < (half + 1) * (M_ / 2); f0 += 32) {
        float v[32];
        tmem_ld32(lane_tm + G::tP + f0, v);
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          uint32_t w4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float a = valid ? ex2(v[8 * g + 2 * e] - nrm) : 0.f;
            const float c = valid ? ex2(v[8 * g + 2 * e + 1] - nrm) : 0.f;
            w4[e] = pack_bf16(a, c);
          }
          st_shared_v4(s0 + G::oPhi + kmajor_off(row, f0 + 8 * g, 16384), w4[0], w4[1], w4[2], w4[3]);
        }
      }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t idv = idesc(128, 64, true, true, false);
      constexpr uint32_t id1 = idesc(128, 16, true, false, false);
#pragma unroll
      for (int mb = 0; mb < G::MB; ++mb) {
#pragma unroll
        for (int s = 0; s < kT / 16; ++s) {
          const uint32_t acc = (t > tb || s > 0) ? 1u : 0u;
          const uint64_t ad = sdesc(s0 + G::oPhi + mb * 32768 + s * 2048, 16384, 1024);
          mma(tmem + G::tD + 80 * mb, ad, sdesc(s0 + G::oV + buf * kTileBytes + s * 2048, 16384, 1024),
              idv, acc);
          mma(tmem + G::tD + 80 * mb + 64, ad, sdesc(s0 + G::oOnes + (s % 4) * 32, 16, 1024), id1, acc);
        }
      }
    }
  }
  if (!abort && te > tb) {
    if (tid == 0) mma_commit(bar_mma);
    if (!wait_all(bar_mma, ph_mma, p.dev_status)) abort = true;
    tc_fence_after();
  }
  if (!abort && half < G::MB) {
    const int f = half * 128 + row;
    float* dst = p.partials + ((size_t)bh * p.nsplit + split) * 65 * M_;
    if (te > tb) {
      float v[32];
      const uint32_t base = lane_tm + G::tD + 80 * half;
      tmem_ld32(base, v);
#pragma unroll
      for (int e = 0; e < 32; ++e) dst[e * M_ + f] = v[e];
      tmem_ld32(base + 32, v);
#pragma unroll
      for (int e = 0; e < 32; ++e) dst[(32 + e) * M_ + f] = v[e];
      dst[64 * M_ + f] = tmem_ld1(base + 64);
    } else {
      for (int e = 0; e < 65; ++e) dst[e * M_ + f] = 0.f;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Sums the split partials of each head in split order and writes the query
// kernel's operand image (hi + lo bf16) and, if requested, the fp32 state.
__global__ void reduce_kernel(const float* __restrict__ partials, int nsplit, int m,
                              uint8_t* __restrict__ images, float* __restrict__ st_kv,
                              float* __restrict__ st_z) {
  const int bh = blockIdx.y;
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= 65 * m) return;
  const int col = idx / m, f = idx % m;
  const float* src = partials + (size_t)bh * nsplit * 65 * m + idx;
  float acc = 0.f;
  for (int s = 0; s < nsplit; ++s) acc += src[(size_t)s * 65 * m];
  const __nv_bfloat16 hi = __float2bfloat16_rn(acc);
  const __nv_bfloat16 lo = __float2bfloat16_rn(acc - __bfloat162float(hi));
  uint8_t* img = images + (size_t)bh * img_bytes(m);
  if (col < 64) {
    const uint32_t off = (uint32_t)(f / 8) * 1024 + (uint32_t)(f % 8) * 128 +
                         (uint32_t)((((col / 8) ^ (f % 8)) * 16)) + (uint32_t)(col % 8) * 2;
    *reinterpret_cast<__nv_bfloat16*>(img + off) = hi;
    *reinterpret_cast<__nv_bfloat16*>(img + img_s_bytes(m) + off) = lo;
    if (st_kv != nullptr) st_kv[((size_t)bh * m + f) * 64 + col] = acc;
  } else {
    uint8_t* zh = img + 2 * img_s_bytes(m);
    uint8_t* zl = zh + img_z_bytes(m);
    for (int n = 0; n < 16; ++n) {
      const uint32_t off = (uint32_t)(f / 64) * 2048 + kmajor_off(n, f % 64, 0);
      *reinterpret_cast<__nv_bfloat16*>(zh + off) = hi;
      *reinterpret_cast<__nv_bfloat16*>(zl + off) = lo;
    }
    if (st_z != nullptr) st_z[(size_t)bh * m + f] = acc;
  }
}

struct QueryParams {
  __nv_bfloat16* out;
  int64_t ob, oh, ol;
  int B, H, L, ntiles, heads_w, total_tiles;
  const uint8_t* images;
  int* dev_status;
};

template <int M_, int R_>
struct QueryCfg {
  static constexpr int NW = M_ + R_;
  static constexpr uint32_t kWq = M_ * 128;       // the m feature rows of W'
  static constexpr uint32_t kPsi = (M_ / 64) * 16384;
  static constexpr uint32_t oW = 0;
  static constexpr uint32_t oImg = (kWq + 1023) / 1024 * 1024;
  static constexpr uint32_t oQ = oImg + (img_bytes(M_) + 1023) / 1024 * 1024;   // 2 buffers
  static constexpr uint32_t oPsi = oQ + 2 * kTileBytes;
  static constexpr uint32_t oBar = oPsi + kPsi;
  static constexpr uint32_t kSmem = oBar + 64 + 1024;
  static constexpr uint32_t tP = 0, tO = 256;
};

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"((uint64_t)src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

template <int M_, int R_>
__global__ void __launch_bounds__(kThreads, 1)
    queries_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_q,
                   const QueryParams p) {
  using G = QueryCfg<M_, R_>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t s0 = smem_u32(sm);
  uint64_t* bar_q = (uint64_t*)(sm + G::oBar);      // [2]
  uint64_t* bar_mma = bar_q + 2;
  uint64_t* bar_head = bar_q + 3;
  uint32_t* tmem_slot = (uint32_t*)(bar_q + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int quad = warp & 3, half = warp >> 2;
  const int row = quad * 32 + lane;
  const int ub = (int)((long long)blockIdx.x * p.total_tiles / gridDim.x);
  const int ue = (int)((long long)(blockIdx.x + 1) * p.total_tiles / gridDim.x);

  if (tid == 0) {
    mbar_init(&bar_q[0], 1);
    mbar_init(&bar_q[1], 1);
    mbar_init(bar_mma, 1);
    mbar_init(bar_head, 1);
    fence_mbar_init();
    if (ue > ub) {
      const int bh = ub / p.ntiles, t = ub % p.ntiles;
      mbar_arrive_expect_tx(&bar_q[0], kTileBytes);
      tma_load_4d(sm + G::oQ, &tm_q, 0, t * kT, bh % p.H, bh / p.H, &bar_q[0]);
    }
  }
  __syncwarp();
  if (warp == 0) tmem_alloc(tmem_slot, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_tm = tmem + ((uint32_t)(quad * 32) << 16);

  uint32_t ph_q[2] = {0, 0}, ph_mma = 0, ph_head = 0;
  int cur_bh = -1;
  bool abort = false;
  for (int u = ub; u < ue; ++u) {
    const int i = u - ub, buf = i & 1;
    const int bh = u / p.ntiles, t = u % p.ntiles, b = bh / p.H, h = bh % p.H;
    if (bh != cur_bh) {
      // W' rows and the [S | z] image of this head (all earlier MMAs have completed)
      if (tid == 0) {
        const int hw = p.heads_w == 1 ? 0 : h;
        mbar_arrive_expect_tx(bar_head, G::kWq + img_bytes(M_));
        for (int r0 = 0; r0 < M_; r0 += 16)
          tma_load_2d(sm + G::oW + r0 * 128, &tm_w, 0, hw * G::NW + r0, bar_head);
        const uint8_t* src = p.images + (size_t)bh * img_bytes(M_);
        for (uint32_t o = 0; o < img_bytes(M_); o += 16384)
          bulk_load(sm + G::oImg + o, src + o, img_bytes(M_) - o < 16384 ? img_bytes(M_) - o : 16384,
                    bar_head);
      }
      if (!wait_all(bar_head, ph_head, p.dev_status)) { abort = true; break; }
      ph_head ^= 1;
      cur_bh = bh;
    }
    if (!wait_all(&bar_q[buf], ph_q[buf], p.dev_status)) { abort = true; break; }
    ph_q[buf] ^= 1;
    to_fp16_inplace(s0 + G::oQ + buf * kTileBytes, kTileBytes, p.dev_status);
    fence_async_smem();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t idq = idesc(128, M_, false, false, true);
#pragma unroll
      for (int s = 0; s < kD / 16; ++s)
        mma(tmem + G::tP, sdesc(s0 + G::oQ + buf * kTileBytes + s * 32, 16, 1024),
            sdesc(s0 + G::oW + s * 32, 16, 1024), idq, s > 0);
      mma_commit(bar_mma);
    }
    if (!wait_all(bar_mma, ph_mma, p.dev_status)) { abort = true; break; }
    ph_mma ^= 1;
    tc_fence_after();
    // prefetch the next query tile into the other buffer (its GEMM completed)
    if (tid == 0 && u + 1 < ue) {
      const int nbh = (u + 1) / p.ntiles, nt = (u + 1) % p.ntiles;
      mbar_arrive_expect_tx(&bar_q[buf ^ 1], kTileBytes);
      tma_load_4d(sm + G::oQ + (buf ^ 1) * kTileBytes, &tm_q, 0, nt * kT, nbh % p.H, nbh / p.H,
                  &bar_q[buf ^ 1]);
    }
#pragma unroll 1
    for (int f0 = half * (M_ / 2); f0 < (half + 1) * (M_ / 2); f0 += 32) {
      float v[32];
      tmem_ld32(lane_tm + G::tP + f0, v);
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        uint32_t w4[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) w4[e] = pack_bf16(ex2(v[8 * g + 2 * e]), ex2(v[8 * g + 2 * e + 1]));
        st_shared_v4(s0 + G::oPsi + kmajor_off(row, f0 + 8 * g, 16384), w4[0], w4[1], w4[2], w4[3]);
      }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t idv = idesc(128, 64, false, true, false);
      constexpr uint32_t id1 = idesc(128, 16, false, false, false);
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        const uint32_t sb = s0 + G::oImg + part * img_s_bytes(M_);
        const uint32_t zb = s0 + G::oImg + 2 * img_s_bytes(M_) + part * img_z_bytes(M_);
#pragma unroll
        for (int s = 0; s < M_ / 16; ++s) {
          const uint64_t ad = sdesc(s0 + G::oPsi + (s / 4) * 16384 + (s % 4) * 32, 16, 1024);
          const uint32_t acc = (part > 0 || s > 0) ? 1u : 0u;
          mma(tmem + G::tO, ad, sdesc(sb + s * 2048, 16384, 1024), idv, acc);
          mma(tmem + G::tO + 64, ad, sdesc(zb + (s / 4) * 2048 + (s % 4) * 32, 16, 1024), id1, acc);
        }
      }
      mma_commit(bar_mma);
    }
    if (!wait_all(bar_mma, ph_mma, p.dev_status)) { abort = true; break; }
    ph_mma ^= 1;
    tc_fence_after();
    {
      const float den = tmem_ld1(lane_tm + G::tO + 64);
      float v[32];
      tmem_ld32(lane_tm + G::tO + half * 32, v);
      const int tok = t * kT + row;
      if (tok < p.L) {
        const float inv = den > 0.f ? 1.f / den : 0.f;
        uint32_t w[16];
        bool bad = !isfinite(den);
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float a = v[2 * e] * inv, c = v[2 * e + 1] * inv;
          bad |= !isfinite(a) || !isfinite(c);
          w[e] = pack_bf16(a, c);
        }
        if (bad) report(p.dev_status, DARK_ERR_NUMERIC);
        uint4* dst = reinterpret_cast<uint4*>(p.out + (int64_t)b * p.ob + (int64_t)h * p.oh +
                                              (int64_t)tok * p.ol + half * 32);
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4)
          dst[q4] = make_uint4(w[4 * q4], w[4 * q4 + 1], w[4 * q4 + 2], w[4 * q4 + 3]);
      }
    }
    tc_fence_before();
    __syncthreads();
  }
  (void)abort;
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

struct Layout {
  int ntiles, nsplit;
  size_t off_part, off_img, total;
};

Layout layout(int B, int H, int L, int m) {
  Layout s;
  const int bh = B * H;
  s.ntiles = (L + kT - 1) / kT;
  s.nsplit = kSms / bh;
  if (s.nsplit < 1) s.nsplit = 1;
  if (s.nsplit > s.ntiles) s.nsplit = s.ntiles;
  s.off_part = kWsHeader;
  s.off_img = align_up(s.off_part + (size_t)bh * s.nsplit * 65 * m * 4, 1024);
  s.total = align_up(s.off_img + (size_t)bh * img_bytes(m), 256);
  return s;
}

bool aligned16(const void* ptr) { return ((uintptr_t)ptr & 15) == 0; }

bool make_maps(const FwdArgs& a, CUtensorMap* tw, CUtensorMap* tq, CUtensorMap* tk, CUtensorMap* tv) {
  const uint64_t wd[2] = {(uint64_t)a.d, (uint64_t)a.heads_w * (a.m + a.r)};
  const uint64_t wsd[1] = {(uint64_t)a.d * 2};
  const uint32_t wb[2] = {64, 16};
  if (!encode_tmap(tw, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, a.w, wd, wsd, wb)) return false;
  const uint64_t xd[4] = {(uint64_t)a.d, (uint64_t)a.L, (uint64_t)a.H, (uint64_t)a.B};
  const uint64_t xs[3] = {(uint64_t)a.qs[2] * 2, (uint64_t)a.qs[1] * 2, (uint64_t)a.qs[0] * 2};
  const uint32_t xb[4] = {64, (uint32_t)kT, 1, 1};
  return encode_tmap(tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, a.q, xd, xs, xb) &&
         encode_tmap(tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, a.k, xd, xs, xb) &&
         encode_tmap(tv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, a.v, xd, xs, xb);
}

template <int M_, int R_>
cudaError_t launch(const FwdArgs& a, const CUtensorMap& tw, const CUtensorMap& tq,
                   const CUtensorMap& tk, const CUtensorMap& tv) {
  const Layout s = layout(a.B, a.H, a.L, a.m);
  char* ws = (char*)a.ws;
  float* partials = (float*)(ws + s.off_part);
  uint8_t* images = (uint8_t*)(ws + s.off_img);
  const int bh = a.B * a.H;

  KeyParams kp;
  kp.mask = a.mask;
  kp.B = a.B;
  kp.H = a.H;
  kp.L = a.L;
  kp.ntiles = s.ntiles;
  kp.nsplit = s.nsplit;
  kp.heads_w = a.heads_w;
  kp.partials = partials;
  kp.dev_status = a.dev_status;
  using KG = KeyCfg<M_, R_>;
  cudaError_t e = cudaFuncSetAttribute(keys_kernel<M_, R_>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)KG::kSmem);
  if (e != cudaSuccess) return e;
  keys_kernel<M_, R_><<<dim3(s.nsplit, bh), kThreads, KG::kSmem, a.stream>>>(tw, tk, tv, kp);

  reduce_kernel<<<dim3((65 * a.m + 255) / 256, bh), 256, 0, a.stream>>>(partials, s.nsplit, a.m,
                                                                         images, a.st_kv, a.st_z);

  QueryParams qp;
  qp.out = (__nv_bfloat16*)a.out;
  qp.ob = a.os[0];
  qp.oh = a.os[1];
  qp.ol = a.os[2];
  qp.B = a.B;
  qp.H = a.H;
  qp.L = a.L;
  qp.ntiles = s.ntiles;
  qp.heads_w = a.heads_w;
  qp.total_tiles = bh * s.ntiles;
  qp.images = images;
  qp.dev_status = a.dev_status;
  using QG = QueryCfg<M_, R_>;
  e = cudaFuncSetAttribute(queries_kernel<M_, R_>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)QG::kSmem);
  if (e != cudaSuccess) return e;
  const int grid = qp.total_tiles < kSms ? qp.total_tiles : kSms;
  queries_kernel<M_, R_><<<grid, kThreads, QG::kSmem, a.stream>>>(tw, tq, qp);
  return cudaGetLastError();
}

}  // namespace

bool tc_noncausal_supported(const FwdArgs& a) {
  if (a.dtype != DARK_BF16 || a.d != kD || (a.flags & DARK_STABILISE)) return false;
  if (!(a.m == 128 || a.m == 256) || a.r % 16 != 0 || a.r < 16 || a.r > 64) return false;
  if (!aligned16(a.q) || !aligned16(a.k) || !aligned16(a.v) || !aligned16(a.out) || !aligned16(a.w))
    return false;
  for (int i = 0; i < 3; ++i)
    if (a.qs[i] % 8 != 0 || a.os[i] % 8 != 0) return false;
  CUtensorMap t[4];
  return make_maps(a, &t[0], &t[1], &t[2], &t[3]);
}

size_t tc_noncausal_workspace_bytes(int B, int H, int L, int m, int d) {
  if (d != kD || !(m == 128 || m == 256)) return 0;
  return layout(B, H, L, m).total;
}

cudaError_t tc_noncausal_forward(const FwdArgs& a) {
  CUtensorMap tw, tq, tk, tv;
  if (!make_maps(a, &tw, &tq, &tk, &tv)) return cudaErrorInvalidValue;
#define DARK_NC_CASE(MM, RR) \
  if (a.m == MM && a.r == RR) return launch<MM, RR>(a, tw, tq, tk, tv);
  DARK_NC_CASE(256, 64)
  DARK_NC_CASE(256, 48)
  DARK_NC_CASE(256, 32)
  DARK_NC_CASE(256, 16)
  DARK_NC_CASE(128, 64)
  DARK_NC_CASE(128, 48)
  DARK_NC_CASE(128, 32)
  DARK_NC_CASE(128, 16)
#undef DARK_NC_CASE
  return cudaErrorInvalidValue;
}

}  // namespace dark
