// Key-side tensor-core kernel shared by the forward paths: per range of
// 128-token key tiles of one (batch, head), the chunk state
// Phi(K)^T [V | 1] (DARKformer README, section "Kernel": the statistics
// Phi(K)^T V and Phi(K)^T 1 of the associative form).
//
// Each CTA walks a contiguous tile range: TMA K/V tiles (double-buffered) ->
// tcgen05 feature GEMM K W'^T (fp16 operands, fp32 in TMEM) -> epilogue: key
// norm, exp2, key mask -> bf16 Phi tile in shared memory -> tcgen05 GEMM
// Phi^T [V | 1] accumulated in TMEM over the range -> fp32 [65][m] partial
// (column 64 is z). With one tile per range the partials are per-chunk
// aggregates.
#include "internal.h"
#include "tc_keys.cuh"

namespace dark {
namespace {

using namespace tc;

constexpr int kD = 64;
constexpr int kT = 128;
constexpr int kThreads = kFwdThreads;
constexpr int kTileBytes = kT * kD * 2;
constexpr uint32_t kTmemCols = 512;

struct KeyParams {
  const uint8_t* mask;
  int B, H, L, ntiles, nsplit, heads_w;
  float* partials;                 // [B*H*nsplit][65][m]
  // stabiliser (null: off): each CTA subtracts the running maximum of its valid
  // key exponents, rescaling the state accumulated so far when it grows, and
  // writes that maximum (-inf without a valid key) to shifts[B*H*nsplit]
  float* shifts;
  int* dev_status;
  long long stall;                 // testing stall before the first wait (0: none)
};

template <int M_, int R_>
struct KeyCfg {
  static constexpr int NW = M_ + R_, MB = M_ / 128;
  static constexpr uint32_t kW = NW * 128;
  static constexpr uint32_t kPhi = (M_ / 64) * 16384;
  static constexpr uint32_t oW = 0;
  static constexpr uint32_t oK = (kW + 1023) / 1024 * 1024;   // 2 buffers
  static constexpr uint32_t oV = oK + 2 * kTileBytes;         // 2 buffers
  // 128 x 64 block of bf16 ones after the V buffers: [V | 1] is one MN-major
  // operand of N = 80 (64-wide blocks LBO apart), one MMA per K-step
  static constexpr uint32_t oOnes = oV + 2 * kTileBytes;
  static constexpr uint32_t oPhi = oOnes + kTileBytes;
  static constexpr uint32_t oBar = oPhi + kPhi;
  static constexpr uint32_t oRed = oBar + 64;              // [8] per-warp maxima
  static constexpr uint32_t kSmem = oRed + 64 + 1024;
  static_assert(kSmem <= 232448, "shared memory");
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
  uint64_t* bar_drain = bar_kv + 4;     // abort path: the issued MMAs completed
  uint64_t* bar_never = bar_kv + 5;     // completed by nothing (testing stall)

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
    mbar_init(bar_drain, 1);
    mbar_init(bar_never, 1);
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
  for (int i = tid; i < kTileBytes / 4; i += kThreads) ((uint32_t*)(sm + G::oOnes))[i] = 0x3F803F80u;
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // a launch that follows with programmatic serialization may start now; it
  // waits for this grid's results where it reads them
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const uint32_t lane_tm = tmem + ((uint32_t)(quad * 32) << 16);

  uint32_t ph_kv = 0, ph_mma = 0;             // bit i: phase parity of buffer i
  float c_run = -INFINITY;                     // stabiliser: running key maximum
  bool abort = false;
  int issued[2] = {te > tb ? 1 : 0, 0}, waited[2] = {0, 0};   // load phases per buffer
  if (te > tb && p.stall > 0 && !wait_all(bar_never, 0, p.dev_status, p.stall)) abort = true;
  for (int t = tb; t < te && !abort; ++t) {
    const int i = t - tb, buf = i & 1;
    if (!wait_all(&bar_kv[buf], (ph_kv >> buf) & 1u, p.dev_status)) { abort = true; break; }
    ph_kv ^= 1u << buf;
    ++waited[buf];
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
      ++issued[nb];
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
      if (p.shifts != nullptr) {
        // the tile's largest valid exponent, then the running maximum; the
        // state accumulated so far (its MMAs completed with this tile's
        // feature GEMM) is rescaled when the maximum grows
        float mx = -INFINITY;
        for (int c0 = half * (M_ / 2); c0 < (half + 1) * (M_ / 2); c0 += 32) {
          float v[32];
          tmem_ld32(lane_tm + G::tP + c0, v);
#pragma unroll
          for (int e = 0; e < 32; ++e) mx = fmaxf(mx, v[e]);
        }
        mx = warp_max(valid ? mx - nrm : -INFINITY);
        float* red = (float*)(sm + G::oRed);
        if (lane == 0) red[warp] = mx;
        __syncthreads();
        float tmx = red[0];
#pragma unroll
        for (int w = 1; w < kThreads / 32; ++w) tmx = fmaxf(tmx, red[w]);
        __syncthreads();
        if (tmx > c_run) {
          if (t > tb && c_run > -INFINITY && half < G::MB) {
            const float sc = exp2f(c_run - tmx);
            const uint32_t base = lane_tm + G::tD + 80 * half;
            float v[32];
#pragma unroll
            for (int c0 = 0; c0 < 64; c0 += 32) {
              tmem_ld32(base + c0, v);
#pragma unroll
              for (int e = 0; e < 32; ++e) v[e] *= sc;
              tmem_st32(base + c0, v);
            }
            tmem_st1(base + 64, tmem_ld1(base + 64) * sc);
          }
          c_run = tmx;
        }
        if (c_run > -INFINITY) nrm += c_run;
      }
      exp2_rows_to_smem(lane_tm + G::tP, half * (M_ / 2), (half + 1) * (M_ / 2), nrm, !valid,
                        s0 + G::oPhi, row);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      // chunk state [S | z] += Phi^T [V | 1] (z in column 64 and its copies)
      constexpr uint32_t id = idesc(128, 80, true, true, false);
      const uint32_t sv = s0 + G::oV + buf * kTileBytes;
      const uint32_t lbo = G::oOnes - (G::oV + buf * kTileBytes);
#pragma unroll
      for (int mb = 0; mb < G::MB; ++mb) {
#pragma unroll
        for (int s = 0; s < kT / 16; ++s) {
          const uint32_t acc = (t > tb || s > 0) ? 1u : 0u;
          mma(tmem + G::tD + 80 * mb, sdesc(s0 + G::oPhi + mb * 32768 + s * 2048, 16384, 1024),
              sdesc(sv + s * 2048, lbo, 1024), id, acc);
        }
      }
    }
  }
  if (!abort && te > tb) {
    if (tid == 0) mma_commit(bar_mma);
    if (!wait_all(bar_mma, ph_mma, p.dev_status)) abort = true;
    tc_fence_after();
  }
  if (abort && tid == 0) {
    // no copy or MMA of this CTA may still be running when TMEM is freed
    drain_loads(&bar_kv[0], issued[0], waited[0]);
    drain_loads(&bar_kv[1], issued[1], waited[1]);
    drain_mmas(bar_drain);
  }
  if (!abort && tid == 0 && p.shifts != nullptr) p.shifts[(size_t)bh * p.nsplit + split] = c_run;
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


template <int M_, int R_>
cudaError_t launch_keys_t(const FwdArgs& a, const CUtensorMap& tw, const CUtensorMap& tk,
                          const CUtensorMap& tv, int ntiles, int nsplit, float* partials,
                          float* shifts) {
  KeyParams kp;
  kp.shifts = shifts;
  kp.mask = a.mask;
  kp.B = a.B;
  kp.H = a.H;
  kp.L = a.Lk;                    // keys (= L for self-attention)
  kp.ntiles = ntiles;
  kp.nsplit = nsplit;
  kp.heads_w = a.heads_w;
  kp.partials = partials;
  kp.dev_status = a.dev_status;
  kp.stall = test_stall_cycles();
  using KG = KeyCfg<M_, R_>;
  static int smem_set[64];
  cudaError_t e = set_smem_limit_once((const void*)keys_kernel<M_, R_>, (int)KG::kSmem, smem_set);
  if (e != cudaSuccess) return e;
  keys_kernel<M_, R_><<<dim3(nsplit, a.B * a.H), kThreads, KG::kSmem, a.stream>>>(tw, tk, tv, kp);
  return cudaGetLastError();
}

}  // namespace

cudaError_t tc_launch_key_states(const FwdArgs& a, const CUtensorMap& tw, const CUtensorMap& tk,
                                 const CUtensorMap& tv, int ntiles, int nsplit, float* partials,
                                 float* shifts) {
#define DARK_KEYS_CASE(MM, RR)                                                              \
  if (a.m == MM && a.r == RR)                                                               \
    return launch_keys_t<MM, RR>(a, tw, tk, tv, ntiles, nsplit, partials, shifts);
  DARK_KEYS_CASE(256, 64)
  DARK_KEYS_CASE(256, 48)
  DARK_KEYS_CASE(256, 32)
  DARK_KEYS_CASE(256, 16)
  DARK_KEYS_CASE(128, 64)
  DARK_KEYS_CASE(128, 48)
  DARK_KEYS_CASE(128, 32)
  DARK_KEYS_CASE(128, 16)
#undef DARK_KEYS_CASE
  return cudaErrorInvalidValue;
}

}  // namespace dark
