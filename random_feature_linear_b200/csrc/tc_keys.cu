// Key-side tensor-core kernel shared by the forward paths: per range of
// 128-token key tiles of one (batch, head), the chunk state
// Phi(K)^T [V | 1] (DARKformer README, section "Kernel": the statistics
// Phi(K)^T V and Phi(K)^T 1 of the associative form).
//
// Each CTA walks a contiguous tile range with three roles: warp 9 loads the
// K/V tiles by TMA (two buffers), warp 8 issues the tcgen05 MMAs, warps 0-7
// run the epilogue. Per tile: feature GEMM K W'^T (fp16 operands, fp32 in
// TMEM) -> epilogue: key norm, exp2, key mask -> bf16 Phi tile in shared
// memory -> GEMM Phi^T [V | 1] accumulated in TMEM over the range -> fp32
// [65][m] partial (column 64 is z). The epilogue reads a tile's features into
// registers and frees the TMEM block at once, then converts the next K tile to
// fp16, so the next tile's feature GEMM runs while this tile's exponentials
// are computed. With one tile per range the partials are per-chunk aggregates.
#include "internal.h"
#include "tc_keys.cuh"
#include "tc_roles.cuh"

namespace dark {
namespace {

using namespace tc;

constexpr int kD = 64;
constexpr int kT = 128;
constexpr int kEpi = kFwdThreads;          // epilogue threads (warps 0-7)
constexpr int kThreads = kEpi + 64;       // + MMA warp 8 + producer warp 9
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
  static constexpr uint32_t kW = NW * 128;                    // one W' image
  // W' as two bf16 images, hi and lo (hi + lo is the fp16 value exactly), so
  // that the feature GEMM reads the bf16 K tile as loaded: K W'^T = K hi^T + K lo^T
  static constexpr uint32_t oWlo = (kW + 1023) / 1024 * 1024;
  static constexpr uint32_t kPhi = (M_ / 64) * 16384;
  static constexpr uint32_t oW = 0;
  static constexpr uint32_t oK = oWlo + (kW + 1023) / 1024 * 1024;   // 2 buffers
  static constexpr uint32_t oV = oK + 2 * kTileBytes;         // 2 buffers
  // 128 x 64 block of bf16 ones after the V buffers: [V | 1] is one MN-major
  // operand of N = 80 (64-wide blocks LBO apart), one MMA per K-step
  static constexpr uint32_t oOnes = oV + 2 * kTileBytes;
  static constexpr uint32_t oPhi = oOnes + kTileBytes;
  static constexpr uint32_t oBar = oPhi + kPhi;
  static constexpr uint32_t oRed = oBar + 256;             // [2][8] per-warp maxima
  static constexpr uint32_t kSmem = oRed + 64 + 1024;
  static_assert(kSmem <= 232448, "shared memory");
  static constexpr uint32_t tP = 0, tD = 320;
};


// The fp16 W' image at `hi` (as loaded) -> bf16 hi in place and bf16 lo at
// `lo` (the same layout), by the 256 epilogue threads. An fp16 value has 11
// significant bits: hi = bf16(x) keeps 8 of them and x - hi, exact in fp32,
// has at most 4, so lo = bf16(x - hi) is exact and hi + lo = x.
__device__ __forceinline__ void split_w(uint32_t hi, uint32_t lo, uint32_t bytes, int etid) {
  for (uint32_t i = etid; i < bytes / 16; i += kEpi) {
    uint4 u = ld_shared_v4(hi + i * 16);
    uint32_t* w32 = &u.x;
    uint32_t l32[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 x = __half22float2(*reinterpret_cast<const __half2*>(&w32[e]));
      const __nv_bfloat162 h2 = __floats2bfloat162_rn(x.x, x.y);
      const float2 hf = __bfloat1622float2(h2);
      const __nv_bfloat162 l2 = __floats2bfloat162_rn(x.x - hf.x, x.y - hf.y);
      w32[e] = *reinterpret_cast<const uint32_t*>(&h2);
      l32[e] = *reinterpret_cast<const uint32_t*>(&l2);
    }
    st_shared_v4(hi + i * 16, u.x, u.y, u.z, u.w);
    st_shared_v4(lo + i * 16, l32[0], l32[1], l32[2], l32[3]);
  }
}

template <int M_, int R_>
__global__ void __launch_bounds__(kThreads, 1)
    keys_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const KeyParams p) {
  using G = KeyCfg<M_, R_>;
  constexpr int NH = M_ / 128;                // 32-column groups per pass (two passes per half)
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t s0 = smem_u32(sm);
  uint64_t* bars = (uint64_t*)(sm + G::oBar);
  uint64_t* k_full = bars + 0;       // [2] producer: K tile loaded (the first with W')
  uint64_t* v_full = bars + 2;       // [2] producer: V tile loaded
  uint64_t* v_empty = bars + 4;      // [2] MMA: chunk-state GEMM has read the V tile
  uint64_t* bar_conv = bars + 6;     // epilogue: W' split into bf16 hi and lo (8)
  // the feature GEMM in two parts: A = features [0, M/2) and the norm
  // columns, B = features [M/2, M); each part is released by the epilogue
  // as soon as it has been read, so the next tile's part can start
  uint64_t* bar_ffullA = bars + 7;   // MMA: part A in TMEM
  uint64_t* bar_ffreeA = bars + 8;   // epilogue: part A read (8)
  uint64_t* bar_ffullB = bars + 15;  // MMA: part B in TMEM
  uint64_t* bar_ffreeB = bars + 16;  // epilogue: part B read (8)
  uint64_t* bar_pfull = bars + 9;    // epilogue: Phi staged (8)
  uint64_t* bar_pfree = bars + 10;   // MMA: chunk-state GEMM done (Phi and the state free)
  uint64_t* bar_drain = bars + 11;   // abort path: the issued MMAs completed
  uint64_t* bar_never = bars + 12;   // completed by nothing (testing stall)
  uint64_t* k_empty = bars + 13;     // [2] MMA: feature GEMM has read the K tile
  uint32_t* tmem_slot = (uint32_t*)(bars + 17);
  volatile int* abort_flag = (volatile int*)(bars + 17) + 1;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x, bh = blockIdx.y, b = bh / p.H, h = bh % p.H;
  const int hw = p.heads_w == 1 ? 0 : h;
  const int tb = (int)((long long)split * p.ntiles / p.nsplit);
  const int te = (int)((long long)(split + 1) * p.ntiles / p.nsplit);
  const int n = te > tb ? te - tb : 0;

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(k_full + i, 1);
      mbar_init(v_full + i, 1);
      mbar_init(v_empty + i, 1);
      mbar_init(k_empty + i, 1);
    }
    mbar_init(bar_conv, 8);
    mbar_init(bar_ffullA, 1);
    mbar_init(bar_ffreeA, 8);
    mbar_init(bar_ffullB, 1);
    mbar_init(bar_ffreeB, 8);
    mbar_init(bar_pfull, 8);
    mbar_init(bar_pfree, 1);
    mbar_init(bar_drain, 1);
    mbar_init(bar_never, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
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

  if (warp == 9) {
    // ------------------------------------------------------------ producer
    // K tile j + 2 loads once tile j's feature GEMM has read its buffer, V tile
    // j + 1 once tile j - 1's chunk-state GEMM has read its buffer.
    if (lane == 0 && n > 0) {
      int nk[2] = {0, 0}, nv[2] = {0, 0};    // loads issued per buffer
      auto load_k = [&](int j) {
        const int buf = j & 1;
        mbar_arrive_expect_tx(k_full + buf, (j == 0 ? G::kW : 0u) + kTileBytes);
        if (j == 0)
          for (int r0 = 0; r0 < G::NW; r0 += 16)
            tma_load_2d(sm + G::oW + r0 * 128, &tm_w, 0, hw * G::NW + r0, k_full);
        tma_load_4d(sm + G::oK + buf * kTileBytes, &tm_k, 0, (tb + j) * kT, h, b, k_full + buf);
        ++nk[buf];
      };
      auto load_v = [&](int j) {
        const int buf = j & 1;
        mbar_arrive_expect_tx(v_full + buf, kTileBytes);
        tma_load_4d(sm + G::oV + buf * kTileBytes, &tm_v, 0, (tb + j) * kT, h, b, v_full + buf);
        ++nv[buf];
      };
      prefetch_tmap(&tm_w);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      load_k(0);
      load_v(0);
      if (n > 1) {
        load_k(1);
        load_v(1);
      }
      bool ok = true;
      for (int j = 0; ok && j + 1 < n; ++j) {
        if (j + 2 < n) {
          if (!(ok = wait_one(k_empty + (j & 1), (j >> 1) & 1, abort_flag, p.dev_status))) break;
          load_k(j + 2);
        }
        if (j >= 1) {
          if (!(ok = wait_one(v_empty + ((j + 1) & 1), ((j - 1) >> 1) & 1, abort_flag, p.dev_status)))
            break;
          load_v(j + 1);
        }
      }
      if (!ok) {
        // aborted: leave no copy in flight (a completed phase passes at once)
        for (int i = 0; i < 2; ++i) {
          if (nk[i] > 0) mbar_wait(k_full + i, (uint32_t)(nk[i] - 1) & 1u);
          if (nv[i] > 0) mbar_wait(v_full + i, (uint32_t)(nv[i] - 1) & 1u);
        }
      }
    }
    __syncwarp();
  } else if (warp == 8) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0 && n > 0) {
      bool ok = true;
      // K W'^T = K hi^T + K lo^T (bf16 operands, fp32 in TMEM), part A or B
      auto features = [&](int i, int part) {
        const uint32_t sk = s0 + G::oK + (i & 1) * kTileBytes;
        constexpr uint32_t idh = idesc(128, M_ / 2, false, false, false);
        constexpr uint32_t idr = idesc(128, R_, false, false, false);
#pragma unroll
        for (int w = 0; w < 2; ++w) {
          const uint32_t sw = s0 + (w == 0 ? G::oW : G::oWlo);
#pragma unroll
          for (int s = 0; s < kD / 16; ++s) {
            const uint64_t ad = sdesc(sk + s * 32, 16, 1024);
            const uint32_t acc = (w | s) != 0 ? 1u : 0u;
            if (part == 0) {
              mma(tmem + G::tP, ad, sdesc(sw + s * 32, 16, 1024), idh, acc);
              mma(tmem + G::tP + M_, ad, sdesc(sw + M_ * 128 + s * 32, 16, 1024), idr, acc);
            } else {
              mma(tmem + G::tP + M_ / 2, ad, sdesc(sw + (M_ / 2) * 128 + s * 32, 16, 1024), idh,
                  acc);
            }
          }
        }
        if (part == 0) {
          mma_commit(bar_ffullA);
        } else {
          mma_commit(bar_ffullB);
          mma_commit(k_empty + (i & 1));
        }
      };
      if ((ok = wait_one(bar_conv, 0, abort_flag, p.dev_status) &&
                wait_one(k_full, 0, abort_flag, p.dev_status))) {
        tc_fence_after();
        features(0, 0);
        features(0, 1);
      }
      for (int i = 0; ok && i < n; ++i) {
        // the next tile's features first (its K tile loaded, each part's TMEM
        // columns read), so that they are computed during this tile's
        // exponentials
        if (i + 1 < n) {
          if (!(ok = wait_one(k_full + ((i + 1) & 1), ((i + 1) >> 1) & 1, abort_flag, p.dev_status)))
            break;
          if (!(ok = wait_one(bar_ffreeA, i & 1, abort_flag, p.dev_status))) break;
          tc_fence_after();
          features(i + 1, 0);
          if (!(ok = wait_one(bar_ffreeB, i & 1, abort_flag, p.dev_status))) break;
          tc_fence_after();
          features(i + 1, 1);
        }
        // chunk state [S | z] += Phi^T [V | 1] (z in column 64 and its copies)
        if (!(ok = wait_one(bar_pfull, i & 1, abort_flag, p.dev_status))) break;
        if (!(ok = wait_one(v_full + (i & 1), (i >> 1) & 1, abort_flag, p.dev_status))) break;
        tc_fence_after();
        constexpr uint32_t id = idesc(128, 80, true, true, false);
        const uint32_t sv = s0 + G::oV + (i & 1) * kTileBytes;
        const uint32_t lbo = G::oOnes - (G::oV + (i & 1) * kTileBytes);
#pragma unroll
        for (int mb = 0; mb < G::MB; ++mb) {
#pragma unroll
          for (int s = 0; s < kT / 16; ++s)
            mma(tmem + G::tD + 80 * mb, sdesc(s0 + G::oPhi + mb * 32768 + s * 2048, 16384, 1024),
                sdesc(sv + s * 2048, lbo, 1024), id, (i > 0 || s > 0) ? 1u : 0u);
        }
        mma_commit(bar_pfree);
        mma_commit(v_empty + (i & 1));
      }
      if (!ok) drain_mmas(bar_drain);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int quad = warp & 3, half = warp >> 2;
    const int row = quad * 32 + lane;
    const uint32_t lane_tm = tmem + ((uint32_t)(quad * 32) << 16);
    float* red = (float*)(sm + G::oRed);
    float c_run = -INFINITY;                   // stabiliser: running key maximum
    bool ok = n > 0;
    if (ok && p.stall > 0) ok = epi_wait(bar_never, 0, abort_flag, p.dev_status, p.stall);
    // W' (loaded with the first K tile) into its bf16 hi and lo images
    if (ok && (ok = epi_wait(k_full, 0, abort_flag, p.dev_status))) {
      split_w(s0 + G::oW, s0 + G::oWlo, G::kW, tid);
      fence_async_smem();
      warp_arrive(bar_conv);
    }
    for (int i = 0; ok && i < n; ++i) {
      const int t = tb + i;
      // ---- this tile's features: the norm columns and pass 0 (part A), the
      // first pass exponentiated while the previous chunk-state GEMM may
      // still read Phi, then pass 1 (part B); each part's TMEM columns are
      // released as soon as they are read. Pass r, chunk q of thread half h
      // holds features r M/2 + h M/4 + 32 q.
      if (!(ok = epi_wait(bar_ffullA, i & 1, abort_flag, p.dev_status))) break;
      tc_fence_after();
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
      const int f_r0 = half * (M_ / 4), f_r1 = M_ / 2 + half * (M_ / 4);
      bool have_b = false;
      float c_old = c_run;
      if (p.shifts != nullptr) {
        // the tile's largest valid exponent (both parts, every row), then the
        // running maximum
        if (!(ok = epi_wait(bar_ffullB, i & 1, abort_flag, p.dev_status))) break;
        tc_fence_after();
        have_b = true;
        float mx = -INFINITY;
#pragma unroll 1
        for (int q = 0; q < 2 * NH; ++q) {
          float v[32];
          tmem_ld32(lane_tm + G::tP + (q < NH ? f_r0 + 32 * q : f_r1 + 32 * (q - NH)), v);
#pragma unroll
          for (int e = 0; e < 32; ++e) mx = fmaxf(mx, v[e]);
        }
        mx = warp_max(valid ? mx - nrm : -INFINITY);
        float* rr = red + 8 * (i & 1);
        if (lane == 0) rr[warp] = mx;
        epi_sync();
        float tmx = rr[0];
#pragma unroll
        for (int w = 1; w < 8; ++w) tmx = fmaxf(tmx, rr[w]);
        c_run = fmaxf(c_run, tmx);
        if (c_run > -INFINITY) nrm += c_run;
      }
      uint32_t fv[NH][32], pk[NH][16];
#pragma unroll
      for (int q = 0; q < NH; ++q) tmem_ld32_async(lane_tm + G::tP + f_r0 + 32 * q, fv[q]);
#pragma unroll
      for (int q = 0; q < NH; ++q) tmem_wait_ld(fv[q]);
      tc_fence_before();
      warp_arrive(bar_ffreeA);
#pragma unroll
      for (int q = 0; q < NH; ++q) exp2_pack32(fv[q], nrm, !valid, pk[q]);
      // ---- Phi and the state are free once the previous chunk-state GEMM is done
      if (i > 0 && !(ok = epi_wait(bar_pfree, (i - 1) & 1, abort_flag, p.dev_status))) break;
      tc_fence_after();
      if (p.shifts != nullptr && c_run > c_old && i > 0 && c_old > -INFINITY && half < G::MB) {
        // the running maximum grew: rescale the state accumulated so far
        const float sc = exp2f(c_old - c_run);
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
#pragma unroll
      for (int q = 0; q < NH; ++q) store_row32(pk[q], s0 + G::oPhi, row, f_r0 + 32 * q);
      // ---- pass 1 (part B)
      if (!have_b) {
        if (!(ok = epi_wait(bar_ffullB, i & 1, abort_flag, p.dev_status))) break;
        tc_fence_after();
      }
#pragma unroll
      for (int q = 0; q < NH; ++q) tmem_ld32_async(lane_tm + G::tP + f_r1 + 32 * q, fv[q]);
#pragma unroll
      for (int q = 0; q < NH; ++q) tmem_wait_ld(fv[q]);
      tc_fence_before();
      warp_arrive(bar_ffreeB);
#pragma unroll
      for (int q = 0; q < NH; ++q) {
        exp2_pack32(fv[q], nrm, !valid, pk[q]);
        store_row32(pk[q], s0 + G::oPhi, row, f_r1 + 32 * q);
      }
      fence_async_smem();
      tc_fence_before();
      warp_arrive(bar_pfull);
    }
    // ---- the range's state [S | z] -> partial
    if (ok && n > 0) ok = epi_wait(bar_pfree, (n - 1) & 1, abort_flag, p.dev_status);
    tc_fence_after();
    if ((ok || n == 0) && tid == 0 && p.shifts != nullptr)
      p.shifts[(size_t)bh * p.nsplit + split] = c_run;   // -inf without a valid key
    if ((ok || n == 0) && half < G::MB) {
      const int f = half * 128 + row;
      float* dst = p.partials + ((size_t)bh * p.nsplit + split) * 65 * M_;
      if (n > 0) {
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
