// Causal (and key-masked) PRF attention forward on sm_100a tensor cores.
//
// DARKformer README, section "Kernel": phi(x) = m^{-1/2} exp(omega^T M x~ -
// 1/2 |M x~|^2), out = Phi(Q)(Phi(K)^T V) / Phi(Q)(Phi(K)^T 1); section
// "Self-attention": the causal constraint (diagonal included) combined with the
// key mask. The causal form is evaluated chunkwise over 128-token chunks c:
//
//   num_c = tril(Psi(Q_c) Phi(K_c)^T) [V_c | 1] + Psi(Q_c) [S_<c | z_<c]
//   out_c = num_c[:, :d] / num_c[:, d]
//   [S_<=c | z_<=c] = [S_<c | z_<c] + Phi(K_c)^T [V_c | 1]
//
// where Psi(Q) drops the per-query factors of phi(q) (they cancel in the ratio).
// One CTA (256 threads, 8 warps) runs a chunk entirely on chip:
//   TMA loads of W', Q_c, K_c, V_c (128B-swizzled tiles)
//   -> tcgen05 feature GEMMs K_c W'^T, Q_c W^T (fp16 operands, fp32 in TMEM)
//   -> epilogue warps: key norm, exp2, key mask, bf16 Phi/Psi tiles in smem
//   -> tcgen05 GEMMs Psi Phi^T (scores) and Phi^T [V | 1] (chunk state)
//   -> causal mask of the scores -> intra GEMM tril(A) [V | 1]
//   -> prefix state (hi/lo bf16 split) -> inter GEMM Psi [S | z] -> divide.
// Phi and Psi never leave shared memory. The prefix state across chunks is
// carried in registers when one CTA walks all chunks of a head (many heads),
// or exchanged between CTAs by a decoupled look-back over per-chunk aggregates
// in the workspace (few heads); every wait there is bounded and a wait that
// runs out reports DARK_ERR_TIMEOUT instead of hanging.
#include <atomic>
#include <string.h>

#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace dark {
namespace {

using namespace tc;

constexpr int kD = 64;          // head dimension handled by this kernel
constexpr int kC = 128;         // tokens per chunk (UMMA M)
constexpr int kThreads = 256;
constexpr int kSms = 148;
constexpr int kTileBytes = kC * kD * 2;   // one 128 x 64 tile of 16-bit elements
constexpr uint32_t kTmemCols = 512;

std::atomic<uint64_t> g_call{0};

template <int M_, int R_>
struct Cfg {
  static constexpr int M = M_, R = R_, MB = M_ / 128;
  static constexpr int NW = M_ + R_;                      // W' rows
  static constexpr uint32_t kW = NW * 128;                // W' bytes (fp16, 128 B rows)
  static constexpr uint32_t kZ = (M_ / 64) * 2048;        // one z16 operand (hi or lo)
  static constexpr uint32_t kWReg = (kW > 2 * kZ ? kW : 2 * kZ);
  static constexpr uint32_t kPhi = (M_ / 64) * 16384;     // 128 tokens x M_ features, bf16
  // shared memory offsets (all 1024-byte aligned)
  static constexpr uint32_t oW = 0;
  static constexpr uint32_t oQ = (oW + kWReg + 1023) / 1024 * 1024;
  static constexpr uint32_t oK = oQ + kTileBytes;
  static constexpr uint32_t oV = oK + kTileBytes;
  static constexpr uint32_t oPhi = oV + kTileBytes;
  static constexpr uint32_t oPsi = oPhi + kPhi;
  static constexpr uint32_t oOnes = oPsi + kPhi;
  static constexpr uint32_t oBar = oOnes + 2048;
  static constexpr uint32_t kSmem = oBar + 64 + 1024;     // + alignment slack
  // TMEM columns
  static constexpr uint32_t tP = 0, tA = 0, tNum = 128, tD = 320;
  static_assert(NW <= 320 && M_ % 128 == 0 && R_ % 16 == 0, "shape");
  static_assert(tD + 80 * MB <= kTmemCols, "tmem");
};

struct Params {
  __nv_bfloat16* out;
  int64_t ob, oh, ol;           // out strides (elements)
  const uint8_t* mask;
  int B, H, L, nc;              // nc = chunks per head
  int heads_w;
  int lookback;                 // 1: one chunk per CTA + look-back; 0: one head per CTA
  uint32_t* ticket;             // workspace header word
  uint64_t* flags;              // [B*H*nc] look-back flags
  float* slots;                 // [B*H*nc][2][65][m] aggregates / inclusive prefixes
  float *st_kv, *st_z;
  uint64_t call;
  int* dev_status;
};

__device__ __forceinline__ bool wait_all(uint64_t* bar, uint32_t parity, int* dev_status) {
  const bool ok = mbar_wait(bar, parity);
  const int bad = __syncthreads_or(ok ? 0 : 1);
  if (bad && threadIdx.x == 0) report(dev_status, DARK_ERR_TIMEOUT);
  return bad == 0;
}

template <int M_, int R_>
__global__ void __launch_bounds__(kThreads, 1)
    causal_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_q,
                  const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                  const Params p) {
  using G = Cfg<M_, R_>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t s0 = smem_u32(sm);
  uint64_t* bar_tma = (uint64_t*)(sm + G::oBar);
  uint64_t* bar_mma = bar_tma + 1;
  uint32_t* tmem_slot = (uint32_t*)(bar_tma + 2);
  int* s_int = (int*)(bar_tma + 3);           // [0]: ticket, [1]: look-back state

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int quad = warp & 3, half = warp >> 2;
  const int row = quad * 32 + lane;           // TMEM lane = tile row of this thread
  const bool has_feat = half < G::MB;         // owns state row `feat`
  const int feat = half * 128 + row;

  if (tid == 0) {
    mbar_init(bar_tma, 1);
    mbar_init(bar_mma, 1);
    fence_mbar_init();
    prefetch_tmap(&tm_w);
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    if (p.lookback) {
      const uint32_t t = atomicAdd(p.ticket, 1u);
      if (t == gridDim.x - 1) atomicExch(p.ticket, 0u);   // every block has its ticket
      s_int[0] = (int)t;
    } else {
      s_int[0] = blockIdx.x;
    }
  }
  __syncwarp();
  if (warp == 0) tmem_alloc(tmem_slot, kTmemCols);
  // ones tile (bf16 1.0) for the z columns: 16 rows x 64 keys, K-major
  for (int i = tid; i < 2048 / 4; i += kThreads) ((uint32_t*)(sm + G::oOnes))[i] = 0x3F803F80u;
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_tm = tmem + ((uint32_t)(quad * 32) << 16);
  const int unit = s_int[0];
  int bh, c_begin, c_end;
  if (p.lookback) {
    bh = unit / p.nc;
    c_begin = unit % p.nc;
    c_end = c_begin + 1;
  } else {
    bh = unit;
    c_begin = 0;
    c_end = p.nc;
  }
  const int b = bh / p.H, h = bh % p.H;
  const int hw = p.heads_w == 1 ? 0 : h;

  uint32_t ph_tma = 0, ph_mma = 0;
  float run[65];                               // prefix state row `feat` (fp32)
#pragma unroll
  for (int i = 0; i < 65; ++i) run[i] = 0.f;
  bool abort = false;

  for (int c = c_begin; c < c_end && !abort; ++c) {
    const int t0 = c * kC;
    // ---------------------------------------------------------------- loads
    if (tid == 0) {
      const bool load_w = (c == c_begin) || !p.lookback;
      mbar_arrive_expect_tx(bar_tma, (load_w ? G::kW : 0) + 3 * kTileBytes);
      if (load_w)
        for (int r0 = 0; r0 < G::NW; r0 += 16)
          tma_load_2d(sm + G::oW + r0 * 128, &tm_w, 0, hw * G::NW + r0, bar_tma);
      tma_load_4d(sm + G::oK, &tm_k, 0, t0, h, b, bar_tma);
      tma_load_4d(sm + G::oV, &tm_v, 0, t0, h, b, bar_tma);
      tma_load_4d(sm + G::oQ, &tm_q, 0, t0, h, b, bar_tma);
    }
    if (!wait_all(bar_tma, ph_tma, p.dev_status)) { abort = true; break; }
    ph_tma ^= 1;
    // q, k: bf16 -> fp16 in place (the feature GEMM runs on fp16 operands)
    {
      bool bad = false;
      for (int i = tid; i < 2 * kTileBytes / 16; i += kThreads) {
        const uint32_t a = s0 + G::oQ + i * 16;        // Q then K (contiguous)
        uint4 u = ld_shared_v4(a);
        uint32_t* w32 = &u.x;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const __nv_bfloat162 bv = *reinterpret_cast<const __nv_bfloat162*>(&w32[e]);
          const float2 f = __bfloat1622float2(bv);
          bad |= fabsf(f.x) > 65504.f || fabsf(f.y) > 65504.f;
          const __half2 hv = __floats2half2_rn(f.x, f.y);
          w32[e] = *reinterpret_cast<const uint32_t*>(&hv);
        }
        st_shared_v4(a, u.x, u.y, u.z, u.w);
      }
      if (bad) report(p.dev_status, DARK_ERR_NUMERIC);
    }
    fence_async_smem();
    __syncthreads();
    // ------------------------------------------------------- feature GEMM K
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t idn0 = idesc(128, (G::NW < 256 ? G::NW : 256), false, false, true);
      constexpr uint32_t idn1 = idesc(128, (G::NW > 256 ? G::NW - 256 : 16), false, false, true);
#pragma unroll
      for (int s = 0; s < kD / 16; ++s) {
        const uint64_t ad = sdesc(s0 + G::oK + s * 32, 16, 1024);
        mma(tmem + G::tP, ad, sdesc(s0 + G::oW + s * 32, 16, 1024), idn0, s > 0);
        if (G::NW > 256)
          mma(tmem + G::tP + 256, ad, sdesc(s0 + G::oW + 256 * 128 + s * 32, 16, 1024), idn1, s > 0);
      }
      mma_commit(bar_mma);
    }
    if (!wait_all(bar_mma, ph_mma, p.dev_status)) { abort = true; break; }
    ph_mma ^= 1;
    tc_fence_after();
    // ------------------------------------------------- epilogue: Phi(K_c)
    {
      float nrm = 0.f;
#pragma unroll
      for (int c0 = 0; c0 < R_; c0 += 16) {
        float v[16];
        tmem_ld16(lane_tm + G::tP + M_ + c0, v);
#pragma unroll
        for (int i = 0; i < 16; ++i) nrm = fmaf(v[i], v[i], nrm);
      }
      nrm += 0.5f * __log2f((float)M_);
      const int tok = t0 + row;
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
            const float bb = valid ? ex2(v[8 * g + 2 * e + 1] - nrm) : 0.f;
            w4[e] = pack_bf16(a, bb);
          }
          const int f = f0 + 8 * g;
          st_shared_v4(s0 + G::oPhi + kmajor_off(row, f, 16384), w4[0], w4[1], w4[2], w4[3]);
        }
      }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    // ------------------------------------------------------- feature GEMM Q
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t idq = idesc(128, (M_ < 256 ? M_ : 256), false, false, true);
#pragma unroll
      for (int s = 0; s < kD / 16; ++s)
        mma(tmem + G::tP, sdesc(s0 + G::oQ + s * 32, 16, 1024),
            sdesc(s0 + G::oW + s * 32, 16, 1024), idq, s > 0);
      mma_commit(bar_mma);
    }
    if (!wait_all(bar_mma, ph_mma, p.dev_status)) { abort = true; break; }
    ph_mma ^= 1;
    tc_fence_after();
    // ------------------------------------------------- epilogue: Psi(Q_c)
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
    // -------------------------------- scores Psi Phi^T and chunk state Phi^T [V|1]
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t ids = idesc(128, 128, false, false, false);
#pragma unroll
      for (int s = 0; s < M_ / 16; ++s) {
        const uint32_t off = (s / 4) * 16384 + (s % 4) * 32;
        mma(tmem + G::tA, sdesc(s0 + G::oPsi + off, 16, 1024), sdesc(s0 + G::oPhi + off, 16, 1024),
            ids, s > 0);
      }
      constexpr uint32_t idv = idesc(128, 64, true, true, false);
      constexpr uint32_t id1 = idesc(128, 16, true, false, false);
#pragma unroll
      for (int mb = 0; mb < G::MB; ++mb) {
#pragma unroll
        for (int s = 0; s < kC / 16; ++s) {
          const uint64_t ad = sdesc(s0 + G::oPhi + mb * 32768 + s * 2048, 16384, 1024);
          mma(tmem + G::tD + 80 * mb, ad, sdesc(s0 + G::oV + s * 2048, 16384, 1024), idv, s > 0);
          mma(tmem + G::tD + 80 * mb + 64, ad, sdesc(s0 + G::oOnes + (s % 4) * 32, 16, 1024), id1,
              s > 0);
        }
      }
      mma_commit(bar_mma);
    }
    if (!wait_all(bar_mma, ph_mma, p.dev_status)) { abort = true; break; }
    ph_mma ^= 1;
    tc_fence_after();
    // ----------------------- causal mask of the scores -> bf16 A operand (Q/K tiles)
    {
      float v[32];
#pragma unroll
      for (int j0 = half * 64; j0 < half * 64 + 64; j0 += 32) {
        tmem_ld32(lane_tm + G::tA + j0, v);
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          uint32_t w4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int j = j0 + 8 * g + 2 * e;
            w4[e] = pack_bf16(j <= row ? v[8 * g + 2 * e] : 0.f, j + 1 <= row ? v[8 * g + 2 * e + 1] : 0.f);
          }
          st_shared_v4(s0 + G::oQ + kmajor_off(row, j0 + 8 * g, 16384), w4[0], w4[1], w4[2], w4[3]);
        }
      }
    }
    // chunk state row `feat` (the aggregate of this chunk)
    float ds[65];
    if (has_feat) {
      float v[32];
      const uint32_t base = tmem + ((uint32_t)(quad * 32) << 16) + G::tD + 80 * half;
      tmem_ld32(base, v);
#pragma unroll
      for (int i = 0; i < 32; ++i) ds[i] = v[i];
      tmem_ld32(base + 32, v);
#pragma unroll
      for (int i = 0; i < 32; ++i) ds[32 + i] = v[i];
      ds[64] = tmem_ld1(base + 64);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    // -------------------------------------------- intra-chunk GEMM tril(A) [V|1]
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t idv = idesc(128, 64, false, true, false);
      constexpr uint32_t id1 = idesc(128, 16, false, false, false);
#pragma unroll
      for (int s = 0; s < kC / 16; ++s) {
        const uint64_t ad = sdesc(s0 + G::oQ + (s / 4) * 16384 + (s % 4) * 32, 16, 1024);
        mma(tmem + G::tNum, ad, sdesc(s0 + G::oV + s * 2048, 16384, 1024), idv, s > 0);
        mma(tmem + G::tNum + 64, ad, sdesc(s0 + G::oOnes + (s % 4) * 32, 16, 1024), id1, s > 0);
      }
    }
    // ---------------------------------------------------------- prefix state
    bool have_prefix;
    if (p.lookback) {
      const size_t unit_idx = (size_t)bh * p.nc + c;
      float* slot_agg = p.slots + unit_idx * 2 * 65 * M_;
      float* slot_inc = slot_agg + 65 * M_;
      // publish the aggregate (chunk 0: it is already the inclusive prefix)
      if (has_feat) {
        float* dst = c == 0 ? slot_inc : slot_agg;
#pragma unroll
        for (int i = 0; i < 65; ++i) __stcg(dst + i * M_ + feat, ds[i]);
      }
      __threadfence();
      __syncthreads();
      if (tid == 0) st_release_u64(p.flags + unit_idx, (p.call << 2) | (c == 0 ? 2u : 1u));
      // look back over the predecessors of this chunk
      for (int pc = c - 1; pc >= 0; --pc) {
        if (tid == 0) {
          const uint64_t* fl = p.flags + (size_t)bh * p.nc + pc;
          uint64_t f = ld_acquire_u64(fl);
          const long long start = clock64();
          while ((f >> 2) != p.call || (f & 3) == 0) {
            if (clock64() - start > kWaitCycles) { f = 0; break; }
            __nanosleep(64);
            f = ld_acquire_u64(fl);
          }
          if (f == 0) report(p.dev_status, DARK_ERR_TIMEOUT);
          s_int[1] = (int)(f & 3);
        }
        __syncthreads();
        const int st = s_int[1];
        __syncthreads();
        if (st == 0) break;
        const float* src = p.slots + ((size_t)bh * p.nc + pc) * 2 * 65 * M_ + (st == 2 ? 65 * M_ : 0);
        if (has_feat) {
#pragma unroll
          for (int i = 0; i < 65; ++i) run[i] += __ldcg(src + i * M_ + feat);
        }
        if (st == 2) break;
      }
      have_prefix = c > 0;
      // publish the inclusive prefix
      if (c > 0) {
        if (has_feat) {
#pragma unroll
          for (int i = 0; i < 65; ++i) __stcg(slot_inc + i * M_ + feat, run[i] + ds[i]);
        }
        __threadfence();
        __syncthreads();
        if (tid == 0) st_release_u64(p.flags + unit_idx, (p.call << 2) | 2u);
      }
      if (c == p.nc - 1 && p.st_kv != nullptr && has_feat) {
        float* kv = p.st_kv + ((size_t)bh * M_ + feat) * kD;
#pragma unroll
        for (int i = 0; i < 64; ++i) kv[i] = run[i] + ds[i];
        p.st_z[(size_t)bh * M_ + feat] = run[64] + ds[64];
      }
    } else {
      have_prefix = c > 0;
    }
    // prefix [S | z] as hi + lo bf16 operands: S (MN-major) in the Phi region,
    // z (16 identical K-major rows) in the W' region
    if (have_prefix && has_feat) {
      const uint32_t sh = s0 + G::oPhi, sl = sh + M_ * 128;
      const uint32_t rowoff = (uint32_t)(feat / 8) * 1024 + (uint32_t)(feat % 8) * 128;
#pragma unroll
      for (int cg = 0; cg < 8; ++cg) {
        uint32_t hi4[4], lo4[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float x0 = run[8 * cg + 2 * e], x1 = run[8 * cg + 2 * e + 1];
          const __nv_bfloat162 hv = __floats2bfloat162_rn(x0, x1);
          const float2 hf = __bfloat1622float2(hv);
          hi4[e] = *reinterpret_cast<const uint32_t*>(&hv);
          lo4[e] = pack_bf16(x0 - hf.x, x1 - hf.y);
        }
        const uint32_t off = rowoff + (uint32_t)((cg ^ (feat % 8)) * 16);
        st_shared_v4(sh + off, hi4[0], hi4[1], hi4[2], hi4[3]);
        st_shared_v4(sl + off, lo4[0], lo4[1], lo4[2], lo4[3]);
      }
      const __nv_bfloat16 zh = __float2bfloat16_rn(run[64]);
      const __nv_bfloat16 zl = __float2bfloat16_rn(run[64] - __bfloat162float(zh));
      const uint16_t zhb = *reinterpret_cast<const uint16_t*>(&zh);
      const uint16_t zlb = *reinterpret_cast<const uint16_t*>(&zl);
      const uint32_t zh_base = s0 + G::oW, zl_base = zh_base + G::kZ;
#pragma unroll
      for (int n = 0; n < 16; ++n) {
        const uint32_t off = (uint32_t)(feat / 64) * 2048 + kmajor_off(n, feat % 64, 0);
        st_shared_u16(zh_base + off, zhb);
        st_shared_u16(zl_base + off, zlb);
      }
    }
    if (!p.lookback && has_feat) {
#pragma unroll
      for (int i = 0; i < 65; ++i) run[i] += ds[i];
    }
    fence_async_smem();
    __syncthreads();
    // -------------------------------------------------- inter-chunk GEMM Psi [S|z]
    if (tid == 0) {
      tc_fence_after();
      if (have_prefix) {
        constexpr uint32_t idv = idesc(128, 64, false, true, false);
        constexpr uint32_t id1 = idesc(128, 16, false, false, false);
#pragma unroll
        for (int part = 0; part < 2; ++part) {
          const uint32_t sb = s0 + G::oPhi + part * M_ * 128;
          const uint32_t zb = s0 + G::oW + part * G::kZ;
#pragma unroll
          for (int s = 0; s < M_ / 16; ++s) {
            const uint64_t ad = sdesc(s0 + G::oPsi + (s / 4) * 16384 + (s % 4) * 32, 16, 1024);
            mma(tmem + G::tNum, ad, sdesc(sb + s * 2048, 16384, 1024), idv, 1);
            mma(tmem + G::tNum + 64, ad, sdesc(zb + (s / 4) * 2048 + (s % 4) * 32, 16, 1024), id1, 1);
          }
        }
      }
      mma_commit(bar_mma);
    }
    if (!wait_all(bar_mma, ph_mma, p.dev_status)) { abort = true; break; }
    ph_mma ^= 1;
    tc_fence_after();
    // ------------------------------------------------------------- output
    {
      const float den = tmem_ld1(lane_tm + G::tNum + 64);
      float v[32];
      tmem_ld32(lane_tm + G::tNum + half * 32, v);
      const int tok = t0 + row;
      if (tok < p.L) {
        const float inv = den > 0.f ? 1.f / den : 0.f;
        uint32_t w[16];
        bool bad = false;
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float a = v[2 * e] * inv, bb = v[2 * e + 1] * inv;
          bad |= !isfinite(a) || !isfinite(bb);
          w[e] = pack_bf16(a, bb);
        }
        if (bad || !isfinite(den)) report(p.dev_status, DARK_ERR_NUMERIC);
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
  if (!abort && !p.lookback && p.st_kv != nullptr && has_feat) {
    float* kv = p.st_kv + ((size_t)bh * M_ + feat) * kD;
#pragma unroll
    for (int i = 0; i < 64; ++i) kv[i] = run[i];
    p.st_z[(size_t)bh * M_ + feat] = run[64];
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

struct Layout {
  int nc, lookback;
  size_t off_flags, off_slots, total;
};

Layout layout(int B, int H, int L, int m) {
  Layout s;
  s.nc = (L + kC - 1) / kC;
  s.lookback = (B * H < kSms) ? 1 : 0;
  const size_t units = (size_t)B * H * s.nc;
  s.off_flags = kWsHeader;
  s.off_slots = align_up(s.off_flags + (s.lookback ? units * 8 : 0), 256);
  s.total = align_up(s.off_slots + (s.lookback ? units * 2 * 65 * (size_t)m * 4 : 0), 256);
  return s;
}

template <int M_, int R_>
cudaError_t launch(const FwdArgs& a, const CUtensorMap& tw, const CUtensorMap& tq,
                   const CUtensorMap& tk, const CUtensorMap& tv) {
  using G = Cfg<M_, R_>;
  const Layout s = layout(a.B, a.H, a.L, a.m);
  Params p;
  memset(&p, 0, sizeof(p));
  p.out = (__nv_bfloat16*)a.out;
  p.ob = a.os[0];
  p.oh = a.os[1];
  p.ol = a.os[2];
  p.mask = a.mask;
  p.B = a.B;
  p.H = a.H;
  p.L = a.L;
  p.nc = s.nc;
  p.heads_w = a.heads_w;
  p.lookback = s.lookback;
  p.ticket = (uint32_t*)a.ws;
  p.flags = (uint64_t*)((char*)a.ws + s.off_flags);
  p.slots = (float*)((char*)a.ws + s.off_slots);
  p.st_kv = a.st_kv;
  p.st_z = a.st_z;
  p.call = ++g_call;
  p.dev_status = a.dev_status;
  cudaError_t e = cudaFuncSetAttribute(causal_kernel<M_, R_>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)G::kSmem);
  if (e != cudaSuccess) return e;
  const int grid = s.lookback ? a.B * a.H * s.nc : a.B * a.H;
  causal_kernel<M_, R_><<<grid, kThreads, G::kSmem, a.stream>>>(tw, tq, tk, tv, p);
  return cudaGetLastError();
}

bool make_maps(const FwdArgs& a, CUtensorMap* tw, CUtensorMap* tq, CUtensorMap* tk, CUtensorMap* tv) {
  const uint64_t wd[2] = {(uint64_t)a.d, (uint64_t)a.heads_w * (a.m + a.r)};
  const uint64_t ws[1] = {(uint64_t)a.d * 2};
  const uint32_t wb[2] = {64, 16};
  if (!encode_tmap(tw, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, a.w, wd, ws, wb)) return false;
  const uint64_t xd[4] = {(uint64_t)a.d, (uint64_t)a.L, (uint64_t)a.H, (uint64_t)a.B};
  const uint64_t xs[3] = {(uint64_t)a.qs[2] * 2, (uint64_t)a.qs[1] * 2, (uint64_t)a.qs[0] * 2};
  const uint32_t xb[4] = {64, (uint32_t)kC, 1, 1};
  return encode_tmap(tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, a.q, xd, xs, xb) &&
         encode_tmap(tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, a.k, xd, xs, xb) &&
         encode_tmap(tv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, a.v, xd, xs, xb);
}

bool aligned16(const void* ptr) { return ((uintptr_t)ptr & 15) == 0; }

}  // namespace

bool tc_causal_supported(const FwdArgs& a) {
  if (a.dtype != DARK_BF16 || a.d != kD || (a.flags & DARK_STABILISE)) return false;
  if (!(a.m == 128 || a.m == 256) || a.r % 16 != 0 || a.r < 16 || a.r > 64) return false;
  if (!aligned16(a.q) || !aligned16(a.k) || !aligned16(a.v) || !aligned16(a.out) || !aligned16(a.w))
    return false;
  for (int i = 0; i < 3; ++i)
    if (a.qs[i] % 8 != 0 || a.os[i] % 8 != 0) return false;
  CUtensorMap t[4];
  return make_maps(a, &t[0], &t[1], &t[2], &t[3]);
}

size_t tc_causal_workspace_bytes(int B, int H, int L, int m, int d) {
  if (d != kD || !(m == 128 || m == 256)) return 0;
  return layout(B, H, L, m).total;
}

cudaError_t tc_causal_forward(const FwdArgs& a) {
  CUtensorMap tw, tq, tk, tv;
  if (!make_maps(a, &tw, &tq, &tk, &tv)) return cudaErrorInvalidValue;
#define DARK_CAUSAL_CASE(MM, RR) \
  if (a.m == MM && a.r == RR) return launch<MM, RR>(a, tw, tq, tk, tv);
  DARK_CAUSAL_CASE(256, 64)
  DARK_CAUSAL_CASE(256, 48)
  DARK_CAUSAL_CASE(256, 32)
  DARK_CAUSAL_CASE(256, 16)
  DARK_CAUSAL_CASE(128, 64)
  DARK_CAUSAL_CASE(128, 48)
  DARK_CAUSAL_CASE(128, 32)
  DARK_CAUSAL_CASE(128, 16)
#undef DARK_CAUSAL_CASE
  return cudaErrorInvalidValue;
}

}  // namespace dark
