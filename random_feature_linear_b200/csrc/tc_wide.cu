// Causal (and key-masked) PRF attention forward for wide heads (d = 128..256,
// m up to 512) on sm_100a tensor cores.
//
// DARKformer README, section "Kernel": phi(x) = m^{-1/2} exp(omega^T M x~ -
// 1/2 |M x~|^2) and out = Phi(Q)(Phi(K)^T V) / Phi(Q)(Phi(K)^T 1); section
// "Self-attention": the causal constraint (diagonal included) combined with the
// key mask. Per 128-token chunk c (Psi drops the per-query factors of phi):
//
//   num_c = tril(Psi(Q_c) Phi(K_c)^T) [V_c | 1] + Psi(Q_c) [S_<c | z_<c]
//   out_c = num_c[:, :d] / num_c[:, d]
//   [S_<=c | z_<=c] = [S_<c | z_<c] + Phi(K_c)^T [V_c | 1]
//
// At d = 256, m = 512 one head's state [S | z] is 512 x 257 fp32 (526 KB),
// more than one SM's shared memory or TMEM, so it cannot ride along with one
// CTA as in the d = 64 kernel. The work is split in two launches:
//
//  1. features_kernel, persistent (one CTA per SM walking a contiguous range of
//     (head, chunk) items): per item the key norms, then per 128-feature block
//     one N = 256 MMA chain over the chunk's keys and queries together (the W'
//     block is the M = 128 operand); the epilogue warps turn the block into
//     Phi(K_c), Psi(Q_c) (bf16), the scores Psi Phi^T accumulate on the tensor
//     cores block by block, and Phi, Psi, the masked causal scores A_c, the
//     chunk's key-feature sums and the row sums of A_c go to the workspace as
//     ready shared-memory operand images (128B-swizzled, so the second launch
//     copies them back verbatim).
//  2. values_kernel, one CTA per (head, 128 value columns, feature half), the
//     two feature halves of a (head, value block) forming a 2-CTA cluster: each
//     CTA walks the chunks in order with its 256 x 128 block of the state in
//     TMEM; per chunk the epilogue warps copy S to shared memory as hi + lo
//     bf16 operands (bf16 alone moves outputs by ~1e-2), the tensor cores run
//       num = A_c [V_c] + Psi [S hi | S lo]   and   S += Phi^T V_c,
//     the denominators come from the key sums on the CUDA cores, and the two
//     halves exchange their partial outputs through distributed shared memory.
//
// The stabiliser (DARK_STABILISE) adds a statistics pass of the features
// kernel before the features: the same GEMMs with an epilogue that only takes
// maxima, the largest valid key exponent of every (b, h) and the largest
// exponent of every query. The features pass subtracts them before exp2, so
// every image, key sum and score is relative to those constants and the values
// launch runs unchanged; the key constant is the state's shift.
//
// In both kernels warp 9 is the producer (TMA / bulk copies), warp 8 issues
// the MMAs and warps 0-7 are the epilogue (TMEM lane quadrant = warp % 4). Every
// wait is bounded: a wait that runs out records DARK_ERR_TIMEOUT and raises the
// CTA's abort flag, every role leaves its loop, in-flight copies are waited for
// (bounded), and TMEM is freed.
#include <string.h>

#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"
#include "tc_roles.cuh"

namespace dark {
namespace {

using namespace tc;

constexpr int kC = 128;              // tokens per chunk (UMMA M)
constexpr int kEpiThreads = 256;     // warps 0-7
constexpr int kThreadsF = kEpiThreads + 64;   // + MMA warp 8 + producer warp 9
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSmemBudget = 229376;   // 224 KB of operands + barriers + alignment slack

// ----------------------------------------------------------- bulk copies --
// shared -> global bulk copy (16-byte aligned, size a multiple of 16) with an
// L2 eviction policy for the written lines
__device__ __forceinline__ void bulk_store_hint(void* gdst, uint32_t ssrc, uint32_t bytes,
                                                uint64_t policy) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group.L2::cache_hint [%0], [%1], %2, %3;" ::"l"(
                   (uint64_t)gdst),
               "r"(ssrc), "r"(bytes), "l"(policy)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_read_all() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}
// ================================================================ launch 1 ==
// Persistent: each CTA walks a contiguous range of (head, chunk) items. Per
// item the key and query tiles sit side by side in shared memory as one
// 256-token operand [K_c ; Q_c] (fp16, d in 64-column slabs), so that every
// feature GEMM is a full-width MMA: W'_f (128 feature rows, M = 128) times the
// 256 tokens (N = 256), accumulated over d. The TMEM result holds feature f of
// the block in lane f and token t in column t (keys 0-127, queries 128-255),
// which is exactly the layout the value launch wants for its operands:
// Phi_f^T with features as rows (the A operand of the state update) and
// Psi_f^T with features as rows (the MN-major A operand of the prefix
// product). The key norms come first from a tokens x r GEMM (keys as M) and go
// to shared memory as one base-2 offset per key, +inf for masked keys (whose
// features are then exp2(-inf) = 0).
template <int D_, int M_, int R_>
struct FeatCfg {
  static constexpr int DS = D_ / 64;                     // 64-column slabs of d
  static constexpr int NB = M_ / 128;                    // feature blocks of 128
  static constexpr int NRH = R_ > 128 ? R_ / 128 : 1;    // norm row groups per slab
  static constexpr int NRROWS = R_ > 128 ? 128 : R_;     // rows per norm item
  static constexpr int NNORM = DS * NRH;                 // ring items: norm rows first,
  static constexpr int NITEMS = NNORM + NB * DS;         // then W' block f, slab s
  static constexpr uint32_t kXSlab = 32768;              // 256 token rows x 128 B
  static constexpr uint32_t oX = 0;
  static constexpr uint32_t oST = DS * kXSlab;           // staging: Phi_f | Psi_f (32 KB each)
  static constexpr uint32_t oW = oST + 65536;            // ring of 16 KB slots
  static constexpr int kSlotsFit = (int)((kSmemBudget - oW) / 16384);
  static constexpr int NSLOT = kSlotsFit > 6 ? 6 : kSlotsFit;
  static constexpr uint32_t oBar = oW + NSLOT * 16384;
  static constexpr uint32_t kSmem = oBar + 2048 + 1024;  // barriers, norms, exchange, slack
  static constexpr uint32_t tF = 0, tN = 256;            // TMEM: F block | norms, then scores
  static_assert(D_ % 64 == 0 && D_ >= 128 && D_ <= 256, "d");
  static_assert(M_ % 128 == 0 && M_ <= 512, "m");
  static_assert(R_ % 64 == 0 && R_ >= 64 && R_ <= 256, "r");
  static_assert(NSLOT >= 2, "shared memory");
};

// One chunk's record in the workspace: the Phi image (m/128 blocks of 128
// features x 128 tokens), the Psi image (the same), the masked score image A
// (128 queries x 128 keys), dz = the chunk's key-feature sums (m floats) and
// the row sums of A over keys 0-63 and over keys 64-127 (2 x 128 floats).
__host__ __device__ constexpr size_t chunk_dz_off(int m) { return (size_t)2 * m * 256 + 32768; }
__host__ __device__ constexpr size_t chunk_den_off(int m) { return chunk_dz_off(m) + (size_t)4 * m; }
__host__ __device__ constexpr size_t chunk_record_bytes(int m) { return chunk_den_off(m) + 1024; }

struct FeatParams {
  const uint8_t* mask;
  uint8_t* img;            // chunk records [B*H][nc]
  int B, H, L, nc, heads_w, nitems;
  // stabiliser: per-(b,h) key maximum as an order-preserving integer (zero
  // before the statistics pass), per-query maxima [B*H][nc*128], the state's
  // key constant (state output, or null)
  unsigned* kmax;
  float* qc;
  float* st_shift;
  int* dev_status;
  long long stall;         // testing stall before the first wait (0: none)
};

// The three forms of the features launch: plain; the statistics pass of the
// stabiliser (feature exponents only: per-(b,h) maximum of the valid key
// exponents, per-query maximum of the query exponents; no images); and the
// stabilised pass, which subtracts those maxima before exp2.
constexpr int kPlain = 0, kStats = 1, kStab = 2;

// float <-> unsigned with the order of the floats (for integer max reductions);
// 0 lies below every float, -inf included
__device__ __forceinline__ unsigned f2ord(float f) {
  const unsigned u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float ord2f(unsigned o) {
  return __uint_as_float((o & 0x80000000u) ? (o & 0x7fffffffu) : ~o);
}

template <int D_, int M_, int R_, int MODE>
__global__ void __launch_bounds__(kThreadsF, 1)
    features_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k, const FeatParams p) {
  using G = FeatCfg<D_, M_, R_>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t s0 = smem_u32(sm);
  uint64_t* bars = (uint64_t*)(sm + G::oBar);
  uint64_t* bar_x = bars + 0;       // producer: token tiles loaded
  uint64_t* bar_conv = bars + 1;    // epilogue: tiles converted; TMEM norm/score region free (8)
  uint64_t* bar_norm = bars + 2;    // MMA: norm GEMM done
  uint64_t* bar_nread = bars + 3;   // epilogue: norms read (8)
  uint64_t* bar_ffull = bars + 4;   // MMA: feature block in TMEM
  uint64_t* bar_ffree = bars + 5;   // epilogue: feature block read (8)
  uint64_t* bar_stage = bars + 6;   // epilogue: Phi_f, Psi_f staged (8)
  uint64_t* bar_sfree = bars + 7;   // MMA: scores GEMM of the staged block done
  uint64_t* bar_xfree = bars + 8;   // MMA: every GEMM reading the token tiles done
  uint64_t* bar_sc = bars + 9;      // MMA: scores complete
  uint64_t* bar_drain = bars + 10;  // MMA: everything issued has completed (abort path)
  uint64_t* bar_never = bars + 11;  // completed by nothing (testing stall)
  uint64_t* bar_full = bars + 16;   // [NSLOT] ring slot loaded
  uint64_t* bar_empty = bars + 24;  // [NSLOT] ring slot read by the MMAs
  uint32_t* tmem_slot = (uint32_t*)(bars + 32);
  volatile int* abort_flag = (volatile int*)(bars + 33);
  float* nrm_s = (float*)(sm + G::oBar + 1024);          // [128] key offsets
  float* nrm_x = (float*)(sm + G::oBar + 1536);          // [128] second half sums
  // stabiliser: the chunk's query maxima (statistics pass: order-preserving
  // integers; stabilised pass: floats)
  unsigned* qmax_s = (unsigned*)(sm + G::oBar + 512);
  float* qc_s = (float*)(sm + G::oBar + 512);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // this CTA's contiguous range of (head, chunk) items
  const int per = p.nitems / gridDim.x, extra = p.nitems % gridDim.x;
  const int it0 = blockIdx.x * per + (blockIdx.x < extra ? blockIdx.x : extra);
  const int nit = per + (blockIdx.x < extra ? 1 : 0);

  if (tid == 0) {
    mbar_init(bar_x, 1);
    mbar_init(bar_conv, 8);
    mbar_init(bar_norm, 1);
    mbar_init(bar_nread, 8);
    mbar_init(bar_ffull, 1);
    mbar_init(bar_ffree, 8);
    mbar_init(bar_stage, 8);
    mbar_init(bar_sfree, 1);
    mbar_init(bar_xfree, 1);
    mbar_init(bar_sc, 1);
    mbar_init(bar_drain, 1);
    mbar_init(bar_never, 1);
    for (int i = 0; i < G::NSLOT; ++i) {
      mbar_init(bar_full + i, 1);
      mbar_init(bar_empty + i, 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(tmem_slot, kTmemCols);
  if (MODE == kStats && tid < kC) qmax_s[tid] = 0u;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 9) {
    // ------------------------------------------------------------ producer
    // per item: the token tiles (once the previous item's GEMMs have read
    // them), then the ring items in consumption order
    if (lane == 0) {
      prefetch_tmap(&tm_w);
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      // projection rows are re-read for every chunk: keep them in L2
      const uint64_t keep = l2_evict_last(), once = l2_evict_first();
      int last[G::NSLOT];
      for (int i = 0; i < G::NSLOT; ++i) last[i] = -1;
      bool ok = true;
      int xlast = -1;
      int g = 0;   // ring items issued so far (over all items)
      for (int j = 0; ok && j < nit; ++j) {
        const int item = it0 + j, bh = item / p.nc, c = item % p.nc;
        const int b = bh / p.H, h = bh % p.H, hw = p.heads_w == 1 ? 0 : h;
        if (j > 0 && !(ok = wait_one(bar_xfree, (j - 1) & 1, abort_flag, p.dev_status))) break;
        mbar_arrive_expect_tx(bar_x, 2 * G::DS * 16384);
        for (int s = 0; s < G::DS; ++s) {
          tma_load_4d_hint(sm + G::oX + s * G::kXSlab, &tm_k, 64 * s, c * kC, h, b, bar_x, once);
          tma_load_4d_hint(sm + G::oX + s * G::kXSlab + 16384, &tm_q, 64 * s, c * kC, h, b, bar_x,
                           once);
        }
        xlast = j;
        for (int i = 0; i < G::NITEMS; ++i, ++g) {
          const int slot = g % G::NSLOT;
          if (g >= G::NSLOT &&
              !(ok = wait_one(bar_empty + slot, ((g / G::NSLOT) - 1) & 1, abort_flag, p.dev_status)))
            break;
          uint8_t* dst = sm + G::oW + slot * 16384;
          const int wrow0 = hw * (M_ + R_);
          if (i < G::NNORM) {          // norm rows: slab i / NRH, row group i % NRH
            const int s = i / G::NRH, rg = i % G::NRH;
            mbar_arrive_expect_tx(bar_full + slot, G::NRROWS * 128);
            for (int q = 0; q < G::NRROWS / 64; ++q)
              tma_load_2d_hint(dst + q * 8192, &tm_w, 64 * s, wrow0 + M_ + rg * 128 + 64 * q,
                               bar_full + slot, keep);
          } else {                     // feature rows of block f, d slab s
            const int f = (i - G::NNORM) / G::DS, s = (i - G::NNORM) % G::DS;
            mbar_arrive_expect_tx(bar_full + slot, 16384);
            tma_load_2d_hint(dst, &tm_w, 64 * s, wrow0 + 128 * f, bar_full + slot, keep);
            tma_load_2d_hint(dst + 8192, &tm_w, 64 * s, wrow0 + 128 * f + 64, bar_full + slot, keep);
          }
          last[slot] = g;
        }
      }
      if (!ok) {
        // leave no copy in flight (a completed phase passes at once)
        if (xlast >= 0) mbar_wait(bar_x, xlast & 1);
        for (int i = 0; i < G::NSLOT; ++i)
          if (last[i] >= 0) mbar_wait(bar_full + i, (last[i] / G::NSLOT) & 1);
      }
    }
    __syncwarp();
  } else if (warp == 8) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      bool ok = true;
      int g = 0, nblk = 0;   // ring items consumed, feature blocks issued (all items)
      auto wait_item = [&](int gi) -> bool {
        return wait_one(bar_full + gi % G::NSLOT, (gi / G::NSLOT) & 1, abort_flag, p.dev_status);
      };
      auto slot_addr = [&](int gi) -> uint32_t { return s0 + G::oW + (gi % G::NSLOT) * 16384; };
      // scores += Psi_f Phi_f^T from the staging (both MN-major, features as K)
      auto scores = [&](int f) {
        constexpr uint32_t id = idesc(128, 128, true, true, false);
#pragma unroll
        for (int k = 0; k < 8; ++k)
          mma(tmem + G::tN, sdesc(s0 + G::oST + 32768 + k * 2048, 16384, 1024),
              sdesc(s0 + G::oST + k * 2048, 16384, 1024), id, (f | k) != 0);
        mma_commit(bar_sfree);
      };
      for (int j = 0; ok && j < nit; ++j) {
        if (!(ok = wait_one(bar_conv, j & 1, abort_flag, p.dev_status))) break;
        tc_fence_after();
        // ---- key norms: (keys x d) (d x r), r in groups of up to 128 columns
        for (int i = 0; ok && i < G::NNORM; ++i, ++g) {
          const int s = i / G::NRH, rg = i % G::NRH;
          if (!(ok = wait_item(g))) break;
          tc_fence_after();
          constexpr uint32_t id = idesc(128, G::NRROWS, false, false, true);
          const uint32_t sw = slot_addr(g), sx = s0 + G::oX + s * G::kXSlab;
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mma(tmem + G::tN + 128 * rg, sdesc(sx + k * 32, 16, 1024), sdesc(sw + k * 32, 16, 1024),
                id, (s | k) != 0);
          mma_commit(bar_empty + g % G::NSLOT);
        }
        if (!ok) break;
        mma_commit(bar_norm);
        // ---- feature blocks: F = W'_f [K_c ; Q_c]^T, one N = 256 MMA per K-step
        for (int f = 0; ok && f < G::NB; ++f, ++nblk) {
          if (nblk > 0 && !(ok = wait_one(bar_ffree, (nblk - 1) & 1, abort_flag, p.dev_status)))
            break;
          tc_fence_after();
          constexpr uint32_t id = idesc(128, 256, false, false, true);
          for (int s = 0; ok && s < G::DS; ++s, ++g) {
            if (!(ok = wait_item(g))) break;
            tc_fence_after();
            const uint32_t sw = slot_addr(g), sx = s0 + G::oX + s * G::kXSlab;
#pragma unroll
            for (int k = 0; k < 4; ++k)
              mma(tmem + G::tF, sdesc(sw + k * 32, 16, 1024), sdesc(sx + k * 32, 16, 1024), id,
                  (s | k) != 0);
            mma_commit(bar_empty + g % G::NSLOT);
          }
          if (!ok) break;
          mma_commit(bar_ffull);
          if (f == G::NB - 1) mma_commit(bar_xfree);
          // scores of the previous block, staged meanwhile by the epilogue
          if (MODE != kStats && f > 0) {
            if (f == 1 && !(ok = wait_one(bar_nread, j & 1, abort_flag, p.dev_status))) break;
            if (!(ok = wait_one(bar_stage, (nblk - 1) & 1, abort_flag, p.dev_status))) break;
            tc_fence_after();
            scores(f - 1);
          }
        }
        if (!ok) break;
        if (MODE == kStats) continue;
        if (G::NB == 1 && !(ok = wait_one(bar_nread, j & 1, abort_flag, p.dev_status))) break;
        if (!(ok = wait_one(bar_stage, (nblk - 1) & 1, abort_flag, p.dev_status))) break;
        tc_fence_after();
        scores(G::NB - 1);
        mma_commit(bar_sc);
      }
      if (!ok) {
        // let every issued MMA finish before TMEM is released
        mma_commit(bar_drain);
        mbar_wait(bar_drain, 0);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int etid = tid, quad = warp & 3, half = warp >> 2;
    const int row = quad * 32 + lane;                    // TMEM lane
    const uint32_t lane_tm = tmem + ((uint32_t)(quad * 32) << 16);
    bool ok = true;
    int nblk = 0;
    float kmax_t = -INFINITY;   // statistics pass: this thread's key maximum
    if (nit > 0 && p.stall > 0) ok = epi_wait(bar_never, 0, abort_flag, p.dev_status, p.stall);
    for (int j = 0; ok && j < nit; ++j) {
      const int item = it0 + j, bh = item / p.nc, c = item % p.nc;
      const int b = bh / p.H;
      uint8_t* rec = p.img + (size_t)item * chunk_record_bytes(M_);
      if (!(ok = epi_wait(bar_x, j & 1, abort_flag, p.dev_status))) break;
      // bf16 -> fp16 in place; a magnitude of 0x4780 (65536) or more in either
      // half of a word (the running unsigned maximum of the magnitude bits) is
      // out of fp16 range and reported
      {
        uint32_t mag = 0;
#pragma unroll 4
        for (int i = etid; i < (int)(G::DS * G::kXSlab / 16); i += kEpiThreads) {
          const uint32_t a = s0 + G::oX + i * 16;
          uint4 u = ld_shared_v4(a);
          uint32_t* w32 = &u.x;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            mag = __vmaxu2(mag, w32[e] & 0x7FFF7FFFu);
            const __half2 hv = __floats2half2_rn(__uint_as_float(w32[e] << 16),
                                                 __uint_as_float(w32[e] & 0xFFFF0000u));
            w32[e] = *reinterpret_cast<const uint32_t*>(&hv);
          }
          st_shared_v4(a, u.x, u.y, u.z, u.w);
        }
        if ((mag & 0xFFFFu) >= 0x4780u || (mag >> 16) >= 0x4780u) report(p.dev_status, DARK_ERR_NUMERIC);
      }
      fence_async_smem();
      tc_fence_before();
      warp_arrive(bar_conv);
      // ---- key offsets: sum of squares of the norm columns + 1/2 log2 m
      // (+ the head's key maximum when stabilised); +inf for a masked or
      // missing key
      float kconst = 0.f;
      if (MODE == kStab) {
        // the statistics pass's maxima: 0 for a head without a valid key
        const float km = ord2f(p.kmax[bh]);
        kconst = km > -INFINITY ? km : 0.f;
        if (etid < kC) qc_s[etid] = p.qc[(size_t)item * kC + etid];
        if (p.st_shift != nullptr && c == 0 && etid == 0) p.st_shift[bh] = kconst;
      }
      if (!(ok = epi_wait(bar_norm, j & 1, abort_flag, p.dev_status))) break;
      tc_fence_after();
      {
        float part = 0.f;
#pragma unroll 1
        for (int c0 = half * (R_ / 2); c0 < (half + 1) * (R_ / 2); c0 += 32) {
          float v[32];
          tmem_ld32(lane_tm + G::tN + c0, v);
#pragma unroll
          for (int i = 0; i < 32; ++i) part = fmaf(v[i], v[i], part);
        }
        if (half == 1) nrm_x[row] = part;
        epi_sync();
        if (half == 0) {
          const int tok = c * kC + row;
          bool valid = tok < p.L;
          if (valid && p.mask != nullptr) valid = p.mask[(size_t)b * p.L + tok] != 0;
          nrm_s[row] = valid ? part + nrm_x[row] + 0.5f * __log2f((float)M_) + kconst
                             : __int_as_float(0x7f800000);
        }
        tc_fence_before();
        epi_sync();
        warp_arrive(bar_nread);
      }
      // ---- feature blocks: Phi_f (keys, half 0) and Psi_f (queries, half 1)
      for (int f = 0; ok && f < G::NB; ++f, ++nblk) {
        if (!(ok = epi_wait(bar_ffull, nblk & 1, abort_flag, p.dev_status))) break;
        tc_fence_after();
        uint32_t v[4][32];
#pragma unroll
        for (int q = 0; q < 4; ++q) tmem_ld32_async(lane_tm + G::tF + 128 * half + 32 * q, v[q]);
#pragma unroll
        for (int q = 0; q < 4; ++q) tmem_wait_ld(v[q]);
        tc_fence_before();
        warp_arrive(bar_ffree);
        if (MODE == kStats) {
          if (half == 0) {
            // keys: the largest exponent over this thread's feature and the
            // chunk's valid keys (a masked key's offset is +inf)
#pragma unroll
            for (int q = 0; q < 4; ++q)
#pragma unroll
              for (int e = 0; e < 32; ++e)
                kmax_t = fmaxf(kmax_t, __uint_as_float(v[q][e]) - nrm_s[32 * q + e]);
          } else {
            // queries: the maximum over the block's 128 features (TMEM lanes)
            // of every query (column): a warp reduction per column, then
            // across the four warps of the half in shared memory
            unsigned mine[4];
#pragma unroll
            for (int q = 0; q < 4; ++q)
#pragma unroll
              for (int e = 0; e < 32; ++e) {
                const unsigned r = __reduce_max_sync(0xffffffffu, f2ord(__uint_as_float(v[q][e])));
                if (lane == e) mine[q] = r;
              }
#pragma unroll
            for (int q = 0; q < 4; ++q) atomicMax(&qmax_s[32 * q + lane], mine[q]);
          }
          continue;
        }
        // exp2 and bf16 packing (keys: minus the key offset; their sum over the
        // chunk, of the rounded values, is the chunk's increment of z)
        uint32_t pk[64];
        float dz = 0.f;
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int t = 32 * q + 2 * e;
            float x0 = __uint_as_float(v[q][2 * e]), x1 = __uint_as_float(v[q][2 * e + 1]);
            if (half == 0) {
              x0 -= nrm_s[t];
              x1 -= nrm_s[t + 1];
            } else if (MODE == kStab) {
              x0 -= qc_s[t];
              x1 -= qc_s[t + 1];
            }
            const __nv_bfloat162 pv = __floats2bfloat162_rn(ex2(x0), ex2(x1));
            pk[16 * q + e] = *reinterpret_cast<const uint32_t*>(&pv);
            if (half == 0) {
              const float2 pf = __bfloat1622float2(pv);
              dz += pf.x + pf.y;
            }
          }
        if (half == 0)
          *reinterpret_cast<float*>(rec + chunk_dz_off(M_) + 4 * (128 * f + row)) = dz;
        // the staging is free once the previous block's scores GEMM and bulk
        // stores (or the previous item's A image store) have read it
        if (nblk > 0) {
          if (f > 0 && !(ok = epi_wait(bar_sfree, (nblk - 1) & 1, abort_flag, p.dev_status))) break;
          if (etid == 0) bulk_wait_read_all();
          epi_sync();
        }
        const uint32_t st = s0 + G::oST + 32768 * half;
#pragma unroll
        for (int cc = 0; cc < 16; ++cc) {
          const uint32_t off = (uint32_t)(cc >> 3) * 16384 + (uint32_t)(row >> 3) * 1024 +
                               (uint32_t)(row & 7) * 128 + (uint32_t)(((cc & 7) ^ (row & 7)) * 16);
          st_shared_v4(st + off, pk[4 * cc], pk[4 * cc + 1], pk[4 * cc + 2], pk[4 * cc + 3]);
        }
        fence_async_smem();
        epi_sync();
        if (etid == 0) {
          // the images stream through L2 once: evict them before the projection rows
          const uint64_t once = l2_evict_first();
          bulk_store_hint(rec + (size_t)f * 32768, s0 + G::oST, 32768, once);
          bulk_store_hint(rec + (size_t)M_ * 256 + (size_t)f * 32768, s0 + G::oST + 32768, 32768,
                          once);
          bulk_commit();
        }
        warp_arrive(bar_stage);
      }
      if (!ok) break;
      if (MODE == kStats) {
        // the chunk's maxima: keys into the head's running maximum, queries
        // (their own, one per query) to the workspace
        if (half == 0) {
          const unsigned km = __reduce_max_sync(0xffffffffu, f2ord(kmax_t));
          if (lane == 0) atomicMax(p.kmax + bh, km);
        }
        kmax_t = -INFINITY;
        epi_sync();
        if (etid < kC) {
          p.qc[(size_t)item * kC + etid] = ord2f(qmax_s[etid]);
          qmax_s[etid] = 0u;
        }
        continue;
      }
      // ---- masked causal scores -> A image (query rows, keys as K)
      if (!(ok = epi_wait(bar_sc, j & 1, abort_flag, p.dev_status))) break;
      if (etid == 0) bulk_wait_read_all();
      epi_sync();
      tc_fence_after();
      {
        uint32_t a[2][32];
        tmem_ld32_async(lane_tm + G::tN + 64 * half, a[0]);
        tmem_ld32_async(lane_tm + G::tN + 64 * half + 32, a[1]);
        tmem_wait_ld(a[0]);
        tmem_wait_ld(a[1]);
        float rs = 0.f;      // row sum of the rounded masked scores over this key half
#pragma unroll
        for (int cc = 0; cc < 8; ++cc) {
          uint32_t w4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int jj = 64 * half + 8 * cc + 2 * e;
            const uint32_t* src = a[cc >> 2] + 8 * (cc & 3) + 2 * e;
            const __nv_bfloat162 pv = __floats2bfloat162_rn(jj <= row ? __uint_as_float(src[0]) : 0.f,
                                                            jj + 1 <= row ? __uint_as_float(src[1]) : 0.f);
            w4[e] = *reinterpret_cast<const uint32_t*>(&pv);
            const float2 pf = __bfloat1622float2(pv);
            rs += pf.x + pf.y;
          }
          st_shared_v4(s0 + G::oST + kmajor_off(row, 64 * half + 8 * cc, 16384), w4[0], w4[1],
                       w4[2], w4[3]);
        }
        *reinterpret_cast<float*>(rec + chunk_den_off(M_) + 4 * (128 * half + row)) = rs;
      }
      tc_fence_before();
      fence_async_smem();
      epi_sync();
      if (etid == 0) {
        bulk_store_hint(rec + (size_t)2 * M_ * 256, s0 + G::oST, 32768, l2_evict_first());
        bulk_commit();
      }
    }
    if (etid == 0) bulk_wait_all();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ================================================================ launch 2 ==
// One CTA per (head, value block of 128 columns, feature half). The CTA keeps
// its block of the state, S[f, v] for its NTC tiles of 128 features and 128
// value columns, in TMEM (NTC x 128 columns) and walks the chunks in order.
// Per chunk c, with Psi_t, Phi_t the images of its feature tiles t:
//
//   num  = sum_t Psi_t [S_t hi | S_t lo]      (one N = 256 MMA per K-step)
//        + A_c[:, my keys] V_c                (intra-chunk part, split by keys)
//   S_t += Phi_t^T V_c
//   den  = sum_t Psi_t z_t + rowsum(A_c[:, my keys])   (CUDA cores, fp32)
//
// with z_t the running key-feature sums of the CTA's features (z_<c; the
// per-chunk increments come from the features launch). With m >= 256 the two
// feature halves of a head form a cluster of two CTAs: each finishes half of
// the chunk's query rows and sends the partner its partial result for the
// other half through distributed shared memory, as num/den in fp16 plus den
// in fp32 (out = (num + den' o') / (den + den')).
//
// Warp 9 streams V_c (TMA) and the images (bulk copies) through a 5-slot ring;
// warp 8 issues the MMAs; warps 0-7 are the epilogue. The S operand [S hi | S lo]
// is rebuilt from TMEM for every chunk in halves of 64 features: epilogue group
// h (the four warps whose TMEM lanes hold features 64h..64h+63) fills buffer h
// while the MMAs read the other one. The numerators are signalled as soon as
// the prefix and intra-chunk products are done, so the epilogue reads them
// while the state update runs; each feature tile's Psi slots go back to the
// producer once the epilogue has read them for the denominators.
template <int D_, int M_>
struct ValCfg {
  static constexpr int FS = M_ >= 256 ? 2 : 1;          // feature halves (cluster size)
  static constexpr int VS = D_ / 128;                   // value blocks of 128 columns
  static constexpr int NTC = M_ / (FS * 128);           // feature tiles of this CTA
  // ring items of 16 KB per chunk: Psi_t in halves of 64 features (2 per tile),
  // A (my key block, or both), Phi_t in blocks of 64 tokens (2 per tile)
  static constexpr int NA = FS == 2 ? 1 : 2;
  static constexpr int NI = 4 * NTC + NA;
  static constexpr int NSLOT = 5;
  static constexpr uint32_t oV = 0;                     // V_c block: 2 x 16 KB (MN-major)
  static constexpr uint32_t oS = 32768;                 // S operand halves: 2 x 32 KB
  static constexpr uint32_t oR = oS + 65536;            // ring: NSLOT x 16 KB
  // received o' (fp16 [64 rows][128 columns], the 16-byte chunks of each
  // 128-byte half-row XOR-swizzled by row, so that eight consecutive rows
  // hit different banks) + den' [64]
  static constexpr uint32_t kXB = 16384 + 1024;
  static constexpr uint32_t kXBytes = 16384 + 256;      // bytes the peer sends per chunk
  static constexpr uint32_t oX = oR + NSLOT * 16384;    // [2] receive buffers (chunk parity)
  static constexpr uint32_t oSm = oX + 2 * kXB;         // [2] small items: dz [NTC*128], den_a [256]
  static constexpr uint32_t kSmB = NTC * 512 + 1024;
  static constexpr uint32_t oZ = oSm + 2 * kSmB;        // z [NTC*128], den partials [2][2][128]
  static constexpr uint32_t oBar = oZ + NTC * 512 + 2048;
  static constexpr uint32_t kSmem = oBar + 1024 + 1024;
  static constexpr uint32_t tNum = 256;                 // TMEM: S tiles [0, 128 NTC), num [256, 512)
  static_assert(D_ % 128 == 0 && D_ <= 256 && NTC >= 1 && NTC <= 2, "shape");
  static_assert(kSmem <= 232448, "shared memory");
};

struct ValParams {
  const uint8_t* img;
  __nv_bfloat16* out;
  int64_t ob, oh, ol;
  int B, H, L, nc;
  float *st_kv, *st_z;
  int* dev_status;
  long long stall;         // testing stall before the first wait (0: none)
};

constexpr int kThreadsV = kEpiThreads + 64;   // + MMA warp 8 + producer warp 9

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}
// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t peer_addr(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
// Arrival on a peer CTA's mbarrier, not ordered after this thread's writes
// (the caller's earlier reads are complete: their values have been used).
__device__ __forceinline__ void arrive_peer_relaxed(uint32_t bar_addr) {
  asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_addr)
               : "memory");
}
// Asynchronous stores into a peer CTA's shared memory; the bytes count towards
// the transaction count of the peer's mbarrier at `bar_addr`.
__device__ __forceinline__ void st_async_v4(uint32_t a, uint32_t x, uint32_t y, uint32_t z,
                                            uint32_t w, uint32_t bar_addr) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(
                   a),
               "r"(x), "r"(y), "r"(z), "r"(w), "r"(bar_addr)
               : "memory");
}
__device__ __forceinline__ void st_async_f32(uint32_t a, float x, uint32_t bar_addr) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];" ::"r"(a),
               "r"(__float_as_uint(x)), "r"(bar_addr)
               : "memory");
}
// Wait for a barrier that peers arrive on (acquire at cluster scope), bounded.
__device__ __forceinline__ bool wait_cluster(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                             int* dev_status) {
  const uint32_t a = smem_u32(bar);
  auto probe = [&]() -> bool {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.b32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(a), "r"(parity)
        : "memory");
    return ok != 0;
  };
  if (probe()) return true;
  const long long t0 = clock64();
  while (!probe()) {
    if (*abort_flag) return false;
    if (clock64() - t0 > kWaitCycles) {
      *abort_flag = 1;
      report(dev_status, DARK_ERR_TIMEOUT);
      return false;
    }
  }
  return true;
}
// Named barrier 2 + g over the 128 threads of epilogue group g; true if any
// of them passes `bad`.
__device__ __forceinline__ bool grp_sync_or(int g, bool bad) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "barrier.cta.red.or.pred q, %2, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)bad), "r"(2 + g)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ bool grp_wait(int g, uint64_t* bar, uint32_t parity,
                                         volatile int* abort_flag, int* dev_status) {
  const bool ok = wait_one(bar, parity, abort_flag, dev_status);
  return !grp_sync_or(g, !ok);
}

template <int D_, int M_>
__global__ void __launch_bounds__(kThreadsV, 1)
    values_kernel(const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                  const ValParams p) {
  using G = ValCfg<D_, M_>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t s0 = smem_u32(sm);
  uint64_t* bars = (uint64_t*)(sm + G::oBar);
  uint64_t* bar_v = bars + 0;           // V_c and the chunk's small items loaded
  uint64_t* bar_vfree = bars + 1;       // MMA: every GEMM reading V_c done
  uint64_t* bar_smfree = bars + 2;      // [2] epilogue: small items of buffer i consumed (8)
  uint64_t* bar_simg = bars + 4;        // [2] group h: S operand half written (4)
  uint64_t* bar_sfree = bars + 6;       // [2] MMA: GEMM reading S operand half h done
  uint64_t* bar_ds = bars + 8;          // [2] MMA: state tile t updated by the chunk
  uint64_t* bar_den = bars + 10;        // [2 t][2 h] group h: Psi_{t,h} read for the denominators (4)
  uint64_t* bar_nfull = bars + 14;      // MMA: numerators complete (before the state update)
  uint64_t* bar_nfree = bars + 15;      // epilogue: numerator read (8)
  uint64_t* bar_recv = bars + 38;       // [2] peer: its half-result for my rows arrived (128)
  uint64_t* bar_rfree = bars + 40;      // [2] peer: my half-result in its buffer consumed (128)
  uint64_t* bar_drain = bars + 18;      // MMA: everything issued has completed (abort path)
  uint64_t* bar_never = bars + 19;      // completed by nothing (testing stall)
  uint64_t* bar_full = bars + 20;       // [NSLOT] ring slot loaded
  uint64_t* bar_empty = bars + 28;      // [NSLOT] ring slot read
  uint32_t* tmem_slot = (uint32_t*)(bars + 36);
  volatile int* abort_flag = (volatile int*)(bars + 37);
  float* zs = (float*)(sm + G::oZ);                    // [NTC*128] z_<c of my features
  float* den_part = (float*)(sm + G::oZ + G::NTC * 512);   // [2 parity][2 groups][128]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int fh = G::FS == 2 ? (int)cluster_rank() : 0;
  const int unit = blockIdx.x / G::FS;                 // (head, value block)
  const int bh = unit / G::VS, vb = unit % G::VS;
  const int b = bh / p.H, h = bh % p.H;
  const size_t rec_bytes = chunk_record_bytes(M_);
  const uint8_t* recs = p.img + (size_t)bh * p.nc * rec_bytes;
  const int ft0 = fh * G::NTC;                         // first global feature tile of this CTA

  if (tid == 0) {
    mbar_init(bar_v, 1);
    mbar_init(bar_vfree, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_smfree + i, 8);
      mbar_init(bar_simg + i, 4);
      mbar_init(bar_sfree + i, 1);
      mbar_init(bar_ds + i, 1);
      mbar_init(bar_den + i, 4);
      mbar_init(bar_den + 2 + i, 4);
    }
    mbar_init(bar_nfull, 1);
    mbar_init(bar_nfree, 8);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_recv + i, 1);
      mbar_init(bar_rfree + i, 1);
    }
    for (int i = 0; i < G::NSLOT; ++i) {
      mbar_init(bar_full + i, 1);
      mbar_init(bar_empty + i, 1);
    }
    mbar_init(bar_drain, 1);
    mbar_init(bar_never, 1);
    *abort_flag = 0;
    fence_mbar_init();
    // the peer's half-results for chunks 0 and 1 (its stores complete these)
    if (G::FS == 2)
      for (int i = 0; i < 2 && i < p.nc; ++i) mbar_arrive_expect_tx(bar_recv + i, G::kXBytes);
  }
  for (int i = tid; i < G::NTC * 128 + 512; i += kThreadsV) zs[i] = 0.f;   // z and den partials
  if (warp == 0) tmem_alloc(tmem_slot, kTmemCols);
  tc_fence_before();
  __syncthreads();
  if (G::FS == 2) cluster_sync();     // both CTAs' barriers exist before any peer arrives
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // ring item index (within a chunk) of Psi_t, Phi_t and A: Psi_0, .., Psi_{NTC-1}, A, Phi_0, ..
  // ring items of a chunk: Psi_{t,h} (features 64h.. of tile t), then A_j (key
  // block j), then Phi_{t,kb} (tokens 64kb.. of tile t)
  auto item_psi = [](int t, int hh) { return 2 * t + hh; };
  auto item_a = [](int j) { return 2 * G::NTC + j; };
  auto item_phi = [](int t, int kb) { return 2 * G::NTC + G::NA + 2 * t + kb; };

  if (warp == 9) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tmap(&tm_v);
      int last[G::NSLOT];
      for (int i = 0; i < G::NSLOT; ++i) last[i] = -1;
      int vlast = -1;
      bool ok = true;
      for (int c = 0; ok && c < p.nc; ++c) {
        const uint8_t* rc = recs + (size_t)c * rec_bytes;
        for (int i = 0; ok && i < G::NI; ++i) {
          if (i == 2 * G::NTC) {
            // V_c (once the previous chunk's GEMMs have read V_{c-1}) and the
            // chunk's small items (into the buffer of chunk c - 2, once consumed)
            if (c > 0 && !(ok = wait_one(bar_vfree, (c - 1) & 1, abort_flag, p.dev_status))) break;
            if (c > 1 && !(ok = wait_one(bar_smfree + (c & 1), ((c >> 1) - 1) & 1, abort_flag,
                                         p.dev_status)))
              break;
            const uint32_t dzb = G::NTC * 512, dab = G::FS == 2 ? 512 : 1024;
            mbar_arrive_expect_tx(bar_v, 32768 + dzb + dab);
            tma_load_4d(sm + G::oV, &tm_v, 128 * vb, c * kC, h, b, bar_v);
            tma_load_4d(sm + G::oV + 16384, &tm_v, 128 * vb + 64, c * kC, h, b, bar_v);
            uint8_t* smb = sm + G::oSm + (c & 1) * G::kSmB;
            bulk_load(smb, rc + chunk_dz_off(M_) + (size_t)ft0 * 512, dzb, bar_v);
            bulk_load(smb + dzb, rc + chunk_den_off(M_) + (G::FS == 2 ? 512 * fh : 0), dab, bar_v);
            vlast = c;
          }
          const int g = c * G::NI + i, slot = g % G::NSLOT;
          if (g >= G::NSLOT &&
              !(ok = wait_one(bar_empty + slot, ((g / G::NSLOT) - 1) & 1, abort_flag, p.dev_status)))
            break;
          uint8_t* dst = sm + G::oR + slot * 16384;
          mbar_arrive_expect_tx(bar_full + slot, 16384);
          if (i < 2 * G::NTC) {
            // Psi_{t,h}: rows 64h.. of both token blocks of the tile's image
            const uint8_t* src = rc + (size_t)M_ * 256 + (size_t)(ft0 + i / 2) * 32768 + (i & 1) * 8192;
            bulk_load(dst, src, 8192, bar_full + slot);
            bulk_load(dst + 8192, src + 16384, 8192, bar_full + slot);
          } else if (i < 2 * G::NTC + G::NA) {
            const int j = G::FS == 2 ? fh : i - 2 * G::NTC;                      // A, key block j
            bulk_load(dst, rc + (size_t)2 * M_ * 256 + 16384 * j, 16384, bar_full + slot);
          } else {
            const int q = i - 2 * G::NTC - G::NA;                               // Phi_{t,kb}
            bulk_load(dst, rc + (size_t)(ft0 + q / 2) * 32768 + (q & 1) * 16384, 16384,
                      bar_full + slot);
          }
          last[slot] = g;
        }
      }
      if (!ok) {
        // leave no copy in flight (a completed phase passes at once)
        if (vlast >= 0) mbar_wait(bar_v, vlast & 1);
        for (int i = 0; i < G::NSLOT; ++i)
          if (last[i] >= 0) mbar_wait(bar_full + i, (last[i] / G::NSLOT) & 1);
      }
    }
    __syncwarp();
  } else if (warp == 8) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      auto wait_item = [&](int g) -> bool {
        return wait_one(bar_full + g % G::NSLOT, (g / G::NSLOT) & 1, abort_flag, p.dev_status);
      };
      auto slot_addr = [&](int g) -> uint32_t { return s0 + G::oR + (g % G::NSLOT) * 16384; };
      bool ok = true;
      const uint32_t tnum = tmem + G::tNum, sV = s0 + G::oV;
      for (int c = 0; ok && c < p.nc; ++c) {
        const int g0 = c * G::NI;
        // ---- num = sum_t Psi_t [S_t hi | S_t lo], in halves of 64 features
        for (int t = 0; ok && t < G::NTC; ++t) {
          for (int hh = 0; ok && hh < 2; ++hh) {
            const int gP = g0 + item_psi(t, hh);
            const int k = c * G::NTC + t;          // use of S operand half hh
            if (!(ok = wait_item(gP))) break;
            if (!(ok = wait_one(bar_simg + hh, k & 1, abort_flag, p.dev_status))) break;
            if (t == 0 && hh == 0 && c > 0 &&
                !(ok = wait_one(bar_nfree, (c - 1) & 1, abort_flag, p.dev_status)))
              break;
            tc_fence_after();
            constexpr uint32_t id = idesc(128, 256, true, true, false);
            const uint32_t sP = slot_addr(gP), sS = s0 + G::oS + hh * 32768;
#pragma unroll
            for (int st = 0; st < 4; ++st)
              mma(tnum, sdesc(sP + st * 2048, 8192, 1024), sdesc(sS + st * 2048, 8192, 1024), id,
                  (t | hh | st) != 0);
            mma_commit(bar_sfree + hh);
          }
          // the epilogue reads the tile's Psi items too (denominators): release
          // them once it has, so that the Phi items taking their slots load
          // while the next tile's prefix product runs
          for (int hh = 0; ok && hh < 2; ++hh) {
            if (!(ok = wait_one(bar_den + 2 * t + hh, c & 1, abort_flag, p.dev_status))) break;
            mma_commit(bar_empty + (g0 + item_psi(t, hh)) % G::NSLOT);
          }
        }
        if (!ok) break;
        // ---- num[:, hi] += A_c[:, my keys] V_c[my keys]
        for (int j = 0; ok && j < G::NA; ++j) {
          const int gA = g0 + item_a(j);
          if (!(ok = wait_item(gA))) break;
          if (j == 0 && !(ok = wait_one(bar_v, c & 1, abort_flag, p.dev_status))) break;
          tc_fence_after();
          constexpr uint32_t id = idesc(128, 128, false, true, false);
          const uint32_t sA = slot_addr(gA);
          const int kb = G::FS == 2 ? fh : j;      // key block of V
#pragma unroll
          for (int st = 0; st < 4; ++st)
            mma(tnum, sdesc(sA + st * 32, 16, 1024), sdesc(sV + (4 * kb + st) * 2048, 16384, 1024), id,
                1u);
          mma_commit(bar_empty + gA % G::NSLOT);
        }
        // the numerators are complete: the epilogue reads them while the state
        // update runs (its own barrier orders the next conversions)
        if (ok) mma_commit(bar_nfull);
        // ---- S_t += Phi_t^T V_c, in blocks of 64 tokens
        for (int t = 0; ok && t < G::NTC; ++t) {
          for (int kb = 0; ok && kb < 2; ++kb) {
            const int gF = g0 + item_phi(t, kb);
            if (!(ok = wait_item(gF))) break;
            tc_fence_after();
            constexpr uint32_t id = idesc(128, 128, false, true, false);
            const uint32_t sF = slot_addr(gF);
#pragma unroll
            for (int st = 0; st < 4; ++st)
              mma(tmem + 128 * t, sdesc(sF + st * 32, 16, 1024),
                  sdesc(sV + (4 * kb + st) * 2048, 16384, 1024), id, (c > 0) || (kb > 0) || (st > 0));
            mma_commit(bar_empty + gF % G::NSLOT);
          }
          if (!ok) break;
          mma_commit(bar_ds + t);
        }
        if (!ok) break;
        mma_commit(bar_vfree);
      }
      // let every issued MMA finish before TMEM is released (the last state
      // update is waited for by no other role unless the state is output)
      mma_commit(bar_drain);
      mbar_wait(bar_drain, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int quad = warp & 3, colh = warp >> 2;
    const int row = quad * 32 + lane;               // TMEM lane
    const int grp = quad >> 1;                      // lanes 64 grp .. 64 grp + 63
    const int gi = (colh << 6) | ((quad & 1) << 5) | lane;   // 0..127 within the group
    const uint32_t lane_tm = tmem + ((uint32_t)(quad * 32) << 16);
    const int hrow = row - 64 * grp;                // feature row within the half
    bool ok = true;
    if (p.stall > 0) ok = epi_wait(bar_never, 0, abort_flag, p.dev_status, p.stall);
    // denominators: this thread sums features 8a + fi (a = 0..7) of a half for
    // the 8 tokens of chunk tcd; the 8 lanes fi of a quarter-warp then reduce
    const int fi = lane & 7;
    const int tcd = (((quad & 1) | (colh << 1)) << 2) | (lane >> 3);   // 0..15
    float dacc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) dacc[e] = 0.f;
    uint32_t po[32];                               // o of my rows, previous chunk (fp16 pairs)
    float pden = 0.f;
#pragma unroll
    for (int e = 0; e < 32; ++e) po[e] = 0u;
    const uint32_t peer = (uint32_t)(1 - fh);
    // out[row] of chunk cc from 64 fp32 numerators and 1/den (bf16); false if not finite
    auto store_row = [&](int cc, const float* nm, float invd, float dd) -> bool {
      uint32_t w[32];
      bool bad = !isfinite(dd);
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const float o0 = nm[2 * e] * invd, o1 = nm[2 * e + 1] * invd;
        bad |= !isfinite(o0) || !isfinite(o1);
        w[e] = pack_bf16(o0, o1);
      }
      uint4* dst = reinterpret_cast<uint4*>(p.out + (int64_t)b * p.ob + (int64_t)h * p.oh +
                                            (int64_t)(cc * kC + row) * p.ol + 128 * vb + 64 * colh);
#pragma unroll
      for (int q4 = 0; q4 < 8; ++q4)
        dst[q4] = make_uint4(w[4 * q4], w[4 * q4 + 1], w[4 * q4 + 2], w[4 * q4 + 3]);
      return !bad;
    };
    // rows of chunk cc this CTA finishes: (den o + den' o') / (den + den') with
    // o, den kept from that chunk and o', den' from the peer's buffer cc & 1.
    // The buffer of chunk cc - 1 goes back to the peer here (its chunk cc + 1),
    // once the tensor stores of cc - 1 have read it: the wait is a chunk late.
    auto finish_prev = [&](int cc) -> bool {
      if (gi == 0 && cc > 0) {
        bulk_wait_group_read();
        if (cc + 1 < p.nc) mbar_arrive_expect_tx(bar_recv + ((cc - 1) & 1), G::kXBytes);
        arrive_peer_relaxed(peer_addr(smem_u32(bar_rfree + ((cc - 1) & 1)), peer));
      }
      const bool arrived = wait_cluster(bar_recv + (cc & 1), (cc >> 1) & 1, abort_flag, p.dev_status);
      if (grp_sync_or(grp, !arrived)) return false;
      const uint32_t xb = s0 + G::oX + (cc & 1) * G::kXB;
      const uint32_t xr = xb + (uint32_t)(row & 63) * 256 + colh * 128;
      const float dp = *reinterpret_cast<const float*>(sm + G::oX + (cc & 1) * G::kXB + 16384 +
                                                       (row & 63) * 4);
      float nm[64];
#pragma unroll
      for (int q4 = 0; q4 < 8; ++q4) {
        const uint4 u = ld_shared_v4(xr + (uint32_t)((q4 ^ (row & 7)) * 16));
        const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 of = __half22float2(*reinterpret_cast<const __half2*>(&w4[e]));
          const float2 mf = __half22float2(*reinterpret_cast<const __half2*>(&po[4 * q4 + e]));
          nm[8 * q4 + 2 * e] = fmaf(pden, mf.x, dp * of.x);
          nm[8 * q4 + 2 * e + 1] = fmaf(pden, mf.y, dp * of.y);
        }
      }
      // every reader of the group is done with o': the rows go out through the
      // same buffer (two 64-column halves, 64 rows x 128 B each, 16-byte chunks
      // XOR-swizzled by row as the output map's 128-byte swizzle expects) by two
      // tensor stores
      grp_sync_or(grp, false);
      const float dt = pden + dp;
      const float invd = dt > 0.f ? 1.f / dt : 0.f;
      float sum = dt;                   // non-finite if any value is
      uint32_t w[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const float o0 = nm[2 * e] * invd, o1 = nm[2 * e + 1] * invd;
        sum += o0 + o1;
        w[e] = pack_bf16(o0, o1);
      }
      if (cc * kC + row < p.L && !isfinite(sum)) report(p.dev_status, DARK_ERR_NUMERIC);
      const int r = row & 63;
      const uint32_t stg = xb + colh * 8192 + (uint32_t)r * 128;
#pragma unroll
      for (int q4 = 0; q4 < 8; ++q4)
        st_shared_v4(stg + (uint32_t)((q4 ^ (r & 7)) * 16), w[4 * q4], w[4 * q4 + 1], w[4 * q4 + 2],
                     w[4 * q4 + 3]);
      fence_async_smem();
      grp_sync_or(grp, false);
      if (gi == 0) {
        tma_store_4d(&tm_o, xb, 128 * vb, cc * kC + 64 * fh, h, b);
        tma_store_4d(&tm_o, xb + 8192, 128 * vb + 64, cc * kC + 64 * fh, h, b);
        bulk_commit_group();
      }
      return true;
    };
    // S operand half of feature tile t for chunk c (group grp's features)
    auto conv = [&](int c, int t) -> bool {
      const int k = c * G::NTC + t;
      if (k > 0 && !(ok = grp_wait(grp, bar_sfree + grp, (k - 1) & 1, abort_flag, p.dev_status)))
        return false;
      if (c > 0 && !(ok = grp_wait(grp, bar_ds + t, (c - 1) & 1, abort_flag, p.dev_status))) return false;
      tc_fence_after();
      // this thread: feature hrow of half grp, value columns 64 colh .. 64 colh + 63
      uint32_t a[2][32];
      if (c > 0) {
        tmem_ld32_async(lane_tm + 128 * t + 64 * colh, a[0]);
        tmem_ld32_async(lane_tm + 128 * t + 64 * colh + 32, a[1]);
        tmem_wait_ld(a[0]);
        tmem_wait_ld(a[1]);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) a[0][i] = a[1][i] = 0u;
      }
      const uint32_t sS = s0 + G::oS + grp * 32768;
      const uint32_t rowoff = (uint32_t)(hrow >> 3) * 1024 + (uint32_t)(hrow & 7) * 128;
#pragma unroll
      for (int cg = 0; cg < 8; ++cg) {
        uint32_t hi4[4], lo4[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int i = 8 * cg + 2 * e;
          const float x0 = __uint_as_float(a[i >> 5][i & 31]);
          const float x1 = __uint_as_float(a[(i + 1) >> 5][(i + 1) & 31]);
          const __nv_bfloat162 hv = __floats2bfloat162_rn(x0, x1);
          const float2 hf = __bfloat1622float2(hv);
          hi4[e] = *reinterpret_cast<const uint32_t*>(&hv);
          lo4[e] = pack_bf16(x0 - hf.x, x1 - hf.y);
        }
        const uint32_t off = rowoff + (uint32_t)((cg ^ (hrow & 7)) * 16);
        st_shared_v4(sS + colh * 8192 + off, hi4[0], hi4[1], hi4[2], hi4[3]);          // hi block
        st_shared_v4(sS + (2 + colh) * 8192 + off, lo4[0], lo4[1], lo4[2], lo4[3]);   // lo block
      }
      tc_fence_before();
      fence_async_smem();
      warp_arrive(bar_simg + grp);
      return true;
    };
    // denominator partials from Psi_{t,grp} of chunk c, then z_<c+1 for the half
    auto den_tile = [&](int c, int t) -> bool {
      const int g0 = c * G::NI;
      // ---- den partial of token gi over features 64 grp .. + 63 of tile t
      const int gP = g0 + item_psi(t, grp);
      if (!(ok = grp_wait(grp, bar_full + gP % G::NSLOT, (gP / G::NSLOT) & 1, abort_flag,
                          p.dev_status)))
        return false;
      {
        // Psi_{t,h}: token block tcd >> 3, rows = features of the half
        const uint32_t psi = s0 + G::oR + (gP % G::NSLOT) * 16384 + (tcd >> 3) * 8192 +
                             (uint32_t)fi * 128 + (uint32_t)(((tcd & 7) ^ fi) << 4);
        const float* zt = zs + 128 * t + 64 * grp + fi;
        float acc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
        for (int a8 = 0; a8 < 8; ++a8) {
          const uint4 u = ld_shared_v4(psi + a8 * 1024);
          const float zf = zt[8 * a8];
          const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            acc[2 * e] = fmaf(__uint_as_float(w4[e] << 16), zf, acc[2 * e]);
            acc[2 * e + 1] = fmaf(__uint_as_float(w4[e] & 0xFFFF0000u), zf, acc[2 * e + 1]);
          }
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          float x = acc[e];
          x += __shfl_xor_sync(0xffffffffu, x, 1);
          x += __shfl_xor_sync(0xffffffffu, x, 2);
          x += __shfl_xor_sync(0xffffffffu, x, 4);
          dacc[e] += x;
        }
      }
      // z_<c+1 = z_<c + dz_c for these 64 features, once every thread has read
      // them and the chunk's small items have arrived
      if (!(ok = grp_wait(grp, bar_v, c & 1, abort_flag, p.dev_status))) return false;
      if (gi < 64) {
        const float* dz = (const float*)(sm + G::oSm + (c & 1) * G::kSmB);
        zs[128 * t + 64 * grp + gi] += dz[128 * t + 64 * grp + gi];
      }
      warp_arrive(bar_den + 2 * t + grp);
      return true;
    };
    // this chunk's denominator partials, for the rows of the output phase (read
    // by other threads after the agreement at the top of the chunk)
    auto put_den = [&](int c) {
      if (fi == 0) {
#pragma unroll
        for (int e = 0; e < 8; ++e) den_part[((c & 1) * 2 + grp) * 128 + 8 * tcd + e] = dacc[e];
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) dacc[e] = 0.f;
    };
    for (int t = 0; ok && t < G::NTC; ++t) ok = conv(0, t) && den_tile(0, t);
    put_den(0);
    // Every epilogue thread passes the agreement at the top of each chunk (the
    // only point where both groups wait together); a failure inside a chunk
    // skips to it, so that the groups always leave the loop together.
    for (int c = 0; c < p.nc; ++c) {
      if (epi_sync_or(!ok)) {
        ok = false;
        break;
      }
      // ---------------- output of chunk c, part 1: numerators and denominators
      if (!wait_one(bar_nfull, c & 1, abort_flag, p.dev_status)) {
        ok = false;
        continue;
      }
      tc_fence_after();
      float num[64];
      {
        uint32_t hi[2][32], lo[2][32];
        tmem_ld32_async(lane_tm + G::tNum + 64 * colh, hi[0]);
        tmem_ld32_async(lane_tm + G::tNum + 64 * colh + 32, hi[1]);
        tmem_ld32_async(lane_tm + G::tNum + 128 + 64 * colh, lo[0]);
        tmem_ld32_async(lane_tm + G::tNum + 128 + 64 * colh + 32, lo[1]);
        tmem_wait_ld(hi[0]);
        tmem_wait_ld(hi[1]);
        tmem_wait_ld(lo[0]);
        tmem_wait_ld(lo[1]);
#pragma unroll
        for (int i = 0; i < 64; ++i)
          num[i] = __uint_as_float(hi[i >> 5][i & 31]) + __uint_as_float(lo[i >> 5][i & 31]);
      }
      tc_fence_before();
      warp_arrive(bar_nfree);
      // den = the two groups' partials for query row `row` + rowsum(A_c[row, my keys])
      const float* da = (const float*)(sm + G::oSm + (c & 1) * G::kSmB + G::NTC * 512);
      const float den = den_part[((c & 1) * 2 + 0) * 128 + row] +
                        den_part[((c & 1) * 2 + 1) * 128 + row] + da[row] +
                        (G::FS == 1 ? da[128 + row] : 0.f);
      const float inv = den > 0.f ? 1.f / den : 0.f;
      uint32_t o[32];
      if (G::FS == 1) {
        if (c * kC + row < p.L && !store_row(c, num, inv, den)) report(p.dev_status, DARK_ERR_NUMERIC);
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const __half2 hv = __floats2half2_rn(num[2 * e] * inv, num[2 * e + 1] * inv);
          o[e] = *reinterpret_cast<const uint32_t*>(&hv);
        }
      }
      // the next chunk's S operands and denominators, so that its MMAs start now
      if (c + 1 < p.nc) {
        for (int t = 0; ok && t < G::NTC; ++t) ok = conv(c + 1, t) && den_tile(c + 1, t);
        if (!ok) continue;
        put_den(c + 1);
      }
      // ---------------- output of chunk c, part 2: the exchange between the halves
      if (G::FS == 2) {
        if ((row >> 6) == fh) {
          // a row this CTA finishes: chunk c - 1's, whose other half has arrived
          // by now; this chunk's part waits in registers until the next chunk
          if (c > 0 && !(ok = finish_prev(c - 1))) continue;
#pragma unroll
          for (int e = 0; e < 32; ++e) po[e] = o[e];
          pden = den;
        } else {
          // a row the peer finishes: num/den (fp16) and den into its buffer c & 1,
          // once it has consumed what the buffer held (chunk c - 2)
          if (c > 1) {
            const bool freed = wait_cluster(bar_rfree + (c & 1), ((c >> 1) - 1) & 1, abort_flag,
                                            p.dev_status);
            if (grp_sync_or(grp, !freed)) {
              ok = false;
              continue;
            }
          }
          const uint32_t xb = s0 + G::oX + (c & 1) * G::kXB;
          const uint32_t xr = peer_addr(xb + (uint32_t)(row & 63) * 256 + colh * 128, peer);
          const uint32_t rb = peer_addr(smem_u32(bar_recv + (c & 1)), peer);
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4)
            st_async_v4(xr + (uint32_t)((q4 ^ (row & 7)) * 16), o[4 * q4], o[4 * q4 + 1], o[4 * q4 + 2],
                        o[4 * q4 + 3], rb);
          if (colh == 0) st_async_f32(peer_addr(xb + 16384 + (uint32_t)(row & 63) * 4, peer), den, rb);
        }
      }
      warp_arrive(bar_smfree + (c & 1));
    }
    if (ok && G::FS == 2 && (row >> 6) == fh && p.nc > 0) ok = finish_prev(p.nc - 1);
    if (G::FS == 2 && (row >> 6) == fh && gi == 0) bulk_wait_group();   // the output stores are done
    ok = !epi_sync_or(!ok);
    // final state: S_t (my features x my 128 value columns) and z (first value block)
    if (ok && p.st_kv != nullptr) {
      for (int t = 0; ok && t < G::NTC; ++t)
        ok = epi_wait(bar_ds + t, (p.nc - 1) & 1, abort_flag, p.dev_status);
      if (ok) {
        tc_fence_after();
        for (int t = 0; t < G::NTC; ++t) {
          uint32_t a[2][32];
          tmem_ld32_async(lane_tm + 128 * t + 64 * colh, a[0]);
          tmem_ld32_async(lane_tm + 128 * t + 64 * colh + 32, a[1]);
          tmem_wait_ld(a[0]);
          tmem_wait_ld(a[1]);
          const int feat = 128 * (ft0 + t) + row;
          float* kv = p.st_kv + ((size_t)bh * M_ + feat) * D_ + 128 * vb + 64 * colh;
#pragma unroll
          for (int i = 0; i < 64; ++i) kv[i] = __uint_as_float(a[i >> 5][i & 31]);
          if (vb == 0 && colh == 0) p.st_z[(size_t)bh * M_ + feat] = zs[128 * t + row];
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (G::FS == 2) cluster_sync();     // no peer may still write into this CTA
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------ host --
bool make_wide_maps(FwdArgs& a) {
  auto al16 = [](const void* p) { return ((uintptr_t)p & 15) == 0; };
  if (!al16(a.q) || !al16(a.k) || !al16(a.v) || !al16(a.out) || !al16(a.w)) return false;
  for (int i = 0; i < 3; ++i)
    if (a.qs[i] % 8 != 0 || a.ks[i] != a.qs[i] || a.os[i] % 8 != 0) return false;
  const uint64_t wd[2] = {(uint64_t)a.d, (uint64_t)a.heads_w * (a.m + a.r)};
  const uint64_t wsd[1] = {(uint64_t)a.d * 2};
  const uint32_t wb[2] = {64, 64};
  const uint64_t xd[4] = {(uint64_t)a.d, (uint64_t)a.L, (uint64_t)a.H, (uint64_t)a.B};
  const uint64_t xs[3] = {(uint64_t)a.qs[2] * 2, (uint64_t)a.qs[1] * 2, (uint64_t)a.qs[0] * 2};
  const uint32_t xb[4] = {64, 128, 1, 1};
  a.maps_ready = encode_tmap(&a.tm_w, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, a.w, wd, wsd, wb) &&
                 encode_tmap(&a.tm_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, a.q, xd, xs, xb) &&
                 encode_tmap(&a.tm_k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, a.k, xd, xs, xb) &&
                 encode_tmap(&a.tm_v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, a.v, xd, xs, xb);
  // out: 64-column x 64-row boxes (the half-chunk rows one CTA of a cluster finishes)
  const uint64_t od[4] = {(uint64_t)a.d, (uint64_t)a.L, (uint64_t)a.H, (uint64_t)a.B};
  const uint64_t ost[3] = {(uint64_t)a.os[2] * 2, (uint64_t)a.os[1] * 2, (uint64_t)a.os[0] * 2};
  const uint32_t ob[4] = {64, 64, 1, 1};
  a.maps_ready = a.maps_ready &&
                 encode_tmap(&a.tm_o, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, a.out, od, ost, ob);
  return a.maps_ready;
}

bool shape_ok(int d, int m, int r) {
  return (d == 256 && m == 512 && r == 256) || (d == 128 && m == 256 && r == 128) ||
         (d == 128 && m == 128 && r == 64);
}

// Workspace after the chunk records: the stabiliser's per-(b,h) key maxima
// (order-preserving integers) and per-query maxima.
size_t stab_kmax_off(int B, int H, int nc, int m) {
  return align_up(kWsHeader + (size_t)B * H * nc * chunk_record_bytes(m), 256);
}
size_t stab_qc_off(int B, int H, int nc, int m) {
  return align_up(stab_kmax_off(B, H, nc, m) + (size_t)B * H * 4, 256);
}

template <int D_, int M_, int R_, int MODE>
cudaError_t launch_features(const FwdArgs& a, const FeatParams& fp) {
  using F = FeatCfg<D_, M_, R_>;
  static int smem_f[64];
  cudaError_t e =
      set_smem_limit_once((const void*)features_kernel<D_, M_, R_, MODE>, (int)F::kSmem, smem_f);
  if (e != cudaSuccess) return e;
  const int grid_f = fp.nitems < num_sms() ? fp.nitems : num_sms();
  features_kernel<D_, M_, R_, MODE><<<grid_f, kThreadsF, F::kSmem, a.stream>>>(a.tm_w, a.tm_q,
                                                                               a.tm_k, fp);
  return cudaGetLastError();
}

template <int D_, int M_, int R_>
cudaError_t launch(const FwdArgs& a) {
  using V = ValCfg<D_, M_>;
  const int nc = (a.L + kC - 1) / kC;
  uint8_t* img = (uint8_t*)a.ws + kWsHeader;
  const bool stab = (a.flags & DARK_STABILISE) != 0;
  FeatParams fp;
  memset(&fp, 0, sizeof(fp));
  fp.mask = a.mask;
  fp.img = img;
  fp.B = a.B;
  fp.H = a.H;
  fp.L = a.L;
  fp.nc = nc;
  fp.heads_w = a.heads_w;
  fp.dev_status = a.dev_status;
  fp.stall = test_stall_cycles();
  static int smem_v[64];
  cudaError_t e = set_smem_limit_once((const void*)values_kernel<D_, M_>, (int)V::kSmem, smem_v);
  if (e != cudaSuccess) return e;
  fp.nitems = a.B * a.H * nc;
  if (stab) {
    // statistics pass, then the features with the maxima subtracted
    fp.kmax = (unsigned*)((uint8_t*)a.ws + stab_kmax_off(a.B, a.H, nc, M_));
    fp.qc = (float*)((uint8_t*)a.ws + stab_qc_off(a.B, a.H, nc, M_));
    fp.st_shift = a.st_shift;
    e = cudaMemsetAsync(fp.kmax, 0, (size_t)a.B * a.H * 4, a.stream);
    if (e != cudaSuccess) return e;
    e = launch_features<D_, M_, R_, kStats>(a, fp);
    if (e != cudaSuccess) return e;
    e = launch_features<D_, M_, R_, kStab>(a, fp);
  } else {
    e = launch_features<D_, M_, R_, kPlain>(a, fp);
  }
  if (e != cudaSuccess) return e;
  ValParams vp;
  memset(&vp, 0, sizeof(vp));
  vp.img = img;
  vp.out = (__nv_bfloat16*)a.out;
  vp.ob = a.os[0];
  vp.oh = a.os[1];
  vp.ol = a.os[2];
  vp.B = a.B;
  vp.H = a.H;
  vp.L = a.L;
  vp.nc = nc;
  vp.st_kv = a.st_kv;
  vp.st_z = a.st_z;
  vp.dev_status = a.dev_status;
  vp.stall = test_stall_cycles();
  // one CTA per (head, 128 value columns, feature half); the feature halves
  // of a (head, value block) form a cluster
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(a.B * a.H * V::VS * V::FS);
  cfg.blockDim = dim3(kThreadsV);
  cfg.dynamicSmemBytes = V::kSmem;
  cfg.stream = a.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = V::FS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, values_kernel<D_, M_>, a.tm_v, a.tm_o, vp);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

bool tc_wide_supported(FwdArgs& a) {
  if (a.dtype != DARK_BF16 || !(a.flags & DARK_CAUSAL)) return false;
  if (!shape_ok(a.d, a.m, a.r)) return false;
  return make_wide_maps(a);
}

size_t tc_wide_workspace_bytes(int B, int H, int L, int m, int d, int r) {
  if (!shape_ok(d, m, r)) return 0;
  const int nc = (L + kC - 1) / kC;
  return align_up(stab_qc_off(B, H, nc, m) + (size_t)B * H * nc * kC * 4, 256);
}

cudaError_t tc_wide_forward(const FwdArgs& a) {
  if (!a.maps_ready) return cudaErrorInvalidValue;
  if (a.d == 256 && a.m == 512 && a.r == 256) return launch<256, 512, 256>(a);
  if (a.d == 128 && a.m == 256 && a.r == 128) return launch<128, 256, 128>(a);
  if (a.d == 128 && a.m == 128 && a.r == 64) return launch<128, 128, 64>(a);
  return cudaErrorInvalidValue;
}

}  // namespace dark
