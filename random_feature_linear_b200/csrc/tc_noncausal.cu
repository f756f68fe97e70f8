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
#include "tc_keys.cuh"
#include "tc_roles.cuh"

namespace dark {
namespace {

using namespace tc;

constexpr int kD = 64;
constexpr int kT = 128;                     // tokens per tile
constexpr int kThreads = kFwdThreads + 128;   // query kernel: + MMA, producer, 2 converter warps
constexpr int kSms = 148;
constexpr int kTileBytes = kT * kD * 2;
constexpr uint32_t kTmemCols = 512;

// The query kernel's B operand [S hi | S lo | (z hi, z lo)] per head: three
// MN-major blocks of m feature rows x 128 B, so that one MMA per K-step (N =
// 64 + 64 + 16) yields both halves of the numerator and of the denominator
// (every MMA with N <= 144 costs about the same, so fewer and wider is faster).
// The third block holds z hi, z lo in columns 0, 1 and zeros up to column 15.
__host__ __device__ constexpr uint32_t img_s_bytes(int m) { return (uint32_t)m * 128; }
__host__ __device__ constexpr uint32_t img_bytes(int m) { return 3 * img_s_bytes(m); }

// Sums the split partials of each head in split order and writes the query
// kernel's operand image (hi + lo bf16) and, if requested, the fp32 state.
// Stabiliser (shifts non-null): partial s is scaled by 2^-shifts[s]; the sum is
// taken relative to the largest of them, c_K (0 when no key is valid), which
// is the state's shift. One thread per (feature f, group of 8 value columns),
// consecutive threads over f (coalesced partial reads); group 8 is z.
__global__ void reduce_kernel(const float* __restrict__ partials, int nsplit, int m,
                              const float* __restrict__ shifts, uint8_t* __restrict__ images,
                              float* __restrict__ st_kv, float* __restrict__ st_z,
                              float* __restrict__ st_shift) {
  // the query launch that follows may start now: it waits for this grid only
  // where it reads the operand image
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int bh = blockIdx.y;
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= 9 * m) return;
  const int cg = idx / m, f = idx % m;
  const int ncol = cg < 8 ? 8 : 1;
  const float* src = partials + (size_t)bh * nsplit * 65 * m + (size_t)(cg * 8) * m + f;
  float acc[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) acc[c] = 0.f;
  const float* sh = shifts == nullptr ? nullptr : shifts + (size_t)bh * nsplit;
  float cmax = -INFINITY;
  if (sh != nullptr)
    for (int s = 0; s < nsplit; ++s) cmax = fmaxf(cmax, sh[s]);
  for (int s = 0; s < nsplit; ++s) {
    float sc = 1.f;
    if (sh != nullptr) {
      if (!(sh[s] > -INFINITY)) continue;
      sc = exp2f(sh[s] - cmax);
    }
    const float* ps = src + (size_t)s * 65 * m;
#pragma unroll
    for (int c = 0; c < 8; ++c)
      if (c < ncol) acc[c] += (sh != nullptr ? sc * ps[(size_t)c * m] : ps[(size_t)c * m]);
  }
  if (sh != nullptr && idx == 0 && st_shift != nullptr)
    st_shift[bh] = cmax > -INFINITY ? cmax : 0.f;
  uint32_t hi2[4], lo2[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const __nv_bfloat16 h0 = __float2bfloat16_rn(acc[2 * e]), h1 = __float2bfloat16_rn(acc[2 * e + 1]);
    const __nv_bfloat16 l0 = __float2bfloat16_rn(acc[2 * e] - __bfloat162float(h0));
    const __nv_bfloat16 l1 = __float2bfloat16_rn(acc[2 * e + 1] - __bfloat162float(h1));
    hi2[e] = (uint32_t)__bfloat16_as_ushort(h0) | ((uint32_t)__bfloat16_as_ushort(h1) << 16);
    lo2[e] = (uint32_t)__bfloat16_as_ushort(l0) | ((uint32_t)__bfloat16_as_ushort(l1) << 16);
  }
  uint8_t* img = images + (size_t)bh * img_bytes(m);
  const uint32_t row = (uint32_t)(f / 8) * 1024 + (uint32_t)(f % 8) * 128;
  if (cg < 8) {
    // columns 8 cg .. 8 cg + 7: one 16-byte chunk of row f in each of the S
    // blocks (hi, lo), chunk index XOR-swizzled by f % 8
    const uint32_t off = row + (uint32_t)((cg ^ (f % 8)) * 16);
    *reinterpret_cast<uint4*>(img + off) = make_uint4(hi2[0], hi2[1], hi2[2], hi2[3]);
    *reinterpret_cast<uint4*>(img + img_s_bytes(m) + off) = make_uint4(lo2[0], lo2[1], lo2[2], lo2[3]);
    if (st_kv != nullptr) {
      float* d = st_kv + ((size_t)bh * m + f) * 64 + cg * 8;
      if ((reinterpret_cast<uintptr_t>(d) & 15) == 0) {
        reinterpret_cast<float4*>(d)[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
        reinterpret_cast<float4*>(d)[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
      } else {
#pragma unroll
        for (int c = 0; c < 8; ++c) d[c] = acc[c];
      }
    }
  } else {
    // columns 0-7 and 8-15 of the third block: (z hi, z lo, 0, ...), zeros
    uint8_t* zz = img + 2 * img_s_bytes(m) + row;
    const uint32_t w0 = (hi2[0] & 0xFFFFu) | ((lo2[0] & 0xFFFFu) << 16);
    *reinterpret_cast<uint4*>(zz + (uint32_t)((0 ^ (f % 8)) * 16)) = make_uint4(w0, 0u, 0u, 0u);
    *reinterpret_cast<uint4*>(zz + (uint32_t)((1 ^ (f % 8)) * 16)) = make_uint4(0u, 0u, 0u, 0u);
    if (st_z != nullptr) st_z[(size_t)bh * m + f] = acc[0];
  }
}

struct QueryParams {
  __nv_bfloat16* out;
  int64_t ob, oh, ol;
  int B, H, L, ntiles, heads_w, total_tiles;   // L, ntiles: queries
  const uint8_t* qmask;         // [B][L] or null: a masked query row outputs 0
  const uint8_t* images;
  int stab_q;                   // stabiliser: query exponents relative to their row maximum
  int* dev_status;
  long long stall;              // testing stall before the first wait (0: none)
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
  static constexpr uint32_t oRed = oBar + 256;             // [2][128] fp32 row maxima
  static constexpr uint32_t kSmem = oRed + 1024 + 1024;
  static constexpr uint32_t tP = 0, tO = 256;
  static_assert(kSmem <= 232448, "shared memory");
};

// bf16 -> fp16 in place for one Q tile by the 64 converter threads. A bf16
// value is out of fp16 range (|x| > 65504) exactly when its magnitude bits are
// 0x4780 (65536) or more.
__device__ __forceinline__ void q_to_fp16(uint32_t saddr, int ctid, int* dev_status) {
  uint32_t mag = 0;
#pragma unroll 4
  for (int i = ctid; i < kTileBytes / 16; i += 64) {
    const uint32_t a = saddr + i * 16;
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
  if ((mag & 0xFFFFu) >= 0x4780u || (mag >> 16) >= 0x4780u) report(dev_status, DARK_ERR_NUMERIC);
}

// Query kernel: each CTA walks a contiguous range of (head, query tile) items
// with four roles. Warp 9 loads the head operands (W' feature rows and the
// [S | z] image, once per head) and the Q tiles (two buffers); warps 10-11
// convert each Q tile to fp16 as it lands; warp 8 issues the MMAs; warps 0-7
// run the epilogue. The feature GEMM Q W^T comes in two parts (features [0, M/2) and
// [M/2, M)), each released by the epilogue as soon as it has read it, so the
// next tile's features are computed during this tile's exponentials; the
// output GEMM of a tile is read back (and the tile's rows stored) while the
// next tile is exponentiated.
template <int M_, int R_>
__global__ void __launch_bounds__(kThreads, 1)
    queries_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_q,
                   const __grid_constant__ CUtensorMap tm_o, const QueryParams p) {
  using G = QueryCfg<M_, R_>;
  constexpr int NH = M_ / 128;                // 32-column chunks per pass
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t s0 = smem_u32(sm);
  uint64_t* bars = (uint64_t*)(sm + G::oBar);
  uint64_t* q_full = bars + 0;       // [2] producer: Q tile loaded
  uint64_t* q_conv = bars + 2;       // [2] converters: Q tile converted to fp16 (2)
  uint64_t* q_empty = bars + 4;      // [2] MMA: the feature GEMM has read the Q tile
  uint64_t* h_full = bars + 6;       // producer: a head's W' rows and image loaded
  uint64_t* h_free = bars + 7;       // MMA: the last GEMMs of a head are done
  uint64_t* bar_ffullA = bars + 8;   // MMA: features [0, M/2) in TMEM
  uint64_t* bar_ffreeA = bars + 9;   // epilogue: read (8)
  uint64_t* bar_ffullB = bars + 10;  // MMA: features [M/2, M) in TMEM
  uint64_t* bar_ffreeB = bars + 11;  // epilogue: read (8)
  uint64_t* bar_pfull = bars + 12;   // epilogue: Psi staged, the previous output read (8)
  uint64_t* bar_ofull = bars + 13;   // MMA: output GEMM done (Psi free)
  uint64_t* bar_drain = bars + 14;   // abort path: the issued MMAs completed
  uint64_t* bar_never = bars + 15;   // completed by nothing (testing stall)
  uint32_t* tmem_slot = (uint32_t*)(bars + 16);
  volatile int* abort_flag = (volatile int*)(bars + 16) + 1;
  float* red = (float*)(sm + G::oRed);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ub = (int)((long long)blockIdx.x * p.total_tiles / gridDim.x);
  const int ue = (int)((long long)(blockIdx.x + 1) * p.total_tiles / gridDim.x);
  const int n = ue > ub ? ue - ub : 0;
  // a new head starts at item i (its operands must be loaded first)
  auto head_starts = [&](int i) { return i == 0 || (ub + i) % p.ntiles == 0; };

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(q_full + i, 1);
      mbar_init(q_conv + i, 2);
      mbar_init(q_empty + i, 1);
    }
    mbar_init(h_full, 1);
    mbar_init(h_free, 1);
    mbar_init(bar_ffullA, 1);
    mbar_init(bar_ffreeA, 8);
    mbar_init(bar_ffullB, 1);
    mbar_init(bar_ffreeB, 8);
    mbar_init(bar_pfull, 8);
    mbar_init(bar_ofull, 1);
    mbar_init(bar_drain, 1);
    mbar_init(bar_never, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(tmem_slot, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= 10) {
    // ---------------------------------------------------------- converters
    const int ctid = tid - 320;
    for (int i = 0; i < n; ++i) {
      const int buf = i & 1;
      bool w = true;
      if (lane == 0) w = wait_one(q_full + buf, (i >> 1) & 1, abort_flag, p.dev_status);
      if (__shfl_sync(0xffffffffu, w ? 1 : 0, 0) == 0) break;
      mbar_wait(q_full + buf, (i >> 1) & 1);   // passes at once (the data's visibility)
      q_to_fp16(s0 + G::oQ + buf * kTileBytes, ctid, p.dev_status);
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(q_conv + buf);
    }
    __syncwarp();
  } else if (warp == 9) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && n > 0) {
      int nq[2] = {0, 0}, nh = 0;        // loads issued: per Q buffer, head operands
      auto load_head = [&](int i) {
        const int bh = (ub + i) / p.ntiles, h = bh % p.H;
        const int hw = p.heads_w == 1 ? 0 : h;
        mbar_arrive_expect_tx(h_full, G::kWq + img_bytes(M_));
        for (int r0 = 0; r0 < M_; r0 += 16)
          tma_load_2d(sm + G::oW + r0 * 128, &tm_w, 0, hw * G::NW + r0, h_full);
        const uint8_t* src = p.images + (size_t)bh * img_bytes(M_);
        for (uint32_t o = 0; o < img_bytes(M_); o += 16384)
          bulk_load(sm + G::oImg + o, src + o,
                    img_bytes(M_) - o < 16384 ? img_bytes(M_) - o : 16384, h_full);
        ++nh;
      };
      auto load_q = [&](int i) {
        const int u = ub + i, bh = u / p.ntiles, t = u % p.ntiles, buf = i & 1;
        mbar_arrive_expect_tx(q_full + buf, kTileBytes);
        tma_load_4d(sm + G::oQ + buf * kTileBytes, &tm_q, 0, t * kT, bh % p.H, bh / p.H,
                    q_full + buf);
        ++nq[buf];
      };
      prefetch_tmap(&tm_w);
      prefetch_tmap(&tm_q);
      load_q(0);
      if (n > 1) load_q(1);
      // the head operands come from the split reduce (this launch may have
      // started before it finished)
      asm volatile("griddepcontrol.wait;" ::: "memory");
      load_head(0);
      bool ok = true;
      int heads_done = 0;                 // h_free phases passed
      for (int i = 0; ok && i + 1 < n; ++i) {
        // Q tile i + 2 into tile i's buffer once tile i's feature GEMM has read it
        if (i + 2 < n) {
          if (!(ok = wait_one(q_empty + (i & 1), (i >> 1) & 1, abort_flag, p.dev_status))) break;
          load_q(i + 2);
        }
        // the next head's operands once this head's last GEMMs are done
        if (head_starts(i + 1)) {
          if (!(ok = wait_one(h_free, heads_done & 1, abort_flag, p.dev_status))) break;
          ++heads_done;
          load_head(i + 1);
        }
      }
      if (!ok) {
        // aborted: leave no copy in flight (a completed phase passes at once)
        for (int i = 0; i < 2; ++i)
          if (nq[i] > 0) mbar_wait(q_full + i, (uint32_t)(nq[i] - 1) & 1u);
        if (nh > 0) mbar_wait(h_full, (uint32_t)(nh - 1) & 1u);
      }
    }
    __syncwarp();
  } else if (warp == 8) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0 && n > 0) {
      bool ok = true;
      int heads_seen = 0;
      // Q W^T, part A (features [0, M/2)) or B ([M/2, M)); fp16, fp32 in TMEM
      auto features = [&](int i, int part) {
        const uint32_t sq = s0 + G::oQ + (i & 1) * kTileBytes;
        constexpr uint32_t idh = idesc(128, M_ / 2, false, false, true);
#pragma unroll
        for (int s = 0; s < kD / 16; ++s)
          mma(tmem + G::tP + part * (M_ / 2), sdesc(sq + s * 32, 16, 1024),
              sdesc(s0 + G::oW + part * (M_ / 2) * 128 + s * 32, 16, 1024), idh, s > 0);
        if (part == 0) {
          mma_commit(bar_ffullA);
        } else {
          mma_commit(bar_ffullB);
          mma_commit(q_empty + (i & 1));
        }
      };
      // features of item i: the head's operands (first item of a head), the
      // converted Q tile, the previous item's TMEM columns released
      auto issue_features = [&](int i) -> bool {
        if (head_starts(i)) {
          if (!wait_one(h_full, heads_seen & 1, abort_flag, p.dev_status)) return false;
          ++heads_seen;
        }
        if (!wait_one(q_conv + (i & 1), (i >> 1) & 1, abort_flag, p.dev_status)) return false;
        if (i > 0 && !wait_one(bar_ffreeA, (i - 1) & 1, abort_flag, p.dev_status)) return false;
        tc_fence_after();
        features(i, 0);
        if (i > 0 && !wait_one(bar_ffreeB, (i - 1) & 1, abort_flag, p.dev_status)) return false;
        tc_fence_after();
        features(i, 1);
        return true;
      };
      auto output = [&](int i) -> bool {
        // [num hi | num lo | den hi, den lo] = Psi [S hi | S lo | (z hi, z lo)]
        if (!wait_one(bar_pfull, i & 1, abort_flag, p.dev_status)) return false;
        tc_fence_after();
        constexpr uint32_t id = idesc(128, 144, false, true, false);
#pragma unroll
        for (int s = 0; s < M_ / 16; ++s)
          mma(tmem + G::tO, sdesc(s0 + G::oPsi + (s / 4) * 16384 + (s % 4) * 32, 16, 1024),
              sdesc(s0 + G::oImg + s * 2048, img_s_bytes(M_), 1024), id, s > 0);
        mma_commit(bar_ofull);
        return true;
      };
      ok = issue_features(0);
      for (int i = 0; ok && i < n; ++i) {
        if (i + 1 < n && !head_starts(i + 1)) {
          // the next tile's features first: they run under this tile's exponentials
          if (!(ok = issue_features(i + 1))) break;
          if (!(ok = output(i))) break;
        } else {
          // last tile of a head: its output GEMM, then the head's operands are free
          if (!(ok = output(i))) break;
          if (i + 1 < n) {
            mma_commit(h_free);
            if (!(ok = issue_features(i + 1))) break;
          }
        }
      }
      if (!ok) drain_mmas(bar_drain);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int quad = warp & 3, half = warp >> 2;
    const int row = quad * 32 + lane;
    const uint32_t lane_tm = tmem + ((uint32_t)(quad * 32) << 16);
    const int f_r0 = half * (M_ / 4), f_r1 = M_ / 2 + half * (M_ / 4);
    // the output rows of item i (num / den read from TMEM): each thread packs
    // its half row into the staging area (the second half of the Psi buffer,
    // which the next tile's first pass does not write; 16-byte chunks
    // XOR-swizzled by row, as the output map's 128-byte swizzle expects), then
    // one thread stores the tile with a tensor store. The staging is free again
    // once that store has read it (thread 0 waits for that before the second
    // pass's Psi stores; an epilogue barrier follows).
    const uint32_t stage = s0 + G::oPsi + M_ * 128;
    auto store_out = [&](int i) {
      const int u = ub + i, bh = u / p.ntiles, t = u % p.ntiles, b = bh / p.H, h = bh % p.H;
      uint32_t vh[32], vl[32];
      tmem_ld32_async(lane_tm + G::tO + half * 32, vh);
      tmem_ld32_async(lane_tm + G::tO + 64 + half * 32, vl);
      // (each synchronous load waits for every load of the thread)
      const float den = tmem_ld1(lane_tm + G::tO + 128) + tmem_ld1(lane_tm + G::tO + 129);
      tmem_wait_ld(vh);
      tmem_wait_ld(vl);
      const int tok = t * kT + row;
      const bool live = tok < p.L && (p.qmask == nullptr || p.qmask[(size_t)b * p.L + tok] != 0);
      const float inv = live && den > 0.f ? 1.f / den : 0.f;
      float sum = den;                  // non-finite if any value is
      uint32_t w[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const float a = (__uint_as_float(vh[2 * e]) + __uint_as_float(vl[2 * e])) * inv;
        const float c = (__uint_as_float(vh[2 * e + 1]) + __uint_as_float(vl[2 * e + 1])) * inv;
        sum += a + c;
        w[e] = pack_bf16(a, c);
      }
      if (tok < p.L && !isfinite(sum)) report(p.dev_status, DARK_ERR_NUMERIC);
#pragma unroll
      for (int c = 0; c < 4; ++c)
        st_shared_v4(stage + row * 128 + (uint32_t)(((half * 4 + c) ^ (row & 7)) * 16), w[4 * c],
                     w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
      fence_async_smem();
      epi_sync();
      if (tid == 0) {
        tma_store_4d(&tm_o, stage, 0, t * kT, h, b);
        bulk_commit_group();
      }
    };
    bool ok = n > 0;
    if (ok && p.stall > 0) ok = epi_wait(bar_never, 0, abort_flag, p.dev_status, p.stall);
    for (int i = 0; ok && i < n; ++i) {
      if (!(ok = epi_wait(bar_ffullA, i & 1, abort_flag, p.dev_status))) break;
      tc_fence_after();
      bool have_b = false;
      float qoff = 0.f;
      if (p.stab_q) {
        // the row maximum over all M features (both parts, both thread halves)
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
        red[half * 128 + row] = mx;
        epi_sync();
        qoff = fmaxf(red[row], red[128 + row]);
        epi_sync();                     // red may be reused
      }
      // ---- pass 0 (part A)
      uint32_t fv[NH][32], pk[NH][16];
#pragma unroll
      for (int q = 0; q < NH; ++q) tmem_ld32_async(lane_tm + G::tP + f_r0 + 32 * q, fv[q]);
#pragma unroll
      for (int q = 0; q < NH; ++q) tmem_wait_ld(fv[q]);
      tc_fence_before();
      warp_arrive(bar_ffreeA);
#pragma unroll
      for (int q = 0; q < NH; ++q) exp2_pack32(fv[q], qoff, false, pk[q]);
      // ---- the previous tile's output GEMM is done: its rows out, Psi free
      if (i > 0) {
        if (!(ok = epi_wait(bar_ofull, (i - 1) & 1, abort_flag, p.dev_status))) break;
        tc_fence_after();
        store_out(i - 1);
      }
#pragma unroll
      for (int q = 0; q < NH; ++q) store_row32(pk[q], s0 + G::oPsi, row, f_r0 + 32 * q);
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
      for (int q = 0; q < NH; ++q) exp2_pack32(fv[q], qoff, false, pk[q]);
      if (i > 0) {
        // the previous tile's tensor store has read the staging
        if (tid == 0) bulk_wait_group_read();
        epi_sync();
      }
#pragma unroll
      for (int q = 0; q < NH; ++q) store_row32(pk[q], s0 + G::oPsi, row, f_r1 + 32 * q);
      fence_async_smem();
      tc_fence_before();
      warp_arrive(bar_pfull);
    }
    if (ok) {
      // the last tile's rows
      ok = epi_wait(bar_ofull, (n - 1) & 1, abort_flag, p.dev_status);
      tc_fence_after();
      if (ok) store_out(n - 1);
    }
    if (tid == 0) bulk_wait_group();    // every tensor store has completed
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

struct Layout {
  int ntiles, nsplit;           // key tiles per head and key ranges per head
  int qtiles;                   // query tiles per head
  size_t off_part, off_img, off_shift, total;   // shift: the stabiliser's per-range maxima
};

// Lq queries over Lk keys (equal for self-attention).
Layout layout(int B, int H, int Lq, int Lk, int m) {
  Layout s;
  const int bh = B * H;
  s.ntiles = (Lk + kT - 1) / kT;
  s.qtiles = (Lq + kT - 1) / kT;
  s.nsplit = kSms / bh;
  if (s.nsplit < 1) s.nsplit = 1;
  if (s.nsplit > s.ntiles) s.nsplit = s.ntiles;
  s.off_part = kWsHeader;
  s.off_img = align_up(s.off_part + (size_t)bh * s.nsplit * 65 * m * 4, 1024);
  s.off_shift = align_up(s.off_img + (size_t)bh * img_bytes(m), 256);
  s.total = align_up(s.off_shift + (size_t)bh * s.nsplit * 4, 256);
  return s;
}



template <int M_, int R_>
cudaError_t launch(const FwdArgs& a, const CUtensorMap& tw, const CUtensorMap& tq,
                   const CUtensorMap& tk, const CUtensorMap& tv) {
  const Layout s = layout(a.B, a.H, a.L, a.Lk, a.m);
  char* ws = (char*)a.ws;
  float* partials = (float*)(ws + s.off_part);
  uint8_t* images = (uint8_t*)(ws + s.off_img);
  const int bh = a.B * a.H;

  const bool stab = (a.flags & DARK_STABILISE) != 0;
  float* shifts = stab ? (float*)(ws + s.off_shift) : nullptr;
  cudaError_t e = tc_launch_key_states(a, tw, tk, tv, s.ntiles, s.nsplit, partials, shifts);
  if (e != cudaSuccess) return e;
  reduce_kernel<<<dim3((9 * a.m + 255) / 256, bh), 256, 0, a.stream>>>(
      partials, s.nsplit, a.m, shifts, images, a.st_kv, a.st_z, a.st_shift);

  QueryParams qp;
  qp.out = (__nv_bfloat16*)a.out;
  qp.ob = a.os[0];
  qp.oh = a.os[1];
  qp.ol = a.os[2];
  qp.B = a.B;
  qp.H = a.H;
  qp.L = a.L;
  qp.ntiles = s.qtiles;
  qp.heads_w = a.heads_w;
  qp.total_tiles = bh * s.qtiles;
  qp.qmask = a.qmask;
  qp.images = images;
  qp.stab_q = stab ? 1 : 0;
  qp.dev_status = a.dev_status;
  qp.stall = test_stall_cycles();
  using QG = QueryCfg<M_, R_>;
  static int smem_set[64];
  e = set_smem_limit_once((const void*)queries_kernel<M_, R_>, (int)QG::kSmem, smem_set);
  if (e != cudaSuccess) return e;
  const int grid = qp.total_tiles < kSms ? qp.total_tiles : kSms;
  // programmatic dependent launch after the reduce: the CTAs set up, load and
  // convert their first Q tiles while the reduce finishes
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = QG::kSmem;
  cfg.stream = a.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, queries_kernel<M_, R_>, tw, tq, a.tm_o, qp);
}

}  // namespace

bool tc_noncausal_supported(FwdArgs& a) {
  if (a.dtype != DARK_BF16 || a.d != kD) return false;
  if (!(a.m == 128 || a.m == 256) || a.r % 16 != 0 || a.r < 16 || a.r > 64) return false;
  return tc_make_maps(a);
}

size_t tc_noncausal_workspace_bytes(int B, int H, int Lq, int Lk, int m, int d) {
  if (d != kD || !(m == 128 || m == 256)) return 0;
  return layout(B, H, Lq, Lk, m).total;
}

cudaError_t tc_noncausal_forward(const FwdArgs& a) {
  if (!a.maps_ready) return cudaErrorInvalidValue;
  const CUtensorMap &tw = a.tm_w, &tq = a.tm_q, &tk = a.tm_k, &tv = a.tm_v;
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
