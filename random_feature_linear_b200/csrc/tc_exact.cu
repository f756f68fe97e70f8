// Exact learned-kernel attention on sm_100a tensor cores (bf16 I/O; d = 64 with
// r <= 64, d = 128 with r <= 128): out_i = sum_j softmax_j(u_i . w_j) v_j with
// u = M q~, w = M k~
// (README, section "Attention modes": in the exact mode M acts on queries and
// keys and ordinary softmax attention with scaled scores follows).
//
// One CTA (256 threads) per 128-query tile of one (batch, head):
//   Q tile (TMA, bf16 -> fp16) x W'_bot^T -> 2 p_q (fp16, a K-major operand; the
//   projection's last r rows are c_m M, so 2 p_q . p_k is the score in base 2);
//   per 128-key tile:
//     K tile (TMA) x W'_bot^T -> p_k (fp16 operand)        tcgen05, N = r
//     scores S = (2 p_q) p_k^T                              tcgen05, N = 128
//     key mask, causal mask, running row maximum (the two thread halves of a
//     row exchange their maxima), P = 2^(S - max) as bf16 into shared memory
//     [num | den] = P [V | 1]                               tcgen05, N = d + 16
//     O = O * 2^(old max - new max) + num, l likewise with den (registers)
//   out = O / l.
// The next key tile loads while the current scores are processed, the next
// value tile while the next projection runs. Every wait is bounded; a wait
// that runs out stores DARK_ERR_TIMEOUT and the CTA leaves its loop.
#include <string.h>

#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"
#include "tc_keys.cuh"

namespace dark {
namespace {

using namespace tc;

constexpr int kT = 128;                    // queries per CTA, keys per tile
constexpr int kThreads = kFwdThreads;
constexpr int kBlk = kT * 64 * 2;          // one 128 x 64 block of 16-bit elements (16 KB)

// Shared memory (1024-byte aligned blocks) and TMEM of the kernel for head
// dimension D_: d = 64 fits two CTAs per SM (~106 KB, 256 TMEM columns each),
// d = 128 one (~177 KB, 512 columns).
template <int D_>
struct ExCfg {
  static constexpr int DS = D_ / 64;                  // 64-column slabs of d
  static constexpr int RMAX = D_;                     // r <= d (projection blocks fit the tiles)
  static constexpr uint32_t kWslab = RMAX * 128;      // W'_bot rows of one slab (fp16)
  static constexpr uint32_t oW = 0;
  static constexpr uint32_t oQ = oW + DS * kWslab;    // Q tile, then 2 p_q (fp16, K-major blocks)
  static constexpr uint32_t oK = oQ + DS * kBlk;      // K tile, then p_k
  static constexpr uint32_t oV = oK + DS * kBlk;      // V tile (bf16, keys x d, DS blocks)
  static constexpr uint32_t oOnes = oV + DS * kBlk;   // bf16 ones: [V | 1] as one N = d + 16 operand
  static constexpr uint32_t oP = oOnes + kBlk;        // P: 128 queries x 128 keys bf16, two K blocks
  static constexpr uint32_t oMax = oP + 2 * kBlk;     // row maxima of the two thread halves
  static constexpr uint32_t oKv = oMax + 2 * kT * 4;  // validity of the tile's 128 keys (bytes)
  static constexpr uint32_t oBar = oKv + kT;
  static constexpr uint32_t kSmem = oBar + 64 + 1024;
  // TMEM columns: scores [0, 128); projection [128, 128 + r) and, later in the
  // same tile, [num | den] [128, 128 + d + 16)
  static constexpr uint32_t tS = 0, tX = 128;
  static constexpr uint32_t kTmemCols = D_ == 64 ? 256 : 512;
  static_assert(tX + D_ + 16 <= kTmemCols, "tmem");
};

struct Params {
  __nv_bfloat16* out;
  int64_t ob, oh, ol;
  const uint8_t* kmask;                    // [B][Lk] or null
  const uint8_t* qmask;                    // [B][Lq] or null
  int B, H, Lq, Lk, nq, causal, heads_w, m, r;
  // key ranges: a query tile's key tiles are cut into splits of at most S
  // tiles, one CTA each (blockIdx: head fastest, then query tile, then split);
  // a tile with more than one split leaves (O, l, m) per split in `part`
  // ([B*H][nq][maxsplits] slots of 128 (d + 2) floats) for the combine kernel
  int S, maxsplits;
  float* part;
  int* dev_status;
  long long stall;                         // testing stall before the first wait (0: none)
};

// Key tiles of query tile qt.
__host__ __device__ inline int exact_key_tiles(int qt, int Lk, int causal) {
  const int nk_all = (Lk + 127) / 128;
  return causal ? (qt + 1 < nk_all ? qt + 1 : nk_all) : nk_all;
}

// Projection epilogue: this thread's row of the N = r projection in TMEM, times
// `scale`, as fp16 into K-major 128B-swizzled 64-column blocks 16 KB apart
// (columns r and up zero); each thread half writes 32 columns of every block.
__device__ __forceinline__ void proj_to_smem(uint32_t lane_taddr, int r, int nblk, float scale,
                                             uint32_t tile, int row, int half) {
  for (int kb = 0; kb < nblk; ++kb) {
    const int c0 = kb * 64 + half * 32;
    uint32_t w[16];
    if (c0 < r) {
      float v[32];
      tmem_ld32(lane_taddr + c0, v);
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const float a = c0 + 2 * e < r ? v[2 * e] * scale : 0.f;
        const float b = c0 + 2 * e + 1 < r ? v[2 * e + 1] * scale : 0.f;
        const __half2 hv = __floats2half2_rn(a, b);
        w[e] = *reinterpret_cast<const uint32_t*>(&hv);
      }
    } else {
#pragma unroll
      for (int e = 0; e < 16; ++e) w[e] = 0u;
    }
#pragma unroll
    for (int g = 0; g < 4; ++g)
      st_shared_v4(tile + kb * kBlk + kmajor_off(row, half * 32 + 8 * g, 0), w[4 * g],
                   w[4 * g + 1], w[4 * g + 2], w[4 * g + 3]);
  }
}

template <int D_>
__global__ void __launch_bounds__(kThreads, D_ == 64 ? 2 : 1)
    exact_tc_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                    const Params p) {
  using G = ExCfg<D_>;
  constexpr int DS = G::DS;
  // this CTA's (head, query tile, split); a split past the tile's key tiles
  // has nothing to do
  const int nbh = p.B * p.H;
  const int bh = blockIdx.x % nbh, qt = p.nq - 1 - (blockIdx.x / nbh) % p.nq;
  const int split = blockIdx.x / (nbh * p.nq);
  const int nk_q = exact_key_tiles(qt, p.Lk, p.causal);
  const int jb = split * p.S, je = jb + p.S < nk_q ? jb + p.S : nk_q;
  if (jb >= je) return;
  const bool whole = jb == 0 && je == nk_q;     // the tile's only split: output directly
  constexpr uint32_t oW = G::oW, oQ = G::oQ, oK = G::oK, oV = G::oV, oOnes = G::oOnes, oP = G::oP;
  constexpr uint32_t tS = G::tS, tX = G::tX;
  constexpr uint32_t kTile = DS * kBlk;         // one 128-token tile of d columns (bf16)
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t s0 = smem_u32(sm);
  uint64_t* bar_k = (uint64_t*)(sm + G::oBar);  // Q, W' (first), then each K tile
  uint64_t* bar_v = bar_k + 1;                  // each V tile
  uint64_t* bar_mma = bar_k + 2;
  uint32_t* tmem_slot = (uint32_t*)(bar_k + 3);
  uint64_t* bar_drain = bar_k + 4;              // abort path: the issued MMAs completed
  uint64_t* bar_never = bar_k + 5;              // completed by nothing (testing stall)
  float* smax = (float*)(sm + G::oMax);
  uint8_t* kval = sm + G::oKv;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int quad = warp & 3, half = warp >> 2;
  const int row = quad * 32 + lane;

  if (tid == 0) {
    mbar_init(bar_k, 1);
    mbar_init(bar_v, 1);
    mbar_init(bar_mma, 1);
    mbar_init(bar_drain, 1);
    mbar_init(bar_never, 1);
    fence_mbar_init();
    prefetch_tmap(&tm_w);
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
  }
  __syncwarp();
  if (warp == 0) tmem_alloc(tmem_slot, G::kTmemCols);
  for (int i = tid; i < kBlk / 16; i += kThreads)
    st_shared_v4(s0 + oOnes + i * 16, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_tm = tmem + ((uint32_t)(quad * 32) << 16);
  // query tiles in decreasing order of work first (causal: tile qt walks qt + 1
  // key tiles), so that the short ones fill in behind the long ones
  const int b = bh / p.H, h = bh % p.H;
  const int hw = p.heads_w == 1 ? 0 : h;
  const int q0 = qt * kT;
  const int qi = q0 + row;
  const int r = p.r;
  const int rb = (r + 63) / 64;                 // 64-column blocks of the projections

  uint32_t ph_k = 0, ph_v = 0, ph_mma = 0;
  bool abort = false;
  int k_issued = 1, k_waited = 0, v_issued = 0, v_waited = 0;   // load phases started / waited
  constexpr int kHalfD = D_ / 2;                // output columns per thread
  float o[kHalfD], l = 0.f, mrow = -INFINITY;
#pragma unroll
  for (int i = 0; i < kHalfD; ++i) o[i] = 0.f;

  // ---- Q and W'_bot, then K_0 and V_0
  if (tid == 0) {
    mbar_arrive_expect_tx(bar_k, (uint32_t)r * 128 * DS + kTile);
    for (int sl = 0; sl < DS; ++sl) {
      for (int r0 = 0; r0 < r; r0 += 16)
        tma_load_2d(sm + oW + sl * G::kWslab + r0 * 128, &tm_w, 64 * sl,
                    hw * (p.m + r) + p.m + r0, bar_k);
      tma_load_4d(sm + oQ + sl * kBlk, &tm_q, 64 * sl, q0, h, b, bar_k);
    }
  }
  if (p.stall > 0 && !wait_all(bar_never, 0, p.dev_status, p.stall)) abort = true;
  if (!abort && !wait_all(bar_k, ph_k, p.dev_status)) abort = true;
  ph_k ^= 1;
  if (!abort) {
    ++k_waited;
    ++k_issued;
    ++v_issued;
    if (tid == 0) {
      mbar_arrive_expect_tx(bar_k, kTile);
      for (int sl = 0; sl < DS; ++sl)
        tma_load_4d(sm + oK + sl * kBlk, &tm_k, 64 * sl, jb * kT, h, b, bar_k);
      mbar_arrive_expect_tx(bar_v, kTile);
      for (int sl = 0; sl < DS; ++sl)
        tma_load_4d(sm + oV + sl * kBlk, &tm_v, 64 * sl, jb * kT, h, b, bar_v);
    }
    to_fp16_inplace(s0 + oQ, kTile, p.dev_status);
    fence_async_smem();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      const uint32_t idp = idesc(128, r, false, false, true);
#pragma unroll
      for (int s = 0; s < D_ / 16; ++s)
        mma(tmem + tX, sdesc(s0 + oQ + (s / 4) * kBlk + (s % 4) * 32, 16, 1024),
            sdesc(s0 + oW + (s / 4) * G::kWslab + (s % 4) * 32, 16, 1024), idp, s > 0);
      mma_commit(bar_mma);
    }
    if (!wait_all(bar_mma, ph_mma, p.dev_status)) abort = true;
    ph_mma ^= 1;
    tc_fence_after();
    // the projection MMA has read the Q tile: 2 p_q over it
    if (!abort) proj_to_smem(lane_tm + tX, r, rb, 2.f, s0 + oQ, row, half);
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
  }

  for (int j = jb; j < je && !abort; ++j) {
    const int k0 = j * kT;
    // ---- K_j: projection p_k
    if (!wait_all(bar_k, ph_k, p.dev_status)) { abort = true; break; }
    ph_k ^= 1;
    ++k_waited;
    to_fp16_inplace(s0 + oK, kTile, p.dev_status);
    fence_async_smem();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      const uint32_t idp = idesc(128, r, false, false, true);
#pragma unroll
      for (int s = 0; s < D_ / 16; ++s)
        mma(tmem + tX, sdesc(s0 + oK + (s / 4) * kBlk + (s % 4) * 32, 16, 1024),
            sdesc(s0 + oW + (s / 4) * G::kWslab + (s % 4) * 32, 16, 1024), idp, s > 0);
      mma_commit(bar_mma);
    }
    if (!wait_all(bar_mma, ph_mma, p.dev_status)) { abort = true; break; }
    ph_mma ^= 1;
    tc_fence_after();
    proj_to_smem(lane_tm + tX, r, rb, 1.f, s0 + oK, row, half);
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    // ---- scores S = (2 p_q) p_k^T
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t ids = idesc(128, 128, false, false, true);
      for (int s = 0; s < rb * 4; ++s)
        mma(tmem + tS, sdesc(s0 + oQ + (s / 4) * kBlk + (s % 4) * 32, 16, 1024),
            sdesc(s0 + oK + (s / 4) * kBlk + (s % 4) * 32, 16, 1024), ids, s > 0);
      mma_commit(bar_mma);
    }
    // key validity of this tile, read from global memory once (the wait below
    // is a block-wide barrier)
    if (tid < kT) {
      const int key = k0 + tid;
      kval[tid] = (key < p.Lk && (p.kmask == nullptr || p.kmask[(size_t)b * p.Lk + key] != 0)) ? 1 : 0;
    }
    if (!wait_all(bar_mma, ph_mma, p.dev_status)) { abort = true; break; }
    ph_mma ^= 1;
    tc_fence_after();
    // the scores MMA has read p_k: the next key tile may load over it
    if (j + 1 < je) ++k_issued;
    if (tid == 0 && j + 1 < je) {
      mbar_arrive_expect_tx(bar_k, kTile);
      for (int sl = 0; sl < DS; ++sl)
        tma_load_4d(sm + oK + sl * kBlk, &tm_k, 64 * sl, k0 + kT, h, b, bar_k);
    }
    // ---- masks, row maximum, P = 2^(S - max) (this half: keys half*64 .. +63);
    // the scores are read from TMEM twice (maximum, then exponentials) rather
    // than held in registers
    auto visible = [&](int key) { return kval[key - k0] != 0 && (!p.causal || key <= qi); };
    float tmax = -INFINITY;
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      float v[32];
      tmem_ld32(lane_tm + tS + half * 64 + c * 32, v);
#pragma unroll
      for (int e = 0; e < 32; ++e)
        if (visible(k0 + half * 64 + c * 32 + e)) tmax = fmaxf(tmax, v[e]);
    }
    smax[half * kT + row] = tmax;
    __syncthreads();
    const float nmax = fmaxf(mrow, fmaxf(smax[row], smax[kT + row]));
    const float off = nmax == -INFINITY ? 0.f : nmax;
    const float scale = nmax == -INFINITY ? 1.f : ex2(mrow - nmax);
    mrow = nmax;
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      float v[32];
      tmem_ld32(lane_tm + tS + half * 64 + c * 32, v);
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        uint32_t w4[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j0 = c * 32 + 8 * g + 2 * e, key = k0 + half * 64 + j0;
          const float p0 = visible(key) ? ex2(v[8 * g + 2 * e] - off) : 0.f;
          const float p1 = visible(key + 1) ? ex2(v[8 * g + 2 * e + 1] - off) : 0.f;
          w4[e] = pack_bf16(p0, p1);
        }
        st_shared_v4(s0 + oP + kmajor_off(row, half * 64 + c * 32 + 8 * g, 16384), w4[0], w4[1],
                     w4[2], w4[3]);
      }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    // ---- [num | den] = P [V | 1]
    if (!wait_all(bar_v, ph_v, p.dev_status)) { abort = true; break; }
    ph_v ^= 1;
    ++v_waited;
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t idv = idesc(128, D_ + 16, false, true, false);
#pragma unroll
      for (int s = 0; s < kT / 16; ++s)
        mma(tmem + tX, sdesc(s0 + oP + (s / 4) * 16384 + (s % 4) * 32, 16, 1024),
            sdesc(s0 + oV + s * 2048, kBlk, 1024), idv, s > 0);
      mma_commit(bar_mma);
    }
    if (!wait_all(bar_mma, ph_mma, p.dev_status)) { abort = true; break; }
    ph_mma ^= 1;
    tc_fence_after();
    // the value MMA has read V: the next value tile may load
    if (j + 1 < je) ++v_issued;
    if (tid == 0 && j + 1 < je) {
      mbar_arrive_expect_tx(bar_v, kTile);
      for (int sl = 0; sl < DS; ++sl)
        tma_load_4d(sm + oV + sl * kBlk, &tm_v, 64 * sl, k0 + kT, h, b, bar_v);
    }
    {
#pragma unroll
      for (int c = 0; c < kHalfD; c += 32) {
        float v[32];
        tmem_ld32(lane_tm + tX + half * kHalfD + c, v);
#pragma unroll
        for (int i = 0; i < 32; ++i) o[c + i] = fmaf(o[c + i], scale, v[i]);
      }
      const float den = tmem_ld1(lane_tm + tX + D_);
      l = fmaf(l, scale, den);
    }
    tc_fence_before();
    __syncthreads();
  }
  if (abort && tid == 0) {
    // no copy or MMA of this CTA may still be running when TMEM is freed
    drain_loads(bar_k, k_issued, k_waited);
    drain_loads(bar_v, v_issued, v_waited);
    drain_mmas(bar_drain);
  }
  if (!abort && !whole) {
    // a partial result: the unnormalised numerator, l and the running maximum
    float* slot = p.part + ((size_t)(bh * p.nq + qt) * p.maxsplits + split) * (kT * (D_ + 2));
    float4* od = reinterpret_cast<float4*>(slot + (size_t)row * D_ + half * kHalfD);
#pragma unroll
    for (int i = 0; i < kHalfD / 4; ++i)
      od[i] = make_float4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
    if (half == 0) {
      slot[kT * D_ + row] = l;
      slot[kT * D_ + kT + row] = mrow;
    }
  }
  if (!abort && whole && qi < p.Lq) {
    const bool live = p.qmask == nullptr || p.qmask[(size_t)b * p.Lq + qi] != 0;
    const float inv = (live && l > 0.f) ? 1.f / l : 0.f;
    uint4* dst = reinterpret_cast<uint4*>(p.out + (int64_t)b * p.ob + (int64_t)h * p.oh +
                                          (int64_t)qi * p.ol + half * kHalfD);
    bool bad = false;
#pragma unroll
    for (int q4 = 0; q4 < kHalfD / 8; ++q4) {
      uint32_t w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float a = o[8 * q4 + 2 * e] * inv, c = o[8 * q4 + 2 * e + 1] * inv;
        bad |= !isfinite(a) || !isfinite(c);
        w[e] = pack_bf16(a, c);
      }
      dst[q4] = make_uint4(w[0], w[1], w[2], w[3]);
    }
    if (bad) report(p.dev_status, DARK_ERR_NUMERIC);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, G::kTmemCols);
  }
}

}  // namespace

// Query tiles with more than one split: per row, m = max_s m_s and
// out = sum_s 2^(m_s - m) O_s / sum_s 2^(m_s - m) l_s (the splits' running
// maxima are base-2 exponents); 256 threads per (query tile, head), each thread
// half a row.
template <int D_>
__global__ void __launch_bounds__(256) exact_combine_kernel(const Params p) {
  const int qt = blockIdx.x, bh = blockIdx.y;
  const int ns = (exact_key_tiles(qt, p.Lk, p.causal) + p.S - 1) / p.S;
  if (ns <= 1) return;
  const int row = threadIdx.x & 127, half = threadIdx.x >> 7;
  const int qi = qt * kT + row;
  if (qi >= p.Lq) return;
  const int b = bh / p.H, h = bh % p.H;
  constexpr int kHalfD = D_ / 2;
  const size_t stride = (size_t)kT * (D_ + 2);
  const float* base = p.part + (size_t)(bh * p.nq + qt) * p.maxsplits * stride;
  float mx = -INFINITY;
  for (int s = 0; s < ns; ++s) mx = fmaxf(mx, base[s * stride + kT * D_ + kT + row]);
  float o[kHalfD], l = 0.f;
#pragma unroll
  for (int i = 0; i < kHalfD; ++i) o[i] = 0.f;
  if (mx > -INFINITY) {
    for (int s = 0; s < ns; ++s) {
      const float* sl = base + s * stride;
      const float ms = sl[kT * D_ + kT + row];
      if (!(ms > -INFINITY)) continue;       // no visible key in this split
      const float sc = exp2f(ms - mx);
      l = fmaf(sc, sl[kT * D_ + row], l);
      const float4* src = reinterpret_cast<const float4*>(sl + (size_t)row * D_ + half * kHalfD);
#pragma unroll
      for (int i = 0; i < kHalfD / 4; ++i) {
        const float4 x = src[i];
        o[4 * i] = fmaf(sc, x.x, o[4 * i]);
        o[4 * i + 1] = fmaf(sc, x.y, o[4 * i + 1]);
        o[4 * i + 2] = fmaf(sc, x.z, o[4 * i + 2]);
        o[4 * i + 3] = fmaf(sc, x.w, o[4 * i + 3]);
      }
    }
  }
  const bool live = p.qmask == nullptr || p.qmask[(size_t)b * p.Lq + qi] != 0;
  const float inv = (live && l > 0.f) ? 1.f / l : 0.f;
  uint4* dst = reinterpret_cast<uint4*>(p.out + (int64_t)b * p.ob + (int64_t)h * p.oh +
                                        (int64_t)qi * p.ol + half * kHalfD);
  bool bad = false;
#pragma unroll
  for (int q4 = 0; q4 < kHalfD / 8; ++q4) {
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float x0 = o[8 * q4 + 2 * e] * inv, x1 = o[8 * q4 + 2 * e + 1] * inv;
      bad |= !isfinite(x0) || !isfinite(x1);
      w[e] = pack_bf16(x0, x1);
    }
    dst[q4] = make_uint4(w[0], w[1], w[2], w[3]);
  }
  if (bad) report(p.dev_status, DARK_ERR_NUMERIC);
}

template <int D_>
cudaError_t launch_exact(const FwdArgs& a, const Params& p) {
  using G = ExCfg<D_>;
  static int smem_set[64];
  cudaError_t e = set_smem_limit_once((const void*)exact_tc_kernel<D_>, (int)G::kSmem, smem_set);
  if (e != cudaSuccess) return e;
  if (D_ == 64) {
    // two CTAs per SM (2 x 106 KB of shared memory, 2 x 256 TMEM columns); set
    // once per device, outside any later stream capture
    static int carveout_set[64];
    int dev = 0;
    e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64 && !carveout_set[dev]) {
      e = cudaFuncSetAttribute((const void*)exact_tc_kernel<D_>,
                               cudaFuncAttributePreferredSharedMemoryCarveout, 100);
      if (e != cudaSuccess) return e;
      carveout_set[dev] = 1;
    }
  }
  exact_tc_kernel<D_><<<a.B * a.H * p.nq * p.maxsplits, kThreads, G::kSmem, a.stream>>>(
      a.tm_w, a.tm_q, a.tm_k, a.tm_v, p);
  e = cudaGetLastError();
  if (e != cudaSuccess || p.maxsplits == 1) return e;
  exact_combine_kernel<D_><<<dim3(p.nq, a.B * a.H), 256, 0, a.stream>>>(p);
  return cudaGetLastError();
}

// Key tiles per split (d = 64 only): none while the query tiles alone give
// two waves of CTAs; otherwise the total key-tile work spread over about two
// waves (at least 2 tiles per split), so that the longest query tiles no
// longer set the time. (At d = 128, one CTA per SM, the splits' repeated
// query projections and the combine cost more than they gain: measured.)
void exact_split_plan(int B, int H, int Lq, int Lk, int causal, int d, int* S, int* maxsplits) {
  const int nq = (Lq + kT - 1) / kT, nk_all = (Lk + kT - 1) / kT;
  const long long ctas = (long long)B * H * nq;
  const long long slots = 2LL * num_sms();
  if (d != 64 || ctas >= 2 * slots || nk_all <= 2) {
    *S = nk_all;
    *maxsplits = 1;
    return;
  }
  long long total = 0;
  for (int qt = 0; qt < nq; ++qt) total += exact_key_tiles(qt, Lk, causal);
  total *= (long long)B * H;
  long long s = (total + 2 * slots - 1) / (2 * slots);
  if (s < 2) s = 2;
  if (s > nk_all) s = nk_all;
  int nk_max = 0;
  for (int qt = 0; qt < nq; ++qt) {
    const int k = exact_key_tiles(qt, Lk, causal);
    nk_max = k > nk_max ? k : nk_max;
  }
  *S = (int)s;
  *maxsplits = (int)((nk_max + s - 1) / s);
}

// d = 64 (r <= 64, two CTAs per SM) and d = 128 (r <= 128, one CTA per SM):
// the projections p_q, p_k overwrite the Q and K tiles, so r <= d
bool tc_exact_supported(FwdArgs& a) {
  if (a.dtype != DARK_BF16 || !(a.d == 64 || a.d == 128)) return false;
  if (a.r % 16 != 0 || a.r < 16 || a.r > a.d) return false;
  if (a.os[2] % 8 != 0) return false;          // 16-byte output stores
  return tc_make_maps(a);
}

cudaError_t tc_exact_forward(const FwdArgs& a) {
  if (!a.maps_ready) return cudaErrorInvalidValue;
  Params p;
  memset(&p, 0, sizeof(p));
  p.out = (__nv_bfloat16*)a.out;
  p.ob = a.os[0];
  p.oh = a.os[1];
  p.ol = a.os[2];
  p.kmask = a.mask;
  p.qmask = a.qmask;
  p.B = a.B;
  p.H = a.H;
  p.Lq = a.L;
  p.Lk = a.Lk;
  p.nq = (a.L + kT - 1) / kT;
  p.causal = (a.flags & DARK_CAUSAL) ? 1 : 0;
  p.heads_w = a.heads_w;
  p.m = a.m;
  p.r = a.r;
  p.dev_status = a.dev_status;
  p.stall = test_stall_cycles();
  exact_split_plan(a.B, a.H, a.L, a.Lk, p.causal, a.d, &p.S, &p.maxsplits);
  if (p.maxsplits > 1 && a.ws_bytes < tc_exact_workspace_bytes(a.B, a.H, a.L, a.Lk, a.d, p.causal)) {
    // a workspace without room for the splits' partials: one CTA per query tile
    p.S = (a.Lk + kT - 1) / kT;
    p.maxsplits = 1;
  }
  p.part = p.maxsplits > 1 ? (float*)((char*)a.ws + kWsHeader) : nullptr;
  return a.d == 64 ? launch_exact<64>(a, p) : launch_exact<128>(a, p);
}

size_t tc_exact_workspace_bytes(int B, int H, int Lq, int Lk, int d, int causal) {
  int S = 0, ms = 1;
  exact_split_plan(B, H, Lq, Lk, causal, d, &S, &ms);
  if (ms <= 1) return kWsHeader;
  const size_t nq = (size_t)(Lq + kT - 1) / kT;
  return align_up(kWsHeader + (size_t)B * H * nq * ms * kT * (d + 2) * 4, 256);
}

}  // namespace dark
