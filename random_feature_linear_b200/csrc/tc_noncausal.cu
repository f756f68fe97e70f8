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

namespace dark {
namespace {

using namespace tc;

constexpr int kD = 64;
constexpr int kT = 128;                     // tokens per tile
constexpr int kThreads = kFwdThreads;
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
// is the state's shift.
__global__ void reduce_kernel(const float* __restrict__ partials, int nsplit, int m,
                              const float* __restrict__ shifts, uint8_t* __restrict__ images,
                              float* __restrict__ st_kv, float* __restrict__ st_z,
                              float* __restrict__ st_shift) {
  const int bh = blockIdx.y;
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= 65 * m) return;
  const int col = idx / m, f = idx % m;
  const float* src = partials + (size_t)bh * nsplit * 65 * m + idx;
  float acc = 0.f;
  if (shifts == nullptr) {
    for (int s = 0; s < nsplit; ++s) acc += src[(size_t)s * 65 * m];
  } else {
    const float* sh = shifts + (size_t)bh * nsplit;
    float cmax = -INFINITY;
    for (int s = 0; s < nsplit; ++s) cmax = fmaxf(cmax, sh[s]);
    for (int s = 0; s < nsplit; ++s)
      if (sh[s] > -INFINITY) acc += exp2f(sh[s] - cmax) * src[(size_t)s * 65 * m];
    if (idx == 0 && st_shift != nullptr) st_shift[bh] = cmax > -INFINITY ? cmax : 0.f;
  }
  const __nv_bfloat16 hi = __float2bfloat16_rn(acc);
  const __nv_bfloat16 lo = __float2bfloat16_rn(acc - __bfloat162float(hi));
  uint8_t* img = images + (size_t)bh * img_bytes(m);
  const uint32_t row = (uint32_t)(f / 8) * 1024 + (uint32_t)(f % 8) * 128;
  if (col < 64) {
    const uint32_t off = row + (uint32_t)((((col / 8) ^ (f % 8)) * 16)) + (uint32_t)(col % 8) * 2;
    *reinterpret_cast<__nv_bfloat16*>(img + off) = hi;
    *reinterpret_cast<__nv_bfloat16*>(img + img_s_bytes(m) + off) = lo;
    if (st_kv != nullptr) st_kv[((size_t)bh * m + f) * 64 + col] = acc;
  } else {
    // columns 0-7 and 8-15 of the third block: (z hi, z lo, 0, ...), zeros
    uint8_t* zz = img + 2 * img_s_bytes(m) + row;
    const uint32_t w0 = (uint32_t)__bfloat16_as_ushort(hi) | ((uint32_t)__bfloat16_as_ushort(lo) << 16);
    *reinterpret_cast<uint4*>(zz + (uint32_t)((0 ^ (f % 8)) * 16)) = make_uint4(w0, 0u, 0u, 0u);
    *reinterpret_cast<uint4*>(zz + (uint32_t)((1 ^ (f % 8)) * 16)) = make_uint4(0u, 0u, 0u, 0u);
    if (st_z != nullptr) st_z[(size_t)bh * m + f] = acc;
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
  static constexpr uint32_t oRed = oBar + 64;              // [2][128] fp32 row maxima
  static constexpr uint32_t kSmem = oRed + 1024 + 1024;
  static constexpr uint32_t tP = 0, tO = 256;
  static_assert(kSmem <= 232448, "shared memory");
};

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
  uint64_t* bar_drain = bar_q + 5;      // abort path: the issued MMAs completed
  uint64_t* bar_never = bar_q + 6;      // completed by nothing (testing stall)

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
    mbar_init(bar_drain, 1);
    mbar_init(bar_never, 1);
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

  uint32_t ph_q = 0, ph_mma = 0, ph_head = 0;  // ph_q bit i: parity of buffer i
  int cur_bh = -1;
  bool abort = false;
  // load phases started / waited for: query buffers, head operands
  int q_issued[2] = {ue > ub ? 1 : 0, 0}, q_waited[2] = {0, 0}, h_issued = 0, h_waited = 0;
  if (ue > ub && p.stall > 0 && !wait_all(bar_never, 0, p.dev_status, p.stall)) abort = true;
  for (int u = ub; u < ue && !abort; ++u) {
    const int i = u - ub, buf = i & 1;
    const int bh = u / p.ntiles, t = u % p.ntiles, b = bh / p.H, h = bh % p.H;
    if (bh != cur_bh) {
      // W' rows and the [S | z] image of this head (all earlier MMAs have completed)
      if (tid == 0) {
        const int hw = p.heads_w == 1 ? 0 : h;
        ++h_issued;
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
      ++h_waited;
      cur_bh = bh;
    }
    if (!wait_all(&bar_q[buf], (ph_q >> buf) & 1u, p.dev_status)) { abort = true; break; }
    ph_q ^= 1u << buf;
    ++q_waited[buf];
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
      ++q_issued[buf ^ 1];
      mbar_arrive_expect_tx(&bar_q[buf ^ 1], kTileBytes);
      tma_load_4d(sm + G::oQ + (buf ^ 1) * kTileBytes, &tm_q, 0, nt * kT, nbh % p.H, nbh / p.H,
                  &bar_q[buf ^ 1]);
    }
    {
      const float qoff = p.stab_q ? row_max_pair(lane_tm + G::tP, half, M_ / 2,
                                                  (float*)(sm + G::oRed), row)
                                  : 0.f;
      exp2_rows_to_smem(lane_tm + G::tP, half * (M_ / 2), (half + 1) * (M_ / 2), qoff, false,
                        s0 + G::oPsi, row);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      // [num hi | num lo | den hi, den lo] = Psi [S hi | S lo | (z hi, z lo)]
      constexpr uint32_t id = idesc(128, 144, false, true, false);
#pragma unroll
      for (int s = 0; s < M_ / 16; ++s)
        mma(tmem + G::tO, sdesc(s0 + G::oPsi + (s / 4) * 16384 + (s % 4) * 32, 16, 1024),
            sdesc(s0 + G::oImg + s * 2048, img_s_bytes(M_), 1024), id, s > 0);
      mma_commit(bar_mma);
    }
    if (!wait_all(bar_mma, ph_mma, p.dev_status)) { abort = true; break; }
    ph_mma ^= 1;
    tc_fence_after();
    {
      const float den = tmem_ld1(lane_tm + G::tO + 128) + tmem_ld1(lane_tm + G::tO + 129);
      float v[32], vl[32];
      tmem_ld32(lane_tm + G::tO + half * 32, v);
      tmem_ld32(lane_tm + G::tO + 64 + half * 32, vl);
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] += vl[i];
      const int tok = t * kT + row;
      if (tok < p.L) {
        const bool live = p.qmask == nullptr || p.qmask[(size_t)b * p.L + tok] != 0;
        const float inv = live && den > 0.f ? 1.f / den : 0.f;
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
  if (abort && tid == 0) {
    // no copy or MMA of this CTA may still be running when TMEM is freed
    drain_loads(bar_head, h_issued, h_waited);
    drain_loads(&bar_q[0], q_issued[0], q_waited[0]);
    drain_loads(&bar_q[1], q_issued[1], q_waited[1]);
    drain_mmas(bar_drain);
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
  reduce_kernel<<<dim3((65 * a.m + 255) / 256, bh), 256, 0, a.stream>>>(
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
  queries_kernel<M_, R_><<<grid, kThreads, QG::kSmem, a.stream>>>(tw, tq, qp);
  return cudaGetLastError();
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
