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
//   -> tcgen05 GEMM Psi Phi^T (scores) -> causal mask -> intra GEMM tril(A) [V | 1]
//   -> inter GEMM Psi [S_<c | z_<c] with the prefix split into hi + lo bf16
//      (bf16 alone moves outputs by ~1e-2) -> divide.
// Phi and Psi never leave shared memory. Every CTA walks a segment of
// consecutive chunks of one head and carries the prefix state in registers,
// adding Phi(K_c)^T [V_c | 1] after each chunk. With many heads (B*H >= #SMs)
// a segment is the whole head; with few heads each head is cut into G
// segments so that all SMs work, and a key-state launch comes first: it sums
// Phi(K)^T [V | 1] over each segment, and each CTA adds the sums of the
// segments before its own in segment order (deterministic, no waiting
// between blocks).
#include <string.h>

#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"
#include "tc_keys.cuh"
#include "tc_roles.cuh"

namespace dark {
namespace {

using namespace tc;

constexpr int kD = 64;          // head dimension handled by this kernel
constexpr int kC = 128;         // tokens per chunk (UMMA M)
constexpr int kThreads = kFwdThreads;
constexpr int kSms = 148;
constexpr int kTileBytes = kC * kD * 2;   // one 128 x 64 tile of 16-bit elements
constexpr uint32_t kTmemCols = 512;

template <int M_, int R_>
struct Cfg {
  static constexpr int MB = M_ / 128;
  static constexpr int NW = M_ + R_;                      // W' rows
  static constexpr uint32_t kW = NW * 128;                // W' bytes (fp16, 128 B rows)
  static constexpr uint32_t kZ = (M_ / 64) * 2048;        // the 16-row z operand
  // after the feature GEMMs the W' region holds the z operand and keys 64-127
  // of the masked-score operand (keys 0-63 sit in the Q tile)
  static constexpr uint32_t oA1 = kZ;
  static constexpr uint32_t kWReg = (kW > kZ + 16384 ? kW : kZ + 16384);
  static constexpr uint32_t kPhi = (M_ / 64) * 16384;     // 128 tokens x M_ features, bf16
  // shared memory offsets (all 1024-byte aligned)
  static constexpr uint32_t oW = 0;
  static constexpr uint32_t oQ = (oW + kWReg + 1023) / 1024 * 1024;
  // V, then K: once the key GEMM is done the K tile is refilled with bf16 ones,
  // so that [V | 1] is one MN-major operand of N = 80 (blocks 16 KB apart)
  static constexpr uint32_t oV = oQ + kTileBytes;
  static constexpr uint32_t oK = oV + kTileBytes;
  static constexpr uint32_t oPhi = oK + kTileBytes;
  static constexpr uint32_t oPsi = oPhi + kPhi;
  static constexpr uint32_t oOnes = oPsi + kPhi;
  static constexpr uint32_t oBar = oOnes + 2048;
  static constexpr uint32_t oRed = oBar + 64;              // [2][128] fp32 row maxima
  static constexpr uint32_t kSmem = oRed + 1024 + 1024;    // + alignment slack
  // TMEM columns
  // key features [0, M_) and norms [M_, M_ + R_); query features [256, 256 + M_)
  // (issued once the norms are read); once both feature blocks are consumed:
  // scores [0, 128), numerator hi | lo [128, 256), denominator hi, lo at 256,
  // 257 (16 columns) and chunk state [320, 480)
  static constexpr uint32_t tP = 0, tQ = 256, tA = 0, tNum = 128, tDen = 256, tD = 320;
  static_assert(NW <= 320 && M_ % 128 == 0 && R_ % 16 == 0, "shape");
  static_assert(tD + 80 * MB <= kTmemCols, "tmem");
};

struct Params {
  __nv_bfloat16* out;
  int64_t ob, oh, ol;           // out strides (elements)
  const uint8_t* mask;
  int B, H, L, nc;              // nc = chunks per head
  int heads_w;
  int nseg;                     // segments per head
  const float* seg_sums;        // [B*H*nseg][65][m] per-segment key states (nseg > 1)
  float *st_kv, *st_z;          // state after the last chunk
  // stabiliser (stab != 0): the key exponents of a CTA are taken relative to the
  // running maximum over the keys seen so far (the earlier segments' maxima in
  // seg_shift, then this segment's chunks), the prefix rescaled when it grows;
  // the query exponents relative to their row maximum
  const float* seg_shift;       // [B*H*nseg] (nseg > 1)
  float* st_shift;              // the state's key constant (state output)
  int stab;
  int* dev_status;
  long long stall;              // testing stall before the first wait (0: none)
};

template <int M_, int R_>
__global__ void __launch_bounds__(kThreads, 1)
    causal_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_q,
                  const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                  const __grid_constant__ CUtensorMap tm_o, const Params p) {
  using G = Cfg<M_, R_>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t s0 = smem_u32(sm);
  uint64_t* bar_tma = (uint64_t*)(sm + G::oBar);
  uint64_t* bar_mma = bar_tma + 1;
  uint32_t* tmem_slot = (uint32_t*)(bar_tma + 2);
  uint64_t* bar_drain = bar_tma + 3;    // abort path: the issued MMAs completed
  uint64_t* bar_never = bar_tma + 4;    // completed by nothing (testing stall)

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int quad = warp & 3, half = warp >> 2;
  const int row = quad * 32 + lane;           // TMEM lane = tile row of this thread
  const bool has_feat = half < G::MB;         // owns prefix-state row `feat`
  const int feat = half * 128 + row;

  if (tid == 0) {
    mbar_init(bar_tma, 1);
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
  if (warp == 0) tmem_alloc(tmem_slot, kTmemCols);
  // ones operand for the z / denominator columns: 16 rows x 64 keys, K-major,
  // 1.0 in row 0 (its first 128 bytes) and zeros in rows 1-15, so that each
  // sum lands in a single column
  for (int i = tid; i < 2048 / 4; i += kThreads)
    ((uint32_t*)(sm + G::oOnes))[i] = i < 32 ? 0x3F803F80u : 0u;
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_tm = tmem + ((uint32_t)(quad * 32) << 16);
  const int bh = blockIdx.x / p.nseg, seg = blockIdx.x % p.nseg;
  const int c_begin = (int)((long long)seg * p.nc / p.nseg);
  const int c_end = (int)((long long)(seg + 1) * p.nc / p.nseg);
  const int b = bh / p.H, h = bh % p.H;
  const int hw = p.heads_w == 1 ? 0 : h;

  uint32_t ph_tma = 0, ph_mma = 0;
  float run[65];                               // prefix state row `feat` (fp32)
  float c_run = -INFINITY;                     // stabiliser: running key maximum
#pragma unroll
  for (int i = 0; i < 65; ++i) run[i] = 0.f;
  bool abort = false;
  int tma_issued = 0, tma_waited = 0;          // load phases started / waited for

  // W', K, V and Q tiles of the chunk starting at token t (one thread)
  auto issue_loads = [&](int t) {
    ++tma_issued;
    mbar_arrive_expect_tx(bar_tma, G::kW + 3 * kTileBytes);
    for (int r0 = 0; r0 < G::NW; r0 += 16)
      tma_load_2d(sm + G::oW + r0 * 128, &tm_w, 0, hw * G::NW + r0, bar_tma);
    tma_load_4d(sm + G::oK, &tm_k, 0, t, h, b, bar_tma);
    tma_load_4d(sm + G::oV, &tm_v, 0, t, h, b, bar_tma);
    tma_load_4d(sm + G::oQ, &tm_q, 0, t, h, b, bar_tma);
  };
  for (int c = c_begin; c < c_end && !abort; ++c) {
    const int t0 = c * kC;
    // ---------------------------------------------------------------- loads
    // (for later chunks they were issued during the previous chunk's output)
    if (tid == 0 && c == c_begin) issue_loads(t0);
    if (c == c_begin && p.stall > 0 && !wait_all(bar_never, 0, p.dev_status, p.stall)) {
      abort = true;
      break;
    }
    if (!wait_all(bar_tma, ph_tma, p.dev_status)) { abort = true; break; }
    ph_tma ^= 1;
    ++tma_waited;
    // this chunk's key validity, read now so that the load's latency passes
    // under the conversion and the key GEMM
    const int tok = t0 + row;
    const bool valid = tok < p.L && (p.mask == nullptr || p.mask[(size_t)b * p.L + tok] != 0);
    // the previous chunk's output tensor store has read its staging (in the
    // Psi region, written again below)
    if (tid == 0) bulk_wait_group_read();
    // k, then q: bf16 -> fp16 in place (the feature GEMMs run on fp16 operands);
    // the key GEMM starts while the query tile converts
    to_fp16_inplace(s0 + G::oK, kTileBytes, p.dev_status);
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
    to_fp16_inplace(s0 + G::oQ, kTileBytes, p.dev_status);
    fence_async_smem();
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
      // the norm columns are read: the query GEMM may now overwrite them
      tc_fence_before();
      __syncthreads();
      if (tid == 0) {
        tc_fence_after();
        constexpr uint32_t idq = idesc(128, (M_ < 256 ? M_ : 256), false, false, true);
#pragma unroll
        for (int s = 0; s < kD / 16; ++s)
          mma(tmem + G::tQ, sdesc(s0 + G::oQ + s * 32, 16, 1024),
              sdesc(s0 + G::oW + s * 32, 16, 1024), idq, s > 0);
        mma_commit(bar_mma);
      }
      if (p.stab) {
        // the running maximum starts from the earlier segments' maxima (the
        // key-state launch's results), then takes each chunk's largest valid
        // key exponent; the prefix carried in registers follows it
        if (c == c_begin && seg > 0) {
          asm volatile("griddepcontrol.wait;" ::: "memory");
          for (int g = 0; g < seg; ++g) c_run = fmaxf(c_run, p.seg_shift[bh * p.nseg + g]);
        }
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
        float cmx = red[0];
#pragma unroll
        for (int w = 1; w < kThreads / 32; ++w) cmx = fmaxf(cmx, red[w]);
        __syncthreads();
        if (cmx > c_run) {
          if (c_run > -INFINITY) {
            const float sc = exp2f(c_run - cmx);
#pragma unroll
            for (int i = 0; i < 65; ++i) run[i] *= sc;
          }
          c_run = cmx;
        }
        if (c_run > -INFINITY) nrm += c_run;
      }
      exp2_rows_to_smem(lane_tm + G::tP, half * (M_ / 2), (half + 1) * (M_ / 2), nrm, !valid,
                        s0 + G::oPhi, row);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    if (!wait_all(bar_mma, ph_mma, p.dev_status)) { abort = true; break; }
    ph_mma ^= 1;
    tc_fence_after();
    // ------------------------------------------------- epilogue: Psi(Q_c)
    {
      const float qoff = p.stab ? row_max_pair(lane_tm + G::tQ, half, M_ / 2,
                                                  (float*)(sm + G::oRed), row)
                                  : 0.f;
      exp2_rows_to_smem(lane_tm + G::tQ, half * (M_ / 2), (half + 1) * (M_ / 2), qoff, false,
                        s0 + G::oPsi, row);
    }
    for (int i = tid; i < kTileBytes / 16; i += kThreads)   // the key tile is consumed
      st_shared_v4(s0 + G::oK + i * 16, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    // ------------------ scores Psi Phi^T and chunk state Phi^T [V | 1] (N = 80)
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t ids = idesc(128, 128, false, false, false);
#pragma unroll
      for (int s = 0; s < M_ / 16; ++s) {
        const uint32_t off = (s / 4) * 16384 + (s % 4) * 32;
        mma(tmem + G::tA, sdesc(s0 + G::oPsi + off, 16, 1024), sdesc(s0 + G::oPhi + off, 16, 1024),
            ids, s > 0);
      }
      constexpr uint32_t idv = idesc(128, 80, true, true, false);
#pragma unroll
      for (int mb = 0; mb < G::MB; ++mb) {
#pragma unroll
        for (int s = 0; s < kC / 16; ++s)
          mma(tmem + G::tD + 80 * mb, sdesc(s0 + G::oPhi + mb * 32768 + s * 2048, 16384, 1024),
              sdesc(s0 + G::oV + s * 2048, G::oK - G::oV, 1024), idv, s > 0);
      }
      mma_commit(bar_mma);
    }
    if (c == c_begin && seg > 0) {
      // exclusive prefix of this segment: the earlier segments' key states
      // (written by the key-state launch, which may still be finishing: this
      // launch starts early and waits for it only here), added in segment order
      asm volatile("griddepcontrol.wait;" ::: "memory");
      // stabiliser: segment g's sum is scaled by 2^-(its maximum); c_run (set
      // in the key epilogue above) is at least every one of them
      if (has_feat) {
        for (int g = 0; g < seg; ++g) {
          const float* sp = p.seg_sums + (size_t)(bh * p.nseg + g) * 65 * M_ + feat;
          float sc = 1.f;
          if (p.stab) {
            const float cg = p.seg_shift[bh * p.nseg + g];
            if (!(cg > -INFINITY)) continue;
            sc = exp2f(cg - c_run);
          }
#pragma unroll
          for (int i = 0; i < 65; ++i) run[i] += sc * sp[(size_t)i * M_];
        }
      }
    }
    if (!wait_all(bar_mma, ph_mma, p.dev_status)) { abort = true; break; }
    ph_mma ^= 1;
    tc_fence_after();
    // ---- causal mask of the scores -> bf16 A operand (Q tile, W' region); the
    // prefix [S_<c | z_<c] as operands; this chunk's state added to the prefix
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
          const uint32_t blk = j0 < 64 ? s0 + G::oQ : s0 + G::oW + G::oA1;
          st_shared_v4(blk + kmajor_off(row, (j0 % 64) + 8 * g, 0), w4[0], w4[1], w4[2], w4[3]);
        }
      }
    }
    const bool have_prefix = c > 0;
    // S hi, S lo: MN-major blocks of M_ feature rows in the Phi region (M_ * 128
    // bytes apart); z hi, z lo: rows 0 and 1 of a 16-row K-major operand in the
    // W' region (rows 2-15 zero)
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
      const uint32_t zb = s0 + G::oW + (uint32_t)(feat / 64) * 2048;
      st_shared_u16(zb + kmajor_off(0, feat % 64, 0), *reinterpret_cast<const uint16_t*>(&zh));
      st_shared_u16(zb + kmajor_off(1, feat % 64, 0), *reinterpret_cast<const uint16_t*>(&zl));
    }
    if (have_prefix) {
      for (int i = tid; i < (M_ / 64) * 14 * 8; i += kThreads) {
        const int blk = i / 112, n = 2 + (i % 112) / 8, ch = i % 8;
        st_shared_v4(s0 + G::oW + blk * 2048 + (n / 8) * 1024 + (n % 8) * 128 + ch * 16, 0u, 0u, 0u, 0u);
      }
    }
    // add this chunk's state row `feat` (Phi(K_c)^T [V_c | 1], in TMEM) to the prefix
    if (has_feat) {
      uint32_t a[32], b2[32];
      const uint32_t base = tmem + ((uint32_t)(quad * 32) << 16) + G::tD + 80 * half;
      tmem_ld32_async(base, a);
      tmem_ld32_async(base + 32, b2);
      tmem_wait_ld(a);
      tmem_wait_ld(b2);
#pragma unroll
      for (int i = 0; i < 32; ++i) run[i] += __uint_as_float(a[i]);
#pragma unroll
      for (int i = 0; i < 32; ++i) run[32 + i] += __uint_as_float(b2[i]);
      run[64] += tmem_ld1(base + 64);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    // ---- [num hi | num lo] = Psi [S hi | S lo], [den hi, den lo] = Psi [z hi; z lo]
    // (one N = 128 and one N = 16 MMA per K-step), then num hi += tril(A) V and
    // den hi += tril(A) 1, all in one commit group
    if (tid == 0) {
      tc_fence_after();
      if (have_prefix) {
        constexpr uint32_t ids = idesc(128, 128, false, true, false);
        constexpr uint32_t idz = idesc(128, 16, false, false, false);
#pragma unroll
        for (int s = 0; s < M_ / 16; ++s) {
          const uint64_t ad = sdesc(s0 + G::oPsi + (s / 4) * 16384 + (s % 4) * 32, 16, 1024);
          mma(tmem + G::tNum, ad, sdesc(s0 + G::oPhi + s * 2048, M_ * 128, 1024), ids, s > 0);
          mma(tmem + G::tDen, ad, sdesc(s0 + G::oW + (s / 4) * 2048 + (s % 4) * 32, 16, 1024), idz,
              s > 0);
        }
      }
      constexpr uint32_t idv = idesc(128, 64, false, true, false);
      constexpr uint32_t id1 = idesc(128, 16, false, false, false);
#pragma unroll
      for (int s = 0; s < kC / 16; ++s) {
        const uint32_t ablk = s < 4 ? s0 + G::oQ : s0 + G::oW + G::oA1;
        const uint64_t ad = sdesc(ablk + (s % 4) * 32, 16, 1024);
        const uint32_t acc = (have_prefix || s > 0) ? 1u : 0u;
        mma(tmem + G::tNum, ad, sdesc(s0 + G::oV + s * 2048, 16384, 1024), idv, acc);
        mma(tmem + G::tDen, ad, sdesc(s0 + G::oOnes + (s % 4) * 32, 16, 1024), id1, acc);
      }
      mma_commit(bar_mma);
    }
    if (!wait_all(bar_mma, ph_mma, p.dev_status)) { abort = true; break; }
    ph_mma ^= 1;
    tc_fence_after();
    // every tile region has been read: the next chunk's tiles load during the output
    if (tid == 0 && c + 1 < c_end) issue_loads(t0 + kC);
    // ------------------------------------------------------------- output
    {
      float den = tmem_ld1(lane_tm + G::tDen);
      float v[32];
      tmem_ld32(lane_tm + G::tNum + half * 32, v);
      if (have_prefix) {
        float vl[32];
        tmem_ld32(lane_tm + G::tNum + 64 + half * 32, vl);
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] += vl[i];
        den += tmem_ld1(lane_tm + G::tDen + 1);
      }
      // the chunk's rows staged in the Psi region (free once the inter GEMM is
      // done; 16-byte chunks XOR-swizzled by row, as the output map's 128-byte
      // swizzle expects), then one tensor store (rows past L are not written)
      const float inv = den > 0.f ? 1.f / den : 0.f;
      uint32_t w[16];
      float sum = den;                  // non-finite if any value is
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const float a = v[2 * e] * inv, bb = v[2 * e + 1] * inv;
        sum += a + bb;
        w[e] = pack_bf16(a, bb);
      }
      if (tok < p.L && !isfinite(sum)) report(p.dev_status, DARK_ERR_NUMERIC);
      const uint32_t stage = s0 + G::oPsi;
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4)
        st_shared_v4(stage + row * 128 + (uint32_t)(((half * 4 + q4) ^ (row & 7)) * 16), w[4 * q4],
                     w[4 * q4 + 1], w[4 * q4 + 2], w[4 * q4 + 3]);
      fence_async_smem();
    }
    __syncthreads();
    if (tid == 0) {
      tma_store_4d(&tm_o, s0 + G::oPsi, 0, t0, h, b);
      bulk_commit_group();
    }
    tc_fence_before();
    __syncthreads();
  }
  if (!abort && p.st_kv != nullptr && has_feat && c_end == p.nc) {
    float* kv = p.st_kv + ((size_t)bh * M_ + feat) * kD;
#pragma unroll
    for (int i = 0; i < 64; ++i) kv[i] = run[i];
    p.st_z[(size_t)bh * M_ + feat] = run[64];
  }
  if (!abort && p.st_shift != nullptr && tid == 0 && c_end == p.nc)
    p.st_shift[bh] = c_run > -INFINITY ? c_run : 0.f;
  if (tid == 0) bulk_wait_group();      // every output tensor store has completed
  if (abort && tid == 0) {
    // no copy or MMA of this CTA may still be running when TMEM is freed
    drain_loads(bar_tma, tma_issued, tma_waited);
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
  int nc, nseg;
  size_t off_seg, off_shift, total;   // shift: the stabiliser's per-segment maxima
};

// Segments per head: 1 when the heads alone fill the SMs, else enough to give
// every SM a segment (at most one per chunk).
Layout layout(int B, int H, int L, int m) {
  Layout s;
  const int bh = B * H;
  s.nc = (L + kC - 1) / kC;
  s.nseg = bh >= kSms ? 1 : kSms / bh;
  if (s.nseg > s.nc) s.nseg = s.nc;
  s.off_seg = kWsHeader;
  s.off_shift = align_up(s.off_seg + (s.nseg > 1 ? (size_t)bh * s.nseg * 65 * m * 4 : 0), 256);
  s.total = align_up(s.off_shift + (size_t)bh * s.nseg * 4, 256);
  return s;
}

template <int M_, int R_>
cudaError_t launch(const FwdArgs& a, const CUtensorMap& tw, const CUtensorMap& tq,
                   const CUtensorMap& tk, const CUtensorMap& tv) {
  using G = Cfg<M_, R_>;
  const Layout s = layout(a.B, a.H, a.L, a.m);
  const int bh = a.B * a.H;
  float* seg = (float*)((char*)a.ws + s.off_seg);
  cudaError_t e;
  const bool stab = (a.flags & DARK_STABILISE) != 0;
  float* seg_shift = (float*)((char*)a.ws + s.off_shift);
  if (s.nseg > 1) {
    e = tc_launch_key_states(a, tw, tk, tv, s.nc, s.nseg, seg, stab ? seg_shift : nullptr);
    if (e != cudaSuccess) return e;
  }
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
  p.nseg = s.nseg;
  p.seg_sums = seg;
  p.st_kv = a.st_kv;
  p.st_z = a.st_z;
  p.seg_shift = seg_shift;
  p.st_shift = stab ? a.st_shift : nullptr;
  p.stab = stab ? 1 : 0;
  p.dev_status = a.dev_status;
  p.stall = test_stall_cycles();
  static int smem_set[64];
  e = set_smem_limit_once((const void*)causal_kernel<M_, R_>, (int)G::kSmem, smem_set);
  if (e != cudaSuccess) return e;
  // after the key-state launch: programmatic dependent launch, so that CTAs
  // start on SMs the key-state CTAs leave and wait for its results only where
  // they read them
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(bh * s.nseg);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = G::kSmem;
  cfg.stream = a.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = s.nseg > 1 ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, causal_kernel<M_, R_>, tw, tq, tk, tv, a.tm_o, p);
}



}  // namespace

bool tc_causal_supported(FwdArgs& a) {
  if (a.dtype != DARK_BF16 || a.d != kD) return false;
  if (!(a.m == 128 || a.m == 256) || a.r % 16 != 0 || a.r < 16 || a.r > 64) return false;
  return tc_make_maps(a);
}

size_t tc_causal_workspace_bytes(int B, int H, int L, int m, int d) {
  if (d != kD || !(m == 128 || m == 256)) return 0;
  return layout(B, H, L, m).total;
}

cudaError_t tc_causal_forward(const FwdArgs& a) {
  if (!a.maps_ready) return cudaErrorInvalidValue;
  const CUtensorMap &tw = a.tm_w, &tq = a.tm_q, &tk = a.tm_k, &tv = a.tm_v;
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
