// Shared by the tensor-core forward kernels: bounded block-wide mbarrier wait
// and the in-place bf16 -> fp16 conversion of a shared-memory operand tile.
#pragma once

#include "common.cuh"
#include "tc_common.cuh"

namespace dark {
namespace tc {

constexpr int kFwdThreads = 256;

// Every thread of the CTA waits (bounded by `limit` cycles); false on all of
// them if any wait ran out (DARK_ERR_TIMEOUT is then recorded).
__device__ __forceinline__ bool wait_all(uint64_t* bar, uint32_t parity, int* dev_status,
                                         long long limit = kWaitCycles) {
  const bool ok = mbar_wait(bar, parity, limit);
  const int bad = __syncthreads_or(ok ? 0 : 1);
  if (bad && threadIdx.x == 0) report(dev_status, DARK_ERR_TIMEOUT);
  return bad == 0;
}

// bf16 -> fp16 in place for `bytes` of a shared tile (feature GEMM operand).
// A bf16 value is out of fp16 range (|x| > 65504) exactly when its magnitude
// bits are 0x4780 (65536) or more; that is reported.
__device__ __forceinline__ void to_fp16_inplace(uint32_t saddr, int bytes, int* dev_status) {
  uint32_t mag = 0;
#pragma unroll 4
  for (int i = threadIdx.x; i < bytes / 16; i += kFwdThreads) {
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

// Stabiliser: the maximum of a row of `ncols_half` * 2 TMEM columns whose two
// halves are read by the threads of warps w and w + 4 (half = 0, 1) at
// lane_taddr + half * ncols_half; the halves meet in red[2][128]. Called by
// every thread of the CTA (it holds a block-wide barrier).
__device__ __forceinline__ float row_max_pair(uint32_t lane_taddr, int half, int ncols_half,
                                              float* red, int row) {
  float mx = -INFINITY;
  for (int c0 = half * ncols_half; c0 < (half + 1) * ncols_half; c0 += 32) {
    float v[32];
    tmem_ld32(lane_taddr + c0, v);
#pragma unroll
    for (int e = 0; e < 32; ++e) mx = fmaxf(mx, v[e]);
  }
  red[half * 128 + row] = mx;
  __syncthreads();
  mx = fmaxf(red[row], red[128 + row]);
  __syncthreads();               // red may be reused
  return mx;
}

// exp2 of 32 values (minus `offset`) packed to bf16 pairs (zeros for a masked key).
__device__ __forceinline__ void exp2_pack32(const uint32_t (&r)[32], float offset, bool zero,
                                            uint32_t (&w)[16]) {
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    const float x0 = __uint_as_float(r[2 * e]) - offset;
    const float x1 = __uint_as_float(r[2 * e + 1]) - offset;
    w[e] = zero ? 0u : pack_bf16(ex2(x0), ex2(x1));
  }
}
// 32 packed bf16 pairs as four 16-byte chunks of a K-major 128B-swizzled row.
__device__ __forceinline__ void store_row32(const uint32_t (&w)[16], uint32_t tile, int row, int f0) {
#pragma unroll
  for (int g = 0; g < 4; ++g)
    st_shared_v4(tile + kmajor_off(row, f0 + 8 * g, 16384), w[4 * g], w[4 * g + 1], w[4 * g + 2],
                 w[4 * g + 3]);
}
}  // namespace tc
}  // namespace dark
