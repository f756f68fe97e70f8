// fp32 operand tiles for tcgen05 MMAs of kind::tf32, staged into shared memory
// by the threads of the CTA (the backward pass reads fp32 feature maps,
// statistics and coefficients that it wrote itself, in whatever orientation the
// next contraction needs, so no tensor maps are involved).
//
// Layouts (128-byte swizzle, 1024-byte aligned atoms of 8 rows x 128 bytes in
// which the 16-byte chunk c of row r sits at chunk c ^ (r mod 8)):
//  * K-major chunk: R rows (M or N index) x 32 K values; row i is 128 bytes at
//    (i / 8) * 1024 + (i % 8) * 128. One MMA consumes K = 8 (32 bytes): K-step
//    j of the chunk starts 32 * j bytes in, 8-row groups are 1024 bytes apart.
//  * MN-major chunk (the 128-byte swizzle on a 32-byte base, the one layout the
//    tensor cores take for MN-major 32-bit operands): 32 K rows x R values of
//    M or N (R a multiple of 32). The 32-value MN block b holds the chunk's 32
//    K rows of 128 bytes at b * 4096; K row k sits at (k / 4) * 512 +
//    (k % 4) * 128 inside it, and its 32-byte piece p at piece p ^ (k % 4).
//    K-step j covers K rows 8j..8j+7 (two 512-byte groups), 1024 bytes in.
#pragma once

#include "tc_common.cuh"

namespace dark {
namespace tc {

// Instruction descriptor of kind::tf32 (tf32 operands, fp32 accumulation).
__host__ __device__ constexpr uint32_t idesc_tf32(int M, int N, bool a_mn, bool b_mn) {
  return (1u << 4) | (2u << 7) | (2u << 10) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// D (TMEM) = A * B (+ D if accumulate), tf32 operands in shared memory.
__device__ __forceinline__ void mma_tf32(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                         uint32_t id, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(id), "r"(accumulate)
      : "memory");
}

constexpr uint32_t kKmRowBytes = 128;      // one K-major row of a chunk
constexpr uint32_t kMnBlockBytes = 4096;   // one 32-wide MN block of an MN-major chunk

// Bytes of a K-major chunk of R rows / an MN-major chunk of R values.
__host__ __device__ constexpr uint32_t km_bytes(int R) { return (uint32_t)R * 128u; }
__host__ __device__ constexpr uint32_t mn_bytes(int R) { return (uint32_t)(R / 32) * 4096u; }

// Descriptors of K-step j (0..3) of a chunk at shared address `base`.
__device__ __forceinline__ uint64_t km_desc(uint32_t base, int j) {
  return sdesc(base + 32u * j, 16, 1024);
}
constexpr uint32_t kSwizzle128Base32 = 1;
__device__ __forceinline__ uint64_t mn_desc(uint32_t base, int j) {
  return sdesc(base + 1024u * j, kMnBlockBytes, 512, kSwizzle128Base32);
}

// Stages a K-major chunk: fn(row, c) returns values 4c..4c+3 of the row's 32.
template <class F>
__device__ __forceinline__ void stage_km(uint8_t* base, int R, F fn) {
  for (int i = threadIdx.x; i < R * 8; i += blockDim.x) {
    const int row = i >> 3, c = i & 7;
    const float4 v = fn(row, c);
    *reinterpret_cast<float4*>(base + (row >> 3) * 1024 + (row & 7) * 128 +
                               (((c ^ row) & 7) << 4)) = v;
  }
}

// Stages an MN-major chunk: fn(k, c) returns MN values 4c..4c+3 at K row k
// (0..31); R is the MN extent (a multiple of 32).
template <class F>
__device__ __forceinline__ void stage_mn(uint8_t* base, int R, F fn) {
  const int per_k = R >> 2;
  for (int i = threadIdx.x; i < 32 * per_k; i += blockDim.x) {
    const int k = i / per_k, c = i - k * per_k;
    const float4 v = fn(k, c);
    *reinterpret_cast<float4*>(base + (c >> 3) * kMnBlockBytes + (k >> 2) * 512 + (k & 3) * 128 +
                               ((((c >> 1) ^ k) & 3) << 5) + ((c & 1) << 4)) = v;
  }
}

// Issues the four K-steps of one 32-deep chunk: D (+)= A * B with A an M = 128
// operand and B an N-wide operand, each K-major or MN-major.
__device__ __forceinline__ void mma_chunk(uint32_t tmem_d, uint32_t a_base, bool a_mn,
                                          uint32_t b_base, bool b_mn, int N, bool accumulate) {
  const uint32_t id = idesc_tf32(128, N, a_mn, b_mn);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint64_t ad = a_mn ? mn_desc(a_base, j) : km_desc(a_base, j);
    const uint64_t bd = b_mn ? mn_desc(b_base, j) : km_desc(b_base, j);
    mma_tf32(tmem_d, ad, bd, id, (accumulate || j > 0) ? 1u : 0u);
  }
}

}  // namespace tc
}  // namespace dark
