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
#include "tc_roles.cuh"

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

// Shared-memory byte offsets of 16-byte piece c (values 4c..4c+3) of K-major
// row `row`, and of MN-major K row k.
__device__ __forceinline__ uint32_t km_off(int row, int c) {
  return (uint32_t)((row >> 3) * 1024 + (row & 7) * 128 + (((c ^ row) & 7) << 4));
}
__device__ __forceinline__ uint32_t mn_off(int k, int c) {
  return (uint32_t)((c >> 3) * kMnBlockBytes + (k >> 2) * 512 + (k & 3) * 128 +
                    ((((c >> 1) ^ k) & 3) << 5) + ((c & 1) << 4));
}

// Register staging for values that need converting: fn(row, c) (K-major) or
// fn(k, c) (MN-major) returns the four values; each thread issues up to four
// loads before it stores any of them. Element i of the rows x per_row pieces
// is (i / per_row, i % per_row); a thread steps its pair instead of dividing.
template <bool MN, class F>
__device__ __forceinline__ void stage_regs(uint8_t* base, int rows, int per_row, F fn, int nt) {
  constexpr int U = 4;
  const int total = rows * per_row;
  const int da = nt / per_row, dc = nt - da * per_row;
  int a = threadIdx.x / per_row, c = threadIdx.x - a * per_row;
  for (int i0 = threadIdx.x; i0 < total; i0 += U * nt) {
    float4 v[U];
    uint32_t off[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const bool ok = i0 + u * nt < total;
      v[u] = ok ? fn(a, c) : make_float4(0.f, 0.f, 0.f, 0.f);
      off[u] = MN ? mn_off(a, c) : km_off(a, c);
      a += da;
      c += dc;
      if (c >= per_row) {
        c -= per_row;
        ++a;
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u)
      if (i0 + u * nt < total) *reinterpret_cast<float4*>(base + off[u]) = v[u];
  }
}
// The staging helpers are called by threads 0 .. nt - 1 of the CTA.
// K-major chunk of R rows: fn(row, c) returns values 4c..4c+3 of the row's 32.
template <class F>
__device__ __forceinline__ void stage_km(uint8_t* base, int R, F fn, int nt) {
  stage_regs<false>(base, R, 8, fn, nt);
}
// MN-major chunk of MN extent R (a multiple of 32): fn(k, c) returns MN values
// 4c..4c+3 at K row k (0..31).
template <class F>
__device__ __forceinline__ void stage_mn(uint8_t* base, int R, F fn, int nt) {
  stage_regs<true>(base, 32, R >> 2, fn, nt);
}

// Asynchronous 16-byte copies global -> shared (zero-filled when `valid` is
// false: no byte of `src` is read then, and `src` is any mapped address).
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
// Copy staging of fp32 values already in place: src(row, c) / src(k, c) gives
// the 16-byte aligned source of the four values, or nullptr for zeros
// (`any` then stands in as the unread source address).
template <bool MN, class F>
__device__ __forceinline__ void stage_async(uint8_t* base, int rows, int per_row, F src,
                                            const float* any, int nt) {
  const uint32_t b = smem_u32(base);
  const int total = rows * per_row;
  const int da = nt / per_row, dc = nt - da * per_row;
  int a = threadIdx.x / per_row, c = threadIdx.x - a * per_row;
#pragma unroll 4
  for (int i = threadIdx.x; i < total; i += nt) {
    const float* p = src(a, c);
    cp_async16(b + (MN ? mn_off(a, c) : km_off(a, c)), p != nullptr ? p : any, p != nullptr);
    a += da;
    c += dc;
    if (c >= per_row) {
      c -= per_row;
      ++a;
    }
  }
}
template <class F>
__device__ __forceinline__ void stage_km_async(uint8_t* base, int R, F src, const float* any,
                                               int nt) {
  stage_async<false>(base, R, 8, src, any, nt);
}
template <class F>
__device__ __forceinline__ void stage_mn_async(uint8_t* base, int R, F src, const float* any,
                                               int nt) {
  stage_async<true>(base, 32, R >> 2, src, any, nt);
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
