// Synchronisation helpers of the warp-specialised tensor-core kernels: one
// producer thread (TMA), one MMA-issuing thread and 256 epilogue threads
// (warps 0-7) hand shared-memory and TMEM buffers to one another through
// mbarriers. Every wait is bounded: a wait that runs out records
// DARK_ERR_TIMEOUT and raises the CTA's abort flag, and a raised flag ends every
// other wait of the CTA, so that all roles leave their loops.
#pragma once

#include "common.cuh"
#include "tc_common.cuh"

namespace dark {
namespace tc {

// One arrival of this thread on a shared-memory mbarrier.
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Named barrier 1 over the 256 epilogue threads; true if any of them passes `bad`.
__device__ __forceinline__ bool epi_sync_or(bool bad) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "barrier.cta.red.or.pred q, 1, 256, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)bad)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void epi_sync() { asm volatile("barrier.cta.sync 1, 256;" ::: "memory"); }

// Bounded wait of one thread (see above).
__device__ __forceinline__ bool wait_one(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                         int* dev_status, long long limit = kWaitCycles) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (*abort_flag) return false;
    if (clock64() - t0 > limit) {
      *abort_flag = 1;
      report(dev_status, DARK_ERR_TIMEOUT);
      return false;
    }
  }
  return true;
}
// The same for the epilogue threads: all 256 wait, then agree.
__device__ __forceinline__ bool epi_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                         int* dev_status, long long limit = kWaitCycles) {
  const bool ok = wait_one(bar, parity, abort_flag, dev_status, limit);
  return !epi_sync_or(!ok);
}
// Epilogue warp -> producer / MMA thread: one arrival per warp (barrier count 8).
__device__ __forceinline__ void warp_arrive(uint64_t* bar) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}

// Tensor store of one 128-row tile from shared memory (128B-swizzled, as the
// map says) to global memory; rows past the tensor's end are not written.
__device__ __forceinline__ void tma_store_4d(const CUtensorMap* map, uint32_t ssrc, int x, int y,
                                             int z, int w) {
  asm volatile(
      "cp.async.bulk.tensor.4d.global.shared::cta.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(
          (uint64_t)map),
      "r"(ssrc), "r"(x), "r"(y), "r"(z), "r"(w)
      : "memory");
}
__device__ __forceinline__ void bulk_commit_group() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_group_read() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_group() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

}  // namespace tc
}  // namespace dark
