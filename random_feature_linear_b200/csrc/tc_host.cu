// Host helper of the tensor-core kernels: tiled TMA descriptors.
#include <cudaTypedefs.h>

#include "internal.h"
#include "tc_common.cuh"

namespace dark {

namespace {
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = []() -> PFN_cuTensorMapEncodeTiled_v12000 {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return (PFN_cuTensorMapEncodeTiled_v12000)p;
  }();
  return fn;
}
}  // namespace

bool encode_tmap(CUtensorMap* map, CUtensorMapDataType type, int rank, const void* base,
                 const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box) {
  PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint32_t elem_strides[5] = {1, 1, 1, 1, 1};
  const CUresult r =
      fn(map, type, (cuuint32_t)rank, const_cast<void*>(base), (const cuuint64_t*)dims,
         (const cuuint64_t*)strides_bytes, (const cuuint32_t*)box, elem_strides,
         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool tc_make_maps(FwdArgs& a) {
  if (a.maps_ready) return true;
  auto al16 = [](const void* p) { return ((uintptr_t)p & 15) == 0; };
  // 64-column boxes: d = 64 is one box per row, d = 128 two
  if (a.dtype != DARK_BF16 || !(a.d == 64 || a.d == 128)) return false;
  if (!al16(a.q) || !al16(a.k) || !al16(a.v) || !al16(a.out) || !al16(a.w)) return false;
  for (int i = 0; i < 3; ++i)
    if (a.qs[i] % 8 != 0 || a.ks[i] % 8 != 0 || a.os[i] % 8 != 0) return false;
  const uint64_t wd[2] = {(uint64_t)a.d, (uint64_t)a.heads_w * (a.m + a.r)};
  const uint64_t wsd[1] = {(uint64_t)a.d * 2};
  const uint32_t wb[2] = {64, 16};
  // queries: L tokens with strides qs; keys and values: Lk tokens with strides ks
  const uint64_t qd[4] = {(uint64_t)a.d, (uint64_t)a.L, (uint64_t)a.H, (uint64_t)a.B};
  const uint64_t qst[3] = {(uint64_t)a.qs[2] * 2, (uint64_t)a.qs[1] * 2, (uint64_t)a.qs[0] * 2};
  const uint64_t kd[4] = {(uint64_t)a.d, (uint64_t)a.Lk, (uint64_t)a.H, (uint64_t)a.B};
  const uint64_t kst[3] = {(uint64_t)a.ks[2] * 2, (uint64_t)a.ks[1] * 2, (uint64_t)a.ks[0] * 2};
  const uint32_t xb[4] = {64, 128, 1, 1};
  a.maps_ready = encode_tmap(&a.tm_w, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, a.w, wd, wsd, wb) &&
                 encode_tmap(&a.tm_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, a.q, qd, qst, xb) &&
                 encode_tmap(&a.tm_k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, a.k, kd, kst, xb) &&
                 encode_tmap(&a.tm_v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, a.v, kd, kst, xb);
  // out: L query rows with strides os
  const uint64_t ost[3] = {(uint64_t)a.os[2] * 2, (uint64_t)a.os[1] * 2, (uint64_t)a.os[0] * 2};
  a.maps_ready = a.maps_ready &&
                 encode_tmap(&a.tm_o, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, a.out, qd, ost, xb);
  return a.maps_ready;
}

int num_sms() {
  static int count[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (count[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    count[dev] = n;
  }
  return count[dev];
}

cudaError_t set_smem_limit_once(const void* kernel, int bytes, int* done_per_device) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  // done_per_device[dev] holds the largest size set so far on that device
  if (dev >= 0 && dev < 64 && done_per_device[dev] >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && dev >= 0 && dev < 64) done_per_device[dev] = bytes;
  return e;
}

}  // namespace dark
