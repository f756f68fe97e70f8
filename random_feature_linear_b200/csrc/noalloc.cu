// dark_attention_fwd_noalloc: the forward pass for callers that cannot
// allocate device memory. Some hosts run this library where cudaMalloc is not
// available to them: under an allocator that forbids extra allocations, or in a
// runtime that hands the library only the tensors of the call. They still own their inputs and
// outputs; the scratch that dark_attention_fwd takes as a caller workspace
// comes here from one fixed array compiled into the library.
#include <mutex>

#include "internal.h"

namespace {

// Scratch for every call of this entry point, on every GPU that loads the
// library, for the life of the process.
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices];

// Device address of the array on the current device; looked up once per device
// and kept for the life of the process (the header tells callers not to use
// this entry point after a device reset, which would invalidate it).
// In host code `g_noalloc_scratch` only names a host-side shadow, so its address
// must come from cudaGetSymbolAddress with the device current.
cudaError_t scratch_for_current_device(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" size_t dark_noalloc_scratch_bytes(void) { return kNoAllocScratchBytes; }

extern "C" dark_status dark_attention_fwd_noalloc(const dark_projection* proj, const void* q,
                                                  const void* k, const void* v, void* out,
                                                  const int64_t* qkv_strides,
                                                  const int64_t* out_strides, int B, int H, int L,
                                                  const uint8_t* key_mask, int flags,
                                                  dark_state* state_out, int* dev_status,
                                                  void* stream) {
  dark::FwdArgs a;
  dark_status st = dark::fwd_prepare(proj, q, k, v, out, qkv_strides, out_strides, B, H, L,
                                     key_mask, flags, state_out, dev_status, stream, &a);
  if (st != DARK_OK) return st;
  if (dark::fwd_workspace_need(a) > kNoAllocScratchBytes) return DARK_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  if (scratch_for_current_device(&scratch) != cudaSuccess) return DARK_ERR_CUDA;
  // the synchronisation header of the workspace layout must read zero
  if (cudaMemsetAsync(scratch, 0, dark::kWsHeader, (cudaStream_t)stream) != cudaSuccess)
    return DARK_ERR_CUDA;
  return dark::fwd_launch(a, scratch, kNoAllocScratchBytes, state_out, proj->generation);
}
