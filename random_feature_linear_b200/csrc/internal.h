// Internal launch interface between the C-ABI layer (api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <cuda.h>

#include "../../include/dark.h"

namespace dark {

// Everything one forward call needs, validated by the C-ABI layer.
struct FwdArgs {
  int heads_w, m, r, d;
  dark_dtype dtype;
  const void* w;                  // projection buffer [heads_w][m + r][d]
  const void *q, *k, *v;
  void* out;
  int64_t qs[3], ks[3], os[3];    // element strides {b, h, l} of q, of k/v, of out
  int B, H, L;                    // L: queries (and keys, for self-attention)
  int Lk;                         // keys/values: L, or the context length
  const uint8_t* mask;            // keys [B][Lk] or null
  const uint8_t* qmask;           // queries [B][L] or null (cross-attention)
  int flags;
  float *st_kv, *st_z, *st_shift; // state_out arrays or null
  void* ws;
  size_t ws_bytes;
  int* dev_status;
  cudaStream_t stream;
  // TMA descriptors of W', q, k, v, encoded once per call by tc_make_maps
  CUtensorMap tm_w, tm_q, tm_k, tm_v;
  CUtensorMap tm_o;               // out, 64 x 128 boxes (tensor stores of the d = 64 paths)
  bool maps_ready;
  int path;                       // kernel path chosen by fwd_prepare
};

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Every workspace starts with this many bytes of synchronisation words (zero
// at first use, restored to zero by the kernels that use them); kernel data
// of every path starts after it.
constexpr size_t kWsHeader = 256;

// The forward call in three steps: validate and choose the kernel path (no
// device work), report the workspace that path needs, enqueue it.
// Lq queries (strides q_strides, optional query mask) over Lk keys/values
// (strides kv_strides, optional key mask); self-attention passes Lq = Lk and the
// same strides for both.
dark_status fwd_prepare_general(const dark_projection* proj, const void* q,
                                const int64_t* q_strides, int Lq, const uint8_t* query_mask,
                                const void* k, const void* v, const int64_t* kv_strides, int Lk,
                                const uint8_t* key_mask, void* out, const int64_t* out_strides,
                                int B, int H, int flags, const dark_state* state_out,
                                int* dev_status, void* stream, FwdArgs* a);
dark_status fwd_prepare(const dark_projection* proj, const void* q, const void* k, const void* v,
                        void* out, const int64_t* qkv_strides, const int64_t* out_strides, int B,
                        int H, int L, const uint8_t* key_mask, int flags,
                        const dark_state* state_out, int* dev_status, void* stream, FwdArgs* a);
size_t fwd_workspace_need(const FwdArgs& a);
dark_status fwd_launch(FwdArgs& a, void* ws, size_t ws_bytes, dark_state* state_out,
                       uint64_t generation);

// Projection W' = [c_w Omega M ; c_m M] (one-off, fp64 accumulation).
cudaError_t launch_projection(const float* omega, int heads_omega, const float* geom,
                              int heads_geom, int heads_w, int m, int r, int d,
                              dark_dtype dtype, void* w, cudaStream_t stream);

// Generic SIMT forward: any strides, any supported sizes, fp32 or bf16 I/O.
size_t simt_workspace_bytes(int B, int H, int Lq, int Lk, int m, int d, int flags);
cudaError_t simt_forward(const FwdArgs& a);

// Tensor-core forward paths (tcgen05/TMEM/TMA). `*_supported` says whether the
// sizes, layout and alignment fit; the launchers assume they do.
// Alignment/stride/shape checks shared by the tensor-core paths, then the
// TMA descriptors (false if any check fails or the driver rejects a layout).
bool tc_make_maps(FwdArgs& a);
// Cycles of the testing stall every tensor-core forward kernel takes first
// (0: none); set through dark_set_test_stall_cycles.
long long test_stall_cycles();
// Streaming multiprocessors of the current device (looked up once per device).
int num_sms();
// Raises a kernel's dynamic shared memory limit to `bytes` on the current device
// when it is below (done_per_device keeps the size set so far per device).
cudaError_t set_smem_limit_once(const void* kernel, int bytes, int* done_per_device);

bool tc_causal_supported(FwdArgs& a);
size_t tc_causal_workspace_bytes(int B, int H, int L, int m, int d);
cudaError_t tc_causal_forward(const FwdArgs& a);

bool tc_noncausal_supported(FwdArgs& a);
// Per-range key states Phi(K)^T [V | 1] as fp32 [B*H*nsplit][65][m] (tcgen05).
// shifts: null, or (stabiliser) [B*H*nsplit] receiving each range's largest
// valid key exponent (-inf without one), which its state is scaled by 2^-shift.
cudaError_t tc_launch_key_states(const FwdArgs& a, const CUtensorMap& tw, const CUtensorMap& tk,
                                 const CUtensorMap& tv, int ntiles, int nsplit, float* partials,
                                 float* shifts);
size_t tc_noncausal_workspace_bytes(int B, int H, int Lq, int Lk, int m, int d);
cudaError_t tc_noncausal_forward(const FwdArgs& a);

// Wide heads (d = 128..256, m up to 512), causal: features/scores launch, then
// a value-block launch carrying the state in TMEM (tcgen05).
bool tc_wide_supported(FwdArgs& a);
size_t tc_wide_workspace_bytes(int B, int H, int L, int m, int d, int r);
cudaError_t tc_wide_forward(const FwdArgs& a);

// Exact learned-kernel attention (softmax over u = M q~, w = M k~), SIMT fp32.
size_t exact_workspace_bytes(int B, int H, int Lq, int Lk, int r);
cudaError_t exact_forward(const FwdArgs& a);
// ... and on tcgen05 for bf16, d = 64, r in {16, 32, 48, 64} (no workspace).
bool tc_exact_supported(FwdArgs& a);
cudaError_t tc_exact_forward(const FwdArgs& a);
// Workspace of the tensor-core exact path (d = 64 or 128): the key-range
// splits' partial results when the query tiles alone are too few for the GPU.
size_t tc_exact_workspace_bytes(int B, int H, int Lq, int Lk, int d, int causal);

// Decode step over [B][H] heads.
struct DecodeArgs {
  int heads_w, m, r, d;
  dark_dtype dtype;
  const void* w;
  float *kv, *z, *shift;
  int B, H;
  const void *q, *k, *v;
  void* out;
  const uint8_t* valid;
  int update;                     // 1: add (k, v) to the state first; 0: read it only
  int* dev_status;
  cudaStream_t stream;
};
cudaError_t launch_decode(const DecodeArgs& a);

// Backward pass of self-attention (SIMT, fp32 arithmetic).
struct BwdArgs {
  const float *omega, *geom;      // [heads_omega][m][r], [heads_geom][r][d]
  int heads_omega, heads_geom, heads_w, m, r, d;
  dark_dtype dtype;
  const void *q, *k, *v, *dout;
  void *dq, *dk, *dv;
  int64_t xs[3], gs[3], ds[3];    // element strides {b, h, l}: q/k/v, dout, dq/dk/dv
  float* dgeom;                   // [heads_geom][r][d] or null
  int B, H, L;
  const uint8_t* mask;
  int flags;
  void* ws;
  int* dev_status;
  cudaStream_t stream;
};
size_t bwd_workspace_bytes(int B, int H, int L, int m, int r, int d, int heads_w);
cudaError_t launch_backward(const BwdArgs& a);
// bf16 I/O on the tensor cores (kind::tf32): d a multiple of 32 up to 128, m a
// multiple of 64 up to 256, r a multiple of 32 up to 128.
bool tc_backward_supported(const BwdArgs& a);
size_t tc_bwd_workspace_bytes(int B, int H, int L, int m, int r, int d, int heads_w);
cudaError_t launch_backward_tc(const BwdArgs& a);
cudaError_t bwd_fill_ordered(int* p, int n, float v, cudaStream_t s);
cudaError_t bwd_shift_keys(float* phik, const int* ck, int L, int m, size_t n, cudaStream_t s);
cudaError_t bwd_tile_scan(float* st, int n, int nt, int bh, int mode, cudaStream_t s);
cudaError_t bwd_dgeom(const float* G, const BwdArgs& a);

// Projection sampler (Philox4x64-10 + Box-Muller; orthogonal blocks by fp64
// Gram-Schmidt).
size_t omega_workspace_bytes(int heads, int m, int r, int orthogonal);
cudaError_t launch_sample_omega(uint64_t seed, uint64_t draw, int heads, int m, int r,
                                int orthogonal, float* omega, void* ws, cudaStream_t stream);

}  // namespace dark
