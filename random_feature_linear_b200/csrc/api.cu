// C ABI of the library (declared in include/dark.h): argument validation on the
// host, choice between the tensor-core kernels and the generic SIMT kernels,
// and launches on the caller's stream. Nothing here allocates device memory.
#include <atomic>
#include <string.h>

#include "common.cuh"
#include "internal.h"

namespace {

std::atomic<uint64_t> g_generation{0};

constexpr int kMaxD = 256, kMaxR = 256, kMaxM = 1024;

bool sizes_ok(int m, int r, int d) {
  return m >= 1 && m <= kMaxM && r >= 1 && r <= kMaxR && d >= 4 && d <= kMaxD && d % 4 == 0;
}

bool dtype_ok(dark_dtype t) { return t == DARK_F32 || t == DARK_BF16; }

size_t elt(dark_dtype t) { return t == DARK_BF16 ? 2 : 4; }

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

dark_status from_cuda(cudaError_t e) { return e == cudaSuccess ? DARK_OK : DARK_ERR_CUDA; }

bool proj_ok(const dark_projection* p) {
  return p != nullptr && p->w != nullptr && aligned(p->w, 16) && dtype_ok(p->dtype) &&
         sizes_ok(p->m, p->r, p->d) && p->heads >= 1;
}

enum class Path { Simt, TcCausal, TcNonCausal, TcWide, Exact, TcExact };

Path choose_path(dark::FwdArgs& a) {
  if (a.flags & DARK_EXACT) return dark::tc_exact_supported(a) ? Path::TcExact : Path::Exact;
  if (a.flags & DARK_CAUSAL) {
    if (dark::tc_causal_supported(a)) return Path::TcCausal;
    if (dark::tc_wide_supported(a)) return Path::TcWide;
  } else {
    if (dark::tc_noncausal_supported(a)) return Path::TcNonCausal;
  }
  return Path::Simt;
}

size_t ws_need(Path p, int B, int H, int Lq, int Lk, int m, int r, int d, int flags) {
  switch (p) {
    case Path::TcCausal: return dark::tc_causal_workspace_bytes(B, H, Lq, m, d);
    case Path::TcWide: return dark::tc_wide_workspace_bytes(B, H, Lq, m, d, r);
    case Path::TcNonCausal: return dark::tc_noncausal_workspace_bytes(B, H, Lq, Lk, m, d);
    case Path::Exact: return dark::exact_workspace_bytes(B, H, Lq, Lk, r);
    // the key-range splits run only when the caller's workspace holds them
    // (the public workspace queries include them)
    case Path::TcExact: return dark::kWsHeader;
    default: return dark::simt_workspace_bytes(B, H, Lq, Lk, m, d, flags);
  }
}

}  // namespace

namespace dark {

dark_status fwd_prepare_general(const dark_projection* proj, const void* q,
                                const int64_t* q_strides, int Lq, const uint8_t* query_mask,
                                const void* k, const void* v, const int64_t* kv_strides, int Lk,
                                const uint8_t* key_mask, void* out, const int64_t* out_strides,
                                int B, int H, int flags, const dark_state* state_out,
                                int* dev_status, void* stream, FwdArgs* out_args) {
  if (proj == nullptr || proj->w == nullptr || !aligned(proj->w, 16) || !dtype_ok(proj->dtype))
    return DARK_ERR_INVALID_ARG;
  if (proj->m < 1 || proj->r < 1 || proj->d < 1) return DARK_ERR_INVALID_ARG;
  if (!sizes_ok(proj->m, proj->r, proj->d)) return DARK_ERR_UNSUPPORTED;
  if (q == nullptr || k == nullptr || v == nullptr || out == nullptr) return DARK_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || Lq < 1 || Lk < 1) return DARK_ERR_INVALID_ARG;
  if ((flags & DARK_CAUSAL) && Lq != Lk) return DARK_ERR_INVALID_ARG;
  if (!(proj->heads == 1 || proj->heads == H)) return DARK_ERR_INVALID_ARG;
  if (flags & ~(DARK_CAUSAL | DARK_STABILISE | DARK_EXACT)) return DARK_ERR_INVALID_ARG;
  // the exact mode keeps no recurrent statistics
  if ((flags & DARK_EXACT) && state_out != nullptr) return DARK_ERR_INVALID_ARG;
  FwdArgs& a = *out_args;
  memset(&a, 0, sizeof(a));
  a.heads_w = proj->heads;
  a.m = proj->m;
  a.r = proj->r;
  a.d = proj->d;
  a.dtype = proj->dtype;
  a.w = proj->w;
  a.q = q;
  a.k = k;
  a.v = v;
  a.out = out;
  const int64_t d = proj->d;
  const int64_t cq[3] = {(int64_t)H * Lq * d, (int64_t)Lq * d, d};
  const int64_t ck[3] = {(int64_t)H * Lk * d, (int64_t)Lk * d, d};
  for (int i = 0; i < 3; ++i) {
    a.qs[i] = q_strides ? q_strides[i] : cq[i];
    a.ks[i] = kv_strides ? kv_strides[i] : ck[i];
    a.os[i] = out_strides ? out_strides[i] : cq[i];
    if (a.qs[i] < 0 || a.ks[i] < 0 || a.os[i] < 0) return DARK_ERR_INVALID_ARG;
  }
  a.B = B;
  a.H = H;
  a.L = Lq;
  a.Lk = Lk;
  a.mask = key_mask;
  a.qmask = query_mask;
  a.flags = flags;
  if (state_out != nullptr) {
    if (state_out->kv == nullptr || state_out->z == nullptr || state_out->B != B ||
        state_out->H != H || state_out->m != proj->m || state_out->d != proj->d)
      return DARK_ERR_INVALID_ARG;
    if ((flags & DARK_STABILISE) && state_out->shift == nullptr) return DARK_ERR_INVALID_ARG;
    a.st_kv = state_out->kv;
    a.st_z = state_out->z;
    a.st_shift = (flags & DARK_STABILISE) ? state_out->shift : nullptr;
  }
  a.dev_status = dev_status;
  a.stream = (cudaStream_t)stream;
  a.path = (int)choose_path(a);   // may encode the TMA descriptors into `a`
  return DARK_OK;
}

dark_status fwd_prepare(const dark_projection* proj, const void* q, const void* k, const void* v,
                        void* out, const int64_t* qkv_strides, const int64_t* out_strides, int B,
                        int H, int L, const uint8_t* key_mask, int flags,
                        const dark_state* state_out, int* dev_status, void* stream,
                        FwdArgs* out_args) {
  return fwd_prepare_general(proj, q, qkv_strides, L, nullptr, k, v, qkv_strides, L, key_mask,
                             out, out_strides, B, H, flags, state_out, dev_status, stream,
                             out_args);
}

size_t fwd_workspace_need(const FwdArgs& a) {
  return ws_need((Path)a.path, a.B, a.H, a.L, a.Lk, a.m, a.r, a.d, a.flags);
}

dark_status fwd_launch(FwdArgs& a, void* ws, size_t ws_bytes, dark_state* state_out,
                       uint64_t generation) {
  a.ws = ws;
  a.ws_bytes = ws_bytes;
  cudaError_t e;
  switch ((Path)a.path) {
    case Path::TcCausal: e = tc_causal_forward(a); break;
    case Path::TcNonCausal: e = tc_noncausal_forward(a); break;
    case Path::TcWide: e = tc_wide_forward(a); break;
    case Path::Exact: e = exact_forward(a); break;
    case Path::TcExact: e = tc_exact_forward(a); break;
    default: e = simt_forward(a); break;
  }
  if (e != cudaSuccess) return DARK_ERR_CUDA;
  if (state_out != nullptr) state_out->generation = generation;
  return DARK_OK;
}

}  // namespace dark

namespace dark {
namespace {
std::atomic<long long> g_test_stall{0};
}
long long test_stall_cycles() { return g_test_stall.load(std::memory_order_relaxed); }
}  // namespace dark

extern "C" {

int dark_abi_version(void) { return DARK_ABI_VERSION; }

void dark_set_test_stall_cycles(long long cycles) {
  dark::g_test_stall.store(cycles > 0 ? cycles : 0, std::memory_order_relaxed);
}

const char* dark_status_string(dark_status s) {
  switch (s) {
    case DARK_OK: return "DARK_OK";
    case DARK_ERR_INVALID_ARG: return "DARK_ERR_INVALID_ARG: invalid size, pointer, alignment or layout";
    case DARK_ERR_UNSUPPORTED: return "DARK_ERR_UNSUPPORTED: sizes outside what this build implements";
    case DARK_ERR_STALE_STATE: return "DARK_ERR_STALE_STATE: decode state belongs to another projection";
    case DARK_ERR_CUDA: return "DARK_ERR_CUDA: a CUDA launch or runtime call failed";
    case DARK_ERR_NUMERIC: return "DARK_ERR_NUMERIC: non-finite output";
    case DARK_ERR_TIMEOUT: return "DARK_ERR_TIMEOUT: a bounded wait between blocks ran out";
  }
  return "unknown dark_status";
}

size_t dark_projection_bytes(int heads, int m, int r, int d, dark_dtype dtype) {
  if (heads < 1 || m < 1 || r < 1 || d < 1 || !dtype_ok(dtype)) return 0;
  return (size_t)heads * (size_t)(m + r) * (size_t)d * elt(dtype);
}

dark_status dark_make_projection(const float* omega, int heads_omega, const float* geom,
                                 int heads_geom, int H, int m, int r, int d, dark_dtype dtype,
                                 void* w_buf, size_t w_bytes, void* stream,
                                 dark_projection* out) {
  if (omega == nullptr || geom == nullptr || w_buf == nullptr || out == nullptr || H < 1 ||
      !dtype_ok(dtype))
    return DARK_ERR_INVALID_ARG;
  if (!(heads_omega == 1 || heads_omega == H) || !(heads_geom == 1 || heads_geom == H))
    return DARK_ERR_INVALID_ARG;
  if (m < 1 || r < 1 || d < 1) return DARK_ERR_INVALID_ARG;
  if (!sizes_ok(m, r, d)) return DARK_ERR_UNSUPPORTED;
  const int heads = heads_omega > heads_geom ? heads_omega : heads_geom;
  if (w_bytes < dark_projection_bytes(heads, m, r, d, dtype) || !aligned(w_buf, 16))
    return DARK_ERR_INVALID_ARG;
  cudaError_t e = dark::launch_projection(omega, heads_omega, geom, heads_geom, heads, m, r, d,
                                          dtype, w_buf, (cudaStream_t)stream);
  if (e != cudaSuccess) return DARK_ERR_CUDA;
  out->heads = heads;
  out->m = m;
  out->r = r;
  out->d = d;
  out->dtype = dtype;
  out->w = w_buf;
  out->generation = ++g_generation;
  return DARK_OK;
}

size_t dark_attention_workspace_bytes(const dark_projection* proj, int B, int H, int L,
                                      int flags) {
  if (!proj_ok(proj) || B < 1 || H < 1 || L < 1) return 0;
  if (flags & DARK_EXACT) {
    // either exact path may run (the tensor-core one for bf16 d = 64, 128)
    const size_t simt = dark::exact_workspace_bytes(B, H, L, L, proj->r);
    const size_t tc = (proj->d == 64 || proj->d == 128)
                          ? dark::tc_exact_workspace_bytes(B, H, L, L, proj->d,
                                                           (flags & DARK_CAUSAL) != 0)
                          : 0;
    return simt > tc ? simt : tc;
  }
  const int m = proj->m, d = proj->d;
  size_t need = dark::simt_workspace_bytes(B, H, L, L, m, d, flags);
  const size_t tc = (flags & DARK_CAUSAL) ? dark::tc_causal_workspace_bytes(B, H, L, m, d)
                                          : dark::tc_noncausal_workspace_bytes(B, H, L, L, m, d);
  const size_t wide =
      (flags & DARK_CAUSAL) ? dark::tc_wide_workspace_bytes(B, H, L, m, d, proj->r) : 0;
  if (need < tc) need = tc;
  return need > wide ? need : wide;
}

dark_status dark_attention_fwd(const dark_projection* proj, const void* q, const void* k,
                               const void* v, void* out, const int64_t* qkv_strides,
                               const int64_t* out_strides, int B, int H, int L,
                               const uint8_t* key_mask, int flags, dark_state* state_out,
                               void* ws, size_t ws_bytes, int* dev_status, void* stream) {
  if (ws == nullptr || !aligned(ws, 256)) return DARK_ERR_INVALID_ARG;
  dark::FwdArgs a;
  const dark_status st = dark::fwd_prepare(proj, q, k, v, out, qkv_strides, out_strides, B, H, L,
                                           key_mask, flags, state_out, dev_status, stream, &a);
  if (st != DARK_OK) return st;
  if (ws_bytes < dark::fwd_workspace_need(a)) return DARK_ERR_INVALID_ARG;
  return dark::fwd_launch(a, ws, ws_bytes, state_out, proj->generation);
}

size_t dark_cross_attention_workspace_bytes(const dark_projection* proj, int B, int H, int Lq,
                                            int Lk, int flags) {
  if (!proj_ok(proj) || B < 1 || H < 1 || Lq < 1 || Lk < 1 || (flags & DARK_CAUSAL)) return 0;
  if (flags & DARK_EXACT) {
    const size_t simt = dark::exact_workspace_bytes(B, H, Lq, Lk, proj->r);
    const size_t tc = (proj->d == 64 || proj->d == 128)
                          ? dark::tc_exact_workspace_bytes(B, H, Lq, Lk, proj->d, 0)
                          : 0;
    return simt > tc ? simt : tc;
  }
  const size_t simt = dark::simt_workspace_bytes(B, H, Lq, Lk, proj->m, proj->d, flags);
  const size_t tc = dark::tc_noncausal_workspace_bytes(B, H, Lq, Lk, proj->m, proj->d);
  return simt > tc ? simt : tc;
}

dark_status dark_cross_attention_fwd(const dark_projection* proj, const void* q,
                                     const int64_t* q_strides, int Lq, const uint8_t* query_mask,
                                     const void* k, const void* v, const int64_t* kv_strides,
                                     int Lk, const uint8_t* context_mask, void* out,
                                     const int64_t* out_strides, int B, int H, int flags,
                                     dark_state* context_out, void* ws, size_t ws_bytes,
                                     int* dev_status, void* stream) {
  if (ws == nullptr || !aligned(ws, 256)) return DARK_ERR_INVALID_ARG;
  if (flags & DARK_CAUSAL) return DARK_ERR_INVALID_ARG;
  dark::FwdArgs a;
  const dark_status st = dark::fwd_prepare_general(
      proj, q, q_strides, Lq, query_mask, k, v, kv_strides, Lk, context_mask, out, out_strides,
      B, H, flags, context_out, dev_status, stream, &a);
  if (st != DARK_OK) return st;
  if (ws_bytes < dark::fwd_workspace_need(a)) return DARK_ERR_INVALID_ARG;
  return dark::fwd_launch(a, ws, ws_bytes, context_out, proj->generation);
}

dark_status dark_cross_decode_step(const dark_projection* proj, const dark_state* context,
                                   const void* q_t, void* out_t, int* dev_status, void* stream) {
  if (proj == nullptr || proj->w == nullptr || !aligned(proj->w, 16) || !dtype_ok(proj->dtype) ||
      context == nullptr)
    return DARK_ERR_INVALID_ARG;
  if (!sizes_ok(proj->m, proj->r, proj->d)) return DARK_ERR_UNSUPPORTED;
  if (context->kv == nullptr || context->z == nullptr || q_t == nullptr || out_t == nullptr)
    return DARK_ERR_INVALID_ARG;
  if (context->B < 1 || context->H < 1 || context->m != proj->m || context->d != proj->d)
    return DARK_ERR_INVALID_ARG;
  if (!(proj->heads == 1 || proj->heads == context->H)) return DARK_ERR_INVALID_ARG;
  if (!aligned(context->kv, 16)) return DARK_ERR_INVALID_ARG;
  if (context->generation != proj->generation) return DARK_ERR_STALE_STATE;
  dark::DecodeArgs a;
  memset(&a, 0, sizeof(a));
  a.heads_w = proj->heads;
  a.m = proj->m;
  a.r = proj->r;
  a.d = proj->d;
  a.dtype = proj->dtype;
  a.w = proj->w;
  a.kv = context->kv;
  a.z = context->z;
  a.shift = context->shift;
  a.B = context->B;
  a.H = context->H;
  a.q = q_t;
  a.out = out_t;
  a.update = 0;
  a.dev_status = dev_status;
  a.stream = (cudaStream_t)stream;
  return from_cuda(dark::launch_decode(a));
}

size_t dark_attention_bwd_workspace_bytes(int heads_omega, int heads_geom, int m, int r, int d,
                                          int B, int H, int L) {
  if (heads_omega < 1 || heads_geom < 1 || B < 1 || H < 1 || L < 1 || !sizes_ok(m, r, d))
    return 0;
  const int heads_w = heads_omega > heads_geom ? heads_omega : heads_geom;
  return dark::bwd_workspace_bytes(B, H, L, m, r, d, heads_w);
}

dark_status dark_attention_bwd(const float* omega, int heads_omega, const float* geom,
                               int heads_geom, int m, int r, int d, dark_dtype dtype,
                               const void* q, const void* k, const void* v,
                               const int64_t* qkv_strides, const void* dout,
                               const int64_t* dout_strides, int B, int H, int L,
                               const uint8_t* key_mask, int flags, void* dq, void* dk, void* dv,
                               const int64_t* grad_strides, float* dgeom, void* ws,
                               size_t ws_bytes, int* dev_status, void* stream) {
  if (omega == nullptr || geom == nullptr || !dtype_ok(dtype)) return DARK_ERR_INVALID_ARG;
  if (q == nullptr || k == nullptr || v == nullptr || dout == nullptr || dq == nullptr ||
      dk == nullptr || dv == nullptr || ws == nullptr)
    return DARK_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || L < 1 || m < 1 || r < 1 || d < 1) return DARK_ERR_INVALID_ARG;
  if (!(heads_omega == 1 || heads_omega == H) || !(heads_geom == 1 || heads_geom == H))
    return DARK_ERR_INVALID_ARG;
  if (flags & ~(DARK_CAUSAL | DARK_STABILISE)) return DARK_ERR_INVALID_ARG;
  if (!sizes_ok(m, r, d)) return DARK_ERR_UNSUPPORTED;
  if ((int64_t)B * H > 65535) return DARK_ERR_UNSUPPORTED;   // grid y/z bound
  if (!aligned(ws, 256) || ws_bytes < dark_attention_bwd_workspace_bytes(
                                          heads_omega, heads_geom, m, r, d, B, H, L))
    return DARK_ERR_INVALID_ARG;
  dark::BwdArgs a;
  memset(&a, 0, sizeof(a));
  a.omega = omega;
  a.geom = geom;
  a.heads_omega = heads_omega;
  a.heads_geom = heads_geom;
  a.heads_w = heads_omega > heads_geom ? heads_omega : heads_geom;
  a.m = m;
  a.r = r;
  a.d = d;
  a.dtype = dtype;
  a.q = q;
  a.k = k;
  a.v = v;
  a.dout = dout;
  a.dq = dq;
  a.dk = dk;
  a.dv = dv;
  const int64_t c[3] = {(int64_t)H * L * d, (int64_t)L * d, (int64_t)d};
  for (int i = 0; i < 3; ++i) {
    a.xs[i] = qkv_strides ? qkv_strides[i] : c[i];
    a.gs[i] = dout_strides ? dout_strides[i] : c[i];
    a.ds[i] = grad_strides ? grad_strides[i] : c[i];
    if (a.xs[i] < 0 || a.gs[i] < 0 || a.ds[i] < 0) return DARK_ERR_INVALID_ARG;
  }
  a.dgeom = dgeom;
  a.B = B;
  a.H = H;
  a.L = L;
  a.mask = key_mask;
  a.flags = flags;
  a.ws = ws;
  a.dev_status = dev_status;
  a.stream = (cudaStream_t)stream;
  return from_cuda(dark::launch_backward(a));
}

int dark_auto_uses_exact(int L, int exact_threshold) {
  return exact_threshold > 0 && L <= exact_threshold ? 1 : 0;
}

size_t dark_sample_omega_workspace_bytes(int heads, int m, int r, int orthogonal) {
  if (heads < 1 || m < 1 || r < 1 || m > kMaxM || r > kMaxR) return 0;
  return dark::omega_workspace_bytes(heads, m, r, orthogonal);
}

dark_status dark_sample_omega(uint64_t seed, uint64_t draw, int heads, int m, int r,
                              int orthogonal, float* omega, void* ws, size_t ws_bytes,
                              void* stream) {
  if (omega == nullptr || !aligned(omega, 4) || heads < 1 || m < 1 || r < 1)
    return DARK_ERR_INVALID_ARG;
  if (m > kMaxM || r > kMaxR || heads > 65535) return DARK_ERR_UNSUPPORTED;
  if (orthogonal) {
    const size_t need = dark::omega_workspace_bytes(heads, m, r, 1);
    if (ws == nullptr || !aligned(ws, 256) || ws_bytes < need) return DARK_ERR_INVALID_ARG;
  }
  return from_cuda(dark::launch_sample_omega(seed, draw, heads, m, r, orthogonal ? 1 : 0, omega,
                                             ws, (cudaStream_t)stream));
}

dark_status dark_redraw_schedule_init(dark_redraw_schedule* s, uint64_t seed, int64_t interval,
                                      int deterministic) {
  if (s == nullptr) return DARK_ERR_INVALID_ARG;
  s->seed = seed;
  s->draw = 0;
  s->interval = interval > 0 ? interval : 0;
  s->count = 0;
  s->fixed = deterministic ? 1 : 0;
  return DARK_OK;
}

int dark_redraw_on_forward(dark_redraw_schedule* s, int training) {
  if (s == nullptr || !training) return 0;
  int redrew = 0;
  if (s->interval > 0 && s->count >= s->interval) {
    s->count = 0;                 // a redraw falling due while fixed is dropped
    if (!s->fixed) {
      ++s->draw;
      redrew = 1;
    }
  }
  ++s->count;
  return redrew;
}

int dark_redraw_request(dark_redraw_schedule* s, int force) {
  if (s == nullptr || (s->fixed && !force)) return 0;
  ++s->draw;
  s->count = 0;
  return 1;
}

void dark_redraw_set_fixed(dark_redraw_schedule* s, int fixed) {
  if (s != nullptr) s->fixed = fixed ? 1 : 0;
}

dark_status dark_state_init(const dark_projection* proj, dark_state* st, void* stream) {
  if (proj == nullptr || st == nullptr || st->kv == nullptr || st->z == nullptr)
    return DARK_ERR_INVALID_ARG;
  if (st->B < 1 || st->H < 1 || st->m != proj->m || st->d != proj->d) return DARK_ERR_INVALID_ARG;
  const size_t n = (size_t)st->B * st->H;
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaMemsetAsync(st->kv, 0, n * st->m * st->d * sizeof(float), s);
  if (e == cudaSuccess) e = cudaMemsetAsync(st->z, 0, n * st->m * sizeof(float), s);
  if (e == cudaSuccess && st->shift != nullptr) e = cudaMemsetAsync(st->shift, 0, n * sizeof(float), s);
  if (e != cudaSuccess) return DARK_ERR_CUDA;
  st->generation = proj->generation;
  return DARK_OK;
}

dark_status dark_decode_step(const dark_projection* proj, dark_state* st, const void* q_t,
                             const void* k_t, const void* v_t, void* out_t,
                             const uint8_t* valid, int* dev_status, void* stream) {
  if (proj == nullptr || proj->w == nullptr || !aligned(proj->w, 16) || !dtype_ok(proj->dtype) ||
      st == nullptr)
    return DARK_ERR_INVALID_ARG;
  if (!sizes_ok(proj->m, proj->r, proj->d)) return DARK_ERR_UNSUPPORTED;
  if (st->kv == nullptr || st->z == nullptr || q_t == nullptr || k_t == nullptr ||
      v_t == nullptr || out_t == nullptr)
    return DARK_ERR_INVALID_ARG;
  if (st->B < 1 || st->H < 1 || st->m != proj->m || st->d != proj->d) return DARK_ERR_INVALID_ARG;
  if (!(proj->heads == 1 || proj->heads == st->H)) return DARK_ERR_INVALID_ARG;
  if (!aligned(st->kv, 16)) return DARK_ERR_INVALID_ARG;
  if (st->generation != proj->generation) return DARK_ERR_STALE_STATE;
  dark::DecodeArgs a;
  a.heads_w = proj->heads;
  a.m = proj->m;
  a.r = proj->r;
  a.d = proj->d;
  a.dtype = proj->dtype;
  a.w = proj->w;
  a.kv = st->kv;
  a.z = st->z;
  a.shift = st->shift;
  a.B = st->B;
  a.H = st->H;
  a.q = q_t;
  a.k = k_t;
  a.v = v_t;
  a.out = out_t;
  a.valid = valid;
  a.update = 1;
  a.dev_status = dev_status;
  a.stream = (cudaStream_t)stream;
  return from_cuda(dark::launch_decode(a));
}

}  // extern "C"
