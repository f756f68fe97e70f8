/*
 * dark.h -- C ABI of the B200 (sm_100a) DARKformer positive-random-feature
 * attention library: forward pass (non-causal, causal, key-masked), its
 * backward pass, cross-attention, the streaming decode steps and the projection
 * sampler with its redraw schedule.
 *
 * Source of the method: the DARKformer README ("Data-Aware Random Feature
 * Kernels for Transformers", darkformer-pytorch 0.1.0 package description).
 *   - section "Kernel": Sigma = M^T M; q and k are scaled by d^{-1/4};
 *     phi(x; omega_j) = m^{-1/2} exp(omega_j^T M x - 1/2 x^T Sigma x),
 *     omega_j ~ N(0, I); Att = Phi(Q)(Phi(K)^T V) / Phi(Q)(Phi(K)^T 1).
 *   - section "Self-attention": B x L boolean key mask (true = valid), causal
 *     constraint combined with the mask, per-head or shared geometry,
 *     orthogonal or independent Gaussian features.
 *   - section "Encoder-decoder model and generation": recurrent statistics
 *     updated per appended token; a state is tied to the projection that made
 *     it, and statistics from before a redraw are refused.
 *   - section "Mixed precision": bf16 I/O with stable (fp32) accumulation.
 *
 * Conventions shared by every call
 *   - Every pointer argument named as "device" must be device memory owned by
 *     the caller; the library allocates nothing, frees nothing, and keeps no
 *     state between calls except a process-wide projection generation counter.
 *   - All calls are asynchronous on `stream` (a cudaStream_t passed as void*;
 *     NULL is the legacy default stream). Argument errors are detected on the
 *     host before anything is enqueued and returned as a status; nothing
 *     crosses the ABI as an exception and no kernel traps.
 *   - `dev_status` (device int, may be NULL): kernels store a nonzero
 *     dark_status there when they detect a problem on the device
 *     (DARK_ERR_NUMERIC: a non-finite output; DARK_ERR_TIMEOUT: a bounded
 *     inter-block wait ran out). The caller zeroes it and reads it after the
 *     stream is synchronised. The first error stored wins.
 *   - Tokens use the layout [B][H][L][d] with d innermost (stride 1) and
 *     caller-given element strides for b, h and l (NULL = contiguous).
 */
#ifndef DARK_H_
#define DARK_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define DARK_ABI_VERSION 6

typedef enum {
  DARK_OK = 0,
  DARK_ERR_INVALID_ARG = 1,   /* a size, pointer, alignment or layout is invalid  */
  DARK_ERR_UNSUPPORTED = 2,   /* valid, but outside what this build implements    */
  DARK_ERR_STALE_STATE = 3,   /* decode state made with another projection        */
  DARK_ERR_CUDA = 4,          /* a CUDA launch or runtime call failed             */
  DARK_ERR_NUMERIC = 5,       /* device: non-finite output                        */
  DARK_ERR_TIMEOUT = 6        /* device: a bounded wait between blocks ran out    */
} dark_status;

typedef enum { DARK_F32 = 0, DARK_BF16 = 1 } dark_dtype;

enum {
  DARK_CAUSAL = 1,     /* key j is visible to query i only if j <= i (diagonal included) */
  DARK_STABILISE = 2,  /* overflow guard; see dark_attention_fwd                          */
  DARK_EXACT = 4       /* the learned kernel evaluated exactly (softmax); see below        */
};

/*
 * A built projection. `w` points to caller-owned device memory holding
 *   W' = [ c_w * (Omega_h M_h) ; c_m * M_h ]   per head, [heads][m + r][d],
 *   c_w = d^{-1/4} * log2(e),  c_m = d^{-1/4} * sqrt(log2(e)/2),
 * so that, for a raw token x, (W' x)_j is the feature exponent omega_j^T M x~
 * in base 2 and sum_i (W' x)_{m+i}^2 is 1/2 x~^T Sigma x~ in base 2.
 * Element type of W': fp32 for DARK_F32 projections; fp16 (IEEE binary16)
 * for DARK_BF16 projections. fp16's 11 significant bits keep the exponents of
 * the largest features accurate to ~2e-3 (bf16's 8 bits would move them by
 * ~1e-2 and causal outputs by ~3e-2, beyond bf16 I/O tolerance). Entries of W'
 * must stay below 65504 in magnitude; the tensor-core kernels also convert bf16
 * q and k to fp16 for the feature GEMM, so |q|, |k| must stay below 65504
 * (a larger value is reported as DARK_ERR_NUMERIC).
 * `heads` is 1 when Omega and M are both shared by all heads, else H.
 * `generation` is unique per dark_make_projection call in this process.
 */
typedef struct dark_projection {
  int heads, m, r, d;
  dark_dtype dtype;
  uint64_t generation;
  void* w;
} dark_projection;

/*
 * Recurrent statistics of linear attention for every (batch, head):
 *   kv = Phi(K)^T V  as [B][H][m][d] fp32,  z = Phi(K)^T 1  as [B][H][m] fp32,
 * both device memory owned by the caller, summed over every valid key seen.
 * `shift` is NULL unless the state was made with DARK_STABILISE: then it is a
 * device [B][H] fp32 array holding the base-2 key constant c_K that every
 * stored feature was divided by (2^{-c_K}); decode reuses it.
 * `generation` ties the state to the projection that made it.
 */
typedef struct dark_state {
  float* kv;
  float* z;
  float* shift;
  int B, H, m, d;
  uint64_t generation;
} dark_state;

/* ABI version of the loaded library (DARK_ABI_VERSION at build time). */
int dark_abi_version(void);

/* Human-readable name of a status code. Never NULL; static storage. */
const char* dark_status_string(dark_status s);

/*
 * Testing hook for the device time-out path; the method's pages have no
 * counterpart of it. With cycles > 0, every tensor-core forward kernel launched
 * afterwards first waits on a barrier that nothing completes, for at most
 * `cycles` SM clock cycles, and then takes the path of a wait that ran out: it
 * records DARK_ERR_TIMEOUT in *dev_status, waits (bounded) for its own copies
 * and MMAs still in flight, frees its TMEM and returns without writing its
 * outputs. 0 (the default) turns the hook off. Process-wide: set it only while
 * no other host thread calls the library.
 */
void dark_set_test_stall_cycles(long long cycles);

/* Bytes of the projection buffer for the given sizes, 0 if a size is not positive. */
size_t dark_projection_bytes(int heads, int m, int r, int d, dark_dtype dtype);

/*
 * Builds W' (layout above) from the random features and the learned geometry
 * (README "Kernel": W = Omega M with omega_j ~ N(0, I) in R^r, M is r x d).
 *   omega       device fp32 [heads_omega][m][r]; heads_omega in {1, H}
 *   geom        device fp32 [heads_geom][r][d];  heads_geom  in {1, H}
 *   H           number of attention heads (>= 1)
 *   dtype       DARK_BF16 or DARK_F32: the element type of the tokens this
 *               projection will be used with (W' is fp16 or fp32, see above)
 *   w_buf       device, w_bytes >= dark_projection_bytes(heads, ...), 16-byte
 *               aligned; heads = max(heads_omega, heads_geom)
 *   out         host struct filled on success (w = w_buf, a new generation)
 * Products are accumulated in fp64 and rounded once to W's element type.
 * Calling it again (a redraw) gives a new generation: states made with the
 * old projection are rejected by dark_decode_step.
 * Supported sizes: 4 <= d <= 256 with d a multiple of 4, 1 <= r <= 256,
 * 1 <= m <= 1024; other positive sizes return DARK_ERR_UNSUPPORTED.
 */
dark_status dark_make_projection(const float* omega, int heads_omega, const float* geom,
                                 int heads_geom, int H, int m, int r, int d, dark_dtype dtype,
                                 void* w_buf, size_t w_bytes, void* stream,
                                 dark_projection* out);

/*
 * Workspace bytes dark_attention_fwd needs for these sizes and flags (the
 * largest need of any kernel path the call may take). The workspace is device
 * memory, 256-byte aligned, owned by the caller. Its first 256 bytes hold
 * synchronisation words: they must be zero before the workspace is first used,
 * and every call that completes without a device error leaves them zero again,
 * so the workspace can be reused without clearing. After a device error
 * (dev_status != 0) zero them again. The rest needs no initialisation. Two
 * calls in flight at the same time need two workspaces.
 */
size_t dark_attention_workspace_bytes(const dark_projection* proj, int B, int H, int L, int flags);

/*
 * Forward pass of PRF attention (README "Kernel", "Self-attention").
 *   q, k, v      device, [B][H][L][d] of proj->dtype with strides qkv_strides
 *                (elements; {b, h, l}; d stride 1; NULL = contiguous)
 *   out          device, [B][H][L][d] of proj->dtype, strides out_strides
 *   key_mask     device uint8 [B][L] (nonzero = valid key) or NULL = all valid.
 *                Masked keys contribute nothing; query rows are not masked.
 *   flags        DARK_CAUSAL: out_i uses keys j <= i only (diagonal included).
 *                DARK_STABILISE: subtract a per-query constant (the row max of
 *                the query exponents) and one per-(b, h) constant shared by
 *                all keys (the max key exponent) before exponentiating; both
 *                cancel exactly in the ratio, so outputs are unchanged in
 *                exact arithmetic while large exponents no longer overflow.
 *   state_out    NULL, or a state whose kv/z (and shift, with DARK_STABILISE)
 *                receive the statistics over all valid keys; its generation is
 *                set to proj->generation.
 *   ws, ws_bytes workspace (see dark_attention_workspace_bytes)
 * A query row whose visible valid keys sum to a zero denominator gets a zero
 * output. bf16 I/O accumulates in fp32; fp32 I/O computes in fp32 throughout.
 * Returns DARK_ERR_INVALID_ARG for inconsistent sizes or pointers,
 * DARK_ERR_UNSUPPORTED for sizes outside dark_make_projection's limits.
 */
dark_status dark_attention_fwd(const dark_projection* proj, const void* q, const void* k,
                               const void* v, void* out, const int64_t* qkv_strides,
                               const int64_t* out_strides, int B, int H, int L,
                               const uint8_t* key_mask, int flags, dark_state* state_out,
                               void* ws, size_t ws_bytes, int* dev_status, void* stream);

/*
 * dark_attention_fwd without a caller workspace, for callers that cannot
 * allocate device memory (for example a runtime that hands the library only the
 * tensors of the call, or code under an allocator that refuses extra
 * allocations). The method's pages have no counterpart of this call; it is a
 * deployment aid.
 * Arguments and results are those of dark_attention_fwd minus ws/ws_bytes; the
 * scratch is a fixed array of dark_noalloc_scratch_bytes() (16 MiB) compiled into
 * the library, which every GPU that loads the library keeps until the process
 * exits. Nothing is allocated and nothing is freed.
 *   - Returns DARK_ERR_UNSUPPORTED, enqueuing nothing, when the call needs more
 *     scratch than that (dark_attention_workspace_bytes tells the size the call
 *     would need with a workspace of its own).
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress); make that first call before any stream capture.
 *     The address is kept for the life of the process: after cudaDeviceReset
 *     (or any other teardown of the device's primary context) do not call this
 *     entry point again in that process.
 *   - Every call shares the one array and it keeps the previous call's
 *     contents: calls whose work overlaps on the GPU (different streams, or
 *     different host threads without ordering) race on it. Serialise them.
 */
size_t dark_noalloc_scratch_bytes(void);
dark_status dark_attention_fwd_noalloc(const dark_projection* proj, const void* q, const void* k,
                                       const void* v, void* out, const int64_t* qkv_strides,
                                       const int64_t* out_strides, int B, int H, int L,
                                       const uint8_t* key_mask, int flags, dark_state* state_out,
                                       int* dev_status, void* stream);

/*
 * Zeroes a state (kv, z and, if non-NULL, shift) and ties it to `proj`, for
 * decoding from an empty prefix.
 */
dark_status dark_state_init(const dark_projection* proj, dark_state* st, void* stream);

/*
 * One streaming decode step for every (batch, head) (README "Encoder-decoder
 * model and generation"): with k_t valid, kv += phi(k_t) v_t^T and
 * z += phi(k_t); then out_t = phi(q_t)^T kv / phi(q_t)^T z (update, then emit).
 *   q_t, k_t, v_t, out_t  device [B][H][d] of proj->dtype, contiguous
 *   valid                 device uint8 [B] (nonzero = this token is a valid key)
 *                         or NULL = all valid
 *   st                    state of sizes (B, H, proj->m, proj->d)
 * Returns DARK_ERR_STALE_STATE, enqueuing nothing, when st->generation !=
 * proj->generation (the projection was rebuilt after the state was made).
 */
dark_status dark_decode_step(const dark_projection* proj, dark_state* st, const void* q_t,
                             const void* k_t, const void* v_t, void* out_t,
                             const uint8_t* valid, int* dev_status, void* stream);

/*
 * Workspace bytes dark_cross_attention_fwd needs (0 for invalid arguments or
 * DARK_CAUSAL). Same rules as dark_attention_workspace_bytes.
 */
size_t dark_cross_attention_workspace_bytes(const dark_projection* proj, int B, int H, int Lq,
                                            int Lk, int flags);

/*
 * Cross-attention of Lq queries over an Lk-token context (README
 * "Cross-attention": separate query and context masks, no causal option):
 * out_i = phi(q_i)^T S / phi(q_i)^T z with S = Phi(K)^T V and z = Phi(K)^T 1
 * over the valid context positions.
 *   q            device, [B][H][Lq][d] of proj->dtype, strides q_strides
 *                (elements; {b, h, l}; d stride 1; NULL = contiguous)
 *   query_mask   device uint8 [B][Lq] or NULL; a masked query row (0) gets a
 *                zero output (the pages leave the query mask's effect open:
 *                this library's reading)
 *   k, v         device, [B][H][Lk][d], strides kv_strides (NULL = contiguous)
 *   context_mask device uint8 [B][Lk] (nonzero = valid context position) or NULL
 *   out          device, [B][H][Lq][d], strides out_strides (NULL = contiguous)
 *   flags        0 or DARK_STABILISE; DARK_CAUSAL returns DARK_ERR_INVALID_ARG
 *   context_out  NULL, or a state that receives the context summary (S, z),
 *                which decoding reuses at every step (see
 *                dark_cross_decode_step); its generation is set
 *   ws, ws_bytes workspace (dark_cross_attention_workspace_bytes)
 * Errors as dark_attention_fwd.
 */
dark_status dark_cross_attention_fwd(const dark_projection* proj, const void* q,
                                     const int64_t* q_strides, int Lq, const uint8_t* query_mask,
                                     const void* k, const void* v, const int64_t* kv_strides,
                                     int Lk, const uint8_t* context_mask, void* out,
                                     const int64_t* out_strides, int B, int H, int flags,
                                     dark_state* context_out, void* ws, size_t ws_bytes,
                                     int* dev_status, void* stream);

/*
 * One decoder step of cross-attention against a context summary made by
 * dark_cross_attention_fwd (README "Encoder-decoder model and generation":
 * decoder cross-attention summarises the encoded source once per layer):
 * out_t = phi(q_t)^T S / phi(q_t)^T z. The summary is read, never written.
 *   q_t, out_t   device [B][H][d] of proj->dtype, contiguous
 *   context      state of sizes (B, H, proj->m, proj->d)
 * Returns DARK_ERR_STALE_STATE, enqueuing nothing, when context->generation !=
 * proj->generation.
 */
dark_status dark_cross_decode_step(const dark_projection* proj, const dark_state* context,
                                   const void* q_t, void* out_t, int* dev_status, void* stream);

/*
 * Backward pass of self-attention (dark_attention_fwd without query mask):
 * gradients of sum(dout * out) with respect to q, k, v and the geometry M.
 * README, section "Kernel": M (r x d per head, or shared) is the learned factor
 * of Sigma = M^T M, whose learning is the method's point; Omega is a fixed draw
 * of the projection and gets no gradient. Section "Self-attention": the key mask
 * and the causal constraint act as in the forward pass. A query row with no
 * visible valid key has output 0 and contributes no gradient; masked keys get
 * zero dk and dv.
 *
 * The projection is rebuilt in fp32 from omega and geom (the forward's W' for
 * bf16 is fp16), features are recomputed, and every step accumulates in fp32.
 *   omega        device fp32 [heads_omega][m][r]  (heads_omega = 1 or H)
 *   geom         device fp32 [heads_geom][r][d]   (heads_geom = 1 or H)
 *   dtype        element type of q, k, v, dout, dq, dk, dv
 *   q, k, v      device [B][H][L][d], element strides qkv_strides {b, h, l}
 *   dout         device [B][H][L][d], strides dout_strides (NULL = contiguous)
 *   key_mask     device uint8 [B][L] (nonzero = valid) or NULL
 *   flags        DARK_CAUSAL and/or DARK_STABILISE (a per-head key shift; the
 *                gradients do not depend on it)
 *   dq, dk, dv   device [B][H][L][d], strides grad_strides; overwritten. They
 *                must not overlap each other or any input.
 *   dgeom        device fp32 [heads_geom][r][d], overwritten with the gradient
 *                summed over batches and over the heads sharing M; NULL skips it.
 *   ws, ws_bytes device workspace of at least
 *                dark_attention_bwd_workspace_bytes(...) bytes, 256-byte
 *                aligned; no initial contents are required.
 * Errors: DARK_ERR_INVALID_ARG for a null pointer, a bad head count, flag,
 * stride or workspace; DARK_ERR_UNSUPPORTED for sizes outside the library's
 * limits or B*H > 65535; DARK_ERR_CUDA for a failed launch; the device may store
 * DARK_ERR_NUMERIC in dev_status for a non-finite gradient.
 */
size_t dark_attention_bwd_workspace_bytes(int heads_omega, int heads_geom, int m, int r, int d,
                                          int B, int H, int L);
dark_status dark_attention_bwd(const float* omega, int heads_omega, const float* geom,
                               int heads_geom, int m, int r, int d, dark_dtype dtype,
                               const void* q, const void* k, const void* v,
                               const int64_t* qkv_strides, const void* dout,
                               const int64_t* dout_strides, int B, int H, int L,
                               const uint8_t* key_mask, int flags, void* dq, void* dk, void* dv,
                               const int64_t* grad_strides, float* dgeom, void* ws,
                               size_t ws_bytes, int* dev_status, void* stream);

/*
 * Exact mode (README, section "Attention modes": M acts on queries and keys and
 * ordinary softmax attention with scaled scores follows).
 * DARK_EXACT in the flags of dark_attention_fwd, dark_attention_fwd_noalloc or
 * dark_cross_attention_fwd evaluates
 *   out_i = sum_j softmax_j(u_i . w_j) v_j,  u = M q~, w = M k~, x~ = d^{-1/4} x,
 * (scores q^T Sigma k / sqrt(d)) over the valid keys (j <= i with DARK_CAUSAL)
 * instead of the random-feature estimate. M is read from the projection's last r
 * rows (c_m M); Omega is not used. A query row with no visible key outputs 0.
 * state_out / context_out must be NULL (the mode keeps no recurrent statistics);
 * DARK_STABILISE is accepted and has no effect (the softmax is computed with a
 * running maximum). The workspace queries account for the flag. bf16 I/O with
 * d = 64 (r <= 64) or d = 128 (r <= 128), r a multiple of 16 and 16-byte aligned
 * rows runs on the tensor cores; every other shape on the fp32 SIMT kernels, with
 * the same results within rounding.
 *
 * Auto mode ("exact_threshold"): the exact mode for sequences up to the threshold
 * length, random features for longer ones. dark_auto_uses_exact returns 1 when L <= exact_threshold and
 * exact_threshold > 0; the caller then adds DARK_EXACT.
 */
int dark_auto_uses_exact(int L, int exact_threshold);

/*
 * Projection sampler: Omega drawn on the device, reproducibly from (seed, draw).
 * README, section "Kernel": omega_j ~ N(0, I_r); section "Self-attention":
 * orthogonal Gaussian blocks by default, independent Gaussian features when
 * orthogonal_features=False; section "Projection lifecycle": projection_seed makes
 * the draws reproducible.
 *
 * Generator (the pages fix none): Philox4x64-10 with key (seed, draw) and counter
 * (block, head, purpose, 0); the block's four 64-bit words give two Box-Muller pairs
 * (u1 = 1 - u(x_a), u2 = u(x_b), u(x) = (x >> 11) 2^-53). Stream element e of
 * (head, purpose) is word e % 4 of block e / 4.
 *   independent: Omega[h][j][i] = z(h, 0, j r + i);
 *   orthogonal:  per block b of r rows, G[i][k] = z(h, 0, b r^2 + i r + k), G = Q R
 *                with diag(R) > 0 (fp64 Gram-Schmidt with re-orthogonalisation),
 *                row i = ||(z(h, 1, b r^2 + i r + k))_k|| * Q[:, i]; a partial last
 *                block keeps its first rows.
 *   omega     device fp32 [heads][m][r], written
 *   ws        device workspace of dark_sample_omega_workspace_bytes(...) bytes,
 *             256-byte aligned (none needed for independent features: NULL is fine)
 * Errors: DARK_ERR_INVALID_ARG for a null or misaligned pointer, bad sizes or a
 * short workspace; DARK_ERR_UNSUPPORTED for m > 1024, r > 256 or heads > 65535;
 * DARK_ERR_CUDA for a failed launch.
 */
size_t dark_sample_omega_workspace_bytes(int heads, int m, int r, int orthogonal);
dark_status dark_sample_omega(uint64_t seed, uint64_t draw, int heads, int m, int r,
                              int orthogonal, float* omega, void* ws, size_t ws_bytes,
                              void* stream);

/*
 * Redraw schedule of one projection (host only; README, section "Projection
 * lifecycle"). The current projection is dark_sample_omega(seed, draw, ...).
 *   interval > 0: once that many training forwards have run, a redraw happens at
 *   the start of the next training forward; forwards outside training are not
 *   counted;
 *   interval <= 0: no scheduled redraws. While fixed, a redraw falling due is
 *   dropped (the interval restarts) and ordinary requests are refused; a forced
 *   request redraws once. Every redraw restarts the interval. deterministic != 0
 *   fixes the projection at construction.
 */
typedef struct dark_redraw_schedule {
  uint64_t seed;       /* projection seed */
  uint64_t draw;       /* redraws so far: the current projection's draw index */
  int64_t interval;    /* training forwards between scheduled redraws; 0: none */
  int64_t count;       /* training forwards since the interval last restarted */
  int fixed;           /* 1: ordinary redraws are ignored */
} dark_redraw_schedule;

dark_status dark_redraw_schedule_init(dark_redraw_schedule* s, uint64_t seed, int64_t interval,
                                      int deterministic);
/* At the start of a forward: 1 if a redraw happened (draw advanced), else 0. */
int dark_redraw_on_forward(dark_redraw_schedule* s, int training);
/* A manual redraw request: 1 if granted (draw advanced), else 0. */
int dark_redraw_request(dark_redraw_schedule* s, int force);
void dark_redraw_set_fixed(dark_redraw_schedule* s, int fixed);

#ifdef __cplusplus
}
#endif

#endif /* DARK_H_ */
