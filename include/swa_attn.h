/*
 * swa_attn.h -- C ABI of the B200 (sm_100a) masked-attention library.
 *
 * One operation, in several masks: the masked attention forward
 *     A = softmax(Q K^T * scale + log M) V,   log M_ij = 0 (allowed) or -inf,
 * from "Learn: Sparse & Sliding-Window Attention", section 3 "The math". The
 * mask is never stored; each query tile visits only the key tiles its mask
 * touches, so the work grows with the number of attended cells.
 *
 * Conventions shared by every entry point:
 *   - Tensors are row-major, contiguous, bf16 unless stated: Q [B, Hq, N, d],
 *     K and V [B, Hkv, N, d]. Query head h reads KV head h / (Hq / Hkv)
 *     (grouped-query attention, "Sliding Window Attention" glossary page,
 *     GQA entry; the consecutive grouping is this library's reading).
 *   - Every pointer argument named as device memory must be device memory of
 *     the current CUDA device, 16-byte aligned. The caller allocates and owns
 *     every buffer; the library allocates nothing at call time and keeps no
 *     pointer after the call returns.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream). Calls
 *     are asynchronous on that stream: on return the work is queued, not
 *     done.
 *   - Argument errors are reported before anything is launched
 *     (SWA_ERR_INVALID_ARG / SWA_ERR_UNSUPPORTED). A failed launch returns
 *     SWA_ERR_CUDA. Every wait inside a kernel is bounded (about two
 *     seconds); a kernel whose wait runs out records SWA_ERR_TIMEOUT in a
 *     device flag, releases what it holds and returns; swa_last_device_error
 *     reports it.
 *   - Outputs are bf16 rounded to nearest even from fp32 accumulators.
 */
#ifndef SWA_ATTN_H
#define SWA_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SWA_OK = 0,
  SWA_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size or ratio  */
  SWA_ERR_UNSUPPORTED = 2, /* valid but not built: head dim outside {64,128} */
  SWA_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed           */
  SWA_ERR_TIMEOUT = 4,     /* a bounded in-kernel wait ran out            */
  SWA_ERR_SCRATCH_TOO_SMALL = 5, /* sizes need more scratch than the library's
                                    static decode array holds              */
  SWA_ERR_BOUNDS = 6       /* bounds-checking debug build only: a TMA
                              coordinate or global index fell outside its
                              tensor (the access was skipped)              */
} swa_status_t;

/* Optional device-side debug outputs of the prefill kernels (pass NULL to
 * skip). Indexing is per (b, hq, query tile of 128 rows):
 * idx = (b * Hq + hq) * ceil(N / 128) + qt.
 *   cells  [B*Hq*nq] int64: attended cells the kernel processed for that
 *          query tile are ADDED here (zero it first).
 *   tiles  [B*Hq*nq*tiles_cap] int32: the key tiles the kernel visited, in
 *          visiting order: a window tile is its index kt (keys kt*128 ..
 *          kt*128+127); a stride tile is 0x40000000 | ct (stride keys
 *          m*S for m in ct*128 .. ct*128+127).
 *   ntiles [B*Hq*nq] int32: how many entries were visited (may exceed
 *          tiles_cap; only the first tiles_cap are written).
 *   inject_timeout: nonzero makes the kernel withhold its first key tile so
 *          that its waits run out and it returns SWA_ERR_TIMEOUT through
 *          swa_last_device_error (a test of the error path; nothing hangs).
 */
typedef struct {
  int64_t* cells;
  int32_t* tiles;
  int32_t* ntiles;
  int32_t tiles_cap;
  int32_t inject_timeout;
} swa_debug_t;

/* Sliding-window attention forward.
 * Source: "Learn: Sparse & Sliding-Window Attention", section 3a, band mask
 * M_ij = 1[i - W < j <= i]; "Attention Variants Compared", swa_mask code
 * (lo = max(0, i - window + 1); window >= n gives full causal).
 *   q [B,Hq,N,d], k, v [B,Hkv,N,d] bf16 (device, read only);
 *   o [B,Hq,N,d] bf16 (device, written);
 *   lse [B,Hq,N] fp32 natural-log sum of exp of the scaled scores, or NULL;
 *   d in {64, 128}; W >= 1 (W >= N is full causal); Hq % Hkv == 0;
 *   scale multiplies Q K^T (1/sqrt(d) for the usual attention); it must be
 *   finite and at least 1e-30 (masked scores are carried as -FLT_MAX, and
 *   this keeps their weights exactly 0). */
swa_status_t swa_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                          int B, int Hq, int Hkv, int N, int d, int W, float scale, void* stream);

/* Local + strided attention forward: the window mask OR every stride-th key
 * (keys j with j % stride == 0 and j <= i). Each attended cell counts once.
 * Source: "Attention Variants Compared", strided_mask code ("local window,
 * then every stride-th token back to 0"); "Exploring Attention Variants",
 * Sparse Attention section (the two masks combined by logical OR).
 * Arguments as swa_attn_fwd, plus stride >= 1. */
swa_status_t strided_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                              int B, int Hq, int Hkv, int N, int d, int W, int stride,
                              float scale, void* stream);

/* Window + global-token attention forward: row i attends key j <= i when
 * i - W < j (the window) or j < n_global (a global token) or i < n_global
 * (a global row). Source: "Learn: Sparse & Sliding-Window Attention",
 * section 3b (Longformer: global tokens attend to everything and are
 * attended to by everything, a full row and column of M each; cost
 * O(s w + s g)) and section 6 (window + global FLOPs). The pages do not
 * place the global tokens; this library takes positions 0 .. n_global-1
 * (a [CLS] or question prefix), where a global row's causal keys are all
 * global. Extra (global) keys below a row's window are visited as whole
 * 128-key tiles of K/V, before the window tiles; every cell counts once.
 *   Arguments as swa_attn_fwd, plus n_global >= 0 (0 is swa_attn_fwd). */
swa_status_t global_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                             int B, int Hq, int Hkv, int N, int d, int W, int n_global,
                             float scale, void* stream);

/* Dilated sliding-window attention forward: row i attends the W keys
 * i, i - dilation, ..., i - (W-1)*dilation (those >= 0).
 * Source: "Learn: Sparse & Sliding-Window Attention", section 3b
 * (Longformer: gaps of size d_dil inside the window, so the same budget of
 * keys reaches d_dil times further). Rows and keys of one residue class mod
 * `dilation` form a plain window of W keys, so the call runs the window
 * kernel once per class on strided views of Q, K, V and O (no copies).
 *   Arguments as swa_attn_fwd, plus dilation >= 1 (1 is swa_attn_fwd);
 *   lse, if given, is written at the original row positions. */
swa_status_t dilated_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                              int B, int Hq, int Hkv, int N, int d, int W, int dilation,
                              float scale, void* stream);

/* Differential attention forward:
 *     o = softmax(Q1 K1^T * scale + log M) V - lambda[h] * softmax(Q2 K2^T * scale + log M) V
 * over one shared V, both maps under the same window mask (W >= N: causal).
 * Source: "Attention Variants -- Sliding Window, Sparse, Differential", the
 * problem statement (two maps from separate Q/K projections, one subtracted
 * from the other); "Attention Variants Compared", variants table
 * (Differential: 2 times N squared compute).
 *   q1, q2 [B,Hq,N,d_qk], k1, k2 [B,Hkv,N,d_qk], v [B,Hkv,N,d_v] bf16;
 *   o [B,Hq,N,d_v] bf16; lambda: device fp32 [Hq];
 *   d_qk == 64 (K1 and K2 tiles share one shared-memory slot), d_v in
 *   {64, 128}; other head dims return SWA_ERR_UNSUPPORTED. */
swa_status_t diff_attn_fwd(const void* q1, const void* k1, const void* q2, const void* k2,
                           const void* v, void* o, const float* lambda, int B, int Hq, int Hkv,
                           int N, int d_qk, int d_v, int W, float scale, void* stream);

/* One decode step over a rolling W-slot KV cache.
 * Source: "Learn: Sparse & Sliding-Window Attention", section 4 (keep a
 * rolling window of the most recent w tokens, evict the oldest) and
 * section 6 (the cache stays O(w)); "Sliding Window Attention" glossary page
 * (fixed-size KV cache).
 *   q [B,Hq,d]; k_new, v_new [B,Hkv,d] bf16 (device, read only);
 *   k_cache, v_cache [B,Hkv,W,d] bf16 (device, updated: slot pos[b] % W of
 *     sequence b receives k_new/v_new);
 *   pos: device int32 [B], absolute position (>= 0) of the new token;
 *   o [B,Hq,d] bf16 (device, written);
 *   workspace: device scratch of at least swa_decode_workspace_bytes(...)
 *     bytes, 16-byte aligned; its contents need not be initialised.
 * The step writes the new token first, then attends over the positions
 * max(0, pos-W+1) .. pos, which the cache's slots hold in rotated order. */
swa_status_t swa_decode_step(const void* q, const void* k_new, const void* v_new, void* k_cache,
                             void* v_cache, const int32_t* pos, void* o, int B, int Hq, int Hkv,
                             int d, int W, float scale, void* workspace, size_t ws_bytes,
                             void* stream);

/* Scratch bytes swa_decode_step needs for these sizes (0 on bad sizes). */
size_t swa_decode_workspace_bytes(int B, int Hq, int Hkv, int d, int W);

/* One decode step with attention sinks over an (n_sink + W)-slot cache.
 * Source: "Learn: Sparse & Sliding-Window Attention", section 4
 * (StreamingLLM: keep the first k tokens -- the attention sinks -- for good
 * plus the most recent w tokens, drop the middle) and section 6 (the cache
 * stays O(k + w)).
 *   k_cache, v_cache [B,Hkv,n_sink+W,d] bf16 (device, updated): positions
 *     p < n_sink live in slot p for good; a later position p takes slot
 *     n_sink + (p - n_sink) % W, replacing the oldest non-sink token;
 *   the step stores its token, then attends over the sink positions
 *     0 .. min(n_sink, pos+1)-1 and the positions max(n_sink, pos-W+1) .. pos;
 *   n_sink >= 0 (0 is swa_decode_step); workspace of at least
 *     swa_sink_decode_workspace_bytes(...) bytes; other arguments as
 *     swa_decode_step. */
swa_status_t swa_sink_decode_step(const void* q, const void* k_new, const void* v_new,
                                  void* k_cache, void* v_cache, const int32_t* pos, void* o,
                                  int B, int Hq, int Hkv, int d, int n_sink, int W, float scale,
                                  void* workspace, size_t ws_bytes, void* stream);

/* Scratch bytes swa_sink_decode_step needs (0 on bad sizes). */
size_t swa_sink_decode_workspace_bytes(int B, int Hq, int Hkv, int d, int n_sink, int W);

/* One differential-attention decode step over a rolling W-slot cache.
 * ("Attention Variants -- Sliding Window, Sparse, Differential", The Problem:
 * two attention maps from separate Q/K projections, one subtracted from the
 * other: out = sum_j (w1_j - lambda_h w2_j) v_j with w1 = softmax(scale q1
 * K1^T), w2 = softmax(scale q2 K2^T) over the same window. "Attention
 * Variants Compared", symptom table: the first differential version's
 * decode loads the value cache twice; here every slot's K1, K2 and V bytes
 * are read once. Window as swa_decode_step: "Learn: Sparse & Sliding-Window
 * Attention", section 4.)
 *   q1, q2            device bf16 [B, Hq, d_qk]
 *   k1_new, k2_new    device bf16 [B, Hkv, d_qk]; v_new [B, Hkv, d_v]
 *   k1_cache, k2_cache device bf16 [B, Hkv, W, d_qk]; v_cache [B, Hkv, W, d_v];
 *                     position p lives in slot p % W; the step first stores
 *                     its token in slot pos % W, then attends over the
 *                     positions max(0, pos-W+1) .. pos
 *   pos               device int32 [B], absolute position of the new token
 *   lambda            device fp32 [Hq]
 *   o                 device bf16 [B, Hq, d_v]
 *   d_qk = 64 and d_v = 128 only (SWA_ERR_UNSUPPORTED otherwise); Hq/Hkv in
 *   {1, 2, 4, 8}; workspace: device, 16-byte aligned, at least
 *   swa_diff_decode_workspace_bytes(...) bytes, owned by the caller.
 * Pointers not 16-byte aligned (pos and lambda: 4), a null pointer, a short
 * workspace or a bad size return SWA_ERR_INVALID_ARG before any launch. */
swa_status_t swa_diff_decode_step(const void* q1, const void* q2, const void* k1_new,
                                  const void* k2_new, const void* v_new, void* k1_cache,
                                  void* k2_cache, void* v_cache, const int32_t* pos,
                                  const float* lambda, void* o, int B, int Hq, int Hkv,
                                  int d_qk, int d_v, int W, float scale, void* workspace,
                                  size_t ws_bytes, void* stream);

/* Scratch bytes swa_diff_decode_step needs (0 on bad or unsupported sizes). */
size_t swa_diff_decode_workspace_bytes(int B, int Hq, int Hkv, int d_qk, int d_v, int W);

/* Bytes of the scratch array compiled into the library for
 * swa_decode_step_static (on every GPU that loads the library). */
#define SWA_DECODE_STATIC_SCRATCH_BYTES (4u << 20)

/* swa_decode_step for callers that cannot allocate device memory. The pages
 * have no counterpart: this is a convenience of this library's ABI.
 * Some callers cannot hand over a workspace: a plugin host that gives a
 * library tensors but no allocator, or a serving loop whose hot path may not
 * allocate. This entry point allocates nothing; its scratch (the per-split
 * partial results) is a fixed array of SWA_DECODE_STATIC_SCRATCH_BYTES inside
 * the library, which every GPU that loads the library holds until the process
 * exits. Arguments, layout and results are those of swa_decode_step, minus
 * the workspace. Sizes whose scratch (swa_decode_workspace_bytes) exceeds the
 * array return SWA_ERR_SCRATCH_TOO_SMALL before anything is launched.
 * The first call on a device looks up the array's device address (once per
 * device, with that device current); make that first call before any stream
 * capture. Every call shares the one array, which keeps the last call's
 * contents (nothing in it needs to start at zero): calls whose work overlaps
 * on the GPU -- on different streams, or from different threads -- race on
 * it and must be serialised by the caller. */
swa_status_t swa_decode_step_static(const void* q, const void* k_new, const void* v_new,
                                    void* k_cache, void* v_cache, const int32_t* pos, void* o,
                                    int B, int Hq, int Hkv, int d, int W, float scale,
                                    void* stream);

/* Backward of swa_attn_fwd: the gradients dQ, dK, dV of a loss whose
 * gradient with respect to the output is dO.
 * The pages define the forward only ("Learn: Sparse & Sliding-Window
 * Attention", section 3: A = softmax(Q K^T * scale + log M) V); this is its
 * chain rule under the same window mask, with P = exp(scale Q K^T - L) from
 * the forward's log-sum-exp L, D = rowsum(dO * O), dS = P * (dO V^T - D):
 *     dV = P^T dO,   dQ = scale dS K,   dK = scale dS^T Q,
 * dK and dV summed over the query heads of each KV head.
 *   q, o, d_o [B,Hq,N,d]; k, v [B,Hkv,N,d] bf16 (device, read only): the
 *     forward's inputs and output and the output's gradient;
 *   lse [B,Hq,N] fp32 (device): the forward's log-sum-exp (swa_attn_fwd
 *     with a non-NULL lse);
 *   dq [B,Hq,N,d], dk, dv [B,Hkv,N,d] bf16 (device, written);
 *   d in {64, 128}; W >= 1 (W >= N is full causal); Hq % Hkv == 0;
 *   workspace: device, 16-byte aligned, at least
 *     swa_attn_bwd_workspace_bytes(B, Hq, N) bytes (caller-owned).
 * Three kernels run on `stream`: row terms, dK/dV, dQ. */
swa_status_t swa_attn_bwd(const void* q, const void* k, const void* v, const void* o,
                          const void* d_o, const float* lse, void* dq, void* dk, void* dv, int B,
                          int Hq, int Hkv, int N, int d, int W, float scale, void* workspace,
                          size_t ws_bytes, void* stream);

/* Scratch bytes swa_attn_bwd needs (0 on bad sizes). */
size_t swa_attn_bwd_workspace_bytes(int B, int Hq, int N);

/* Backward of strided_attn_fwd (window OR keys j % stride == 0, j <= i):
 * the same chain rule as swa_attn_bwd over the union mask. Stride keys below
 * a row's window are gathered through a strided view of K and V (no copies);
 * their dK/dV contributions from every later query row are accumulated in
 * fp32 in the workspace and added to the window pass's before rounding.
 *   Arguments as swa_attn_bwd, plus stride >= 1; lse from strided_attn_fwd;
 *   workspace of at least strided_attn_bwd_workspace_bytes(...) bytes. */
swa_status_t strided_attn_bwd(const void* q, const void* k, const void* v, const void* o,
                              const void* d_o, const float* lse, void* dq, void* dk, void* dv,
                              int B, int Hq, int Hkv, int N, int d, int W, int stride,
                              float scale, void* workspace, size_t ws_bytes, void* stream);

/* Note on determinism: the stride keys' partial dK/dV are summed in fp32 with
 * atomic adds, in an order that varies from run to run, so strided_attn_bwd's
 * dK and dV can differ in the last bit between identical calls (within the
 * stated accuracy). swa_attn_bwd and every forward entry point are
 * deterministic. */

/* Scratch bytes strided_attn_bwd needs (0 on bad sizes). */
size_t strided_attn_bwd_workspace_bytes(int B, int Hq, int Hkv, int N, int d, int stride);

/* Prefill with debug outputs. kind 0 = sliding window (stride ignored),
 * kind 1 = local + strided, kind 3 = window + global tokens (stride carries
 * n_global). Same arithmetic as swa_attn_fwd / strided_attn_fwd /
 * global_attn_fwd; dbg may be NULL. */
swa_status_t swa_prefill_debug(int kind, const void* q, const void* k, const void* v, void* o,
                               float* lse, int B, int Hq, int Hkv, int N, int d, int W,
                               int stride, float scale, const swa_debug_t* dbg, void* stream);

/* The key tiles each query tile visits, as the kernels enumerate them
 * (host only; the kernels call the same function). kind 0 = window,
 * 1 = window + stride, 2 = full causal, 3 = window + global tokens (stride
 * carries n_global >= 0; extra tiles hold keys ct*Bk .. ct*Bk+Bk-1). Query tiles are Bq rows, key tiles
 * Bk keys (the kernels use 128 x 128). qtile_offsets [nq + 1] receives the
 * start of each query tile's list in `tiles`; tiles receives up to cap
 * entries in the encoding of swa_debug_t. Returns the total number of
 * entries (which may exceed cap), or -1 on bad arguments. Either output
 * may be NULL to just count. Source: "Learn: Sparse & Sliding-Window
 * Attention", section 3 (cost proportional to ||M||_0);
 * "Attention Variants Compared", glossary (zero blocks skipped in the
 * kernel). */
int64_t swa_schedule(int kind, int N, int W, int stride, int Bq, int Bk, int32_t* qtile_offsets,
                     int32_t* tiles, int64_t cap);

/* ||M||_0, the attended cells of one (b, head) N x N mask, in closed form
 * (kind as swa_schedule; stride ignored unless kind is 1 or 3). -1 on bad
 * arguments. Source: "Attention Variants Compared", count_nonmasked. */
int64_t swa_count_nonmasked(int kind, int N, int W, int stride);

/* Debug: y[i] = 2^x[i] through the prefill kernels' own FMA-pipe exponential
 * (Cody-Waite range reduction plus a cubic minimax polynomial, evaluated in
 * fp32 on pairs), which the differential kernel uses for a quarter of its
 * exponentials instead of the MUFU unit. Exposed so that a test can hold it
 * to its bound: relative error at most 1.02e-4 for x in [-125, 8], exactly 0
 * for x <= -127 (-inf included), finite everywhere below 8 (in the kernels
 * the argument never exceeds 8). Not part of the attention path.
 *   x, y: device fp32 [n], 4-byte aligned (y written); n >= 0 (0: no-op).
 *   A null or misaligned pointer or n < 0 returns SWA_ERR_INVALID_ARG. */
swa_status_t swa_debug_exp2(const float* x, float* y, int64_t n, void* stream);

/* Synchronises `stream`, then returns and clears the device error flag of
 * the current device (SWA_OK if no kernel recorded an error). */
swa_status_t swa_last_device_error(void* stream);

/* A static, human-readable name for a status code. */
const char* swa_status_string(swa_status_t status);

#ifdef __cplusplus
}
#endif

#endif /* SWA_ATTN_H */
