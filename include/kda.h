/*
 * kda.h -- C ABI of libkda.so: Kimi Delta Attention (KDA) on NVIDIA B200 (sm_100a).
 *
 * KDA is delta-rule linear attention with a channel-wise forget gate, computed
 * chunk-parallel, with a lower-bounded decay ("KimiDelta Attention (KDA)",
 * section 一.1 of the CSDN post analysing the Kimi K3 technical report).  Per
 * request and head, with a fixed-size state S in R^{dk x dv}:
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *     o_t = S_t^T q_t                      alpha_t = exp(g_t), g_t in [-5, 0]^{dk}
 *
 * The pages describe this in words; the algebraic form above is the plain
 * reading used throughout the library (decay first, then the delta-rule
 * write, output from the post-update state, no 1/sqrt(d) scale).
 *
 * Conventions shared by every call
 *   - All tensor pointers are DEVICE pointers to caller-owned, C-contiguous,
 *     16-byte-aligned memory.  The library allocates nothing and keeps no
 *     pointer after a call returns; scratch space is passed in as `workspace`.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Every compute call is asynchronous on that stream.
 *   - Argument errors are detected on the host before anything is launched and
 *     returned synchronously; no kernel runs in that case.
 *   - Errors found on the device (input validation when the environment
 *     variable KDA_VALIDATE=1 is set, or a bounded wait that gave up) are
 *     recorded in a per-device status word; read it with
 *     kda_get_device_status().  Kernels never trap and never spin unbounded.
 *   - Layouts are token-major and packed over requests ("THD"):
 *       q, k, g : [T_total, H, dk]     v, o : [T_total, H, dv]
 *       beta    : [T_total, H]         states : [n, H, dk, dv], dv contiguous
 *     Page 4 ("从 KDA 到 Stable LatentMoE：Kimi K3 底层架构全拆解", section 三)
 *     writes per-sequence tensors as (B, H, T, D); packing the token axis is
 *     what variable-length requests need, and a fixed-length batch is the
 *     special case cu_seqlens[r] = r * T.
 *   - Supported shapes: dk == dv in {64, 128}; H >= 1; chunk size is 64.
 *   - Results are deterministic: the same inputs give bit-identical outputs
 *     (no floating-point atomics), and a request's results do not depend on
 *     which other requests share the batch.
 */
#ifndef KDA_H_
#define KDA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define KDA_CHUNK 64           /* tokens per chunk of the chunked form */
#define KDA_VERSION 100        /* 1.0.0 */

typedef enum {
  KDA_OK = 0,
  KDA_ERR_INVALID_ARG = 1,  /* a pointer, size, stride or layout is invalid */
  KDA_ERR_UNSUPPORTED = 2,  /* valid but not implemented (e.g. dk != dv, d not 64/128) */
  KDA_ERR_CUDA = 3,         /* a CUDA runtime call or kernel launch failed */
  KDA_ERR_GATE_RANGE = 4,   /* (device, KDA_VALIDATE=1) g outside [-5, 0] or beta outside [0, 1] */
  KDA_ERR_TIMEOUT = 5,      /* (device) a bounded wait inside a kernel gave up */
  KDA_ERR_WORKSPACE = 6     /* workspace pointer NULL or smaller than required */
} kda_status;

typedef enum { KDA_BF16 = 0, KDA_F32 = 1 } kda_dtype;

/* ------------------------------------------------------------------------ */
/* Chunked prefill over packed variable-length requests.                    */
/* ------------------------------------------------------------------------ */

/*
 * Arguments of kda_prefill_chunked.
 *
 * Source of the operation: the chunk-parallel KDA forward -- tokens inside a
 * chunk are processed together, the state passes between chunks in order
 * ("Kimi K3 开源日来了", FlashKDA section) -- over requests that each carry a
 * fixed-size recurrent state, with sparse state snapshots at 512-token block
 * boundaries for prefix-cache reuse ("Kimi K3 开源日来了", Infra section,
 * second layer).  The result equals the token-by-token recurrence above up
 * to floating-point rounding.
 *
 *   n_req          number of packed requests, >= 0 (0 launches nothing).
 *   total_tokens   T_total; must equal cu_seqlens[n_req] (not checked on the
 *                  device unless KDA_VALIDATE=1).
 *   H, dk, dv      heads and head dims; dk == dv in {64, 128}.
 *   in_dtype       dtype of q, k, v (KDA_BF16 or KDA_F32).
 *   out_dtype      dtype of o (KDA_F32 recommended for parity checks).
 *   q, k           [T_total, H, dk] in_dtype.  No normalisation or scaling is
 *                  applied by the library; o is linear in q.
 *   v              [T_total, H, dv] in_dtype.
 *   g              [T_total, H, dk] fp32, g = log(alpha) per key channel.
 *                  Precondition -5 <= g <= 0 (alpha >= exp(-5)): the
 *                  lower-bounded decay that keeps the chunked form's
 *                  exponentials finite.  Checked only when KDA_VALIDATE=1.
 *                  NULL when g_logits is given (exactly one of the two).
 *   beta           [T_total, H] fp32, precondition 0 <= beta <= 1.
 *   cu_seqlens     DEVICE int32 [n_req + 1]; cu_seqlens[0] == 0, non-decreasing.
 *                  Request r owns tokens cu_seqlens[r] .. cu_seqlens[r+1]-1.
 *                  Empty requests are allowed (final state = initial state).
 *   cu_seqlens_host optional HOST copy of cu_seqlens (may be NULL).  When
 *                  given, the host validates it and schedules the longest
 *                  requests first; when NULL, requests are scheduled in index
 *                  order.  Results are identical either way.
 *   initial_state  [n_req, H, dk, dv] fp32 or NULL (zeros).
 *   o              [T_total, H, dv] out_dtype; must not be NULL.
 *   final_state    [n_req, H, dk, dv] fp32 or NULL (not written).  May alias
 *                  initial_state exactly (in-place update); no other overlap
 *                  between outputs and inputs is allowed.
 *   snapshot_stride 0 (no snapshots) or a positive multiple of 64 (512 in
 *                  the standard workloads).
 *   cu_snapshots   DEVICE int32 [n_req + 1] when snapshot_stride > 0:
 *                  cu_snapshots[0] == 0 and cu_snapshots[r+1] - cu_snapshots[r]
 *                  == floor(L_r / snapshot_stride) (see kda_snapshot_count).
 *   snapshots      [cu_snapshots[n_req], H, dk, dv] fp32 when
 *                  snapshot_stride > 0.  Snapshot j (1-based) of request r is
 *                  the state after the request's first j*snapshot_stride
 *                  tokens, stored at row cu_snapshots[r] + j - 1.  When L_r is
 *                  a multiple of the stride the last snapshot equals the
 *                  final state.
 *   g_logits       fused gate activation: NULL, or bf16 [T_total, H, dk] gate
 *                  logits x with g == NULL.  The kernels then use
 *                  log(alpha) = -5 * sigmoid(x), computed in fp32 as the tiles
 *                  are loaded: the lower-bounded decay (CSDN post on the Kimi
 *                  K3 technical report, section 一.1), alpha >= exp(-5) for
 *                  every x, with half the gate bytes of fp32 g and no range
 *                  precondition.
 */
typedef struct kda_prefill_args {
  int32_t n_req;
  int32_t total_tokens;
  int32_t H, dk, dv;
  kda_dtype in_dtype;
  kda_dtype out_dtype;
  const void *q, *k, *v;
  const float *g;
  const float *beta;
  const int32_t *cu_seqlens;
  const int32_t *cu_seqlens_host;
  const float *initial_state;
  void *o;
  float *final_state;
  int32_t snapshot_stride;
  const int32_t *cu_snapshots;
  float *snapshots;
  const void *g_logits;
} kda_prefill_args;

/* Bytes of device workspace kda_prefill_chunked needs for these arguments
 * (a multiple of 256; 0 is possible).  Host computation (it reads the current
 * device's SM count); returns 0 for invalid arguments (kda_prefill_chunked then
 * reports the error).  When the call would be split (see below) this is the
 * split's workspace: the segment tables and three fp32 states per segment and
 * head, for example 19 MB for one 8,192-token request with H = 32, d = 128. */
size_t kda_prefill_workspace_size(const kda_prefill_args *args);

/* Run chunked prefill.  workspace: device memory of at least
 * kda_prefill_workspace_size(args) bytes, 256-byte aligned, owned by the
 * caller and not used concurrently by another call; workspace_bytes: its
 * size.  Returns KDA_OK once the work is enqueued on `stream`.
 *
 * Few chains.  A (request, head) chain runs its chunks in order on one SM, so
 * a call with few chains leaves most SMs idle.  When the tensor-core kernel
 * runs, cu_seqlens_host is given, the chains fill at most half of the SMs and
 * some request is long enough (segments of at least 1,024 tokens, starting on
 * multiples of 32 or of snapshot_stride), the call is split the way KDA
 * context parallelism splits a sequence ("Kimi K3 开源日来了", Infra section,
 * first layer): every split request's first segment from its initial state
 * (on a second stream of the library's, forked from and joined to `stream`)
 * beside the local states and transitions of the middle segments
 * (kda_chunk_local_state), an exact combine per request (kda_state_combine)
 * from the first segment's final state, then every other segment from its
 * start state.  o, the snapshots and the final
 * states equal the unsplit call's up to rounding (not bit for bit); the call
 * then also makes small host-to-device copies of its segment tables from
 * pageable memory, which a CUDA graph capture does not accept.  The split is
 * skipped when the workspace is smaller than kda_prefill_workspace_size asks
 * for (the call then needs only the unsplit workspace), and when the
 * environment variable KDA_NO_SPLIT is set to a non-zero value. */
kda_status kda_prefill_chunked(const kda_prefill_args *args, void *workspace,
                               size_t workspace_bytes, void *stream);

/* Segments the call would run after the context-parallel split described
 * above, 0 when it would not be split.  Host computation, like
 * kda_prefill_workspace_size. */
int32_t kda_prefill_split_segments(const kda_prefill_args *args);

/* Largest n_req that kda_prefill_chunked_noalloc accepts. */
#define KDA_NOALLOC_MAX_REQUESTS 16384

/*
 * Allocation-free variant of kda_prefill_chunked.  The pages have no
 * counterpart to this entry point; it exists for callers that cannot hand
 * the library a device workspace, for example:
 *   - an inference engine that reserves all device memory for its own pools
 *     at start-up and has no buffer to spare for a plug-in kernel;
 *   - a custom-op or plug-in host whose interface gives the op no way to
 *     request scratch memory;
 *   - latency-critical code that cannot call cudaMalloc, which may
 *     synchronise the device and take milliseconds.
 *
 * Same arguments, results and error codes as kda_prefill_chunked, never
 * split (its scratch has no room for segment states), and except
 * that the scratch (one int32 per request: the longest-first work order)
 * lives in a fixed array inside libkda.so instead of a caller workspace:
 *   - the array holds KDA_NOALLOC_MAX_REQUESTS int32 (64 KiB) and is resident
 *     on every GPU that loads the library until the process exits;
 *   - n_req > KDA_NOALLOC_MAX_REQUESTS returns KDA_ERR_WORKSPACE and launches
 *     nothing;
 *   - the first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current, and so does the first
 *     call after the device's context changes (cudaDeviceReset); make that
 *     first call before any stream capture.  The lookup is guarded by a
 *     lock, so first calls from several host threads are safe;
 *   - every call on a device shares the one array, which keeps the last
 *     call's contents.  Nothing in it needs to start at zero: each call
 *     rewrites entries 0 .. n_req-1 before reading them.  Calls that overlap
 *     on the GPU (for example on two streams of the same device) race on the
 *     array, so serialise them;
 *   - it calls no cudaMalloc, cudaFree or other allocating routine.
 */
kda_status kda_prefill_chunked_noalloc(const kda_prefill_args *args, void *stream);

/* ------------------------------------------------------------------------ */
/* Context-parallel split of one long sequence into segments.               */
/* ------------------------------------------------------------------------ */

/*
 * Arguments of kda_chunk_local_state.
 *
 * Source: KDA context parallelism ("Kimi K3 开源日来了", Infra section, first
 * layer; also section 三.1 of the CSDN post): a segment's effect on the state
 * splits into (i) the state the segment produces from a zero start and (ii)
 * the linear map it applies to whatever state enters it.  Both are computed
 * locally per segment; kda_state_combine then recovers every segment's true
 * start state exactly.  Per segment s and head h:
 *
 *     S_loc[s] = state after the segment's tokens starting from S = 0
 *     M[s]     = A_L ... A_2 A_1,   A_t = (I - beta_t k_t k_t^T) Diag(alpha_t)
 *
 * so that running the segment from any start state X gives M[s] X + S_loc[s].
 *
 *   n_seg          number of segments, >= 1.
 *   total_tokens   T_total = seg_cu[n_seg].
 *   H, dk, dv      as for prefill (dk == dv in {64, 128}).
 *   in_dtype       dtype of k, v.
 *   k              [T_total, H, dk];  v [T_total, H, dv];  g [T_total, H, dk] fp32;
 *   beta           [T_total, H] fp32 -- same layouts and preconditions as prefill.
 *   seg_cu         DEVICE int32 [n_seg + 1] segment token offsets (0 first,
 *                  non-decreasing).
 *   seg_cu_host    optional HOST copy (may be NULL), used only for validation.
 *   s_loc          [n_seg, H, dk, dv] fp32 output.
 *   m              [n_seg, H, dk, dk] fp32 output (row-major: m[.., i, j]).
 *   g_logits       as in kda_prefill_args: bf16 gate logits instead of g
 *                  (then g == NULL).
 */
typedef struct kda_local_state_args {
  int32_t n_seg;
  int32_t total_tokens;
  int32_t H, dk, dv;
  kda_dtype in_dtype;
  const void *k, *v;
  const float *g;
  const float *beta;
  const int32_t *seg_cu;
  const int32_t *seg_cu_host;
  float *s_loc;
  float *m;
  const void *g_logits;
} kda_local_state_args;

size_t kda_local_state_workspace_size(const kda_local_state_args *args);
kda_status kda_chunk_local_state(const kda_local_state_args *args, void *workspace,
                                 size_t workspace_bytes, void *stream);

/*
 * Combine of the per-segment results: the "one exchange among all ranks" of
 * KDA context parallelism ("Kimi K3 开源日来了", Infra section, first layer),
 * done here on one device as an exact serial scan over segments:
 *
 *     S_in[0] = S_init (zeros if NULL),  S_in[s+1] = M[s] S_in[s] + S_loc[s],
 *     S_final = S_in[n_seg].
 *
 *   s_loc  [n_seg, H, dk, dv] fp32;  m [n_seg, H, dk, dk] fp32  (inputs)
 *   s_init [H, dk, dv] fp32 or NULL
 *   s_in   [n_seg, H, dk, dv] fp32 output: each segment's true start state
 *          (feed it to kda_prefill_chunked as initial_state, one request per
 *          segment).  May be NULL.
 *   s_final [H, dk, dv] fp32 output or NULL.
 * Outputs must not overlap inputs.  dk == dv in {64, 128}.
 */
kda_status kda_state_combine(const float *s_loc, const float *m, const float *s_init,
                             int32_t n_seg, int32_t H, int32_t dk, int32_t dv,
                             float *s_in, float *s_final, void *stream);

/* ------------------------------------------------------------------------ */
/* Decode: one new token per request against its fixed-size state.          */
/* ------------------------------------------------------------------------ */

/*
 * Arguments of kda_decode_step.
 *
 * Source: KDA keeps one fixed-size recurrent state per request, unlike the
 * MLA KV cache that grows with the conversation ("Kimi K3 开源日来了", Infra
 * section, second layer).  One call advances every listed request by one
 * token:  S <- (I - beta k k^T) Diag(alpha) S + beta k v^T,  o = S^T q.
 *
 *   n              number of requests this step, >= 0.
 *   H, dk, dv      dk == dv in {64, 128}.
 *   in_dtype       dtype of q, k, v;  out_dtype: dtype of o.
 *   q, k           [n, H, dk];  v [n, H, dv];  g [n, H, dk] fp32;  beta [n, H] fp32.
 *   state          [n_slots, H, dk, dv] fp32 state pool, updated IN PLACE.
 *   n_slots        number of states in the pool (>= n when slot == NULL).
 *   slot           DEVICE int32 [n] or NULL: request i uses state slot[i]
 *                  (values in [0, n_slots), pairwise distinct -- duplicates
 *                  race).  NULL means slot i for request i.
 *   o              [n, H, dv] out_dtype.
 */
typedef struct kda_decode_args {
  int32_t n;
  int32_t H, dk, dv;
  kda_dtype in_dtype;
  kda_dtype out_dtype;
  const void *q, *k, *v;
  const float *g;
  const float *beta;
  float *state;
  int32_t n_slots;
  const int32_t *slot;
  void *o;
} kda_decode_args;

kda_status kda_decode_step(const kda_decode_args *args, void *stream);

/* ------------------------------------------------------------------------ */
/* Backward (training): gradients of the chunked prefill.                   */
/* ------------------------------------------------------------------------ */

/*
 * Arguments of kda_prefill_backward.
 *
 * Source: FlashKDA also speeds up training ("Kimi K3 开源日来了", FlashKDA
 * section), which needs the derivative of the same prefill map.  For the
 * inputs of a kda_prefill_chunked call, this computes the gradients of
 *
 *     L = sum(d_o * o) + sum(d_final * final_state)
 *
 * with respect to q, k, v, g (= log alpha), beta and the initial state, where
 * (o, final_state) is what kda_prefill_chunked returns for those inputs.
 * Snapshots take no cotangent.  The chunk-start states are recomputed by a
 * forward pass inside the call; nothing from an earlier forward is needed.
 *
 *   n_req, total_tokens, H, dk, dv, in_dtype, q, k, v, g, beta, cu_seqlens,
 *   initial_state   as in kda_prefill_args (dk == dv in {64, 128}).
 *   cu_seqlens_host HOST int32 [n_req + 1], REQUIRED: it sizes the workspace
 *                   and the chunk table.  Same values as cu_seqlens.
 *   d_o             fp32 [total_tokens, H, dv] or NULL (zero cotangent).
 *   d_final         fp32 [n_req, H, dk, dv] or NULL (zero cotangent).
 *   d_q, d_k, d_g   fp32 [total_tokens, H, dk] outputs: gradients of q, k, g.
 *   d_v             fp32 [total_tokens, H, dv] output: gradient of v.
 *   d_beta          fp32 [total_tokens, H] output: gradient of beta.
 *   d_initial       fp32 [n_req, H, dk, dv] output, or NULL (not returned).
 *   g_logits        as in kda_prefill_args: bf16 gate logits x instead of g
 *                   (then g == NULL).  d_g then receives dL/dx, the gradient
 *                   of the logits: dL/dg * (-5) sigmoid(x) (1 - sigmoid(x)).
 * Outputs must not overlap each other, the inputs or the workspace.  The
 * workspace (kda_prefill_backward_workspace_size bytes, 256-byte aligned) is
 * scratch owned by the caller for the duration of the call.  The host tables
 * are copied into the workspace before the call returns, so cu_seqlens_host
 * may be freed afterwards.
 */
typedef struct kda_backward_args {
  int32_t n_req;
  int32_t total_tokens;
  int32_t H, dk, dv;
  kda_dtype in_dtype;
  const void *q, *k, *v;
  const float *g;
  const float *beta;
  const int32_t *cu_seqlens;
  const int32_t *cu_seqlens_host;
  const float *initial_state;
  const float *d_o;
  const float *d_final;
  float *d_q, *d_k, *d_v, *d_g, *d_beta;
  float *d_initial;
  const void *g_logits;
} kda_backward_args;

/* Workspace bytes for kda_prefill_backward (0 if the arguments are invalid). */
size_t kda_prefill_backward_workspace_size(const kda_backward_args *args);
kda_status kda_prefill_backward(const kda_backward_args *args, void *workspace,
                                size_t workspace_bytes, void *stream);

/* ------------------------------------------------------------------------ */
/* Prefix cache over state snapshots (serving).                             */
/* ------------------------------------------------------------------------ */

/*
 * Source: the serving cache keeps sparse state snapshots at 512-token block
 * boundaries, and a request whose prompt starts with a cached prefix resumes
 * from the longest one ("Kimi K3 开源日来了", Infra section, second layer).
 * The state after a prefix depends only on the prefix, so the cache maps
 * prompt prefixes that end on a block boundary to states.
 *
 * kda_prefix_cache is a HOST index (no device memory of its own): the chained
 * 64-bit FNV-1a hash of a prompt's first j blocks of token ids (block j hashed
 * over the hash of block j-1, 0 before the first, and its ids, little-endian)
 * maps to a slot of a caller-owned device state pool [n_slots, H, dk, dv]
 * fp32.  Each entry keeps its parent's hash and its block's ids, and lookups
 * compare both, so a hash collision cannot return another prompt's state.
 * When every slot is taken, an insert evicts the least recently used entry;
 * lookups and inserts refresh the blocks they walk, deepest first, so a
 * chain's leading blocks are evicted last.  Calls on one cache are serialised
 * by an internal lock.  A slot returned by a lookup holds its state until a
 * later insert evicts it: enqueue the copy out of the pool (kda_state_gather)
 * before the next insert's copies into it, on the same stream.
 *
 * Typical resume of one request with prompt ids t[0..n):
 *   m = kda_prefix_cache_lookup(c, t, n, n - 1, &slot);   (keep >= 1 token)
 *   kda_state_gather(pool, n_slots, &slot, 1, ...) -> initial state;
 *   prefill tokens m..n from it with snapshot_stride = block_tokens;
 *   kda_prefix_cache_insert(c, t, n, m / block_tokens, slots_out), then
 *   kda_state_scatter of snapshot j - m / block_tokens into slots_out[j].
 */
typedef struct kda_prefix_cache kda_prefix_cache;

/* New empty cache of n_slots states, keyed by blocks of block_tokens ids
 * (512 in the standard workloads).  NULL if an argument is <= 0 or memory runs
 * out.  Release it with kda_prefix_cache_destroy. */
kda_prefix_cache *kda_prefix_cache_create(int32_t block_tokens, int32_t n_slots);
void kda_prefix_cache_destroy(kda_prefix_cache *cache);

/* Longest cached prefix of tokens[0..n_tokens) that ends on a block boundary
 * and is at most max_tokens long.  Returns its length in tokens (a multiple of
 * block_tokens, 0 for none) and writes the slot holding the state after it
 * to *slot (-1 for none); -1 on invalid arguments.  tokens: HOST int32. */
int32_t kda_prefix_cache_lookup(kda_prefix_cache *cache, const int32_t *tokens,
                                int32_t n_tokens, int32_t max_tokens, int32_t *slot);

/* Registers the complete blocks of tokens[0..n_tokens) (HOST int32).
 * slots_out (HOST int32 [n_tokens / block_tokens]) receives, for block j
 * (0-based), the slot the caller must fill with the state after tokens
 * [0, (j+1) * block_tokens), or -1 when nothing is to be written (the block
 * was cached already, or was not registered).  Blocks before first_block must
 * be cached already (their states are not at hand): the walk stops at the
 * first one that is not.  The walk also stops when the only slot left to
 * evict belongs to this prompt.  Returns how many leading blocks are cached
 * afterwards, or -1 on invalid arguments. */
int32_t kda_prefix_cache_insert(kda_prefix_cache *cache, const int32_t *tokens,
                                int32_t n_tokens, int32_t first_block, int32_t *slots_out);

/* Number of cached blocks (-1 for a NULL cache). */
int32_t kda_prefix_cache_size(const kda_prefix_cache *cache);

/* Device copies between the state pool [n_slots, H, dk, dv] fp32 and dense
 * states [n, H, dk, dv] fp32.  slots: DEVICE int32 [n].
 *   gather:  dst[i] = pool[slots[i]], zeros where slots[i] < 0;
 *   scatter: pool[slots[i]] = src[i] where slots[i] >= 0.
 * All pointers 16-byte aligned; the pool must not overlap dst / src.  A slot
 * >= n_slots copies nothing and is reported through the device status word
 * (KDA_ERR_INVALID_ARG from kda_get_device_status).  Asynchronous on stream. */
kda_status kda_state_gather(const float *pool, int32_t n_slots, const int32_t *slots,
                            int32_t n, int32_t H, int32_t dk, int32_t dv, float *dst,
                            void *stream);
kda_status kda_state_scatter(const float *src, const int32_t *slots, int32_t n, int32_t H,
                             int32_t dk, int32_t dv, float *pool, int32_t n_slots,
                             void *stream);

/* ------------------------------------------------------------------------ */
/* Helpers.                                                                 */
/* ------------------------------------------------------------------------ */

/* floor(len / stride): snapshots a request of `len` tokens gets (0 if stride <= 0). */
int32_t kda_snapshot_count(int32_t len, int32_t stride);

/* Synchronises `stream`, then reads and clears the device status word of the
 * current device.  Returns KDA_OK, KDA_ERR_GATE_RANGE, KDA_ERR_TIMEOUT or
 * KDA_ERR_CUDA (the synchronisation itself failed). */
kda_status kda_get_device_status(void *stream);

/* Static, human-readable name of a status code. */
const char *kda_status_string(kda_status status);

/* KDA_VERSION of the loaded library. */
int32_t kda_version(void);

/* 1 if kda_prefill_chunked serves these head dims and input dtype with the
 * tensor-core (tcgen05) kernel, 0 if with the SIMT fp32 kernel.  The
 * environment variable KDA_FORCE_SIMT=1 forces the SIMT kernel (and makes
 * this return 0).  Both kernels compute the same result up to rounding. */
int32_t kda_prefill_uses_tensor_cores(int32_t dk, int32_t dv, kda_dtype in_dtype);

#ifdef __cplusplus
}
#endif

#endif /* KDA_H_ */
