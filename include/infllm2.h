/*
 * libinfllm2 — InfLLM-V2 sparse-attention forward path for grouped-query
 * attention on NVIDIA B200 (sm_100a).  C ABI.
 *
 * The method (InfLLM-V2: dense-sparse switchable attention) is described on
 * these pages, cited below by their titles:
 *   [blog]   "论文阅读：InfLLM-V2 — 把可训练稀疏注意力做成全注意力的'受限版本'"
 *            (xiaohongrsx.github.io paper-reading notes)
 *   [news]   "从密集到稀疏：InfLLM-V2 如何实现零参数开销的长文本高效处理" (dtcms.com)
 *   [top168] top168.com article on InfLLM-V2 (Tsinghua / OpenBMB,
 *            arXiv 2509.24663), sections 三, 四, 七
 *
 * Data layout (all calls).
 *   Sequences are packed token-major ("THD"): Q [total, h_q, d],
 *   K and V [total, h_kv, d], bf16, row-major, contiguous in d.  Sequence s
 *   holds rows cu_seqlens[s] .. cu_seqlens[s+1]-1.  Blocks (64 tokens) and
 *   pooling windows restart at every sequence start.  Query head h belongs
 *   to kv group h / (h_q / h_kv).  d is 64 or 128; h_q % h_kv == 0 and
 *   G = h_q / h_kv is a power of two <= 16.  Every device pointer must be
 *   16-byte aligned.
 *
 * Ownership.  The caller allocates every buffer (workspaces included) and
 * keeps ownership; no call allocates or frees device memory, none
 * synchronises the stream, and no pointer is kept after a call returns.
 * Calls are asynchronous on the given stream (a cudaStream_t passed as
 * void*; NULL is the legacy default stream).
 *
 * Errors.  Every call returns INFLLM2_OK (0) or a negative INFLLM2_ERR_*
 * code.  Arguments are checked before anything is launched; on an argument
 * error nothing is written.  INFLLM2_ERR_CUDA means a launch failed (the
 * CUDA error text is kept for infllm2_status_string).  Kernels that detect a
 * problem on the device (a bounded wait that ran out, an index out of range)
 * record it in a per-device status word instead of trapping; read it with
 * infllm2_get_device_status after synchronising.
 */
#ifndef INFLLM2_H_
#define INFLLM2_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
  INFLLM2_OK = 0,
  INFLLM2_ERR_INVALID_ARG = -1,        /* null pointer, bad size, misalignment */
  INFLLM2_ERR_UNSUPPORTED = -2,        /* valid but not implemented (d, G, params) */
  INFLLM2_ERR_WORKSPACE_TOO_SMALL = -3,
  INFLLM2_ERR_CUDA = -4,               /* a CUDA runtime call or launch failed */
  INFLLM2_ERR_DEVICE_TIMEOUT = -5,     /* device status: a bounded wait ran out */
  INFLLM2_ERR_DEVICE_BOUNDS = -6       /* device status: an index check failed */
};

enum { INFLLM2_OUT_BF16 = 0, INFLLM2_OUT_F32 = 1 };
/* lse_mode: APPROX takes each head's log-sum-exp from the coarse C2 scores
 * (the pages' approximation, 1.25x the cost of one scoring pass); EXACT
 * takes it from the C1 scores themselves (the two-pass computation it
 * replaces, 2x; each row of S then sums to G).  [top168] §四. */
enum { INFLLM2_LSE_APPROX = 0, INFLLM2_LSE_EXACT = 1 };

/* Method parameters.  Defaults (infllm2_default_params) are the pages'
 * values: block B = 64 ([blog] worked example "每块 64 个 token");
 * stage-1 windows l_C1 = B/2 = 32, s_C1 = B/4 = 16 and stage-3 max-pool
 * kernel 5, stride 4 ([top168] §三); coarse windows for the LSE approximation
 * l_C2 = 4 l_C1 = 128, s_C2 = 4 s_C1 = 64 ([top168] §四); 1 initial block,
 * 32 local blocks and 63 top-k blocks, |I| = 96 ([blog] worked example).
 * The kernels implement exactly these pooling geometries; any other value of
 * block_size, c1_*, c2_*, pool_* returns INFLLM2_ERR_UNSUPPORTED.  n_init,
 * n_local (>= 1) and top_k are free (|I| = n_init + n_local + top_k <= 4096). */
typedef struct {
  int32_t block_size;      /* B = 64 */
  int32_t c1_len;          /* 32 */
  int32_t c1_stride;       /* 16 */
  int32_t c2_len;          /* 128 */
  int32_t c2_stride;       /* 64 */
  int32_t pool_len;        /* 5 */
  int32_t pool_stride;     /* 4 */
  int32_t pool_pad;        /* 1 */
  int32_t n_init;          /* 1 */
  int32_t n_local;         /* 32, includes the query's own block */
  int32_t top_k;           /* 63 */
  float scale;             /* softmax scale; <= 0 selects 1/sqrt(d) */
  int32_t lse_mode;        /* INFLLM2_LSE_APPROX */
  int32_t dense_threshold; /* 8192: sequences of at most this length take the dense path */
} infllm2_params;

/* Packed variable-length batch geometry.  cu_seqlens is a DEVICE array of
 * batch+1 int32 offsets (cu_seqlens[0] = 0, cu_seqlens[batch] = total);
 * the other fields are host values: max_seqlen = longest sequence, total =
 * number of packed tokens, total_c1 / total_c2 = number of pooled rows
 * (the sum over sequences of infllm2_window_count(len, 32, 16) and
 * infllm2_window_count(len, 128, 64)); these are the row capacities of the
 * pooled-key buffers. */
typedef struct {
  const int32_t* cu_seqlens;
  int32_t batch;
  int32_t max_seqlen;
  int64_t total;
  int64_t total_c1;
  int64_t total_c2;
} infllm2_varlen;

infllm2_params infllm2_default_params(void);
const char* infllm2_status_string(int status);

/* Number of complete pooling windows of `len` tokens taken every `stride`
 * tokens inside a sequence of n tokens (partial windows are dropped). */
int64_t infllm2_window_count(int64_t n, int32_t len, int32_t stride);

/* Leading dimension (floats) of the S_shared rows for this batch:
 * max window count rounded up to a multiple of 4. */
int64_t infllm2_scores_ld(const infllm2_varlen* vl, const infllm2_params* p);

/* ---------------------------------------------------------------------
 * Step 1: stage-1 and coarse mean pooling of K  ([top168] §三 first stage,
 * §四 coarse scores S_C2).  For each sequence and kv head g:
 *   K_c1[g, c1_off(s) + j] = bf16_rne(mean(K[16j .. 16j+31, g]))  j < n_c1(len)
 *   K_c2[g, c2_off(s) + m] = bf16_rne(mean(K[64m .. 64m+127, g])) m < n_c2(len)
 * where c1_off(s) is the number of C1 windows of the sequences before s.
 * The mean is exact (fp64 sum) before the single rounding to bf16.
 *   K     bf16 [total, h_kv, d]                  (input)
 *   K_c1  bf16 [h_kv, total_c1, d]               (output)
 *   K_c2  bf16 [h_kv, total_c2, d]               (output)
 * ------------------------------------------------------------------- */
int infllm2_compress_k(const void* K, const infllm2_varlen* vl, int32_t h_kv, int32_t d,
                       void* K_c1, void* K_c2, const infllm2_params* p, void* stream);

/* ---------------------------------------------------------------------
 * Step 2: compressed scores with the LSE approximation and the fused
 * head-group sum ([top168] §三 second stage, §四).  For query token t of a
 * sequence and kv group g, with s_h(j) = scale * q[t,h] . K_c1[g,j]:
 *   LSE_h  = log sum_{m visible} exp(scale * q[t,h] . K_c2[g,m])
 *   S[g, t, j] = sum_{h in group g} exp(s_h(j) - LSE_h)   for visible j
 * A C1 window j is visible when 16j+31 <= t, a C2 window m when 64m+127 <= t
 * (positions within the sequence).  Rows with no visible C2 window
 * (t < 127) take the exact log-sum-exp over their visible C1 windows.
 * With p->lse_mode == INFLLM2_LSE_EXACT, LSE_h is the log-sum-exp of s_h
 * over the visible C1 windows for every row.
 * Only visible entries are written; the per-head scores never reach HBM.
 *   Q          bf16 [total, h_q, d]
 *   K_c1, K_c2 as written by infllm2_compress_k
 *   S          fp32 [h_kv, total, ld], ld = infllm2_scores_ld(vl, p)
 * ------------------------------------------------------------------- */
int infllm2_shared_scores(const void* Q, const void* K_c1, const void* K_c2,
                          const infllm2_varlen* vl, int32_t h_q, int32_t h_kv, int32_t d,
                          float* S, int64_t ld, const infllm2_params* p, void* stream);

/* ---------------------------------------------------------------------
 * Step 3: stage-3 max-pool and block selection ([top168] §三 third stage,
 * §七; [blog] worked example).  For query token t (block b_t = t / 64):
 *   score(b) = max{ S[g,t,j] : 4b-1 <= j <= 4b+3, j visible }
 *   I = {0..n_init-1} U {b_t-n_local+1 .. b_t} U top_k of the remaining
 *       blocks 0..b_t by score (ties go to the lower block index),
 * clipped to [0, b_t]; listed ascending, padded with -1.
 *   S          fp32 [h_kv, total, ld]
 *   block_idx  int32 [h_kv, total, n_init+n_local+top_k]   (output)
 * ------------------------------------------------------------------- */
int infllm2_topk_blocks(const float* S, int64_t ld, const infllm2_varlen* vl, int32_t h_kv,
                        int32_t* block_idx, const infllm2_params* p, void* stream);

/* ---------------------------------------------------------------------
 * Steps 2 and 3 with the first step of the max-pool fused into the score
 * kernel ([top168] §三 third stage; S_shared itself is not written).  For
 * query token t and each group of four C1 windows 4i .. 4i+3 whose first
 * window is visible, the score kernel writes the pair
 *   P[g, t, 2i]   = max{ S[g,t,j] : 4i <= j <= 4i+3, j visible }
 *   P[g, t, 2i+1] = S[g,t,4i+3] if visible, else -inf
 * (S as defined for infllm2_shared_scores; entries of groups with no visible
 * window are not written), so that
 *   score(b) = max(P[g,t,2b], P[g,t,2b-1])      (the second term for b >= 1)
 * equals infllm2_topk_blocks' score(b) bit for bit, and
 * infllm2_topk_blocks_pooled returns the same lists.  The pairs take half
 * the bytes of S_shared.
 *   P          fp32 [h_kv, total, ldp], ldp = infllm2_pooled_ld(vl, p)
 *              (2 * ceil(max window count / 4), rounded up to a multiple of 4)
 * Arguments, errors and the other buffers as for infllm2_shared_scores and
 * infllm2_topk_blocks.
 * ------------------------------------------------------------------- */
int64_t infllm2_pooled_ld(const infllm2_varlen* vl, const infllm2_params* p);
int infllm2_pooled_scores(const void* Q, const void* K_c1, const void* K_c2,
                          const infllm2_varlen* vl, int32_t h_q, int32_t h_kv, int32_t d,
                          float* P, int64_t ldp, const infllm2_params* p, void* stream);
int infllm2_topk_blocks_pooled(const float* P, int64_t ldp, const infllm2_varlen* vl, int32_t h_kv,
                               int32_t* block_idx, const infllm2_params* p, void* stream);

/* Steps 2 and 3 in one call.  S_shared goes to `workspace` (at least
 * infllm2_select_workspace_bytes bytes) unless s_shared_out is non-NULL, in
 * which case it is written there ([h_kv, total, ld] fp32) and the workspace
 * may be NULL. */
size_t infllm2_select_workspace_bytes(const infllm2_varlen* vl, int32_t h_kv, const infllm2_params* p);
int infllm2_select_blocks(const void* Q, const void* K_c1, const void* K_c2,
                          const infllm2_varlen* vl, int32_t h_q, int32_t h_kv, int32_t d,
                          void* workspace, size_t workspace_bytes, int32_t* block_idx,
                          float* s_shared_out, const infllm2_params* p, void* stream);

/* Allocation-free variant of infllm2_select_blocks.  The paper has no
 * counterpart: this is a convenience of this library for callers that cannot
 * allocate device memory when they select blocks (code running inside a
 * custom allocator or memory pool, plugins whose host owns every device
 * allocation, paths that must not call cudaMalloc because it can
 * synchronise the device).  Same arguments and results as
 * infllm2_select_blocks, without a workspace: S_shared is kept in a
 * fixed array of INFLLM2_NOALLOC_SCRATCH_BYTES in the library's device
 * memory, held on every GPU that loads the library until the process exits.
 *   - Problems whose S_shared (h_kv * total * ld floats, ld =
 *     infllm2_scores_ld) exceeds the array return
 *     INFLLM2_ERR_WORKSPACE_TOO_SMALL before anything is launched.
 *   - Every call looks up the array's device address on the current
 *     device (cudaGetSymbolAddress, which allocates nothing); the first call
 *     on a device is also the one that sets the array up there, so make that
 *     first call before any stream capture.
 *   - Every call uses the same array: calls whose kernels can overlap on the
 *     GPU race on it.  It keeps the last call's scores; none of it needs to
 *     start at zero.
 *   - It calls no cudaMalloc, cudaFree or other allocating routine. */
#define INFLLM2_NOALLOC_SCRATCH_BYTES (64u << 20)
int infllm2_select_blocks_noalloc(const void* Q, const void* K_c1, const void* K_c2,
                                  const infllm2_varlen* vl, int32_t h_q, int32_t h_kv, int32_t d,
                                  int32_t* block_idx, const infllm2_params* p, void* stream);

/* ---------------------------------------------------------------------
 * Step 4: block-sparse causal attention ([blog] "对齐计算图": selected and
 * sliding attention merged into one sparse attention with a single output;
 * [top168] §七).  For token t of a sequence and query head h of group g:
 *   out[t,h] = softmax_u(scale * q[t,h] . K[u,g]) V[u,g]
 * over u <= t with u / 64 in block_idx[g, t, :] (entries < 0 ignored).
 *   out  [total, h_q, d], bf16 (INFLLM2_OUT_BF16) or fp32 (INFLLM2_OUT_F32)
 * Each row of block_idx must be ascending (valid entries first, then -1)
 * and must hold the row's init blocks (0 .. min(n_init, b_t + 1) - 1) and
 * its local run (the n_local blocks ending at b_t = t / 64), as every list
 * of infllm2_select_blocks / infllm2_topk_blocks does: the shared init and
 * local blocks are attended once per group of query tokens and the other
 * entries per token, and the two partials are merged.  A row that breaks
 * this rule (also: entries out of [0, b_t], repeated, unsorted, or valid
 * entries after a -1) is detected on the device and recorded in the device
 * status word as INFLLM2_ERR_DEVICE_BOUNDS; its output is then undefined
 * (no fault, no out-of-range read).
 * workspace: device, 16-byte aligned, at least
 * infllm2_sparse_workspace_bytes(vl, h_q) bytes (one fp32 per (token,
 * query head)).  When the call's kernels have completed, its first
 * total * h_q floats hold, for every token row t and query head h (index
 * t * h_q + h), the row's log-sum-exp in log2 units over the keys it
 * attended: lse = log2 sum_u 2^(scale * log2(e) * q[t,h] . K[u,g]) — the
 * statistic infllm2_sparse_attn_backward takes.
 * ------------------------------------------------------------------- */
size_t infllm2_sparse_workspace_bytes(const infllm2_varlen* vl, int32_t h_q);
int infllm2_sparse_attn(const void* Q, const void* K, const void* V, const int32_t* block_idx,
                        const infllm2_varlen* vl, int32_t h_q, int32_t h_kv, int32_t d,
                        void* out, int32_t out_dtype, void* workspace, size_t workspace_bytes,
                        const infllm2_params* p, void* stream);

/* ---------------------------------------------------------------------
 * Backward of step 4: gradients of the block-sparse attention over a fixed
 * selection (the method trains the sparse attention end to end with no added
 * parameters: [news] §二, [top168] §一; [blog] "训练是怎么做的").  The block
 * lists carry no gradient.  For row (t, h) of kv group g and its attended
 * keys u (those infllm2_sparse_attn attends), with P = softmax_u(scale *
 * q[t,h] . K[u,g]) and dS = P * (dO[t,h] . V[u,g] - sum_d dO[t,h] * out[t,h]):
 *   dQ[t,h] = scale * sum_u dS K[u,g]
 *   dK[u,g] = scale * sum over rows (t,h) that attend u of dS q[t,h]
 *   dV[u,g] = sum over rows (t,h) that attend u of P dO[t,h]
 *   Q, K, V, block_idx, vl, h_q, h_kv, d, p: as given to infllm2_sparse_attn
 *   out        its output [total, h_q, d], out_dtype INFLLM2_OUT_BF16 / _F32
 *   dout       bf16 [total, h_q, d], the gradient of the loss w.r.t. out
 *   lse        fp32 [total, h_q]: the first total * h_q floats of
 *              infllm2_sparse_attn's workspace after that call (row
 *              log-sum-exps, log2 units)
 *   dQ         fp32 [total, h_q, d]   (output, every element written)
 *   dK, dV     fp32 [total, h_kv, d]  (output, every element written)
 *   workspace  device, at least infllm2_sparse_backward_workspace_bytes
 *              bytes (per-row sums, the inverse of the block lists); its
 *              contents need no initialisation and carry nothing between
 *              calls.
 * Supported: G = h_q / h_kv of 8 or 16, d of 64 or 128 (other shapes:
 * INFLLM2_ERR_UNSUPPORTED).  Lists must have the form infllm2_sparse_attn
 * requires; a list that breaks it is recorded as INFLLM2_ERR_DEVICE_BOUNDS.
 * The result does not depend on scheduling: each key block's gradient is
 * summed by one CTA over its rows in ascending token order.
 * ------------------------------------------------------------------- */
size_t infllm2_sparse_backward_workspace_bytes(const infllm2_varlen* vl, int32_t h_q, int32_t h_kv,
                                               const infllm2_params* p);
int infllm2_sparse_attn_backward(const void* Q, const void* K, const void* V, const void* out, int32_t out_dtype,
                                 const void* dout, const float* lse, const int32_t* block_idx,
                                 const infllm2_varlen* vl, int32_t h_q, int32_t h_kv, int32_t d, float* dQ, float* dK,
                                 float* dV, void* workspace, size_t workspace_bytes, const infllm2_params* p,
                                 void* stream);

/* Dense causal attention, the short-sequence side of the dense/sparse switch
 * ([blog] "Dense-Sparse Switchable Attention"; [news] §二.2.c).  Same
 * arguments and output form as infllm2_sparse_attn, all u <= t attended. */
int infllm2_dense_attn(const void* Q, const void* K, const void* V,
                       const infllm2_varlen* vl, int32_t h_q, int32_t h_kv, int32_t d,
                       void* out, int32_t out_dtype, const infllm2_params* p, void* stream);

/* ---------------------------------------------------------------------
 * Step 5: one decode step per sequence (dtcms article §二.2.b: the sparse
 * pattern serves prefill and decode alike).  The caller owns the state:
 *   k_cache, v_cache  bf16 [batch, capacity, h_kv, d]
 *   k_c1              bf16 [batch, h_kv, cap_c1, d], cap_c1 = infllm2_window_count(capacity, 32, 16)
 *   k_c2              bf16 [batch, h_kv, cap_c2, d], cap_c2 = infllm2_window_count(capacity, 128, 64)
 *   seq_len           int32 [batch] on the device: tokens already cached.
 * infllm2_decode_step appends k_new / v_new ([batch, h_kv, d]) at position
 * t = seq_len[b], pools the stage-1 window ending at t when 16 divides t+1
 * (t+1 >= 32) and the coarse window ending at t when 64 divides t+1
 * (t+1 >= 128), then computes for the query q ([batch, h_q, d]) exactly
 * row t of the prefill path (scores, max-pool, selection, sparse attention
 * over keys <= t) and writes out ([batch, h_q, d] bf16); finally
 * seq_len[b] += 1.  t must be < capacity (else the device status records
 * INFLLM2_ERR_DEVICE_BOUNDS and that sequence's step is skipped: no output,
 * seq_len[b] unchanged).  The step is three kernel launches with no host
 * synchronisation, so it can be captured in a CUDA graph.  workspace:
 * infllm2_decode_workspace_bytes (device, caller-owned, no alignment beyond
 * 16 bytes, contents need no initialisation and carry nothing from one step
 * to the next; one workspace must not serve two steps in flight at once).
 * The decode step takes the LSE approximation only (lse_mode EXACT is
 * INFLLM2_ERR_UNSUPPORTED here).
 * Capacities above 1441792 tokens (more than 22528 candidate blocks) and
 * batch * h_kv above 65535 are INFLLM2_ERR_UNSUPPORTED, and
 * infllm2_decode_workspace_bytes returns 0 for them.  The three kernels are
 * chained with programmatic dependent launch among themselves only: the
 * first waits for whatever precedes it on the stream, and the last releases
 * nothing early to what follows.  infllm2_decode_build_caches pools the seq_len[b] tokens already in
 * the cache into k_c1 / k_c2 (for a prefix written by the caller).
 * ------------------------------------------------------------------- */
typedef struct {
  void* k_cache;
  void* v_cache;
  void* k_c1;
  void* k_c2;
  int32_t* seq_len;
  int32_t batch;
  int32_t capacity;
  int32_t h_q;
  int32_t h_kv;
  int32_t d;
} infllm2_decode_state;

size_t infllm2_decode_workspace_bytes(const infllm2_decode_state* st, const infllm2_params* p);

/* The blocks each decode step selected ([top168] §三 third stage, §七: the
 * same init U local U top-k rule as infllm2_topk_blocks, applied to row t).
 * Returns the byte offset inside the decode workspace of an int32 array
 * [batch, h_kv, n_init + n_local + top_k]: for sequence b and kv group g,
 * the blocks attended by the new token, ascending, padded with -1.  The
 * array is written by infllm2_decode_step and holds the lists of the last
 * step that ran on this workspace, for every sequence whose step ran (t <
 * capacity), until the next step on the same workspace overwrites it; read
 * it after that step's kernels have completed (stream order).  The call
 * launches nothing.  Returns -1 where infllm2_decode_workspace_bytes
 * returns 0 (invalid or unsupported state or parameters). */
int64_t infllm2_decode_block_idx_offset(const infllm2_decode_state* st, const infllm2_params* p);
int infllm2_decode_build_caches(const infllm2_decode_state* st, const infllm2_params* p, void* stream);
int infllm2_decode_step(const infllm2_decode_state* st, const void* q, const void* k_new, const void* v_new,
                        void* out, void* workspace, size_t workspace_bytes, const infllm2_params* p,
                        void* stream);

/* Device status word (per device).  Returns INFLLM2_OK or the first
 * INFLLM2_ERR_DEVICE_* recorded by a kernel since the last clear.
 * Synchronises the device. */
int infllm2_get_device_status(void);
int infllm2_clear_device_status(void);

/* Diagnostic: launches one block that waits on a barrier nothing will ever
 * complete, with a bound of `limit_ns` nanoseconds; the wait gives up,
 * records INFLLM2_ERR_DEVICE_TIMEOUT in the device status word and returns.
 * Used to test the bounded-wait path without hanging a GPU. */
int infllm2_debug_wait_timeout(uint64_t limit_ns, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* INFLLM2_H_ */
