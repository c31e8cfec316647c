// libinfllm2: the C-ABI entry points declared in include/infllm2.h.
//
// The library is one translation unit (the kernel files are included
// below) so that the per-device status word has a single definition.
// Host code here checks arguments, builds TMA tensor maps and launches; it
// never allocates device memory and never synchronises a stream (except
// infllm2_get_device_status, which is documented to).
#include <math.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <mutex>

#include "sm100.cuh"

// The LOCAL part of the sparse attention and the dense path run on the kernel
// with two query tiles per CTA (pair_attn.cu); 0 selects the one-tile kernel.
#ifndef INFLLM2_PAIR_ATTN
#define INFLLM2_PAIR_ATTN 1
#endif

#include "compress.cu"
#include "score.cu"
#include "select.cu"
#include "sparse_attn.cu"
#include "dense_attn.cu"
#include "pair_attn.cu"
#include "decode.cu"
#include "backward.cu"
#include "probe.cu"
#include "../../include/infllm2_measure.h"

namespace infllm2 {

static thread_local char g_err_text[256] = "";

static int cuda_fail(cudaError_t e) {
  snprintf(g_err_text, sizeof(g_err_text), "CUDA error: %s", cudaGetErrorString(e));
  return INFLLM2_ERR_CUDA;
}

PFN_encodeTiled get_encode_tiled() {
  static PFN_encodeTiled fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_encodeTiled>(p);
  });
  return fn;
}

int num_sms() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static bool geometry_supported(const infllm2_params* p) {
  return p->block_size == 64 && p->c1_len == 32 && p->c1_stride == 16 && p->c2_len == 128 &&
         p->c2_stride == 64 && p->pool_len == 5 && p->pool_stride == 4 && p->pool_pad == 1 &&
         (p->lse_mode == INFLLM2_LSE_APPROX || p->lse_mode == INFLLM2_LSE_EXACT);
}

static int check_varlen(const infllm2_varlen* vl) {
  if (!vl || !vl->cu_seqlens || vl->batch < 1 || vl->batch > 65535 || vl->max_seqlen < 0 || vl->total < 0 ||
      vl->total_c1 < 0 || vl->total_c2 < 0 || vl->total > INT32_MAX || vl->max_seqlen > vl->total)
    return INFLLM2_ERR_INVALID_ARG;
  return INFLLM2_OK;
}

static int check_heads(int32_t h_q, int32_t h_kv, int32_t d) {
  if (h_q <= 0 || h_kv <= 0 || h_q % h_kv != 0) return INFLLM2_ERR_INVALID_ARG;
  const int G = h_q / h_kv;
  if (d != 64 && d != 128) return INFLLM2_ERR_UNSUPPORTED;
  if (G > 16 || (G & (G - 1)) != 0) return INFLLM2_ERR_UNSUPPORTED;
  return INFLLM2_OK;
}

static int check_params(const infllm2_params* p) {
  if (!p) return INFLLM2_ERR_INVALID_ARG;
  if (!geometry_supported(p)) return INFLLM2_ERR_UNSUPPORTED;
  if (p->n_init < 0 || p->n_local < 1 || p->top_k < 0) return INFLLM2_ERR_INVALID_ARG;
  if (p->n_init + p->n_local + p->top_k > 4096) return INFLLM2_ERR_UNSUPPORTED;
  return INFLLM2_OK;
}

// A single thread waits on a barrier that nothing will ever complete; the
// bounded wait gives up after limit_ns and records the timeout status.
__global__ void debug_wait_kernel(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, limit_ns);
  __syncthreads();
}

static float softmax_scale(const infllm2_params* p, int d) {
  return p->scale > 0.f ? p->scale : 1.0f / sqrtf(static_cast<float>(d));
}

}  // namespace infllm2

using namespace infllm2;

extern "C" {

infllm2_params infllm2_default_params(void) {
  infllm2_params p;
  p.block_size = 64;
  p.c1_len = 32;
  p.c1_stride = 16;
  p.c2_len = 128;
  p.c2_stride = 64;
  p.pool_len = 5;
  p.pool_stride = 4;
  p.pool_pad = 1;
  p.n_init = 1;
  p.n_local = 32;
  p.top_k = 63;
  p.scale = 0.f;
  p.lse_mode = INFLLM2_LSE_APPROX;
  p.dense_threshold = 8192;
  return p;
}

const char* infllm2_status_string(int status) {
  switch (status) {
    case INFLLM2_OK: return "ok";
    case INFLLM2_ERR_INVALID_ARG: return "invalid argument";
    case INFLLM2_ERR_UNSUPPORTED: return "unsupported configuration";
    case INFLLM2_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case INFLLM2_ERR_CUDA: return g_err_text[0] ? g_err_text : "CUDA error";
    case INFLLM2_ERR_DEVICE_TIMEOUT: return "device: a bounded wait ran out";
    case INFLLM2_ERR_DEVICE_BOUNDS: return "device: an index check failed";
    default: return "unknown status";
  }
}

int64_t infllm2_window_count(int64_t n, int32_t len, int32_t stride) {
  if (len <= 0 || stride <= 0 || n < len) return 0;
  return (n - len) / stride + 1;
}

int64_t infllm2_scores_ld(const infllm2_varlen* vl, const infllm2_params* p) {
  if (!vl || !p || vl->max_seqlen < 0) return 0;
  const int64_t n1 = infllm2_window_count(vl->max_seqlen, p->c1_len, p->c1_stride);
  return std::max<int64_t>(4, (n1 + 3) & ~int64_t(3));
}

int infllm2_compress_k(const void* K, const infllm2_varlen* vl, int32_t h_kv, int32_t d, void* K_c1, void* K_c2,
                       const infllm2_params* p, void* stream) {
  int r;
  if ((r = check_varlen(vl)) || (r = check_params(p))) return r;
  if (!K || !K_c1 || !K_c2 || !aligned16(K) || !aligned16(K_c1) || !aligned16(K_c2)) return INFLLM2_ERR_INVALID_ARG;
  if (h_kv <= 0) return INFLLM2_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return INFLLM2_ERR_UNSUPPORTED;
  cudaError_t e = launch_compress_k(K, vl->cu_seqlens, vl->batch, vl->max_seqlen, h_kv, d, K_c1, vl->total_c1,
                                    K_c2, vl->total_c2, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? INFLLM2_OK : cuda_fail(e);
}

static int scores_common(const void* Q, const void* K_c1, const void* K_c2, const infllm2_varlen* vl, int32_t h_q,
                         int32_t h_kv, int32_t d, float* S, int64_t ld, int64_t ld_min, bool pool,
                         const infllm2_params* p, void* stream) {
  int r;
  if ((r = check_varlen(vl)) || (r = check_params(p)) || (r = check_heads(h_q, h_kv, d))) return r;
  if (!Q || !K_c1 || !K_c2 || !S || !aligned16(Q) || !aligned16(K_c1) || !aligned16(K_c2) || !aligned16(S))
    return INFLLM2_ERR_INVALID_ARG;
  if (ld < ld_min || (ld & 3)) return INFLLM2_ERR_INVALID_ARG;
  bool map_fail = false;
  cudaError_t e = launch_shared_scores(Q, K_c1, K_c2, vl->cu_seqlens, vl->batch, vl->max_seqlen, vl->total,
                                       vl->total_c1, vl->total_c2, h_q, h_kv, d, S, ld, softmax_scale(p, d),
                                       p->lse_mode == INFLLM2_LSE_EXACT, pool, static_cast<cudaStream_t>(stream),
                                       &map_fail);
  if (map_fail) return INFLLM2_ERR_INVALID_ARG;
  return e == cudaSuccess ? INFLLM2_OK : cuda_fail(e);
}

int infllm2_shared_scores(const void* Q, const void* K_c1, const void* K_c2, const infllm2_varlen* vl, int32_t h_q,
                          int32_t h_kv, int32_t d, float* S, int64_t ld, const infllm2_params* p, void* stream) {
  return scores_common(Q, K_c1, K_c2, vl, h_q, h_kv, d, S, ld, infllm2_scores_ld(vl, p), false, p, stream);
}

int64_t infllm2_pooled_ld(const infllm2_varlen* vl, const infllm2_params* p) {
  if (!vl || !p || vl->max_seqlen < 0) return 0;
  const int64_t n1 = infllm2_window_count(vl->max_seqlen, p->c1_len, p->c1_stride);
  return std::max<int64_t>(4, (2 * ((n1 + 3) / 4) + 3) & ~int64_t(3));
}

int infllm2_pooled_scores(const void* Q, const void* K_c1, const void* K_c2, const infllm2_varlen* vl, int32_t h_q,
                          int32_t h_kv, int32_t d, float* P, int64_t ldp, const infllm2_params* p, void* stream) {
  return scores_common(Q, K_c1, K_c2, vl, h_q, h_kv, d, P, ldp, infllm2_pooled_ld(vl, p), true, p, stream);
}

static int topk_common(const float* S, int64_t ld, int64_t ld_min, bool pool, const infllm2_varlen* vl,
                       int32_t h_kv, int32_t* block_idx, const infllm2_params* p, void* stream) {
  int r;
  if ((r = check_varlen(vl)) || (r = check_params(p))) return r;
  if (!S || !block_idx || !aligned16(S) || h_kv <= 0) return INFLLM2_ERR_INVALID_ARG;
  if (ld < ld_min || (ld & 3)) return INFLLM2_ERR_INVALID_ARG;
  cudaError_t e = launch_topk(S, ld, vl->cu_seqlens, vl->batch, vl->max_seqlen, vl->total, h_kv, p->n_init,
                              p->n_local, p->top_k, pool, static_cast<cudaStream_t>(stream), block_idx);
  if (e == cudaErrorInvalidValue) return INFLLM2_ERR_UNSUPPORTED;
  return e == cudaSuccess ? INFLLM2_OK : cuda_fail(e);
}

int infllm2_topk_blocks(const float* S, int64_t ld, const infllm2_varlen* vl, int32_t h_kv, int32_t* block_idx,
                        const infllm2_params* p, void* stream) {
  return topk_common(S, ld, infllm2_scores_ld(vl, p), false, vl, h_kv, block_idx, p, stream);
}

int infllm2_topk_blocks_pooled(const float* P, int64_t ldp, const infllm2_varlen* vl, int32_t h_kv,
                               int32_t* block_idx, const infllm2_params* p, void* stream) {
  return topk_common(P, ldp, infllm2_pooled_ld(vl, p), true, vl, h_kv, block_idx, p, stream);
}

size_t infllm2_select_workspace_bytes(const infllm2_varlen* vl, int32_t h_kv, const infllm2_params* p) {
  if (!vl || !p || h_kv <= 0 || vl->total < 0) return 0;
  return static_cast<size_t>(h_kv) * static_cast<size_t>(vl->total) * static_cast<size_t>(infllm2_scores_ld(vl, p)) *
         sizeof(float);
}

int infllm2_select_blocks(const void* Q, const void* K_c1, const void* K_c2, const infllm2_varlen* vl, int32_t h_q,
                          int32_t h_kv, int32_t d, void* workspace, size_t workspace_bytes, int32_t* block_idx,
                          float* s_shared_out, const infllm2_params* p, void* stream) {
  int r;
  if ((r = check_varlen(vl)) || (r = check_params(p)) || (r = check_heads(h_q, h_kv, d))) return r;
  if (!block_idx) return INFLLM2_ERR_INVALID_ARG;
  float* S = s_shared_out;
  if (!S) {
    if (!workspace) return INFLLM2_ERR_INVALID_ARG;
    if (workspace_bytes < infllm2_select_workspace_bytes(vl, h_kv, p)) return INFLLM2_ERR_WORKSPACE_TOO_SMALL;
    S = static_cast<float*>(workspace);
  }
  const int64_t ld = infllm2_scores_ld(vl, p);
  if ((r = infllm2_shared_scores(Q, K_c1, K_c2, vl, h_q, h_kv, d, S, ld, p, stream))) return r;
  return infllm2_topk_blocks(S, ld, vl, h_kv, block_idx, p, stream);
}

size_t infllm2_sparse_workspace_bytes(const infllm2_varlen* vl, int32_t h_q) {
  if (check_varlen(vl) || h_q <= 0) return 0;
  return (static_cast<size_t>(vl->total) * h_q * sizeof(float) + 255) & ~size_t(255);
}

int infllm2_sparse_attn(const void* Q, const void* K, const void* V, const int32_t* block_idx,
                        const infllm2_varlen* vl, int32_t h_q, int32_t h_kv, int32_t d, void* out, int32_t out_dtype,
                        void* workspace, size_t workspace_bytes, const infllm2_params* p, void* stream) {
  int r;
  if ((r = check_varlen(vl)) || (r = check_params(p)) || (r = check_heads(h_q, h_kv, d))) return r;
  if (!Q || !K || !V || !block_idx || !out || !aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(out))
    return INFLLM2_ERR_INVALID_ARG;
  if (out_dtype != INFLLM2_OUT_BF16 && out_dtype != INFLLM2_OUT_F32) return INFLLM2_ERR_INVALID_ARG;
  if (!workspace || !aligned16(workspace)) return INFLLM2_ERR_INVALID_ARG;
  if (workspace_bytes < infllm2_sparse_workspace_bytes(vl, h_q)) return INFLLM2_ERR_WORKSPACE_TOO_SMALL;
  bool map_fail = false;
  const int n_sel = p->n_init + p->n_local + p->top_k;
  const float scale = softmax_scale(p, d);
  const bool f32 = out_dtype == INFLLM2_OUT_F32;
  float* lse = static_cast<float*>(workspace);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the top-k blocks of each token, then the init and local blocks once per 128/G tokens, merged in
  cudaError_t e = launch_sparse_attn(Q, K, V, block_idx, vl->cu_seqlens, vl->batch, vl->total, h_q, h_kv, d, n_sel,
                                     p->n_init, p->n_local, scale, out, f32, lse, st, &map_fail);
  if (e == cudaSuccess && !map_fail)
    e = (INFLLM2_PAIR_ATTN ? launch_pair_attn : launch_dense_attn)(Q, K, V, vl->cu_seqlens, vl->batch, vl->max_seqlen,
                          vl->total, h_q, h_kv, d, scale, out, f32, p->n_init, p->n_local, lse, st, &map_fail);
  if (map_fail) return INFLLM2_ERR_INVALID_ARG;
  return e == cudaSuccess ? INFLLM2_OK : cuda_fail(e);
}

int infllm2_dense_attn(const void* Q, const void* K, const void* V, const infllm2_varlen* vl, int32_t h_q,
                       int32_t h_kv, int32_t d, void* out, int32_t out_dtype, const infllm2_params* p, void* stream) {
  int r;
  if ((r = check_varlen(vl)) || (r = check_params(p)) || (r = check_heads(h_q, h_kv, d))) return r;
  if (!Q || !K || !V || !out || !aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(out))
    return INFLLM2_ERR_INVALID_ARG;
  if (out_dtype != INFLLM2_OUT_BF16 && out_dtype != INFLLM2_OUT_F32) return INFLLM2_ERR_INVALID_ARG;
  bool map_fail = false;
  cudaError_t e = (INFLLM2_PAIR_ATTN ? launch_pair_attn : launch_dense_attn)(
      Q, K, V, vl->cu_seqlens, vl->batch, vl->max_seqlen, vl->total, h_q, h_kv, d, softmax_scale(p, d), out,
      out_dtype == INFLLM2_OUT_F32, 0, 0, nullptr, static_cast<cudaStream_t>(stream), &map_fail);
  if (map_fail) return INFLLM2_ERR_INVALID_ARG;
  return e == cudaSuccess ? INFLLM2_OK : cuda_fail(e);
}

size_t infllm2_sparse_backward_workspace_bytes(const infllm2_varlen* vl, int32_t h_q, int32_t h_kv,
                                               const infllm2_params* p) {
  if (check_varlen(vl) || check_params(p) || h_q <= 0 || h_kv <= 0) return 0;
  const BwdPlan P = bwd_plan(vl->batch, vl->max_seqlen, vl->total, h_q, h_kv, p->n_init + p->n_local + p->top_k);
  return P.bytes;
}

int infllm2_sparse_attn_backward(const void* Q, const void* K, const void* V, const void* out, int32_t out_dtype,
                                 const void* dout, const float* lse, const int32_t* block_idx,
                                 const infllm2_varlen* vl, int32_t h_q, int32_t h_kv, int32_t d, float* dQ, float* dK,
                                 float* dV, void* workspace, size_t workspace_bytes, const infllm2_params* p,
                                 void* stream) {
  int r;
  if ((r = check_varlen(vl)) || (r = check_params(p)) || (r = check_heads(h_q, h_kv, d))) return r;
  const void* ptrs[] = {Q, K, V, out, dout, lse, block_idx, dQ, dK, dV, workspace};
  for (const void* q : ptrs)
    if (!q || !aligned16(q)) return INFLLM2_ERR_INVALID_ARG;
  if (out_dtype != INFLLM2_OUT_BF16 && out_dtype != INFLLM2_OUT_F32) return INFLLM2_ERR_INVALID_ARG;
  const int G = h_q / h_kv;
  if (G != 8 && G != 16) return INFLLM2_ERR_UNSUPPORTED;
  const int n_sel = p->n_init + p->n_local + p->top_k;
  const BwdPlan P = bwd_plan(vl->batch, vl->max_seqlen, vl->total, h_q, h_kv, n_sel);
  if (static_cast<int64_t>(h_kv) * vl->total * n_sel > INT32_MAX ||
      static_cast<int64_t>(h_kv) * vl->batch * P.nb_max > (int64_t(1) << 24))
    return INFLLM2_ERR_UNSUPPORTED;
  if (workspace_bytes < P.bytes) return INFLLM2_ERR_WORKSPACE_TOO_SMALL;
  if (vl->total == 0) return INFLLM2_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the lists' form first (recorded in the device status word when broken)
  {
    sparse::SparseArgs a{};
    a.block_idx = block_idx; a.cu = vl->cu_seqlens; a.batch = vl->batch; a.total = vl->total; a.h_q = h_q;
    a.h_kv = h_kv; a.n_sel = n_sel; a.n_init = p->n_init; a.n_local = p->n_local;
    const int64_t warps = static_cast<int64_t>(h_kv) * vl->total;
    const int64_t grid = std::min<int64_t>((warps + 7) / 8, static_cast<int64_t>(num_sms()) * 8);
    sparse::check_lists_kernel<<<static_cast<unsigned>(grid), 256, 0, st>>>(a);
  }
  bool map_fail = false;
  cudaError_t e = launch_sparse_backward(Q, K, V, out, out_dtype == INFLLM2_OUT_F32, dout, lse, block_idx,
                                         vl->cu_seqlens, vl->batch, vl->max_seqlen, vl->total, h_q, h_kv, d, n_sel,
                                         p->n_init, p->n_local, softmax_scale(p, d), dQ, dK, dV, workspace, P, st,
                                         &map_fail);
  if (map_fail) return INFLLM2_ERR_INVALID_ARG;
  return e == cudaSuccess ? INFLLM2_OK : cuda_fail(e);
}

static int check_decode_state(const infllm2_decode_state* s) {
  if (!s || !s->k_cache || !s->v_cache || !s->k_c1 || !s->k_c2 || !s->seq_len) return INFLLM2_ERR_INVALID_ARG;
  if (!aligned16(s->k_cache) || !aligned16(s->v_cache) || !aligned16(s->k_c1) || !aligned16(s->k_c2))
    return INFLLM2_ERR_INVALID_ARG;
  if (s->batch < 1 || s->batch > 65535 || s->capacity < 1) return INFLLM2_ERR_INVALID_ARG;
  if (static_cast<int64_t>(s->batch) * s->capacity > INT32_MAX) return INFLLM2_ERR_UNSUPPORTED;
  return check_heads(s->h_q, s->h_kv, s->d);
}

static DecodePlan plan_of(const infllm2_decode_state* st, const infllm2_params* p) {
  return decode_plan(st->batch, st->capacity, st->h_q, st->h_kv, st->d, p->n_init + p->n_local + p->top_k,
                     num_sms());
}

size_t infllm2_decode_workspace_bytes(const infllm2_decode_state* st, const infllm2_params* p) {
  if (check_decode_state(st) || check_params(p) || p->lse_mode != INFLLM2_LSE_APPROX) return 0;
  const DecodePlan P = plan_of(st, p);
  return decode_plan_supported(P) ? P.bytes : 0;
}

int64_t infllm2_decode_block_idx_offset(const infllm2_decode_state* st, const infllm2_params* p) {
  if (check_decode_state(st) || check_params(p) || p->lse_mode != INFLLM2_LSE_APPROX) return -1;
  const DecodePlan P = plan_of(st, p);
  return decode_plan_supported(P) ? static_cast<int64_t>(P.off_idx) : -1;
}

int infllm2_decode_build_caches(const infllm2_decode_state* st, const infllm2_params* p, void* stream) {
  int r;
  if ((r = check_decode_state(st)) || (r = check_params(p))) return r;
  if (p->lse_mode != INFLLM2_LSE_APPROX) return INFLLM2_ERR_UNSUPPORTED;
  const DecodePlan P = plan_of(st, p);
  if (!decode_plan_supported(P)) return INFLLM2_ERR_UNSUPPORTED;
  cudaError_t e = launch_decode_build_caches(st, P, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? INFLLM2_OK : cuda_fail(e);
}

int infllm2_decode_step(const infllm2_decode_state* st, const void* q, const void* k_new, const void* v_new,
                        void* out, void* workspace, size_t workspace_bytes, const infllm2_params* p, void* stream) {
  int r;
  if ((r = check_decode_state(st)) || (r = check_params(p))) return r;
  if (p->lse_mode != INFLLM2_LSE_APPROX) return INFLLM2_ERR_UNSUPPORTED;   // decode keeps the approximation
  if (!q || !k_new || !v_new || !out || !workspace || !aligned16(q) || !aligned16(k_new) || !aligned16(v_new) ||
      !aligned16(out) || !aligned16(workspace))
    return INFLLM2_ERR_INVALID_ARG;
  const DecodePlan P = plan_of(st, p);
  if (!decode_plan_supported(P)) return INFLLM2_ERR_UNSUPPORTED;
  if (workspace_bytes < P.bytes) return INFLLM2_ERR_WORKSPACE_TOO_SMALL;
  cudaError_t e = launch_decode_step(st, q, k_new, v_new, out, workspace, P, p->n_init, p->n_local, p->top_k,
                                     softmax_scale(p, st->d), static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? INFLLM2_OK : cuda_fail(e);
}

int infllm2_get_device_status(void) {
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e);
  int v = 0;
  e = cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e);
  return v;
}

int infllm2_clear_device_status(void) {
  const int zero = 0;
  cudaError_t e = cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e);
  e = cudaDeviceSynchronize();
  return e == cudaSuccess ? INFLLM2_OK : cuda_fail(e);
}

int infllm2_probe_l2_gather(const void* K, const void* V, int64_t rows, int32_t h_kv, int32_t nblk,
                            int32_t tiles, int32_t producers, void* stream) {
  if (!K || !V || !aligned16(K) || !aligned16(V) || rows < 64 || h_kv < 1 || nblk < 1 ||
      static_cast<int64_t>(nblk) * 64 > rows || tiles < 1)
    return INFLLM2_ERR_INVALID_ARG;
  if (producers != 1 && producers != 2 && producers != 3 && producers != 6) return INFLLM2_ERR_UNSUPPORTED;
  bool map_fail = false;
  cudaError_t e = launch_l2_gather_probe(K, V, rows, h_kv, nblk, tiles, producers, static_cast<cudaStream_t>(stream),
                                         &map_fail);
  if (map_fail) return INFLLM2_ERR_INVALID_ARG;
  return e == cudaSuccess ? INFLLM2_OK : cuda_fail(e);
}

int infllm2_debug_wait_timeout(uint64_t limit_ns, void* stream) {
  if (limit_ns == 0 || limit_ns > 10000000000ull) return INFLLM2_ERR_INVALID_ARG;
  debug_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? INFLLM2_OK : cuda_fail(e);
}

}  // extern "C"

// Allocation-free variant of infllm2_select_blocks (fixed device scratch).
#include "noalloc.cu"
