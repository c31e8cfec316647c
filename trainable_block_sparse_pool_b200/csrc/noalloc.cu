// Allocation-free block selection.
//
// infllm2_select_blocks needs scratch memory for S_shared, which the caller
// normally provides as a workspace it allocated.  Some callers cannot
// allocate device memory at the point where they select blocks: code that
// runs inside a custom allocator or memory pool, plugins and runtimes whose
// host does all device allocation up front, or paths that must not call
// cudaMalloc because it can synchronise the device.  For them this entry
// point keeps the scratch in a fixed-size array in the library's own device
// memory instead.  It is a convenience of this library; the paper has no
// counterpart.
//
// The array lives for as long as the library is loaded, on every GPU that
// loads it.  All calls share it, so calls whose kernels overlap on the GPU
// (different streams, or different host threads without ordering) race on
// it; it keeps the last call's contents.  Nothing in it has to start at
// zero: the score kernel writes every entry that the top-k kernel reads.
#include "sm100.cuh"

namespace infllm2 {

// 64 MiB of fp32 S_shared: h_kv * total * ld floats.  At h_kv = 2 this
// covers one 8192-token sequence (ld = 512), the longest the dense/sparse
// switch keeps on the dense path by default, or any batch of that size.
constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;
static_assert(kNoAllocScratchBytes == INFLLM2_NOALLOC_SCRATCH_BYTES,
              "the array's size is the limit the public header documents");

static __device__ __align__(256) float g_noalloc_scores[kNoAllocScratchBytes / sizeof(float)];

// Device address of g_noalloc_scores on the current device.  In host code
// the array's name is only a host-side stand-in, so the address is looked up
// with cudaGetSymbolAddress (which allocates nothing) with the device
// current.  It is looked up on every call rather than cached, so a primary
// context that was torn down and created again never leaves a stale address.
static int noalloc_scratch(float** out) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scores);
  if (e != cudaSuccess) return cuda_fail(e);
  *out = static_cast<float*>(p);
  return INFLLM2_OK;
}

}  // namespace infllm2

extern "C" int infllm2_select_blocks_noalloc(const void* Q, const void* K_c1, const void* K_c2,
                                             const infllm2_varlen* vl, int32_t h_q, int32_t h_kv, int32_t d,
                                             int32_t* block_idx, const infllm2_params* p, void* stream) {
  using namespace infllm2;
  int r;
  if ((r = check_varlen(vl)) || (r = check_params(p)) || (r = check_heads(h_q, h_kv, d))) return r;
  if (!block_idx) return INFLLM2_ERR_INVALID_ARG;
  if (infllm2_select_workspace_bytes(vl, h_kv, p) > kNoAllocScratchBytes) return INFLLM2_ERR_WORKSPACE_TOO_SMALL;
  float* S = nullptr;
  if ((r = noalloc_scratch(&S))) return r;
  const int64_t ld = infllm2_scores_ld(vl, p);
  if ((r = infllm2_shared_scores(Q, K_c1, K_c2, vl, h_q, h_kv, d, S, ld, p, stream))) return r;
  return infllm2_topk_blocks(S, ld, vl, h_kv, block_idx, p, stream);
}
