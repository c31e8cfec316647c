// Measurement: the L2 -> SM gather bandwidth that bounds the block-sparse
// attention.  Persistent CTAs (one per SM); NPROD producer warps each keep
// 6/NPROD stages of 32 KB in flight, every stage a pair of random 64-key
// blocks of one kv group gathered by TMA with the attention kernel's tensor
// map shape and box (64 rows x 64 dims, 128-byte swizzle), from K (even
// producers) or V (odd producers).  Nothing consumes the data: a producer
// reuses a stage as soon as its copy has landed, so the loop runs at the
// rate the memory system delivers tiles.  Blocks are drawn from the first
// nblk blocks of the sequence with a per-producer linear congruential
// generator, so the footprint is nblk * 64 rows of K and of V.
#include "sm100.cuh"

namespace infllm2 {

namespace probe {

constexpr int kStagesPerSm = 6;
constexpr uint32_t kStage = 32768;    // 2 blocks x 64 keys x 128 dims x 2 B

template <int NPROD>
__global__ void __launch_bounds__(32 * NPROD, 1) l2_gather_kernel(const __grid_constant__ CUtensorMap tmK,
                                                                  const __grid_constant__ CUtensorMap tmV,
                                                                  int nblk, int tiles) {
  constexpr int NST = kStagesPerSm / NPROD;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t full[kStagesPerSm];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kStagesPerSm; ++i) mbar_init(&full[i], 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (lane != 0) return;
  const CUtensorMap* tm = (warp & 1) ? &tmV : &tmK;
  uint64_t* bars = full + warp * NST;
  uint8_t* ring = smem + warp * NST * kStage;
  uint32_t rng = 2654435761u * (blockIdx.x * NPROD + warp + 1);
  int i = 0;
  for (; i < tiles; ++i) {
    const int st = i % NST;
    if (i >= NST && !mbar_wait(&bars[st], ((i / NST) - 1) & 1)) break;
    rng = rng * 1664525u + 1013904223u;
    const int b0 = static_cast<int>((rng >> 8) % static_cast<uint32_t>(nblk));
    rng = rng * 1664525u + 1013904223u;
    const int b1 = static_cast<int>((rng >> 8) % static_cast<uint32_t>(nblk));
    uint8_t* dst = ring + st * kStage;
    mbar_arrive_expect_tx(&bars[st], kStage);
    for (int ch = 0; ch < 2; ++ch) {
      tma_load_3d(dst + ch * 16384, tm, &bars[st], ch * 64, 0, 64 * b0);
      tma_load_3d(dst + ch * 16384 + 8192, tm, &bars[st], ch * 64, 0, 64 * b1);
    }
  }
  // wait for every copy still in flight before the CTA exits
  for (int k = max(0, i - NST); k < i; ++k) mbar_wait(&bars[k % NST], (k / NST) & 1);
}

}  // namespace probe

bool make_tmap(CUtensorMap* map, const void* base, int rank, const uint64_t* dims, const uint64_t* strides_bytes,
               const uint32_t* box);
int num_sms();

template <int NPROD>
static cudaError_t launch_probe_t(const CUtensorMap& mK, const CUtensorMap& mV, int nblk, int tiles, cudaStream_t st) {
  auto kern = probe::l2_gather_kernel<NPROD>;
  const uint32_t smem = 1024 + probe::kStagesPerSm * probe::kStage;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  kern<<<num_sms(), 32 * NPROD, smem, st>>>(mK, mV, nblk, tiles);
  return cudaGetLastError();
}

// K, V: [rows, h_kv, 128] bf16.  Each producer gathers `tiles` tiles of 32 KB.
cudaError_t launch_l2_gather_probe(const void* K, const void* V, int64_t rows, int h_kv, int nblk, int tiles,
                                   int nprod, cudaStream_t st, bool* map_fail) {
  CUtensorMap mK, mV;
  const uint64_t dims[3] = {128, (uint64_t)h_kv, (uint64_t)rows};
  const uint64_t strides[2] = {256, (uint64_t)h_kv * 256};
  const uint32_t box[3] = {64, 1, 64};
  if (!make_tmap(&mK, K, 3, dims, strides, box) || !make_tmap(&mV, V, 3, dims, strides, box)) {
    *map_fail = true;
    return cudaErrorInvalidValue;
  }
  if (nprod == 1) return launch_probe_t<1>(mK, mV, nblk, tiles, st);
  if (nprod == 2) return launch_probe_t<2>(mK, mV, nblk, tiles, st);
  if (nprod == 3) return launch_probe_t<3>(mK, mV, nblk, tiles, st);
  if (nprod == 6) return launch_probe_t<6>(mK, mV, nblk, tiles, st);
  return cudaErrorInvalidValue;
}

}  // namespace infllm2
