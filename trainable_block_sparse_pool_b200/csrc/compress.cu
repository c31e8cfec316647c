// Step 1: stage-1 and coarse mean pooling of K (InfLLM-V2, top168 article
// §三 first stage: mean pooling over windows of l_C1 = 32 keys every
// s_C1 = 16; §四: the coarse keys for the LSE approximation pool the raw
// keys with l_C2 = 128, s_C2 = 64).
//
// HBM-bound.  One CTA covers 512 tokens of one (sequence, kv head): it sums
// the 40 16-row chunks starting at its first token (the 8 chunks past the
// end are the halo its last windows need) in fp64 — exact for bf16 inputs —
// then forms every C1 window as two adjacent chunk sums and every C2 window
// as eight, divides by the (power-of-two) window length and rounds once to
// bf16.  Loads are 16-byte vectors, one thread per (chunk, 8-wide slice of d).
#include "sm100.cuh"

namespace infllm2 {

// Round an fp64 value to the nearest bf16 (ties to even), written from the
// IEEE-754 formats: keep the top 8 significant bits of the fp64 significand.
__device__ __forceinline__ uint16_t f64_to_bf16_rne(double x) {
  const uint64_t b = static_cast<uint64_t>(__double_as_longlong(x));
  const uint16_t sign = static_cast<uint16_t>((b >> 48) & 0x8000u);
  const int ex = static_cast<int>((b >> 52) & 0x7FF);
  const uint64_t man = b & ((1ull << 52) - 1);
  if (ex == 0x7FF) return man ? static_cast<uint16_t>(sign | 0x7FC0u) : static_cast<uint16_t>(sign | 0x7F80u);
  if (ex == 0) return sign;  // fp64 subnormals are far below the bf16 range
  int e = ex - 1023;                              // unbiased exponent
  uint64_t sig = (1ull << 52) | man;              // 53-bit significand
  int shift = 45;                                 // keep 8 bits
  int be = e + 127;                               // bf16 biased exponent
  if (be <= 0) shift += 1 - be;                   // bf16 subnormal: fewer bits kept
  if (shift > 54) return sign;
  uint64_t q = sig >> shift;
  const uint64_t rem = sig & ((1ull << shift) - 1);
  const uint64_t half = 1ull << (shift - 1);
  if (rem > half || (rem == half && (q & 1))) ++q;
  if (be <= 0) {
    // subnormal result (q < 128) or rounded up into the smallest normal (q == 128)
    return static_cast<uint16_t>(sign | static_cast<uint16_t>(q));
  }
  if (q == 256) { q = 128; ++be; }
  if (be >= 255) return static_cast<uint16_t>(sign | 0x7F80u);
  return static_cast<uint16_t>(sign | (be << 7) | (q & 0x7F));
}

constexpr int kCompTok = 512;                 // tokens per CTA
constexpr int kChunk = 16;                    // rows per chunk (= s_C1)
constexpr int kNChunk = kCompTok / kChunk + 8;  // 32 + halo of 8 (a C2 window spans 8 chunks)
constexpr int kCompThreads = 256;

template <int D>
__global__ void __launch_bounds__(kCompThreads) compress_k_kernel(
    const __nv_bfloat16* __restrict__ K, const int32_t* __restrict__ cu, int h_kv,
    __nv_bfloat16* __restrict__ Kc1, int64_t total_c1, __nv_bfloat16* __restrict__ Kc2, int64_t total_c2) {
  constexpr int SL = D / 8;  // 16-byte slices per row
  __shared__ double csum[kNChunk][D];
  __shared__ int red[32];
  const int s = blockIdx.y, g = blockIdx.z;
  const int row0 = cu[s];
  const int len = cu[s + 1] - row0;
  const int t0 = blockIdx.x * kCompTok;
  if (t0 >= len) return;
  const int c1_off = pooled_offset_block(cu, s, 32, 16, red);
  const int c2_off = pooled_offset_block(cu, s, 128, 64, red);
  const int n_c1 = window_count_dev(len, 32, 16);
  const int n_c2 = window_count_dev(len, 128, 64);

  // chunk sums
  for (int item = threadIdx.x; item < kNChunk * SL; item += kCompThreads) {
    const int c = item / SL, sl = item % SL;
    double acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.0;
    const int tb = t0 + c * kChunk;
#pragma unroll 4
    for (int r = 0; r < kChunk; ++r) {
      const int t = tb + r;
      if (t < len) {
        const uint4 raw =
            *reinterpret_cast<const uint4*>(K + ((static_cast<int64_t>(row0 + t) * h_kv + g) * D + sl * 8));
        const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 f = __bfloat1622float2(p2[i]);
          acc[2 * i] += static_cast<double>(f.x);
          acc[2 * i + 1] += static_cast<double>(f.y);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) csum[c][sl * 8 + i] = acc[i];
  }
  __syncthreads();

  // C1 windows j = t0/16 + w, w < 32: chunks w and w+1
  const int j0 = t0 / kChunk;
  for (int item = threadIdx.x; item < 32 * SL; item += kCompThreads) {
    const int w = item / SL, sl = item % SL;
    const int j = j0 + w;
    if (j >= n_c1) continue;
    const int64_t orow = static_cast<int64_t>(c1_off) + j;
    if (orow >= total_c1) { record_status(INFLLM2_ERR_DEVICE_BOUNDS); continue; }
    uint16_t o[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i] = f64_to_bf16_rne((csum[w][sl * 8 + i] + csum[w + 1][sl * 8 + i]) * (1.0 / 32.0));
    uint4 v;
    v.x = o[0] | (static_cast<uint32_t>(o[1]) << 16);
    v.y = o[2] | (static_cast<uint32_t>(o[3]) << 16);
    v.z = o[4] | (static_cast<uint32_t>(o[5]) << 16);
    v.w = o[6] | (static_cast<uint32_t>(o[7]) << 16);
    *reinterpret_cast<uint4*>(Kc1 + ((static_cast<int64_t>(g) * total_c1 + orow) * D + sl * 8)) = v;
  }
  // C2 windows m = t0/64 + w, w < 8: chunks 4w .. 4w+7
  const int m0 = t0 / 64;
  for (int item = threadIdx.x; item < 8 * SL; item += kCompThreads) {
    const int w = item / SL, sl = item % SL;
    const int m = m0 + w;
    if (m >= n_c2) continue;
    const int64_t orow = static_cast<int64_t>(c2_off) + m;
    if (orow >= total_c2) { record_status(INFLLM2_ERR_DEVICE_BOUNDS); continue; }
    uint16_t o[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      double a = 0.0;
#pragma unroll
      for (int c = 0; c < 8; ++c) a += csum[4 * w + c][sl * 8 + i];
      o[i] = f64_to_bf16_rne(a * (1.0 / 128.0));
    }
    uint4 v;
    v.x = o[0] | (static_cast<uint32_t>(o[1]) << 16);
    v.y = o[2] | (static_cast<uint32_t>(o[3]) << 16);
    v.z = o[4] | (static_cast<uint32_t>(o[5]) << 16);
    v.w = o[6] | (static_cast<uint32_t>(o[7]) << 16);
    *reinterpret_cast<uint4*>(Kc2 + ((static_cast<int64_t>(g) * total_c2 + orow) * D + sl * 8)) = v;
  }
}

cudaError_t launch_compress_k(const void* K, const int32_t* cu, int batch, int max_seqlen, int h_kv, int d,
                              void* Kc1, int64_t total_c1, void* Kc2, int64_t total_c2, cudaStream_t st) {
  dim3 grid((max_seqlen + kCompTok - 1) / kCompTok, batch, h_kv);
  if (grid.x == 0) return cudaSuccess;
  if (d == 128)
    compress_k_kernel<128><<<grid, kCompThreads, 0, st>>>(static_cast<const __nv_bfloat16*>(K), cu, h_kv,
                                                          static_cast<__nv_bfloat16*>(Kc1), total_c1,
                                                          static_cast<__nv_bfloat16*>(Kc2), total_c2);
  else
    compress_k_kernel<64><<<grid, kCompThreads, 0, st>>>(static_cast<const __nv_bfloat16*>(K), cu, h_kv,
                                                         static_cast<__nv_bfloat16*>(Kc1), total_c1,
                                                         static_cast<__nv_bfloat16*>(Kc2), total_c2);
  return cudaGetLastError();
}

}  // namespace infllm2
