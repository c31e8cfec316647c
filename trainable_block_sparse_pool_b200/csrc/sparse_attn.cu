// Step 4: block-sparse causal attention over the selected blocks (InfLLM-V2:
// selected and sliding attention merged into one sparse attention with a
// single output — paper-reading blog, "对齐计算图"; top168 article §七).
//
// Work unit: one (kv group g, query token t).  Its G query heads share the
// selected block list I(g,t) (|I| <= 96 blocks of 64 keys).  With G = 16 a
// unit is too small for the M dimension of tcgen05 (64 or 128), so the
// contractions are transposed ("swap AB"): keys fill M, heads fill N.
//   S^T [128 keys, 16] = K_pair[128, d]  . Q_t[16, d]^T      (M=128, N=16)
//   O^T [d, 16]       = V_pair[128, d]^T . P^T[128, 16]      (M=d,   N=16)
// A "pair" is two selected blocks side by side in shared memory (each
// loaded by TMA straight from K / V — the gather is the TMA coordinate).
// Softmax: one thread per key lane holds the 16 head scores of its key;
// the per-head maximum over the 128 keys is a shuffle + shared-memory
// reduction; each thread keeps partial row sums and every thread holds the
// running maxima, so the rescale factors are known everywhere.  P goes to
// shared memory as bf16 in the no-swizzle MN-major core-matrix layout.  The
// PV product of each pair lands in a fresh TMEM accumulator and is folded
// into registers (O = O * alpha + O_pair) by the thread that owns that row
// of d, so TMEM never needs an in-place rescale.
// Warp roles: warp 0 TMA producer, warp 1 MMA issuer / TMEM owner,
// warps 2-5 softmax + correction.  Persistent CTAs, one per SM, take units
// round-robin (consecutive CTAs work on consecutive tokens of one group, so
// the group's shared init/local blocks stay hot in L2).
#include "sm100.cuh"

namespace infllm2 {

namespace sparse {

constexpr int kThreads = 192;
constexpr int kWG = 128;         // softmax / correction threads
constexpr int kPairKeys = 128;   // keys per tile (two 64-key blocks)
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct Cfg {
  static constexpr int KCH = D / 64;
  static constexpr uint32_t kChunk = kPairKeys * 128;         // 16 KB: 128 keys x 64 dims
  static constexpr uint32_t kHalf = 64 * 128;                 // one block inside a chunk
  static constexpr uint32_t kKBytes = kChunk * KCH;
  static constexpr uint32_t kStageBytes = 2 * kKBytes;        // K then V
  static constexpr int kStages = (D == 128) ? 3 : 5;
  static constexpr uint32_t kQBuf = 16 * 128 * KCH;           // 16 head rows
  static constexpr uint32_t kPBuf = kPairKeys * 16 * 2;       // 4 KB
  static constexpr uint32_t kSmem =
      1024 + kStages * kStageBytes + 2 * kQBuf + 2 * kPBuf + 2 * 4 * 16 * 4 + 4 * 16 * 4 + 512;
};

struct Bars {
  uint64_t kv_full[8];
  uint64_t kv_empty[8];
  uint64_t q_full[2];
  uint64_t q_empty[2];
  uint64_t s_full[2];
  uint64_t s_empty[2];
  uint64_t p_full[2];
  uint64_t o_full[2];
  uint64_t o_empty[2];
  uint64_t mma_done;
  uint64_t wg;          // rendezvous of the four softmax warps
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ bool aborted(const Bars* b) {
  return *reinterpret_cast<const volatile int*>(&b->abort) != 0;
}
__device__ __forceinline__ void set_abort(Bars* b) {
  *reinterpret_cast<volatile int*>(&b->abort) = 1;
}

// Rendezvous of the four softmax warps on an mbarrier (count 4) with a
// bounded wait, so a warp that gave up cannot leave the others blocked.
__device__ __forceinline__ bool wg_sync(uint64_t* bar, uint32_t& phase) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
  const bool ok = mbar_wait(bar, phase & 1);
  ++phase;
  return ok;
}

struct Unit {
  int g, t, seq_start, nvalid;
  int64_t row;
  const int32_t* I;
};

__device__ __forceinline__ Unit get_unit(int64_t u, const int32_t* cu, int batch, int64_t total,
                                         const int32_t* block_idx, int n_sel) {
  Unit x;
  x.g = static_cast<int>(u / total);
  x.row = u - static_cast<int64_t>(x.g) * total;
  const int s = find_sequence(cu, batch, x.row);
  x.seq_start = cu[s];
  x.t = static_cast<int>(x.row - x.seq_start);
  x.I = block_idx + u * n_sel;
  int nv = 0;
  while (nv < n_sel && x.I[nv] >= 0) ++nv;
  x.nvalid = nv;
  return x;
}

template <int D, int G, bool OUT_F32>
__global__ void __launch_bounds__(kThreads, 1) sparse_attn_kernel(
    const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
    const __grid_constant__ CUtensorMap tmV, const int32_t* __restrict__ block_idx, const int32_t* __restrict__ cu,
    int batch, int64_t total, int h_q, int h_kv, int n_sel, float scale, void* __restrict__ out) {
  using C = Cfg<D>;
  static_assert(G >= 1 && G <= 16, "group size <= 16");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sKV = smem;
  uint8_t* sQ = sKV + C::kStages * C::kStageBytes;
  uint8_t* sP = sQ + 2 * C::kQBuf;
  float* red_max = reinterpret_cast<float*>(sP + 2 * C::kPBuf);  // [2][4][16]
  float* red_l = red_max + 2 * 4 * 16;                             // [4][16]
  Bars* bars = reinterpret_cast<Bars*>(red_l + 4 * 16);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t n_units = static_cast<int64_t>(h_kv) * total;

  // zero both Q buffers so the head rows past G contribute zeros
  for (int i = threadIdx.x; i < static_cast<int>(2 * C::kQBuf / 16); i += kThreads)
    reinterpret_cast<uint4*>(sQ)[i] = make_uint4(0, 0, 0, 0);
  fence_proxy_async_smem();
  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kStages; ++i) { mbar_init(&bars->kv_full[i], 1); mbar_init(&bars->kv_empty[i], 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->q_full[i], 1);
      mbar_init(&bars->q_empty[i], 1);
      mbar_init(&bars->s_full[i], 1);
      mbar_init(&bars->s_empty[i], 4);
      mbar_init(&bars->p_full[i], 4);
      mbar_init(&bars->o_full[i], 1);
      mbar_init(&bars->o_empty[i], 4);
    }
    mbar_init(&bars->mma_done, 1);
    mbar_init(&bars->wg, 4);
    bars->abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) { tmem_alloc(&bars->tmem_base, 64); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ); tma_prefetch_desc(&tmK); tma_prefetch_desc(&tmV);
      int it = 0, qi = 0;
      bool ok = true;
      for (int64_t u = blockIdx.x; ok && u < n_units; u += gridDim.x, ++qi) {
        const Unit x = get_unit(u, cu, batch, total, block_idx, n_sel);
        const int qb = qi & 1;
        if (!mbar_wait(&bars->q_empty[qb], ((qi >> 1) & 1) ^ 1)) { set_abort(bars); break; }
        mbar_arrive_expect_tx(&bars->q_full[qb], C::KCH * G * 128);
        for (int ch = 0; ch < C::KCH; ++ch)
          tma_load_4d(sQ + qb * C::kQBuf + ch * 2048, &tmQ, &bars->q_full[qb], ch * 64, 0, x.g,
                      static_cast<int>(x.row));
        const int ntile = (x.nvalid + 1) >> 1;
        for (int i = 0; i < ntile; ++i, ++it) {
          const int st = it % C::kStages;
          if (!mbar_wait(&bars->kv_empty[st], ((it / C::kStages) & 1) ^ 1) || aborted(bars)) {
            set_abort(bars); ok = false; break;
          }
          const int b0 = x.I[2 * i];
          const int b1 = (2 * i + 1 < x.nvalid) ? x.I[2 * i + 1] : b0;   // odd count: reload, masked later
          uint8_t* dK = sKV + st * C::kStageBytes;
          uint8_t* dV = dK + C::kKBytes;
          mbar_arrive_expect_tx(&bars->kv_full[st], C::kStageBytes);
          for (int ch = 0; ch < C::KCH; ++ch) {
            tma_load_3d(dK + ch * C::kChunk, &tmK, &bars->kv_full[st], ch * 64, x.g, x.seq_start + 64 * b0);
            tma_load_3d(dK + ch * C::kChunk + C::kHalf, &tmK, &bars->kv_full[st], ch * 64, x.g,
                        x.seq_start + 64 * b1);
            tma_load_3d(dV + ch * C::kChunk, &tmV, &bars->kv_full[st], ch * 64, x.g, x.seq_start + 64 * b0);
            tma_load_3d(dV + ch * C::kChunk + C::kHalf, &tmV, &bars->kv_full[st], ch * 64, x.g,
                        x.seq_start + 64 * b1);
          }
        }
      }
      // wait for every copy still in flight before the CTA may exit
      for (int i = max(0, it - C::kStages); i < it; ++i) mbar_wait(&bars->kv_full[i % C::kStages], (i / C::kStages) & 1);
      for (int i = max(0, qi - 2); i < qi; ++i) mbar_wait(&bars->q_full[i & 1], (i >> 1) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idS = idesc_bf16_f32(128, 16, 0, 0);
      const uint32_t idO = idesc_bf16_f32(128, 16, 1, 1);
      const uint32_t lboV = (D == 128) ? C::kChunk : 0u;   // d = 64: rows 64-127 of O^T repeat 0-63
      int it = 0, qi = 0;
      bool ok = true;
      auto issue_pv = [&](int j) -> bool {
        const int pb = j & 1;
        const int st = j % C::kStages;
        if (!mbar_wait(&bars->p_full[pb], (j >> 1) & 1)) return false;
        if (!mbar_wait(&bars->o_empty[pb], ((j >> 1) & 1) ^ 1)) return false;
        tc_fence_after();
        const uint32_t v_base = smem_u32(sKV + st * C::kStageBytes + C::kKBytes);
        const uint32_t p_base = smem_u32(sP + pb * C::kPBuf);
#pragma unroll
        for (int k = 0; k < kPairKeys / 16; ++k) {
          const uint64_t a = make_sdesc(v_base + k * 2048, lboV, 1024, kLayoutSW128);
          const uint64_t b = make_sdesc(p_base + k * 512, 256, 128, kLayoutNone);
          umma_bf16(tmem + 32 + pb * 16, a, b, idO, k > 0);
        }
        umma_commit(&bars->kv_empty[st]);
        umma_commit(&bars->o_full[pb]);
        return true;
      };
      for (int64_t u = blockIdx.x; ok && u < n_units; u += gridDim.x, ++qi) {
        const Unit x = get_unit(u, cu, batch, total, block_idx, n_sel);
        const int qb = qi & 1;
        if (!mbar_wait(&bars->q_full[qb], (qi >> 1) & 1)) { set_abort(bars); break; }
        const uint32_t q_base = smem_u32(sQ + qb * C::kQBuf);
        const int ntile = (x.nvalid + 1) >> 1;
        for (int i = 0; i < ntile; ++i, ++it) {
          const int st = it % C::kStages;
          const int sb = it & 1;
          if (!mbar_wait(&bars->kv_full[st], (it / C::kStages) & 1) ||
              !mbar_wait(&bars->s_empty[sb], ((it >> 1) & 1) ^ 1) || aborted(bars)) {
            set_abort(bars); ok = false; break;
          }
          tc_fence_after();
          const uint32_t k_base = smem_u32(sKV + st * C::kStageBytes);
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint64_t a = make_sdesc(k_base + (k >> 2) * C::kChunk + (k & 3) * 32, 16, 1024, kLayoutSW128);
            const uint64_t b = make_sdesc(q_base + (k >> 2) * 2048 + (k & 3) * 32, 16, 1024, kLayoutSW128);
            umma_bf16(tmem + sb * 16, a, b, idS, k > 0);
          }
          umma_commit(&bars->s_full[sb]);
          if (i == ntile - 1) umma_commit(&bars->q_empty[qb]);
          if (it > 0 && !issue_pv(it - 1)) { set_abort(bars); ok = false; ++it; break; }
        }
      }
      if (ok && it > 0 && !issue_pv(it - 1)) set_abort(bars);
      umma_commit(&bars->mma_done);
      mbar_wait(&bars->mma_done, 0);
    }
  } else {
    // ------------------------------------------------------------ softmax + correction
    const int wq = warp & 3;                 // TMEM lane quadrant of this warp
    const int kl = wq * 32 + lane;           // key lane (softmax) / d row (correction)
    const uint32_t lane_addr = static_cast<uint32_t>(wq * 32) << 16;
    const float c = scale * kLog2e;
    uint32_t wg_phase = 0;
    int it = 0;
    for (int64_t u = blockIdx.x; u < n_units && !aborted(bars); u += gridDim.x) {
      const Unit x = get_unit(u, cu, batch, total, block_idx, n_sel);
      float m_run[16], l_part[16], o_acc[16];
#pragma unroll
      for (int h = 0; h < 16; ++h) { m_run[h] = -INFINITY; l_part[h] = 0.f; o_acc[h] = 0.f; }
      const int ntile = (x.nvalid + 1) >> 1;
      bool ok = true;
      for (int i = 0; i < ntile; ++i, ++it) {
        const int sb = it & 1;
        // ---- softmax of tile it
        if (!mbar_wait(&bars->s_full[sb], (it >> 1) & 1)) { set_abort(bars); ok = false; break; }
        tc_fence_after();
        float v[16];
        tmem_ld16(tmem + lane_addr + sb * 16, v);
        tmem_wait_ld16(v);
        const int half = kl >> 6;
        const int bsel = 2 * i + half;
        const int blk = (bsel < x.nvalid) ? x.I[bsel] : -1;
        const int pos = 64 * blk + (kl & 63);
        const bool valid = (blk >= 0) && (pos <= x.t);
        float mx[16];
#pragma unroll
        for (int h = 0; h < 16; ++h) {
          v[h] = valid ? v[h] * c : -INFINITY;
          mx[h] = v[h];
        }
#pragma unroll
        for (int h = 0; h < 16; ++h) {
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], o));
        }
        float* rm = red_max + (it & 1) * 64;
        if (lane < 16) {
          float mine = mx[0];
#pragma unroll
          for (int h = 1; h < 16; ++h) if (lane == h) mine = mx[h];
          rm[wq * 16 + lane] = mine;
        }
        if (!wg_sync(&bars->wg, wg_phase)) { set_abort(bars); ok = false; ++it; break; }
        float alpha[16];
        uint32_t pk[8];
#pragma unroll
        for (int h = 0; h < 16; ++h) {
          const float tmax = fmaxf(fmaxf(rm[h], rm[16 + h]), fmaxf(rm[32 + h], rm[48 + h]));
          const float m_new = fmaxf(m_run[h], tmax);
          const bool none = (m_new == -INFINITY);
          alpha[h] = none ? 1.f : ex2(m_run[h] - m_new);
          const float p = none ? 0.f : ex2(v[h] - m_new);
          l_part[h] = l_part[h] * alpha[h] + p;
          m_run[h] = m_new;
          v[h] = p;
        }
#pragma unroll
        for (int h = 0; h < 8; ++h) {
          __nv_bfloat162 b2 = __floats2bfloat162_rn(v[2 * h], v[2 * h + 1]);
          pk[h] = *reinterpret_cast<uint32_t*>(&b2);
        }
        uint8_t* pbuf = sP + sb * C::kPBuf;
        const uint32_t poff = (kl >> 3) * 256 + (kl & 7) * 16;
        *reinterpret_cast<uint4*>(pbuf + poff) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        *reinterpret_cast<uint4*>(pbuf + poff + 128) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) { mbar_arrive(&bars->p_full[sb]); mbar_arrive(&bars->s_empty[sb]); }
        // ---- correction: fold this tile's P.V into the register accumulator
        if (!mbar_wait(&bars->o_full[sb], (it >> 1) & 1)) { set_abort(bars); ok = false; ++it; break; }
        tc_fence_after();
        float ov[16];
        tmem_ld16(tmem + lane_addr + 32 + sb * 16, ov);
        tmem_wait_ld16(ov);
#pragma unroll
        for (int h = 0; h < 16; ++h) o_acc[h] = fmaf(o_acc[h], alpha[h], ov[h]);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->o_empty[sb]);
      }
      if (!ok) break;
      // ---- row sums over the 128 key lanes, then the normalised output
#pragma unroll
      for (int h = 0; h < 16; ++h) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) l_part[h] += __shfl_xor_sync(0xffffffffu, l_part[h], o);
      }
      if (lane < 16) {
        float mine = l_part[0];
#pragma unroll
        for (int h = 1; h < 16; ++h) if (lane == h) mine = l_part[h];
        red_l[wq * 16 + lane] = mine;
      }
      if (!wg_sync(&bars->wg, wg_phase)) { set_abort(bars); break; }
      if (kl < D) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float l = red_l[h] + red_l[16 + h] + red_l[32 + h] + red_l[48 + h];
          const float o = (l > 0.f) ? o_acc[h] / l : 0.f;
          const int64_t idx = (x.row * h_q + static_cast<int64_t>(x.g) * G + h) * D + kl;
          if (OUT_F32) reinterpret_cast<float*>(out)[idx] = o;
          else reinterpret_cast<__nv_bfloat16*>(out)[idx] = __float2bfloat16_rn(o);
        }
      }
      if (!wg_sync(&bars->wg, wg_phase)) { set_abort(bars); break; }   // red_l is reused by the next unit
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 64);
}

}  // namespace sparse

bool make_tmap(CUtensorMap* map, const void* base, int rank, const uint64_t* dims, const uint64_t* strides_bytes,
               const uint32_t* box);
int num_sms();

template <int D, int G, bool F32>
static cudaError_t launch_sparse_t(const void* Q, const void* K, const void* V, const int32_t* idx,
                                   const int32_t* cu, int batch, int64_t total, int h_q, int h_kv, int n_sel,
                                   float scale, void* out, cudaStream_t st, bool* map_fail) {
  using C = sparse::Cfg<D>;
  CUtensorMap mQ, mK, mV;
  {
    const uint64_t dims[4] = {(uint64_t)D, (uint64_t)G, (uint64_t)h_kv, (uint64_t)total};
    const uint64_t strides[3] = {(uint64_t)D * 2, (uint64_t)G * D * 2, (uint64_t)h_q * D * 2};
    const uint32_t box[4] = {64, (uint32_t)G, 1, 1};
    if (!make_tmap(&mQ, Q, 4, dims, strides, box)) { *map_fail = true; return cudaErrorInvalidValue; }
  }
  {
    const uint64_t dims[3] = {(uint64_t)D, (uint64_t)h_kv, (uint64_t)total};
    const uint64_t strides[2] = {(uint64_t)D * 2, (uint64_t)h_kv * D * 2};
    const uint32_t box[3] = {64, 1, 64};
    if (!make_tmap(&mK, K, 3, dims, strides, box)) { *map_fail = true; return cudaErrorInvalidValue; }
    if (!make_tmap(&mV, V, 3, dims, strides, box)) { *map_fail = true; return cudaErrorInvalidValue; }
  }
  auto kern = sparse::sparse_attn_kernel<D, G, F32>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return e;
  const int64_t units = static_cast<int64_t>(h_kv) * total;
  if (units == 0) return cudaSuccess;
  const int64_t grid = std::min<int64_t>(units, num_sms());
  kern<<<static_cast<unsigned>(grid), sparse::kThreads, C::kSmem, st>>>(mQ, mK, mV, idx, cu, batch, total, h_q,
                                                                        h_kv, n_sel, scale, out);
  return cudaGetLastError();
}

cudaError_t launch_sparse_attn(const void* Q, const void* K, const void* V, const int32_t* idx, const int32_t* cu,
                               int batch, int64_t total, int h_q, int h_kv, int d, int n_sel, float scale,
                               void* out, bool out_f32, cudaStream_t st, bool* map_fail) {
  const int G = h_q / h_kv;
#define INFLLM2_SPARSE_CASE(DD, GG)                                                                            \
  if (d == DD && G == GG)                                                                                     \
    return out_f32 ? launch_sparse_t<DD, GG, true>(Q, K, V, idx, cu, batch, total, h_q, h_kv, n_sel, scale, out, \
                                                   st, map_fail)                                              \
                   : launch_sparse_t<DD, GG, false>(Q, K, V, idx, cu, batch, total, h_q, h_kv, n_sel, scale,   \
                                                    out, st, map_fail);
  INFLLM2_SPARSE_CASE(128, 16)
  INFLLM2_SPARSE_CASE(128, 8)
  INFLLM2_SPARSE_CASE(128, 4)
  INFLLM2_SPARSE_CASE(128, 2)
  INFLLM2_SPARSE_CASE(128, 1)
  INFLLM2_SPARSE_CASE(64, 16)
  INFLLM2_SPARSE_CASE(64, 8)
  INFLLM2_SPARSE_CASE(64, 4)
  INFLLM2_SPARSE_CASE(64, 2)
  INFLLM2_SPARSE_CASE(64, 1)
#undef INFLLM2_SPARSE_CASE
  return cudaErrorInvalidValue;
}

}  // namespace infllm2
