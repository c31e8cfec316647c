// Step 2: compressed scores with the LSE approximation and the fused
// head-group sum (InfLLM-V2, top168 article §三 second stage and §四).
//
// For one kv group g and a tile of TQ = 256/G query tokens (256 query rows
// (t, h), h the G heads of the group) a CTA computes
//   phase A  LSE(t,h) = logsumexp_m  scale * q[t,h] . K_c2[g,m]  over the
//            visible coarse windows (the LSE approximation), or, in the
//            EXACT form, over the visible stage-1 windows K_c1 themselves
//            (the two-pass computation the approximation replaces: the
//            rows of S then sum to G),
//   phase B  S[g,t,j] = sum_h exp(scale * q[t,h] . K_c1[g,j] - LSE(t,h))
//            over the visible stage-1 windows,
// and writes only S (the group sum happens on chip, the per-head scores
// never reach HBM).  With POOL the kernel writes, instead of S, the first
// step of the 5/4/1 max-pool: for every group of four windows 4i .. 4i+3 the
// pair (max of its visible windows, window 4i+3 or -inf), half the bytes of
// S.  Block i's score is then max(pair i's max, pair i-1's last window).
//
// Both contractions run on the tcgen05 tensor cores with the Q tile resident
// in shared memory:
//   phase A  D[(t,h), m] = Q[(t,h), :] . K_c2[m, :]   M = 128 rows (two
//            halves of the Q tile), N = 128 coarse keys;
//   phase B  D[j, (t,h)] = K_c1[j, :] . Q[(t,h), :]   M = 128 keys, N = 256
//            rows; keys sit on TMEM lanes and the (t,h) pairs along columns,
//            so one thread owns one key and sums its token's G head columns
//            in registers: the group sum needs no shuffles.
// Warp roles: warps 0-7 epilogue (256 threads; warp w reads TMEM lane
// quadrant w%4 and column half w/4), warp 8 TMA producer, warp 9 MMA issuer
// and TMEM owner.  Two 256-column TMEM accumulators alternate so the MMA of
// tile i+1 overlaps the exponentials of tile i.
#include "sm100.cuh"

namespace infllm2 {

namespace score {

constexpr int kThreads = 320;
constexpr int kEpiThreads = 256;
constexpr int kKeysPerTile = 128;
constexpr int kStages = 4;
constexpr float kLog2e = 1.4426950408889634f;

template <int D, int G>
struct Cfg {
  static constexpr int TQ = 256 / G;                      // tokens per tile
  static constexpr int KCH = D / 64;                      // 128-byte chunks of d
  static constexpr uint32_t kQChunk = 256 * 128;          // bytes per chunk of the Q tile
  static constexpr uint32_t kKChunk = kKeysPerTile * 128; // bytes per chunk of a key tile
  static constexpr uint32_t kQBytes = kQChunk * KCH;
  static constexpr uint32_t kStageBytes = kKChunk * KCH;
  static constexpr uint32_t kSmem = 1024 /*align slack*/ + kQBytes + kStages * kStageBytes + 256 * 4 + 256;
};

struct Bars {
  uint64_t q_full;
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ bool aborted(const Bars* b) {
  return *reinterpret_cast<const volatile int*>(&b->abort) != 0;
}
__device__ __forceinline__ void set_abort(Bars* b) {
  *reinterpret_cast<volatile int*>(&b->abort) = 1;
}

template <int D, int G, bool EXACT, bool POOL>
__global__ void __launch_bounds__(kThreads, 1) score_kernel(
    const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK1,
    const __grid_constant__ CUtensorMap tmK2, const __nv_bfloat16* __restrict__ Q,
    const __nv_bfloat16* __restrict__ Kc1, const int32_t* __restrict__ cu, int h_q, int h_kv,
    int64_t total, int64_t total_c1, float* __restrict__ S, int64_t ld, float scale) {
  using C = Cfg<D, G>;
  constexpr int TQ = C::TQ;
  static_assert(G >= 1 && G <= 16 && (16 % G) == 0, "group size must be a power of two <= 16");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = smem + C::kQBytes;
  float* nlse = reinterpret_cast<float*>(sK + kStages * C::kStageBytes);   // -LSE (log2 units) per Q row
  Bars* bars = reinterpret_cast<Bars*>(nlse + 256);
  __shared__ int red[32];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int s = blockIdx.y, g = blockIdx.z;
  const int row0 = cu[s];
  const int len = cu[s + 1] - row0;
  const int ntiles = (len + TQ - 1) / TQ;
  if (static_cast<int>(blockIdx.x) >= ntiles) return;
  const int tile = ntiles - 1 - blockIdx.x;      // heaviest tiles first
  const int t0 = tile * TQ;
  const int t_last = min(len - 1, t0 + TQ - 1);
  const int c1_off = pooled_offset_block(cu, s, 32, 16, red);
  const int c2_off = pooled_offset_block(cu, s, 128, 64, red);
  const int n1_max = visible_windows_dev(t_last, 32, 16);
  const int n2_max = EXACT ? n1_max : visible_windows_dev(t_last, 128, 64);
  const int nA = (n2_max + kKeysPerTile - 1) / kKeysPerTile;   // key tiles of phase A
  const int nB = (n1_max + kKeysPerTile - 1) / kKeysPerTile;   // stage-1 key tiles
  const float c = scale * kLog2e;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int i = 0; i < kStages; ++i) { mbar_init(&bars->full[i], 1); mbar_init(&bars->empty[i], 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(&bars->tfull[i], 1); mbar_init(&bars->tempty[i], 8); }
    mbar_init(&bars->mma_done, 1);
    bars->abort = 0;
    fence_barrier_init();
  }
  if (warp == 9) { tmem_alloc(&bars->tmem_base, 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ); tma_prefetch_desc(&tmK1); tma_prefetch_desc(&tmK2);
      mbar_arrive_expect_tx(&bars->q_full, C::kQBytes);
      for (int ch = 0; ch < C::KCH; ++ch)
        tma_load_4d(sQ + ch * C::kQChunk, &tmQ, &bars->q_full, ch * 64, 0, g, row0 + t0);
      int it = 0;
      for (; it < nA + nB; ++it) {
        const int st = it % kStages;
        if (!mbar_wait(&bars->empty[st], ((it / kStages) & 1) ^ 1)) { set_abort(bars); break; }
        if (aborted(bars)) break;
        mbar_arrive_expect_tx(&bars->full[st], C::kStageBytes);
        uint8_t* dst = sK + st * C::kStageBytes;
        if (it < nA) {
          for (int ch = 0; ch < C::KCH; ++ch)
            tma_load_3d(dst + ch * C::kKChunk, EXACT ? &tmK1 : &tmK2, &bars->full[st], ch * 64,
                        (EXACT ? c1_off : c2_off) + it * kKeysPerTile, g);
        } else {
          const int kt = it - nA;
          for (int ch = 0; ch < C::KCH; ++ch)
            tma_load_3d(dst + ch * C::kKChunk, &tmK1, &bars->full[st], ch * 64, c1_off + kt * kKeysPerTile, g);
        }
      }
      // make sure every copy this CTA issued has landed before it can exit
      mbar_wait(&bars->q_full, 0);
      for (int i = max(0, it - kStages); i < it; ++i) mbar_wait(&bars->full[i % kStages], (i / kStages) & 1);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idA = idesc_bf16_f32(128, 128, 0, 0);
      const uint32_t idB = idesc_bf16_f32(128, 256, 0, 0);
      bool ok = mbar_wait(&bars->q_full, 0);
      if (!ok) set_abort(bars);
      tc_fence_after();
      const uint32_t q_base = smem_u32(sQ);
      for (int it = 0; ok && it < nA + nB; ++it) {
        const int st = it % kStages;
        const int buf = it & 1;
        if (!mbar_wait(&bars->tempty[buf], ((it >> 1) & 1) ^ 1)) { set_abort(bars); break; }
        if (!mbar_wait(&bars->full[st], (it / kStages) & 1)) { set_abort(bars); break; }
        if (aborted(bars)) break;
        tc_fence_after();
        const uint32_t k_base = smem_u32(sK + st * C::kStageBytes);
        const uint32_t d_base = tmem + buf * 256;
        if (it < nA) {
          for (int mh = 0; mh < 2; ++mh) {
#pragma unroll
            for (int k = 0; k < D / 16; ++k) {
              const uint32_t koff = (k >> 2) * C::kQChunk + (k & 3) * 32;
              const uint64_t a = make_sdesc(q_base + koff + mh * 128 * 128, 16, 1024, kLayoutSW128);
              const uint64_t b = make_sdesc(k_base + (k >> 2) * C::kKChunk + (k & 3) * 32, 16, 1024, kLayoutSW128);
              umma_bf16(d_base + mh * 128, a, b, idA, k > 0);
            }
          }
        } else {
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint64_t a = make_sdesc(k_base + (k >> 2) * C::kKChunk + (k & 3) * 32, 16, 1024, kLayoutSW128);
            const uint64_t b = make_sdesc(q_base + (k >> 2) * C::kQChunk + (k & 3) * 32, 16, 1024, kLayoutSW128);
            umma_bf16(d_base, a, b, idB, k > 0);
          }
        }
        umma_commit(&bars->empty[st]);
        umma_commit(&bars->tfull[buf]);
      }
      umma_commit(&bars->mma_done);
      mbar_wait(&bars->mma_done, 0);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q4 = warp & 3, hh = warp >> 2;
    const uint32_t lane_addr = static_cast<uint32_t>(q4 * 32) << 16;
    // phase A: this thread owns Q-tile row r = (t_local, h)
    const int r = hh * 128 + q4 * 32 + lane;
    const int t_loc = r / G, h = r % G;
    const int t = t0 + t_loc;
    const int n2 = EXACT ? visible_windows_dev(t, 32, 16) : visible_windows_dev(t, 128, 64);
    float m_run = -INFINITY, l_run = 0.f;
    int it = 0;
    bool ok = true;
    for (; it < nA; ++it) {
      const int buf = it & 1;
      if (!mbar_wait(&bars->tfull[buf], (it >> 1) & 1)) { set_abort(bars); ok = false; break; }
      tc_fence_after();
      const uint32_t tcol = tmem + lane_addr + buf * 256 + hh * 128;
      float va[32], vb[32];
      tmem_ld32(tcol, va);
      tmem_wait_ld32(va);
#pragma unroll
      for (int cc = 0; cc < 128; cc += 32) {
        float (&v)[32] = ((cc >> 5) & 1) ? vb : va;
        float (&vn)[32] = ((cc >> 5) & 1) ? va : vb;
        if (cc + 32 < 128) tmem_ld32(tcol + cc + 32, vn);
        const int m0 = it * kKeysPerTile + cc;
        float mx = -INFINITY;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          v[i] = (m0 + i < n2) ? v[i] * c : -INFINITY;
          mx = fmaxf(mx, v[i]);
        }
        const float m_new = fmaxf(m_run, mx);
        if (m_new != -INFINITY) {
          float acc = 0.f;
#pragma unroll
          for (int i = 0; i < 32; ++i) acc += ex2(v[i] - m_new);
          l_run = l_run * ex2(m_run - m_new) + acc;
          m_run = m_new;
        }
        if (cc + 32 < 128) tmem_wait_ld32(vn);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->tempty[buf]);
    }
    float lse;
    if (n2 > 0) {
      lse = m_run + log2f(l_run);
    } else if (EXACT) {
      lse = INFINITY;                   // no visible window: the row is empty
    } else {
      // no coarse window visible yet (t < 127): exact log-sum-exp over the
      // visible stage-1 windows (at most 6), straight from global memory
      const int n1 = visible_windows_dev(t, 32, 16);
      float mm = -INFINITY, ll = 0.f;
      if (t < len) {
        const __nv_bfloat16* qp = Q + (static_cast<int64_t>(row0 + t) * h_q + g * G + h) * D;
        for (int j = 0; j < n1 && c1_off + j < total_c1; ++j) {
          const __nv_bfloat16* kp = Kc1 + (static_cast<int64_t>(g) * total_c1 + c1_off + j) * D;
          float dot = 0.f;
          for (int e = 0; e < D; ++e) dot += __bfloat162float(qp[e]) * __bfloat162float(kp[e]);
          const float x = dot * c;
          const float mn = fmaxf(mm, x);
          ll = ll * ex2(mm - mn) + ex2(x - mn);
          mm = mn;
        }
      }
      lse = (n1 > 0) ? mm + log2f(ll) : INFINITY;
    }

    // phase B: this thread owns key j; columns hh*128 .. +128 are tokens
    // hh*TQ/2 .. (hh+1)*TQ/2 - 1, G heads each
    nlse[r] = -lse;                     // stored negated: exp2(s*c - lse) = ex2(fma(s, c, nlse))
    named_bar_sync(2, kEpiThreads);
    const int tt0 = t0 + hh * (TQ / 2);
    float* srow0 = S + (static_cast<int64_t>(g) * total + row0 + tt0) * ld;
    for (; ok && it < nA + nB; ++it) {
      const int buf = it & 1;
      const int kt = it - nA;
      if (!mbar_wait(&bars->tfull[buf], (it >> 1) & 1)) { set_abort(bars); ok = false; break; }
      tc_fence_after();
      const int j = kt * kKeysPerTile + q4 * 32 + lane;
      const int need = 16 * j + 31;     // window j is visible to tokens at or after this position
      // software-pipelined over four 32-column chunks: the load of chunk
      // c+1 is in flight while chunk c is computed
      const uint32_t tcol = tmem + lane_addr + buf * 256 + hh * 128;
      float va[32], vb[32];
      tmem_ld32(tcol, va);
      tmem_wait_ld32(va);
#pragma unroll
      for (int cc = 0; cc < 128; cc += 32) {
        float (&v)[32] = ((cc >> 5) & 1) ? vb : va;
        float (&vn)[32] = ((cc >> 5) & 1) ? va : vb;
        if (cc + 32 < 128) tmem_ld32(tcol + cc + 32, vn);
        const float4* l4 = reinterpret_cast<const float4*>(nlse + hh * 128 + cc);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float4 L = l4[q];
          v[4 * q + 0] = ex2(fmaf(v[4 * q + 0], c, L.x));
          v[4 * q + 1] = ex2(fmaf(v[4 * q + 1], c, L.y));
          v[4 * q + 2] = ex2(fmaf(v[4 * q + 2], c, L.z));
          v[4 * q + 3] = ex2(fmaf(v[4 * q + 3], c, L.w));
        }
        // group sums: tree over each token's G head columns
#pragma unroll
        for (int w = 1; w < G; w <<= 1) {
#pragma unroll
          for (int i = 0; i < 32; i += 2 * w) v[i] += v[i + w];
        }
        if constexpr (POOL) {
          // lanes 4k .. 4k+3 hold windows 4i .. 4i+3 of one group (j is a
          // multiple of 4 on lane 4k): two xor shuffles give all four the
          // group's maximum, and lane 4k+3, which holds the last window,
          // writes the pair when the group's first window (48 positions
          // earlier) is visible
#pragma unroll
          for (int i = 0; i < 32; i += G) {
            const int tl = (cc + i) / G;
            const int tt = tt0 + tl;
            const float x = (tt < len && tt >= need) ? v[i] : -INFINITY;
            float m = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 1));
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
            if ((lane & 3) == 3 && tt < len && tt >= need - 48)
              *reinterpret_cast<float2*>(srow0 + static_cast<int64_t>(tl) * ld + 2 * (j >> 2)) = make_float2(m, x);
          }
        } else {
#pragma unroll
          for (int i = 0; i < 32; i += G) {
            const int tl = (cc + i) / G;          // token index within this half
            const int tt = tt0 + tl;
            if (tt < len && tt >= need) srow0[static_cast<int64_t>(tl) * ld + j] = v[i];
          }
        }
        if (cc + 32 < 128) tmem_wait_ld32(vn);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->tempty[buf]);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 9) tmem_dealloc(tmem, 512);
}

}  // namespace score

// Host side: tensor maps and launch.
typedef CUresult (*PFN_encodeTiled)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                    const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                    CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
PFN_encodeTiled get_encode_tiled();

bool make_tmap(CUtensorMap* map, const void* base, int rank, const uint64_t* dims, const uint64_t* strides_bytes,
               const uint32_t* box) {
  PFN_encodeTiled enc = get_encode_tiled();
  if (!enc) return false;
  cuuint64_t gd[5], gs[4];
  cuuint32_t bx[5], es[5];
  for (int i = 0; i < rank; ++i) { gd[i] = dims[i]; bx[i] = box[i]; es[i] = 1; }
  for (int i = 0; i < rank - 1; ++i) gs[i] = strides_bytes[i];
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), gd, gs, bx, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D, int G, bool EXACT, bool POOL>
static cudaError_t launch_score_t(const void* Q, const void* Kc1, const void* Kc2, const int32_t* cu, int batch,
                                  int max_seqlen, int64_t total, int64_t total_c1, int64_t total_c2, int h_q,
                                  int h_kv, float* S, int64_t ld, float scale, cudaStream_t st, bool* map_fail) {
  using C = score::Cfg<D, G>;
  CUtensorMap mQ, mK1, mK2;
  {
    const uint64_t dims[4] = {(uint64_t)D, (uint64_t)G, (uint64_t)h_kv, (uint64_t)total};
    const uint64_t strides[3] = {(uint64_t)D * 2, (uint64_t)G * D * 2, (uint64_t)h_q * D * 2};
    const uint32_t box[4] = {64, (uint32_t)G, 1, (uint32_t)C::TQ};
    if (!make_tmap(&mQ, Q, 4, dims, strides, box)) { *map_fail = true; return cudaErrorInvalidValue; }
  }
  {
    const uint64_t dims[3] = {(uint64_t)D, (uint64_t)(total_c1 > 0 ? total_c1 : 1), (uint64_t)h_kv};
    const uint64_t strides[2] = {(uint64_t)D * 2, (uint64_t)(total_c1 > 0 ? total_c1 : 1) * D * 2};
    const uint32_t box[3] = {64, score::kKeysPerTile, 1};
    if (!make_tmap(&mK1, Kc1, 3, dims, strides, box)) { *map_fail = true; return cudaErrorInvalidValue; }
  }
  {
    const uint64_t dims[3] = {(uint64_t)D, (uint64_t)(total_c2 > 0 ? total_c2 : 1), (uint64_t)h_kv};
    const uint64_t strides[2] = {(uint64_t)D * 2, (uint64_t)(total_c2 > 0 ? total_c2 : 1) * D * 2};
    const uint32_t box[3] = {64, score::kKeysPerTile, 1};
    if (!make_tmap(&mK2, Kc2, 3, dims, strides, box)) { *map_fail = true; return cudaErrorInvalidValue; }
  }
  auto kern = score::score_kernel<D, G, EXACT, POOL>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return e;
  dim3 grid((max_seqlen + C::TQ - 1) / C::TQ, batch, h_kv);
  if (grid.x == 0) return cudaSuccess;
  kern<<<grid, score::kThreads, C::kSmem, st>>>(mQ, mK1, mK2, static_cast<const __nv_bfloat16*>(Q),
                                                 static_cast<const __nv_bfloat16*>(Kc1), cu, h_q, h_kv, total,
                                                 total_c1, S, ld, scale);
  return cudaGetLastError();
}

cudaError_t launch_shared_scores(const void* Q, const void* Kc1, const void* Kc2, const int32_t* cu, int batch,
                                 int max_seqlen, int64_t total, int64_t total_c1, int64_t total_c2, int h_q,
                                 int h_kv, int d, float* S, int64_t ld, float scale, bool exact, bool pool,
                                 cudaStream_t st, bool* map_fail) {
  const int G = h_q / h_kv;
#define INFLLM2_SCORE_ARGS Q, Kc1, Kc2, cu, batch, max_seqlen, total, total_c1, total_c2, h_q, h_kv, S, ld, scale, st, map_fail
#define INFLLM2_SCORE_CASE(DD, GG)                                                                                 \
  if (d == DD && G == GG)                                                                                         \
    return exact ? (pool ? launch_score_t<DD, GG, true, true>(INFLLM2_SCORE_ARGS)                                 \
                         : launch_score_t<DD, GG, true, false>(INFLLM2_SCORE_ARGS))                               \
                 : (pool ? launch_score_t<DD, GG, false, true>(INFLLM2_SCORE_ARGS)                                \
                         : launch_score_t<DD, GG, false, false>(INFLLM2_SCORE_ARGS));
  INFLLM2_SCORE_CASE(128, 16)
  INFLLM2_SCORE_CASE(128, 8)
  INFLLM2_SCORE_CASE(128, 4)
  INFLLM2_SCORE_CASE(128, 2)
  INFLLM2_SCORE_CASE(128, 1)
  INFLLM2_SCORE_CASE(64, 16)
  INFLLM2_SCORE_CASE(64, 8)
  INFLLM2_SCORE_CASE(64, 4)
  INFLLM2_SCORE_CASE(64, 2)
  INFLLM2_SCORE_CASE(64, 1)
#undef INFLLM2_SCORE_CASE
#undef INFLLM2_SCORE_ARGS
  return cudaErrorInvalidValue;
}

}  // namespace infllm2
