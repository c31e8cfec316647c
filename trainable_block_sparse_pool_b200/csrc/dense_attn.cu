// Dense causal attention: the short-sequence side of InfLLM-V2's dense/sparse
// switch (paper-reading blog, "Dense-Sparse Switchable Attention"; dtcms
// article §二.2.c).  Same inputs and output form as the sparse kernel.
//
// The same kernel, in its LOCAL form, computes the shared part of the
// block-sparse attention: every query token attends to its init blocks and
// to the n_local blocks that end at its own block (top168 article §七), and
// these are the same for all tokens of a 64-token block.  Attending to them
// once per CTA of 128/G tokens (instead of once per token) leaves only the
// top-k blocks to the per-token sparse kernel, which runs first and leaves
// its normalised partial in out and its log-sum-exp in lse; the row's thread
// here merges the two partials through their log-sum-exps.
//
// A CTA owns one kv group and TQ = 128/G consecutive query tokens: its 128
// query rows (t, h) share every key of the group, so one K/V tile feeds all
// of them (GQA packing).  A tile is two 64-key blocks, each gathered by TMA
// (dense: blocks 2i, 2i+1; LOCAL: consecutive blocks of the CTA's init and
// local range).  Per 128-key tile:
//   S[128 rows, 128 keys] = Q . K^T        tcgen05, A = Q (smem), B = K (smem)
//   softmax, two threads per row (warps w and w + 4 share TMEM lane
//   quadrant w % 4; each owns 64 of the tile's score columns): one TMEM
//   read of its 64 scores, the row maximum exchanged with the partner
//   through shared memory at the pair's barrier, exp2, and bf16 P written
//   back to TMEM over the tile's own score columns (key k in column k/2)
//   O_tile[128 rows, d] = P . V            A = P (TMEM), B = V (smem, MN-major)
// O_tile lands in a fresh TMEM accumulator; each thread folds its d/2
// columns into registers (O = O * alpha + O_tile) one tile later, after it
// has written the next tile's P, so the softmax never waits for the P.V of
// the tile it has just produced.
// Warp roles: warp 0 loads Q and the K ring, warp 10 the V ring (a K slot is
// free once its QK product is done, a V slot only once its P.V product is),
// warp 1 issues the MMAs and owns TMEM, warps 2-9 softmax + correction.
#include "sm100.cuh"

namespace infllm2 {

namespace dense {

constexpr int kSoftWarps = 8;                // two per TMEM lane quadrant
constexpr int kVWarp = 2 + kSoftWarps;        // the V producer
constexpr int kThreads = 64 + 32 * kSoftWarps + 32;
constexpr int kKeys = 128;
constexpr int kKStages = 3;
constexpr int kVStages = 2;
constexpr float kLog2e = 1.4426950408889634f;

template <int D, int G>
struct Cfg {
  static constexpr int TQ = 128 / G;
  static constexpr int KCH = D / 64;
  static constexpr uint32_t kQBytes = 128 * 128 * KCH;
  static constexpr uint32_t kChunk = kKeys * 128;            // 16 KB
  static constexpr uint32_t kKBytes = kChunk * KCH;
  static constexpr uint32_t kRed = 3 * 128 * 2 * 4;            // row-max exchange (two slots), row-sum exchange
  static constexpr uint32_t kSmem = 1024 + kQBytes + (kKStages + kVStages) * kKBytes + kRed + 512;
  static constexpr uint32_t kOCol = 256;                     // O buffers after the two S buffers
};

struct Bars {
  uint64_t q_full;
  uint64_t k_full[kKStages];
  uint64_t k_empty[kKStages];
  uint64_t v_full[kVStages];
  uint64_t v_empty[kVStages];
  uint64_t s_full[2];
  uint64_t s_empty[2];
  uint64_t p_full;
  uint64_t o_full[2];
  uint64_t o_empty[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ bool aborted(const Bars* b) { return *reinterpret_cast<const volatile int*>(&b->abort) != 0; }
__device__ __forceinline__ void set_abort(Bars* b) { *reinterpret_cast<volatile int*>(&b->abort) = 1; }

// The blocks a CTA walks.  Dense: 0 .. t_last/64.  LOCAL: the init blocks
// [0, i_hi) followed by [l_start, b_hi], the union of the init and local
// blocks of the CTA's query tokens (blocks b_lo .. b_hi); block(p) < 0 past
// the end.  in_set tells whether block blk is shared for query token t.
struct BlockWalk {
  int i_hi, l_start, nblk;
  __device__ int block(int p) const { return p >= nblk ? -1 : (p < i_hi ? p : l_start + (p - i_hi)); }
};
__device__ __forceinline__ BlockWalk local_walk(int b_lo, int b_hi, int n_init, int n_local) {
  BlockWalk w;
  w.i_hi = min(n_init, b_hi + 1);
  w.l_start = max(w.i_hi, max(0, b_lo - n_local + 1));
  w.nblk = w.i_hi + max(0, b_hi - w.l_start + 1);
  return w;
}
__device__ __forceinline__ bool in_set(int blk, int t, int n_init, int n_local) {
  const int bt = t >> 6;
  return blk < min(n_init, bt + 1) || blk >= bt - n_local + 1;
}

template <int D, int G, bool OUT_F32, bool LOCAL>
__global__ void __launch_bounds__(kThreads, 1) dense_attn_kernel(
    const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
    const __grid_constant__ CUtensorMap tmV, const int32_t* __restrict__ cu, int h_q, float scale,
    void* __restrict__ out, int n_init, int n_local, float* __restrict__ lse) {
  using C = Cfg<D, G>;
  constexpr int TQ = C::TQ;
  static_assert(G >= 1 && G <= 16 && (16 % G) == 0, "group size must be a power of two <= 16");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sKV = sQ + C::kQBytes;
  uint8_t* sKr = sKV;                                       // K ring [kKStages][kKBytes]
  uint8_t* sVr = sKV + kKStages * C::kKBytes;               // V ring [kVStages][kKBytes]
  float* xch = reinterpret_cast<float*>(sKV + (kKStages + kVStages) * C::kKBytes);   // [slot][row][half]: maxima (slots 0, 1), sums (2)
  Bars* bars = reinterpret_cast<Bars*>(xch + 3 * 128 * 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int s = blockIdx.y, g = blockIdx.z;
  const int row0 = cu[s];
  const int len = cu[s + 1] - row0;
  const int ntiles = (len + TQ - 1) / TQ;
  if (static_cast<int>(blockIdx.x) >= ntiles) return;
  const int t0 = (ntiles - 1 - blockIdx.x) * TQ;        // heaviest query tiles first
  const int t_last = min(len - 1, t0 + TQ - 1);
  BlockWalk walk;
  if (LOCAL) {
    walk = local_walk(t0 >> 6, t_last >> 6, n_init, n_local);
  } else {
    walk.i_hi = t_last / 64 + 1;
    walk.l_start = walk.i_hi;
    walk.nblk = walk.i_hi;
  }
  const int nkt = (walk.nblk + 1) / 2;                   // tiles of two blocks

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int i = 0; i < kKStages; ++i) { mbar_init(&bars->k_full[i], 1); mbar_init(&bars->k_empty[i], 1); }
    for (int i = 0; i < kVStages; ++i) { mbar_init(&bars->v_full[i], 1); mbar_init(&bars->v_empty[i], 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->s_full[i], 1);
      mbar_init(&bars->s_empty[i], kSoftWarps);
      mbar_init(&bars->o_full[i], 1);
      mbar_init(&bars->o_empty[i], kSoftWarps);
    }
    mbar_init(&bars->p_full, kSoftWarps);
    mbar_init(&bars->mma_done, 1);
    bars->abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) { tmem_alloc(&bars->tmem_base, 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0 || warp == kVWarp) {
    if (lane == 0) {
      const bool isV = (warp == kVWarp);
      const int nst = isV ? kVStages : kKStages;
      const CUtensorMap* tm = isV ? &tmV : &tmK;
      uint8_t* ring = isV ? sVr : sKr;
      uint64_t* full = isV ? bars->v_full : bars->k_full;
      uint64_t* empty = isV ? bars->v_empty : bars->k_empty;
      tma_prefetch_desc(tm);
      if (!isV) {
        tma_prefetch_desc(&tmQ);
        mbar_arrive_expect_tx(&bars->q_full, C::kQBytes);
        for (int ch = 0; ch < C::KCH; ++ch) tma_load_4d(sQ + ch * 16384, &tmQ, &bars->q_full, ch * 64, 0, g, row0 + t0);
      }
      int it = 0;
      for (; it < nkt; ++it) {
        const int st = it % nst;
        if (!mbar_wait(&empty[st], ((it / nst) & 1) ^ 1) || aborted(bars)) { set_abort(bars); break; }
        uint8_t* dst = ring + st * C::kKBytes;
        const int ba = walk.block(2 * it);
        int bb = walk.block(2 * it + 1);
        if (bb < 0) bb = ba;                             // odd count: reload, masked by the softmax
        mbar_arrive_expect_tx(&full[st], C::kKBytes);
        for (int ch = 0; ch < C::KCH; ++ch) {
          tma_load_3d(dst + ch * C::kChunk, tm, &full[st], ch * 64, g, row0 + 64 * ba);
          tma_load_3d(dst + ch * C::kChunk + C::kChunk / 2, tm, &full[st], ch * 64, g, row0 + 64 * bb);
        }
      }
      // wait for every copy still in flight before the CTA may exit
      if (!isV) mbar_wait(&bars->q_full, 0);
      for (int i = max(0, it - nst); i < it; ++i) mbar_wait(&full[i % nst], (i / nst) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idS = idesc_bf16_f32(128, kKeys, 0, 0);
      const uint32_t idO = idesc_bf16_f32(128, D, 0, 1);
      const uint32_t q_base = smem_u32(sQ);
      bool ok = mbar_wait(&bars->q_full, 0);
      if (!ok) set_abort(bars);
      auto issue_pv = [&](int j) -> bool {
        const int pb = j & 1;
        const int st = j % kVStages;
        if (!mbar_wait(&bars->p_full, j & 1)) return false;
        if (!mbar_wait(&bars->o_empty[pb], ((j >> 1) & 1) ^ 1)) return false;
        if (!mbar_wait(&bars->v_full[st], (j / kVStages) & 1)) return false;
        tc_fence_after();
        const uint32_t v_base = smem_u32(sVr + st * C::kKBytes);
        const uint32_t p_tmem = tmem + (j & 1) * kKeys;     // P(j) over S(j)'s columns: keys 16k.. in column 8k..
#pragma unroll
        for (int k = 0; k < kKeys / 16; ++k) {
          const uint64_t b = make_sdesc(v_base + k * 2048, C::kChunk, 1024, kLayoutSW128);
          umma_bf16_ts(tmem + C::kOCol + pb * D, p_tmem + k * 8, b, idO, k > 0);
        }
        umma_commit(&bars->v_empty[st]);
        umma_commit(&bars->o_full[pb]);
        return true;
      };
      int it = 0;
      for (; ok && it < nkt; ++it) {
        const int st = it % kKStages;
        const int sb = it & 1;
        if (!mbar_wait(&bars->k_full[st], (it / kKStages) & 1) ||
            !mbar_wait(&bars->s_empty[sb], ((it >> 1) & 1) ^ 1) || aborted(bars)) {
          set_abort(bars); ok = false; break;
        }
        tc_fence_after();
        const uint32_t k_base = smem_u32(sKr + st * C::kKBytes);
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint64_t a = make_sdesc(q_base + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024, kLayoutSW128);
          const uint64_t b = make_sdesc(k_base + (k >> 2) * C::kChunk + (k & 3) * 32, 16, 1024, kLayoutSW128);
          umma_bf16(tmem + sb * kKeys, a, b, idS, k > 0);
        }
        umma_commit(&bars->s_full[sb]);
        umma_commit(&bars->k_empty[st]);                 // the K slot is free once this product is done
        if (it > 0 && !issue_pv(it - 1)) { set_abort(bars); ok = false; break; }
      }
      if (ok && nkt > 0 && !issue_pv(nkt - 1)) set_abort(bars);
      umma_commit(&bars->mma_done);
      mbar_wait(&bars->mma_done, 0);
    }
  } else {
    const int wq = warp & 3;                      // TMEM lane quadrant
    const int hf = (warp - 2) >> 2;               // which half of the columns
    const int r = wq * 32 + lane;                 // query row (t_loc, h)
    const int t = t0 + r / G;
    const int h = r % G;
    const int pair = 1 + wq;                      // named barrier of the two warps of this quadrant
    const uint32_t lane_addr = static_cast<uint32_t>(wq * 32) << 16;
    constexpr int DH = D / 2;                     // output columns of this thread
    const float c = scale * kLog2e;
    float o_acc[DH];
#pragma unroll
    for (int j = 0; j < DH; ++j) o_acc[j] = 0.f;
    float m_run = -INFINITY, l_run = 0.f;         // l_run: this thread's 64 columns only
    float alpha_prev = 1.f;                       // rescale of o_acc that goes with the pending fold
    bool ok = true;
    // o_acc = o_acc * alpha + (P.V of tile j): this thread's d/2 columns
    auto fold = [&](int j, float alpha) {
      const int pb = j & 1;
      const bool gotO = __all_sync(0xffffffffu, mbar_wait(&bars->o_full[pb], (j >> 1) & 1));
      if (!gotO) { set_abort(bars); ok = false; }
      tc_fence_after();
      if (gotO) {
#pragma unroll
        for (int cc = 0; cc < DH; cc += 16) {
          float w[16];
          tmem_load16(tmem + lane_addr + C::kOCol + pb * D + hf * DH + cc, w);
#pragma unroll
          for (int i = 0; i < 16; ++i) o_acc[cc + i] = fmaf(o_acc[cc + i], alpha, w[i]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->o_empty[pb]);
    };
    int done = 0;                                 // tiles whose P has been handed to the MMA warp
    for (int it = 0; it < nkt; ++it) {
      const int sb = it & 1;
      const bool got = __all_sync(0xffffffffu, mbar_wait(&bars->s_full[sb], (it >> 1) & 1));
      if (!got) set_abort(bars);
      tc_fence_after();
      // the tile's keys: half e is block walk.block(2 it + e), this thread's
      // is e = hf; key i of it is token ub + i (visible when <= t); a block
      // the row does not share is masked whole
      int ub;
      {
        const int blk = walk.block(2 * it + hf);
        ub = (blk >= 0 && (!LOCAL || in_set(blk, t, n_init, n_local))) ? 64 * blk : INT_MAX / 2;
      }
      float v[64];                                // raw scores; the scale c > 0 goes into the exponent
      if (got) tmem_load64(tmem + lane_addr + sb * kKeys + hf * 64, v);
      float mx = -INFINITY;
      if (__all_sync(0xffffffffu, ub + 63 <= t)) {          // every key of this half visible to every row of the warp
#pragma unroll
        for (int i = 0; i < 64; ++i) mx = fmaxf(mx, v[i]);
      } else {
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          v[i] = (ub + i <= t) ? v[i] : -INFINITY;
          mx = fmaxf(mx, v[i]);
        }
      }
      mx *= c;                                    // -inf stays -inf
      float* slot = xch + sb * 256;
      slot[r * 2 + hf] = mx;
      // one barrier per tile for the pair: the partner's maximum, and a
      // stop decision both warps take alike; both have read their scores
      // before it, so P may overwrite them after it
      if (bar_red_or(pair, 64, !got || aborted(bars))) { set_abort(bars); ok = false; break; }
      const float m_new = fmaxf(m_run, fmaxf(mx, slot[r * 2 + (hf ^ 1)]));
      const bool none = (m_new == -INFINITY);
      const float alpha = none ? 1.f : ex2(m_run - m_new);
      // P (bf16 pairs) into TMEM columns sb * 128 + hf * 32 .. + 31: key k of the tile in column k / 2
      float lsum = 0.f;
      uint32_t pk[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float p0 = none ? 0.f : ex2(fmaf(v[2 * i], c, -m_new));
        const float p1 = none ? 0.f : ex2(fmaf(v[2 * i + 1], c, -m_new));
        lsum += p0 + p1;
        __nv_bfloat162 b2 = __floats2bfloat162_rn(p0, p1);
        pk[i] = *reinterpret_cast<uint32_t*>(&b2);
      }
      tmem_store32u(tmem + lane_addr + sb * kKeys + hf * 32, pk);
      l_run = l_run * alpha + lsum;
      m_run = m_new;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) { mbar_arrive(&bars->p_full); mbar_arrive(&bars->s_empty[sb]); }
      done = it + 1;
      // the previous tile's P.V has had this tile's softmax to finish
      if (it > 0) fold(it - 1, alpha_prev);
      alpha_prev = alpha;
    }
    if (ok && done > 0) fold(done - 1, alpha_prev);
    // the row sum over both halves (both warps of the pair get here alike)
    xch[512 + r * 2 + hf] = l_run;
    bar_red_or(pair, 64, false);
    const float l_row = l_run + xch[512 + r * 2 + (hf ^ 1)];
    float lse_row = -INFINITY;                    // LOCAL: the row's log-sum-exp over all its keys (log2 units)
    if (ok && t < len) {
      const float inv = (l_row > 0.f) ? 1.f / l_row : 0.f;
      const int64_t base = (static_cast<int64_t>(row0 + t) * h_q + static_cast<int64_t>(g) * G + h) * D + hf * DH;
      float w_own = inv;   // weight of o_acc; the top-k partial (if any) gets w_top
      float w_top = 0.f;
      if (LOCAL) {
        // out[row] holds the top-k partial (normalised) when its log-sum-exp
        // lb (log2 units) is finite; la is this partial's
        const float lb = lse[static_cast<int64_t>(row0 + t) * h_q + static_cast<int64_t>(g) * G + h];
        const float la = (l_row > 0.f) ? m_run + log2f(l_row) : -INFINITY;
        lse_row = la;
        if (lb != -INFINITY && l_row > 0.f) {
          const float mm = fmaxf(la, lb);
          const float wa = ex2(la - mm), wb = ex2(lb - mm);
          const float iw = 1.f / (wa + wb);
          w_own = inv * wa * iw;
          w_top = wb * iw;
          lse_row = mm + log2f(wa + wb);
        }
      }
      if (OUT_F32) {
        float4* o4 = reinterpret_cast<float4*>(reinterpret_cast<float*>(out) + base);
#pragma unroll
        for (int j = 0; j < DH; j += 4) {
          float4 v4 = make_float4(o_acc[j] * w_own, o_acc[j + 1] * w_own, o_acc[j + 2] * w_own, o_acc[j + 3] * w_own);
          if (LOCAL && w_top != 0.f) {
            const float4 b4 = o4[j / 4];
            v4.x = fmaf(b4.x, w_top, v4.x); v4.y = fmaf(b4.y, w_top, v4.y);
            v4.z = fmaf(b4.z, w_top, v4.z); v4.w = fmaf(b4.w, w_top, v4.w);
          }
          o4[j / 4] = v4;
        }
      } else {
        uint4* o4 = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(out) + base);
#pragma unroll
        for (int j = 0; j < DH; j += 8) {
          float top[8];
#pragma unroll
          for (int q = 0; q < 8; ++q) top[q] = 0.f;
          if (LOCAL && w_top != 0.f) {
            const uint4 b4 = o4[j / 8];
            const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&b4);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const float2 f = __bfloat1622float2(b2[q]);
              top[2 * q] = f.x * w_top;
              top[2 * q + 1] = f.y * w_top;
            }
          }
          uint32_t w[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            __nv_bfloat162 b2 = __floats2bfloat162_rn(fmaf(o_acc[j + 2 * q], w_own, top[2 * q]),
                                                      fmaf(o_acc[j + 2 * q + 1], w_own, top[2 * q + 1]));
            w[q] = *reinterpret_cast<uint32_t*>(&b2);
          }
          o4[j / 8] = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
    }
    if (LOCAL) {
      // both threads of the row have read the top-k log-sum-exp: the slot
      // now takes the row's complete one (the statistic a backward pass
      // needs: P = 2^(scale log2(e) q.k - lse))
      bar_red_or(pair, 64, false);
      if (hf == 0 && ok && t < len)
        lse[static_cast<int64_t>(row0 + t) * h_q + static_cast<int64_t>(g) * G + h] = lse_row;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

}  // namespace dense

bool make_tmap(CUtensorMap* map, const void* base, int rank, const uint64_t* dims, const uint64_t* strides_bytes,
               const uint32_t* box);

template <int D, int G, bool F32, bool LOCAL>
static cudaError_t launch_dense_t(const void* Q, const void* K, const void* V, const int32_t* cu, int batch,
                                  int max_seqlen, int64_t total, int h_q, int h_kv, float scale, void* out,
                                  int n_init, int n_local, float* lse, cudaStream_t st, bool* map_fail) {
  using C = dense::Cfg<D, G>;
  CUtensorMap mQ, mK, mV;
  {
    const uint64_t dims[4] = {(uint64_t)D, (uint64_t)G, (uint64_t)h_kv, (uint64_t)total};
    const uint64_t strides[3] = {(uint64_t)D * 2, (uint64_t)G * D * 2, (uint64_t)h_q * D * 2};
    const uint32_t box[4] = {64, (uint32_t)G, 1, (uint32_t)C::TQ};
    if (!make_tmap(&mQ, Q, 4, dims, strides, box)) { *map_fail = true; return cudaErrorInvalidValue; }
  }
  {
    const uint64_t dims[3] = {(uint64_t)D, (uint64_t)h_kv, (uint64_t)total};
    const uint64_t strides[2] = {(uint64_t)D * 2, (uint64_t)h_kv * D * 2};
    const uint32_t box[3] = {64, 1, 64};
    if (!make_tmap(&mK, K, 3, dims, strides, box)) { *map_fail = true; return cudaErrorInvalidValue; }
    if (!make_tmap(&mV, V, 3, dims, strides, box)) { *map_fail = true; return cudaErrorInvalidValue; }
  }
  auto kern = dense::dense_attn_kernel<D, G, F32, LOCAL>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return e;
  dim3 grid((max_seqlen + C::TQ - 1) / C::TQ, batch, h_kv);
  if (grid.x == 0) return cudaSuccess;
  kern<<<grid, dense::kThreads, C::kSmem, st>>>(mQ, mK, mV, cu, h_q, scale, out, n_init, n_local, lse);
  return cudaGetLastError();
}

// Dense causal attention (lse == nullptr), or the LOCAL part of the sparse
// attention: attention over each token's init and local blocks, merged with
// the top-k partial that out and lse ([total, h_q] fp32, log2 units) hold.
cudaError_t launch_dense_attn(const void* Q, const void* K, const void* V, const int32_t* cu, int batch,
                              int max_seqlen, int64_t total, int h_q, int h_kv, int d, float scale, void* out,
                              bool out_f32, int n_init, int n_local, float* lse, cudaStream_t st, bool* map_fail) {
  const int G = h_q / h_kv;
#define INFLLM2_DENSE_CASE(DD, GG)                                                                               \
  if (d == DD && G == GG) {                                                                                     \
    if (lse)                                                                                                    \
      return out_f32 ? launch_dense_t<DD, GG, true, true>(Q, K, V, cu, batch, max_seqlen, total, h_q, h_kv, scale, \
                                                          out, n_init, n_local, lse, st, map_fail)             \
                     : launch_dense_t<DD, GG, false, true>(Q, K, V, cu, batch, max_seqlen, total, h_q, h_kv, scale, \
                                                           out, n_init, n_local, lse, st, map_fail);           \
    return out_f32 ? launch_dense_t<DD, GG, true, false>(Q, K, V, cu, batch, max_seqlen, total, h_q, h_kv, scale, \
                                                         out, 0, 0, nullptr, st, map_fail)                     \
                   : launch_dense_t<DD, GG, false, false>(Q, K, V, cu, batch, max_seqlen, total, h_q, h_kv, scale, \
                                                          out, 0, 0, nullptr, st, map_fail);                   \
  }
  INFLLM2_DENSE_CASE(128, 16)
  INFLLM2_DENSE_CASE(128, 8)
  INFLLM2_DENSE_CASE(128, 4)
  INFLLM2_DENSE_CASE(128, 2)
  INFLLM2_DENSE_CASE(128, 1)
  INFLLM2_DENSE_CASE(64, 16)
  INFLLM2_DENSE_CASE(64, 8)
  INFLLM2_DENSE_CASE(64, 4)
  INFLLM2_DENSE_CASE(64, 2)
  INFLLM2_DENSE_CASE(64, 1)
#undef INFLLM2_DENSE_CASE
  return cudaErrorInvalidValue;
}

}  // namespace infllm2
