// Dense causal attention and the LOCAL part of the block-sparse attention,
// two query tiles per CTA (the short-sequence side of InfLLM-V2's dense/sparse
// switch: paper-reading blog, "Dense-Sparse Switchable Attention"; dtcms
// article §二.2.c; the shared init and local blocks: top168 article §七).
//
// A CTA owns one kv group and 2 TQ consecutive query tokens, TQ = 128/G: two
// 128-row query tiles A and B (rows (t, h), the G heads of each token) that
// share every K/V tile (two 64-key blocks gathered by TMA).  Per key tile j
// the MMA warp issues, in this order,
//   S_A(j) = Q_A . K(j)^T,  O_B += P_B(j-1) . V(j-1),  S_B(j) = Q_B . K(j)^T,
//   O_A += P_A(j) . V(j)
// so the softmax of one tile runs while the tensor core works on the other.
// One thread per row: it reads its 128 scores from TMEM, keeps its own
// reference maximum m (raised only when a score passes it by more than 2^8;
// then it rescales its O row in TMEM after the pending P.V product is done),
// and writes P (bf16) back over its scores, where the P.V product reads it
// as the A operand.  O accumulates in TMEM; nothing crosses threads per tile.
// LOCAL: a row attends only to its own init blocks and local run (the union
// of the CTA's rows is walked) and its partial is merged with the top-k
// partial that out and lse hold (both log-sum-exps, log2 units); the row's
// complete log-sum-exp is written back to lse.
// Warp roles: warp 0 loads Q and the K and V rings (in the order the MMA
// warp frees their slots), warp 1 issues the MMAs and owns TMEM, warps 2-5
// are tile A's rows, 6-9 tile B's.
#include "sm100.cuh"

namespace infllm2 {

namespace pair {

constexpr int kThreads = 320;              // 10 warps
constexpr int kKeys = 128;
#ifndef INFLLM2_PAIR_KSTAGES
#define INFLLM2_PAIR_KSTAGES 2
#endif
#ifndef INFLLM2_PAIR_PIPE
#define INFLLM2_PAIR_PIPE 0
#endif
// LOCAL with bf16 output: the row's top-k partial (d bf16) and its
// log-sum-exp are loaded before the wait for the last P.V, in one batch,
// instead of chunk by chunk between the TMEM reads of the epilogue (each
// TMEM read orders the loads around it, so they went out one round trip
// at a time).
#ifndef INFLLM2_PAIR_PREFETCH
#define INFLLM2_PAIR_PREFETCH 1
#endif
constexpr int kKStages = INFLLM2_PAIR_KSTAGES;
constexpr int kVStages = 2;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescale = 8.f;            // raise m only past this margin (log2 units)

template <int D, int G>
struct Cfg {
  static constexpr int TQ = 128 / G;                      // tokens per query tile
  static constexpr int KCH = D / 64;
  static constexpr uint32_t kQBytes = 128 * 128 * KCH;    // one query tile
  static constexpr uint32_t kChunk = kKeys * 128;         // 128 keys x 64 dims
  static constexpr uint32_t kKBytes = kChunk * KCH;
  static constexpr uint32_t kSmem = 1024 + 2 * kQBytes + (kKStages + kVStages) * kKBytes + 512;
};

struct Bars {
  uint64_t q_full;
  uint64_t k_full[kKStages], k_empty[kKStages];
  uint64_t v_full[kVStages], v_empty[kVStages];
  uint64_t s_full[2];          // per query tile: its S(j) is in TMEM
  uint64_t p_full[2];          // per query tile: its P(j) is in TMEM (4 warps)
  uint64_t pv_done[2];         // per query tile: its P.V product of tile j has completed
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
};
__device__ __forceinline__ bool aborted(const Bars* b) { return *reinterpret_cast<const volatile int*>(&b->abort) != 0; }
__device__ __forceinline__ void set_abort(Bars* b) { *reinterpret_cast<volatile int*>(&b->abort) = 1; }

// The blocks a CTA walks.  Dense: 0 .. t_last/64.  LOCAL: the init blocks
// [0, i_hi) followed by [l_start, b_hi], the union of the init and local
// blocks of the CTA's query tokens (blocks b_lo .. b_hi); block(p) < 0 past
// the end.
struct BlockWalk {
  int i_hi, l_start, nblk;
  __device__ int block(int p) const { return p >= nblk ? -1 : (p < i_hi ? p : l_start + (p - i_hi)); }
};
__device__ __forceinline__ bool in_set(int blk, int t, int n_init, int n_local) {
  const int bt = t >> 6;
  return blk < min(n_init, bt + 1) || blk >= bt - n_local + 1;
}

template <int D, int G, bool OUT_F32, bool LOCAL>
__global__ void __launch_bounds__(kThreads, 1) pair_attn_kernel(
    const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
    const __grid_constant__ CUtensorMap tmV, const int32_t* __restrict__ cu, int h_q, float scale,
    void* __restrict__ out, int n_init, int n_local, float* __restrict__ lse) {
  using C = Cfg<D, G>;
  constexpr int TQ = C::TQ;
  static_assert(G >= 1 && G <= 16 && (16 % G) == 0, "group size must be a power of two <= 16");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                                        // [2] query tiles
  uint8_t* sKr = sQ + 2 * C::kQBytes;                        // K ring
  uint8_t* sVr = sKr + kKStages * C::kKBytes;                // V ring
  Bars* bars = reinterpret_cast<Bars*>(sVr + kVStages * C::kKBytes);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int s = blockIdx.y, g = blockIdx.z;
  const int row0 = cu[s];
  const int len = cu[s + 1] - row0;
  const int ncta = (len + 2 * TQ - 1) / (2 * TQ);
  if (static_cast<int>(blockIdx.x) >= ncta) return;
  const int t0 = (ncta - 1 - blockIdx.x) * 2 * TQ;          // heaviest tiles first
  const int t_last = min(len - 1, t0 + 2 * TQ - 1);
  BlockWalk walk;
  if (LOCAL) {
    const int b_lo = t0 >> 6, b_hi = t_last >> 6;
    walk.i_hi = min(n_init, b_hi + 1);
    walk.l_start = max(walk.i_hi, max(0, b_lo - n_local + 1));
    walk.nblk = walk.i_hi + max(0, b_hi - walk.l_start + 1);
  } else {
    walk.i_hi = t_last / 64 + 1;
    walk.l_start = walk.i_hi;
    walk.nblk = walk.i_hi;
  }
  const int nkt = (walk.nblk + 1) / 2;                   // key tiles of two blocks

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int i = 0; i < kKStages; ++i) { mbar_init(&bars->k_full[i], 1); mbar_init(&bars->k_empty[i], 1); }
    for (int i = 0; i < kVStages; ++i) { mbar_init(&bars->v_full[i], 1); mbar_init(&bars->v_empty[i], 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->s_full[i], 1);
      mbar_init(&bars->p_full[i], 4);
      mbar_init(&bars->pv_done[i], 1);
    }
    mbar_init(&bars->mma_done, 1);
    bars->abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) { tmem_alloc(&bars->tmem_base, 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  // TMEM columns: S / P of tile w at 128 w, O of tile w at 256 + 128 w (d <= 128)

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(&bars->q_full, 2 * C::kQBytes);
      for (int w = 0; w < 2; ++w)
        for (int ch = 0; ch < C::KCH; ++ch)
          tma_load_4d(sQ + w * C::kQBytes + ch * 16384, &tmQ, &bars->q_full, ch * 64, 0, g, row0 + t0 + w * TQ);
      // K(j) then V(j): the MMA warp frees K(j) after S_B(j) and V(j) after
      // O_B += P_B(j) V(j), in that order, so loading in this order never
      // waits on a slot out of turn
      int it = 0;
      bool ok = true;
      for (; ok && it < nkt; ++it) {
        const int ba = walk.block(2 * it);
        int bb = walk.block(2 * it + 1);
        if (bb < 0) bb = ba;                             // odd count: reload, masked by the softmax
        for (int isv = 0; isv < 2; ++isv) {
          const int nst = isv ? kVStages : kKStages;
          const int st = it % nst;
          uint64_t* full = isv ? bars->v_full : bars->k_full;
          uint64_t* empty = isv ? bars->v_empty : bars->k_empty;
          if (!mbar_wait(&empty[st], ((it / nst) & 1) ^ 1) || aborted(bars)) { set_abort(bars); ok = false; break; }
          uint8_t* dst = (isv ? sVr : sKr) + st * C::kKBytes;
          const CUtensorMap* tm = isv ? &tmV : &tmK;
          mbar_arrive_expect_tx(&full[st], C::kKBytes);
          for (int ch = 0; ch < C::KCH; ++ch) {
            tma_load_3d(dst + ch * C::kChunk, tm, &full[st], ch * 64, g, row0 + 64 * ba);
            tma_load_3d(dst + ch * C::kChunk + C::kChunk / 2, tm, &full[st], ch * 64, g, row0 + 64 * bb);
          }
        }
      }
      // wait for every copy still in flight before the CTA may exit (the
      // last tile's K may have been issued without its V)
      mbar_wait(&bars->q_full, 0);
      for (int i = max(0, it - kKStages); i < it; ++i) mbar_wait(&bars->k_full[i % kKStages], (i / kKStages) & 1);
      const int itv = ok ? it : it - 1;
      for (int i = max(0, itv - kVStages); i < itv; ++i) mbar_wait(&bars->v_full[i % kVStages], (i / kVStages) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idS = idesc_bf16_f32(128, kKeys, 0, 0);
      const uint32_t idO = idesc_bf16_f32(128, D, 0, 1);
      bool ok = mbar_wait(&bars->q_full, 0);
      tc_fence_after();
      auto issue_s = [&](int w, int j) -> bool {          // S_w(j) = Q_w . K(j)^T
        const int st = j % kKStages;
        if (w == 0 && !mbar_wait(&bars->k_full[st], (j / kKStages) & 1)) return false;
        tc_fence_after();
        const uint32_t q_base = smem_u32(sQ + w * C::kQBytes);
        const uint32_t k_base = smem_u32(sKr + st * C::kKBytes);
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint64_t a = make_sdesc(q_base + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024, kLayoutSW128);
          const uint64_t b = make_sdesc(k_base + (k >> 2) * C::kChunk + (k & 3) * 32, 16, 1024, kLayoutSW128);
          umma_bf16(tmem + w * 128, a, b, idS, k > 0);
        }
        umma_commit(&bars->s_full[w]);
        if (w == 1) umma_commit(&bars->k_empty[st]);    // both tiles have read K(j)
        return true;
      };
      auto issue_pv = [&](int w, int j) -> bool {         // O_w += P_w(j) . V(j)
        const int st = j % kVStages;
        if (!mbar_wait(&bars->p_full[w], j & 1)) return false;
        if (w == 0 && !mbar_wait(&bars->v_full[st], (j / kVStages) & 1)) return false;
        tc_fence_after();
        const uint32_t v_base = smem_u32(sVr + st * C::kKBytes);
        const uint32_t p_tmem = tmem + w * 128;          // key 2c, 2c+1 of P in column c
#pragma unroll
        for (int k = 0; k < kKeys / 16; ++k) {
          const uint64_t b = make_sdesc(v_base + k * 2048, C::kChunk, 1024, kLayoutSW128);
          umma_bf16_ts(tmem + 256 + w * 128, p_tmem + k * 8, b, idO, (j > 0 || k > 0) ? 1u : 0u);
        }
        umma_commit(&bars->pv_done[w]);
        if (w == 1) umma_commit(&bars->v_empty[st]);    // both tiles have read V(j)
        return true;
      };
      // S_A(j), O_B += P_B(j-1) V(j-1), S_B(j), O_A += P_A(j) V(j)
      for (int j = 0; ok && j < nkt; ++j) {
        if (!issue_s(0, j) || aborted(bars)) { ok = false; break; }
        if (j > 0 && !issue_pv(1, j - 1)) { ok = false; break; }
        if (!issue_s(1, j)) { ok = false; break; }
        if (!issue_pv(0, j)) { ok = false; break; }
      }
      if (ok && nkt > 0 && !issue_pv(1, nkt - 1)) ok = false;
      if (!ok) set_abort(bars);
      umma_commit(&bars->mma_done);
      mbar_wait(&bars->mma_done, 0);
    }
  } else {
    // ------------------------------------------------------------ softmax: one thread per row
    const int w = (warp - 2) >> 2;                // query tile
    const int wq = warp & 3;                      // TMEM lane quadrant
    const int r = wq * 32 + lane;                 // row (t_loc, h) of tile w
    const int t = t0 + w * TQ + r / G;
    const int h = r % G;
    const uint32_t lane_addr = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t t_s = tmem + lane_addr + w * 128;
    const uint32_t t_o = tmem + lane_addr + 256 + w * 128;
    const float c = scale * kLog2e;
    float m_ref = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < nkt; ++j) {
      bool got = mbar_wait(&bars->s_full[w], j & 1);
      tc_fence_after();
      // keys of the tile: half e is block walk.block(2 j + e); key i of it is
      // token ub + i (visible when <= t); a block the row does not share is
      // masked whole
      int ub[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int blk = walk.block(2 * j + e);
        ub[e] = (blk >= 0 && (!LOCAL || in_set(blk, t, n_init, n_local))) ? 64 * blk : INT_MAX / 2;
      }
      // pass 1: the row maximum over both halves (raw scores; the scale c > 0
      // goes into the exponent); the second half stays in registers.  Tiles
      // whose keys every row of the warp sees skip the masking.
      const bool vis = __all_sync(0xffffffffu, ub[0] + 63 <= t && ub[1] + 63 <= t);
      float va[64], vb[64];
      tmem_load64(t_s, va);
#if INFLLM2_PAIR_PIPE
      // the second half's read is in flight while the first half is reduced
      float (&vb0)[32] = *reinterpret_cast<float(*)[32]>(&vb[0]);
      float (&vb1)[32] = *reinterpret_cast<float(*)[32]>(&vb[32]);
      tmem_ld32(t_s + 64, vb0);
      tmem_ld32(t_s + 96, vb1);
#endif
      float mx = -INFINITY;
      if (vis) {
#pragma unroll
        for (int i = 0; i < 64; ++i) mx = fmaxf(mx, va[i]);
      } else {
#pragma unroll
        for (int i = 0; i < 64; ++i) mx = fmaxf(mx, (ub[0] + i <= t) ? va[i] : -INFINITY);
      }
#if INFLLM2_PAIR_PIPE
      tmem_wait_ld32(vb0);
      tmem_wait_ld32(vb1);
#else
      tmem_load64(t_s + 64, vb);
#endif
      if (vis) {
#pragma unroll
        for (int i = 0; i < 64; ++i) mx = fmaxf(mx, vb[i]);
      } else {
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          vb[i] = (ub[1] + i <= t) ? vb[i] : -INFINITY;
          mx = fmaxf(mx, vb[i]);
        }
      }
      mx *= c;                                    // -inf stays -inf
      // a raise of the reference: O (once the pending P.V product is done) and
      // l scale by 2^(m_ref - mx); TMEM is read and written by whole warps
      const bool need = mx > m_ref + kRescale;
      const bool scale_o = need && m_ref != -INFINITY;
      if (__any_sync(0xffffffffu, scale_o)) {
        got = mbar_wait(&bars->pv_done[w], (j - 1) & 1) && got;
        tc_fence_after();
        const float alpha = scale_o ? ex2(m_ref - mx) : 1.f;
#pragma unroll
        for (int cc = 0; cc < D; cc += 16) {
          float o[16];
          tmem_load16(t_o + cc, o);
#pragma unroll
          for (int i = 0; i < 16; ++i) o[i] *= alpha;
          tmem_store16(t_o + cc, o);
        }
        l_run *= alpha;
      }
      if (need) m_ref = mx;
      const bool none = (m_ref == -INFINITY);
      // pass 2: P (bf16 pairs) over the score columns, key 2i, 2i+1 in column
      // i: the second half from registers, then the first half reloaded
      float lsum = 0.f;
      {
        uint32_t pk[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float p0 = none ? 0.f : ex2(fmaf(vb[2 * i], c, -m_ref));
          const float p1 = none ? 0.f : ex2(fmaf(vb[2 * i + 1], c, -m_ref));
          lsum += p0 + p1;
          __nv_bfloat162 b2 = __floats2bfloat162_rn(p0, p1);
          pk[i] = *reinterpret_cast<uint32_t*>(&b2);
        }
        tmem_load64(t_s, va);                     // keys 0..63 again, before columns 32..63 take P of keys 64..127
        tmem_store32u(t_s + 32, pk);
      }
      {
        uint32_t pk[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float x0 = (vis || ub[0] + 2 * i <= t) ? va[2 * i] : -INFINITY;
          const float x1 = (vis || ub[0] + 2 * i + 1 <= t) ? va[2 * i + 1] : -INFINITY;
          const float p0 = none ? 0.f : ex2(fmaf(x0, c, -m_ref));
          const float p1 = none ? 0.f : ex2(fmaf(x1, c, -m_ref));
          lsum += p0 + p1;
          __nv_bfloat162 b2 = __floats2bfloat162_rn(p0, p1);
          pk[i] = *reinterpret_cast<uint32_t*>(&b2);
        }
        tmem_store32u(t_s, pk);
      }
      l_run += lsum;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_full[w]);
      if (__any_sync(0xffffffffu, !got || aborted(bars))) { set_abort(bars); ok = false; break; }
    }
    // ---- the row's output: O / l, merged with the top-k partial (LOCAL).
    // TMEM is read by whole warps; only rows of the sequence are written.
    constexpr bool kPre = LOCAL && !OUT_F32 && INFLLM2_PAIR_PREFETCH;
    uint4 topv[kPre ? D / 8 : 1];
    float lb_pre = -INFINITY;
    if (kPre && t < len) {
      const int64_t rh = static_cast<int64_t>(row0 + t) * h_q + static_cast<int64_t>(g) * G + h;
      lb_pre = lse[rh];
      const uint4* src = reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(out) + rh * D);
#pragma unroll
      for (int q = 0; q < (kPre ? D / 8 : 1); ++q) topv[q] = src[q];
    }
    const bool got = __all_sync(0xffffffffu, ok && (nkt == 0 || mbar_wait(&bars->pv_done[w], (nkt - 1) & 1)));
    tc_fence_after();
    if (!got) {
      set_abort(bars);
    } else {
      const bool row_ok = t < len;
      const int64_t rh = static_cast<int64_t>(row0 + min(t, len - 1)) * h_q + static_cast<int64_t>(g) * G + h;
      const float inv = (l_run > 0.f) ? 1.f / l_run : 0.f;
      float w_own = inv, w_top = 0.f;
      if (LOCAL && row_ok) {
        // lse[rh] holds the top-k partial's log-sum-exp (log2 units; -inf: none)
        const float lb = kPre ? lb_pre : lse[rh];
        const float la = (l_run > 0.f) ? m_ref + log2f(l_run) : -INFINITY;
        float lse_row = la;
        if (lb != -INFINITY && l_run > 0.f) {
          const float mm = fmaxf(la, lb);
          const float wa = ex2(la - mm), wb = ex2(lb - mm);
          const float iw = 1.f / (wa + wb);
          w_own = inv * wa * iw;
          w_top = wb * iw;
          lse_row = mm + log2f(wa + wb);
        }
        lse[rh] = lse_row;                        // one thread per row reads and writes its slot
      }
#pragma unroll
      for (int cc = 0; cc < D; cc += 16) {
        float o[16];
        tmem_load16(t_o + cc, o);
        if (!row_ok) continue;
        if (OUT_F32) {
          float4* o4 = reinterpret_cast<float4*>(reinterpret_cast<float*>(out) + rh * D + cc);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float4 x = make_float4(o[4 * q] * w_own, o[4 * q + 1] * w_own, o[4 * q + 2] * w_own, o[4 * q + 3] * w_own);
            if (LOCAL && w_top != 0.f) {
              const float4 b4 = o4[q];
              x.x = fmaf(b4.x, w_top, x.x); x.y = fmaf(b4.y, w_top, x.y);
              x.z = fmaf(b4.z, w_top, x.z); x.w = fmaf(b4.w, w_top, x.w);
            }
            o4[q] = x;
          }
        } else {
          uint4* o4 = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(out) + rh * D + cc);
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            float top[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) top[e] = 0.f;
            if (LOCAL && w_top != 0.f) {
              const uint4 b4 = kPre ? topv[(cc >> 3) + q] : o4[q];
              const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&b4);
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float2 f = __bfloat1622float2(b2[e]);
                top[2 * e] = f.x * w_top;
                top[2 * e + 1] = f.y * w_top;
              }
            }
            uint32_t wv[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              __nv_bfloat162 b2 = __floats2bfloat162_rn(fmaf(o[8 * q + 2 * e], w_own, top[2 * e]),
                                                        fmaf(o[8 * q + 2 * e + 1], w_own, top[2 * e + 1]));
              wv[e] = *reinterpret_cast<uint32_t*>(&b2);
            }
            o4[q] = make_uint4(wv[0], wv[1], wv[2], wv[3]);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

}  // namespace pair

bool make_tmap(CUtensorMap* map, const void* base, int rank, const uint64_t* dims, const uint64_t* strides_bytes,
               const uint32_t* box);

template <int D, int G, bool F32, bool LOCAL>
static cudaError_t launch_pair_t(const void* Q, const void* K, const void* V, const int32_t* cu, int batch,
                                 int max_seqlen, int64_t total, int h_q, int h_kv, float scale, void* out, int n_init,
                                 int n_local, float* lse, cudaStream_t st, bool* map_fail) {
  using C = pair::Cfg<D, G>;
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
  auto kern = pair::pair_attn_kernel<D, G, F32, LOCAL>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return e;
  dim3 grid((max_seqlen + 2 * C::TQ - 1) / (2 * C::TQ), batch, h_kv);
  if (grid.x == 0) return cudaSuccess;
  kern<<<grid, pair::kThreads, C::kSmem, st>>>(mQ, mK, mV, cu, h_q, scale, out, n_init, n_local, lse);
  return cudaGetLastError();
}

cudaError_t launch_pair_attn(const void* Q, const void* K, const void* V, const int32_t* cu, int batch,
                             int max_seqlen, int64_t total, int h_q, int h_kv, int d, float scale, void* out,
                             bool out_f32, int n_init, int n_local, float* lse, cudaStream_t st, bool* map_fail) {
  const int G = h_q / h_kv;
#define INFLLM2_PAIR_CASE(DD, GG)                                                                              \
  if (d == DD && G == GG) {                                                                                   \
    if (lse)                                                                                                  \
      return out_f32 ? launch_pair_t<DD, GG, true, true>(Q, K, V, cu, batch, max_seqlen, total, h_q, h_kv, scale, \
                                                         out, n_init, n_local, lse, st, map_fail)            \
                     : launch_pair_t<DD, GG, false, true>(Q, K, V, cu, batch, max_seqlen, total, h_q, h_kv, scale, \
                                                          out, n_init, n_local, lse, st, map_fail);          \
    return out_f32 ? launch_pair_t<DD, GG, true, false>(Q, K, V, cu, batch, max_seqlen, total, h_q, h_kv, scale, \
                                                        out, 0, 0, nullptr, st, map_fail)                    \
                   : launch_pair_t<DD, GG, false, false>(Q, K, V, cu, batch, max_seqlen, total, h_q, h_kv, scale, \
                                                         out, 0, 0, nullptr, st, map_fail);                  \
  }
  INFLLM2_PAIR_CASE(128, 16)
  INFLLM2_PAIR_CASE(128, 8)
  INFLLM2_PAIR_CASE(128, 4)
  INFLLM2_PAIR_CASE(128, 2)
  INFLLM2_PAIR_CASE(128, 1)
  INFLLM2_PAIR_CASE(64, 16)
  INFLLM2_PAIR_CASE(64, 8)
  INFLLM2_PAIR_CASE(64, 4)
  INFLLM2_PAIR_CASE(64, 2)
  INFLLM2_PAIR_CASE(64, 1)
#undef INFLLM2_PAIR_CASE
  return cudaErrorInvalidValue;
}

}  // namespace infllm2
