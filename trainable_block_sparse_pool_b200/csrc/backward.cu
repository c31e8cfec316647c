// Backward of the block-sparse attention over a fixed selection (InfLLM-V2
// trains the sparse attention end to end with no added parameters: dtcms
// article §二 and top168 article §一; the paper-reading blog, "训练是怎么做的").
// The block lists carry no gradient; the loss reaches Q, K and V through the
// attention over the selected keys.  For row (t, h) of kv group g, with
// c = scale * log2(e), P = 2^(c q.k - lse) (lse: the forward's row
// log-sum-exp, log2 units), Dsum = sum_d dO . O:
//   dV[u]  = sum_rows P dO            dP = dO . V[u]
//   dS     = P (dP - Dsum)
//   dQ     = scale sum_u dS K[u]      dK[u] = scale sum_rows dS q
//
// Seven launches, all on the caller's stream, none waiting on another CTA:
//   prep     Dsum per row; clears the inverse-list bitmap
//   bitmap   bit t of (g, s, kb) set when token t's top-k part holds block kb
//   count    rows per (g, s, kb): the init/local tokens (a contiguous range)
//            plus the bitmap's bits
//   scan     exclusive offsets of those counts (one CTA)
//   fill     the row list of every (g, s, kb), ascending in t
//   dQ       per (kv group, token), over the row's whole list: the forward's
//            swap-AB form (keys on the MMA's M side, the G heads on N)
//              S^T  = K_pair . Q^T,  dP^T = V_pair . dO^T      (M=128, N=16)
//              dQ^T += K_pair^T . dS^T                          (M=d,   N=16)
//   dK/dV    one CTA per (kv group, sequence, key block), over the rows
//            that selected the block, TQ = 128/G tokens (128 rows) at a time:
//              S  = Q_c . K_blk^T,  dP = dO_c . V_blk^T        (M=128, N=64)
//              dV^T += dO_c^T . P,  dK^T += Q_c^T . dS         (M=d,   N=64)
//            The row lists are ascending and each key block is summed by one
//            CTA, so the result is the same from run to run (no atomics on
//            the gradients).
#include "sm100.cuh"

namespace infllm2 {

namespace bwd {

constexpr float kLog2e = 1.4426950408889634f;

struct Args {
  const int32_t* block_idx;   // [h_kv, total, n_sel]
  const int32_t* cu;          // [batch + 1]
  int batch, max_seqlen, nb_max, words;   // nb_max = ceil(max_seqlen / 64), words = ceil(max_seqlen / 32)
  int64_t total;
  int h_q, h_kv, n_sel, n_init, n_local;
  float scale;
  const float* lse;           // [total, h_q] log2 units
  float* dsum;                // [total, h_q]
  uint32_t* bitmap;           // [h_kv, batch, nb_max, words]
  int32_t* counts;            // [h_kv * batch * nb_max]
  int32_t* offsets;           // [h_kv * batch * nb_max + 1]
  int32_t* rows;              // the row lists: token positions within the sequence
  float* dQ;                  // [total, h_q, d]
  float* dK;                  // [total, h_kv, d]
  float* dV;
};

__device__ __forceinline__ int ntasks(const Args& a) { return a.h_kv * a.batch * a.nb_max; }

// The list of unit (g, row): positions [0, i_hi) init, [i_hi, i_hi + ntop)
// top-k, then the local run (the form check_lists_kernel verifies).
struct ListForm {
  int t, s, row0, i_hi, l_start, bt, ntop, nall;
};
__device__ __forceinline__ ListForm list_form(const Args& a, int g, int64_t row, const int32_t* list) {
  ListForm f;
  f.s = find_sequence(a.cu, a.batch, row);
  f.row0 = a.cu[f.s];
  f.t = static_cast<int>(row - f.row0);
  f.bt = f.t >> 6;
  f.i_hi = min(a.n_init, f.bt + 1);
  f.l_start = max(f.i_hi, max(0, f.bt - a.n_local + 1));
  int nall = 0;
  for (int i = 0; i < a.n_sel; ++i) nall += (__ldg(list + i) >= 0);
  f.nall = nall;
  f.ntop = max(0, nall - (f.i_hi + max(0, f.bt - f.l_start + 1)));
  return f;
}

// ---------------------------------------------------------------- prep: Dsum, bitmap clear
// Dsum[row, h] = sum_d dO[row, h, d] * O[row, h, d]: 16 lanes per (row, h),
// 8 elements (one 16-byte load of dO) each.
template <int D, bool O_F32>
__global__ void __launch_bounds__(256) prep_kernel(const Args a, const __nv_bfloat16* __restrict__ dO,
                                                   const void* __restrict__ O) {
  const int64_t nrh = a.total * a.h_q;
  const int64_t nthr = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  constexpr int LPR = D / 8;                       // lanes per (row, h)
  const int lane = threadIdx.x & 31;
  // warp-uniform trip count: the shuffles below need every lane
  for (int64_t base = tid - lane; base < nrh * LPR; base += nthr) {
    const int64_t i = base + lane;
    const bool in = i < nrh * LPR;
    const int64_t rh = in ? i / LPR : 0;
    const int part = static_cast<int>(i % LPR);
    const uint4 g4 = in ? __ldg(reinterpret_cast<const uint4*>(dO + rh * D) + part) : make_uint4(0, 0, 0, 0);
    const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&g4);
    float acc = 0.f;
    if (!in) {
    } else if (O_F32) {
      const float4* o4 = reinterpret_cast<const float4*>(static_cast<const float*>(O) + rh * D) + 2 * part;
      const float4 a0 = __ldg(o4), a1 = __ldg(o4 + 1);
      const float ov[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 gf = __bfloat1622float2(g2[q]);
        acc = fmaf(gf.x, ov[2 * q], fmaf(gf.y, ov[2 * q + 1], acc));
      }
    } else {
      const uint4 o4 = __ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(O) + rh * D) + part);
      const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&o4);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 gf = __bfloat1622float2(g2[q]);
        const float2 of = __bfloat1622float2(o2[q]);
        acc = fmaf(gf.x, of.x, fmaf(gf.y, of.y, acc));
      }
    }
    // the LPR lanes of (row, h) are consecutive threads of one warp (LPR divides 32)
#pragma unroll
    for (int o = LPR / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (in && part == 0) a.dsum[rh] = acc;
  }
  const int64_t nw = static_cast<int64_t>(ntasks(a)) * a.words;
  for (int64_t i = tid; i < nw; i += nthr) a.bitmap[i] = 0u;
}

// ---------------------------------------------------------------- bitmap of the top-k parts
// One warp per unit (g, row): bit t of (g, s, kb) for each top-k entry kb.
__global__ void __launch_bounds__(256) bitmap_kernel(const Args a) {
  const int lane = threadIdx.x & 31;
  const int64_t n_units = static_cast<int64_t>(a.h_kv) * a.total;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t u = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); u < n_units;
       u += stride) {
    const int g = static_cast<int>(u / a.total);
    const int64_t row = u - static_cast<int64_t>(g) * a.total;
    const int32_t* list = a.block_idx + u * a.n_sel;
    const ListForm f = list_form(a, g, row, list);
    uint32_t* bm = a.bitmap + (static_cast<int64_t>(g) * a.batch + f.s) * a.nb_max * a.words;
    for (int i = lane; i < f.ntop; i += 32) {
      const int kb = __ldg(list + f.i_hi + i);
      if (kb >= 0 && kb < a.nb_max && kb <= f.bt)
        atomicOr(bm + static_cast<int64_t>(kb) * a.words + (f.t >> 5), 1u << (f.t & 31));
    }
  }
}

// Token range of (s, kb) whose lists hold kb outside their top-k part: every
// token from 64 kb on when kb is an init block, else the tokens whose local
// run holds kb (blocks kb .. kb + n_local - 1).
__device__ __forceinline__ void shared_range(const Args& a, int len, int kb, int* lo, int* hi) {
  *lo = 64 * kb;
  *hi = (kb < a.n_init) ? len : min(len, 64 * (kb + a.n_local));
  if (*lo > *hi) *hi = *lo;
}

// ---------------------------------------------------------------- counts: one warp per task
__global__ void __launch_bounds__(256) count_kernel(const Args a) {
  const int lane = threadIdx.x & 31;
  const int n = ntasks(a);
  for (int task = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); task < n;
       task += gridDim.x * (blockDim.x >> 5)) {
    const int kb = task % a.nb_max;
    const int s = (task / a.nb_max) % a.batch;
    const int len = a.cu[s + 1] - a.cu[s];
    int c = 0;
    if (64 * kb < len) {
      const uint32_t* bm = a.bitmap + static_cast<int64_t>(task) * a.words;
      const int wn = (len + 31) >> 5;
      for (int w = lane; w < wn; w += 32) c += __popc(__ldg(bm + w));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
      int lo, hi;
      shared_range(a, len, kb, &lo, &hi);
      c += hi - lo;
    }
    if (lane == 0) a.counts[task] = c;
  }
}

// ---------------------------------------------------------------- exclusive scan of the counts (one CTA)
__global__ void __launch_bounds__(1024) scan_kernel(const Args a) {
  __shared__ int wsum[32];
  __shared__ int carry;
  const int n = ntasks(a);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < n; base += 1024) {
    const int i = base + threadIdx.x;
    const int v = (i < n) ? a.counts[i] : 0;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) wsum[warp] = x;
    __syncthreads();
    int before = 0, tot = 0;
    for (int w = 0; w < 32; ++w) {
      before += (w < warp) ? wsum[w] : 0;
      tot += wsum[w];
    }
    if (i < n) a.offsets[i] = carry + before + x - v;
    __syncthreads();
    if (threadIdx.x == 0) carry += tot;
    __syncthreads();
  }
  if (threadIdx.x == 0) a.offsets[n] = carry;
}

// ---------------------------------------------------------------- fill: one warp per task, ascending t
__global__ void __launch_bounds__(256) fill_kernel(const Args a) {
  const int lane = threadIdx.x & 31;
  const int n = ntasks(a);
  for (int task = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); task < n;
       task += gridDim.x * (blockDim.x >> 5)) {
    const int kb = task % a.nb_max;
    const int s = (task / a.nb_max) % a.batch;
    const int len = a.cu[s + 1] - a.cu[s];
    if (64 * kb >= len) continue;
    int32_t* out = a.rows + a.offsets[task];
    int lo, hi;
    shared_range(a, len, kb, &lo, &hi);
    // the bitmap's tokens all come after the shared range (a top-k block is
    // at least n_local blocks before its token's block); merge by position
    int pos = 0;
    const uint32_t* bm = a.bitmap + static_cast<int64_t>(task) * a.words;
    const int wn = (len + 31) >> 5;
    for (int w0 = 0; w0 < wn; w0 += 32) {
      const int w = w0 + lane;
      const uint32_t bits = (w < wn) ? __ldg(bm + w) : 0u;
      // shared-range tokens in this lane's 32 positions
      const int r_lo = max(lo, 32 * w), r_hi = min(hi, 32 * w + 32);
      const int nsh = max(0, r_hi - r_lo);
      const int cnt = nsh + __popc(bits);
      int x = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      int p = pos + x - cnt;
      // positions 32 w .. 32 w + 31 in order: each is either in the shared
      // range or a bitmap bit (never both)
      uint32_t b = bits;
      for (int q = r_lo; q < r_hi; ++q) {
        // bits below q come first
        while (b && (32 * w + __ffs(b) - 1) < q) {
          out[p++] = 32 * w + __ffs(b) - 1;
          b &= b - 1;
        }
        out[p++] = q;
      }
      while (b) {
        out[p++] = 32 * w + __ffs(b) - 1;
        b &= b - 1;
      }
      pos += __shfl_sync(0xffffffffu, x, 31);
    }
  }
}

// ---------------------------------------------------------------- dQ: per (kv group, token)
// One thread issues tcgen05.mma at about one product per 100-180 cycles
// (measured on the B200 for M=128 chains, whatever N), so the products of a
// tile are spread over several issuing threads: S and dP of the dQ kernel
// from two threads (1 and 2), and the dK/dV kernel's four products from two
// threads ({S, dV^T}, {dP, dK^T}: 1) or four (one each: 2).  0 restores one
// issuer for them.
#ifndef INFLLM2_BWD_SPLIT
#define INFLLM2_BWD_SPLIT 2
#endif
constexpr bool kBwdSplit = INFLLM2_BWD_SPLIT != 0;
// The dK/dV kernel's row threads fetch their rows' token ids two chunks
// ahead and the rows' log-sum-exp and Dsum one chunk ahead, so the two
// dependent global loads of a chunk are in flight during the chunk before
// instead of opening it.
#ifndef INFLLM2_BWD_ROWS_AHEAD
#define INFLLM2_BWD_ROWS_AHEAD 1
#endif
// warp 0 K/Q/dO producer, 1 S (and dP) MMA, 2-5 softmax, 6 V producer, 7 dQ MMA, 8 (split) dP MMA
constexpr int kQThreads = kBwdSplit ? 288 : 256;
constexpr int kQVWarp = 6;
constexpr int kQDqWarp = 7;
constexpr int kQDpWarp = 8;

template <int D>
struct QCfg {
  static constexpr int KCH = D / 64;
  static constexpr uint32_t kChunk = 128 * 128;                // 128 keys x 64 dims
  static constexpr uint32_t kHalf = 64 * 128;
  static constexpr uint32_t kKBytes = kChunk * KCH;
  static constexpr int kKStages = (D == 128) ? 3 : 5;
  static constexpr int kVStages = (D == 128) ? 2 : 4;
  static constexpr uint32_t kQBuf = 2048 * KCH;                // 16 head rows x d
  static constexpr uint32_t kDSBuf = 128 * 16 * 2;
  static constexpr uint32_t kSmem =
      1024 + (kKStages + kVStages) * kKBytes + 4 * kQBuf + 2 * kDSBuf + 512;
};

struct QBars {
  uint64_t k_full[8], k_empty[8], v_full[8], v_empty[8];
  uint64_t q_full[2], q_empty[2];
  uint64_t s_full[2], s_empty[2];
  uint64_t ds_full[2], ds_empty[2];
  uint64_t dq_full[2], dq_empty[2];
  uint64_t mma_done, dq_done, dp_done;   // each MMA issuer's own products have completed
  uint32_t tmem_base;
  int abort;
};
__device__ __forceinline__ bool q_aborted(const QBars* b) { return *reinterpret_cast<const volatile int*>(&b->abort) != 0; }
__device__ __forceinline__ void q_set_abort(QBars* b) { *reinterpret_cast<volatile int*>(&b->abort) = 1; }

struct QUnit {
  int g, t, row0, nvalid;
  int64_t row;
  const int32_t* I;
};
__device__ __forceinline__ QUnit q_unit(int64_t u, const Args& a) {
  QUnit x;
  x.g = static_cast<int>(u / a.total);
  x.row = u - static_cast<int64_t>(x.g) * a.total;
  const int s = find_sequence(a.cu, a.batch, x.row);
  x.row0 = a.cu[s];
  x.t = static_cast<int>(x.row - x.row0);
  x.I = a.block_idx + u * a.n_sel;
  int nv = 0;
  if ((a.n_sel & 3) == 0) {                 // rows of n_sel ints start 16-byte aligned
    const int4* I4 = reinterpret_cast<const int4*>(x.I);
#pragma unroll 8
    for (int i = 0; i < a.n_sel / 4; ++i) {
      const int4 v = __ldg(I4 + i);
      nv += (v.x >= 0) + (v.y >= 0) + (v.z >= 0) + (v.w >= 0);
    }
  } else {
    for (int i = 0; i < a.n_sel; ++i) nv += (__ldg(x.I + i) >= 0);
  }
  x.nvalid = nv;
  return x;
}
__device__ __forceinline__ int list_at(const QUnit& x, int e) { return (e < x.nvalid) ? __ldg(x.I + e) : -1; }

template <int D, int G>
__global__ void __launch_bounds__(kQThreads, 1) dq_kernel(const __grid_constant__ CUtensorMap tmQ,
                                                          const __grid_constant__ CUtensorMap tmdO,
                                                          const __grid_constant__ CUtensorMap tmK,
                                                          const __grid_constant__ CUtensorMap tmV, const Args a) {
  using C = QCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sKr = smem;
  uint8_t* sVr = sKr + C::kKStages * C::kKBytes;
  uint8_t* sQ = sVr + C::kVStages * C::kKBytes;            // [2] Q buffers, then [2] dO buffers
  uint8_t* sdO = sQ + 2 * C::kQBuf;
  uint8_t* sdS = sdO + 2 * C::kQBuf;                        // [2]
  QBars* bars = reinterpret_cast<QBars*>(sdS + 2 * C::kDSBuf);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t n_units = static_cast<int64_t>(a.h_kv) * a.total;
  const int64_t my_units = (n_units > blockIdx.x) ? (n_units - 1 - blockIdx.x) / gridDim.x + 1 : 0;

  for (int i = threadIdx.x; i < static_cast<int>(4 * C::kQBuf / 16); i += kQThreads)
    reinterpret_cast<uint4*>(sQ)[i] = make_uint4(0, 0, 0, 0);   // head rows past G stay zero
  fence_proxy_async_smem();
  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kKStages; ++i) { mbar_init(&bars->k_full[i], 1); mbar_init(&bars->k_empty[i], 1); }
    for (int i = 0; i < C::kVStages; ++i) { mbar_init(&bars->v_full[i], 1); mbar_init(&bars->v_empty[i], 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->q_full[i], 1);
      mbar_init(&bars->q_empty[i], kBwdSplit ? 2 : 1);   // Q read by S, dO by dP
      mbar_init(&bars->s_full[i], kBwdSplit ? 2 : 1);    // S and dP both in TMEM
      mbar_init(&bars->s_empty[i], 4);
      mbar_init(&bars->ds_full[i], 4);
      mbar_init(&bars->ds_empty[i], 1);
      mbar_init(&bars->dq_full[i], 1);
      mbar_init(&bars->dq_empty[i], 4);
    }
    mbar_init(&bars->mma_done, 1);
    mbar_init(&bars->dq_done, 1);
    mbar_init(&bars->dp_done, 1);
    bars->abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) { tmem_alloc(&bars->tmem_base, 128); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  // TMEM columns: S^T[sb] at 16 sb, dP^T[sb] at 32 + 16 sb, dQ^T[ub] at 64 + 16 ub

  if (warp == 0 || warp == kQVWarp) {
    // ------------------------------------------------------------ producers (lane 0)
    if (lane == 0) {
      const bool isV = (warp == kQVWarp);
      const int nst = isV ? C::kVStages : C::kKStages;
      const CUtensorMap* tm = isV ? &tmV : &tmK;
      uint8_t* ring = isV ? sVr : sKr;
      uint64_t* full = isV ? bars->v_full : bars->k_full;
      uint64_t* empty = isV ? bars->v_empty : bars->k_empty;
      tma_prefetch_desc(tm);
      if (!isV) { tma_prefetch_desc(&tmQ); tma_prefetch_desc(&tmdO); }
      int it = 0, uc = 0;
      bool ok = true;
      for (int64_t k = 0; ok && k < my_units; ++k, ++uc) {
        const QUnit x = q_unit(blockIdx.x + k * gridDim.x, a);
        if (!isV) {
          const int qb = uc & 1;
          if (!mbar_wait(&bars->q_empty[qb], ((uc >> 1) & 1) ^ 1) || q_aborted(bars)) { q_set_abort(bars); ok = false; break; }
          mbar_arrive_expect_tx(&bars->q_full[qb], 2 * C::KCH * G * 128);
          for (int ch = 0; ch < C::KCH; ++ch) {
            tma_load_4d(sQ + qb * C::kQBuf + ch * 2048, &tmQ, &bars->q_full[qb], ch * 64, 0, x.g, static_cast<int>(x.row));
            tma_load_4d(sdO + qb * C::kQBuf + ch * 2048, &tmdO, &bars->q_full[qb], ch * 64, 0, x.g, static_cast<int>(x.row));
          }
        }
        const int nt = (x.nvalid + 1) >> 1;
        for (int j = 0; ok && j < nt; ++j, ++it) {
          const int b0 = list_at(x, 2 * j);
          int b1 = list_at(x, 2 * j + 1);
          if (b1 < 0) b1 = b0;             // odd count: reload the first block, masked by the softmax
          const int st = it % nst;
          if (!mbar_wait(&empty[st], ((it / nst) & 1) ^ 1) || q_aborted(bars)) { q_set_abort(bars); ok = false; break; }
          uint8_t* dst = ring + st * C::kKBytes;
          mbar_arrive_expect_tx(&full[st], C::kKBytes);
          for (int ch = 0; ch < C::KCH; ++ch) {
            tma_load_3d(dst + ch * C::kChunk, tm, &full[st], ch * 64, x.g, x.row0 + 64 * b0);
            tma_load_3d(dst + ch * C::kChunk + C::kHalf, tm, &full[st], ch * 64, x.g, x.row0 + 64 * b1);
          }
        }
      }
      // wait for every copy still in flight before the CTA may exit
      for (int i = max(0, it - nst); i < it; ++i) mbar_wait(&full[i % nst], (i / nst) & 1);
      if (!isV)
        for (int i = max(0, uc - 2); i < uc; ++i) mbar_wait(&bars->q_full[i & 1], (i >> 1) & 1);
    }
  } else if (warp == 1 || (kBwdSplit && warp == kQDpWarp)) {
    // ------------------------------------------------------------ S / dP issuer(s)
    // per tile: S^T = K_pair Q^T and dP^T = V_pair dO^T (with the split, S
    // from warp 1 and dP from warp kQDpWarp); the V slot is free once dP is
    // done, the K slot only after the dQ product (warp kQDqWarp)
    const bool do_s = (warp == 1), do_dp = !kBwdSplit || warp == kQDpWarp;
    if (lane == 0) {
      const uint32_t idS = idesc_bf16_f32(128, 16, 0, 0);
      int kit = 0, vit = 0, tc = 0, uc = 0;
      bool ok = true;
      for (int64_t k = 0; ok && k < my_units; ++k, ++uc) {
        const QUnit x = q_unit(blockIdx.x + k * gridDim.x, a);
        const int nt = (x.nvalid + 1) >> 1;
        const int qb = uc & 1;
        if (!mbar_wait(&bars->q_full[qb], (uc >> 1) & 1) || q_aborted(bars)) { q_set_abort(bars); ok = false; break; }
        tc_fence_after();
        const uint32_t q_base = smem_u32(sQ + qb * C::kQBuf);
        const uint32_t do_base = smem_u32(sdO + qb * C::kQBuf);
        for (int j = 0; ok && j < nt; ++j, ++kit, ++vit, ++tc) {
          const int kst = kit % C::kKStages, vst = vit % C::kVStages, sb = tc & 1;
          if ((do_s && !mbar_wait(&bars->k_full[kst], (kit / C::kKStages) & 1)) ||
              (do_dp && !mbar_wait(&bars->v_full[vst], (vit / C::kVStages) & 1)) ||
              !mbar_wait(&bars->s_empty[sb], ((tc >> 1) & 1) ^ 1) || q_aborted(bars)) {
            q_set_abort(bars); ok = false; break;
          }
          tc_fence_after();
          const uint32_t k_base = smem_u32(sKr + kst * C::kKBytes);
          const uint32_t v_base = smem_u32(sVr + vst * C::kKBytes);
          if (do_s) {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint64_t ak = make_sdesc(k_base + (kk >> 2) * C::kChunk + (kk & 3) * 32, 16, 1024, kLayoutSW128);
              const uint64_t bq = make_sdesc(q_base + (kk >> 2) * 2048 + (kk & 3) * 32, 16, 1024, kLayoutSW128);
              umma_bf16(tmem + 16 * sb, ak, bq, idS, kk > 0);
            }
          }
          if (do_dp) {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint64_t av = make_sdesc(v_base + (kk >> 2) * C::kChunk + (kk & 3) * 32, 16, 1024, kLayoutSW128);
              const uint64_t bo = make_sdesc(do_base + (kk >> 2) * 2048 + (kk & 3) * 32, 16, 1024, kLayoutSW128);
              umma_bf16(tmem + 32 + 16 * sb, av, bo, idS, kk > 0);
            }
          }
          umma_commit(&bars->s_full[sb]);
          if (do_dp) umma_commit(&bars->v_empty[vst]);
        }
        if (ok) umma_commit(&bars->q_empty[qb]);         // Q and dO are read by S and dP only
      }
      uint64_t* done = do_s ? &bars->mma_done : &bars->dp_done;
      umma_commit(done);
      mbar_wait(done, 0);
    }
  } else if (warp == kQDqWarp) {
    // ------------------------------------------------------------ dQ issuer
    // per tile, once its dS is in shared memory: dQ^T += K_pair^T dS^T
    if (lane == 0) {
      const uint32_t idQ = idesc_bf16_f32(128, 16, 1, 1);
      const uint32_t lboK = (D == 128) ? C::kChunk : 0u;    // d = 64: rows 64-127 of dQ^T repeat 0-63
      int kit = 0, tc = 0, uc = 0;
      bool ok = true;
      for (int64_t k = 0; ok && k < my_units; ++k, ++uc) {
        const QUnit x = q_unit(blockIdx.x + k * gridDim.x, a);
        const int nt = (x.nvalid + 1) >> 1;
        const int ub = uc & 1;
        if (!mbar_wait(&bars->dq_empty[ub], ((uc >> 1) & 1) ^ 1) || q_aborted(bars)) {
          q_set_abort(bars); ok = false; break;
        }
        tc_fence_after();
        const uint32_t dq_addr = tmem + 64 + 16 * ub;
        for (int j = 0; ok && j < nt; ++j, ++kit, ++tc) {
          const int kst = kit % C::kKStages, sb = tc & 1;
          if (!mbar_wait(&bars->ds_full[sb], (tc >> 1) & 1) || q_aborted(bars)) { q_set_abort(bars); ok = false; break; }
          tc_fence_after();
          const uint32_t k_base = smem_u32(sKr + kst * C::kKBytes);
          const uint32_t ds_base = smem_u32(sdS + sb * C::kDSBuf);
#pragma unroll
          for (int kk = 0; kk < 128 / 16; ++kk) {
            const uint64_t ad = make_sdesc(k_base + kk * 2048, lboK, 1024, kLayoutSW128);
            const uint64_t bd = make_sdesc(ds_base + kk * 512, 256, 128, kLayoutNone);
            umma_bf16(dq_addr, ad, bd, idQ, (j > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&bars->k_empty[kst]);
          umma_commit(&bars->ds_empty[sb]);
        }
        if (ok) umma_commit(&bars->dq_full[ub]);
      }
      umma_commit(&bars->dq_done);
      mbar_wait(&bars->dq_done, 0);
    }
  } else {
    // ------------------------------------------------------------ softmax warps 2..5 (one key lane each)
    const int wq = warp & 3;
    const int kl = wq * 32 + lane;            // key lane of the pair tile; d row of dQ^T
    const int half = kl >> 6;
    const uint32_t lane_addr = static_cast<uint32_t>(wq * 32) << 16;
    const float c = a.scale * kLog2e;
    int tc = 0, uc = 0;
    bool stop = false;
    for (int64_t k = 0; !stop && k < my_units; ++k, ++uc) {
      const QUnit x = q_unit(blockIdx.x + k * gridDim.x, a);
      const int nt = (x.nvalid + 1) >> 1;
      const int ub = uc & 1;
      float lse[16], ds0[16];
#pragma unroll
      for (int h = 0; h < 16; ++h) {
        const int64_t rh = x.row * a.h_q + static_cast<int64_t>(x.g) * G + h;
        lse[h] = (h < G) ? __ldg(a.lse + rh) : 0.f;
        ds0[h] = (h < G) ? __ldg(a.dsum + rh) : 0.f;
      }
      for (int j = 0; j < nt; ++j, ++tc) {
        const int sb = tc & 1;
        bool ab = !mbar_wait(&bars->s_full[sb], (tc >> 1) & 1);
        tc_fence_after();
        float sv[16], pv[16];
        tmem_load16(tmem + lane_addr + 16 * sb, sv);
        tmem_load16(tmem + lane_addr + 32 + 16 * sb, pv);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->s_empty[sb]);
        const int blk = list_at(x, 2 * j + half);
        const int pos = 64 * blk + (kl & 63);
        const bool valid = (blk >= 0) && (pos <= x.t);
        uint32_t pk[8];
#pragma unroll
        for (int h = 0; h < 16; h += 2) {
          float d0 = 0.f, d1 = 0.f;
          if (valid && h < G) {
            const float p0 = ex2(fmaf(sv[h], c, -lse[h]));
            d0 = p0 * (pv[h] - ds0[h]);
          }
          if (valid && h + 1 < G) {
            const float p1 = ex2(fmaf(sv[h + 1], c, -lse[h + 1]));
            d1 = p1 * (pv[h + 1] - ds0[h + 1]);
          }
          __nv_bfloat162 b2 = __floats2bfloat162_rn(d0, d1);
          pk[h >> 1] = *reinterpret_cast<uint32_t*>(&b2);
        }
        // dS buffer sb was last read by the dQ product of tile tc - 2
        if (tc >= 2 && !mbar_wait(&bars->ds_empty[sb], ((tc - 2) >> 1) & 1)) ab = true;
        uint8_t* dbuf = sdS + sb * C::kDSBuf;
        const uint32_t off = (kl >> 3) * 256 + (kl & 7) * 16;
        *reinterpret_cast<uint4*>(dbuf + off) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        *reinterpret_cast<uint4*>(dbuf + off + 128) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->ds_full[sb]);
        // the four warps need no common step per tile: each stops on its own
        // failed wait (the others' bounded waits then run out too)
        if (__any_sync(0xffffffffu, ab || q_aborted(bars))) { q_set_abort(bars); stop = true; break; }
      }
      if (stop) break;
      // ---- unit done: dQ = scale * dQ^T, this lane's d row
      const bool got = mbar_wait(&bars->dq_full[ub], (uc >> 1) & 1);
      tc_fence_after();
      float qv[16];
      tmem_load16(tmem + lane_addr + 64 + 16 * ub, qv);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->dq_empty[ub]);
      if (__any_sync(0xffffffffu, !got || q_aborted(bars))) { q_set_abort(bars); stop = true; break; }
      if (kl < D) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const int64_t idx = (x.row * a.h_q + static_cast<int64_t>(x.g) * G + h) * D + kl;
          a.dQ[idx] = (nt > 0) ? a.scale * qv[h] : 0.f;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 128);
}

// ---------------------------------------------------------------- dK / dV: per (kv group, sequence, key block)
// MMA issuers of the dK/dV kernel and the products each issues (bit 1 S,
// 2 dP, 4 dV^T, 8 dK^T): one issuer for all four, two ({S, dV^T}, {dP,
// dK^T}), or, with INFLLM2_BWD_SPLIT=2, one per product.
constexpr int kKVIssuers = (INFLLM2_BWD_SPLIT >= 2) ? 4 : (kBwdSplit ? 2 : 1);
__host__ __device__ constexpr uint32_t kv_issuer_mask(int i) {
  return kKVIssuers == 1 ? 15u : kKVIssuers == 2 ? (i == 0 ? 5u : 10u) : (1u << i);
}
// warp 0 producer, 1 the first MMA issuer, 2-5 softmax / epilogue, 6 .. the other issuers
constexpr int kKVThreads = 192 + 32 * (kKVIssuers - 1);
constexpr int kKVIssuerB = 6;
constexpr uint32_t kKVFront = (kKVIssuers == 4) ? 2u : static_cast<uint32_t>(kKVIssuers);   // issuers of S / dP
constexpr uint32_t kKVBack = kKVFront;                                                       // issuers of dV^T / dK^T

template <int D>
struct KVCfg {
  static constexpr int KCH = D / 64;
  static constexpr uint32_t kBlk = 64 * 128 * KCH;             // one 64-key block (K or V), all d
  static constexpr uint32_t kRowsChunk = 128 * 128;            // 128 rows x 64 dims
  static constexpr uint32_t kRows = kRowsChunk * KCH;          // Q_c or dO_c
  static constexpr uint32_t kPB = 128 * 64 * 2;                // P or dS: 128 rows x 64 keys
  static constexpr uint32_t kSmem = 1024 + 2 * kBlk + 2 * 2 * kRows + 2 * 2 * kPB + 512;
};

struct KVBars {
  uint64_t kv_full;
  uint64_t qd_full[2], qd_empty[2];
  uint64_t s_full[2], s_empty[2];
  uint64_t pd_full[2], pd_empty[2];
  uint64_t acc_full;
  uint64_t mma_done[4];
  uint32_t tmem_base;
  int abort;
};
__device__ __forceinline__ bool kv_aborted(const KVBars* b) { return *reinterpret_cast<const volatile int*>(&b->abort) != 0; }
__device__ __forceinline__ void kv_set_abort(KVBars* b) { *reinterpret_cast<volatile int*>(&b->abort) = 1; }

// Launch order of the tasks: every init block first (they hold the most
// rows: every later token of the sequence), then the others.
__device__ __forceinline__ int task_of_block(const Args& a, int i) {
  const int ni = min(a.n_init, a.nb_max);
  const int gs_n = a.h_kv * a.batch;
  if (i < gs_n * ni) return (i / ni) * a.nb_max + (i % ni);
  const int j = i - gs_n * ni, rest = a.nb_max - ni;
  return (j / rest) * a.nb_max + ni + (j % rest);
}

template <int D, int G>
__global__ void __launch_bounds__(kKVThreads, 1) dkdv_kernel(const __grid_constant__ CUtensorMap tmQ,
                                                             const __grid_constant__ CUtensorMap tmdO,
                                                             const __grid_constant__ CUtensorMap tmQc,
                                                             const __grid_constant__ CUtensorMap tmdOc,
                                                             const __grid_constant__ CUtensorMap tmK,
                                                             const __grid_constant__ CUtensorMap tmV, const Args a) {
  using C = KVCfg<D>;
  constexpr int TQ = 128 / G;
  const int task = task_of_block(a, blockIdx.x);
  const int kb = task % a.nb_max;
  const int s = (task / a.nb_max) % a.batch;
  const int g = task / (a.nb_max * a.batch);
  const int row0 = a.cu[s];
  const int len = a.cu[s + 1] - row0;
  if (64 * kb >= len) return;                       // uniform: no such block
  const int off = a.offsets[task];
  const int count = a.offsets[task + 1] - off;
  const int nchunks = (count + TQ - 1) / TQ;
  if (nchunks == 0) return;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = smem;
  uint8_t* sV = sK + C::kBlk;
  uint8_t* sQ = sV + C::kBlk;                 // [2]
  uint8_t* sdO = sQ + 2 * C::kRows;           // [2]
  uint8_t* sP = sdO + 2 * C::kRows;           // [2]
  uint8_t* sdS = sP + 2 * C::kPB;             // [2]
  KVBars* bars = reinterpret_cast<KVBars*>(sdS + 2 * C::kPB);
  const int32_t* rows = a.rows + off;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(&bars->kv_full, 1);
    // one commit per MMA issuer that reads the buffer or writes the product
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->qd_full[i], 1);
      mbar_init(&bars->qd_empty[i], kKVIssuers);
      mbar_init(&bars->s_full[i], kKVFront);
      mbar_init(&bars->s_empty[i], 4);
      mbar_init(&bars->pd_full[i], 4);
      mbar_init(&bars->pd_empty[i], kKVBack);
    }
    mbar_init(&bars->acc_full, kKVBack);
    for (int i = 0; i < 4; ++i) mbar_init(&bars->mma_done[i], 1);
    bars->abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) { tmem_alloc(&bars->tmem_base, 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  // TMEM columns: S[sb] at 64 sb, dP[sb] at 128 + 64 sb, dV^T at 256, dK^T at 320

  if (warp == 0) {
    // ------------------------------------------------------------ producer: K/V block, then Q_c / dO_c rows
    if (lane == 0) {
      tma_prefetch_desc(&tmK); tma_prefetch_desc(&tmV); tma_prefetch_desc(&tmQ); tma_prefetch_desc(&tmdO);
      mbar_arrive_expect_tx(&bars->kv_full, 2 * C::kBlk);
      for (int ch = 0; ch < C::KCH; ++ch) {
        tma_load_3d(sK + ch * 8192, &tmK, &bars->kv_full, ch * 64, g, row0 + 64 * kb);
        tma_load_3d(sV + ch * 8192, &tmV, &bars->kv_full, ch * 64, g, row0 + 64 * kb);
      }
    }
    int c = 0;
    for (; c < nchunks; ++c) {
      const int qb = c & 1;
      // the chunk's tokens, one per lane (slots past the row list repeat its first token: their rows are masked)
      const int i = c * TQ + lane;
      const int t_l = (lane < TQ && i < count) ? __ldg(rows + i) : __ldg(rows + c * TQ);
      int good = 1;
      if (lane == 0) {
        good = mbar_wait(&bars->qd_empty[qb], ((c >> 1) & 1) ^ 1) && !kv_aborted(bars);
        if (good) mbar_arrive_expect_tx(&bars->qd_full[qb], 2 * C::KCH * TQ * G * 128);
        else kv_set_abort(bars);
      }
      if (!__shfl_sync(0xffffffffu, good, 0)) break;
      // a chunk of TQ consecutive tokens (the init / local part of the list is
      // one contiguous range) loads as one box per 64 dims; scattered tokens
      // (the top-k part) one box each
      const int t_first = __shfl_sync(0xffffffffu, t_l, 0);
      const int t_lastq = __shfl_sync(0xffffffffu, t_l, TQ - 1);
      const bool contig = (c * TQ + TQ <= count) && (t_lastq - t_first == TQ - 1);
      if (contig) {
        if (lane == 0) {
          for (int ch = 0; ch < C::KCH; ++ch) {
            tma_load_4d(sQ + qb * C::kRows + ch * C::kRowsChunk, &tmQc, &bars->qd_full[qb], ch * 64, 0, g,
                        row0 + t_first);
            tma_load_4d(sdO + qb * C::kRows + ch * C::kRowsChunk, &tmdOc, &bars->qd_full[qb], ch * 64, 0, g,
                        row0 + t_first);
          }
        }
      } else {
        for (int q = 0; q < TQ; ++q) {
          const int t = __shfl_sync(0xffffffffu, t_l, q);
          if (lane == 0) {
            for (int ch = 0; ch < C::KCH; ++ch) {
              tma_load_4d(sQ + qb * C::kRows + ch * C::kRowsChunk + q * G * 128, &tmQ, &bars->qd_full[qb], ch * 64,
                          0, g, row0 + t);
              tma_load_4d(sdO + qb * C::kRows + ch * C::kRowsChunk + q * G * 128, &tmdO, &bars->qd_full[qb],
                          ch * 64, 0, g, row0 + t);
            }
          }
        }
      }
    }
    if (lane == 0) {
      mbar_wait(&bars->kv_full, 0);
      for (int i = max(0, c - 2); i < c; ++i) mbar_wait(&bars->qd_full[i & 1], (i >> 1) & 1);
    }
  } else if (warp == 1 || (warp >= kKVIssuerB && warp < kKVIssuerB + kKVIssuers - 1)) {
    // ------------------------------------------------------------ MMA issuer(s)
    // Issuer ir issues the products of kv_issuer_mask(ir).  An issuer of S or
    // dP ("front") walks the chunks as they land; an issuer of dV^T or dK^T
    // ("back") as their P and dS are written.  One that does both issues the
    // gradient products of chunk cc-1 after S / dP of chunk cc.
    const int ir = (warp == 1) ? 0 : warp - kKVIssuerB + 1;
    const uint32_t mask = kv_issuer_mask(ir);
    const bool do_s = mask & 1u, do_dp = mask & 2u, do_dv = mask & 4u, do_dk = mask & 8u;
    const bool front = do_s || do_dp, back = do_dv || do_dk;
    if (lane == 0) {
      const uint32_t idS = idesc_bf16_f32(128, 64, 0, 0);
      const uint32_t idG = idesc_bf16_f32(128, 64, 1, 1);
      const uint32_t lboR = (D == 128) ? C::kRowsChunk : 0u;   // d = 64: rows 64-127 of dV^T / dK^T repeat 0-63
      bool ok = mbar_wait(&bars->kv_full, 0);
      tc_fence_after();
      const uint32_t k_base = smem_u32(sK), v_base = smem_u32(sV);
      auto issue_grad = [&](int cc) -> bool {
        const int pb = cc & 1;
        if (!mbar_wait(&bars->pd_full[pb], (cc >> 1) & 1) || kv_aborted(bars)) return false;
        tc_fence_after();
        const uint32_t q_base = smem_u32(sQ + pb * C::kRows), do_base = smem_u32(sdO + pb * C::kRows);
        const uint32_t p_base = smem_u32(sP + pb * C::kPB), ds_base = smem_u32(sdS + pb * C::kPB);
        if (do_dv) {
#pragma unroll
          for (int kk = 0; kk < 128 / 16; ++kk) {
            const uint64_t ad = make_sdesc(do_base + kk * 2048, lboR, 1024, kLayoutSW128);
            const uint64_t bp = make_sdesc(p_base + kk * 2048, 1024, 128, kLayoutNone);
            umma_bf16(tmem + 256, ad, bp, idG, (cc > 0 || kk > 0) ? 1u : 0u);
          }
        }
        if (do_dk) {
#pragma unroll
          for (int kk = 0; kk < 128 / 16; ++kk) {
            const uint64_t aq = make_sdesc(q_base + kk * 2048, lboR, 1024, kLayoutSW128);
            const uint64_t bs = make_sdesc(ds_base + kk * 2048, 1024, 128, kLayoutNone);
            umma_bf16(tmem + 320, aq, bs, idG, (cc > 0 || kk > 0) ? 1u : 0u);
          }
        }
        umma_commit(&bars->pd_empty[pb]);
        umma_commit(&bars->qd_empty[pb]);
        return true;
      };
      int cc = 0;
      for (; ok && cc < nchunks; ++cc) {
        if (!front) {
          if (!issue_grad(cc)) { kv_set_abort(bars); ok = false; break; }
          continue;
        }
        const int qb = cc & 1, sb = cc & 1;
        if (!mbar_wait(&bars->qd_full[qb], (cc >> 1) & 1) ||
            !mbar_wait(&bars->s_empty[sb], ((cc >> 1) & 1) ^ 1) || kv_aborted(bars)) {
          kv_set_abort(bars); ok = false; break;
        }
        tc_fence_after();
        const uint32_t q_base = smem_u32(sQ + qb * C::kRows), do_base = smem_u32(sdO + qb * C::kRows);
        if (do_s) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t aq = make_sdesc(q_base + (kk >> 2) * C::kRowsChunk + (kk & 3) * 32, 16, 1024, kLayoutSW128);
            const uint64_t bk = make_sdesc(k_base + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024, kLayoutSW128);
            umma_bf16(tmem + 64 * sb, aq, bk, idS, kk > 0);
          }
        }
        if (do_dp) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t ao = make_sdesc(do_base + (kk >> 2) * C::kRowsChunk + (kk & 3) * 32, 16, 1024, kLayoutSW128);
            const uint64_t bv = make_sdesc(v_base + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024, kLayoutSW128);
            umma_bf16(tmem + 128 + 64 * sb, ao, bv, idS, kk > 0);
          }
        }
        umma_commit(&bars->s_full[sb]);
        if (!back) umma_commit(&bars->qd_empty[qb]);     // this issuer's last read of the chunk
        if (back && cc > 0 && !issue_grad(cc - 1)) { kv_set_abort(bars); ok = false; break; }
      }
      if (ok && front && back && !issue_grad(nchunks - 1)) { kv_set_abort(bars); ok = false; }
      if (back) umma_commit(&bars->acc_full);
      umma_commit(&bars->mma_done[ir]);
      mbar_wait(&bars->mma_done[ir], 0);
    }
  } else {
    // ------------------------------------------------------------ softmax warps 2..5: row r = (token i, head h)
    const int wq = warp & 3;
    const int r = wq * 32 + lane;
    const int qi = r / G, h = r % G;
    const uint32_t lane_addr = static_cast<uint32_t>(wq * 32) << 16;
    const float c = a.scale * kLog2e;
    bool stop = false;
    auto row_of = [&](int c2) { const int i2 = c2 * TQ + qi; return (c2 < nchunks && i2 < count) ? __ldg(rows + i2) : -1; };
    auto stat_of = [&](const float* v, int t2) {
      return (t2 >= 0) ? __ldg(v + static_cast<int64_t>(row0 + t2) * a.h_q + static_cast<int64_t>(g) * G + h) : 0.f;
    };
    int t_a = 0, t_b = 0;
    float lse_a = 0.f, ds_a = 0.f;
    if (INFLLM2_BWD_ROWS_AHEAD) {
      t_a = row_of(0);
      t_b = row_of(1);
      lse_a = stat_of(a.lse, t_a);
      ds_a = stat_of(a.dsum, t_a);
    }
    for (int cc = 0; cc < nchunks; ++cc) {
      const int sb = cc & 1;
      const int i = cc * TQ + qi;
      const bool rv = i < count;
      int t;
      float lse, dsum;
      if (INFLLM2_BWD_ROWS_AHEAD) {
        t = t_a; lse = lse_a; dsum = ds_a;
        lse_a = stat_of(a.lse, t_b);           // chunk cc + 1
        ds_a = stat_of(a.dsum, t_b);
        t_a = t_b;
        t_b = row_of(cc + 2);                   // chunk cc + 2
      } else {
        t = rv ? __ldg(rows + i) : -1;
        const int64_t rh = static_cast<int64_t>(row0 + max(t, 0)) * a.h_q + static_cast<int64_t>(g) * G + h;
        lse = rv ? __ldg(a.lse + rh) : 0.f;
        dsum = rv ? __ldg(a.dsum + rh) : 0.f;
      }
      bool ab = !mbar_wait(&bars->s_full[sb], (cc >> 1) & 1);
      tc_fence_after();
      float sv[64], pv[64];
      tmem_load64(tmem + lane_addr + 64 * sb, sv);
      tmem_load64(tmem + lane_addr + 128 + 64 * sb, pv);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->s_empty[sb]);
      // P and dS buffers sb were last read by the gradient products of chunk cc - 2
      if (cc >= 2 && !mbar_wait(&bars->pd_empty[sb], ((cc - 2) >> 1) & 1)) ab = true;
      uint8_t* pbuf = sP + sb * C::kPB;
      uint8_t* dbuf = sdS + sb * C::kPB;
      const int key0 = 64 * kb;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        uint32_t pp[4], dd[4];
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
          const int n = 8 * q + e;
          float p0 = 0.f, p1 = 0.f;
          if (rv && key0 + n <= t) p0 = ex2(fmaf(sv[n], c, -lse));
          if (rv && key0 + n + 1 <= t) p1 = ex2(fmaf(sv[n + 1], c, -lse));
          const float d0 = p0 * (pv[n] - dsum), d1 = p1 * (pv[n + 1] - dsum);
          __nv_bfloat162 pb2 = __floats2bfloat162_rn(p0, p1);
          __nv_bfloat162 db2 = __floats2bfloat162_rn(d0, d1);
          pp[e >> 1] = *reinterpret_cast<uint32_t*>(&pb2);
          dd[e >> 1] = *reinterpret_cast<uint32_t*>(&db2);
        }
        const uint32_t o = (r >> 3) * 1024 + q * 128 + (r & 7) * 16;
        *reinterpret_cast<uint4*>(pbuf + o) = make_uint4(pp[0], pp[1], pp[2], pp[3]);
        *reinterpret_cast<uint4*>(dbuf + o) = make_uint4(dd[0], dd[1], dd[2], dd[3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->pd_full[sb]);
      if (bar_red_or(1, 128, ab || kv_aborted(bars))) { kv_set_abort(bars); stop = true; break; }
    }
    // ---- the block's gradients: lane r of dV^T / dK^T is d row r, columns the 64 keys
    const bool got = !stop && mbar_wait(&bars->acc_full, 0);
    tc_fence_after();
    if (!bar_red_or(1, 128, !got || kv_aborted(bars))) {
      float gv[64], gk[64];
      tmem_load64(tmem + lane_addr + 256, gv);
      tmem_load64(tmem + lane_addr + 320, gk);
      if (r < D) {
#pragma unroll
        for (int n = 0; n < 64; ++n) {
          const int u = 64 * kb + n;
          if (u < len) {
            const int64_t idx = (static_cast<int64_t>(row0 + u) * a.h_kv + g) * D + r;
            a.dV[idx] = gv[n];
            a.dK[idx] = a.scale * gk[n];
          }
        }
      }
    } else {
      kv_set_abort(bars);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

}  // namespace bwd

// ---------------------------------------------------------------- host side
bool make_tmap(CUtensorMap* map, const void* base, int rank, const uint64_t* dims, const uint64_t* strides_bytes,
               const uint32_t* box);
int num_sms();

struct BwdPlan {
  int nb_max, words, ntasks;
  size_t off_dsum, off_bitmap, off_counts, off_offsets, off_rows, bytes;
};

BwdPlan bwd_plan(int batch, int max_seqlen, int64_t total, int h_q, int h_kv, int n_sel) {
  BwdPlan p{};
  p.nb_max = (max_seqlen + 63) / 64;
  p.words = (max_seqlen + 31) / 32;
  p.ntasks = h_kv * batch * p.nb_max;
  auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
  size_t off = 0;
  p.off_dsum = off;    off = al(off + static_cast<size_t>(total) * h_q * sizeof(float));
  p.off_bitmap = off;  off = al(off + static_cast<size_t>(p.ntasks) * p.words * sizeof(uint32_t));
  p.off_counts = off;  off = al(off + static_cast<size_t>(p.ntasks) * sizeof(int32_t));
  p.off_offsets = off; off = al(off + (static_cast<size_t>(p.ntasks) + 1) * sizeof(int32_t));
  p.off_rows = off;    off = al(off + static_cast<size_t>(h_kv) * total * n_sel * sizeof(int32_t));
  p.bytes = off;
  return p;
}

template <int D, int G>
static cudaError_t launch_bwd_t(const void* Q, const void* K, const void* V, const void* O, bool o_f32,
                                const void* dO, bwd::Args a, cudaStream_t st, bool* map_fail) {
  using bf = __nv_bfloat16;
  const int h_q = a.h_q, h_kv = a.h_kv;
  CUtensorMap mQ, mdO, mQc, mdOc, mK, mV;
  {
    const uint64_t dims[4] = {(uint64_t)D, (uint64_t)G, (uint64_t)h_kv, (uint64_t)a.total};
    const uint64_t strides[3] = {(uint64_t)D * 2, (uint64_t)G * D * 2, (uint64_t)h_q * D * 2};
    const uint32_t box[4] = {64, (uint32_t)G, 1, 1};
    const uint32_t boxc[4] = {64, (uint32_t)G, 1, (uint32_t)(128 / G)};   // 128/G consecutive tokens
    if (!make_tmap(&mQ, Q, 4, dims, strides, box) || !make_tmap(&mdO, dO, 4, dims, strides, box) ||
        !make_tmap(&mQc, Q, 4, dims, strides, boxc) || !make_tmap(&mdOc, dO, 4, dims, strides, boxc)) {
      *map_fail = true;
      return cudaErrorInvalidValue;
    }
  }
  {
    const uint64_t dims[3] = {(uint64_t)D, (uint64_t)h_kv, (uint64_t)a.total};
    const uint64_t strides[2] = {(uint64_t)D * 2, (uint64_t)h_kv * D * 2};
    const uint32_t box[3] = {64, 1, 64};
    if (!make_tmap(&mK, K, 3, dims, strides, box) || !make_tmap(&mV, V, 3, dims, strides, box)) {
      *map_fail = true;
      return cudaErrorInvalidValue;
    }
  }
  const int sms = num_sms();
  const int64_t units = static_cast<int64_t>(h_kv) * a.total;
  const int64_t warp_grid = std::min<int64_t>((units + 7) / 8, static_cast<int64_t>(sms) * 8);
  const int task_grid = std::min<int>((a.h_kv * a.batch * a.nb_max + 7) / 8, sms * 8);
  if (o_f32) bwd::prep_kernel<D, true><<<sms * 8, 256, 0, st>>>(a, static_cast<const bf*>(dO), O);
  else bwd::prep_kernel<D, false><<<sms * 8, 256, 0, st>>>(a, static_cast<const bf*>(dO), O);
  bwd::bitmap_kernel<<<static_cast<unsigned>(warp_grid), 256, 0, st>>>(a);
  bwd::count_kernel<<<task_grid, 256, 0, st>>>(a);
  bwd::scan_kernel<<<1, 1024, 0, st>>>(a);
  bwd::fill_kernel<<<task_grid, 256, 0, st>>>(a);
  {
    using C = bwd::QCfg<D>;
    auto kern = bwd::dq_kernel<D, G>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
    if (e != cudaSuccess) return e;
    const int64_t grid = std::min<int64_t>(units, sms);
    kern<<<static_cast<unsigned>(grid), bwd::kQThreads, C::kSmem, st>>>(mQ, mdO, mK, mV, a);
  }
  {
    using C = bwd::KVCfg<D>;
    auto kern = bwd::dkdv_kernel<D, G>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
    if (e != cudaSuccess) return e;
    kern<<<static_cast<unsigned>(a.h_kv * a.batch * a.nb_max), bwd::kKVThreads, C::kSmem, st>>>(mQ, mdO, mQc, mdOc,
                                                                                                  mK, mV, a);
  }
  return cudaGetLastError();
}

cudaError_t launch_sparse_backward(const void* Q, const void* K, const void* V, const void* O, bool o_f32,
                                   const void* dO, const float* lse, const int32_t* idx, const int32_t* cu, int batch,
                                   int max_seqlen, int64_t total, int h_q, int h_kv, int d, int n_sel, int n_init,
                                   int n_local, float scale, float* dQ, float* dK, float* dV, void* ws,
                                   const BwdPlan& P, cudaStream_t st, bool* map_fail) {
  bwd::Args a{};
  uint8_t* w = static_cast<uint8_t*>(ws);
  a.block_idx = idx; a.cu = cu; a.batch = batch; a.max_seqlen = max_seqlen; a.nb_max = P.nb_max; a.words = P.words;
  a.total = total; a.h_q = h_q; a.h_kv = h_kv; a.n_sel = n_sel; a.n_init = n_init; a.n_local = n_local;
  a.scale = scale; a.lse = lse;
  a.dsum = reinterpret_cast<float*>(w + P.off_dsum);
  a.bitmap = reinterpret_cast<uint32_t*>(w + P.off_bitmap);
  a.counts = reinterpret_cast<int32_t*>(w + P.off_counts);
  a.offsets = reinterpret_cast<int32_t*>(w + P.off_offsets);
  a.rows = reinterpret_cast<int32_t*>(w + P.off_rows);
  a.dQ = dQ; a.dK = dK; a.dV = dV;
  const int G = h_q / h_kv;
#define INFLLM2_BWD_CASE(DD, GG) \
  if (d == DD && G == GG) return launch_bwd_t<DD, GG>(Q, K, V, O, o_f32, dO, a, st, map_fail);
  INFLLM2_BWD_CASE(128, 16)
  INFLLM2_BWD_CASE(128, 8)
  INFLLM2_BWD_CASE(64, 16)
  INFLLM2_BWD_CASE(64, 8)
#undef INFLLM2_BWD_CASE
  return cudaErrorInvalidValue;
}

}  // namespace infllm2
