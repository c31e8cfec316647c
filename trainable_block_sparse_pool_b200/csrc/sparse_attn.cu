// Step 4: block-sparse causal attention over the selected blocks (InfLLM-V2:
// selected and sliding attention merged into one sparse attention with a
// single output — paper-reading blog, "对齐计算图"; top168 article §七).
//
// Work unit: one (kv group g, query token t).  Its G query heads share the
// selected block list I(g,t) (|I| <= 96 blocks of 64 keys).  The init and
// local blocks of I are the same for every token of a 64-token block, so
// the dense kernel's LOCAL form attends to them once per 128/G tokens; this
// kernel gathers only the top-k blocks of each token (the entries of the
// ascending list between the init and the local run) and leaves its
// normalised partial in out with its log-sum-exp, which the LOCAL kernel
// (launched next) merges with its own.  With G = 16 a
// unit is too small for the M dimension of tcgen05 (64 or 128), so the
// contractions are transposed ("swap AB"): keys fill M, heads fill N.
//   S^T [128 keys, 16] = K_pair[128, d]  . Q_t[16, d]^T      (M=128, N=16)
//   O^T [d, 16]      += V_pair[128, d]^T . P^T[128, 16]      (M=d,   N=16)
// A "pair" is two selected blocks side by side in shared memory, each
// loaded by TMA straight from K / V (the gather is the TMA coordinate).
//
// Throughput comes from keeping the per-tile critical path short:
//  * O accumulates in TMEM across the unit's tiles.  The softmax uses a
//    per-head reference maximum m_ref that is only raised when a score
//    exceeds it by more than 2^8 (then O and the partial row sums are
//    rescaled once); otherwise P = 2^(x - m_ref) <= 2^8 is exact enough in
//    bf16/fp32, so the common tile needs no cross-thread maximum, and no
//    round trip through the PV product.
//  * The rescale decision is one `bar.red.or` over the warpgroup.
//  * Two softmax warpgroups work on alternating units of the CTA, so one
//    group's waits overlap the other's work; the TMA producer and the QK
//    issuer interleave the two units' tiles, and each group has its own PV
//    issuer, so no issuer blocks on another group's progress.
// Warp roles: warp 0 TMA producer, warp 1 QK issuer / TMEM owner,
// warps 2-5 softmax group 0, warps 6-9 softmax group 1, warps 10-11 issue
// the PV products of groups 0 and 1.  Persistent CTAs,
// one per SM, take units round-robin (consecutive CTAs work on consecutive
// tokens of one group, so the group's init/local blocks stay hot in L2).
#include "sm100.cuh"

namespace infllm2 {

namespace sparse {

// One thread issues tcgen05.mma at a limited rate: measured on the B200,
// about one M=128, N=16, K=16 product per 100 cycles when independent and per
// 180 cycles in the 8-step chains of a QK or PV product, while the tensor pipe
// takes one every ~40 cycles from several issuing threads.  A single QK issuer
// for both softmax groups (8 chained products per tile) caps the kernel near
// 0.7 us per tile, so each group has its own QK issuer, as it has its own PV
// issuer.  0 restores the single QK issuer.
#ifndef INFLLM2_SPARSE_QK_SPLIT
#define INFLLM2_SPARSE_QK_SPLIT 1
#endif

// The softmax groups fetch the next unit's list (two dependent L2 round
// trips: its length, then this lane's entries) before waiting for the last
// P.V of the current unit, so the fetch hides under that wait instead of
// stalling the group's pipeline at every unit boundary (measured: 43.8 ->
// 42.7 ms for the sparse step at 128K).  The same fetch in the producers and
// issuers, ahead of their last tile of a unit pair, stalled them instead.
#ifndef INFLLM2_SPARSE_PREFETCH
#define INFLLM2_SPARSE_PREFETCH 1
#endif

constexpr int kNumWG = 2;
constexpr bool kQKSplit = INFLLM2_SPARSE_QK_SPLIT != 0;
// K producer, QK issuer(s), softmax groups, PV issuers, V producer
constexpr int kThreads = 64 + 128 * kNumWG + 32 * kNumWG + 32 + (kQKSplit ? 32 * (kNumWG - 1) : 0);
constexpr int kVWarp = 2 + 5 * kNumWG;   // the V producer
constexpr int kQK1Warp = kVWarp + 1;     // with the split: the QK issuer of softmax group 1 (group 0: warp 1)
constexpr int kPairKeys = 128;       // keys per tile (two 64-key blocks)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescale = 8.f;      // raise m_ref only past this margin (log2 units)

template <int D>
struct Cfg {
  static constexpr int KCH = D / 64;
  static constexpr uint32_t kChunk = kPairKeys * 128;         // 16 KB: 128 keys x 64 dims
  static constexpr uint32_t kHalf = 64 * 128;                 // one block inside a chunk
  static constexpr uint32_t kKBytes = kChunk * KCH;
  // ring depths (measured at 128K: 3 + 3 beats 2 + 4 and 4 + 2)
  static constexpr int kKStages = (D == 128) ? 3 : 6;
  static constexpr int kVStages = (D == 128) ? 3 : 6;
  static constexpr int kStages = kKStages + kVStages;           // K and V slots in all
  static constexpr uint32_t kQBuf = 2048 * KCH;               // 16 head rows x d
  static constexpr uint32_t kPBuf = kPairKeys * 16 * 2;       // 4 KB
  static constexpr uint32_t kRed = kNumWG * 4 * 16 * 4;       // per-warp partial maxima / sums
  static constexpr uint32_t kSmem =
      1024 + kStages * kKBytes + kNumWG * 2 * kQBuf + kNumWG * 2 * kPBuf + kRed + 1024;
};

struct Bars {
  uint64_t k_full[8];     // K ring: filled by the K producer, freed when the QK product completes
  uint64_t k_empty[8];
  uint64_t v_full[8];     // V ring: filled by the V producer, freed when the PV product completes
  uint64_t v_empty[8];
  uint64_t q_full[kNumWG][2];
  uint64_t q_empty[kNumWG][2];
  uint64_t s_full[kNumWG][2];
  uint64_t s_empty[kNumWG][2];
  uint64_t p_full[kNumWG][2];
  uint64_t pv_done[kNumWG][2];
  uint64_t o_free[kNumWG][2];
  uint64_t mma_done[2 + kNumWG];   // QK issuer(s) of group 0 and 1 at 0 and 1 + kNumWG, PV issuers between
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ bool aborted(const Bars* b) {
  return *reinterpret_cast<const volatile int*>(&b->abort) != 0;
}
__device__ __forceinline__ void set_abort(Bars* b) {
  *reinterpret_cast<volatile int*>(&b->abort) = 1;
}

// Number of valid (>= 0) entries of a block list, with independent vector
// loads (lists hold their valid entries first, then -1 padding).
__device__ __forceinline__ int count_valid(const int32_t* I, int n_sel) {
  int nv = 0;
  if ((n_sel & 3) == 0 && (reinterpret_cast<uintptr_t>(I) & 15) == 0) {
    const int4* I4 = reinterpret_cast<const int4*>(I);
#pragma unroll 8
    for (int i = 0; i < n_sel / 4; ++i) {
      const int4 v = __ldg(I4 + i);
      nv += (v.x >= 0) + (v.y >= 0) + (v.z >= 0) + (v.w >= 0);
    }
  } else {
    for (int i = 0; i < n_sel; ++i) nv += (__ldg(I + i) >= 0);
  }
  return nv;
}

// Block list entries in registers: lane l of a warp holds entries
// base + 2*(l + 32*r) + half for r = 0, 1 (tiles j = l + 32 r), so tile j's
// block is shfl(reg[j >> 5], j & 31).  Lists longer than 128 entries are
// read from global memory instead.
struct WarpList {
  int r0, r1;
};
__device__ __forceinline__ WarpList load_warp_list(const int32_t* I, int nvalid, int half, int lane) {
  WarpList L;
  const int e0 = 2 * lane + half, e1 = 2 * (lane + 32) + half;
  L.r0 = (e0 < nvalid) ? __ldg(I + e0) : -1;
  L.r1 = (e1 < nvalid) ? __ldg(I + e1) : -1;
  return L;
}
__device__ __forceinline__ int warp_list_get(const WarpList& L, const int32_t* I, int nvalid, int n_sel, int j,
                                             int half) {
  if (n_sel <= 128) {
    const int v0 = __shfl_sync(0xffffffffu, L.r0, j & 31);
    const int v1 = __shfl_sync(0xffffffffu, L.r1, j & 31);
    return (j < 32) ? v0 : v1;
  }
  const int e = 2 * j + half;
  return (e < nvalid) ? __ldg(I + e) : -1;
}

struct Unit {
  int g, t, seq_start, nvalid, nlist;
  int64_t row;
  const int32_t* I;
};

// Unit u = (kv group, packed row), u = g * total + row; its list is
// block_idx[g, row, :] without the shared (init and local) blocks.
struct SparseArgs {
  const int32_t* block_idx;
  const int32_t* cu;
  int batch;
  int64_t total;       // packed rows
  int h_q, h_kv, n_sel, n_init, n_local;
  float scale;
  void* out;           // the top-k partial, normalised (rows without top-k blocks are not written)
  float* lse;          // [total, h_q] its log-sum-exp, log2 units (-inf: no top-k block)
};

__device__ __forceinline__ int64_t num_units(const SparseArgs& a) { return static_cast<int64_t>(a.h_kv) * a.total; }

__device__ __forceinline__ Unit get_unit(int64_t u, const SparseArgs& a) {
  Unit x;
  x.g = static_cast<int>(u / a.total);
  x.row = u - static_cast<int64_t>(x.g) * a.total;
  const int s = find_sequence(a.cu, a.batch, x.row);
  x.seq_start = a.cu[s];
  x.t = static_cast<int>(x.row - x.seq_start);
  const int32_t* list = a.block_idx + u * a.n_sel;
  const int nall = count_valid(list, a.n_sel);
  // the ascending list starts with the i_hi init blocks and ends with the
  // local run; the top-k entries sit between them
  const int bt = x.t >> 6;
  const int i_hi = min(a.n_init, bt + 1);
  const int l_start = max(i_hi, max(0, bt - a.n_local + 1));
  const int nshared = i_hi + max(0, bt - l_start + 1);
  x.I = list + i_hi;
  x.nlist = a.n_sel - i_hi;
  x.nvalid = max(0, nall - nshared);
  return x;
}

__device__ __forceinline__ int ntiles_of(const Unit& x) { return (x.nvalid + 1) >> 1; }

// Does every list have the form the split into a shared part and a top-k
// part relies on?  One warp per unit (kv group, packed row): positions
// [0, i_hi) hold the init blocks 0 .. i_hi-1, the next nvalid positions
// strictly ascending blocks in [i_hi, l_start), the next ones the local run
// l_start .. b_t, and the rest -1.  A list that breaks it is recorded as
// INFLLM2_ERR_DEVICE_BOUNDS (the output of such a row is not the attention
// over its list).  Runs before the attention kernels, off their critical
// path: 4 bytes per list entry, read once.
__global__ void __launch_bounds__(256) check_lists_kernel(const SparseArgs a) {
  const int lane = threadIdx.x & 31;
  const int64_t n_units = num_units(a);
  const int64_t stride = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  bool bad = false;
  for (int64_t u = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); u < n_units;
       u += stride) {
    const Unit x = get_unit(u, a);
    const int32_t* list = a.block_idx + u * a.n_sel;
    const int bt = x.t >> 6;
    const int i_hi = min(a.n_init, bt + 1);
    const int l_start = max(i_hi, max(0, bt - a.n_local + 1));
    const int e_loc = i_hi + x.nvalid, e_pad = e_loc + max(0, bt - l_start + 1);
    int carry = -1;                            // entry 32 r - 1 (the previous round's lane 31)
    for (int e0 = 0; e0 < a.n_sel; e0 += 32) {
      const int e = e0 + lane;
      const int v = (e < a.n_sel) ? __ldg(list + e) : -1;
      int prev = __shfl_up_sync(0xffffffffu, v, 1);
      if (lane == 0) prev = carry;
      carry = __shfl_sync(0xffffffffu, v, 31);
      if (e < a.n_sel) {
        if (e < i_hi) bad |= v != e;
        else if (e < e_loc) bad |= v < i_hi || v >= l_start || (e > i_hi && v <= prev);
        else if (e < e_pad) bad |= v != l_start + (e - e_loc);
        else bad |= v != -1;
      }
    }
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) record_status(INFLLM2_ERR_DEVICE_BOUNDS);
}

template <int D, int G, bool OUT_F32>
__global__ void __launch_bounds__(kThreads, 1) sparse_attn_kernel(
    const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
    const __grid_constant__ CUtensorMap tmV, const SparseArgs args) {
  using C = Cfg<D>;
  static_assert(G >= 1 && G <= 16, "group size <= 16");
  static_assert(sizeof(Bars) <= 1024, "barrier area");
  static_assert(C::kSmem <= 232448, "shared memory per CTA");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sKV = smem;
  uint8_t* sKr = sKV;                                                  // K ring [kKStages][kKBytes]
  uint8_t* sVr = sKV + C::kKStages * C::kKBytes;                       // V ring [kVStages][kKBytes]
  uint8_t* sQ = sKV + C::kStages * C::kKBytes;                        // [wg][2]
  uint8_t* sP = sQ + kNumWG * 2 * C::kQBuf;                           // [wg][2]
  float* red = reinterpret_cast<float*>(sP + kNumWG * 2 * C::kPBuf);  // [wg][4][16]
  Bars* bars = reinterpret_cast<Bars*>(red + kNumWG * 4 * 16);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t n_units = num_units(args);
  // units of this CTA: u_k = blockIdx.x + k * gridDim.x; unit k goes to group k & 1
  const int64_t my_units = (n_units > blockIdx.x) ? (n_units - 1 - blockIdx.x) / gridDim.x + 1 : 0;

  for (int i = threadIdx.x; i < static_cast<int>(kNumWG * 2 * C::kQBuf / 16); i += kThreads)
    reinterpret_cast<uint4*>(sQ)[i] = make_uint4(0, 0, 0, 0);   // head rows past G stay zero
  fence_proxy_async_smem();
  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kKStages; ++i) {
      mbar_init(&bars->k_full[i], 1);
      mbar_init(&bars->k_empty[i], 1);
    }
    for (int i = 0; i < C::kVStages; ++i) {
      mbar_init(&bars->v_full[i], 1);
      mbar_init(&bars->v_empty[i], 1);
    }
    for (int w = 0; w < kNumWG; ++w)
      for (int i = 0; i < 2; ++i) {
        mbar_init(&bars->q_full[w][i], 1);
        mbar_init(&bars->q_empty[w][i], 1);
        mbar_init(&bars->s_full[w][i], 1);
        mbar_init(&bars->s_empty[w][i], 4);
        mbar_init(&bars->p_full[w][i], 4);
        mbar_init(&bars->pv_done[w][i], 1);
        mbar_init(&bars->o_free[w][i], 4);
      }
    for (int i = 0; i < 2 + kNumWG; ++i) mbar_init(&bars->mma_done[i], 1);
    bars->abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) { tmem_alloc(&bars->tmem_base, 128); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  // TMEM columns of group w: S buffers at w*64 + {0,16}, O buffers at w*64 + {32,48}

  if (warp == 0 || warp == kVWarp) {
    // ------------------------------------------------------------ producers
    // Warp 0 loads Q and the K ring, warp kVWarp the V ring; both walk the
    // same stream of tiles.  The whole warp walks the units (their block
    // lists live in its registers); lane 0 waits and issues the copies.
    const bool isV = (warp == kVWarp);
    const int nst = isV ? C::kVStages : C::kKStages;
    const CUtensorMap* tm = isV ? &tmV : &tmK;
    uint8_t* ring = isV ? sVr : sKr;
    uint64_t* full = isV ? bars->v_full : bars->k_full;
    uint64_t* empty = isV ? bars->v_empty : bars->k_empty;
    if (lane == 0) { tma_prefetch_desc(&tmQ); tma_prefetch_desc(tm); }
    int it = 0;
    int ucnt[kNumWG] = {0, 0};
    bool ok = true;
    for (int64_t k0 = 0; ok && k0 < my_units; k0 += kNumWG) {
      Unit x[kNumWG];
      WarpList Le[kNumWG], Lo[kNumWG];
      int nt[kNumWG];
      for (int w = 0; w < kNumWG; ++w) {
        nt[w] = 0;
        if (k0 + w >= my_units) continue;
        x[w] = get_unit(blockIdx.x + (k0 + w) * gridDim.x, args);
        nt[w] = ntiles_of(x[w]);
        Le[w] = load_warp_list(x[w].I, x[w].nvalid, 0, lane);
        Lo[w] = load_warp_list(x[w].I, x[w].nvalid, 1, lane);
        if (isV) continue;
        const int qb = ucnt[w] & 1;
        int good = 1;
        if (lane == 0) {
          good = mbar_wait(&bars->q_empty[w][qb], ((ucnt[w] >> 1) & 1) ^ 1);
          if (good) {
            mbar_arrive_expect_tx(&bars->q_full[w][qb], C::KCH * G * 128);
            for (int ch = 0; ch < C::KCH; ++ch)
              tma_load_4d(sQ + (w * 2 + qb) * C::kQBuf + ch * 2048, &tmQ, &bars->q_full[w][qb], ch * 64, 0,
                          x[w].g, static_cast<int>(x[w].row));
          } else {
            set_abort(bars);
          }
        }
        if (!__shfl_sync(0xffffffffu, good, 0)) { ok = false; break; }
        ++ucnt[w];
      }
      const int nmax = max(nt[0], nt[1]);
      for (int j = 0; ok && j < nmax; ++j) {
        for (int w = 0; w < kNumWG; ++w) {
          if (j >= nt[w]) continue;
          const int b0 = warp_list_get(Le[w], x[w].I, x[w].nvalid, x[w].nlist, j, 0);
          int b1 = warp_list_get(Lo[w], x[w].I, x[w].nvalid, x[w].nlist, j, 1);
          if (b1 < 0) b1 = b0;   // odd count: reload the first block, masked by the softmax
          const int st = it % nst;
          int good = 1;
          if (lane == 0) {
            good = mbar_wait(&empty[st], ((it / nst) & 1) ^ 1) && !aborted(bars);
            if (good) {
              uint8_t* dst = ring + st * C::kKBytes;
              mbar_arrive_expect_tx(&full[st], C::kKBytes);
              for (int ch = 0; ch < C::KCH; ++ch) {
                tma_load_3d(dst + ch * C::kChunk, tm, &full[st], ch * 64, x[w].g, x[w].seq_start + 64 * b0);
                tma_load_3d(dst + ch * C::kChunk + C::kHalf, tm, &full[st], ch * 64, x[w].g,
                            x[w].seq_start + 64 * b1);
              }
            } else {
              set_abort(bars);
            }
          }
          if (!__shfl_sync(0xffffffffu, good, 0)) { ok = false; break; }
          ++it;
        }
      }
    }
    // wait for every copy still in flight before the CTA may exit
    if (lane == 0) {
      for (int i = max(0, it - nst); i < it; ++i) mbar_wait(&full[i % nst], (i / nst) & 1);
      if (!isV)
        for (int w = 0; w < kNumWG; ++w)
          for (int i = max(0, ucnt[w] - 2); i < ucnt[w]; ++i) mbar_wait(&bars->q_full[w][i & 1], (i >> 1) & 1);
    }
  } else if (warp == 1 || (kQKSplit && warp == kQK1Warp)) {
    // ------------------------------------------------------------ QK issuer(s)
    // Walk the stream in order: a QK product goes out as soon as its K stage
    // has landed and its group's S buffer is free.  With the split each
    // issuer takes one group's tiles and steps over the other's.
    const int mine = kQKSplit ? (warp == 1 ? 0 : 1) : -1;   // -1: both groups
    if (lane == 0) {
      const uint32_t idS = idesc_bf16_f32(128, 16, 0, 0);
      int it = 0;
      int tcnt[kNumWG] = {0, 0}, ucnt[kNumWG] = {0, 0};
      bool ok = true;
      for (int64_t k0 = 0; ok && k0 < my_units; k0 += kNumWG) {
        int nt[kNumWG], qb[kNumWG];
        for (int w = 0; w < kNumWG; ++w) {
          nt[w] = 0;
          if (k0 + w >= my_units) continue;
          const Unit x = get_unit(blockIdx.x + (k0 + w) * gridDim.x, args);
          nt[w] = ntiles_of(x);
          qb[w] = ucnt[w] & 1;
          if (mine >= 0 && w != mine) continue;
          if (!mbar_wait(&bars->q_full[w][qb[w]], (ucnt[w] >> 1) & 1)) { set_abort(bars); ok = false; break; }
          if (nt[w] == 0) umma_commit(&bars->q_empty[w][qb[w]]);   // empty list: Q is free at once
          ++ucnt[w];
        }
        const int nmax = max(nt[0], nt[1]);
        for (int j = 0; ok && j < nmax; ++j) {
          for (int w = 0; w < kNumWG; ++w) {
            if (j >= nt[w]) continue;
            if (mine >= 0 && w != mine) { ++it; continue; }
            const int st = it % C::kKStages;
            const int sb = tcnt[w] & 1;
            if (!mbar_wait(&bars->k_full[st], (it / C::kKStages) & 1) ||
                !mbar_wait(&bars->s_empty[w][sb], ((tcnt[w] >> 1) & 1) ^ 1) || aborted(bars)) {
              set_abort(bars); ok = false; break;
            }
            tc_fence_after();
            const uint32_t k_base = smem_u32(sKr + st * C::kKBytes);
            const uint32_t q_base = smem_u32(sQ + (w * 2 + qb[w]) * C::kQBuf);
#pragma unroll
            for (int k = 0; k < D / 16; ++k) {
              const uint64_t a = make_sdesc(k_base + (k >> 2) * C::kChunk + (k & 3) * 32, 16, 1024, kLayoutSW128);
              const uint64_t b = make_sdesc(q_base + (k >> 2) * 2048 + (k & 3) * 32, 16, 1024, kLayoutSW128);
              umma_bf16(tmem + w * 64 + sb * 16, a, b, idS, k > 0);
            }
            umma_commit(&bars->s_full[w][sb]);
            umma_commit(&bars->k_empty[st]);        // K slot free once this product completes
            if (j == nt[w] - 1) umma_commit(&bars->q_empty[w][qb[w]]);
            ++tcnt[w];
            ++it;
          }
        }
      }
      const int done = (warp == 1) ? 0 : 1 + kNumWG;
      umma_commit(&bars->mma_done[done]);
      mbar_wait(&bars->mma_done[done], 0);
    }
  } else if (warp >= 2 + 4 * kNumWG && warp < kVWarp) {
    // ------------------------------------------------------------ PV issuers
    // One warp per softmax group: the group's PV products in order, each as
    // soon as its P is in shared memory.  The stream is replayed to find
    // which K/V stage each tile occupies.
    const int pw = warp - (2 + 4 * kNumWG);
    if (lane == 0) {
      const uint32_t idO = idesc_bf16_f32(128, 16, 1, 1);
      const uint32_t lboV = (D == 128) ? C::kChunk : 0u;   // d = 64: rows 64-127 of O^T repeat 0-63
      int it = 0, tcnt = 0, ucnt = 0;
      bool ok = true;
      for (int64_t k0 = 0; ok && k0 < my_units; k0 += kNumWG) {
        int nt[kNumWG];
        for (int w = 0; w < kNumWG; ++w) {
          nt[w] = 0;
          if (k0 + w >= my_units) continue;
          const Unit x = get_unit(blockIdx.x + (k0 + w) * gridDim.x, args);
          nt[w] = ntiles_of(x);
        }
        const bool mine = (k0 + pw < my_units);
        const int obuf = ucnt & 1;
        if (mine && nt[pw] > 0 &&
            !mbar_wait(&bars->o_free[pw][obuf], ((ucnt >> 1) & 1) ^ 1)) { set_abort(bars); ok = false; break; }
        const int nmax = max(nt[0], nt[1]);
        for (int j = 0; ok && j < nmax; ++j) {
          for (int w = 0; w < kNumWG; ++w) {
            if (j >= nt[w]) continue;
            if (w == pw) {
              const int st = it % C::kVStages;
              const int pb = tcnt & 1;
              if (!mbar_wait(&bars->p_full[pw][pb], (tcnt >> 1) & 1) ||
                  !mbar_wait(&bars->v_full[st], (it / C::kVStages) & 1) || aborted(bars)) {
                set_abort(bars); ok = false; break;
              }
              tc_fence_after();
              const uint32_t v_base = smem_u32(sVr + st * C::kKBytes);
              const uint32_t p_base = smem_u32(sP + (pw * 2 + pb) * C::kPBuf);
              const uint32_t o_addr = tmem + pw * 64 + 32 + obuf * 16;
#pragma unroll
              for (int k = 0; k < kPairKeys / 16; ++k) {
                const uint64_t a = make_sdesc(v_base + k * 2048, lboV, 1024, kLayoutSW128);
                const uint64_t b = make_sdesc(p_base + k * 512, 256, 128, kLayoutNone);
                umma_bf16(o_addr, a, b, idO, (j == 0 && k == 0) ? 0u : 1u);
              }
              umma_commit(&bars->v_empty[st]);
              umma_commit(&bars->pv_done[pw][pb]);
              ++tcnt;
            }
            ++it;
          }
        }
        if (mine) ++ucnt;
      }
      umma_commit(&bars->mma_done[1 + pw]);
      mbar_wait(&bars->mma_done[1 + pw], 0);
    }
  } else {
    // ------------------------------------------------------------ softmax groups (warps 2 .. 2+4*kNumWG-1)
    const int w = (warp - 2) >> 2;           // softmax group
    const int wq = warp & 3;                 // TMEM lane quadrant of this warp
    const int kl = wq * 32 + lane;           // key lane (softmax) / d row (output)
    const int bar_id = 1 + w;
    const uint32_t lane_addr = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t t_s = tmem + w * 64;
    const uint32_t t_o = tmem + w * 64 + 32;
    float* red_w = red + w * 64;
    const float c = args.scale * kLog2e;
    int tcnt = 0, ucnt = 0;
    bool stop = false;
    const int half = kl >> 6;                // this warp's keys come from the pair's first or second block
    Unit xn{};
    WarpList Ln{};
    if (INFLLM2_SPARSE_PREFETCH && w < my_units) {
      xn = get_unit(blockIdx.x + static_cast<int64_t>(w) * gridDim.x, args);
      Ln = load_warp_list(xn.I, xn.nvalid, half, lane);
    }
    for (int64_t k = w; !stop && k < my_units; k += kNumWG, ++ucnt) {
      const Unit x = INFLLM2_SPARSE_PREFETCH ? xn : get_unit(blockIdx.x + k * gridDim.x, args);
      const int nt = ntiles_of(x);
      const int obuf = ucnt & 1;
      const WarpList L = INFLLM2_SPARSE_PREFETCH ? Ln : load_warp_list(x.I, x.nvalid, half, lane);
      float m_ref[16], l_part[16];
#pragma unroll
      for (int h = 0; h < 16; ++h) { m_ref[h] = -INFINITY; l_part[h] = 0.f; }
      for (int j = 0; j < nt; ++j, ++tcnt) {
        const int sb = tcnt & 1;
        bool ab = !mbar_wait(&bars->s_full[w][sb], (tcnt >> 1) & 1);
        if (ab) set_abort(bars);
        tc_fence_after();
        float v[16];
        tmem_load16(t_s + lane_addr + sb * 16, v);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->s_empty[w][sb]);   // S is in registers: the buffer is free
        const int blk = warp_list_get(L, x.I, x.nvalid, x.nlist, j, half);
        const int pos = 64 * blk + (kl & 63);
        const bool valid = (blk >= 0) && (pos <= x.t);
        bool exceed = false;
#pragma unroll
        for (int h = 0; h < 16; ++h) {
          v[h] = valid ? v[h] * c : -INFINITY;
          exceed |= v[h] > m_ref[h] + kRescale;
        }
        ab = ab || aborted(bars);
        if (bar_red_or(bar_id, 128, exceed || ab)) {
          if (bar_red_or(bar_id, 128, ab)) { stop = true; break; }
          // raise the reference maxima: full per-head maximum over the 128 keys
          float mx[16];
#pragma unroll
          for (int h = 0; h < 16; ++h) {
            mx[h] = v[h];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], o));
          }
          if (lane < 16) {
            float mine = mx[0];
#pragma unroll
            for (int h = 1; h < 16; ++h) if (lane == h) mine = mx[h];
            red_w[wq * 16 + lane] = mine;
          }
          named_bar_sync(bar_id, 128);
          float alpha[16];
          bool any_scale = false;
#pragma unroll
          for (int h = 0; h < 16; ++h) {
            const float tmax = fmaxf(fmaxf(red_w[h], red_w[16 + h]), fmaxf(red_w[32 + h], red_w[48 + h]));
            const float m_new = fmaxf(m_ref[h], tmax);
            alpha[h] = (m_ref[h] == -INFINITY) ? 0.f : ex2(m_ref[h] - m_new);
            any_scale |= (m_ref[h] != -INFINITY) && (m_new > m_ref[h]);
            m_ref[h] = m_new;
            l_part[h] *= alpha[h];
          }
          named_bar_sync(bar_id, 128);   // red_w is read by everyone before it is reused
          if (j > 0 && any_scale) {
            // rescale O in TMEM once every PV of this unit so far is done
            const int prev = tcnt - 1;
            const bool okw = mbar_wait(&bars->pv_done[w][prev & 1], (prev >> 1) & 1);
            if (!okw) set_abort(bars);
            tc_fence_after();
            float o[16];
            tmem_load16(t_o + lane_addr + obuf * 16, o);
#pragma unroll
            for (int h = 0; h < 16; ++h) o[h] *= alpha[h];
            tmem_store16(t_o + lane_addr + obuf * 16, o);
          }
        }
        // P buffer sb was last read by the PV of tile tcnt-2
        if (tcnt >= 2 && !mbar_wait(&bars->pv_done[w][sb], ((tcnt - 2) >> 1) & 1)) set_abort(bars);
        uint32_t pk[8];
#pragma unroll
        for (int h = 0; h < 16; h += 2) {
          const float p0 = ex2(v[h] - m_ref[h]);
          const float p1 = ex2(v[h + 1] - m_ref[h + 1]);
          l_part[h] += p0;
          l_part[h + 1] += p1;
          __nv_bfloat162 b2 = __floats2bfloat162_rn(p0, p1);
          pk[h >> 1] = *reinterpret_cast<uint32_t*>(&b2);
        }
        uint8_t* pbuf = sP + (w * 2 + sb) * C::kPBuf;
        const uint32_t poff = (kl >> 3) * 256 + (kl & 7) * 16;
        *reinterpret_cast<uint4*>(pbuf + poff) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        *reinterpret_cast<uint4*>(pbuf + poff + 128) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->p_full[w][sb]);
      }
      if (stop) break;
      if (INFLLM2_SPARSE_PREFETCH && k + kNumWG < my_units) {
        xn = get_unit(blockIdx.x + (k + kNumWG) * gridDim.x, args);
        Ln = load_warp_list(xn.I, xn.nvalid, half, lane);
      }
      // ---- unit done: reduce the row sums (they do not depend on O, so this
      // runs while the last PV completes), wait for that PV, write out
#pragma unroll
      for (int h = 0; h < 16; ++h) {
#pragma unroll
        for (int s2 = 16; s2 > 0; s2 >>= 1) l_part[h] += __shfl_xor_sync(0xffffffffu, l_part[h], s2);
      }
      if (lane < 16) {
        float mine = l_part[0];
#pragma unroll
        for (int h = 1; h < 16; ++h) if (lane == h) mine = l_part[h];
        red_w[wq * 16 + lane] = mine;
      }
      bool ab = (nt > 0) && !mbar_wait(&bars->pv_done[w][(tcnt - 1) & 1], ((tcnt - 1) >> 1) & 1);
      if (ab) set_abort(bars);
      tc_fence_after();
      float o[16];
      tmem_load16(t_o + lane_addr + obuf * 16, o);
      if (nt == 0) {                         // empty list: no PV wrote this buffer
#pragma unroll
        for (int h = 0; h < 16; ++h) o[h] = 0.f;
      }
      ab = ab || aborted(bars);
      if (bar_red_or(bar_id, 128, ab)) { stop = true; break; }
      if (kl < D && nt > 0) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float l = red_w[h] + red_w[16 + h] + red_w[32 + h] + red_w[48 + h];
          const float r = (l > 0.f) ? o[h] / l : 0.f;
          const int64_t idx = (x.row * args.h_q + static_cast<int64_t>(x.g) * G + h) * D + kl;
          if (OUT_F32) reinterpret_cast<float*>(args.out)[idx] = r;
          else reinterpret_cast<__nv_bfloat16*>(args.out)[idx] = __float2bfloat16_rn(r);
        }
      }
      if (kl < G) {
        float mr = m_ref[0];
#pragma unroll
        for (int h = 1; h < 16; ++h) if (kl == h) mr = m_ref[h];
        const float l = red_w[kl] + red_w[16 + kl] + red_w[32 + kl] + red_w[48 + kl];
        args.lse[x.row * args.h_q + static_cast<int64_t>(x.g) * G + kl] =
            (nt > 0 && l > 0.f) ? mr + log2f(l) : -INFINITY;
      }
      tc_fence_before();
      named_bar_sync(bar_id, 128);           // red_w and this O buffer are free again
      if (lane == 0) mbar_arrive(&bars->o_free[w][obuf]);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 128);
}

}  // namespace sparse

bool make_tmap(CUtensorMap* map, const void* base, int rank, const uint64_t* dims, const uint64_t* strides_bytes,
               const uint32_t* box);
int num_sms();

template <int D, int G, bool F32>
static cudaError_t launch_sparse_t(const void* Q, const void* K, const void* V, int64_t rows,
                                   const sparse::SparseArgs& args, cudaStream_t st, bool* map_fail) {
  using C = sparse::Cfg<D>;
  const int h_q = args.h_q, h_kv = args.h_kv;
  CUtensorMap mQ, mK, mV;
  {
    const uint64_t dims[4] = {(uint64_t)D, (uint64_t)G, (uint64_t)h_kv, (uint64_t)rows};
    const uint64_t strides[3] = {(uint64_t)D * 2, (uint64_t)G * D * 2, (uint64_t)h_q * D * 2};
    const uint32_t box[4] = {64, (uint32_t)G, 1, 1};
    if (!make_tmap(&mQ, Q, 4, dims, strides, box)) { *map_fail = true; return cudaErrorInvalidValue; }
  }
  {
    const uint64_t dims[3] = {(uint64_t)D, (uint64_t)h_kv, (uint64_t)rows};
    const uint64_t strides[2] = {(uint64_t)D * 2, (uint64_t)h_kv * D * 2};
    const uint32_t box[3] = {64, 1, 64};
    if (!make_tmap(&mK, K, 3, dims, strides, box)) { *map_fail = true; return cudaErrorInvalidValue; }
    if (!make_tmap(&mV, V, 3, dims, strides, box)) { *map_fail = true; return cudaErrorInvalidValue; }
  }
  auto kern = sparse::sparse_attn_kernel<D, G, F32>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return e;
  const int64_t units = static_cast<int64_t>(h_kv) * args.total;
  if (units == 0) return cudaSuccess;
  const int64_t grid = std::min<int64_t>((units + 1) / 2, num_sms());
  kern<<<static_cast<unsigned>(grid), sparse::kThreads, C::kSmem, st>>>(mQ, mK, mV, args);
  return cudaGetLastError();
}

// The top-k part of the sparse attention: its normalised partial into out,
// its log-sum-exp into lse (the LOCAL kernel merges its own into both).
cudaError_t launch_sparse_attn(const void* Q, const void* K, const void* V, const int32_t* idx, const int32_t* cu,
                               int batch, int64_t total, int h_q, int h_kv, int d, int n_sel, int n_init,
                               int n_local, float scale, void* out, bool out_f32, float* lse, cudaStream_t st,
                               bool* map_fail) {
  sparse::SparseArgs a{};
  a.block_idx = idx; a.cu = cu; a.batch = batch; a.total = total; a.h_q = h_q; a.h_kv = h_kv; a.n_sel = n_sel;
  a.n_init = n_init; a.n_local = n_local; a.scale = scale; a.out = out; a.lse = lse;
  const int G = h_q / h_kv;
  if (total > 0) {
    const int64_t warps = static_cast<int64_t>(h_kv) * total;
    const int64_t grid = std::min<int64_t>((warps + 7) / 8, static_cast<int64_t>(num_sms()) * 8);
    sparse::check_lists_kernel<<<static_cast<unsigned>(grid), 256, 0, st>>>(a);
  }
#define INFLLM2_SPARSE_CASE(DD, GG)                                                            \
  if (d == DD && G == GG)                                                                     \
    return out_f32 ? launch_sparse_t<DD, GG, true>(Q, K, V, total, a, st, map_fail)           \
                   : launch_sparse_t<DD, GG, false>(Q, K, V, total, a, st, map_fail);
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
