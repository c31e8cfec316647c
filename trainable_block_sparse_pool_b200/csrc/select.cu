// Step 3: stage-3 max-pool to block scores and block selection (InfLLM-V2,
// top168 article §三 third stage and §七; paper-reading blog, worked example).
//
// One warp per (kv group, query token).  HBM-bound on reading the S_shared
// row.  The warp
//   1. max-pools the row into one score per candidate block
//      (block b takes the maximum of windows 4b-1 .. 4b+3 that are visible)
//      with 16-byte loads, keeping the scores' bit patterns in shared memory
//      (scores are >= 0, so their IEEE bits order like the values);
//   2. finds the exact k-th largest score with a radix select over the bits
//      of (score - min score), 8 bits per pass, using a 256-bin warp-private
//      histogram; the result is the threshold T and how many of the blocks
//      equal to T are taken;
//   3. writes init blocks, then in one ascending pass over the candidates
//      every block above T plus the lowest-indexed blocks equal to T
//      (ties go to the lower block index), then the local blocks — the list
//      comes out sorted without a sort.
#include "sm100.cuh"

namespace infllm2 {

namespace sel {

constexpr int kHistBins = 256;

__device__ __forceinline__ uint32_t warp_min_u32(uint32_t v) {
  for (int o = 16; o > 0; o >>= 1) v = min(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ uint32_t warp_max_u32(uint32_t v) {
  for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Block score of candidate block b from a row of visible length n1.
__device__ __forceinline__ float block_score(const float* __restrict__ row, int b, int n1) {
  const int j0 = 4 * b - 1;
  float m = -INFINITY;
  if (j0 >= 0 && 4 * b + 3 < n1) {
    const float4 v = *reinterpret_cast<const float4*>(row + 4 * b);
    m = fmaxf(fmaxf(row[j0], v.x), fmaxf(fmaxf(v.y, v.z), v.w));
  } else {
#pragma unroll
    for (int j = j0; j < j0 + 5; ++j)
      if (j >= 0 && j < n1) m = fmaxf(m, row[j]);
  }
  return m;
}

// Writes the selected block list of one query row, given the candidates'
// keys (bit patterns of non-negative scores, candidate i is block
// cand_lo + i) in this warp's shared memory, each lane's partial min / max of
// the keys (reduced over the warp here), and the init / local
// ranges.  Shared by the prefill and decode selections.
__device__ __noinline__ void warp_select_write(uint32_t* keys, int* hist, int ncand, int cand_lo, int init_hi,
                                               int loc_lo, int b_t, int top_k, int n_sel, uint32_t kmin,
                                               uint32_t kmax, int32_t* out, int lane) {
  kmin = warp_min_u32(kmin);
  kmax = warp_max_u32(kmax);
  __syncwarp();

  // 2. radix select of the top_k-th largest key, on u = key - kmin
  const uint32_t range = kmax - kmin;
  int hi = range ? 32 - __clz(range) : 0;  // bits of u still undecided: [0, hi)
  uint32_t prefix = 0;
  int k_rem = top_k;
  while (hi > 0) {
    const int shift = max(0, hi - 8);
    const int nb = 1 << (hi - shift);
    for (int i = lane; i < nb; i += 32) hist[i] = 0;
    __syncwarp();
    const uint64_t want = static_cast<uint64_t>(prefix) >> hi;
    for (int i = lane; i < ncand; i += 32) {
      const uint32_t u = keys[i] - kmin;
      if ((static_cast<uint64_t>(u) >> hi) == want) atomicAdd(&hist[(u >> shift) & (nb - 1)], 1);
    }
    __syncwarp();
    // lane L looks after bins [8L, 8L+8); counts of all higher bins come from
    // a suffix sum over the lanes
    int lsum = 0;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int b = lane * 8 + q;
      lsum += (b < nb) ? hist[b] : 0;
    }
    int suf = lsum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_down_sync(0xffffffffu, suf, o);
      if (lane + o < 32) suf += v;
    }
    int above = suf - lsum;  // keys in bins above this lane's range
    int digit = -1, above_digit = 0, in_digit = 0;
    if (above < k_rem && suf >= k_rem) {
      for (int q = 7; q >= 0; --q) {
        const int b = lane * 8 + q;
        const int h = (b < nb) ? hist[b] : 0;
        if (above + h >= k_rem) { digit = b; above_digit = above; in_digit = h; break; }
        above += h;
      }
    }
    const uint32_t who = __ballot_sync(0xffffffffu, digit >= 0);
    const int src = __ffs(who) - 1;
    digit = __shfl_sync(0xffffffffu, digit, src);
    above_digit = __shfl_sync(0xffffffffu, above_digit, src);
    in_digit = __shfl_sync(0xffffffffu, in_digit, src);
    prefix |= static_cast<uint32_t>(digit) << shift;
    k_rem -= above_digit;
    hi = shift;
    __syncwarp();
    if (hi > 0 && in_digit <= 32) {
      // at most 32 keys share the boundary digit: gather them (the histogram
      // is free now), sort them across the lanes and take the k_rem-th
      // largest exactly, instead of more passes over every key
      const uint32_t want_hi = prefix >> hi;
      int n = 0;
      for (int base = 0; base < ncand; base += 32) {
        const int i = base + lane;
        const uint32_t u = (i < ncand) ? keys[i] - kmin : 0u;
        const bool m = (i < ncand) && (u >> hi) == want_hi;
        const uint32_t bm = __ballot_sync(0xffffffffu, m);
        if (m) hist[n + __popc(bm & lanemask_lt())] = static_cast<int>(u);
        n += __popc(bm);
      }
      __syncwarp();
      uint32_t x = (lane < n) ? static_cast<uint32_t>(hist[lane]) : 0u;   // 0 sorts last: no key of the bin is below it
#pragma unroll
      for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1) {
          const uint32_t y = __shfl_xor_sync(0xffffffffu, x, j);
          const bool keep_max = ((lane & j) == 0) == ((lane & k) == 0);
          x = keep_max ? max(x, y) : min(x, y);
        }
      }
      const uint32_t tu = __shfl_sync(0xffffffffu, x, k_rem - 1);
      k_rem -= __popc(__ballot_sync(0xffffffffu, lane < n && x > tu));
      prefix = tu;
      hi = 0;
      __syncwarp();
    }
  }
  const uint32_t T = kmin + prefix;  // the top_k-th largest key; take k_rem of the keys equal to it

  // 3. ordered output: INIT, chosen candidates ascending, LOCAL, padding
  for (int i = lane; i < init_hi; i += 32) out[i] = i;
  int pos = init_hi;
  int eq_seen = 0;
  for (int base = 0; base < ncand; base += 32) {
    const int i = base + lane;
    const bool valid = i < ncand;
    const uint32_t k = valid ? keys[i] : 0u;
    const bool gt = valid && k > T;
    const bool eq = valid && k == T;
    const uint32_t eqm = __ballot_sync(0xffffffffu, eq);
    const int eq_rank = eq_seen + __popc(eqm & lanemask_lt());
    const bool take = gt || (eq && eq_rank < k_rem);
    const uint32_t tm = __ballot_sync(0xffffffffu, take);
    if (take) out[pos + __popc(tm & lanemask_lt())] = cand_lo + i;
    pos += __popc(tm);
    eq_seen += __popc(eqm);
  }
  const int nloc = b_t - loc_lo + 1;
  for (int i = lane; i < nloc; i += 32) out[pos + i] = loc_lo + i;
  pos += nloc;
  for (int i = pos + lane; i < n_sel; i += 32) out[i] = -1;
}

// POOL: S holds the score kernel's pooled pairs (per group of four windows,
// its visible maximum and its last window); block b takes the maximum of
// pair b's first value and pair b-1's second.
template <bool POOL>
__global__ void __launch_bounds__(256) topk_kernel(const float* __restrict__ S, int64_t ld,
                                                   const int32_t* __restrict__ cu, int batch, int64_t total,
                                                   int h_kv, int n_init, int n_local, int top_k, int n_sel,
                                                   int cand_cap, int32_t* __restrict__ out_idx) {
  extern __shared__ uint32_t sel_smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int wpb = blockDim.x >> 5;
  uint32_t* keys = sel_smem + warp * (cand_cap + kHistBins);
  int* hist = reinterpret_cast<int*>(keys + cand_cap);

  const int64_t unit = static_cast<int64_t>(blockIdx.x) * wpb + warp;
  if (unit >= static_cast<int64_t>(h_kv) * total) return;
  const int g = static_cast<int>(unit / total);
  const int64_t row = unit - static_cast<int64_t>(g) * total;
  const int s = find_sequence(cu, batch, row);
  const int t = static_cast<int>(row - cu[s]);
  const int b_t = t / 64;
  int32_t* out = out_idx + unit * n_sel;

  const int init_hi = min(n_init, b_t + 1);          // INIT  = [0, init_hi)
  const int loc_lo = max(0, b_t - n_local + 1);      // LOCAL = [loc_lo, b_t]
  const int cand_lo = init_hi;
  const int ncand = max(0, loc_lo - init_hi);        // CAND  = [init_hi, loc_lo)

  if (ncand <= top_k) {
    // every causal block is taken
    for (int i = lane; i < n_sel; i += 32) out[i] = (i <= b_t) ? i : -1;
    return;
  }
  if (ncand > cand_cap) {  // host sizes cand_cap from max_seqlen; never expected
    if (lane == 0) record_status(INFLLM2_ERR_DEVICE_BOUNDS);
    return;
  }

  // 1. block scores of the candidates
  const float* srow = S + (static_cast<int64_t>(g) * total + row) * ld;
  const int n1 = visible_windows_dev(t, 32, 16);
  uint32_t kmin = 0xffffffffu, kmax = 0u;
  // a candidate ends at least n_local blocks before b_t, so its five
  // windows 4b-1 .. 4b+3 are all visible: one 16-byte load and one scalar;
  // eight candidates per lane are loaded before any is used
  constexpr int kU = 8;
  for (int i0 = 0; i0 < ncand; i0 += 32 * kU) {
    float4 v4[kU];
    float pv[kU];
    if constexpr (POOL) {
      // pair b and the second value of pair b-1 (every candidate's first
      // window is visible, so both pairs were written)
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int i = i0 + u * 32 + lane;
        const int b = cand_lo + i;
        const bool ok = i < ncand;
        const float2 pr = ok ? __ldg(reinterpret_cast<const float2*>(srow + 2 * b)) : make_float2(0.f, 0.f);
        v4[u] = make_float4(pr.x, pr.y, 0.f, 0.f);
        pv[u] = (ok && b >= 1) ? __ldg(srow + 2 * b - 1) : -INFINITY;
      }
    } else {
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int i = i0 + u * 32 + lane;
        const int b = cand_lo + i;
        const bool fast = i < ncand && b >= 1 && 4 * b + 3 < n1;
        v4[u] = fast ? __ldg(reinterpret_cast<const float4*>(srow + 4 * b)) : make_float4(0.f, 0.f, 0.f, 0.f);
        pv[u] = fast ? __ldg(srow + 4 * b - 1) : 0.f;
      }
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int i = i0 + u * 32 + lane;
      if (i < ncand) {
        const int b = cand_lo + i;
        float m;
        if constexpr (POOL)
          m = fmaxf(v4[u].x, pv[u]);
        else
          m = (b >= 1 && 4 * b + 3 < n1)
                  ? fmaxf(fmaxf(pv[u], v4[u].x), fmaxf(fmaxf(v4[u].y, v4[u].z), v4[u].w))
                  : block_score(srow, b, n1);
        const uint32_t k = __float_as_uint(fmaxf(m, 0.f));
        keys[i] = k;
        kmin = min(kmin, k);
        kmax = max(kmax, k);
      }
    }
  }
  warp_select_write(keys, hist, ncand, cand_lo, init_hi, loc_lo, b_t, top_k, n_sel, kmin, kmax, out, lane);
}

}  // namespace sel

cudaError_t launch_topk(const float* S, int64_t ld, const int32_t* cu, int batch, int max_seqlen, int64_t total,
                        int h_kv, int n_init, int n_local, int top_k, bool pool, cudaStream_t st, int32_t* out) {
  const int n_sel = n_init + n_local + top_k;
  const int cand_cap = ((max_seqlen + 63) / 64 + 31) & ~31;
  const size_t per_warp = (static_cast<size_t>(cand_cap) + sel::kHistBins) * 4;
  int wpb = static_cast<int>((160 * 1024) / per_warp);
  wpb = max(1, min(8, wpb));
  const size_t smem = per_warp * wpb;
  if (smem > 220 * 1024) return cudaErrorInvalidValue;
  auto kern = pool ? sel::topk_kernel<true> : sel::topk_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int64_t units = static_cast<int64_t>(h_kv) * total;
  const int64_t blocks = (units + wpb - 1) / wpb;
  if (blocks == 0) return cudaSuccess;
  kern<<<static_cast<unsigned>(blocks), wpb * 32, smem, st>>>(S, ld, cu, batch, total, h_kv, n_init, n_local, top_k,
                                                              n_sel, cand_cap, out);
  return cudaGetLastError();
}

}  // namespace infllm2
