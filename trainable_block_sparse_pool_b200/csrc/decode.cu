// Step 5: one decode step — a new token per sequence against a KV cache,
// with the pooled key caches kept current (InfLLM-V2 keeps the sparse
// pattern for decoding too: dtcms article §二.2.b, "prefill 与 decode 全链路";
// the pages' end-to-end decode measurement at |I| = 96).
//
// The new token of sequence b sits at position t = seq_len[b]; the step is
// row t of the prefill rule applied to the sequence extended by one token.
// Three kernels (four with INFLLM2_DEC_SPLIT_SELECT=1):
//   K1 append k, v at t; if a stage-1 window ends at t (t+1 >= 32,
//      (t+1) % 16 == 0) pool it into K_c1, likewise a coarse window
//      (t+1 >= 128, (t+1) % 64 == 0) into K_c2 (exact mean, one bf16
//      rounding); per-head log-sum-exp partials over the visible coarse
//      windows, split over CTAs
//   K2 S over the visible stage-1 windows (head-group sum fused) and the
//      max-pool to block scores, streamed through TMA in one wave of CTAs
//   K2b the selection of each (sequence, group), one CTA each, once every
//      block score of the step is written (built with
//      INFLLM2_DEC_SPLIT_SELECT=0, K2's CTA that completes the last piece of a
//      (sequence, group) selects instead)
//   K3 split-KV block-sparse attention: before the wait for K2b each split
//      streams its share of the init and local blocks (every list holds
//      them), after it its share of the top-k blocks and of the query's own
//      block; the splits
//      of a (sequence, group) merge through distributed shared memory inside
//      a thread-block cluster (or, past 8 splits, through the workspace and
//      a completion counter), and the last group of a sequence advances
//      seq_len
// The hand-offs between CTAs are completion counters (threadfence, then
// atomicAdd) and cluster barriers; the kernels are chained with
// programmatic dependent launch.  No CTA spins on another's progress.
// All of it is HBM-bound (the pooled keys and the selected K/V are read
// once); the small contractions (16 heads against 8 keys or windows per
// instruction) use warp-level mma.sync, which is far from being the limit.
#include "sm100.cuh"

namespace infllm2 {

namespace dec {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kLseWin = 128;   // coarse windows per LSE CTA
constexpr int kMaxSplits = 256; // attention splits per (sequence, group)
constexpr float kRescaleLog2 = 8.f; // attention: raise the reference max only past this margin

// D = A(16x16, bf16, row) * B(16x8, bf16, col) + C, fp32 accumulate.
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// The contraction over d uses a fixed permutation of d inside each pair of
// 16-wide k steps, so a thread's operands are one 16-byte load: for
// k-step 2p+e, thread (gid, tig) covers d = 32p + 8 tig + 4e + {0,1} (as
// logical k 2tig, 2tig+1) and + {2,3} (as k 2tig+8, 2tig+9).  A and B use
// the same map, so the sum is unchanged.
template <int D>
struct QFrag {
  uint4 lo[D / 32], hi[D / 32];   // heads gid and gid + 8
};

template <int D>
__device__ __forceinline__ void load_qfrag(QFrag<D>& f, const __nv_bfloat16* q_heads /* [16][D] */, int lane,
                                           int G) {
  const int gid = lane >> 2, tig = lane & 3;
#pragma unroll
  for (int p = 0; p < D / 32; ++p) {
    const int off = 32 * p + 8 * tig;
    f.lo[p] = (gid < G) ? *reinterpret_cast<const uint4*>(q_heads + gid * D + off) : make_uint4(0, 0, 0, 0);
    f.hi[p] = (gid + 8 < G) ? *reinterpret_cast<const uint4*>(q_heads + (gid + 8) * D + off) : make_uint4(0, 0, 0, 0);
  }
}

// Scores of 16 heads against 8 keys whose rows (one per lane group gid)
// are already in registers: c[0..1] head gid, keys 2tig, 2tig+1; c[2..3]
// head gid+8.  load_krow fetches a row (nullptr = zero row), so a warp can
// issue every load it needs before the first MMA.
template <int D>
__device__ __forceinline__ void load_krow(uint4 (&kv)[D / 32], const __nv_bfloat16* row, int lane) {
  const int tig = lane & 3;
#pragma unroll
  for (int p = 0; p < D / 32; ++p)
    kv[p] = row ? *reinterpret_cast<const uint4*>(row + 32 * p + 8 * tig) : make_uint4(0, 0, 0, 0);
}
template <int D>
__device__ __forceinline__ void scores_16x8_reg(float (&c)[4], const QFrag<D>& f, const uint4 (&kv)[D / 32]) {
  c[0] = c[1] = c[2] = c[3] = 0.f;
#pragma unroll
  for (int p = 0; p < D / 32; ++p) {
    const uint32_t a0[4] = {f.lo[p].x, f.hi[p].x, f.lo[p].y, f.hi[p].y};
    mma16816(c, a0, kv[p].x, kv[p].y);
    const uint32_t a1[4] = {f.lo[p].z, f.hi[p].z, f.lo[p].w, f.hi[p].w};
    mma16816(c, a1, kv[p].z, kv[p].w);
  }
}

// ---------------------------------------------------------------- cp.async staging
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool full) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(full ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait0() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait_n() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr)
               : "memory");
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr)
               : "memory");
}
// ---------------------------------------------------------------- programmatic dependent launch
// The three kernels of a step are chained with programmatic stream
// serialization: a kernel lets its dependent launch as soon as all of its
// CTAs have started, and the dependent does its setup (which reads nothing
// the primary writes) before waiting for the primary grid to complete.
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// ---------------------------------------------------------------- thread-block clusters
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// every thread of every CTA of the cluster: writes before are visible to reads after
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// the address of this CTA's shared-memory word `local` in the CTA of the cluster with rank `rank`
__device__ __forceinline__ uint32_t dsmem_addr(uint32_t local, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
  return r;
}
// (volatile: kept in order with the cluster barriers; no memory clobber, so
// loads of independent items can be in flight together)
__device__ __forceinline__ float ld_dsmem(uint32_t a) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ float4 ld_dsmem4(uint32_t a) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(a));
  return v;
}

// ---------------------------------------------------------------- pooling of the window that ends at t
// Window [t - len + 1, t] of kv group g: rows before t from the cache, row t
// from k_new (it may not be in the cache yet).  Exact mean in fp64, one bf16
// rounding, written to dst.  All 128 threads of the CTA take part; `part` is
// shared scratch of (128 / (D/8)) x D doubles.
template <int D>
__device__ void pool_window(int len, const __nv_bfloat16* kc, int64_t seq0, int h_kv, int g, int t,
                            const __nv_bfloat16* kn, __nv_bfloat16* dst, double* part) {
  constexpr int SL = D / 8;
  constexpr int NRG = 128 / SL;                 // row groups of the 128 threads
  const int sl = threadIdx.x % SL, rg = threadIdx.x / SL;
  double acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.0;
#pragma unroll 4
  for (int r = rg; r < len; r += NRG) {
    const int u = t - len + 1 + r;
    const __nv_bfloat16* src = (u == t) ? kn : kc + ((seq0 + u) * h_kv + g) * D;
    const uint4 raw = reinterpret_cast<const uint4*>(src)[sl];
    const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(p2[i]);
      acc[2 * i] += static_cast<double>(f.x);
      acc[2 * i + 1] += static_cast<double>(f.y);
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) part[rg * D + sl * 8 + i] = acc[i];
  __syncthreads();
  if (threadIdx.x < SL) {
    uint16_t o[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      double s = 0.0;
      for (int q = 0; q < NRG; ++q) s += part[q * D + threadIdx.x * 8 + i];
      o[i] = f64_to_bf16_rne(s / len);
    }
    uint4 v;
    v.x = o[0] | (static_cast<uint32_t>(o[1]) << 16);
    v.y = o[2] | (static_cast<uint32_t>(o[3]) << 16);
    v.z = o[4] | (static_cast<uint32_t>(o[5]) << 16);
    v.w = o[6] | (static_cast<uint32_t>(o[7]) << 16);
    reinterpret_cast<uint4*>(dst)[threadIdx.x] = v;
  }
  __syncthreads();                              // part is free again; dst is visible to the CTA
}

// ---------------------------------------------------------------- K1: append, pooling, coarse LSE partials
// grid (batch*h_kv, nsplit2), 4 warps; CTA c covers coarse windows
// [128c, 128c + 128).
//  * CTA 0 of (b, g) clears the step's completion counters, appends k, v at
//    row t and pools the stage-1 window that ends at t, when one does.
//  * The CTA whose range holds a coarse window ending at t pools it first and
//    then uses it.
//  * Every CTA writes (max, sum) in log2 units of its windows' scores, per
//    head: part2[(bg*nsplit2 + c)*16 + h].
// Counters (cnt): [0, nbg) score pieces done per (b, g); [nbg, 2 nbg)
// attention CTAs done per (b, g); [2 nbg, 2 nbg + batch) groups of b merged.
template <int D>
__global__ void __launch_bounds__(128) lse_append_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k_new,
    const __nv_bfloat16* __restrict__ v_new, __nv_bfloat16* kc, __nv_bfloat16* vc, __nv_bfloat16* kc1,
    __nv_bfloat16* kc2, const int32_t* __restrict__ seq_len, int capacity, int h_q, int h_kv, int cap_c1, int cap_c2,
    float scale, float2* __restrict__ part2, unsigned* __restrict__ cnt) {
  constexpr int SL = D / 8;
  __shared__ double pool_part[(128 / SL) * D];
  __shared__ float2 red[4][16];
  const int bg = blockIdx.x, c = blockIdx.y, nbg = gridDim.x;
  const int b = bg / h_kv, g = bg % h_kv;
  const int G = h_q / h_kv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gid = lane >> 2, tig = lane & 3;
  griddep_launch_dependents();
  if (c == 0 && threadIdx.x == 0) {
    cnt[bg] = 0u;
    cnt[nbg + bg] = 0u;
    if (g == 0) cnt[2 * nbg + b] = 0u;
  }
  const int t = seq_len[b];
  if (t < 0 || t >= capacity) {
    if (c == 0 && g == 0 && threadIdx.x == 0) record_status(INFLLM2_ERR_DEVICE_BOUNDS);
    return;
  }
  const int64_t seq0 = static_cast<int64_t>(b) * capacity;
  const __nv_bfloat16* kn = k_new + (static_cast<int64_t>(b) * h_kv + g) * D;
  if (c == 0) {
    if (threadIdx.x < SL) {
      const __nv_bfloat16* vn = v_new + (static_cast<int64_t>(b) * h_kv + g) * D;
      reinterpret_cast<uint4*>(kc + ((seq0 + t) * h_kv + g) * D)[threadIdx.x] = reinterpret_cast<const uint4*>(kn)[threadIdx.x];
      reinterpret_cast<uint4*>(vc + ((seq0 + t) * h_kv + g) * D)[threadIdx.x] = reinterpret_cast<const uint4*>(vn)[threadIdx.x];
    }
    if (t + 1 >= 32 && (t + 1 - 32) % 16 == 0) {
      const int j = (t + 1 - 32) / 16;
      if (j < cap_c1) pool_window<D>(32, kc, seq0, h_kv, g, t, kn, kc1 + (static_cast<int64_t>(bg) * cap_c1 + j) * D, pool_part);
      else if (threadIdx.x == 0) record_status(INFLLM2_ERR_DEVICE_BOUNDS);
    }
  }
  if (t + 1 >= 128 && (t + 1 - 128) % 64 == 0) {
    const int j = (t + 1 - 128) / 64;
    if (j / kLseWin == c) {
      if (j < cap_c2) pool_window<D>(128, kc, seq0, h_kv, g, t, kn, kc2 + (static_cast<int64_t>(bg) * cap_c2 + j) * D, pool_part);
      else if (threadIdx.x == 0) record_status(INFLLM2_ERR_DEVICE_BOUNDS);
    }
  }
  const int n2 = min(visible_windows_dev(t, 128, 64), cap_c2);
  QFrag<D> f;
  load_qfrag<D>(f, q + (static_cast<int64_t>(b) * h_q + g * G) * D, lane, G);
  const float cs = scale * kLog2e;
  float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};   // heads gid, gid+8
  const __nv_bfloat16* base = kc2 + static_cast<int64_t>(bg) * cap_c2 * D;
  constexpr int kMaxNt = kLseWin / 8 / 4;
  uint4 kv[kMaxNt][D / 32];
#pragma unroll
  for (int i = 0; i < kMaxNt; ++i) {
    const int wr = c * kLseWin + (warp + 4 * i) * 8 + gid;
    load_krow<D>(kv[i], (wr < n2) ? base + static_cast<int64_t>(wr) * D : nullptr, lane);
  }
#pragma unroll
  for (int i = 0; i < kMaxNt; ++i) {
    const int nt = warp + 4 * i;
    const int w0 = c * kLseWin + nt * 8;
    if (w0 >= n2) break;
    float sc[4];
    scores_16x8_reg<D>(sc, f, kv[i]);
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      float x0 = (w0 + 2 * tig < n2) ? sc[2 * r] * cs : -INFINITY;
      float x1 = (w0 + 2 * tig + 1 < n2) ? sc[2 * r + 1] * cs : -INFINITY;
      const float mn = fmaxf(m[r], fmaxf(x0, x1));
      if (mn != -INFINITY) {
        l[r] = l[r] * ex2(m[r] - mn) + ex2(x0 - mn) + ex2(x1 - mn);
        m[r] = mn;
      }
    }
  }
  // combine over the 4 lanes of a head row, then over warps
#pragma unroll
  for (int r = 0; r < 2; ++r) {
#pragma unroll
    for (int o = 1; o <= 2; o <<= 1) {
      const float mo = __shfl_xor_sync(0xffffffffu, m[r], o);
      const float lo = __shfl_xor_sync(0xffffffffu, l[r], o);
      const float mn = fmaxf(m[r], mo);
      if (mn != -INFINITY) {
        l[r] = l[r] * ex2(m[r] - mn) + lo * ex2(mo - mn);
        m[r] = mn;
      }
    }
  }
  if (tig == 0) {
    red[warp][gid] = make_float2(m[0], l[0]);
    red[warp][gid + 8] = make_float2(m[1], l[1]);
  }
  __syncthreads();
  if (threadIdx.x < 16) {
    float mm = -INFINITY, ll = 0.f;
    for (int w = 0; w < 4; ++w) {
      const float2 v = red[w][threadIdx.x];
      const float mn = fmaxf(mm, v.x);
      if (mn != -INFINITY) {
        ll = ll * ex2(mm - mn) + v.y * ex2(v.x - mn);
        mm = mn;
      }
    }
    part2[(static_cast<int64_t>(bg) * gridDim.y + c) * 16 + threadIdx.x] = make_float2(mm, ll);
  }
}

// ---------------------------------------------------------------- block selection of one (sequence, group)
// Run by the 256 threads of one CTA.  Candidates are the blocks after the
// init blocks and before the local run; the top_k largest block scores are
// found with an exact radix select (8-bit digits of the fp32 bit pattern of
// score - min; the scores are >= 0, so the bit order is the value order),
// ties go to the lower block.  Output: init blocks, the chosen candidates
// ascending, the local run, -1 padding ([top168] §三 third stage, §七).
constexpr int kSelThreads = 256;
struct SelScratch {
  int hist[256];
  uint32_t red[2][kSelThreads / 32];
  int wsum[kSelThreads / 32];
  int digit, above;
  uint32_t small[32];                 // the keys of a boundary bin of at most 32
  int nsmall, gt;
  uint32_t tu;
};
constexpr int kSelBins = 2048;        // first radix pass: the top 11 bits

// exclusive prefix sum of v over the CTA's threads in index order; *total
// gets the sum over all threads
__device__ __forceinline__ int cta_exclusive_scan(int v, int* wsum, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wsum[warp] = x;
  __syncthreads();
  int before = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < kSelThreads / 32; ++w) {
    const int s = wsum[w];
    before += (w < warp) ? s : 0;
    tot += s;
  }
  __syncthreads();                              // wsum may be reused
  *total = tot;
  return before + x - v;
}

// keys: shared scratch of cand_cap entries; big: shared scratch of kSelBins ints.
__device__ void select_blocks_cta(const float* row, int t, int n_init, int n_local, int top_k, int n_sel,
                                  int cand_cap, int32_t* out, uint32_t* keys, int* big, SelScratch& sh) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int NW = kSelThreads / 32;
  const int b_t = t / 64;
  const int init_hi = min(n_init, b_t + 1);
  const int loc_lo = max(0, b_t - n_local + 1);
  const int ncand = max(0, loc_lo - init_hi);
  if (ncand <= top_k) {                         // every causal block fits
    for (int i = tid; i < n_sel; i += kSelThreads) out[i] = (i <= b_t) ? i : -1;
    return;
  }
  if (ncand > cand_cap) {
    if (tid == 0) record_status(INFLLM2_ERR_DEVICE_BOUNDS);
    return;
  }
  // the first pass's bins are cleared while the keys load (the barrier after
  // the key range covers both)
  for (int i = tid; i < kSelBins; i += kSelThreads) big[i] = 0;
  uint32_t kmin = 0xffffffffu, kmax = 0u;
  for (int i0 = 0; i0 < ncand; i0 += 8 * kSelThreads) {        // eight loads in flight per thread
    float v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = i0 + u * kSelThreads + tid;
      v[u] = (i < ncand) ? __ldcg(row + init_hi + i) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = i0 + u * kSelThreads + tid;
      if (i < ncand) {
        const uint32_t k = __float_as_uint(fmaxf(v[u], 0.f));
        keys[i] = k;
        kmin = min(kmin, k);
        kmax = max(kmax, k);
      }
    }
  }
  kmin = sel::warp_min_u32(kmin);
  kmax = sel::warp_max_u32(kmax);
  if (lane == 0) { sh.red[0][warp] = kmin; sh.red[1][warp] = kmax; }
  __syncthreads();
  kmin = 0xffffffffu; kmax = 0u;
#pragma unroll
  for (int w = 0; w < NW; ++w) { kmin = min(kmin, sh.red[0][w]); kmax = max(kmax, sh.red[1][w]); }
  const uint32_t range = kmax - kmin;
  int hi = range ? 32 - __clz(range) : 0;
  uint32_t prefix = 0;
  int k_rem = top_k;                            // how many of the keys matching prefix are still to take
  if (hi > 0) {
    // first pass over the top (up to) 11 bits of u, 2048 bins; thread tid
    // owns bins [8 tid, 8 tid + 8)
    const int d1 = min(hi, 11), shift1 = hi - d1, nb1 = 1 << d1;
    for (int i = tid; i < ncand; i += kSelThreads) atomicAdd(&big[(keys[i] - kmin) >> shift1], 1);
    __syncthreads();
    int loc = 0;
#pragma unroll
    for (int q = 0; q < 8; ++q) loc += (8 * tid + q < nb1) ? big[8 * tid + q] : 0;
    int tot;
    const int below = cta_exclusive_scan(loc, sh.wsum, &tot);
    const int above = tot - below - loc;        // keys in bins above this thread's
    if (above < k_rem && above + loc >= k_rem) {
      int acc = above;
      for (int q = 7; q >= 0; --q) {
        const int bb = 8 * tid + q;
        const int hh = (bb < nb1) ? big[bb] : 0;
        if (acc + hh >= k_rem) { sh.digit = bb; sh.above = acc; break; }
        acc += hh;
      }
    }
    __syncthreads();
    const int dg = sh.digit;
    const int in_bin = big[dg];
    prefix = static_cast<uint32_t>(dg) << shift1;
    k_rem -= sh.above;
    hi = shift1;
    if (tid == 0) sh.nsmall = 0;
    __syncthreads();                            // big, digit and above are read by everyone
    if (hi > 0 && in_bin <= 32) {
      // the few keys of the boundary bin: one warp sorts them and takes the
      // k_rem-th largest exactly
      for (int i = tid; i < ncand; i += kSelThreads) {
        const uint32_t u = keys[i] - kmin;
        if ((u >> shift1) == static_cast<uint32_t>(dg)) sh.small[atomicAdd(&sh.nsmall, 1)] = u;
      }
      __syncthreads();
      if (warp == 0) {
        const int n = sh.nsmall;
        uint32_t x = (lane < n) ? sh.small[lane] : 0u;   // 0 sorts last: no key of the bin is below it
        // bitonic sort, descending across the 32 lanes
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
        const int gt = __popc(__ballot_sync(0xffffffffu, lane < n && x > tu));
        if (lane == 0) { sh.tu = tu; sh.gt = gt; }
      }
      __syncthreads();
      prefix = sh.tu;
      k_rem -= sh.gt;
      hi = 0;
    }
  }
  while (hi > 0) {                              // a crowded boundary bin: 8 more bits per pass
    const int shift = max(0, hi - 8);
    const int nb = 1 << (hi - shift);
    sh.hist[tid] = 0;
    __syncthreads();
    const uint64_t want = static_cast<uint64_t>(prefix) >> hi;
    for (int i = tid; i < ncand; i += kSelThreads) {
      const uint32_t u = keys[i] - kmin;
      if ((static_cast<uint64_t>(u) >> hi) == want) atomicAdd(&sh.hist[(u >> shift) & (nb - 1)], 1);
    }
    __syncthreads();
    if (warp == 0) {
      // suffix sums from the top digit down: the digit where they reach k_rem
      int lsum = 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) lsum += (lane * 8 + q < nb) ? sh.hist[lane * 8 + q] : 0;
      int suf = lsum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_down_sync(0xffffffffu, suf, o);
        if (lane + o < 32) suf += v;
      }
      int above = suf - lsum;
      if (above < k_rem && suf >= k_rem) {
        for (int q = 7; q >= 0; --q) {
          const int bb = lane * 8 + q;
          const int hh = (bb < nb) ? sh.hist[bb] : 0;
          if (above + hh >= k_rem) { sh.digit = bb; sh.above = above; break; }
          above += hh;
        }
      }
    }
    __syncthreads();
    prefix |= static_cast<uint32_t>(sh.digit) << shift;
    k_rem -= sh.above;
    hi = shift;
    __syncthreads();                            // hist, digit and above are rewritten by the next pass
  }
  const uint32_t T = kmin + prefix;             // the top_k-th largest key; k_rem keys equal to it are taken
  // one ordered pass: thread tid owns candidates [tid*per, tid*per + per),
  // per a multiple of 4 so they load as 16-byte vectors; one scan of the
  // packed counts (greater in the low 16 bits, equal in the high) gives each
  // thread its output position and its share of the equal keys
  const int per = ((ncand + 4 * kSelThreads - 1) / (4 * kSelThreads)) * 4;
  const int c0 = min(ncand, tid * per), c1 = min(ncand, c0 + per);
  int n_gt = 0, n_eq = 0;
  for (int i = c0; i < c1; i += 4) {
    const uint4 k4 = *reinterpret_cast<const uint4*>(keys + i);
    const uint32_t kk[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      n_gt += (i + u < c1) && kk[u] > T;
      n_eq += (i + u < c1) && kk[u] == T;
    }
  }
  int tot;
  const int before = cta_exclusive_scan(n_gt | (n_eq << 16), sh.wsum, &tot);
  const int gt_before = before & 0xffff, eq_before = before >> 16;
  const int eq_take = max(0, min(n_eq, k_rem - eq_before));
  int pos = init_hi + gt_before + min(eq_before, k_rem), eq_seen = 0;
  for (int i = c0; i < c1; i += 4) {
    const uint4 k4 = *reinterpret_cast<const uint4*>(keys + i);
    const uint32_t kk[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (i + u < c1) {
        const bool take = (kk[u] > T) || (kk[u] == T && eq_seen++ < eq_take);
        if (take) out[pos++] = init_hi + i + u;
      }
    }
  }
  for (int i = tid; i < init_hi; i += kSelThreads) out[i] = i;
  const int nloc = b_t - loc_lo + 1;
  for (int i = tid; i < nloc; i += kSelThreads) out[init_hi + top_k + i] = loc_lo + i;
  for (int i = init_hi + top_k + nloc + tid; i < n_sel; i += kSelThreads) out[i] = -1;
}

// ---------------------------------------------------------------- K2: scores, max-pool, selection
// The scoring streams over pieces.  A piece is kPieceWin = 128 consecutive
// stage-1 windows (32 blocks) of one (sequence, group); (b, g) has np(b)
// pieces, enough to cover its candidate blocks [0, loc_lo), or a single empty
// piece when the selection needs no scores.  The pieces of all (b, g), in
// (b, g) order, are cut into gridDim.x contiguous ranges of near-equal
// length, and a CTA walks its range through a kScoreStages-deep cp.async
// ring, so the pooled-key reads of the whole step stream without the gaps of
// a grid of short-lived CTAs.
// Per window: the 16 heads' scores, normalised by their LSE and summed over
// the group ([top168] §三 second stage, §四); per block i: the max over
// windows 4i-1 .. 4i+3.  A stage is one TMA box of kPieceRows rows starting
// 8 windows before the piece (zeros before window 0): its first n-tile holds
// the window before the piece (the first block's halo), which is scored only
// when the range does not hold the previous piece (else that piece's last
// window is carried over).  The box is 128-byte swizzled (16-byte chunk c of
// row r at chunk c ^ (r & 7)); lane group gid of an n-tile reads row
// (gid >> 1) | ((gid & 1) << 2), so the two rows of each 8-lane phase of a
// fragment load differ in swizzle bit 2 and the loads are free of bank
// conflicts.
// A completion counter per (b, g) counts the pieces done; the CTA that
// completes the last one runs that selection once its range is done.
#ifndef INFLLM2_DEC_PIECE
#define INFLLM2_DEC_PIECE 128
#endif
#ifndef INFLLM2_DEC_STAGES
#define INFLLM2_DEC_STAGES 2
#endif
#ifndef INFLLM2_DEC_EARLY
#define INFLLM2_DEC_EARLY 0
#endif
constexpr int kPieceWin = INFLLM2_DEC_PIECE;    // stage-1 windows per piece
constexpr int kPieceBlk = kPieceWin / 4;        // blocks per piece
constexpr int kPieceRows = kPieceWin + 8;       // the n-tile before the piece, then the piece
constexpr int kScoreStages = INFLLM2_DEC_STAGES;
static_assert(kPieceBlk <= 32 && (kPieceRows * 128) % 1024 == 0, "piece geometry");
constexpr int kMaxRange = 64;                   // pieces per CTA at most (the host sizes the grid)

template <int D>
struct ScoreCfg {
  static constexpr uint32_t kHalf = kPieceRows * 128;               // one 64-column box (1024-byte multiple)
  static constexpr uint32_t kStage = kPieceRows * D * 2;            // D / 64 boxes
  static constexpr uint32_t kRing = kScoreStages * kStage;
  static constexpr uint32_t kSmem = kRing + 1024;                   // + alignment of the swizzled boxes
  static_assert(kHalf % 1024 == 0, "128-byte swizzled boxes start on 1024-byte boundaries");
};

// Pieces of a (sequence, group) whose new token is at t: its scored blocks
// are [0, loc_lo); a single empty piece when every candidate is taken (or t
// is out of range, which the append kernel records).
__device__ __forceinline__ bool needs_scores(int t, int n_init, int n_local, int top_k) {
  const int b_t = t / 64;
  return max(0, b_t - n_local + 1) - min(n_init, b_t + 1) > top_k;
}
__device__ __forceinline__ int score_pieces(int t, int capacity, int n_init, int n_local, int top_k) {
  if (t < 0 || t >= capacity || !needs_scores(t, n_init, n_local, top_k)) return 1;
  return (max(0, t / 64 - n_local + 1) + kPieceBlk - 1) / kPieceBlk;
}

template <int D>
__global__ void __launch_bounds__(kSelThreads, 3) score_select_kernel(
    const __grid_constant__ CUtensorMap tmK1, const __nv_bfloat16* __restrict__ q,
    const __nv_bfloat16* __restrict__ kc1, const int32_t* __restrict__ seq_len,
    const float2* __restrict__ part2, int nsplit2, int batch, int capacity, int h_q, int h_kv, int cap_c1,
    int nblk_cap, int cand_cap, float scale, int n_init, int n_local, int top_k, int n_sel,
    float* __restrict__ bscore, int32_t* __restrict__ idx, unsigned* __restrict__ cnt, int select_here) {
  using C = ScoreCfg<D>;
  extern __shared__ __align__(128) uint8_t sc_smem[];   // the ring; the selection's keys and bins reuse it
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(sc_smem) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t full_bar[kScoreStages];
  __shared__ uint32_t plist[kMaxRange];                // bg << 16 | piece index within (b, g)
  __shared__ int pn1[kMaxRange];                       // visible stage-1 windows; -1: t out of range
  __shared__ int pnp[kMaxRange];                       // pieces of the piece's (b, g); 0: not scored
  __shared__ float nlse[16];
  __shared__ float sw[2][kPieceWin + 8];
  __shared__ SelScratch sel_sh;
  __shared__ int owed[kMaxRange];
  __shared__ int nowed;
  const int G = h_q / h_kv;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gid = lane >> 2, tig = lane & 3;
  const float cs = scale * kLog2e;

  // ---- this CTA's pieces.  With at least one CTA per (b, g), (b, g) gets
  // np(b) * (n - nbg) / total + 1 CTAs (at most n in all), each a contiguous
  // share of its pieces, so no CTA switches groups; otherwise the flattened
  // list of all pieces is cut into n contiguous ranges.
  __shared__ int s_R;
  griddep_launch_dependents();
  int R = 0;
  {
    const int n = gridDim.x, nbg = batch * h_kv;
    const bool aligned = n >= nbg;
    if (tid == 0) s_R = 0;
    int total = 0;
    for (int b0 = 0; b0 < batch; b0 += kSelThreads) {
      const int b = b0 + tid;
      const int v = (b < batch) ? h_kv * score_pieces(seq_len[b], capacity, n_init, n_local, top_k) : 0;
      int tot;
      cta_exclusive_scan(v, sel_sh.wsum, &tot);
      total += tot;
    }
    const int64_t P0 = static_cast<int64_t>(total) * blockIdx.x / n;
    const int64_t P1 = static_cast<int64_t>(total) * (blockIdx.x + 1) / n;
    if (!aligned) {
      R = static_cast<int>(P1 - P0);
      if (R > kMaxRange) {                     // the host sizes the grid so that this cannot happen
        if (tid == 0) record_status(INFLLM2_ERR_DEVICE_BOUNDS);
        return;
      }
    }
    int base = 0;                              // aligned: CTAs before sequence b; else pieces before it
    for (int b0 = 0; b0 < batch; b0 += kSelThreads) {
      const int b = b0 + tid;
      const int tb = (b < batch) ? seq_len[b] : -1;
      const int np = (b < batch) ? score_pieces(tb, capacity, n_init, n_local, top_k) : 0;
      const int cg = (b < batch) ? static_cast<int>(static_cast<int64_t>(np) * (n - nbg) / total) + 1 : 0;
      int tot;
      const int ex = cta_exclusive_scan(h_kv * (aligned ? cg : np), sel_sh.wsum, &tot);
      const bool valid = tb >= 0 && tb < capacity;
      const int n1 = valid ? min(visible_windows_dev(tb, 32, 16), cap_c1) : -1;
      const bool sc = valid && needs_scores(tb, n_init, n_local, top_k);
      if (aligned) {
        // CTAs [base + ex, base + ex + h_kv * cg) belong to sequence b
        const int i = static_cast<int>(blockIdx.x) - (base + ex);
        if (b < batch && i >= 0 && i < h_kv * cg) {
          const int g = i / cg, u = i - g * cg;
          const int p0 = np * u / cg, p1 = np * (u + 1) / cg;
          if (p1 - p0 > kMaxRange) {           // the host sizes the grid so that this cannot happen
            record_status(INFLLM2_ERR_DEVICE_BOUNDS);
            s_R = -1;
          } else {
            for (int j = 0; j < p1 - p0; ++j) {
              plist[j] = (static_cast<uint32_t>(b * h_kv + g) << 16) | static_cast<uint32_t>(p0 + j);
              pn1[j] = n1;
              pnp[j] = sc ? np : 0;
            }
            s_R = p1 - p0;
          }
        }
      } else {
        // pieces [base + ex, base + ex + h_kv * np) belong to sequence b
        const int64_t lo = max(static_cast<int64_t>(base) + ex, P0);
        const int64_t hi = min(static_cast<int64_t>(base) + ex + h_kv * np, P1);
        for (int64_t i = lo; i < hi; ++i) {
          const int rem = static_cast<int>(i - base - ex);
          const int g = rem / np, p = rem - g * np;
          const int j = static_cast<int>(i - P0);
          plist[j] = (static_cast<uint32_t>(b * h_kv + g) << 16) | static_cast<uint32_t>(p);
          pn1[j] = n1;
          pnp[j] = sc ? np : 0;
        }
      }
      base += tot;
      if (!aligned && base >= P1) break;      // uniform: base and P1 are the same in every thread
    }
    if (tid == 0) {
      nowed = 0;
      for (int st = 0; st < kScoreStages; ++st) mbar_init(&full_bar[st], 1);
      fence_barrier_init();
    }
    __syncthreads();
    if (aligned) R = s_R;
  }
  // The mapping read only seq_len; the LSE partials (and the completion
  // counters) come from the append kernel.  The stage-1 windows the
  // selection reads do not: the only window the append kernel may pool ends
  // at t, and with n_local >= 2 it lies past the pooling range of every
  // candidate block (4(b_t - n_local) + 3 < (t - 31) / 16), so the first
  // pieces' copies can go out before the wait and overlap the append kernel.
  const bool early = INFLLM2_DEC_EARLY && n_local >= 2;
  if (!early) griddep_wait();
  if (R <= 0) return;
  auto bg_of = [&](int j) { return static_cast<int>(plist[j] >> 16); };
  auto p_of = [&](int j) { return static_cast<int>(plist[j] & 0xffffu); };
  auto seg_first = [&](int j) { return j == 0 || bg_of(j - 1) != bg_of(j); };
  auto seg_last = [&](int j) { return j == R - 1 || bg_of(j + 1) != bg_of(j); };

  // stage piece j: one box per 64 columns, windows w0 - 8 .. w0 + 127 (rows
  // outside the pooled cache read as zeros; rows of windows not yet visible
  // are masked below)
  auto stage = [&](int j) {
    if (tid == 0 && j < R && pnp[j] > 0) {
      const int st = j % kScoreStages;
      mbar_arrive_expect_tx(&full_bar[st], C::kStage);
#pragma unroll
      for (int h = 0; h < D / 64; ++h)
        tma_load_3d(ring + st * C::kStage + h * C::kHalf, &tmK1, &full_bar[st], 64 * h, p_of(j) * kPieceWin - 8,
                    bg_of(j));
    }
  };
  // the group's negated log-sum-exp per head (log2 units) from the coarse
  // partials: thread (h, k0) folds partials k0, k0 + 16, ..., then the 16
  // lanes of h combine
  auto group_lse = [&](int j) {                // every thread; scored pieces only
    const int bg = bg_of(j), n1 = pn1[j];
    const int b = bg / h_kv, g = bg - b * h_kv;
    const int tb = seq_len[b];
    const int n2 = visible_windows_dev(tb, 128, 64);
    const int h = tid >> 4, k0 = tid & 15;
    float mm = -INFINITY, ll = 0.f;
    if (h < G && n2 > 0) {
      for (int kk = k0; kk < nsplit2; kk += 16) {
        const float2 v = part2[(static_cast<int64_t>(bg) * nsplit2 + kk) * 16 + h];
        const float mn = fmaxf(mm, v.x);
        if (mn != -INFINITY) {
          ll = ll * ex2(mm - mn) + v.y * ex2(v.x - mn);
          mm = mn;
        }
      }
    }
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) {
      const float mo = __shfl_xor_sync(0xffffffffu, mm, o);
      const float lo = __shfl_xor_sync(0xffffffffu, ll, o);
      const float mn = fmaxf(mm, mo);
      if (mn != -INFINITY) {
        ll = ll * ex2(mm - mn) + lo * ex2(mo - mn);
        mm = mn;
      }
    }
    if (k0 == 0) {
      if (h < G && n2 <= 0 && n1 > 0) {
        // no coarse window yet (t < 127): exact log-sum-exp over the visible stage-1 windows
        const __nv_bfloat16* qh = q + (static_cast<int64_t>(b) * h_q + g * G) * D;
        const __nv_bfloat16* base = kc1 + static_cast<int64_t>(bg) * cap_c1 * D;
        mm = -INFINITY;
        ll = 0.f;
        for (int w = 0; w < n1; ++w) {
          float dot = 0.f;
          for (int e = 0; e < D; ++e)
            dot += __bfloat162float(qh[h * D + e]) * __bfloat162float(base[static_cast<int64_t>(w) * D + e]);
          const float x = dot * cs;
          const float mn = fmaxf(mm, x);
          ll = ll * ex2(mm - mn) + ex2(x - mn);
          mm = mn;
        }
      }
      nlse[h] = (h < G && ll > 0.f) ? -(mm + log2f(ll)) : -INFINITY;
    }
  };

#pragma unroll
  for (int s = 0; s < kScoreStages - 1; ++s) stage(s);
  if (early) griddep_wait();
  if (pnp[0] > 0) group_lse(0);
  QFrag<D> f;
  {
    const int bg = bg_of(0), b = bg / h_kv, g = bg - b * h_kv;
    load_qfrag<D>(f, q + (static_cast<int64_t>(b) * h_q + g * G) * D, lane, G);
  }
  int seg_start = 0;
  uint32_t phase = 0;                          // bit s: parity of stage s's next fill
  for (int j = 0; j < R; ++j) {
    __syncthreads();                           // stage (j - 1) % S and sw[(j + 1) & 1] are free
    stage(j + kScoreStages - 1);
    const int bg = bg_of(j), p = p_of(j), n1 = pn1[j];
    const bool live = pnp[j] > 0;
    if (j > 0 && seg_first(j)) {
      seg_start = j;
      if (live) {
        group_lse(j);
        __syncthreads();
        const int b = bg / h_kv, g = bg - b * h_kv;
        load_qfrag<D>(f, q + (static_cast<int64_t>(b) * h_q + g * G) * D, lane, G);
      }
    }
    const int w0 = p * kPieceWin;
    const bool halo = seg_first(j) && p > 0;
    float* swc = sw[j & 1];
    if (live) {
      const int st = j % kScoreStages;
      mbar_wait(&full_bar[st], (phase >> st) & 1u);
      phase ^= 1u << st;
      const float nl0 = nlse[gid], nl1 = nlse[gid + 8];
      const uint8_t* rows = ring + st * C::kStage;
      const int ntiles = halo ? kPieceWin / 8 + 1 : kPieceWin / 8;
      for (int i = warp; i < ntiles; i += kSelThreads / 32) {
        // the piece's n-tiles are box n-tiles 1 .. 16; the halo n-tile (box n-tile 0) comes last
        const int r = (i < kPieceWin / 8 ? 8 * (i + 1) : 0) + ((gid >> 1) | ((gid & 1) << 2));
        uint4 kv[D / 32];
#pragma unroll
        for (int pp = 0; pp < D / 32; ++pp) {
          const int ch = 4 * pp + tig;         // 16-byte chunk of the row: box ch >> 3, chunk ch & 7
          kv[pp] = *reinterpret_cast<const uint4*>(rows + (ch >> 3) * C::kHalf + r * 128 +
                                                   (((ch & 7) ^ (r & 7)) << 4));
        }
        float sc[4];
        scores_16x8_reg<D>(sc, f, kv);
        // head-group sum for windows 2tig and 2tig+1 of the n-tile: two heads here, the other 14 on the lanes with the same tig
        float e0 = ((gid < G) ? ex2(fmaf(sc[0], cs, nl0)) : 0.f) + ((gid + 8 < G) ? ex2(fmaf(sc[2], cs, nl1)) : 0.f);
        float e1 = ((gid < G) ? ex2(fmaf(sc[1], cs, nl0)) : 0.f) + ((gid + 8 < G) ? ex2(fmaf(sc[3], cs, nl1)) : 0.f);
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
          e0 += __shfl_xor_sync(0xffffffffu, e0, o);
          e1 += __shfl_xor_sync(0xffffffffu, e1, o);
        }
        // columns 2tig, 2tig + 1 are rows tig, tig + 4 of the n-tile
        if (gid == 0) {
          if (i < kPieceWin / 8) {
            const int wa = w0 + 8 * i + tig;
            swc[1 + 8 * i + tig] = (wa < n1) ? e0 : -INFINITY;
            swc[5 + 8 * i + tig] = (wa + 4 < n1) ? e1 : -INFINITY;
          } else if (tig == 3) {
            swc[0] = (w0 - 1 < n1) ? e1 : -INFINITY;   // row 7: the halo window w0 - 1 (w0 >= 128 here)
          }
        }
      }
    }
    __syncthreads();                           // sw[j & 1] complete
    if (warp == 0) {
      if (live && lane < kPieceBlk) {
        // block 32p + lane takes windows 4(32p + lane) - 1 .. + 3 = swc[4 lane .. 4 lane + 4],
        // where swc[0] (window w0 - 1) is the staged halo, the previous piece's
        // last window, or none (p == 0)
        const int blk = p * kPieceBlk + lane;
        float m = halo ? swc[0] : (p == 0 ? -INFINITY : sw[(j + 1) & 1][kPieceWin]);
        m = (lane == 0) ? m : swc[4 * lane];
#pragma unroll
        for (int q4 = 1; q4 < 5; ++q4) m = fmaxf(m, swc[4 * lane + q4]);
        if (blk < nblk_cap) bscore[static_cast<int64_t>(bg) * nblk_cap + blk] = m;
      }
      if (select_here && seg_last(j)) {
        // the segment's pieces are done: count them; the CTA that completes
        // the last piece of (b, g) owes its selection
        __threadfence();
        __syncwarp();
        if (lane == 0 && n1 >= 0) {
          const unsigned done = static_cast<unsigned>(j - seg_start + 1);
          const unsigned np = static_cast<unsigned>(live ? pnp[j] : 1);
          if (atomicAdd(&cnt[bg], done) + done == np) owed[nowed++] = bg;
        }
      }
    }
  }
  __syncthreads();                             // every fill was consumed: the ring is free
  const int no = nowed;
  if (no == 0) return;
  __threadfence();
  for (int o = 0; o < no; ++o) {
    const int bg = owed[o];
    const int t = seq_len[bg / h_kv];
    select_blocks_cta(bscore + static_cast<int64_t>(bg) * nblk_cap, t, n_init, n_local, top_k, n_sel, cand_cap,
                      idx + static_cast<int64_t>(bg) * n_sel, reinterpret_cast<uint32_t*>(sc_smem),
                      reinterpret_cast<int*>(sc_smem + ((static_cast<size_t>(cand_cap) * 4 + 15) & ~size_t(15))),
                      sel_sh);
    __syncthreads();                           // the scratch is reused by the next selection
  }
}

// ---------------------------------------------------------------- K2b: the selection of each (sequence, group)
// One CTA per (b, g), launched between the score kernel and the attention
// kernel (programmatic dependent launch on both sides): it waits for every
// block score of the step, then selects as select_blocks_cta does.  The
// attention kernel meanwhile streams the blocks every list holds (init and
// local), which need no selection.
__global__ void __launch_bounds__(kSelThreads) select_kernel(const float* __restrict__ bscore,
                                                             const int32_t* __restrict__ seq_len, int capacity,
                                                             int h_kv, int n_init, int n_local, int top_k, int n_sel,
                                                             int nblk_cap, int cand_cap, int32_t* __restrict__ idx) {
  extern __shared__ __align__(16) uint8_t sel_dyn[];
  __shared__ SelScratch sel_sh;
  griddep_launch_dependents();
  griddep_wait();                              // the block scores of the step
  const int bg = blockIdx.x;
  const int t = seq_len[bg / h_kv];
  if (t < 0 || t >= capacity) return;          // recorded by the append kernel
  select_blocks_cta(bscore + static_cast<int64_t>(bg) * nblk_cap, t, n_init, n_local, top_k, n_sel, cand_cap,
                    idx + static_cast<int64_t>(bg) * n_sel, reinterpret_cast<uint32_t*>(sel_dyn),
                    reinterpret_cast<int*>(sel_dyn + ((static_cast<size_t>(cand_cap) * 4 + 15) & ~size_t(15))), sel_sh);
}

constexpr int kAttWarps = 6;
constexpr int kChunkKeys = 32;

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

template <int D>
struct AttCfg {
  static constexpr int CH = D / 8;                            // 16-byte pieces per key row
  static constexpr int kRow = D + 8;                          // merge rows: D values, m, l, padding (bank spread)
  static constexpr int kPart = D + 4;                         // partial rows in HBM: D values, m, l, padding (16 B rows)
  static constexpr uint32_t kTile = kChunkKeys * D * 2;       // one K or V chunk
  static constexpr uint32_t kSmem = kAttWarps * 4 * kTile;    // per warp: two K and two V buffers
  static_assert(kAttWarps * 16 * kRow * 4 <= kSmem, "warp merge area fits in the staging buffers");
  static_assert(kMaxSplits * 16 * 4 * 2 <= kSmem, "split maxima and sums fit in the staging buffers");
  static_assert((kAttWarps * 16 * kRow + 16 * kPart) * 4 <= kSmem, "the warp rows and the CTA partial fit");
};

// ---------------------------------------------------------------- K3: split-KV sparse attention + merge
// grid (batch*h_kv, nsplit), kAttWarps warps.  CTA (bg, sp) covers the
// entries [sp*bps, sp*bps + bps) of the block list of (sequence b, group g);
// each entry is two 32-key chunks, and warp w takes chunks w, w + kAttWarps, ...
// Per chunk the warp stages K and V (cp.async, 16 B pieces; the 16-byte
// pieces of a key row are XOR-swizzled by the row index so ldmatrix is free
// of bank conflicts), then
//   S[16 heads, 32 keys] = Q . K^T     (mma.sync m16n8k16, K via ldmatrix)
//   P = 2^(S*scale*log2e - m_ref)      (m_ref per head, raised only when a
//                                        score passes it by more than 2^8;
//                                        then O and l are rescaled once)
//   O[16, D] += P . V                  (P re-used from the S fragments,
//                                        V via ldmatrix.trans)
// Each warp holds two K and two V buffers: chunk i + 2's K is issued as soon
// as chunk i's S is done and its V as soon as chunk i's PV product is done,
// so every warp keeps two chunks' copies in flight.  The warps'
// (m_ref, l, O) are merged in shared memory into one partial per CTA.  With
// CLUSTER the nsplit CTAs of (b, g) form one thread-block cluster: each keeps
// its partial in its shared memory and, after a cluster barrier, rank 0 reads
// them all through distributed shared memory, merges them and writes the
// output (a second barrier keeps the partials alive until it is done).
// Otherwise each CTA writes its partial to the workspace and the last CTA of
// (b, g) to finish (a completion counter) merges them.  The merging CTA of the
// last group of b to finish advances seq_len[b].
// Keys past t (and chunks of invalid or not yet visible blocks) are never
// read: their staging rows are zero-filled and their scores are -inf.
// PHASED: the CTA's work comes in two phases.  Phase 0, before the wait for
// the selection, covers the CTA's share of the blocks every list holds (the
// init blocks and the local run, without the query's own block b_t, whose
// row t the append kernel of this step writes); phase 1, after it, the CTA's
// share of the top-k blocks and b_t.  Without PHASED the CTA covers entries
// [sp*bps, sp*bps + bps) of the list, after the wait.
template <int D, bool CLUSTER, bool PHASED>
__global__ void __launch_bounds__(32 * kAttWarps, 1) attend_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ kc, const __nv_bfloat16* __restrict__ vc,
    const int32_t* __restrict__ idx, int32_t* seq_len, int capacity, int h_q, int h_kv, int n_sel, int bps,
    float scale, float* __restrict__ part, __nv_bfloat16* __restrict__ out, unsigned* __restrict__ cnt, int n_init,
    int n_local, int top_k) {
  using C = AttCfg<D>;
  extern __shared__ __align__(128) uint8_t att_smem[];
  __shared__ float s_wgt[kAttWarps][16], s_M[16], s_L[16];
  __shared__ int s_last;
  const int bg = blockIdx.x, sp = blockIdx.y, nsplit = gridDim.y, nbg = gridDim.x;
  const int b = bg / h_kv, g = bg % h_kv;
  const int G = h_q / h_kv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gid = lane >> 2, tig = lane & 3;
  // the new token's position; keys 0..t are visible
  const int t = seq_len[b];
  const int32_t* list = idx + static_cast<int64_t>(bg) * n_sel + static_cast<int64_t>(sp) * bps;
  const int nb = max(0, min(bps, n_sel - sp * bps));
  // PHASED partition (from t alone): S = init blocks below b_t, then the local
  // run below b_t; P = the list's top-k entries, then b_t.  This CTA takes
  // the sp-th share of each.
  const int b_t = t >> 6;
  const int i_hi = min(n_init, b_t + 1);
  const int l_start = max(i_hi, max(0, b_t - n_local + 1));
  const int s_init = min(i_hi, b_t);
  const int s_all = s_init + max(0, b_t - l_start);
  const int ntop = min(top_k, max(0, l_start - i_hi));
  const int p_all = ntop + 1;
  const int s_lo = s_all * sp / nsplit, s_cnt = s_all * (sp + 1) / nsplit - s_lo;
  const int p_lo = p_all * sp / nsplit, p_cnt = p_all * (sp + 1) / nsplit - p_lo;
  const int32_t* list_all = idx + static_cast<int64_t>(bg) * n_sel;
  const int64_t kstride = static_cast<int64_t>(h_kv) * D;    // elements from one key row to the next
  const int64_t row0 = (static_cast<int64_t>(b) * capacity * h_kv + g) * D;
  // the warp's buffers: K of chunks i and i + 1, then V of chunks i and i + 1
  const uint32_t sbuf = smem_u32(att_smem) + warp * 4 * C::kTile;

  // Q of the group's 16 heads (rows >= G are zero) as m16n8k16 A fragments
  uint32_t qa[D / 16][4];
  {
    const __nv_bfloat16* qh = q + (static_cast<int64_t>(b) * h_q + g * G) * D;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const int d0 = 16 * kk + 2 * tig;
      qa[kk][0] = (gid < G) ? *reinterpret_cast<const uint32_t*>(qh + gid * D + d0) : 0u;
      qa[kk][1] = (gid + 8 < G) ? *reinterpret_cast<const uint32_t*>(qh + (gid + 8) * D + d0) : 0u;
      qa[kk][2] = (gid < G) ? *reinterpret_cast<const uint32_t*>(qh + gid * D + d0 + 8) : 0u;
      qa[kk][3] = (gid + 8 < G) ? *reinterpret_cast<const uint32_t*>(qh + (gid + 8) * D + d0 + 8) : 0u;
    }
  }
  // the block lists come from the selection (PHASED: only phase 1 reads them)
  if (!PHASED) griddep_wait();
  if (t < 0 || t >= capacity) return;          // recorded by the append kernel

  // chunks of the warp in the current phase, and the first key of its i-th
  // chunk (-1 when it has no visible key)
  int phase = 0, nmine = 0;
  auto phase_chunks = [&](int ph) -> int {
    const int ne = !PHASED ? nb : (ph == 0 ? s_cnt : p_cnt);
    return (2 * ne > warp) ? (2 * ne - 1 - warp) / kAttWarps + 1 : 0;
  };
  auto chunk_key0 = [&](int i) -> int {
    if (i >= nmine) return -1;
    const int ch = warp + kAttWarps * i;
    int blk;
    if (!PHASED) {
      blk = list[ch >> 1];
    } else if (phase == 0) {
      const int e = s_lo + (ch >> 1);
      blk = (e < s_init) ? e : l_start + (e - s_init);
    } else {
      const int e = p_lo + (ch >> 1);
      blk = (e < ntop) ? list_all[i_hi + e] : b_t;
    }
    const int k0 = 64 * blk + kChunkKeys * (ch & 1);
    return (blk >= 0 && blk <= b_t && k0 <= t) ? k0 : -1;
  };
  auto stage = [&](uint32_t dst, const __nv_bfloat16* cache, int k0) {
    if (k0 >= 0) {
#pragma unroll
      for (int j = 0; j < kChunkKeys * C::CH / 32; ++j) {
        const int pc = lane + 32 * j;
        const int r = pc / C::CH, c = pc % C::CH;
        const bool ok = k0 + r <= t;
        const __nv_bfloat16* src = cache + row0 + static_cast<int64_t>(ok ? k0 + r : k0) * kstride + c * 8;
        cp_async16(dst + r * (D * 2) + ((c ^ (r & 7)) << 4), src, ok);
      }
    }
    cp_async_commit();
  };

  float o[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;   // heads gid, gid + 8: reference max, row sum
  const float cs = scale * kLog2e;

  // copies in flight per warp: two chunks ahead.  Commit order: K0 V0 K1 V1,
  // then per chunk i: K(i+2) after its S product, V(i+2) after its P.V
  // product, so K(i) and V(i) each have exactly three younger groups.  Each
  // phase starts and drains its own stream of copies.
  for (phase = 0; phase < (PHASED ? 2 : 1); ++phase) {
  if (PHASED && phase == 1) griddep_wait();     // the lists of this step are selected
  nmine = phase_chunks(phase);
  int k0 = chunk_key0(0);
  int k1 = chunk_key0(1);
  stage(sbuf, kc, k0);
  stage(sbuf + 2 * C::kTile, vc, k0);
  stage(sbuf + C::kTile, kc, k1);
  stage(sbuf + 3 * C::kTile, vc, k1);
  for (int i = 0; i < nmine; ++i) {
    const uint32_t sK = sbuf + (i & 1) * C::kTile;
    const uint32_t sV = sK + 2 * C::kTile;
    const int k0n = chunk_key0(i + 2);
    cp_async_wait_n<3>();                    // K of chunk i
    __syncwarp();
    float s[4][4];
    if (k0 >= 0) {
#pragma unroll
      for (int j = 0; j < 4; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
#pragma unroll
      for (int p = 0; p < D / 32; ++p) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int r = 8 * j + (lane & 7), c = 4 * p + (lane >> 3);
          uint32_t kb[4];
          ldsm_x4(kb, sK + r * (D * 2) + ((c ^ (r & 7)) << 4));
          mma16816(s[j], qa[2 * p], kb[0], kb[1]);
          mma16816(s[j], qa[2 * p + 1], kb[2], kb[3]);
        }
      }
    }
    __syncwarp();                            // every lane is done with this K buffer
    stage(sK, kc, k0n);
    if (k0 >= 0) {
      float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const bool ok = k0 + 8 * j + 2 * tig + e <= t;
          s[j][e] = ok ? s[j][e] * cs : -INFINITY;
          s[j][2 + e] = ok ? s[j][2 + e] * cs : -INFINITY;
          mx0 = fmaxf(mx0, s[j][e]);
          mx1 = fmaxf(mx1, s[j][2 + e]);
        }
      }
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
      // key k0 is visible, so both maxima are finite; the reference maxima
      // move only past the margin (the first chunk always sets them)
      const bool up0 = mx0 > m0 + kRescaleLog2, up1 = mx1 > m1 + kRescaleLog2;
      if (__any_sync(0xffffffffu, up0 || up1)) {
        const float n0 = up0 ? mx0 : m0, n1 = up1 ? mx1 : m1;
        const float a0 = (m0 == -INFINITY) ? 0.f : ex2(m0 - n0);
        const float a1 = (m1 == -INFINITY) ? 0.f : ex2(m1 - n1);
        m0 = n0;
        m1 = n1;
        l0 *= a0;
        l1 *= a1;
#pragma unroll
        for (int n = 0; n < D / 8; ++n) {
          o[n][0] *= a0;
          o[n][1] *= a0;
          o[n][2] *= a1;
          o[n][3] *= a1;
        }
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          s[j][e] = ex2(s[j][e] - m0);
          s[j][2 + e] = ex2(s[j][2 + e] - m1);
          l0 += s[j][e];
          l1 += s[j][2 + e];
        }
      }
    }
    cp_async_wait_n<3>();                    // V of chunk i
    __syncwarp();
    if (k0 >= 0) {
#pragma unroll
      for (int s2 = 0; s2 < 2; ++s2) {
        const uint32_t pa[4] = {pack_bf16(s[2 * s2][0], s[2 * s2][1]), pack_bf16(s[2 * s2][2], s[2 * s2][3]),
                                pack_bf16(s[2 * s2 + 1][0], s[2 * s2 + 1][1]),
                                pack_bf16(s[2 * s2 + 1][2], s[2 * s2 + 1][3])};
#pragma unroll
        for (int n = 0; n < D / 8; n += 2) {
          const int r = 16 * s2 + (lane & 7) + ((lane >> 3) & 1) * 8, c = n + (lane >> 4);
          uint32_t vb[4];
          ldsm_x4_t(vb, sV + r * (D * 2) + ((c ^ (r & 7)) << 4));
          mma16816(o[n], pa, vb[0], vb[1]);
          mma16816(o[n + 1], pa, vb[2], vb[3]);
        }
      }
    }
    __syncwarp();                            // every lane is done with this V buffer
    stage(sV, vc, k0n);
    k0 = k1;
    k1 = k0n;
  }
  cp_async_wait0();
  __syncwarp();
  }                                            // phases
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);

  // ---- merge the warps in the (now idle) staging buffers: [warp][16][kRow]
  __syncthreads();
  float* mw = reinterpret_cast<float*>(att_smem);
  {
    float* r0 = mw + (warp * 16 + gid) * C::kRow;
    float* r1 = mw + (warp * 16 + gid + 8) * C::kRow;
#pragma unroll
    for (int n = 0; n < D / 8; ++n) {
      *reinterpret_cast<float2*>(r0 + 8 * n + 2 * tig) = make_float2(o[n][0], o[n][1]);
      *reinterpret_cast<float2*>(r1 + 8 * n + 2 * tig) = make_float2(o[n][2], o[n][3]);
    }
    if (tig == 0) {
      r0[D] = m0;
      r0[D + 1] = l0;
      r1[D] = m1;
      r1[D + 1] = l1;
    }
  }
  __syncthreads();
  if (threadIdx.x < 16) {
    const int h = threadIdx.x;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kAttWarps; ++w) M = fmaxf(M, mw[(w * 16 + h) * C::kRow + D]);
    float L = 0.f;
#pragma unroll
    for (int w = 0; w < kAttWarps; ++w) {
      const float mwh = mw[(w * 16 + h) * C::kRow + D];
      const float wg = (mwh == -INFINITY) ? 0.f : ex2(mwh - M);
      s_wgt[w][h] = wg;
      L += wg * mw[(w * 16 + h) * C::kRow + D + 1];
    }
    s_M[h] = M;
    s_L[h] = L;
  }
  __syncthreads();
  if constexpr (CLUSTER) {
    float* mine = reinterpret_cast<float*>(att_smem) + kAttWarps * 16 * C::kRow;   // [G][kPart], after the warp rows
    for (int e = threadIdx.x; e < G * D; e += 32 * kAttWarps) {
      const int h = e / D, d = e % D;
      float acc = 0.f;
#pragma unroll
      for (int w = 0; w < kAttWarps; ++w) acc += s_wgt[w][h] * mw[(w * 16 + h) * C::kRow + d];
      mine[h * C::kPart + d] = acc;
    }
    if (threadIdx.x < G) {
      mine[threadIdx.x * C::kPart + D] = s_M[threadIdx.x];
      mine[threadIdx.x * C::kPart + D + 1] = s_L[threadIdx.x];
    }
    cluster_sync_all();
    if (cluster_rank() == 0) {
      const uint32_t mine_s = smem_u32(mine);
      __shared__ float s_cw[8][16];            // split weights
      if (threadIdx.x < G) {
        const int h = threadIdx.x;
        float ms[8], ls[8];
        float M = -INFINITY;
#pragma unroll
        for (int s2 = 0; s2 < 8; ++s2) {
          if (s2 < nsplit) {
            const uint32_t a = dsmem_addr(mine_s + (h * C::kPart + D) * 4, s2);
            ms[s2] = ld_dsmem(a);
            ls[s2] = ld_dsmem(a + 4);
            M = fmaxf(M, ms[s2]);
          }
        }
        float L = 0.f;
#pragma unroll
        for (int s2 = 0; s2 < 8; ++s2)
          if (s2 < nsplit && ms[s2] != -INFINITY) L += ex2(ms[s2] - M) * ls[s2];
        const float inv = (L > 0.f) ? 1.f / L : 0.f;
#pragma unroll
        for (int s2 = 0; s2 < 8; ++s2)
          if (s2 < nsplit) s_cw[s2][h] = (ms[s2] == -INFINITY) ? 0.f : ex2(ms[s2] - M) * inv;
      }
      __syncthreads();
      constexpr int kIt = (16 * (D / 4) + 32 * kAttWarps - 1) / (32 * kAttWarps);
      const int nitems = G * (D / 4);
      // every item's loads first, so they are all in flight together
      float4 v[kIt][8];
#pragma unroll
      for (int k = 0; k < kIt; ++k) {
        const int it = min(threadIdx.x + 32 * kAttWarps * k, nitems - 1);
        const int h = it / (D / 4), q4 = it % (D / 4);
        const uint32_t local = mine_s + (h * C::kPart + 4 * q4) * 4;
#pragma unroll
        for (int s2 = 0; s2 < 8; ++s2)
          if (s2 < nsplit) v[k][s2] = ld_dsmem4(dsmem_addr(local, s2));
      }
#pragma unroll
      for (int k = 0; k < kIt; ++k) {
        const int it = threadIdx.x + 32 * kAttWarps * k;
        if (it < nitems) {
          const int h = it / (D / 4), q4 = it % (D / 4);
          float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
          for (int s2 = 0; s2 < 8; ++s2) {
            if (s2 < nsplit) {
              const float wg = s_cw[s2][h];
              acc.x = fmaf(wg, v[k][s2].x, acc.x);
              acc.y = fmaf(wg, v[k][s2].y, acc.y);
              acc.z = fmaf(wg, v[k][s2].z, acc.z);
              acc.w = fmaf(wg, v[k][s2].w, acc.w);
            }
          }
          uint2 w2;
          w2.x = pack_bf16(acc.x, acc.y);
          w2.y = pack_bf16(acc.z, acc.w);
          *reinterpret_cast<uint2*>(out + (static_cast<int64_t>(b) * h_q + g * G + h) * D + 4 * q4) = w2;
        }
      }
      // every CTA of every group of b has read seq_len[b] once all groups got here
      if (threadIdx.x == 0 && atomicAdd(&cnt[2 * nbg + b], 1u) == static_cast<unsigned>(h_kv) - 1)
        seq_len[b] = t + 1;
    }
    cluster_sync_all();                        // the partials stay readable until rank 0 is done
    return;
  }
  float* pb = part + static_cast<int64_t>(bg) * nsplit * G * C::kPart;
  {
    float* dst = pb + static_cast<int64_t>(sp) * G * C::kPart;
    for (int e = threadIdx.x; e < G * D; e += 32 * kAttWarps) {
      const int h = e / D, d = e % D;
      float acc = 0.f;
#pragma unroll
      for (int w = 0; w < kAttWarps; ++w) acc += s_wgt[w][h] * mw[(w * 16 + h) * C::kRow + d];
      dst[h * C::kPart + d] = acc;
    }
    if (threadIdx.x < G) {
      dst[threadIdx.x * C::kPart + D] = s_M[threadIdx.x];
      dst[threadIdx.x * C::kPart + D + 1] = s_L[threadIdx.x];
    }
  }

  // ---- the last CTA of (b, g) to finish merges the splits
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = (atomicAdd(&cnt[nbg + bg], 1u) == nsplit - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // split maxima and sums, all loaded at once
  float* wsp = reinterpret_cast<float*>(att_smem);          // [nsplit][16] maxima, then weights
  float* lsp = wsp + kMaxSplits * 16;                        // [nsplit][16] row sums
  for (int e = threadIdx.x; e < nsplit * 16; e += 32 * kAttWarps) {
    const int s2 = e >> 4, h = e & 15;
    const float2 ml = (h < G) ? __ldcg(reinterpret_cast<const float2*>(pb + (static_cast<int64_t>(s2) * G + h) * C::kPart + D))
                              : make_float2(-INFINITY, 0.f);
    wsp[e] = ml.x;
    lsp[e] = ml.y;
  }
  __syncthreads();
  if (threadIdx.x < 16) {
    const int h = threadIdx.x;
    float M = -INFINITY;
    for (int s2 = 0; s2 < nsplit; ++s2) M = fmaxf(M, wsp[s2 * 16 + h]);
    float L = 0.f;
    for (int s2 = 0; s2 < nsplit; ++s2) {
      const float ms = wsp[s2 * 16 + h];
      if (ms != -INFINITY) L += ex2(ms - M) * lsp[s2 * 16 + h];
    }
    s_M[h] = M;
    s_L[h] = (L > 0.f) ? 1.f / L : 0.f;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < nsplit * 16; e += 32 * kAttWarps) {
    const int h = e & 15;
    const float ms = wsp[e];
    wsp[e] = (ms == -INFINITY) ? 0.f : ex2(ms - s_M[h]) * s_L[h];
  }
  __syncthreads();
  // out[h, 4 q .. 4 q + 3] = sum over splits of weight * O: thread items
  // it = tid + 32 kAttWarps k (k < kIt) cover the G * D / 4 (head, quad)
  // pairs; four splits of every item are in flight at once
  {
    constexpr int kIt = (16 * (D / 4) + 32 * kAttWarps - 1) / (32 * kAttWarps), kU = 4;
    const int nitems = G * (D / 4);
    float4 acc[kIt];
#pragma unroll
    for (int k = 0; k < kIt; ++k) acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s0 = 0; s0 < nsplit; s0 += kU) {
      float4 v[kIt][kU];
#pragma unroll
      for (int k = 0; k < kIt; ++k) {
        const int it = threadIdx.x + 32 * kAttWarps * k;
        const int h = it / (D / 4), q4 = it % (D / 4);
#pragma unroll
        for (int u = 0; u < kU; ++u) {
          const bool ok = it < nitems && s0 + u < nsplit;
          v[k][u] = ok ? __ldcg(reinterpret_cast<const float4*>(pb + (static_cast<int64_t>(s0 + u) * G + h) * C::kPart) + q4)
                       : make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
#pragma unroll
      for (int k = 0; k < kIt; ++k) {
        const int it = threadIdx.x + 32 * kAttWarps * k;
        const int h = min(it / (D / 4), 15);
#pragma unroll
        for (int u = 0; u < kU; ++u) {
          const float wg = (s0 + u < nsplit) ? wsp[(s0 + u) * 16 + h] : 0.f;
          acc[k].x = fmaf(wg, v[k][u].x, acc[k].x);
          acc[k].y = fmaf(wg, v[k][u].y, acc[k].y);
          acc[k].z = fmaf(wg, v[k][u].z, acc[k].z);
          acc[k].w = fmaf(wg, v[k][u].w, acc[k].w);
        }
      }
    }
#pragma unroll
    for (int k = 0; k < kIt; ++k) {
      const int it = threadIdx.x + 32 * kAttWarps * k;
      if (it < nitems) {
        const int h = it / (D / 4), q4 = it % (D / 4);
        uint2 w2;
        w2.x = pack_bf16(acc[k].x, acc[k].y);
        w2.y = pack_bf16(acc[k].z, acc[k].w);
        *reinterpret_cast<uint2*>(out + (static_cast<int64_t>(b) * h_q + g * G + h) * D + 4 * q4) = w2;
      }
    }
  }
  // every CTA of every group of b has read seq_len[b] once all groups got here
  if (threadIdx.x == 0 && atomicAdd(&cnt[2 * nbg + b], 1u) == static_cast<unsigned>(h_kv) - 1) seq_len[b] = t + 1;
}

// ---------------------------------------------------------------- pooled caches of a prefix
// grid (ceil(capacity/512), batch, h_kv): the compress algorithm on the
// decode cache layout, for the seq_len[b] tokens already in the cache.
template <int D>
__global__ void __launch_bounds__(256) build_caches_kernel(const __nv_bfloat16* __restrict__ kc,
                                                           const int32_t* __restrict__ seq_len, int capacity, int h_kv,
                                                           __nv_bfloat16* __restrict__ kc1, int cap_c1,
                                                           __nv_bfloat16* __restrict__ kc2, int cap_c2) {
  constexpr int SL = D / 8;
  constexpr int NCH = 512 / 16 + 8;
  __shared__ double csum[NCH][D];
  const int b = blockIdx.y, g = blockIdx.z;
  const int len = min(seq_len[b], capacity);
  const int t0 = blockIdx.x * 512;
  if (t0 >= len) return;
  const int64_t seq0 = static_cast<int64_t>(b) * capacity;
  for (int item = threadIdx.x; item < NCH * SL; item += 256) {
    const int ch = item / SL, sl = item % SL;
    double acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.0;
    for (int r = 0; r < 16; ++r) {
      const int t = t0 + ch * 16 + r;
      if (t < len) {
        const uint4 raw = *reinterpret_cast<const uint4*>(kc + ((seq0 + t) * h_kv + g) * D + sl * 8);
        const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 f2 = __bfloat1622float2(p2[i]);
          acc[2 * i] += static_cast<double>(f2.x);
          acc[2 * i + 1] += static_cast<double>(f2.y);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) csum[ch][sl * 8 + i] = acc[i];
  }
  __syncthreads();
  const int n_c1 = window_count_dev(len, 32, 16), n_c2 = window_count_dev(len, 128, 64);
  for (int item = threadIdx.x; item < 40 * SL; item += 256) {
    const bool is2 = item >= 32 * SL;
    const int w = is2 ? (item - 32 * SL) / SL : item / SL;
    const int sl = item % SL;
    const int j = is2 ? t0 / 64 + w : t0 / 16 + w;
    if (j >= (is2 ? n_c2 : n_c1) || j >= (is2 ? cap_c2 : cap_c1)) continue;
    uint16_t o[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      double a = 0.0;
      if (is2) {
        for (int q4 = 0; q4 < 8; ++q4) a += csum[4 * w + q4][sl * 8 + i];
        o[i] = f64_to_bf16_rne(a * (1.0 / 128.0));
      } else {
        a = csum[w][sl * 8 + i] + csum[w + 1][sl * 8 + i];
        o[i] = f64_to_bf16_rne(a * (1.0 / 32.0));
      }
    }
    uint4 v;
    v.x = o[0] | (static_cast<uint32_t>(o[1]) << 16);
    v.y = o[2] | (static_cast<uint32_t>(o[3]) << 16);
    v.z = o[4] | (static_cast<uint32_t>(o[5]) << 16);
    v.w = o[6] | (static_cast<uint32_t>(o[7]) << 16);
    __nv_bfloat16* dst = (is2 ? kc2 : kc1) + ((static_cast<int64_t>(b) * h_kv + g) * (is2 ? cap_c2 : cap_c1) + j) * D;
    reinterpret_cast<uint4*>(dst)[sl] = v;
  }
}

}  // namespace dec

// ---------------------------------------------------------------- host side
struct DecodePlan {
  int cap_c1, cap_c2, nblk_cap, cand_cap, nsplit2, np_cap, nsplit, bps, n_sel, sms, nbg;
  size_t off_part2, off_bscore, off_idx, off_part, off_cnt, bytes;
};

static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Limits: the selecting CTA's candidate keys fit its shared memory (capacity
// up to about 1.44 M tokens), and the piece list packs (sequence, group) and
// piece indices into 16 bits each.
static bool decode_plan_supported(const DecodePlan& p) {
  return static_cast<size_t>(p.cand_cap) * 4 <= 88 * 1024 && p.nbg <= 65535 && p.np_cap <= 65535;
}

DecodePlan decode_plan(int batch, int capacity, int h_q, int h_kv, int d, int n_sel, int sms) {
  DecodePlan p{};
  p.n_sel = n_sel;
  p.cap_c1 = static_cast<int>(infllm2_window_count(capacity, 32, 16));
  p.cap_c2 = static_cast<int>(infllm2_window_count(capacity, 128, 64));
  p.nblk_cap = (capacity + 63) / 64;
  p.cand_cap = (p.nblk_cap + 31) & ~31;
  p.nsplit2 = std::max(1, (p.cap_c2 + dec::kLseWin - 1) / dec::kLseWin);
  p.np_cap = std::max(1, (p.nblk_cap + dec::kPieceBlk - 1) / dec::kPieceBlk);
  p.sms = std::max(1, sms);
  const int bg = batch * h_kv;
  p.nbg = bg;
  // attention splits: one wave of one CTA per SM (its shared memory holds
  // two chunks ahead per warp); 16 x 131072 decode: 4 splits of 24 blocks
  const int per_bg = std::min(dec::kMaxSplits, std::max(1, sms / std::max(1, bg)));
  p.bps = std::max(1, (n_sel + per_bg - 1) / per_bg);
  p.nsplit = std::max(1, (n_sel + p.bps - 1) / p.bps);
  const int G = h_q / h_kv;
  size_t off = 0;
  p.off_part2 = off; off = align256(off + static_cast<size_t>(bg) * p.nsplit2 * 16 * sizeof(float2));
  p.off_bscore = off; off = align256(off + static_cast<size_t>(bg) * p.nblk_cap * sizeof(float));
  p.off_idx = off; off = align256(off + static_cast<size_t>(bg) * n_sel * sizeof(int32_t));
  p.off_part = off; off = align256(off + static_cast<size_t>(bg) * p.nsplit * G * (d + 4) * sizeof(float));
  p.off_cnt = off; off = align256(off + static_cast<size_t>(2 * bg + batch) * sizeof(unsigned));
  p.bytes = off;
  return p;
}

// 1: the selection runs as its own launch and the attention streams the init
// and local blocks while it runs (measured slower: 53.9 vs 49.4 us per step at
// 16 x 131072); 0: the CTA that completes a (sequence, group)'s last piece in
// the score kernel selects.
#ifndef INFLLM2_DEC_SPLIT_SELECT
#define INFLLM2_DEC_SPLIT_SELECT 0
#endif
constexpr bool kSplitSelect = INFLLM2_DEC_SPLIT_SELECT != 0;

template <int D>
static cudaError_t decode_step_t(const infllm2_decode_state* s, const void* q, const void* k_new, const void* v_new,
                                 void* out, void* ws, const DecodePlan& P, int n_init, int n_local, int top_k,
                                 float scale, cudaStream_t st) {
  using bf = __nv_bfloat16;
  const int bg = s->batch * s->h_kv;
  uint8_t* w = static_cast<uint8_t*>(ws);
  float2* part2 = reinterpret_cast<float2*>(w + P.off_part2);
  float* bscore = reinterpret_cast<float*>(w + P.off_bscore);
  int32_t* idx = reinterpret_cast<int32_t*>(w + P.off_idx);
  float* part = reinterpret_cast<float*>(w + P.off_part);
  unsigned* cnt = reinterpret_cast<unsigned*>(w + P.off_cnt);
  dec::lse_append_kernel<D><<<dim3(bg, P.nsplit2), 128, 0, st>>>(
      static_cast<const bf*>(q), static_cast<const bf*>(k_new), static_cast<const bf*>(v_new),
      static_cast<bf*>(s->k_cache), static_cast<bf*>(s->v_cache), static_cast<bf*>(s->k_c1), static_cast<bf*>(s->k_c2),
      s->seq_len, s->capacity, s->h_q, s->h_kv, P.cap_c1, P.cap_c2, scale, part2, cnt);
  CUtensorMap mK1;
  {
    const uint64_t rows = static_cast<uint64_t>(std::max(1, P.cap_c1));
    const uint64_t dims[3] = {(uint64_t)D, rows, (uint64_t)bg};
    const uint64_t strides[2] = {(uint64_t)D * 2, rows * D * 2};
    const uint32_t box[3] = {64, (uint32_t)dec::kPieceRows, 1};
    if (!make_tmap(&mK1, s->k_c1, 3, dims, strides, box)) return cudaErrorInvalidValue;
  }
  const size_t k2_smem = std::max<size_t>(dec::ScoreCfg<D>::kSmem,
                                          static_cast<size_t>(P.cand_cap) * 4 + 16 + dec::kSelBins * 4);
  cudaError_t e = cudaFuncSetAttribute(dec::score_select_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(k2_smem));
  if (e != cudaSuccess) return e;
  // one wave of streaming CTAs, each with at most kMaxRange pieces
  int occ = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, dec::score_select_kernel<D>, dec::kSelThreads, k2_smem);
  if (e != cudaSuccess) return e;
  const int64_t p_cap = static_cast<int64_t>(bg) * P.np_cap;
  int64_t grid2 = std::min<int64_t>(p_cap, static_cast<int64_t>(std::max(1, occ)) * P.sms);
  // flattened ranges hold at most ceil(total / grid) pieces; group-aligned
  // shares (the kernel's choice when grid >= groups) at most
  // total / (grid - groups) + 1
  grid2 = std::max<int64_t>(grid2, (p_cap + dec::kMaxRange - 1) / dec::kMaxRange);
  if (grid2 >= bg) grid2 = std::max<int64_t>(grid2, bg + (p_cap + dec::kMaxRange - 2) / (dec::kMaxRange - 1));
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(static_cast<unsigned>(grid2));
    cfg.blockDim = dim3(dec::kSelThreads);
    cfg.dynamicSmemBytes = k2_smem;
    cfg.stream = st;
    cfg.attrs = pdl;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, dec::score_select_kernel<D>, mK1, static_cast<const bf*>(q),
                           static_cast<const bf*>(s->k_c1), static_cast<const int32_t*>(s->seq_len),
                           static_cast<const float2*>(part2), P.nsplit2, s->batch, s->capacity, s->h_q, s->h_kv,
                           P.cap_c1, P.nblk_cap, P.cand_cap, scale, n_init, n_local, top_k, P.n_sel, bscore, idx, cnt,
                           kSplitSelect ? 0 : 1);
    if (e != cudaSuccess) return e;
  }
  if (kSplitSelect) {
    // the selection as its own launch, between the scores and the attention
    const size_t sel_smem = ((static_cast<size_t>(P.cand_cap) * 4 + 15) & ~size_t(15)) + dec::kSelBins * 4;
    e = cudaFuncSetAttribute(dec::select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(sel_smem));
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(bg);
    cfg.blockDim = dim3(dec::kSelThreads);
    cfg.dynamicSmemBytes = sel_smem;
    cfg.stream = st;
    cfg.attrs = pdl;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, dec::select_kernel, static_cast<const float*>(bscore),
                           static_cast<const int32_t*>(s->seq_len), s->capacity, s->h_kv, n_init, n_local, top_k,
                           P.n_sel, P.nblk_cap, P.cand_cap, idx);
    if (e != cudaSuccess) return e;
  }
  if (P.nsplit <= 8) {
    // the splits of (b, g) as one cluster: the merge goes through distributed shared memory
    e = cudaFuncSetAttribute(dec::attend_kernel<D, true, kSplitSelect>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(dec::AttCfg<D>::kSmem));
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(bg, P.nsplit);
    cfg.blockDim = dim3(32 * dec::kAttWarps);
    cfg.dynamicSmemBytes = dec::AttCfg<D>::kSmem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = P.nsplit;
    attr[0].val.clusterDim.z = 1;
    attr[1] = pdl[0];
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    e = cudaLaunchKernelEx(&cfg, dec::attend_kernel<D, true, kSplitSelect>, static_cast<const bf*>(q),
                           static_cast<const bf*>(s->k_cache), static_cast<const bf*>(s->v_cache),
                           static_cast<const int32_t*>(idx), s->seq_len, s->capacity, s->h_q, s->h_kv, P.n_sel, P.bps,
                           scale, part, static_cast<bf*>(out), cnt, n_init, n_local, top_k);
    if (e != cudaSuccess) return e;
  } else {
    e = cudaFuncSetAttribute(dec::attend_kernel<D, false, kSplitSelect>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(dec::AttCfg<D>::kSmem));
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(bg, P.nsplit);
    cfg.blockDim = dim3(32 * dec::kAttWarps);
    cfg.dynamicSmemBytes = dec::AttCfg<D>::kSmem;
    cfg.stream = st;
    cfg.attrs = pdl;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, dec::attend_kernel<D, false, kSplitSelect>, static_cast<const bf*>(q),
                           static_cast<const bf*>(s->k_cache), static_cast<const bf*>(s->v_cache),
                           static_cast<const int32_t*>(idx), s->seq_len, s->capacity, s->h_q, s->h_kv, P.n_sel, P.bps,
                           scale, part, static_cast<bf*>(out), cnt, n_init, n_local, top_k);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

cudaError_t launch_decode_step(const infllm2_decode_state* s, const void* q, const void* k_new, const void* v_new,
                               void* out, void* ws, const DecodePlan& P, int n_init, int n_local, int top_k,
                               float scale, cudaStream_t st) {
  if (s->d == 128) return decode_step_t<128>(s, q, k_new, v_new, out, ws, P, n_init, n_local, top_k, scale, st);
  return decode_step_t<64>(s, q, k_new, v_new, out, ws, P, n_init, n_local, top_k, scale, st);
}

cudaError_t launch_decode_build_caches(const infllm2_decode_state* s, const DecodePlan& P, cudaStream_t st) {
  dim3 grid((s->capacity + 511) / 512, s->batch, s->h_kv);
  using bf = __nv_bfloat16;
  if (s->d == 128)
    dec::build_caches_kernel<128><<<grid, 256, 0, st>>>(static_cast<const bf*>(s->k_cache), s->seq_len, s->capacity,
                                                        s->h_kv, static_cast<bf*>(s->k_c1), P.cap_c1,
                                                        static_cast<bf*>(s->k_c2), P.cap_c2);
  else
    dec::build_caches_kernel<64><<<grid, 256, 0, st>>>(static_cast<const bf*>(s->k_cache), s->seq_len, s->capacity,
                                                       s->h_kv, static_cast<bf*>(s->k_c1), P.cap_c1,
                                                       static_cast<bf*>(s->k_c2), P.cap_c2);
  return cudaGetLastError();
}

}  // namespace infllm2
