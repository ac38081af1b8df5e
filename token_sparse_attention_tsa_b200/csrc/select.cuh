// select.cuh -- Dynamic Token Coverage budget and per-head top-k selection.
//
// Source: gist.science summary page "Token Sparse Attention: Efficient
// Long-Context Inference with Interleaved Token Selection", section 2,
// "Cobertura Dinamica de Tokens": tokens are ordered by ascending importance
// and the low-importance tail is pruned as long as its share of the total
// importance stays within the coverage threshold tau; the resulting budget is
// shared (global), and each head keeps its own top-k tokens by its own scores.
//
// Exact arithmetic (so every device and the CPU agree bit for bit):
//   mass  q_j = ceil(score_j * 2^40) as an integer (score_j >= 0 fp32; the
//         product is exact in fp64 and ceil is exact),
//   T     = floor(tau * (double)sum_j q_j) (one fp64 multiply),
//   p_h   = the largest count of least-important tokens whose masses sum to
//           <= T; k_head = max(L - p_h, r) with r the forced recent tokens;
//   k_seq[b] = max over the heads of b, or the ceiling of their mean.
// The page calls the budget global without saying how heads combine: the
// maximum is the default reading; the mean and a per-head budget (every
// head keeps its own k_head) are the two other plain readings, selectable.
// Ascending order of q_j is the ascending order of the fp32 bit patterns, so
// neither kernel sorts: both run a most-significant-digit radix descent over
// the bit patterns, then (select) compact the chosen indices in index order,
// which yields S_h ascending.  Ties at the threshold go to the smaller index.
// The descent runs on r = key - min_key with 11-bit digits taken from the top
// of the head's own key range (at most three levels), after one pass that
// finds the range: the scores of a head span a few binary orders of
// magnitude, so digits of the raw bit pattern's top bits would put nearly
// every key of a warp into the same few bins and serialise the shared-memory
// histogram atomics.
#pragma once

#include <cstdint>

#include "sm100.cuh"

namespace tsa {

constexpr int BS_THREADS = 1024;
constexpr int BS_WARPS = BS_THREADS / 32;

// Order key of a score: its bit pattern for finite scores >= 0 (-0 maps to
// 0); NaN, infinities and negative values map to 0 and are reported.
__device__ __forceinline__ uint32_t score_key(float s, bool& bad) {
  const uint32_t u = __float_as_uint(s);
  const bool ok = (u & 0x80000000u) ? ((u & 0x7fffffffu) == 0) : (u < 0x7f800000u);
  bad |= !ok;
  return ok ? (u & 0x7fffffffu) : 0u;
}

// ceil(s * 2^40) for the score with order key u.
__device__ __forceinline__ uint64_t mass_of_key(uint32_t u) {
  const double x = static_cast<double>(__uint_as_float(u)) * 1099511627776.0;
  return static_cast<uint64_t>(ceil(x));
}

template <typename T>
__device__ __forceinline__ T block_sum(T v, T* red) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  if (warp == 0) {
    T x = lane < BS_WARPS ? red[lane] : T(0);
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    if (lane == 0) red[0] = x;
  }
  __syncthreads();
  const T r = red[0];
  __syncthreads();
  return r;
}

// Exclusive prefix sum over the block (thread order); returns the total too.
// red: at least 33 entries of shared memory.
template <typename T>
__device__ __forceinline__ T block_exclusive_scan(T v, T* red, T& total) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  T inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const T y = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += y;
  }
  __syncthreads();
  if (lane == 31) red[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    const T x = lane < BS_WARPS ? red[lane] : T(0);
    T xi = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const T y = __shfl_up_sync(0xffffffffu, xi, o);
      if (lane >= o) xi += y;
    }
    red[lane] = xi - x;       // exclusive prefix of warp totals
    if (lane == 31) red[32] = xi;
  }
  __syncthreads();
  const T r = red[warp] + inc - v;
  total = red[32];
  __syncthreads();
  return r;
}

// Block-wide minimum and maximum of u32 values (red: at least 2 * 32 entries).
__device__ __forceinline__ void block_minmax(uint32_t& mn, uint32_t& mx, uint32_t* red) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  mn = __reduce_min_sync(0xffffffffu, mn);
  mx = __reduce_max_sync(0xffffffffu, mx);
  __syncthreads();
  if (lane == 0) {
    red[warp] = mn;
    red[32 + warp] = mx;
  }
  __syncthreads();
  if (warp == 0) {
    uint32_t a = lane < BS_WARPS ? red[lane] : 0xffffffffu;
    uint32_t b = lane < BS_WARPS ? red[32 + lane] : 0u;
    a = __reduce_min_sync(0xffffffffu, a);
    b = __reduce_max_sync(0xffffffffu, b);
    if (lane == 0) {
      red[0] = a;
      red[32] = b;
    }
  }
  __syncthreads();
  mn = red[0];
  mx = red[32];
  __syncthreads();
}

// Visit scores sc[j] for j = threadIdx.x, +1024, ... below n, loading BATCH
// of them before using any: one CTA per head walks a 4L-byte row several
// times, and with one load in flight per thread the walk is bound by L2
// latency, not bandwidth.  f(j, value) is called in index order per thread.
constexpr int BS_BATCH = 8;
template <typename F>
__device__ __forceinline__ void for_each_score(const float* __restrict__ sc, int n, F&& f) {
  for (int j0 = threadIdx.x; j0 < n; j0 += BS_THREADS * BS_BATCH) {
    float v[BS_BATCH];
#pragma unroll
    for (int u = 0; u < BS_BATCH; ++u) {
      const int j = j0 + u * BS_THREADS;
      v[u] = j < n ? __ldg(sc + j) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < BS_BATCH; ++u) {
      const int j = j0 + u * BS_THREADS;
      if (j < n) f(j, v[u]);
    }
  }
}

constexpr int RD_BITS = 11;                 // digit width of the radix descent
constexpr int RD_BINS = 1 << RD_BITS;       // 2048 bins per level
constexpr int BUD_COPIES = 4;               // budget histogram copies (eight warps each)
constexpr int SEL_COPIES = 8;               // select histogram copies (four warps each)
// Each head is one thread-block cluster of BS_CLUSTER CTAs, each taking a
// contiguous quarter of the keys; a CTA publishes its merged histogram in
// its shared memory (two buffers, by level parity) and every CTA reads the
// BS_CLUSTER published histograms in rank order, so all of them take the
// same, timing-independent decision.
constexpr int BS_CLUSTER = 4;
constexpr int BUD_PUB = RD_BINS * (8 + 4);          // one published histogram (sum, count)
constexpr int BUD_SMEM = BUD_COPIES * RD_BINS * (8 + 4) + 2 * BUD_PUB;
constexpr int SEL_PUB = RD_BINS * 4;
constexpr int SEL_SMEM = SEL_COPIES * RD_BINS * 4 + 2 * SEL_PUB;

// Digit plan of a descent over r = key - kmin: nb is the bit length of
// kmax - kmin; level l covers bits [lo(l), hi(l)) of r, 11 bits at a time
// from the top, and the last level ends at bit 0.  An element takes part in
// level l when its bits above hi(l) equal the prefix chosen so far.
struct DigitPlan {
  uint32_t kmin;
  int nb;
  __device__ __forceinline__ int levels() const { return nb <= RD_BITS ? 1 : (nb + RD_BITS - 1) / RD_BITS; }
  __device__ __forceinline__ int hi(int l) const { return nb - RD_BITS * l; }
  __device__ __forceinline__ int lo(int l) const {
    const int x = nb - RD_BITS * (l + 1);
    return x < 0 ? 0 : x;
  }
  // digit of key u at level l, or -1 when it is not a candidate there
  __device__ __forceinline__ int digit(uint32_t u, int l, uint32_t prefix) const {
    const uint32_t r = u - kmin;
    const int h = hi(l), w = h - lo(l);
    if ((static_cast<uint64_t>(r) >> h) != prefix) return -1;
    return static_cast<int>((r >> lo(l)) & ((1u << w) - 1u));
  }
};

struct BudgetArgs {
  const float* scores;  // [B*Hq, L]: the first L_b entries of each row are read
  int32_t* k_head;      // [B*Hq]
  uint32_t* status;     // or null
  int L, Hq;
  int keep_recent;      // r in [0, L]: every k_head is raised to at least min(r, L_b)
  double tau;           // fp32 tau widened
  Seqs seqs;            // sequence lengths L_b
};

// grid: B*Hq clusters of BS_CLUSTER CTAs of 1024 threads; dynamic smem:
// BUD_SMEM (count and mass histograms, BUD_COPIES working copies, two
// published buffers).
__global__ void __cluster_dims__(BS_CLUSTER, 1, 1) __launch_bounds__(BS_THREADS, 1)
    budget_kernel(const BudgetArgs a) {
  extern __shared__ __align__(16) uint8_t bsm[];
  unsigned long long* hsum = reinterpret_cast<unsigned long long*>(bsm);           // [copies][bins]
  uint32_t* hcnt = reinterpret_cast<uint32_t*>(bsm + BUD_COPIES * RD_BINS * 8);    // [copies][bins]
  uint8_t* pub = bsm + BUD_COPIES * RD_BINS * 12;                                  // [2][sum bins, count bins]
  __shared__ unsigned long long red64[33];
  __shared__ uint32_t red32[64];
  __shared__ unsigned long long s_rem, s_stat_tot;
  __shared__ uint32_t s_below, s_chosen, s_stat_min, s_stat_max;

  const uint32_t crank = cluster_rank();
  const int bh = blockIdx.x / BS_CLUSTER;
  const float* sc = a.scores + static_cast<size_t>(bh) * a.L;
  const int copy = (threadIdx.x >> 5) % BUD_COPIES;
  bool bad = false, bad_seq = false;
  const int Lb = a.seqs.len_ok(bh / a.Hq, bad_seq);
  const int span = (Lb + BS_CLUSTER - 1) / BS_CLUSTER;
  const int j0 = min(Lb, static_cast<int>(crank) * span), n = min(Lb, j0 + span) - j0;
  const float* scc = sc + j0;                       // this CTA's keys [j0, j0 + n)

  // pass 0: total mass and the key range (this CTA's part, then the cluster's)
  unsigned long long tot = 0;
  uint32_t kmin = 0xffffffffu, kmax = 0u;
  for_each_score(scc, n, [&](int, float x) {
    const uint32_t u = score_key(x, bad);
    tot += mass_of_key(u);
    kmin = min(kmin, u);
    kmax = max(kmax, u);
  });
  tot = block_sum<unsigned long long>(tot, red64);
  block_minmax(kmin, kmax, red32);
  if (threadIdx.x == 0) {
    s_stat_tot = tot;
    s_stat_min = kmin;
    s_stat_max = kmax;
  }
  cluster_sync();
  if (threadIdx.x == 0) {
    unsigned long long t = 0;
    uint32_t mn = 0xffffffffu, mx = 0u;
    for (uint32_t rk = 0; rk < BS_CLUSTER; ++rk) {
      t += ld_cluster_u64(cluster_map(smem_u32(&s_stat_tot), rk));
      mn = min(mn, ld_cluster_u32(cluster_map(smem_u32(&s_stat_min), rk)));
      mx = max(mx, ld_cluster_u32(cluster_map(smem_u32(&s_stat_max), rk)));
    }
    red64[0] = t;
    red32[0] = mn;
    red32[1] = mx;
  }
  __syncthreads();
  tot = red64[0];
  kmin = red32[0];
  kmax = red32[1];
  __syncthreads();
  const unsigned long long T =
      static_cast<unsigned long long>(floor(__dmul_rn(a.tau, __ull2double_rn(tot))));
  const DigitPlan plan{kmin, Lb > 0 ? 32 - __clz(static_cast<int>(kmax - kmin)) : 0};
  unsigned long long rem = T;
  uint32_t below = 0, prefix = 0;
  bool done = Lb == 0;
  for (int l = 0; !done && l < plan.levels(); ++l) {
    for (int i = threadIdx.x; i < BUD_COPIES * RD_BINS; i += BS_THREADS) {
      hsum[i] = 0;
      hcnt[i] = 0;
    }
    __syncthreads();
    for_each_score(scc, n, [&](int, float x) {
      const uint32_t u = score_key(x, bad);
      const int dg = plan.digit(u, l, prefix);
      if (dg >= 0) {
        atomicAdd(&hcnt[copy * RD_BINS + dg], 1u);
        atomicAdd(&hsum[copy * RD_BINS + dg], static_cast<unsigned long long>(mass_of_key(u)));
      }
    });
    __syncthreads();
    // publish this CTA's histogram (its copies merged) in buffer l & 1
    unsigned long long* ps = reinterpret_cast<unsigned long long*>(pub + (l & 1) * BUD_PUB);
    uint32_t* pc = reinterpret_cast<uint32_t*>(pub + (l & 1) * BUD_PUB + RD_BINS * 8);
    for (int i = threadIdx.x; i < RD_BINS; i += BS_THREADS) {
      unsigned long long sv = 0;
      uint32_t cv = 0;
#pragma unroll
      for (int c = 0; c < BUD_COPIES; ++c) {
        sv += hsum[c * RD_BINS + i];
        cv += hcnt[c * RD_BINS + i];
      }
      ps[i] = sv;
      pc[i] = cv;
    }
    cluster_sync();
    // thread t owns bins 2t and 2t+1 (ascending key order): the cluster's
    // totals, summed over the CTAs in rank order
    unsigned long long s2[2] = {0, 0}, c2[2] = {0, 0};
    for (uint32_t rk = 0; rk < BS_CLUSTER; ++rk) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int bin = 2 * threadIdx.x + e;
        s2[e] += ld_cluster_u64(cluster_map(smem_u32(ps + bin), rk));
        c2[e] += ld_cluster_u32(cluster_map(smem_u32(pc + bin), rk));
      }
    }
    unsigned long long tot_s, tot_c;
    const unsigned long long es = block_exclusive_scan<unsigned long long>(s2[0] + s2[1], red64, tot_s);
    const unsigned long long ec = block_exclusive_scan<unsigned long long>(c2[0] + c2[1], red64, tot_c);
    if (tot_s <= rem) {        // every candidate fits under the threshold: all are pruned
      below += static_cast<uint32_t>(tot_c);
      done = true;
      break;
    }
    // the one bin where the running mass first exceeds rem: bins before it
    // are pruned whole, bins after it are kept whole
    if (es <= rem && rem < es + s2[0]) {
      s_chosen = 2 * threadIdx.x;
      s_rem = rem - es;
      s_below = below + static_cast<uint32_t>(ec);
    } else if (es + s2[0] <= rem && rem < es + s2[0] + s2[1]) {
      s_chosen = 2 * threadIdx.x + 1;
      s_rem = rem - es - s2[0];
      s_below = below + static_cast<uint32_t>(ec + c2[0]);
    }
    __syncthreads();
    rem = s_rem;
    below = s_below;
    prefix = (prefix << (plan.hi(l) - plan.lo(l))) | s_chosen;
    __syncthreads();
  }
  if (threadIdx.x == 0 && crank == 0) {
    uint32_t p = below;
    if (!done) {  // the descent ended on one key value: its tokens share one mass
      const unsigned long long qstar = mass_of_key(kmin + prefix);   // > 0 here
      p += static_cast<uint32_t>(rem / qstar);
    }
    const int32_t kh = Lb - static_cast<int32_t>(p);
    const int32_t r = a.keep_recent < Lb ? a.keep_recent : Lb;
    a.k_head[bh] = kh > r ? kh : r;
    if (bad_seq && a.status) atomicOr(a.status, 0x4u);
  }
  if (a.status && __syncthreads_or(bad) && threadIdx.x == 0) atomicOr(a.status, 0x1u);
  cluster_sync();   // no CTA leaves while another may still read its shared memory
}

// k_seq[b] from the heads' counts: mode 1 the ceiling of their mean, mode 2
// their sum (the partial a device contributes when a sequence's heads are
// split over devices and the budget is the mean), else their maximum.
// grid: B CTAs of 32 threads.
__global__ void __launch_bounds__(32) budget_finalize_kernel(const int32_t* k_head, int32_t* k_seq, int Hq,
                                                             int mode) {
  const int b = blockIdx.x;
  long long sum = 0;
  int mx = 0;
  for (int h = threadIdx.x; h < Hq; h += 32) {
    const int k = k_head[static_cast<size_t>(b) * Hq + h];
    sum += k;
    mx = k > mx ? k : mx;
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    sum += __shfl_xor_sync(0xffffffffu, sum, o);
    const int y = __shfl_xor_sync(0xffffffffu, mx, o);
    mx = y > mx ? y : mx;
  }
  if (threadIdx.x == 0)
    k_seq[b] = mode == 1 ? static_cast<int32_t>((sum + Hq - 1) / Hq) : (mode == 2 ? static_cast<int32_t>(sum) : mx);
}

// The mean-mode budget from the heads' count sum over all devices:
// k_seq[b] = ceil(k_sum[b] / Hq_total) (in place allowed).  One thread per
// sequence.
__global__ void __launch_bounds__(128) budget_mean_kernel(const int32_t* k_sum, int32_t* k_seq, int B,
                                                          int Hq_total) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B) return;
  const long long s = k_sum[b];
  k_seq[b] = static_cast<int32_t>((s + Hq_total - 1) / Hq_total);
}

struct SelectArgs {
  const float* scores;   // [B*Hq, L]: the first L_b entries of each row are read
  Kept kept;             // rows kept per (b, h)
  int32_t* idx;          // [B*Hq, L]
  int L, Hq;
  int keep_recent;       // tokens [L_b - r, L_b) rank above every score
  Seqs seqs;             // sequence lengths L_b
};

// Selection key: the score's order key, or the top key for a forced token
// (no score maps there: order keys of valid scores stay below 2^31).
__device__ __forceinline__ uint32_t select_key(float s, int j, int first_forced, bool& bad) {
  const uint32_t u = score_key(s, bad);
  return j >= first_forced ? 0xffffffffu : u;
}

// grid: B*Hq clusters of BS_CLUSTER CTAs of 1024 threads; dynamic smem:
// SEL_SMEM (count histograms, SEL_COPIES working copies, two published
// buffers).
__global__ void __cluster_dims__(BS_CLUSTER, 1, 1) __launch_bounds__(BS_THREADS, 1)
    select_kernel(const SelectArgs a) {
  extern __shared__ __align__(16) uint8_t ssm[];
  uint32_t* hcnt = reinterpret_cast<uint32_t*>(ssm);                     // [copies][bins]
  uint32_t* pub = reinterpret_cast<uint32_t*>(ssm + SEL_COPIES * RD_BINS * 4);   // [2][bins]
  __shared__ uint32_t red[64];
  __shared__ uint32_t s_rem, s_chosen, s_min, s_max, s_gt, s_eq;
  __shared__ uint32_t w_gt[BS_WARPS], w_eq[BS_WARPS], w_base[BS_WARPS], w_eqb[BS_WARPS];

  const uint32_t crank = cluster_rank();
  const int bh = blockIdx.x / BS_CLUSTER;
  const int cap = a.L;                               // row capacity of idx
  const int L = a.seqs.len(bh / a.Hq);               // this sequence's length
  const float* sc = a.scores + static_cast<size_t>(bh) * cap;
  int32_t* out = a.idx + static_cast<size_t>(bh) * cap;
  const int k = a.kept.of(bh / a.Hq, bh % a.Hq, L);
  const int first_forced = L - (a.keep_recent < L ? a.keep_recent : L);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int copy = warp % SEL_COPIES;
  // this CTA's keys [c0, c0 + n) and its share of the index row
  const int span = (L + BS_CLUSTER - 1) / BS_CLUSTER;
  const int c0 = min(L, static_cast<int>(crank) * span), n = min(L, c0 + span) - c0;
  const int cspan = (cap + BS_CLUSTER - 1) / BS_CLUSTER;
  const int o0 = min(cap, static_cast<int>(crank) * cspan), o1 = min(cap, o0 + cspan);
  bool bad = false;

  if (k == L || k == 0) {  // everything kept, or nothing (the same for the whole cluster)
    for (int i = o0 + threadIdx.x; i < o1; i += BS_THREADS) out[i] = (k == L && i < L) ? i : -1;
    return;
  }
  auto key_at = [&](int j, float x) { return select_key(x, j, first_forced, bad); };
  // pass 0: the key range (this CTA's part, then the cluster's)
  uint32_t kmin = 0xffffffffu, kmax = 0u;
  for_each_score(sc + c0, n, [&](int jl, float x) {
    const uint32_t u = key_at(c0 + jl, x);
    kmin = min(kmin, u);
    kmax = max(kmax, u);
  });
  block_minmax(kmin, kmax, red);
  if (threadIdx.x == 0) {
    s_min = kmin;
    s_max = kmax;
  }
  cluster_sync();
  if (threadIdx.x == 0) {
    uint32_t mn = 0xffffffffu, mx = 0u;
    for (uint32_t rk = 0; rk < BS_CLUSTER; ++rk) {
      mn = min(mn, ld_cluster_u32(cluster_map(smem_u32(&s_min), rk)));
      mx = max(mx, ld_cluster_u32(cluster_map(smem_u32(&s_max), rk)));
    }
    red[0] = mn;
    red[1] = mx;
  }
  __syncthreads();
  kmin = red[0];
  kmax = red[1];
  __syncthreads();
  const DigitPlan plan{kmin, 32 - __clz(static_cast<int>(kmax - kmin))};
  // radix descent from the top: the k-th largest key ut, and how many of the
  // keys equal to ut are taken (rem)
  uint32_t rem = static_cast<uint32_t>(k), prefix = 0;
  for (int l = 0; l < plan.levels(); ++l) {
    for (int i = threadIdx.x; i < SEL_COPIES * RD_BINS; i += BS_THREADS) hcnt[i] = 0;
    __syncthreads();
    for_each_score(sc + c0, n, [&](int jl, float x) {
      const int dg = plan.digit(key_at(c0 + jl, x), l, prefix);
      if (dg >= 0) atomicAdd(&hcnt[copy * RD_BINS + dg], 1u);
    });
    __syncthreads();
    uint32_t* pb = pub + (l & 1) * RD_BINS;          // publish the merged copies
    for (int i = threadIdx.x; i < RD_BINS; i += BS_THREADS) {
      uint32_t cv = 0;
#pragma unroll
      for (int c = 0; c < SEL_COPIES; ++c) cv += hcnt[c * RD_BINS + i];
      pb[i] = cv;
    }
    cluster_sync();
    // thread t owns bins B-1-2t and B-2-2t (descending key order): the
    // cluster's counts, summed over the CTAs in rank order
    uint32_t c2[2] = {0, 0};
    for (uint32_t rk = 0; rk < BS_CLUSTER; ++rk) {
#pragma unroll
      for (int e = 0; e < 2; ++e)
        c2[e] += ld_cluster_u32(cluster_map(smem_u32(pb + RD_BINS - 1 - 2 * threadIdx.x - e), rk));
    }
    uint32_t tot;
    const uint32_t ex = block_exclusive_scan<uint32_t>(c2[0] + c2[1], red, tot);
    // the one bin where the running count from the top reaches rem
    if (ex < rem && rem <= ex + c2[0]) {
      s_chosen = RD_BINS - 1 - 2 * threadIdx.x;
      s_rem = rem - ex;
    } else if (ex + c2[0] < rem && rem <= ex + c2[0] + c2[1]) {
      s_chosen = RD_BINS - 2 - 2 * threadIdx.x;
      s_rem = rem - ex - c2[0];
    }
    __syncthreads();
    rem = s_rem;
    prefix = (prefix << (plan.hi(l) - plan.lo(l))) | s_chosen;
    __syncthreads();
  }
  const uint32_t ut = kmin + prefix;
  const uint32_t need = rem;  // keys equal to ut to take, 1..count(ut)

  // compaction in index order: warp w of the CTA walks its contiguous
  // segment of the CTA's keys 32 at a time (coalesced); pass A counts,
  // pass B writes
  const int seg = (n + BS_WARPS - 1) / BS_WARPS;
  const int j0 = c0 + min(n, warp * seg), j1 = c0 + min(n, warp * seg + seg);
  // keys of the warp's segment, BS_BATCH steps of 32 loaded at a time
  auto seg_keys = [&](int jb, uint32_t (&u)[BS_BATCH]) {
    float v[BS_BATCH];
#pragma unroll
    for (int t = 0; t < BS_BATCH; ++t) {
      const int j = jb + t * 32 + lane;
      v[t] = j < j1 ? __ldg(sc + j) : 0.f;
    }
#pragma unroll
    for (int t = 0; t < BS_BATCH; ++t) u[t] = key_at(jb + t * 32 + lane, v[t]);
  };
  uint32_t gt = 0, eq = 0;
  for (int jb = j0; jb < j1; jb += 32 * BS_BATCH) {
    uint32_t u[BS_BATCH];
    seg_keys(jb, u);
#pragma unroll
    for (int t = 0; t < BS_BATCH; ++t) {
      const bool in = jb + t * 32 + lane < j1;
      gt += __popc(__ballot_sync(0xffffffffu, in && u[t] > ut));
      eq += __popc(__ballot_sync(0xffffffffu, in && u[t] == ut));
    }
  }
  if (lane == 0) {
    w_gt[warp] = gt;
    w_eq[warp] = eq;
  }
  __syncthreads();
  if (warp == 0) {   // this CTA's totals, published for the later ranks
    uint32_t g = w_gt[lane], e = w_eq[lane];
    g = __reduce_add_sync(0xffffffffu, g);
    e = __reduce_add_sync(0xffffffffu, e);
    if (lane == 0) {
      s_gt = g;
      s_eq = e;
    }
  }
  cluster_sync();
  if (warp == 0) {   // per-warp bases: ties go to the earlier ranks and warps first
    uint32_t eq_before = 0, base = 0;
    for (uint32_t rk = 0; rk < crank; ++rk) {
      const uint32_t g = ld_cluster_u32(cluster_map(smem_u32(&s_gt), rk));
      const uint32_t e = ld_cluster_u32(cluster_map(smem_u32(&s_eq), rk));
      base += g + (need > eq_before ? min(e, need - eq_before) : 0u);
      eq_before += e;
    }
    const uint32_t e = w_eq[lane], g = w_gt[lane];
    uint32_t ei = e;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, ei, o);
      if (lane >= o) ei += y;
    }
    const uint32_t eb = eq_before + ei - e;           // ties in earlier ranks and warps
    const uint32_t te = need > eb ? min(e, need - eb) : 0u;
    const uint32_t t = g + te;
    uint32_t ti = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, ti, o);
      if (lane >= o) ti += y;
    }
    w_base[lane] = base + ti - t;
    w_eqb[lane] = eb;
  }
  __syncthreads();
  uint32_t pos = w_base[warp], eq_seen = w_eqb[warp];
  const uint32_t lt = (1u << lane) - 1u;
  for (int jb = j0; jb < j1; jb += 32 * BS_BATCH) {
    uint32_t u[BS_BATCH];
    seg_keys(jb, u);
#pragma unroll
    for (int t = 0; t < BS_BATCH; ++t) {
      const int j = jb + t * 32 + lane;
      const bool is_eq = j < j1 && u[t] == ut;
      const uint32_t eqm = __ballot_sync(0xffffffffu, is_eq);
      const bool take = j < j1 && (u[t] > ut || (is_eq && eq_seen + __popc(eqm & lt) < need));
      const uint32_t tm = __ballot_sync(0xffffffffu, take);
      if (take) out[pos + __popc(tm & lt)] = j;
      pos += __popc(tm);
      eq_seen += __popc(eqm);
    }
  }
  for (int i = max(k, o0) + threadIdx.x; i < o1; i += BS_THREADS) out[i] = -1;
  cluster_sync();   // no CTA leaves while another may still read its shared memory
}

}  // namespace tsa
