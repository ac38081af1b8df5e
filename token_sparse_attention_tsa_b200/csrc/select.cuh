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
// neither kernel sorts: both run a most-significant-digit radix descent
// (4 levels of 8 bits) over the score bit patterns with per-warp shared
// histograms, then (select) compact the chosen indices in index order, which
// yields S_h ascending.  Ties at the threshold go to the smaller index.
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
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t* red, uint32_t& total) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint32_t inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += y;
  }
  __syncthreads();
  if (lane == 31) red[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    uint32_t x = red[lane];
    uint32_t xi = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, xi, o);
      if (lane >= o) xi += y;
    }
    red[lane] = xi - x;       // exclusive prefix of warp totals
    if (lane == 31) red[32] = xi;
  }
  __syncthreads();
  const uint32_t r = red[warp] + inc - v;
  total = red[32];
  __syncthreads();
  return r;
}

struct BudgetArgs {
  const float* scores;  // [B*Hq, L]: the first L_b entries of each row are read
  int32_t* k_head;      // [B*Hq]
  uint32_t* status;     // or null
  int L, Hq;
  int keep_recent;      // r in [0, L]: every k_head is raised to at least min(r, L_b)
  double tau;           // fp32 tau widened
  Seqs seqs;            // sequence lengths L_b
};

// grid: B*Hq CTAs of 1024 threads; dynamic smem: per-warp histograms.
__global__ void __launch_bounds__(BS_THREADS, 1) budget_kernel(const BudgetArgs a) {
  extern __shared__ __align__(16) uint8_t bsm[];
  unsigned long long* hsum = reinterpret_cast<unsigned long long*>(bsm);             // [32][256]
  uint32_t* hcnt = reinterpret_cast<uint32_t*>(bsm + BS_WARPS * 256 * 8);            // [32][256]
  __shared__ unsigned long long red64[BS_WARPS];
  __shared__ unsigned long long s_rem;
  __shared__ uint32_t s_below, s_prefix, s_mask, s_done;

  const int bh = blockIdx.x;
  const float* sc = a.scores + static_cast<size_t>(bh) * a.L;
  const int warp = threadIdx.x >> 5;
  bool bad = false, bad_seq = false;
  const int Lb = a.seqs.len_ok(bh / a.Hq, bad_seq);

  unsigned long long tot = 0;
  for (int j = threadIdx.x; j < Lb; j += BS_THREADS) tot += mass_of_key(score_key(sc[j], bad));
  tot = block_sum<unsigned long long>(tot, red64);
  const unsigned long long T =
      static_cast<unsigned long long>(floor(__dmul_rn(a.tau, __ull2double_rn(tot))));
  if (threadIdx.x == 0) {
    s_rem = T;
    s_below = 0;
    s_prefix = 0;
    s_mask = 0;
    s_done = 0;
  }
  __syncthreads();

  for (int level = 0; level < 4; ++level) {
    const int shift = 24 - 8 * level;
    for (int i = threadIdx.x; i < BS_WARPS * 256; i += BS_THREADS) {
      hsum[i] = 0;
      hcnt[i] = 0;
    }
    __syncthreads();
    const uint32_t prefix = s_prefix, mask = s_mask;
    for (int j = threadIdx.x; j < Lb; j += BS_THREADS) {
      const uint32_t u = score_key(sc[j], bad);
      if ((u & mask) == prefix) {
        const uint32_t dgt = (u >> shift) & 255u;
        atomicAdd(&hcnt[warp * 256 + dgt], 1u);
        atomicAdd(&hsum[warp * 256 + dgt], static_cast<unsigned long long>(mass_of_key(u)));
      }
    }
    __syncthreads();
    if (threadIdx.x < 256) {
      unsigned long long s = 0;
      uint32_t c = 0;
      for (int w = 0; w < BS_WARPS; ++w) {
        s += hsum[w * 256 + threadIdx.x];
        c += hcnt[w * 256 + threadIdx.x];
      }
      hsum[threadIdx.x] = s;
      hcnt[threadIdx.x] = c;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      unsigned long long rem = s_rem;
      uint32_t below = s_below;
      int chosen = -1;
      for (int dgt = 0; dgt < 256; ++dgt) {
        if (hsum[dgt] <= rem) {
          rem -= hsum[dgt];
          below += hcnt[dgt];
        } else {
          chosen = dgt;
          break;
        }
      }
      s_rem = rem;
      s_below = below;
      if (chosen < 0) {
        s_done = 1;  // everything left fits under T
      } else {
        s_prefix = prefix | (static_cast<uint32_t>(chosen) << shift);
        s_mask = mask | (255u << shift);
      }
    }
    __syncthreads();
    if (s_done) break;
  }
  if (threadIdx.x == 0) {
    uint32_t p = s_below;
    if (!s_done) {
      const unsigned long long qstar = mass_of_key(s_prefix);  // > 0 here
      p += static_cast<uint32_t>(s_rem / qstar);
    }
    const int32_t kh = Lb - static_cast<int32_t>(p);
    const int32_t r = a.keep_recent < Lb ? a.keep_recent : Lb;
    a.k_head[bh] = kh > r ? kh : r;
    if (bad_seq && a.status) atomicOr(a.status, 0x4u);
  }
  if (a.status && __syncthreads_or(bad) && threadIdx.x == 0) atomicOr(a.status, 0x1u);
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

// grid: B*Hq CTAs of 1024 threads; dynamic smem: per-warp count histograms.
__global__ void __launch_bounds__(BS_THREADS, 1) select_kernel(const SelectArgs a) {
  extern __shared__ __align__(16) uint8_t ssm[];
  uint32_t* hcnt = reinterpret_cast<uint32_t*>(ssm);  // [32][256]
  __shared__ uint32_t red[33];
  __shared__ uint32_t s_rem, s_prefix, s_mask;

  const int bh = blockIdx.x;
  const int cap = a.L;                               // row capacity of idx
  const int L = a.seqs.len(bh / a.Hq);               // this sequence's length
  const float* sc = a.scores + static_cast<size_t>(bh) * cap;
  int32_t* out = a.idx + static_cast<size_t>(bh) * cap;
  const int k = a.kept.of(bh / a.Hq, bh % a.Hq, L);
  const int first_forced = L - (a.keep_recent < L ? a.keep_recent : L);
  const int warp = threadIdx.x >> 5;
  bool bad = false;

  if (k == L) {  // everything kept
    for (int i = threadIdx.x; i < cap; i += BS_THREADS) out[i] = i < L ? i : -1;
    return;
  }
  if (k == 0) {
    for (int i = threadIdx.x; i < cap; i += BS_THREADS) out[i] = -1;
    return;
  }
  if (threadIdx.x == 0) {
    s_rem = static_cast<uint32_t>(k);
    s_prefix = 0;
    s_mask = 0;
  }
  __syncthreads();
  // radix descent from the top: the k-th largest key u_t, and how many of
  // the keys equal to u_t are taken (s_rem)
  for (int level = 0; level < 4; ++level) {
    const int shift = 24 - 8 * level;
    for (int i = threadIdx.x; i < BS_WARPS * 256; i += BS_THREADS) hcnt[i] = 0;
    __syncthreads();
    const uint32_t prefix = s_prefix, mask = s_mask;
    for (int j = threadIdx.x; j < L; j += BS_THREADS) {
      const uint32_t u = select_key(sc[j], j, first_forced, bad);
      if ((u & mask) == prefix) atomicAdd(&hcnt[warp * 256 + ((u >> shift) & 255u)], 1u);
    }
    __syncthreads();
    if (threadIdx.x < 256) {
      uint32_t c = 0;
      for (int w = 0; w < BS_WARPS; ++w) c += hcnt[w * 256 + threadIdx.x];
      hcnt[threadIdx.x] = c;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      uint32_t rem = s_rem;
      int chosen = 0;
      for (int dgt = 255; dgt >= 0; --dgt) {
        if (hcnt[dgt] < rem) {
          rem -= hcnt[dgt];
        } else {
          chosen = dgt;
          break;
        }
      }
      s_rem = rem;
      s_prefix = prefix | (static_cast<uint32_t>(chosen) << shift);
      s_mask = mask | (255u << shift);
    }
    __syncthreads();
  }
  const uint32_t ut = s_prefix;
  const uint32_t need = s_rem;  // keys equal to ut to take, 1..count(ut)

  // compaction in index order: thread t owns the contiguous range [j0, j1)
  const int per = (L + BS_THREADS - 1) / BS_THREADS;
  const int j0 = min(L, static_cast<int>(threadIdx.x) * per);
  const int j1 = min(L, j0 + per);
  uint32_t gt = 0, eq = 0;
  for (int j = j0; j < j1; ++j) {
    const uint32_t u = select_key(sc[j], j, first_forced, bad);
    gt += (u > ut);
    eq += (u == ut);
  }
  uint32_t eq_total;
  const uint32_t eq_before = block_exclusive_scan(eq, red, eq_total);
  const uint32_t take_eq = need > eq_before ? min(eq, need - eq_before) : 0u;
  uint32_t cnt_total;
  uint32_t pos = block_exclusive_scan(gt + take_eq, red, cnt_total);
  uint32_t eq_seen = eq_before;
  for (int j = j0; j < j1; ++j) {
    const uint32_t u = select_key(sc[j], j, first_forced, bad);
    bool take = u > ut;
    if (u == ut) {
      take = eq_seen < need;
      ++eq_seen;
    }
    if (take) out[pos++] = j;
  }
  for (int i = k + threadIdx.x; i < cap; i += BS_THREADS) out[i] = -1;
}

}  // namespace tsa
