// score.cuh -- proxy importance scores of the Token Sparse Attention method.
//
// Source: gist.science summary page "Token Sparse Attention: Efficient
// Long-Context Inference with Interleaved Token Selection", section 2,
// "Cobertura Dinamica de Tokens", scoring: a light attention map of the most
// recent queries against all keys; a key's importance is the sum of its
// column of attention weights.
//
// Here: for each (b, h) and window row i in [L_b-w_b, L_b), x_ij = scale *
// q[b,h,i].k[b,h/G,j] over keys j <= i; p_ij = softmax_j(x_ij);
// score[b,h,j] = sum_i p_ij (L_b the sequence's length, w_b = min(w, L_b)).
//
// The logits come from tcgen05 tensor cores (bf16 products are exact; fp32
// accumulation).  To keep the scores within 1e-5 relative of the exact value,
// d is split into four independent accumulators (d/4 terms each) that are
// summed in registers, which cuts the accumulation error about fourfold; the
// stage is bound by its exponentials, not by the tensor core.  Two passes:
//   stats  per key chunk: row max m_c and sum Z_c of 2^(x log2e - m_c)
//   merge  per row: m = max_c m_c, Z = sum_c Z_c 2^(m_c - m)  (fp64)
//   sums   per key tile: score_j = sum_i 2^(x_ij log2e - m_i) / Z_i, the column
//          sum done by a warp butterfly and a cross-warp pass in shared memory
// One CTA: warps 0..3 one thread per window row (TMEM lane), warp 4 MMA
// issuer, warp 5 TMA producer.  S is double-buffered in TMEM (64 keys x 4
// partial accumulators = 256 columns per buffer).  Every wait is bounded.
#pragma once

#include <cuda_bf16.h>

#include "sm100.cuh"

namespace tsa {

constexpr int SC_KEYS = 64;          // keys per tile (MMA N)
constexpr int SC_ROWS = 128;         // window rows per block (MMA M)
constexpr int SC_MIN_CHUNK_TILES = 16;   // smallest key span of a CTA, in tiles (1024 keys)
constexpr int SC_THREADS = 192;
constexpr int SC_STAGES = 3;

struct ScoreArgs {
  float* scores;           // [B*Hq, L]
  float* part_m;           // [B*Hq, w, n_chunks] chunk row max (log2 units)
  double* part_z;          // [B*Hq, w, n_chunks] chunk row sum
  float2* stats;           // [B*Hq, w] (m, 1/Z), log2 units
  uint32_t* status;        // or null
  uint32_t* abort_word;    // launch-wide abort word (zeroed before launch) or null
  int L, w, Hq, Hkv, G;
  int n_chunks;            // key chunks per head
  int chunk_tiles;         // key tiles per chunk (one CTA each)
  int n_rb;                // window row blocks of 128
  float scale_log2;        // scale * log2(e)
  uint64_t limit_ns;
  int token_major;         // q, k maps are (d, H, L, B) (else (d, L, H, B))
  int test_stall;          // failure-path test: the MMA issuer first waits on a barrier nothing completes
  Seqs seqs;               // sequence lengths (and packed token offsets)
};

template <int D>
struct ScoreLayout {
  static constexpr int CHUNK = 128 * 128;                // 128 rows x 64 bf16 (SW128)
  static constexpr int NCH = D / 64;
  static constexpr int Q_BYTES = SC_ROWS * D * 2;
  static constexpr int K_BYTES = SC_KEYS * D * 2;
  static constexpr int K_CHUNK = SC_KEYS * 128;          // 64 rows x 64 bf16
  static constexpr int STAGE = Q_BYTES + K_BYTES;
  static constexpr int OFF_RED = SC_STAGES * STAGE;      // [4 warps][64] floats
  static constexpr int OFF_BAR = OFF_RED + 4 * SC_KEYS * 4;
  static constexpr int TOTAL = OFF_BAR + 256;
  static constexpr int ALLOC = TOTAL + 1024;
  static constexpr int PART = D / 4;                     // d columns per partial accumulator
  static constexpr int KSTEPS = PART / 16;               // MMA k-steps per partial
};

enum : int { SB_FULL = 0, SB_EMPTY = SC_STAGES, SB_S = 2 * SC_STAGES, SB_SFREE = SB_S + 2,
             SB_DRAIN = SB_SFREE + 2, SB_COUNT = SB_DRAIN + 1 };

// Sum of 32 values held one per lane... done for 32 columns at once: on entry
// lane l holds v[c] for columns c = 0..31 of its row; on exit lane l holds the
// sum over the warp's 32 rows of column l (recursive halving).
__device__ __forceinline__ float warp_column_sums(float (&v)[32], int lane) {
#pragma unroll
  for (int width = 16; width >= 1; width >>= 1) {
    const bool upper = (lane & width) != 0;
#pragma unroll
    for (int c = 0; c < width; ++c) {
      // keep the half of the columns this lane will own, send the other half
      const float send = upper ? v[c] : v[c + width];
      const float keep = upper ? v[c + width] : v[c];
      v[c] = keep + __shfl_xor_sync(0xffffffffu, send, width);
    }
  }
  return v[0];
}

// Shared pipeline: producer and MMA issuer for `steps` (row block, key tile)
// pairs; step s -> (rb, kt) by the caller's mapping.  kPass2 selects the
// order: pass 1 walks key tiles inside a row block, pass 2 row blocks inside a
// key tile.
template <int D, bool kPass2>
__global__ void __launch_bounds__(SC_THREADS, 1)
    score_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 const ScoreArgs a) {
  using C = ScoreLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int chunk = blockIdx.x;
  const int bh = blockIdx.y;
  const int b = bh / a.Hq, h = bh - (bh / a.Hq) * a.Hq;
  const int Lb = a.seqs.len(b);                  // this sequence's length
  const int wb = a.w < Lb ? a.w : Lb;              // its window
  const int pos0 = Lb - wb;                        // position of window row 0
  const int key0 = chunk * a.chunk_tiles * SC_KEYS;
  int n_kt = Lb > key0 ? (Lb - key0 + SC_KEYS - 1) / SC_KEYS : 0;
  n_kt = n_kt > a.chunk_tiles ? a.chunk_tiles : n_kt;
  const int steps = n_kt * a.n_rb;
  auto step_rb = [&](int s) { return kPass2 ? s % a.n_rb : s / n_kt; };
  auto step_kt = [&](int s) { return kPass2 ? s / a.n_rb : s % n_kt; };

  auto bar = [&](int i) -> uint32_t { return base + C::OFF_BAR + 8u * static_cast<uint32_t>(i); };
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(gbase + C::OFF_BAR + 8 * SB_COUNT);
  volatile int* cta_abort = reinterpret_cast<volatile int*>(gbase + C::OFF_BAR + 8 * SB_COUNT + 4);
  if (threadIdx.x == 0) {
    for (int s = 0; s < SC_STAGES; ++s) {
      mbar_init(bar(SB_FULL + s), 1);
      mbar_init(bar(SB_EMPTY + s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar(SB_S + t), 1);
      mbar_init(bar(SB_SFREE + t), 4);
    }
    mbar_init(bar(SB_DRAIN), 1);
    *cta_abort = (a.abort_word && *reinterpret_cast<volatile uint32_t*>(a.abort_word)) ? 1 : 0;
    fence_mbar_init();
  }
  if (warp == 4) {
    tmem_alloc(smem_u32(tmem_holder), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const WaitCtl wc{cta_abort, a.status, a.abort_word, a.limit_ns};
  const bool run = (*cta_abort == 0);

  if (!run) {
    // another CTA of this launch timed out: nothing to do
  } else if (warp == 5) {
    // ------------------------------------------------------------ producer
    const bool leader = elect_one();
    int issued = 0;
    for (int s = 0; s < steps; ++s) {
      const int st = s % SC_STAGES, u = s / SC_STAGES;
      if (u >= 1 && !__all_sync(0xffffffffu, mbar_wait(bar(SB_EMPTY + st), (u - 1) & 1, wc))) break;
      if (leader) {
        const uint32_t sb = base + st * C::STAGE;
        mbar_arrive_expect_tx(bar(SB_FULL + st), C::STAGE);
        const int qrow = a.seqs.map_t(b, pos0 + step_rb(s) * SC_ROWS);
        const int krow = a.seqs.map_t(b, key0 + step_kt(s) * SC_KEYS);
        const int bc = a.seqs.map_b(b);
#pragma unroll
        for (int c = 0; c < C::NCH; ++c) {
          tma_load_rows(sb + c * C::CHUNK, &tmQ, bar(SB_FULL + st), a.token_major, c * 64, qrow, h, bc);
          tma_load_rows(sb + C::Q_BYTES + c * C::K_CHUNK, &tmK, bar(SB_FULL + st), a.token_major, c * 64, krow,
                        h / a.G, bc);
        }
      }
      issued = s + 1;
    }
    if (elect_one() && *cta_abort) {
      for (int s = issued - SC_STAGES < 0 ? 0 : issued - SC_STAGES; s < issued; ++s)
        mbar_wait_drain(bar(SB_FULL + s % SC_STAGES), (s / SC_STAGES) & 1, 1000000000ull);
    }
  } else if (warp == 4) {
    // ------------------------------------------------------------ MMA issuer
    const bool leader = elect_one();
    constexpr uint32_t idS = idesc_bf16_f32(128, SC_KEYS, 0, 0);
    // test hook: phase 0 of the drain barrier completes only at teardown, so
    // this bounded wait runs out and the CTA takes the abort path
    const bool stalled = a.test_stall && !__all_sync(0xffffffffu, mbar_wait(bar(SB_DRAIN), 0, wc));
    for (int s = 0; !stalled && s < steps; ++s) {
      const int st = s % SC_STAGES, buf = s & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(bar(SB_FULL + st), (s / SC_STAGES) & 1, wc))) break;
      if (s >= 2 && !__all_sync(0xffffffffu, mbar_wait(bar(SB_SFREE + buf), ((s >> 1) - 1) & 1, wc))) break;
      tc_fence_after();
      if (leader) {
        const uint32_t qa = base + st * C::STAGE;
        const uint32_t ka = qa + C::Q_BYTES;
#pragma unroll
        for (int p = 0; p < 4; ++p) {
#pragma unroll
          for (int k = 0; k < C::KSTEPS; ++k) {
            const int kk = p * C::KSTEPS + k;                  // 16-column step of d
            const uint32_t qoff = (kk >> 2) * C::CHUNK + (kk & 3) * 32;
            const uint32_t koff = (kk >> 2) * C::K_CHUNK + (kk & 3) * 32;
            mma_bf16_ss(tmem + buf * 256 + p * SC_KEYS, smem_desc(qa + qoff, 16, 1024, kSwizzle128B),
                        smem_desc(ka + koff, 16, 1024, kSwizzle128B), idS, k > 0 ? 1u : 0u);
          }
        }
        mma_commit(bar(SB_S + buf));
        mma_commit(bar(SB_EMPTY + st));
      }
    }
    if (leader) {
      mma_commit(bar(SB_DRAIN));
      mbar_wait_drain(bar(SB_DRAIN), 0, 1000000000ull);
    }
  } else {
    // ------------------------------------------------------------ rows
    const int r = warp * 32 + lane;                 // row within the block (TMEM lane)
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const float sl2 = a.scale_log2;
    float m_run = -INFINITY;                        // pass 1: running max (log2 units)
    double z_run = 0.0;
    float colsum[2] = {0.f, 0.f};                   // pass 2: this lane's two columns
    float2 st_row = make_float2(0.f, 0.f);
    int cur_rb = -1;
    for (int s = 0; s < steps; ++s) {
      const int buf = s & 1, rb = step_rb(s), kt = step_kt(s);
      const int wr = rb * SC_ROWS + r;              // window row
      const int pos = pos0 + wr;                    // its position
      const bool row_ok = wr < wb;
      // the four row warps agree before going on, so the shared-memory column
      // exchange below can never leave a warp waiting alone
      const bool ok = __all_sync(0xffffffffu, mbar_wait(bar(SB_S + buf), (s >> 1) & 1, wc));
      if (!bar_and(1, 128, ok)) break;
      tc_fence_after();
      float x[2][32];
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        float pa[32], pb[32], pc[32], pd[32];
        tmem_ld32(tmem + lane_off + buf * 256 + 0 * SC_KEYS + c * 32, pa);
        tmem_ld32(tmem + lane_off + buf * 256 + 1 * SC_KEYS + c * 32, pb);
        tmem_ld32(tmem + lane_off + buf * 256 + 2 * SC_KEYS + c * 32, pc);
        tmem_ld32(tmem + lane_off + buf * 256 + 3 * SC_KEYS + c * 32, pd);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 32; ++e) x[c][e] = (pa[e] + pb[e]) + (pc[e] + pd[e]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(SB_SFREE + buf));
      const int kbase = key0 + kt * SC_KEYS;
      if constexpr (!kPass2) {
        if (rb != cur_rb) {                         // a new row block starts
          if (cur_rb >= 0 && cur_rb * SC_ROWS + r < a.w) {
            const size_t o = (static_cast<size_t>(bh) * a.w + cur_rb * SC_ROWS + r) * a.n_chunks + chunk;
            a.part_m[o] = m_run;
            a.part_z[o] = z_run;
          }
          cur_rb = rb;
          m_run = -INFINITY;
          z_run = 0.0;
        }
        float mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int key = kbase + c * 32 + e;
            x[c][e] = (row_ok && key <= pos && key < Lb) ? x[c][e] * sl2 : -INFINITY;
            mx = fmaxf(mx, x[c][e]);
          }
        if (mx != -INFINITY) {
          float z8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int c = 0; c < 2; ++c)
#pragma unroll
            for (int e = 0; e < 32; ++e) z8[e & 7] += ex2_approx(x[c][e] - mx);
          const float zs = ((z8[0] + z8[1]) + (z8[2] + z8[3])) + ((z8[4] + z8[5]) + (z8[6] + z8[7]));
          if (mx > m_run) {
            z_run = z_run * exp2(static_cast<double>(m_run) - mx) + zs;
            m_run = mx;
          } else {
            z_run += static_cast<double>(zs) * exp2(static_cast<double>(mx) - m_run);
          }
        }
      } else {
        if (rb != cur_rb) {
          cur_rb = rb;
          st_row = row_ok ? a.stats[static_cast<size_t>(bh) * a.w + wr] : make_float2(0.f, 0.f);
        }
#pragma unroll
        for (int c = 0; c < 2; ++c) {
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int key = kbase + c * 32 + e;
            x[c][e] = (row_ok && key <= pos && key < Lb) ? ex2_approx(fmaf(x[c][e], sl2, -st_row.x)) * st_row.y
                                                        : 0.f;
          }
          colsum[c] += warp_column_sums(x[c], lane);
        }
        const bool tile_done = (rb == a.n_rb - 1);
        if (tile_done) {                            // combine the four warps, store the tile
          float* red = reinterpret_cast<float*>(gbase + C::OFF_RED);
          bar_and(1, 128, true);                      // previous tile's reads are done
          red[warp * SC_KEYS + lane] = colsum[0];
          red[warp * SC_KEYS + 32 + lane] = colsum[1];
          bar_and(1, 128, true);
          if (warp < 2) {
            const int col = warp * 32 + lane;
            const float v = (red[col] + red[SC_KEYS + col]) + (red[2 * SC_KEYS + col] + red[3 * SC_KEYS + col]);
            if (kbase + col < Lb) a.scores[static_cast<size_t>(bh) * a.L + kbase + col] = v;
          }
          colsum[0] = colsum[1] = 0.f;
        }
      }
    }
    if constexpr (!kPass2) {
      if (cur_rb >= 0 && cur_rb * SC_ROWS + r < a.w) {
        const size_t o = (static_cast<size_t>(bh) * a.w + cur_rb * SC_ROWS + r) * a.n_chunks + chunk;
        a.part_m[o] = m_run;
        a.part_z[o] = z_run;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Merge the chunk statistics: one thread per (head, window row), over the
// key chunks its sequence has.
static __global__ void score_merge_kernel(const ScoreArgs a, int total_rows) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= total_rows) return;
  const int Lb = a.seqs.len(idx / a.w / a.Hq);
  const int span = a.chunk_tiles * SC_KEYS;
  const int nc = (Lb + span - 1) / span;
  const float* pm = a.part_m + static_cast<size_t>(idx) * a.n_chunks;
  const double* pz = a.part_z + static_cast<size_t>(idx) * a.n_chunks;
  float m = -INFINITY;
  for (int c = 0; c < nc; ++c) m = fmaxf(m, pm[c]);
  double z = 0.0;
  for (int c = 0; c < nc; ++c)
    if (pm[c] != -INFINITY) z += pz[c] * exp2(static_cast<double>(pm[c]) - m);
  a.stats[idx] = make_float2(m, static_cast<float>(1.0 / z));
}

}  // namespace tsa
