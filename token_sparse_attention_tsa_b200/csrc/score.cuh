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
// Work split.  One CTA takes one KV head of one sequence, GH of its G query
// heads and a chunk of keys.  The window rows of those heads are packed one
// head after another, each head padded to W32 = w rounded up to 32 rows (so
// a warp's 32 TMEM lanes never straddle two heads), into up to four 128-row
// MMA tiles; each K tile is loaded once and multiplied by every packed row,
// so the key stream crosses L2 once per GQA group, not once per query head.
// Windows longer than 512 rows are taken in several row passes per CTA.
//
// The logits come from tcgen05 tensor cores (bf16 products are exact; fp32
// accumulation).  To keep the scores within 1e-5 relative of the exact value,
// d is split into two halves accumulated separately and summed in registers,
// which halves the accumulation error of one long sum.  Two passes:
//   stats  per key chunk: row max m_c and sum Z_c of 2^(x log2e - m_c)
//   merge  per row: m = max_c m_c, Z = sum_c Z_c 2^(m_c - m)  (fp64)
//   sums   per key tile: score_j = sum_i 2^(x_ij log2e - m_i) / Z_i
// Warps 0..15 own the rows: warp w reads TMEM lanes 32(w%4).. and key
// columns 16(w/4)..+16 of every M tile; warp 16 issues the MMAs, warp 17
// the TMA loads.  Each M tile of S has its own ready/free barriers, so the
// MMA of the next key tile into tile m starts as soon as the 16 row warps
// have loaded tile m.  Column sums: a warp butterfly over its 32 rows, then
// a fixed-order sum over a head's 32-row slots in shared memory (no float
// atomics: the result does not depend on timing).  Every wait is bounded.
#pragma once

#include <cuda_bf16.h>

#include "sm100.cuh"

namespace tsa {

constexpr int SC_KEYS = 64;              // keys per tile (MMA N)
constexpr int SC_QBOX = 32;              // query rows per TMA box (one head slot)
constexpr int SC_ROW_WARPS = 16;
constexpr int SC_THREADS = (SC_ROW_WARPS + 2) * 32;
constexpr int SC_MMA_WARP = SC_ROW_WARPS;
constexpr int SC_LOAD_WARP = SC_ROW_WARPS + 1;
constexpr int SC_MAX_MT = 4;             // M tiles (128 packed rows each) per row pass
constexpr int SC_PASS_ROWS = SC_MAX_MT * 128;
constexpr int SC_STAGES = 3;
constexpr int SC_MIN_CHUNK_TILES = 16;   // smallest key span of a CTA, in tiles (1024 keys)

struct ScoreArgs {
  float* scores;           // [B*Hq, L]
  float* part_m;           // [B*Hq, w, n_chunks] chunk row max (log2 units)
  double* part_z;          // [B*Hq, w, n_chunks] chunk row sum
  float2* stats;           // [B*Hq, w] (m, 1/Z), log2 units
  uint32_t* status;        // or null
  uint32_t* abort_word;    // launch-wide abort word (zeroed before launch) or null
  int L, w, Hq, Hkv, G;
  int W32;                 // w rounded up to a multiple of 32: packed rows per head
  int GH;                  // query heads per CTA
  int n_hg;                // head groups per KV head: ceil(G / GH)
  int n_rp;                // row passes per CTA: ceil(GH * W32 / 512)
  int MT;                  // M tiles per row pass
  int n_chunks;            // key chunks per head
  int chunk_tiles;         // key tiles per chunk (one CTA each)
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
  static constexpr int Q_TILE = NCH * CHUNK;             // one 128-row M tile of Q
  static constexpr int K_CHUNK = SC_KEYS * 128;          // 64 rows x 64 bf16
  static constexpr int K_BYTES = NCH * K_CHUNK;
  static constexpr int OFF_K = SC_MAX_MT * Q_TILE;
  static constexpr int OFF_RED = OFF_K + SC_STAGES * K_BYTES;
  // pass 1: per column group, per packed row: float max + double sum;
  // pass 2: two buffers of [M tile][lane quarter][64 keys] floats
  static constexpr int RED_BYTES = 4 * SC_PASS_ROWS * (4 + 8);
  static constexpr int OFF_BAR = OFF_RED + RED_BYTES;
  static constexpr int TOTAL = OFF_BAR + 256;
  static constexpr int ALLOC = TOTAL + 1024;
  static constexpr int HALF = D / 2;                     // d columns per partial accumulator
  static constexpr int KSTEPS = HALF / 16;               // MMA k-steps per partial
  static_assert(2 * SC_MAX_MT * 4 * SC_KEYS * 4 <= RED_BYTES, "pass-2 buffer");
};

enum : int { SB_QFULL = 0, SB_QEMPTY = 1, SB_FULL = 2, SB_EMPTY = SB_FULL + SC_STAGES,
             SB_SREADY = SB_EMPTY + SC_STAGES, SB_SFREE = SB_SREADY + SC_MAX_MT,
             SB_DRAIN = SB_SFREE + SC_MAX_MT, SB_COUNT = SB_DRAIN + 1 };

// Column sums of 16 values per lane over the warp's 32 rows: on entry lane l
// holds v[c] (c = 0..15) of its row; on exit lanes l and l^16 hold the sum
// over all 32 rows of column l & 15 (recursive halving, then one exchange).
__device__ __forceinline__ float warp_column_sums16(float (&v)[16], int lane) {
#pragma unroll
  for (int width = 8; width >= 1; width >>= 1) {
    const bool upper = (lane & width) != 0;
#pragma unroll
    for (int c = 0; c < width; ++c) {
      // keep the half of the columns this lane will own, send the other half
      const float send = upper ? v[c] : v[c + width];
      const float keep = upper ? v[c + width] : v[c];
      v[c] = keep + __shfl_xor_sync(0xffffffffu, send, width);
    }
  }
  return v[0] + __shfl_xor_sync(0xffffffffu, v[0], 16);
}

// kPass2 = false: row statistics of the CTA's key chunk (part_m, part_z);
// kPass2 = true: column sums into scores.  grid (n_chunks, B * Hkv * n_hg).
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
  const int bkg = blockIdx.y;                              // (b, KV head, head group)
  const int hgi = bkg % a.n_hg;
  const int bkv = bkg / a.n_hg;
  const int b = bkv / a.Hkv, kvh = bkv - b * a.Hkv;
  const int h0 = kvh * a.G + hgi * a.GH;                   // first query head of this CTA
  const int GHr = min(a.GH, a.G - hgi * a.GH);             // query heads of this CTA
  const int R = GHr * a.W32;                               // packed rows
  const int Lb = a.seqs.len(b);                            // this sequence's length
  const int wb = a.w < Lb ? a.w : Lb;                      // its window
  const int pos0 = Lb - wb;                                // position of window row 0
  const int key0 = chunk * a.chunk_tiles * SC_KEYS;
  int n_kt = Lb > key0 ? (Lb - key0 + SC_KEYS - 1) / SC_KEYS : 0;
  n_kt = n_kt > a.chunk_tiles ? a.chunk_tiles : n_kt;
  const int n_rp = a.n_rp, MT = a.MT;
  const int steps = n_rp * n_kt;

  auto bar = [&](int i) -> uint32_t { return base + C::OFF_BAR + 8u * static_cast<uint32_t>(i); };
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(gbase + C::OFF_BAR + 8 * SB_COUNT);
  volatile int* cta_abort = reinterpret_cast<volatile int*>(gbase + C::OFF_BAR + 8 * SB_COUNT + 4);
  if (threadIdx.x == 0) {
    mbar_init(bar(SB_QFULL), 1);
    mbar_init(bar(SB_QEMPTY), 1);
    for (int s = 0; s < SC_STAGES; ++s) {
      mbar_init(bar(SB_FULL + s), 1);
      mbar_init(bar(SB_EMPTY + s), 1);
    }
    for (int m = 0; m < SC_MAX_MT; ++m) {
      mbar_init(bar(SB_SREADY + m), 1);
      mbar_init(bar(SB_SFREE + m), SC_ROW_WARPS);
    }
    mbar_init(bar(SB_DRAIN), 1);
    *cta_abort = (a.abort_word && *reinterpret_cast<volatile uint32_t*>(a.abort_word)) ? 1 : 0;
    fence_mbar_init();
  }
  if (warp == SC_MMA_WARP) {
    tmem_alloc(smem_u32(tmem_holder), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const WaitCtl wc{cta_abort, a.status, a.abort_word, a.limit_ns};
  const bool run = (*cta_abort == 0) && steps > 0;

  if (!run) {
    // no keys in this chunk, or another CTA of this launch timed out
  } else if (warp == SC_LOAD_WARP) {
    // ------------------------------------------------------------ producer
    const bool leader = elect_one();
    const int bc = a.seqs.map_b(b);
    int issued = 0, q_issued = 0;
    bool go = true;
    for (int rp = 0; go && rp < n_rp; ++rp) {
      if (rp >= 1 && !__all_sync(0xffffffffu, mbar_wait(bar(SB_QEMPTY), (rp - 1) & 1, wc))) break;
      const int rows = min(SC_PASS_ROWS, R - rp * SC_PASS_ROWS);
      const int slots = (rows + SC_QBOX - 1) / SC_QBOX;
      if (leader) {
        mbar_arrive_expect_tx(bar(SB_QFULL), static_cast<uint32_t>(slots * SC_QBOX * D * 2));
        for (int s = 0; s < slots; ++s) {
          const int gr = rp * SC_PASS_ROWS + s * SC_QBOX;   // packed row of the slot
          const int hl = gr / a.W32, wr = gr - hl * a.W32;
          const uint32_t dst = base + (s >> 2) * C::Q_TILE + (s & 3) * (SC_QBOX * 128);
#pragma unroll
          for (int c = 0; c < C::NCH; ++c)
            tma_load_rows(dst + c * C::CHUNK, &tmQ, bar(SB_QFULL), a.token_major, c * 64,
                          a.seqs.map_t(b, pos0 + wr), h0 + hl, bc);
        }
      }
      q_issued = rp + 1;
      for (int kt = 0; kt < n_kt; ++kt) {
        const int n = rp * n_kt + kt;
        const int st = n % SC_STAGES, u = n / SC_STAGES;
        if (u >= 1 && !__all_sync(0xffffffffu, mbar_wait(bar(SB_EMPTY + st), (u - 1) & 1, wc))) {
          go = false;
          break;
        }
        if (leader) {
          const uint32_t sb = base + C::OFF_K + st * C::K_BYTES;
          mbar_arrive_expect_tx(bar(SB_FULL + st), C::K_BYTES);
          const int krow = a.seqs.map_t(b, key0 + kt * SC_KEYS);
#pragma unroll
          for (int c = 0; c < C::NCH; ++c)
            tma_load_rows(sb + c * C::K_CHUNK, &tmK, bar(SB_FULL + st), a.token_major, c * 64, krow, kvh, bc);
        }
        issued = n + 1;
      }
    }
    if (elect_one() && *cta_abort) {  // let every copy still in flight land before exit
      if (q_issued >= 1) mbar_wait_drain(bar(SB_QFULL), (q_issued - 1) & 1, 1000000000ull);
      for (int n = issued - SC_STAGES < 0 ? 0 : issued - SC_STAGES; n < issued; ++n)
        mbar_wait_drain(bar(SB_FULL + n % SC_STAGES), (n / SC_STAGES) & 1, 1000000000ull);
    }
  } else if (warp == SC_MMA_WARP) {
    // ------------------------------------------------------------ MMA issuer
    const bool leader = elect_one();
    constexpr uint32_t idS = idesc_bf16_f32(128, SC_KEYS, 0, 0);
    auto wait_all = [&](uint32_t br, uint32_t par) { return __all_sync(0xffffffffu, mbar_wait(br, par, wc)); };
    // test hook: phase 0 of the drain barrier completes only at teardown, so
    // this bounded wait runs out and the CTA takes the abort path
    bool ok = !(a.test_stall && !wait_all(bar(SB_DRAIN), 0));
    for (int rp = 0; ok && rp < n_rp; ++rp) {
      if (!(ok = wait_all(bar(SB_QFULL), rp & 1))) break;
      for (int kt = 0; ok && kt < n_kt; ++kt) {
        const int n = rp * n_kt + kt;
        const int st = n % SC_STAGES;
        if (!(ok = wait_all(bar(SB_FULL + st), (n / SC_STAGES) & 1))) break;
        const uint32_t ka = base + C::OFF_K + st * C::K_BYTES;
        for (int m = 0; m < MT; ++m) {
          if (n >= 1 && !(ok = wait_all(bar(SB_SFREE + m), (n - 1) & 1))) break;
          tc_fence_after();
          if (leader) {
            const uint32_t qa = base + m * C::Q_TILE;
#pragma unroll
            for (int p = 0; p < 2; ++p) {
#pragma unroll
              for (int k = 0; k < C::KSTEPS; ++k) {
                const int kk = p * C::KSTEPS + k;               // 16-column step of d
                const uint32_t qoff = (kk >> 2) * C::CHUNK + (kk & 3) * 32;
                const uint32_t koff = (kk >> 2) * C::K_CHUNK + (kk & 3) * 32;
                mma_bf16_ss(tmem + m * 128 + p * SC_KEYS, smem_desc(qa + qoff, 16, 1024, kSwizzle128B),
                            smem_desc(ka + koff, 16, 1024, kSwizzle128B), idS, k > 0 ? 1u : 0u);
              }
            }
            mma_commit(bar(SB_SREADY + m));
          }
        }
        if (!ok) break;
        if (leader) mma_commit(bar(SB_EMPTY + st));
      }
      if (ok && leader) mma_commit(bar(SB_QEMPTY));
    }
    if (leader) {
      mma_commit(bar(SB_DRAIN));
      mbar_wait_drain(bar(SB_DRAIN), 0, 1000000000ull);
    }
  } else {
    // ------------------------------------------------------------ rows
    const int lq = warp & 3;                        // TMEM lane quarter
    const int cg = warp >> 2;                       // key column group
    const uint32_t lane_off = static_cast<uint32_t>(lq * 32) << 16;
    const float sl2 = a.scale_log2;
    float* red = reinterpret_cast<float*>(gbase + C::OFF_RED);
    bool live = true;
    for (int rp = 0; live && rp < n_rp; ++rp) {
      // this thread's packed row in M tile m: rp*512 + m*128 + 32*lq + lane;
      // its head, position (or -1: padding or outside the window) and, in
      // the second pass, its (max, 1/sum) statistics
      float m_run[SC_MAX_MT];
      double z_run[SC_MAX_MT];
      float2 st_row[SC_MAX_MT];
      int pos_m[SC_MAX_MT];
#pragma unroll
      for (int m = 0; m < SC_MAX_MT; ++m) {
        m_run[m] = -INFINITY;
        z_run[m] = 0.0;
        st_row[m] = make_float2(0.f, 0.f);
        const int gr = rp * SC_PASS_ROWS + m * 128 + lq * 32 + lane;
        const int hl = gr / a.W32, wr = gr - hl * a.W32;
        const bool row_ok = m < MT && gr < R && wr < wb;
        pos_m[m] = row_ok ? pos0 + wr : -1;
        if constexpr (kPass2) {
          if (row_ok) st_row[m] = a.stats[(static_cast<size_t>(b) * a.Hq + h0 + hl) * a.w + wr];
        }
      }
      for (int kt = 0; live && kt < n_kt; ++kt) {
        const int n = rp * n_kt + kt;
        const int kbase = key0 + kt * SC_KEYS + cg * 16;   // this warp's first key
#pragma unroll
        for (int m = 0; m < SC_MAX_MT; ++m) {
          if (m >= MT) break;
          if (!(live = __all_sync(0xffffffffu, mbar_wait(bar(SB_SREADY + m), n & 1, wc)))) break;
          tc_fence_after();
          float x[16], xb[16];
          const uint32_t ta = tmem + lane_off + m * 128 + cg * 16;
          tmem_ld16(ta, x);
          tmem_ld16(ta + SC_KEYS, xb);
          tmem_ld_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(SB_SFREE + m));
          // logits: the two partial accumulators summed (packed pairs)
          uint64_t xs[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) xs[e] = f2_add(f2_pack(x[2 * e], x[2 * e + 1]), f2_pack(xb[2 * e], xb[2 * e + 1]));
          // every key of this thread's 16 is visible to its row (the common
          // case), or some are masked: past the row's position (causal) or
          // past the sequence (this only happens near the window)
          const int pos = pos_m[m];
          const bool full = kbase + 15 <= pos && kbase + 15 < Lb;
          if (!full) {
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              float v0, v1;
              f2_unpack(xs[e], v0, v1);
              const int k0 = kbase + 2 * e;
              v0 = (k0 <= pos && k0 < Lb) ? v0 : -INFINITY;
              v1 = (k0 + 1 <= pos && k0 + 1 < Lb) ? v1 : -INFINITY;
              xs[e] = f2_pack(v0, v1);
            }
          }
          if constexpr (!kPass2) {
            float mx = -INFINITY;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              float v0, v1;
              f2_unpack(xs[e], v0, v1);
              mx = fmax3(mx, v0, v1);
            }
            mx *= sl2;                                       // sl2 > 0: the max of the scaled logits
            if (mx != -INFINITY) {
              // lazy reference: keep m_run unless this tile's max passes it
              // by more than 2^8 (terms up to 256 are summed safely in fp32)
              if (mx > m_run[m] + 8.0f) {
                if (m_run[m] != -INFINITY) z_run[m] *= exp2(static_cast<double>(m_run[m]) - mx);
                m_run[m] = mx;
              }
              const uint64_t sl2x2 = f2_pack(sl2, sl2), nref = f2_pack(-m_run[m], -m_run[m]);
              uint64_t z2[2] = {0ull, 0ull};
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                float v0, v1;
                f2_unpack(f2_fma(xs[e], sl2x2, nref), v0, v1);
                z2[e & 1] = f2_add(z2[e & 1], f2_pack(ex2_approx(v0), ex2_approx(v1)));
              }
              float za, zb2, zc, zd;
              f2_unpack(z2[0], za, zb2);
              f2_unpack(z2[1], zc, zd);
              z_run[m] += static_cast<double>((za + zb2) + (zc + zd));
            }
          } else {
            const float2 sr = st_row[m];
            const uint64_t sl2x2 = f2_pack(sl2, sl2), nm = f2_pack(-sr.x, -sr.x), iz = f2_pack(sr.y, sr.y);
            float pv[16];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              float v0, v1;
              f2_unpack(f2_fma(xs[e], sl2x2, nm), v0, v1);
              // a masked logit is -inf, and ex2 of -inf is +0
              f2_unpack(f2_mul(f2_pack(ex2_approx(v0), ex2_approx(v1)), iz), pv[2 * e], pv[2 * e + 1]);
            }
            const float cs = warp_column_sums16(pv, lane);
            if (lane < 16) red[((n & 1) * SC_MAX_MT * 4 + m * 4 + lq) * SC_KEYS + cg * 16 + lane] = cs;
          }
        }
        if constexpr (kPass2) {
          // the row warps agree before going on, so the exchange below can
          // never leave one of them waiting alone
          if (!(live = bar_and(1, SC_ROW_WARPS * 32, live))) break;
          // per head: fixed-order sum over its 32-row slots of this pass
          const int r0 = rp * SC_PASS_ROWS, r1 = min(R, r0 + SC_PASS_ROWS);
          const int hfirst = r0 / a.W32, hlast = (r1 - 1) / a.W32;
          for (int t = threadIdx.x; t < (hlast - hfirst + 1) * SC_KEYS; t += SC_ROW_WARPS * 32) {
            const int hl = hfirst + t / SC_KEYS, col = t % SC_KEYS;
            const int s0 = (max(hl * a.W32, r0) - r0) / SC_QBOX;
            const int s1 = (min((hl + 1) * a.W32, r1) - r0) / SC_QBOX;
            float v = 0.f;
            for (int s = s0; s < s1; ++s) v += red[((n & 1) * SC_MAX_MT * 4 + s) * SC_KEYS + col];
            const int key = key0 + kt * SC_KEYS + col;
            if (key < Lb) {
              float* dst = a.scores + (static_cast<size_t>(b) * a.Hq + h0 + hl) * a.L + key;
              *dst = (hl * a.W32 >= r0) ? v : *dst + v;      // a head's later passes add to its first
            }
          }
        }
      }
      if constexpr (!kPass2) {
        // merge the four column groups of every row, then store its chunk stats
        float* mb = reinterpret_cast<float*>(gbase + C::OFF_RED);                          // [4][512]
        double* zb = reinterpret_cast<double*>(gbase + C::OFF_RED + 4 * SC_PASS_ROWS * 4);  // [4][512]
        if (!(live = bar_and(1, SC_ROW_WARPS * 32, live))) break;
#pragma unroll
        for (int m = 0; m < SC_MAX_MT; ++m) {
          const int r = m * 128 + lq * 32 + lane;
          mb[cg * SC_PASS_ROWS + r] = m_run[m];
          zb[cg * SC_PASS_ROWS + r] = z_run[m];
        }
        if (!(live = bar_and(1, SC_ROW_WARPS * 32, live))) break;
        for (int r = threadIdx.x; r < SC_MAX_MT * 128; r += SC_ROW_WARPS * 32) {
          const int gr = rp * SC_PASS_ROWS + r;
          const int hl = gr / a.W32, wr = gr - hl * a.W32;
          if (r >= MT * 128 || gr >= R || wr >= a.w) continue;
          float mm = -INFINITY;
#pragma unroll
          for (int c = 0; c < 4; ++c) mm = fmaxf(mm, mb[c * SC_PASS_ROWS + r]);
          double z = 0.0;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const float mc = mb[c * SC_PASS_ROWS + r];
            if (mc != -INFINITY) z += zb[c * SC_PASS_ROWS + r] * exp2(static_cast<double>(mc) - mm);
          }
          const size_t o = ((static_cast<size_t>(b) * a.Hq + h0 + hl) * a.w + wr) * a.n_chunks + chunk;
          a.part_m[o] = mm;
          a.part_z[o] = z;
        }
        if (!(live = bar_and(1, SC_ROW_WARPS * 32, live))) break;   // buffers free for the next pass
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == SC_MMA_WARP) {
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
