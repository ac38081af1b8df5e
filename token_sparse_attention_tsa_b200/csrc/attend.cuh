// attend.cuh -- causal attention on sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// Computes, for every valid row i of a head, o_i = sum_{j<=i} softmax_j(scale *
// q_i.k_j) v_j -- the ordinary dense causal attention that the Token Sparse
// Attention method runs on its compressed, contiguous Q/K/V tensors
// (gist.science summary page "Token Sparse Attention: Efficient Long-Context
// Inference with Interleaved Token Selection", section 2, "Arquitectura
// Central": the compressed tensors stay dense so an optimised dense kernel
// applies).  With the identity selection the same kernel is the dense
// baseline.
//
// Two 128-row query tiles of one head per CTA, warp-specialised (see the
// comment above attend2_kernel for the roles, TMEM plan and MMA order).
// Every wait is bounded (WaitCtl); a timeout sets the device status word,
// the CTA drains its in-flight copies/MMAs, frees TMEM and returns.
#pragma once

#include <cuda_bf16.h>

#include <type_traits>

#include "sm100.cuh"

namespace tsa {

struct AttnArgs {
  const int32_t* k_seq;   // valid rows per sequence (null: L)
  __nv_bfloat16* o;       // [B*Hq, L, D]
  float* lse;             // [B*Hq, L] or null
  uint32_t* status;       // device status word or null
  uint32_t* abort_word;   // launch-wide abort word (zeroed before launch) or null
  const int32_t* idx;     // gather mode: [B*Hq, L] selected rows (S_h ascending, then -1)
  int L;
  int Hq;
  int Hkv_map;            // heads of the K/V tensors
  int G_map;              // query heads per K/V head
  int n_tiles;            // ceil(L / 128)
  float scale_log2;       // softmax scale * log2(e)
  uint64_t limit_ns;      // per-wait time limit
  int test_stall;         // failure-path test: the MMA issuer first waits on a barrier nothing completes
};

// ---------------------------------------------------------------------------
// Two query tiles per CTA (rows [256c, 256c+256) of one head), ping-ponged,
// with PARTS softmax warpgroups per tile (each row's 128 S columns split in
// PARTS parts):
//   warps 0..4*PARTS-1          softmax of query tile 0 (warp w: rows
//                               32(w%4)..+32, part w/4)
//   warps 4*PARTS..8*PARTS-1    softmax of query tile 1 (same split)
//   warp 8*PARTS                TMEM allocator + MMA issuer
//   warp 8*PARTS+1              TMA producer
// PARTS = 1 is the configuration in use: one thread owns a whole row, holds
// its 128 S values in registers between the max and the exponentials, and
// needs no exchange.  With PARTS = 2 (18 warps, so at most 96 registers a
// thread) each row's max and sum are combined across its two halves through
// shared memory behind a named barrier of the tile's 256 threads that also
// ANDs the threads' progress flags, so both halves always take the same
// branch, and S is re-read from TMEM for the exponentials.
// TMEM: S0 [0,128), S1 [128,256), O0 [256,256+D), O1 [256+D, 256+2D).  Each
// part writes its P values (bf16, two per 32-bit column) over the first half
// of its own S columns, and the P.V MMA reads P from TMEM, so P never touches
// shared memory.  K and V
// tiles stream through one TMA ring of NSLOT slots in the order K0 V0 K1 V1 ...
// Per KV tile j the MMA warp issues S0_j, PV1_{j-1}, S1_j, PV0_j: while one
// tile's softmax runs the tensor core works on the other tile.  S0_{j+1}
// overwrites the columns P0_j is read from by PV0_j, issued just before it by
// the same thread; tcgen05.mma ops of one thread execute in issue order, so
// the read precedes the overwrite (the same reliance as the open CUTLASS
// sm100 attention mainloop).
template <int D, int PARTS>
struct Attn2Layout {
  static constexpr int BM = 128;
  static constexpr int BN = 128;
  static constexpr int SOFT_WARPS = 8 * PARTS;        // 4 warps per part per tile
  static constexpr int COLS = BN / PARTS;              // S columns per softmax thread
  static constexpr int THREADS = (SOFT_WARPS + 2) * 32;
  static constexpr int MMA_WARP = SOFT_WARPS;
  static constexpr int LOAD_WARP = SOFT_WARPS + 1;
  static constexpr int CHUNK = 128 * 128;            // 128 rows x 64 bf16 columns, SW128
  static constexpr int NCH = D / 64;
  static constexpr int TILE = 128 * D * 2;            // bytes of one Q, K or V tile
  static constexpr int NSLOT = D == 128 ? 4 : 9;      // K/V ring slots
  static constexpr int OFF_Q0 = 0;
  static constexpr int OFF_Q1 = TILE;
  static constexpr int OFF_RING = 2 * TILE;
  static constexpr int OFF_X = OFF_RING + NSLOT * TILE;        // row max / sum exchange
  static constexpr int X_BYTES = 2 * 2 * 2 * 128 * 4;          // [parity][tile][half][row]
  static constexpr int OFF_BAR = OFF_X + X_BYTES;
  static constexpr int TOTAL = OFF_BAR + 512;
  static constexpr int ALLOC = (TOTAL + 1024) > 120 * 1024 ? (TOTAL + 1024) : 120 * 1024;
  static constexpr int TMEM_COLS = 512;
  static constexpr int TMEM_O = 256;
  // barrier indices
  static constexpr int B_Q = 0;
  static constexpr int B_FULL = 1;                    // + slot
  static constexpr int B_EMPTY = 1 + NSLOT;           // + slot
  static constexpr int B_S = 1 + 2 * NSLOT;           // + tile (S ready)
  static constexpr int B_P = B_S + 2;                 // + tile (P written)
  static constexpr int B_PV = B_P + 2;                // + tile (P.V complete)
  static constexpr int B_DRAIN = B_PV + 2;
  static constexpr int B_COUNT = B_DRAIN + 1;
};

// kGather: Q, K and V rows are gathered by index (tile::gather4 from 2D maps
// over [heads * L, d] with one-row boxes) instead of read as contiguous
// compressed tiles.  (Each K/V tile is read by every later query tile of the
// head, so gathering in the kernel repeats the gather many times; one gather
// pass before the kernel is faster when compressed buffers can be held.)
// kScatter: output row i is written to row idx[i] of o (in place in the
// full-length output) instead of row i of a compressed output.
template <int D, int PARTS, bool kGather, bool kScatter>
__global__ void __launch_bounds__(Attn2Layout<D, PARTS>::THREADS, 1)
    attend2_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const AttnArgs a) {
  using C = Attn2Layout<D, PARTS>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int bh = blockIdx.y;
  const int b = bh / a.Hq;
  const int h = bh - b * a.Hq;
  const int n_pairs = (a.n_tiles + 1) >> 1;
  const int t0 = 2 * (n_pairs - 1 - static_cast<int>(blockIdx.x));  // longest pairs first

  int valid = a.k_seq ? a.k_seq[b] : a.L;
  valid = valid < 0 ? 0 : (valid > a.L ? a.L : valid);
  if (t0 * C::BM >= valid) return;                 // uniform, before any barrier
  const bool two = (t0 + 1) * C::BM < valid;       // second query tile has rows
  const int last0 = t0;                            // tile 0 attends KV tiles 0..t0
  const int n_kv = two ? t0 + 2 : t0 + 1;          // tile 1 attends 0..t0+1

  auto bar = [&](int i) -> uint32_t { return base + C::OFF_BAR + 8u * static_cast<uint32_t>(i); };
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(gbase + C::OFF_BAR + 8 * C::B_COUNT);
  volatile int* cta_abort = reinterpret_cast<volatile int*>(gbase + C::OFF_BAR + 8 * C::B_COUNT + 4);
  auto slot_of = [](int n) { return n % C::NSLOT; };
  auto use_of = [](int n) { return n / C::NSLOT; };
  auto ring = [&](int n) -> uint32_t { return base + C::OFF_RING + slot_of(n) * C::TILE; };

  if (threadIdx.x == 0) {
    mbar_init(bar(C::B_Q), 1);
    for (int s = 0; s < C::NSLOT; ++s) {
      mbar_init(bar(C::B_FULL + s), 1);
      mbar_init(bar(C::B_EMPTY + s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar(C::B_S + t), 1);
      mbar_init(bar(C::B_P + t), 4 * PARTS);      // one arrival per softmax warp
      mbar_init(bar(C::B_PV + t), 1);
    }
    mbar_init(bar(C::B_DRAIN), 1);
    *cta_abort = (a.abort_word && *reinterpret_cast<volatile uint32_t*>(a.abort_word)) ? 1 : 0;
    fence_mbar_init();
  }
  if (warp == C::MMA_WARP) {
    tmem_alloc(smem_u32(tmem_holder), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const WaitCtl wc{cta_abort, a.status, a.abort_word, a.limit_ns};
  const bool run = (*cta_abort == 0);

  if (warp == C::LOAD_WARP) {
    // ------------------------------------------------------------ producer
    // The whole warp runs the loop (uniform values); one elected lane issues.
    if (run) {
      const bool leader = elect_one();
      if (leader) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
      }
      const int zkv = b * a.Hkv_map + h / a.G_map;
      // One 128-row tile into dst: a box load, or 32 four-row gathers whose
      // row numbers come from idx (lane l reads entries 4l..4l+3; rows past
      // the selection read row 0 of the head, masked or zeroed downstream).
      auto load_tile = [&](auto by_index, uint32_t dst, const CUtensorMap* m, uint32_t br, int tile, int z) {
        if constexpr (!decltype(by_index)::value) {
          if (leader) {
#pragma unroll
            for (int c = 0; c < C::NCH; ++c) tma_load_3d(dst + c * C::CHUNK, m, br, c * 64, tile * C::BM, z);
          }
        } else {
          int rr[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int i = tile * C::BM + 4 * lane + u;
            const int v = i < valid ? __ldg(a.idx + static_cast<size_t>(bh) * a.L + i) : 0;
            rr[u] = z * a.L + (v >= 0 && v < a.L ? v : 0);
          }
#pragma unroll 4
          for (int g = 0; g < 32; ++g) {
            const int r0 = __shfl_sync(0xffffffffu, rr[0], g), r1 = __shfl_sync(0xffffffffu, rr[1], g);
            const int r2 = __shfl_sync(0xffffffffu, rr[2], g), r3 = __shfl_sync(0xffffffffu, rr[3], g);
            if (leader) {
#pragma unroll
              for (int c = 0; c < C::NCH; ++c) tma_gather4(dst + c * C::CHUNK + g * 512, m, br, c * 64, r0, r1, r2, r3);
            }
          }
        }
      };
      if (leader) mbar_arrive_expect_tx(bar(C::B_Q), (two ? 2 : 1) * C::TILE);
      __syncwarp();
      constexpr std::integral_constant<bool, kGather> q_by_index{};
      constexpr std::integral_constant<bool, kGather> kv_by_index{};
      load_tile(q_by_index, base + C::OFF_Q0, &tmQ, bar(C::B_Q), t0, bh);
      if (two) load_tile(q_by_index, base + C::OFF_Q1, &tmQ, bar(C::B_Q), t0 + 1, bh);
      int issued = 0;
      for (int n = 0; n < 2 * n_kv; ++n) {
        const int s = slot_of(n), u = use_of(n);
        if (u >= 1 && !__all_sync(0xffffffffu, mbar_wait(bar(C::B_EMPTY + s), (u - 1) & 1, wc))) break;
        if (leader) mbar_arrive_expect_tx(bar(C::B_FULL + s), C::TILE);
        __syncwarp();
        load_tile(kv_by_index, ring(n), (n & 1) ? &tmV : &tmK, bar(C::B_FULL + s), n >> 1, zkv);
        issued = n + 1;
      }
      if (leader && *cta_abort) {  // let every copy still in flight land before exit
        mbar_wait_drain(bar(C::B_Q), 0, 1000000000ull);
        for (int n = issued - C::NSLOT < 0 ? 0 : issued - C::NSLOT; n < issued; ++n)
          mbar_wait_drain(bar(C::B_FULL + slot_of(n)), use_of(n) & 1, 1000000000ull);
      }
    }
  } else if (warp == C::MMA_WARP) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the loop so loop state and descriptors are uniform;
    // one elected lane issues every MMA and commit.  Descriptors are built
    // once; a k-step only adds its byte offset >> 4 to the start-address
    // field (shared-memory addresses stay below 2^18, so the field never
    // carries over).
    if (run) {
      const bool leader = elect_one();
      constexpr uint32_t idS = idesc_bf16_f32(128, C::BN, 0, 0);
      constexpr uint32_t idO = idesc_bf16_f32(128, D, 0, 1);
      const uint64_t dq0 = smem_desc(base + C::OFF_Q0, 16, 1024, kSwizzle128B);
      const uint64_t dq1 = smem_desc(base + C::OFF_Q1, 16, 1024, kSwizzle128B);
      const uint64_t dk0 = smem_desc(base + C::OFF_RING, 16, 1024, kSwizzle128B);
      const uint64_t dv0 = smem_desc(base + C::OFF_RING, C::CHUNK, 1024, kSwizzle128B);
      auto issue_s = [&](int t, int j) {
        const uint64_t dq = t ? dq1 : dq0;
        const uint64_t dk = dk0 + static_cast<uint64_t>((slot_of(2 * j) * C::TILE) >> 4);
        if (leader) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t off = static_cast<uint64_t>(((kk >> 2) * C::CHUNK + (kk & 3) * 32) >> 4);
            mma_bf16_ss(tmem + t * 128, dq + off, dk + off, idS, kk > 0 ? 1u : 0u);
          }
          mma_commit(bar(C::B_S + t));
        }
      };
      auto issue_pv = [&](int t, int j) {
        const uint64_t dv = dv0 + static_cast<uint64_t>((slot_of(2 * j + 1) * C::TILE) >> 4);
        if (leader) {
#pragma unroll
          for (int kk = 0; kk < C::BN / 16; ++kk) {
            // P of keys [16kk, 16kk+16): part p = 16kk / COLS holds them from
            // column p*COLS, two keys per column.
            const uint32_t pcol = (16 * kk / C::COLS) * C::COLS + (16 * kk % C::COLS) / 2;
            mma_bf16_ts(tmem + C::TMEM_O + t * D, tmem + t * 128 + pcol,
                        dv + static_cast<uint64_t>((kk * 2048) >> 4), idO, (j > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(bar(C::B_PV + t));
        }
      };
      auto commit_to = [&](uint32_t br) {
        if (leader) mma_commit(br);
      };
      auto wait_all = [&](uint32_t br, uint32_t par) {
        return __all_sync(0xffffffffu, mbar_wait(br, par, wc));
      };
      auto full = [&](int n) { return wait_all(bar(C::B_FULL + slot_of(n)), use_of(n) & 1); };
      // test hook: phase 0 of the drain barrier completes only at teardown,
      // so this bounded wait runs out and takes the abort path
      // The waits for K_{j+1} and V_j come before the wait for P0_j: those
      // tiles have normally landed long before, and once P0_j arrives PV0_j
      // and S0_{j+1} go out back to back.  Every slot these loads need was
      // released by a commit issued earlier in this loop, so waiting for them
      // here cannot deadlock the ring.
      bool ok = !(a.test_stall && !wait_all(bar(C::B_DRAIN), 0)) && wait_all(bar(C::B_Q), 0) && full(0);
      for (int j = 0; ok && j < n_kv; ++j) {
        tc_fence_after();                                                // K_j has landed
        if (j <= last0) issue_s(0, j);
        if (two && j >= 1) {
          if (!(ok = wait_all(bar(C::B_P + 1), (j - 1) & 1))) break;
          tc_fence_after();
          issue_pv(1, j - 1);
          commit_to(bar(C::B_EMPTY + slot_of(2 * j - 1)));               // V_{j-1} done
        }
        if (two) issue_s(1, j);
        commit_to(bar(C::B_EMPTY + slot_of(2 * j)));                     // K_j done
        const bool more = j + 1 < n_kv;
        if (j <= last0) {
          if (!(ok = full(2 * j + 1))) break;                            // V_j
          if (more && !(ok = full(2 * j + 2))) break;                    // K_{j+1}
          if (!(ok = wait_all(bar(C::B_P + 0), j & 1))) break;
          tc_fence_after();
          issue_pv(0, j);
          if (!two) commit_to(bar(C::B_EMPTY + slot_of(2 * j + 1)));
        } else if (more && !(ok = full(2 * j + 2))) {
          break;
        }
      }
      if (ok && two) {
        const int j = n_kv - 1;
        if (wait_all(bar(C::B_P + 1), j & 1) && full(2 * j + 1)) {
          tc_fence_after();
          issue_pv(1, j);
          commit_to(bar(C::B_EMPTY + slot_of(2 * j + 1)));
        }
      }
      commit_to(bar(C::B_DRAIN));
      if (leader) mbar_wait_drain(bar(C::B_DRAIN), 0, 1000000000ull);
    }
  } else if (run && (warp < C::SOFT_WARPS / 2 || two)) {
    // ------------------------------------------------------------ softmax
    const int tt = warp / (4 * PARTS);           // query tile of this warp
    const int half = (warp >> 2) % PARTS;        // columns [COLS*half, COLS*half+COLS)
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;                // row within the tile
    const int tile = t0 + tt;
    const int row = tile * C::BM + r;
    const int last = tile;                       // its diagonal KV tile
    const bool last_active = tt == (two ? 1 : 0);
    const uint32_t named = 1 + tt;               // named barrier of the tile's 256 threads
    const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
    const uint32_t s_col = tmem + lane_off + tt * 128 + half * C::COLS;
    const uint32_t p_col = s_col;                // P over the first COLS/2 of the part's columns
    const uint32_t o_col = tmem + lane_off + C::TMEM_O + tt * D + half * (D / PARTS);
    float* xch = reinterpret_cast<float*>(gbase + C::OFF_X);   // [parity][tile][half][row]
    auto xidx = [&](int par, int hf) { return ((par * 2 + tt) * 2 + hf) * 128 + r; };
    const float sl2 = a.scale_log2;
    float m_used = -INFINITY;
    float l = 0.f;                               // this half's share of the row sum
    bool live = true;
    for (int j = 0; j <= last; ++j) {
      live = live && __all_sync(0xffffffffu, mbar_wait(bar(C::B_S + tt), j & 1, wc));
      float mh = -INFINITY;
      const bool diag = (j == last);
      constexpr int NC = C::COLS / 32;
      float sv[NC][32];
      if (live) {  // pass 1: this part's row max
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < NC; ++c) tmem_ld32(s_col + c * 32, sv[c]);
        tmem_ld_wait();
        if (diag) {  // causal mask, only on the diagonal tile
#pragma unroll
          for (int c = 0; c < NC; ++c)
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if ((half * C::COLS + c * 32 + e) > r) sv[c][e] = -INFINITY;
        }
        // row max: four chains of three-input maxima over value pairs
        float m4[4] = {sv[0][0], sv[0][1], sv[0][2], sv[0][3]};
#pragma unroll
        for (int i = 4; i < C::COLS; i += 2) {       // i even: i, i+1 lie in one 32-chunk
          const int u = (i >> 1) & 3;
          m4[u] = fmax3(m4[u], sv[i >> 5][i & 31], sv[i >> 5][(i & 31) + 1]);
        }
        mh = fmaxf(fmax3(m4[0], m4[1], m4[2]), m4[3]);
      }
      float mx = mh;
      if constexpr (PARTS == 2) {
        xch[xidx(j & 1, half)] = mh;
        live = bar_and(named, 256, live);        // both halves agree to go on
        if (!live) continue;                     // keep the barrier count uniform
        mx = fmaxf(mh, xch[xidx(j & 1, half ^ 1)]);
      } else {
        if (!live) continue;
      }
      const float m_new = fmaxf(m_used, mx * sl2);
      const bool resc = m_new > m_used + 8.0f;   // lazy rescale (factor <= 2^8 tolerated)
      const float alpha = resc ? ex2_approx(m_used - m_new) : 1.f;
      if (resc) m_used = m_new;
      const float nm = -m_used;
      const uint64_t sl2x2 = f2_pack(sl2, sl2), nmx2 = f2_pack(nm, nm);
      uint64_t r4[4];                               // packed partial row sums
#pragma unroll
      for (int u = 0; u < 4; ++u) r4[u] = 0ull;
      // pass 2: S columns [32c, 32c+32) of the part give P columns
      // [16c, 16c+16), which lie in columns already read.  A thread that
      // owns a whole row still holds its S values from pass 1; with the row
      // split in parts the register budget only allows re-reading them.
#pragma unroll
      for (int c = 0; c < NC; ++c) {
        float (&s32)[32] = sv[c];
        if constexpr (PARTS > 1) {
          tmem_ld32(s_col + c * 32, s32);
          tmem_ld_wait();
          if (diag) {
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if ((half * C::COLS + c * 32 + e) > r) s32[e] = -INFINITY;
          }
        }
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          float x0, x1;
          f2_unpack(f2_fma(f2_pack(s32[2 * e], s32[2 * e + 1]), sl2x2, nmx2), x0, x1);
          const float p0 = ex2_approx(x0);
          const float p1 = ex2_approx(x1);
          r4[e & 3] = f2_add(r4[e & 3], f2_pack(p0, p1));
          pk[e] = pack_bf16x2(p0, p1);
        }
        tmem_st16u(p_col + c * 16, pk);
      }
      float rs[8];
#pragma unroll
      for (int u = 0; u < 4; ++u) f2_unpack(r4[u], rs[2 * u], rs[2 * u + 1]);
      l = l * alpha + (((rs[0] + rs[1]) + (rs[2] + rs[3])) + ((rs[4] + rs[5]) + (rs[6] + rs[7])));
      // O is rescaled only when a row's max grew past the lazy threshold, and
      // then only once the previous P.V into O has completed (and before this
      // tile's P.V, which waits for P_FULL).  Otherwise the wait is skipped:
      // P.V MMAs into one accumulator run in issue order.  The PV barrier can
      // never be two phases ahead here (P.V j needs this tile's P first), so a
      // parity wait after skipped ones still names the right phase.
      if (j > 0 && __any_sync(0xffffffffu, resc)) {
        live = __all_sync(0xffffffffu, mbar_wait(bar(C::B_PV + tt), (j - 1) & 1, wc));
        if (live) {
          tc_fence_after();
          {
#pragma unroll
            for (int c = 0; c < D / PARTS / 32; ++c) {
              float ov[32];
              tmem_ld32(o_col + c * 32, ov);
              tmem_ld_wait();
#pragma unroll
              for (int e = 0; e < 32; ++e) ov[e] *= alpha;
              tmem_st32(o_col + c * 32, ov);
            }
          }
        }
      }
      // Rows of the KV tile that holds `valid` may carry any bits beyond it;
      // their P weights are 0 but 0 * NaN would poison O, so zero them.
      if (live && half == 0 && diag && last_active && (j * C::BN + C::BN > valid)) {
        const int n = 2 * j + 1;
        live = __all_sync(0xffffffffu, mbar_wait(bar(C::B_FULL + slot_of(n)), use_of(n) & 1, wc));
        if (live && j * C::BN + r >= valid) {
#pragma unroll
          for (int c = 0; c < C::NCH; ++c) {
            uint4* vrow = reinterpret_cast<uint4*>(gbase + C::OFF_RING + slot_of(n) * C::TILE + c * C::CHUNK + r * 128);
#pragma unroll
            for (int e = 0; e < 8; ++e) vrow[e] = make_uint4(0, 0, 0, 0);
          }
        }
        fence_proxy_async_smem();
      }
      if (live) {
        // the warp's TMEM stores (and V zeroing) are complete; one lane
        // arrives for the warp
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(C::B_P + tt));
      }
    }
    // ------------------------------------------------------------ epilogue
    live = live && __all_sync(0xffffffffu, mbar_wait(bar(C::B_PV + tt), last & 1, wc));
    float lt = l;
    if constexpr (PARTS == 2) {
      xch[xidx(0, half)] = l;  // parity-0 slots are free: every read of them is behind us
      live = bar_and(named, 256, live);
      if (live) lt = l + xch[xidx(0, half ^ 1)];
    }
    if (live) {
      tc_fence_after();
      const float inv_l = 1.f / lt;
      int orow_index = row;
      bool store = row < valid;
      if constexpr (kScatter) {  // compressed row i goes to token S_h[i]
        orow_index = store ? __ldg(a.idx + static_cast<size_t>(bh) * a.L + row) : 0;
        if (store && (orow_index < 0 || orow_index >= a.L)) {
          store = false;
          if (a.status) atomicOr(a.status, 0x4u);
        }
      }
      __nv_bfloat16* orow = a.o + (static_cast<size_t>(bh) * a.L + (store ? orow_index : 0)) * D + half * (D / PARTS);
#pragma unroll
      for (int c = 0; c < D / PARTS / 32; ++c) {
        float ov[32];
        tmem_ld32(o_col + c * 32, ov);
        tmem_ld_wait();
        if (store) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            uint4 pk;
            pk.x = pack_bf16x2(ov[g * 8 + 0] * inv_l, ov[g * 8 + 1] * inv_l);
            pk.y = pack_bf16x2(ov[g * 8 + 2] * inv_l, ov[g * 8 + 3] * inv_l);
            pk.z = pack_bf16x2(ov[g * 8 + 4] * inv_l, ov[g * 8 + 5] * inv_l);
            pk.w = pack_bf16x2(ov[g * 8 + 6] * inv_l, ov[g * 8 + 7] * inv_l);
            dst[g] = pk;
          }
        }
      }
      if (a.lse && half == 0 && row < valid)
        a.lse[static_cast<size_t>(bh) * a.L + row] = (m_used + __log2f(lt)) * 0.69314718055994531f;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == C::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace tsa
