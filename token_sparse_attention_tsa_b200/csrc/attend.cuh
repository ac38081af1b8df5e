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

// Pairs e (of the 16 value pairs of each 32-column chunk of a softmax row)
// whose two exponentials are computed by exp2_poly_x2 on the FMA pipe; the
// others use ex2.approx on the MUFU unit.  The split balances the two units.
#ifndef TSA_P_SPLITS
#define TSA_P_SPLITS 2
#endif

#ifndef TSA_EXP_EMU_PAIRS
#define TSA_EXP_EMU_PAIRS 0x0000u
#endif
constexpr uint32_t kExpEmuPairs = TSA_EXP_EMU_PAIRS;

struct AttnArgs {
  Kept kept;              // valid rows per (b, h) (null counts: L)
  __nv_bfloat16* o;       // B x Hq heads of L rows of D
  RowStrides os;          // row strides of o
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
  int token_major;        // Q/K/V maps are (d, H, L, B) (else (d, L, H, B)); gather rows likewise
  int in_packed;          // Q/K/V are packed sequences (token coordinate cu[b] + t, one map "sequence")
  Seqs seqs;              // sequence lengths L_b (and packed token offsets)
  const uint8_t* block_mask;  // [B*Hq, n_tiles, n_tiles] or null: query tile i may attend key tile j
                              // (j < i) only where the entry is nonzero; diagonal tiles always
};

// ---------------------------------------------------------------------------
// Two query tiles per CTA (rows [256c, 256c+256) of one head), ping-ponged:
//   warps 0..3   softmax of query tile 0 (warp w: rows 32w..32w+31, one
//                thread per row, all 128 S columns of its row)
//   warps 4..7   softmax of query tile 1 (same split)
//   warp 8       TMEM allocator + MMA issuer
//   warp 9       TMA producer
// TMEM: S0 [0,128), S1 [128,256), O0 [256,256+D), O1 [256+D, 256+2D).  A
// softmax thread reads its 128 S values into registers once, takes the row
// max, and writes its P values (bf16, two per 32-bit column) over the first
// 64 of its tile's S columns; the P.V MMA reads P from TMEM, so P never
// touches shared memory.  P is released to the MMA warp in P_SPLITS column
// groups (one barrier each), so the first k-steps of P.V run while the
// softmax still computes the later columns.  K and V
// tiles stream through one TMA ring of NSLOT slots in the order K0 V0 K1 V1 ...
// Per KV tile j the MMA warp issues S0_j, PV1_{j-1}, S1_j, PV0_j: while one
// tile's softmax runs the tensor core works on the other tile.  S0_{j+1}
// overwrites the columns P0_j is read from by PV0_j, issued just before it by
// the same thread; tcgen05.mma ops of one thread execute in issue order, so
// the read precedes the overwrite (the same reliance as the open CUTLASS
// sm100 attention mainloop).
template <int D>
struct Attn2Layout {
  static constexpr int BM = 128;
  static constexpr int BN = 128;
  static constexpr int SOFT_WARPS = 8;
  static constexpr int THREADS = (SOFT_WARPS + 2) * 32;
  static constexpr int MMA_WARP = SOFT_WARPS;
  static constexpr int LOAD_WARP = SOFT_WARPS + 1;
  static constexpr int CHUNK = 128 * 128;            // 128 rows x 64 bf16 columns, SW128
  static constexpr int NCH = D / 64;
  static constexpr int TILE = 128 * D * 2;            // bytes of one Q, K or V tile
  static constexpr int NSLOT = D == 128 ? 4 : 9;      // K/V ring slots
  static constexpr int P_SPLITS = TSA_P_SPLITS;       // P released in this many column groups
  static constexpr int KSTEPS = BN / 16;              // P.V k-steps per KV tile
  static constexpr int OFF_Q0 = 0;
  static constexpr int OFF_Q1 = TILE;
  static constexpr int OFF_RING = 2 * TILE;
  static constexpr int OFF_BAR = OFF_RING + NSLOT * TILE;
  static constexpr int OFF_PROC = OFF_BAR + 512;      // bit j: KV tile j is processed (block masks)
  static constexpr int MAX_TILES = 32768;             // L <= 2^22 tokens
  static constexpr int TOTAL = OFF_PROC + MAX_TILES / 8;
  static constexpr int ALLOC = (TOTAL + 1024) > 120 * 1024 ? (TOTAL + 1024) : 120 * 1024;
  static constexpr int TMEM_COLS = 512;
  static constexpr int TMEM_O = 256;
  // barrier indices
  static constexpr int B_Q = 0;
  static constexpr int B_FULL = 1;                    // + slot
  static constexpr int B_EMPTY = 1 + NSLOT;           // + slot
  static constexpr int B_S = 1 + 2 * NSLOT;           // + tile (S ready)
  static constexpr int B_P = B_S + 2;                 // + tile * P_SPLITS + group (P written)
  static constexpr int B_PV = B_P + 2 * P_SPLITS;     // + tile (P.V complete)
  static constexpr int B_DRAIN = B_PV + 2;
  static constexpr int B_COUNT = B_DRAIN + 1;
  static_assert(8 * B_COUNT + 8 <= 512, "barrier area");
  static_assert(KSTEPS % P_SPLITS == 0 && (BN / 32) % P_SPLITS == 0, "P groups");
};

// kGather: Q, K and V rows are gathered by index (tile::gather4 from 2D maps
// over [heads * L, d] with one-row boxes) instead of read as contiguous
// compressed tiles.  (Each K/V tile is read by every later query tile of the
// head, so gathering in the kernel repeats the gather many times; one gather
// pass before the kernel is faster when compressed buffers can be held.)
// kScatter: output row i is written to row idx[i] of o (in place in the
// full-length output) instead of row i of a compressed output.
// kBlocks: KV tiles are filtered by the block mask (without it every tile
// in the causal range is processed and the checks compile away).
template <int D, bool kGather, bool kScatter, bool kBlocks = false>
__global__ void __launch_bounds__(Attn2Layout<D>::THREADS, 1)
    attend2_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const AttnArgs a) {
  using C = Attn2Layout<D>;
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

  const int seq_len = a.seqs.len(b);
  const int valid = a.kept.of(b, h, seq_len);
  if (t0 * C::BM >= valid) return;                 // uniform, before any barrier
  const bool two = (t0 + 1) * C::BM < valid;       // second query tile has rows
  const int last0 = t0;                            // tile 0 attends KV tiles 0..t0
  const int n_kv = two ? t0 + 2 : t0 + 1;          // tile 1 attends 0..t0+1

  // KV tiles this CTA processes: those one of its query tiles attends (its
  // causal range, the diagonal always, earlier tiles where the block mask
  // allows).  Producer, MMA issuer and softmax walk the same list; barrier
  // phases and ring slots count processed tiles, not j.
  const uint8_t* bmask = kBlocks ? a.block_mask + static_cast<size_t>(bh) * a.n_tiles * a.n_tiles : nullptr;
  auto needs = [&](int qt, int j) {
    if constexpr (kBlocks) return j <= qt && (j == qt || __ldg(bmask + static_cast<size_t>(qt) * a.n_tiles + j) != 0);
    return j <= qt;
  };
  // With a block mask the CTA's processed tiles are computed once into a
  // shared bitmask (below); next_proc(j) is the first processed tile >= j
  // (n_kv when none is left).  Without one every tile is processed.
  const uint32_t* proc_bits = reinterpret_cast<const uint32_t*>(gbase + C::OFF_PROC);
  auto next_proc = [&](int j) -> int {
    if constexpr (kBlocks) {
      while (j < n_kv) {
        const uint32_t w = proc_bits[j >> 5] >> (j & 31);
        if (w) return j + __ffs(static_cast<int>(w)) - 1;
        j = (j | 31) + 1;
      }
      return n_kv;
    }
    return j;
  };

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
      for (int g = 0; g < C::P_SPLITS; ++g) mbar_init(bar(C::B_P + t * C::P_SPLITS + g), 4);  // one arrival per warp
      mbar_init(bar(C::B_PV + t), 1);
    }
    mbar_init(bar(C::B_DRAIN), 1);
    *cta_abort = (a.abort_word && *reinterpret_cast<volatile uint32_t*>(a.abort_word)) ? 1 : 0;
    fence_mbar_init();
  }
  if constexpr (kBlocks) {  // processed tiles: one of the pair's query tiles attends them
    uint32_t* bits = reinterpret_cast<uint32_t*>(gbase + C::OFF_PROC);
    for (int w = warp; w * 32 < n_kv; w += C::THREADS / 32) {
      const int j = w * 32 + lane;
      const bool pj = j < n_kv && (needs(t0, j) || (two && needs(t0 + 1, j)));
      const uint32_t word = __ballot_sync(0xffffffffu, pj);
      if (lane == 0) bits[w] = word;
    }
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
      const bool tm = a.token_major != 0;
      // One 128-row tile of head hz (of the map's nh heads) of sequence b
      // into dst: a box load, or 32 four-row gathers whose row numbers come
      // from idx (lane l reads entries 4l..4l+3; rows past the selection read
      // token 0 of the head, masked or zeroed downstream).
      auto load_tile = [&](auto by_index, uint32_t dst, const CUtensorMap* m, uint32_t br, int tile, int hz,
                           int nh) {
        if constexpr (!decltype(by_index)::value) {
          if (leader) {
#pragma unroll
            for (int c = 0; c < C::NCH; ++c)
              tma_load_rows(dst + c * C::CHUNK, m, br, tm, c * 64, a.in_packed ? a.seqs.map_t(b, tile * C::BM) : tile * C::BM,
                            hz, a.in_packed ? 0 : b);
          }
        } else {
          int rr[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int i = tile * C::BM + 4 * lane + u;
            int v = i < valid ? __ldg(a.idx + static_cast<size_t>(bh) * a.L + i) : 0;
            v = (v >= 0 && v < seq_len) ? v : 0;
            const int tok = a.in_packed ? a.seqs.tok0(b) + v : b * a.L + v;
            rr[u] = tm ? tok * nh + hz : (b * nh + hz) * a.L + v;
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
      load_tile(q_by_index, base + C::OFF_Q0, &tmQ, bar(C::B_Q), t0, h, a.Hq);
      if (two) load_tile(q_by_index, base + C::OFF_Q1, &tmQ, bar(C::B_Q), t0 + 1, h, a.Hq);
      int issued = 0;
      bool go = true;
      for (int j = next_proc(0), cb = 0; go && j < n_kv; j = next_proc(j + 1)) {
        const int c = kBlocks ? cb++ : j;      // processed-tile count (j itself without a mask)
        for (int kv = 0; kv < 2; ++kv) {        // K_j, V_j into ring positions 2c, 2c+1
          const int n = 2 * c + kv;
          const int s = slot_of(n), u = use_of(n);
          if (u >= 1 && !__all_sync(0xffffffffu, mbar_wait(bar(C::B_EMPTY + s), (u - 1) & 1, wc))) {
            go = false;
            break;
          }
          if (leader) mbar_arrive_expect_tx(bar(C::B_FULL + s), C::TILE);
          __syncwarp();
          load_tile(kv_by_index, ring(n), kv ? &tmV : &tmK, bar(C::B_FULL + s), j, h / a.G_map, a.Hkv_map);
          issued = n + 1;
        }
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
      auto issue_s = [&](int t, int c) {         // c: processed-tile count of the KV tile
        const uint64_t dq = t ? dq1 : dq0;
        const uint64_t dk = dk0 + static_cast<uint64_t>((slot_of(2 * c) * C::TILE) >> 4);
        if (leader) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t off = static_cast<uint64_t>(((kk >> 2) * C::CHUNK + (kk & 3) * 32) >> 4);
            mma_bf16_ss(tmem + t * 128, dq + off, dk + off, idS, kk > 0 ? 1u : 0u);
          }
          mma_commit(bar(C::B_S + t));
        }
      };
      auto commit_to = [&](uint32_t br) {
        if (leader) mma_commit(br);
      };
      auto wait_all = [&](uint32_t br, uint32_t par) {
        return __all_sync(0xffffffffu, mbar_wait(br, par, wc));
      };
      auto full = [&](int n) { return wait_all(bar(C::B_FULL + slot_of(n)), use_of(n) & 1); };
      // O_t += P_t,j V_j, one group of k-steps per released P group.  P of
      // keys [16kk, 16kk+16) sits in TMEM column 8kk of the tile's S columns.
      auto issue_pv = [&](int t, int c) -> bool {
        const uint64_t dv = dv0 + static_cast<uint64_t>((slot_of(2 * c + 1) * C::TILE) >> 4);
        constexpr int KPG = C::KSTEPS / C::P_SPLITS;
#pragma unroll
        for (int g = 0; g < C::P_SPLITS; ++g) {
          if (!wait_all(bar(C::B_P + t * C::P_SPLITS + g), c & 1)) return false;
          tc_fence_after();
          if (leader) {
#pragma unroll
            for (int kk = g * KPG; kk < (g + 1) * KPG; ++kk)
              mma_bf16_ts(tmem + C::TMEM_O + t * D, tmem + t * 128 + 8 * kk,
                          dv + static_cast<uint64_t>((kk * 2048) >> 4), idO, (c > 0 || kk > 0) ? 1u : 0u);
          }
        }
        commit_to(bar(C::B_PV + t));
        return true;
      };
      // The waits for K_{j+1} and V_j come before the P waits of PV0_j: those
      // tiles have normally landed long before, and once P0_j is released
      // PV0_j and S0_{j+1} go out back to back.  Every slot these loads need
      // was released by a commit issued earlier in this loop, so waiting for
      // them here cannot deadlock the ring.
      // test hook: phase 0 of the drain barrier completes only at teardown,
      // so this bounded wait runs out and takes the abort path
      int n_proc = n_kv;
      if constexpr (kBlocks) {
        n_proc = 0;
        for (int w = 0; w * 32 < n_kv; ++w) n_proc += __popc(proc_bits[w]);   // >= 1: tile 0's diagonal
      }
      bool ok = !(a.test_stall && !wait_all(bar(C::B_DRAIN), 0)) && wait_all(bar(C::B_Q), 0) && full(0);
      for (int j = next_proc(0), cb = 0; ok && j < n_kv; j = next_proc(j + 1)) {
        const int c = kBlocks ? cb++ : j;        // processed-tile count (j itself without a mask)
        tc_fence_after();                                                // K of tile c has landed
        if (j <= last0) issue_s(0, c);
        if (two && c >= 1) {
          if (!(ok = issue_pv(1, c - 1))) break;
          commit_to(bar(C::B_EMPTY + slot_of(2 * c - 1)));               // V of tile c-1 done
        }
        if (two) issue_s(1, c);
        commit_to(bar(C::B_EMPTY + slot_of(2 * c)));                     // K of tile c done
        const bool more = c + 1 < n_proc;
        if (j <= last0) {
          if (!(ok = full(2 * c + 1))) break;                            // V of tile c
          if (more && !(ok = full(2 * c + 2))) break;                    // K of tile c+1
          if (!(ok = issue_pv(0, c))) break;
          if (!two) commit_to(bar(C::B_EMPTY + slot_of(2 * c + 1)));
        } else if (more && !(ok = full(2 * c + 2))) {
          break;
        }
      }
      if (ok && two) {
        const int c = n_proc - 1;
        if (full(2 * c + 1) && issue_pv(1, c)) commit_to(bar(C::B_EMPTY + slot_of(2 * c + 1)));
      }
      commit_to(bar(C::B_DRAIN));
      if (leader) mbar_wait_drain(bar(C::B_DRAIN), 0, 1000000000ull);
    }
  } else if (run && warp < C::SOFT_WARPS && (warp < 4 || two)) {
    // ------------------------------------------------------------ softmax
    const int tt = warp >> 2;                    // query tile of this warp
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;                // row within the tile
    const int tile = t0 + tt;
    const int row = tile * C::BM + r;
    const int last = tile;                       // its diagonal KV tile
    const bool last_active = tt == (two ? 1 : 0);
    const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
    const uint32_t s_col = tmem + lane_off + tt * 128;
    const uint32_t o_col = tmem + lane_off + C::TMEM_O + tt * D;
    const float sl2 = a.scale_log2;
    float m_used = -INFINITY;
    float l = 0.f;
    bool live = true;
    int pc = -1;                                 // processed-tile count of the current KV tile
    for (int j = next_proc(0); j <= last; j = next_proc(j + 1)) {
      pc = kBlocks ? pc + 1 : j;
      if (!(live = __all_sync(0xffffffffu, mbar_wait(bar(C::B_S + tt), pc & 1, wc)))) break;
      tc_fence_after();
      if (kBlocks && !needs(tile, j)) {
        // a tile only the other query tile attends: P = 0 (S is not read)
        uint32_t z[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) z[e] = 0u;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) tmem_st16u(s_col + cc * 16, z);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
#pragma unroll
          for (int g = 0; g < C::P_SPLITS; ++g) mbar_arrive(bar(C::B_P + tt * C::P_SPLITS + g));
        }
        continue;
      }
      const bool diag = (j == last);
      float sv[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(s_col + c * 32, sv[c]);
      tmem_ld_wait();
      if (diag) {  // causal mask, only on the diagonal tile
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (c * 32 + e > r) sv[c][e] = -INFINITY;
      }
      // row max: eight chains of three-input maxima over value pairs
      float m8[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) m8[u] = sv[0][u];
#pragma unroll
      for (int i = 8; i < C::BN; i += 2) {       // i even: i, i+1 lie in one 32-chunk
        const int u = (i >> 1) & 7;
        m8[u] = fmax3(m8[u], sv[i >> 5][i & 31], sv[i >> 5][(i & 31) + 1]);
      }
      const float mx = fmax3(fmax3(m8[0], m8[1], m8[2]), fmax3(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7]));
      const float m_new = fmaxf(m_used, mx * sl2);
      const bool resc = m_new > m_used + 8.0f;   // lazy rescale (factor <= 2^8 tolerated)
      const float alpha = resc ? ex2_approx(m_used - m_new) : 1.f;
      if (resc) m_used = m_new;
      const float nm = -m_used;
      const uint64_t sl2x2 = f2_pack(sl2, sl2), nmx2 = f2_pack(nm, nm);
      uint64_t r4[4];                               // packed partial row sums
#pragma unroll
      for (int u = 0; u < 4; ++u) r4[u] = 0ull;
      // S columns [32c, 32c+32) give P columns [16c, 16c+16); every S value
      // is already in registers, so P may overwrite any S column.  The plain
      // kernel stores a group's P (its two chunks, 32 columns) in one go; the
      // scatter and block-mask variants (more registers live) chunk by chunk.
      constexpr int CPG = 4 / C::P_SPLITS;          // 32-column chunks per P group
      constexpr bool kWide = !kScatter && !kBlocks && CPG == 2;
#pragma unroll
      for (int g = 0; g < C::P_SPLITS; ++g) {
        uint32_t pk32[32];
#pragma unroll
        for (int cc = 0; cc < CPG; ++cc) {
          const int c = g * CPG + cc;
          uint32_t (&pk)[16] = *reinterpret_cast<uint32_t(*)[16]>(&pk32[kWide ? cc * 16 : 0]);
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const uint64_t xx = f2_fma(f2_pack(sv[c][2 * e], sv[c][2 * e + 1]), sl2x2, nmx2);
            float p0, p1;
            if ((kExpEmuPairs >> e) & 1u) {            // this pair on the FMA pipe
              exp2_poly_x2(xx, p0, p1);
            } else {                                   // this pair on the MUFU unit
              float x0, x1;
              f2_unpack(xx, x0, x1);
              p0 = ex2_approx(x0);
              p1 = ex2_approx(x1);
            }
            r4[e & 3] = f2_add(r4[e & 3], f2_pack(p0, p1));
            pk[e] = pack_bf16x2(p0, p1);
          }
          if constexpr (!kWide) tmem_st16u(s_col + c * 16, pk);
        }
        if constexpr (kWide) tmem_st32(s_col + g * 32, *reinterpret_cast<float(*)[32]>(pk32));
        if (g == 0) {
          // Before the first P group is released: O is rescaled when a
          // row's max grew past the lazy threshold, and V rows past `valid`
          // are zeroed (those rows may carry any bits; their P weights are 0
          // but 0 * NaN would poison O).  P.V j-1 has completed by now, as
          // S_j was committed after it, so the PV wait returns at once; the
          // PV barrier can never be two phases ahead here because P.V j
          // needs this tile's P first, so a parity wait after skipped ones
          // still names the right phase.
          if (pc > 0 && __any_sync(0xffffffffu, resc)) {
            if (!(live = __all_sync(0xffffffffu, mbar_wait(bar(C::B_PV + tt), (pc - 1) & 1, wc)))) break;
            tc_fence_after();
            if constexpr (C::P_SPLITS == 2) {
#pragma unroll
              for (int c = 0; c < D / 32; ++c) {
                float ov[32];
                tmem_ld32(o_col + c * 32, ov);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 32; ++e) ov[e] *= alpha;
                tmem_st32(o_col + c * 32, ov);
              }
            } else {  // more S values still live at group 0: 16 columns at a time
#pragma unroll
              for (int c = 0; c < D / 16; ++c) {
                float ov[16];
                tmem_ld16(o_col + c * 16, ov);
                tmem_ld_wait();
                uint32_t ou[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) ou[e] = __float_as_uint(ov[e] * alpha);
                tmem_st16u(o_col + c * 16, ou);
              }
            }
          }
          if (diag && last_active && (j * C::BN + C::BN > valid)) {
            const int n = 2 * pc + 1;                // ring position of this tile's V
            if (!(live = __all_sync(0xffffffffu, mbar_wait(bar(C::B_FULL + slot_of(n)), use_of(n) & 1, wc)))) break;
            if (j * C::BN + r >= valid) {
#pragma unroll
              for (int c = 0; c < C::NCH; ++c) {
                uint4* vrow = reinterpret_cast<uint4*>(gbase + C::OFF_RING + slot_of(n) * C::TILE + c * C::CHUNK + r * 128);
#pragma unroll
                for (int e = 0; e < 8; ++e) vrow[e] = make_uint4(0, 0, 0, 0);
              }
            }
            fence_proxy_async_smem();
          }
        }
        // the warp's TMEM stores (O rescale, P) and V zeroing are complete;
        // one lane arrives for the warp
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(C::B_P + tt * C::P_SPLITS + g));
      }
      if (!live) break;                            // a wait above ran out
      float rs[8];
#pragma unroll
      for (int u = 0; u < 4; ++u) f2_unpack(r4[u], rs[2 * u], rs[2 * u + 1]);
      l = l * alpha + (((rs[0] + rs[1]) + (rs[2] + rs[3])) + ((rs[4] + rs[5]) + (rs[6] + rs[7])));
    }
    // ------------------------------------------------------------ epilogue
    live = live && __all_sync(0xffffffffu, mbar_wait(bar(C::B_PV + tt), pc & 1, wc));
    if (live) {
      tc_fence_after();
      const float inv_l = 1.f / l;
      int orow_index = row;
      bool store = row < valid;
      if constexpr (kScatter) {  // compressed row i goes to token S_h[i]
        orow_index = store ? __ldg(a.idx + static_cast<size_t>(bh) * a.L + row) : 0;
        if (store && (orow_index < 0 || orow_index >= seq_len)) {
          store = false;
          if (a.status) atomicOr(a.status, 0x4u);
        }
      }
      __nv_bfloat16* orow = a.o + a.os.at(b, h, store ? orow_index : 0);
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
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
      if (a.lse && row < valid)
        a.lse[static_cast<size_t>(bh) * a.L + row] = (m_used + __log2f(l)) * 0.69314718055994531f;
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
