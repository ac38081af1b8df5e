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
// One CTA computes one 128-row query tile of one head.  Warp roles:
//   warp 0      TMA producer: Q tile once, then K/V tiles into a 2-stage ring
//   warp 1      TMEM allocator and single-thread tcgen05.mma issuer
//   warps 2..5  softmax: one thread per query row (TMEM lane), online softmax
//               with lazy rescaling, P written to shared memory as bf16,
//               epilogue normalises O and stores it.
// TMEM columns: S double buffer [0,128) and [128,256), O [256, 256+D).
// S = Q K^T and O += P V are kind::f16 MMAs (bf16 in, fp32 accumulate),
// M = 128, operands in 128-byte-swizzled shared memory.
//
// Every wait is bounded (WaitCtl); a timeout sets the device status word,
// the CTA drains its in-flight copies/MMAs, frees TMEM and returns.
#pragma once

#include <cuda_bf16.h>

#include "sm100.cuh"

namespace tsa {

template <int D>
struct AttnLayout {
  static constexpr int BM = 128;                 // query rows per CTA
  static constexpr int BN = 128;                 // keys per KV tile
  static constexpr int NS = 2;                   // K/V pipeline stages
  static constexpr int CHUNK = 128 * 128;        // one 128-row x 64-col bf16 SW128 block
  static constexpr int NCH = D / 64;             // 64-column chunks of a row
  static constexpr int Q_BYTES = BM * D * 2;
  static constexpr int KV_BYTES = BN * D * 2;
  static constexpr int P_BYTES = BM * BN * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + NS * KV_BYTES;
  static constexpr int OFF_P = OFF_V + NS * KV_BYTES;
  static constexpr int OFF_BAR = OFF_P + P_BYTES;
  static constexpr int TOTAL = OFF_BAR + 256;
  // +1 KiB for aligning the base to 1024 B; padded so only one CTA fits per
  // SM (each CTA allocates all 512 TMEM columns).
  static constexpr int ALLOC = (TOTAL + 1024) > 120 * 1024 ? (TOTAL + 1024) : 120 * 1024;
  static constexpr int TMEM_COLS = 512;
  static constexpr int TMEM_O = 256;
};

struct AttnArgs {
  const int32_t* k_seq;   // valid rows per sequence (null: L)
  __nv_bfloat16* o;       // [B*Hq, L, D]
  float* lse;             // [B*Hq, L] or null
  uint32_t* status;       // device status word or null
  uint32_t* abort_word;   // launch-wide abort word (zeroed before launch) or null
  int L;
  int Hq;
  int Hkv_map;            // heads of the K/V tensors
  int G_map;              // query heads per K/V head
  int n_tiles;            // ceil(L / 128)
  float scale_log2;       // softmax scale * log2(e)
  uint64_t limit_ns;      // per-wait time limit
};

enum : int {
  BAR_Q = 0,
  BAR_KFULL = 1,   // +stage
  BAR_VFULL = 3,   // +stage
  BAR_KVEMPTY = 5, // +stage
  BAR_SFULL = 7,   // +buffer
  BAR_SFREE = 9,   // +buffer
  BAR_PFULL = 11,
  BAR_PVDONE = 12,
  BAR_DRAIN = 13,
  BAR_COUNT = 14
};

template <int D>
__global__ void __launch_bounds__(192, 1)
    attend_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const AttnArgs a) {
  using C = AttnLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int bh = blockIdx.y;
  const int b = bh / a.Hq;
  const int h = bh - b * a.Hq;
  const int t = a.n_tiles - 1 - static_cast<int>(blockIdx.x);  // longest tiles first

  int valid = a.k_seq ? a.k_seq[b] : a.L;
  valid = valid < 0 ? 0 : (valid > a.L ? a.L : valid);
  if (t * C::BM >= valid) return;  // uniform over the CTA, before any barrier
  const int n_kv = t + 1;           // causal: KV tiles 0..t

  auto bar = [&](int i) -> uint32_t { return base + C::OFF_BAR + 8u * static_cast<uint32_t>(i); };
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(gbase + C::OFF_BAR + 8 * BAR_COUNT);
  volatile int* cta_abort = reinterpret_cast<volatile int*>(gbase + C::OFF_BAR + 8 * BAR_COUNT + 4);

  if (threadIdx.x == 0) {
    mbar_init(bar(BAR_Q), 1);
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(bar(BAR_KFULL + s), 1);
      mbar_init(bar(BAR_VFULL + s), 1);
      mbar_init(bar(BAR_KVEMPTY + s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(BAR_SFULL + s), 1);
      mbar_init(bar(BAR_SFREE + s), 128);
    }
    mbar_init(bar(BAR_PFULL), 128);
    mbar_init(bar(BAR_PVDONE), 1);
    mbar_init(bar(BAR_DRAIN), 1);
    // another CTA of this launch already timed out: skip the work (still
    // tear down cleanly)
    *cta_abort = (a.abort_word && *reinterpret_cast<volatile uint32_t*>(a.abort_word)) ? 1 : 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const WaitCtl wc{cta_abort, a.status, a.abort_word, a.limit_ns};
  const bool run = (*cta_abort == 0);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && run) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      const int zq = bh;
      const int zkv = b * a.Hkv_map + h / a.G_map;
      mbar_arrive_expect_tx(bar(BAR_Q), C::Q_BYTES);
#pragma unroll
      for (int c = 0; c < C::NCH; ++c)
        tma_load_3d(base + C::OFF_Q + c * C::CHUNK, &tmQ, bar(BAR_Q), c * 64, t * C::BM, zq);
      int issued = 0;
      for (int j = 0; j < n_kv; ++j) {
        const int s = j % C::NS;
        const int n = j / C::NS;
        if (j >= C::NS && !mbar_wait(bar(BAR_KVEMPTY + s), (n - 1) & 1, wc)) break;
        mbar_arrive_expect_tx(bar(BAR_KFULL + s), C::KV_BYTES);
#pragma unroll
        for (int c = 0; c < C::NCH; ++c)
          tma_load_3d(base + C::OFF_K + s * C::KV_BYTES + c * C::CHUNK, &tmK, bar(BAR_KFULL + s),
                      c * 64, j * C::BN, zkv);
        mbar_arrive_expect_tx(bar(BAR_VFULL + s), C::KV_BYTES);
#pragma unroll
        for (int c = 0; c < C::NCH; ++c)
          tma_load_3d(base + C::OFF_V + s * C::KV_BYTES + c * C::CHUNK, &tmV, bar(BAR_VFULL + s),
                      c * 64, j * C::BN, zkv);
        issued = j + 1;
      }
      if (*cta_abort) {  // let every copy still in flight land before exit
        mbar_wait_drain(bar(BAR_Q), 0, 1000000000ull);
        for (int j = issued - C::NS < 0 ? 0 : issued - C::NS; j < issued; ++j) {
          mbar_wait_drain(bar(BAR_KFULL + j % C::NS), (j / C::NS) & 1, 1000000000ull);
          mbar_wait_drain(bar(BAR_VFULL + j % C::NS), (j / C::NS) & 1, 1000000000ull);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && run) {
      constexpr uint32_t idS = idesc_bf16_f32(128, C::BN, 0, 0);
      constexpr uint32_t idO = idesc_bf16_f32(128, D, 0, 1);
      bool ok = mbar_wait(bar(BAR_Q), 0, wc);
      for (int j = 0; ok && j <= n_kv; ++j) {
        if (j < n_kv) {
          const int sb = j & 1;
          const int s = j % C::NS;
          if (j >= 2 && !(ok = mbar_wait(bar(BAR_SFREE + sb), ((j >> 1) - 1) & 1, wc))) break;
          if (!(ok = mbar_wait(bar(BAR_KFULL + s), (j / C::NS) & 1, wc))) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * C::CHUNK + (kk & 3) * 32;
            mma_bf16_ss(tmem + sb * 128, smem_desc(base + C::OFF_Q + off, 16, 1024, kSwizzle128B),
                        smem_desc(base + C::OFF_K + s * C::KV_BYTES + off, 16, 1024, kSwizzle128B),
                        idS, kk > 0 ? 1u : 0u);
          }
          mma_commit(bar(BAR_SFULL + sb));
        }
        if (j >= 1) {
          const int jj = j - 1;
          const int s = jj % C::NS;
          if (!(ok = mbar_wait(bar(BAR_PFULL), jj & 1, wc))) break;
          if (!(ok = mbar_wait(bar(BAR_VFULL + s), (jj / C::NS) & 1, wc))) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < C::BN / 16; ++kk) {
            const uint32_t pa = (kk >> 2) * C::CHUNK + (kk & 3) * 32;
            mma_bf16_ss(tmem + C::TMEM_O, smem_desc(base + C::OFF_P + pa, 16, 1024, kSwizzle128B),
                        smem_desc(base + C::OFF_V + s * C::KV_BYTES + kk * 2048, C::CHUNK, 1024,
                                  kSwizzle128B),
                        idO, (jj > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(bar(BAR_PVDONE));
          mma_commit(bar(BAR_KVEMPTY + s));
        }
      }
      // all issued MMAs complete before TMEM is released
      mma_commit(bar(BAR_DRAIN));
      mbar_wait_drain(bar(BAR_DRAIN), 0, 1000000000ull);
    }
  } else if (run) {
    // ------------------------------------------------------------ softmax
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;                       // row within the tile
    const int row = t * C::BM + r;                      // compressed row index
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const float sl2 = a.scale_log2;
    float m_used = -INFINITY;                           // running max (log2 units)
    float l = 0.f;
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      const int sb = j & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(bar(BAR_SFULL + sb), (j >> 1) & 1, wc));
      if (!ok) break;
      tc_fence_after();
      float sv[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(lane_base + sb * 128 + c * 32, sv[c]);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(bar(BAR_SFREE + sb));

      const bool diag = (j == n_kv - 1);
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          if (diag && (c * 32 + e) > r) sv[c][e] = -INFINITY;
          mx = fmaxf(mx, sv[c][e]);
        }
      const float m_new = fmaxf(m_used, mx * sl2);
      const bool resc = m_new > m_used + 8.0f;         // lazy rescale (factor <= 2^8 tolerated)

      if (j > 0) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar(BAR_PVDONE), (j - 1) & 1, wc));
        if (!ok) break;
        tc_fence_after();
        if (__any_sync(0xffffffffu, resc)) {
          const float alpha = resc ? ex2_approx(m_used - m_new) : 1.f;
          l *= alpha;
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            float ov[32];
            tmem_ld32(lane_base + C::TMEM_O + c * 32, ov);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) ov[e] *= alpha;
            tmem_st32(lane_base + C::TMEM_O + c * 32, ov);
          }
          tmem_st_wait();
        }
      }
      if (resc) m_used = m_new;

      // P = exp2(s * scale_log2 - m_used) in bf16, row r of a K-major SW128 tile
      const float nm = -m_used;
      float rs = 0.f;
      uint8_t* prow = gbase + C::OFF_P + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          float pv[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            pv[e] = ex2_approx(fmaf(sv[c][g * 8 + e], sl2, nm));
            rs += pv[e];
          }
          const int ch = c * 4 + g;                     // 16-byte chunk 0..15 of the row
          const int blk = ch >> 3;                      // 64-column block
          const int cc = (ch & 7) ^ (r & 7);            // 128B swizzle
          uint4 pk;
          pk.x = pack_bf16x2(pv[0], pv[1]);
          pk.y = pack_bf16x2(pv[2], pv[3]);
          pk.z = pack_bf16x2(pv[4], pv[5]);
          pk.w = pack_bf16x2(pv[6], pv[7]);
          *reinterpret_cast<uint4*>(prow + blk * C::CHUNK + cc * 16) = pk;
        }
      }
      l += rs;

      // Rows of the last KV tile at or beyond `valid` may hold any bits; their
      // P weights are 0 but 0 * NaN would poison O, so zero them in smem.
      if (diag && (j * C::BN + C::BN > valid)) {
        const int s = j % C::NS;
        ok = __all_sync(0xffffffffu, mbar_wait(bar(BAR_VFULL + s), (j / C::NS) & 1, wc));
        if (!ok) break;
        if (j * C::BN + r >= valid) {
#pragma unroll
          for (int c = 0; c < C::NCH; ++c) {
            uint4* vrow = reinterpret_cast<uint4*>(gbase + C::OFF_V + s * C::KV_BYTES + c * C::CHUNK + r * 128);
#pragma unroll
            for (int e = 0; e < 8; ++e) vrow[e] = make_uint4(0, 0, 0, 0);
          }
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar(BAR_PFULL));
    }

    // ------------------------------------------------------------ epilogue
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(BAR_PVDONE), (n_kv - 1) & 1, wc));
    if (ok) {
      tc_fence_after();
      const float inv_l = 1.f / l;
      __nv_bfloat16* orow = a.o + (static_cast<size_t>(bh) * a.L + row) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        float ov[32];
        tmem_ld32(lane_base + C::TMEM_O + c * 32, ov);
        tmem_ld_wait();
        if (row < valid) {
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
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace tsa
