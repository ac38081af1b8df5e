// copy.cuh -- gather of Q/K/V into compressed tensors and scatter of the
// compressed output back to full length.
//
// Source: gist.science summary page "Token Sparse Attention: Efficient
// Long-Context Inference with Interleaved Token Selection", section 2,
// "Arquitectura Central": compression gathers each head's selected rows of
// Q, K and V into dense, contiguous tensors; decompression places each row of
// the compressed output back at its token position in an output that is zero
// everywhere else.
//
// Both kernels are pure HBM traffic: each row (d bf16 = 128 or 256 bytes) is
// moved by d/8 lanes with one 16-byte load and store per lane, so a warp moves
// whole rows with full 32-byte sectors.
#pragma once

#include <cuda_bf16.h>

#include "sm100.cuh"

namespace tsa {

struct GatherArgs {
  const __nv_bfloat16 *q, *k, *v;  // q: B x Hq heads, k, v: B x Hkv heads of L rows of D
  RowStrides qs, kvs;              // their row strides (head-major or token-major)
  const int32_t* idx;              // [B*Hq, L]
  Kept kept;                       // rows kept per (b, h)
  Seqs seqs;                       // sequence lengths L_b
  __nv_bfloat16 *qc, *kc, *vc;     // [B*Hq, L, D]; qc may be null (K and V only)
  uint32_t* status;                // or null
  int B, L, Hq, Hkv, G;
};

constexpr int GT_ROWS = 32;        // compressed rows per gather work item (per query head)

// Work item: (sequence b, KV head g, GT_ROWS compressed rows i) for all G
// query heads of the group, rows visited with the query head fastest: the
// G heads copy their i-th selected rows back to back.  Their selections
// ascend and overlap heavily, so the K and V rows they read are close
// together and come from L2 after the first head's read: each K/V row
// crosses HBM about once per group rather than once per query head.  Index
// arithmetic is 32-bit and done once per item; each thread keeps two rows'
// loads in flight.
template <int D>
__global__ void __launch_bounds__(256, 4) gather_kernel(const GatherArgs a) {
  constexpr int LPR = D / 8;       // lanes per row
  constexpr int RPP = 256 / LPR;   // rows per pass of the CTA
  const int sub = threadIdx.x % LPR;
  const int slot = threadIdx.x / LPR;
  const int tiles = (a.L + GT_ROWS - 1) / GT_ROWS;
  const int items = a.B * a.Hkv * tiles;
  const int per_item = GT_ROWS * a.G;
  bool bad = false;
  for (int w = blockIdx.x; w < items; w += gridDim.x) {
    const int bg = w / tiles, tile = w - bg * tiles;
    const int b = bg / a.Hkv, g = bg - b * a.Hkv;
    const int Lb = a.seqs.len(b);
    const int i0 = tile * GT_ROWS;
    if (i0 >= Lb) continue;
    for (int r0 = slot; r0 < per_item; r0 += 2 * RPP) {
      int h[2], i[2], j[2];
      bool live[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int r = r0 + u * RPP;
        const int di = r / a.G;
        i[u] = i0 + di;
        h[u] = g * a.G + (r - di * a.G);
        live[u] = r < per_item && i[u] < a.kept.of(b, h[u], Lb);
        j[u] = live[u] ? __ldg(a.idx + (static_cast<size_t>(b) * a.Hq + h[u]) * a.L + i[u]) : 0;
      }
      uint4 vq[2], vk[2], vv[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        vq[u] = vk[u] = vv[u] = make_uint4(0, 0, 0, 0);
        const bool ok = j[u] >= 0 && j[u] < Lb;
        bad |= live[u] && !ok;           // a bad index: a zero row, reported
        if (live[u] && ok) {
          const size_t skv = a.kvs.at(b, g, j[u]) + sub * 8;
          vk[u] = __ldg(reinterpret_cast<const uint4*>(a.k + skv));
          vv[u] = __ldg(reinterpret_cast<const uint4*>(a.v + skv));
          if (a.qc) vq[u] = __ldg(reinterpret_cast<const uint4*>(a.q + a.qs.at(b, h[u], j[u]) + sub * 8));
        }
      }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        if (live[u]) {
          const size_t dst = ((static_cast<size_t>(b) * a.Hq + h[u]) * a.L + i[u]) * D + sub * 8;
          if (a.qc) *reinterpret_cast<uint4*>(a.qc + dst) = vq[u];
          *reinterpret_cast<uint4*>(a.kc + dst) = vk[u];
          *reinterpret_cast<uint4*>(a.vc + dst) = vv[u];
        }
      }
    }
  }
  if (bad && a.status) atomicOr(a.status, 0x4u);
}

struct ScatterArgs {
  const __nv_bfloat16* oc;  // [B*Hq, L, D] compressed (head-major)
  const int32_t* idx;       // [B*Hq, L]
  Kept kept;                // rows kept per (b, h)
  __nv_bfloat16* o;         // B x Hq heads of L rows of D
  RowStrides os;            // row strides of o (head-major or token-major)
  uint32_t* status;         // or null
  int L, Hq;
  Seqs seqs;                // sequence lengths L_b: rows [0, L_b) of o are written
};

constexpr int SCAT_ROWS = 256;  // output rows per CTA

// grid (ceil(L/256), B*Hq), 256 threads.  The CTA maps its 256 output rows to
// compressed positions through a shared table built from the ascending idx
// (one binary search for the first entry), then writes every row once.
// kZeroOnly: write only the unselected rows (zeros) and leave the selected
// ones, which the attention epilogue has already written in place.
template <int D, bool kZeroOnly = false>
__global__ void __launch_bounds__(256) scatter_kernel(const ScatterArgs a) {
  constexpr int LPR = D / 8;
  __shared__ int32_t where[SCAT_ROWS];
  __shared__ int32_t s_first;
  const int bh = blockIdx.y;
  const int r0 = blockIdx.x * SCAT_ROWS;
  const int b = bh / a.Hq;
  const int Lb = a.seqs.len(b);
  const int kb = a.kept.of(b, bh - b * a.Hq, Lb);
  const int32_t* ix = a.idx + static_cast<size_t>(bh) * a.L;
  where[threadIdx.x] = -1;
  if (threadIdx.x == 0) {  // first i with ix[i] >= r0
    int lo = 0, hi = kb;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (__ldg(ix + mid) < r0) lo = mid + 1; else hi = mid;
    }
    s_first = lo;
  }
  __syncthreads();
  bool bad = false;
  {
    // an entry outside [0, L_b), or one not above its predecessor (idx must
    // ascend strictly for the binary search above), is reported, not written
    const int i = s_first + threadIdx.x;
    if (i < kb) {
      const int j = __ldg(ix + i);
      const int r = j - r0;
      if (j < 0 || j >= Lb || (i > 0 && __ldg(ix + i - 1) >= j)) bad = true;
      else if (r >= 0 && r < SCAT_ROWS) where[r] = i;
    }
  }
  __syncthreads();
  const int sub = threadIdx.x % LPR;
  constexpr int ROWS_PER_PASS = 256 / LPR;
  for (int rr = threadIdx.x / LPR; rr < SCAT_ROWS; rr += ROWS_PER_PASS) {
    const int r = r0 + rr;
    if (r >= Lb) break;
    const int i = where[rr];
    if (kZeroOnly && i >= 0) continue;
    uint4 val = make_uint4(0, 0, 0, 0);
    if (!kZeroOnly && i >= 0)
      val = __ldg(reinterpret_cast<const uint4*>(a.oc + (static_cast<size_t>(bh) * a.L + i) * D + sub * 8));
    __stcs(reinterpret_cast<uint4*>(a.o + a.os.at(b, bh - b * a.Hq, r) + sub * 8), val);
  }
  if (bad && a.status) atomicOr(a.status, 0x4u);
}

}  // namespace tsa
