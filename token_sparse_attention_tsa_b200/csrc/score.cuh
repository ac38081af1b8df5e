// score.cuh -- proxy importance scores of the Token Sparse Attention method.
//
// Source: gist.science summary page "Token Sparse Attention: Efficient
// Long-Context Inference with Interleaved Token Selection", section 2,
// "Cobertura Dinamica de Tokens", scoring: a light attention map of the most
// recent queries against all keys; a key's importance is the sum of its
// column of attention weights.
//
// Here: for each (b, h) and window row i in [L-w, L), x_ij = scale *
// q[b,h,i].k[b,h/G,j] over keys j <= i; p_ij = softmax_j(x_ij);
// score[b,h,j] = sum_i p_ij.
//
// Two passes over the keys, both tiled 128 window rows x 128 keys with the
// dot products on the fp32 FMA pipe (each bf16 product is exact in fp32 and
// every FMA rounds once, which keeps the scores within ~1e-6 relative of the
// fp64 definition; the window is short, so this stage is small next to the
// attention):
//   pass 1  per key chunk: row max m_c and sum Z_c = sum_j exp(x_ij - m_c),
//           tile sums accumulated in fp64
//   merge   per row: m = max_c m_c, Z = sum_c Z_c exp(m_c - m) (fp64)
//   pass 2  per key tile: score_j = sum_i exp(x_ij - m_i) / Z_i
// Scratch (workspace): partial (m, Z) per (head, row, chunk) and the merged
// (m, 1/Z) per (head, row).
#pragma once

#include <cuda_bf16.h>

namespace tsa {

constexpr int SC_ROWS = 128;     // window rows per block
constexpr int SC_KEYS = 128;     // keys per tile
constexpr int SC_CHUNK_TILES = 8;  // key tiles per pass-1 CTA
constexpr int SC_THREADS = 256;

struct ScoreArgs {
  const __nv_bfloat16* q;  // [B*Hq, L, D]
  const __nv_bfloat16* k;  // [B*Hkv, L, D]
  float* scores;           // [B*Hq, L]
  float* part_m;           // [B*Hq, w, n_chunks] chunk row max m_c
  double* part_z;          // [B*Hq, w, n_chunks] chunk row sum Z_c (fp64)
  float2* stats;           // [B*Hq, w] (m, 1/Z)
  int L, w, Hq, Hkv, G;
  int n_chunks;
  float scale;
};

// Load a [rows x D] bf16 block (rows starting at row0 of a head) into shared
// memory as fp32, transposed to [D][128] so a thread reads 4 consecutive rows
// of one dimension with one 16-byte load.  Rows outside [0, nrows) read 0.
template <int D>
__device__ __forceinline__ void load_block_t(float* dst, const __nv_bfloat16* src, int row0,
                                             int nrows) {
  // each thread converts 8 consecutive elements (16 bytes) of one row;
  // consecutive threads take consecutive rows so the transposed shared
  // stores fall in distinct banks
  for (int e = threadIdx.x; e < 128 * (D / 8); e += SC_THREADS) {
    const int r = e & 127;
    const int c8 = (e >> 7) * 8;
    const int gr = row0 + r;
    uint4 raw = make_uint4(0, 0, 0, 0);
    if (gr >= 0 && gr < nrows) raw = *reinterpret_cast<const uint4*>(src + static_cast<size_t>(gr) * D + c8);
    const uint32_t w4[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      dst[(c8 + 2 * u) * 128 + r] = __uint_as_float(w4[u] << 16);
      dst[(c8 + 2 * u + 1) * 128 + r] = __uint_as_float(w4[u] & 0xFFFF0000u);
    }
  }
}

// 8 rows x 8 keys of scale * q.k per thread.  Thread (ty, tx) = (tid/16,
// tid%16) owns rows ty*8..+7 and keys tx*4..+3, 64+tx*4..+3 of the tile.
template <int D>
__device__ __forceinline__ void tile_dots(const float* sQ, const float* sK, float (&acc)[8][8]) {
  const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
#pragma unroll 4
  for (int d = 0; d < D; ++d) {
    const float4 qa = *reinterpret_cast<const float4*>(sQ + d * 128 + ty * 8);
    const float4 qb = *reinterpret_cast<const float4*>(sQ + d * 128 + ty * 8 + 4);
    const float4 ka = *reinterpret_cast<const float4*>(sK + d * 128 + tx * 4);
    const float4 kb = *reinterpret_cast<const float4*>(sK + d * 128 + 64 + tx * 4);
    const float qv[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
    const float kv[8] = {ka.x, ka.y, ka.z, ka.w, kb.x, kb.y, kb.z, kb.w};
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(qv[i], kv[j], acc[i][j]);
  }
}

__device__ __forceinline__ int tile_key(int tx, int j) { return j < 4 ? tx * 4 + j : 64 + tx * 4 + (j - 4); }

// Pass 1: grid (n_chunks, B*Hq).  One CTA: all window rows (in blocks of
// 128) against SC_CHUNK_TILES key tiles.
template <int D>
__global__ void __launch_bounds__(SC_THREADS, 1) score_stats_kernel(const ScoreArgs a) {
  extern __shared__ float sm[];
  float* sQ = sm;              // [D][128]
  float* sK = sm + D * 128;    // [D][128]
  const int chunk = blockIdx.x;
  const int bh = blockIdx.y;
  const int b = bh / a.Hq, h = bh % a.Hq;
  const __nv_bfloat16* qh = a.q + static_cast<size_t>(bh) * a.L * D;
  const __nv_bfloat16* kh = a.k + (static_cast<size_t>(b) * a.Hkv + h / a.G) * a.L * D;
  const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
  const int key0 = chunk * SC_CHUNK_TILES * SC_KEYS;

  for (int rb = 0; rb < a.w; rb += SC_ROWS) {
    // rows of this block: window rows rb..rb+127 -> positions L-w+rb+r
    const int pos0 = a.L - a.w + rb;
    __syncthreads();
    load_block_t<D>(sQ, qh, pos0, a.L);
    float m_run[8];
    double z_run[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) { m_run[i] = -INFINITY; z_run[i] = 0.0; }
    for (int tile = 0; tile < SC_CHUNK_TILES; ++tile) {
      const int kt0 = key0 + tile * SC_KEYS;
      if (kt0 >= a.L) break;
      __syncthreads();
      load_block_t<D>(sK, kh, kt0, a.L);
      __syncthreads();
      float acc[8][8];
      tile_dots<D>(sQ, sK, acc);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int wr = rb + ty * 8 + i;          // window row
        const int pos = a.L - a.w + wr;          // its position
        float mx = -INFINITY;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int key = kt0 + tile_key(tx, j);
          const float x = acc[i][j] * a.scale;
          acc[i][j] = (wr < a.w && key <= pos && key < a.L) ? x : -INFINITY;
          mx = fmaxf(mx, acc[i][j]);
        }
#pragma unroll
        for (int o = 8; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        float zs = 0.f;
        if (mx != -INFINITY) {
#pragma unroll
          for (int j = 0; j < 8; ++j) zs += expf(acc[i][j] - mx);
        }
#pragma unroll
        for (int o = 8; o >= 1; o >>= 1) zs += __shfl_xor_sync(0xffffffffu, zs, o);
        // merge the tile into the running (m, Z) of the chunk
        if (mx != -INFINITY) {
          if (mx > m_run[i]) {
            z_run[i] = z_run[i] * exp(static_cast<double>(m_run[i]) - mx) + zs;
            m_run[i] = mx;
          } else {
            z_run[i] += static_cast<double>(zs) * exp(static_cast<double>(mx) - m_run[i]);
          }
        }
      }
    }
    if (tx == 0) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int wr = rb + ty * 8 + i;
        if (wr < a.w) {
          const size_t o = (static_cast<size_t>(bh) * a.w + wr) * a.n_chunks + chunk;
          a.part_m[o] = m_run[i];
          a.part_z[o] = z_run[i];
        }
      }
    }
  }
}

// Merge: one thread per (head, window row).
__global__ void score_merge_kernel(const ScoreArgs a, int total_rows) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= total_rows) return;
  const float* pm = a.part_m + static_cast<size_t>(idx) * a.n_chunks;
  const double* pz = a.part_z + static_cast<size_t>(idx) * a.n_chunks;
  float m = -INFINITY;
  for (int c = 0; c < a.n_chunks; ++c) m = fmaxf(m, pm[c]);
  double z = 0.0;
  for (int c = 0; c < a.n_chunks; ++c)
    if (pm[c] != -INFINITY) z += pz[c] * exp(static_cast<double>(pm[c]) - m);
  a.stats[idx] = make_float2(m, static_cast<float>(1.0 / z));
}

// Pass 2: grid (n_key_tiles, B*Hq).  Column sums of the normalised weights.
template <int D>
__global__ void __launch_bounds__(SC_THREADS, 1) score_sum_kernel(const ScoreArgs a) {
  extern __shared__ float sm[];
  float* sQ = sm;
  float* sK = sm + D * 128;
  float* red = sm + 2 * D * 128;  // [16][128] column partials
  const int kt0 = blockIdx.x * SC_KEYS;
  const int bh = blockIdx.y;
  const int b = bh / a.Hq, h = bh % a.Hq;
  const __nv_bfloat16* qh = a.q + static_cast<size_t>(bh) * a.L * D;
  const __nv_bfloat16* kh = a.k + (static_cast<size_t>(b) * a.Hkv + h / a.G) * a.L * D;
  const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;

  load_block_t<D>(sK, kh, kt0, a.L);
  float col[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) col[j] = 0.f;
  for (int rb = 0; rb < a.w; rb += SC_ROWS) {
    __syncthreads();
    load_block_t<D>(sQ, qh, a.L - a.w + rb, a.L);
    __syncthreads();
    float acc[8][8];
    tile_dots<D>(sQ, sK, acc);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int wr = rb + ty * 8 + i;
      if (wr >= a.w) continue;
      const int pos = a.L - a.w + wr;
      const float2 st = a.stats[static_cast<size_t>(bh) * a.w + wr];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int key = kt0 + tile_key(tx, j);
        if (key <= pos && key < a.L) col[j] += expf(acc[i][j] * a.scale - st.x) * st.y;
      }
    }
  }
  __syncthreads();
#pragma unroll
  for (int j = 0; j < 8; ++j) red[ty * 128 + tile_key(tx, j)] = col[j];
  __syncthreads();
  if (threadIdx.x < SC_KEYS) {
    const int key = kt0 + threadIdx.x;
    float s = 0.f;
#pragma unroll
    for (int y = 0; y < 16; ++y) s += red[y * 128 + threadIdx.x];
    if (key < a.L) a.scores[static_cast<size_t>(bh) * a.L + key] = s;
  }
}

}  // namespace tsa
