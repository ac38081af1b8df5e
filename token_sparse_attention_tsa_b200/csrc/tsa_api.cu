// tsa_api.cu -- host side of the C ABI declared in include/tsa.h: argument
// validation, workspace carving, TMA descriptor encoding and kernel launches
// for the Token Sparse Attention prefill path on sm_100a.
//
// Method source: gist.science summary page "Token Sparse Attention: Efficient
// Long-Context Inference with Interleaved Token Selection", section 2
// ("Arquitectura Central", "Cobertura Dinamica de Tokens"); each kernel file
// cites the part it implements.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "tsa.h"
#include "attend.cuh"
#include "copy.cuh"
#include "score.cuh"
#include "select.cuh"

namespace {

constexpr size_t kAlign = 256;
constexpr int kMaxDevices = 64;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Proxy-score work split (see score.cuh): each head's window padded to a
// multiple of 32 rows, as many query heads of a KV group per CTA as fit in
// 512 packed rows, and key chunks sized so the grid is one wave of 148 SMs
// (one CTA per SM), never below 16 key tiles: a CTA loads its packed query
// rows once, so short chunks would spend their time reloading them.
struct ScorePlan {
  int W32, GH, n_hg, n_rp, MT, chunk_tiles, n_chunks;
};

ScorePlan score_plan(const tsa_params* p) {
  ScorePlan s;
  const int G = p->Hq / p->Hkv;
  s.W32 = (p->w + 31) / 32 * 32;
  const int tiles = (p->L + tsa::SC_KEYS - 1) / tsa::SC_KEYS;
  const int max_chunks = std::max(1, tiles / tsa::SC_MIN_CHUNK_TILES);
  // the most heads per CTA that fit, halved while a grid of such CTAs
  // (keys split no finer than SC_MIN_CHUNK_TILES) leaves SMs idle: short
  // sequences gain more from parallel heads than from sharing K tiles
  s.GH = s.W32 <= tsa::SC_PASS_ROWS ? std::min(G, tsa::SC_PASS_ROWS / s.W32) : 1;
  while (s.GH > 1 && p->B * p->Hkv * ((G + s.GH - 1) / s.GH) * max_chunks < 148) s.GH = (s.GH + 1) / 2;
  s.n_hg = (G + s.GH - 1) / s.GH;
  const int rows = s.GH * s.W32;
  s.n_rp = (rows + tsa::SC_PASS_ROWS - 1) / tsa::SC_PASS_ROWS;
  s.MT = s.n_rp > 1 ? tsa::SC_MAX_MT : (rows + 127) / 128;
  const int ctas = p->B * p->Hkv * s.n_hg;
  const int per = std::max(1, 148 / ctas);
  s.chunk_tiles = std::max(tsa::SC_MIN_CHUNK_TILES, (tiles + per - 1) / per);
  const int span = s.chunk_tiles * tsa::SC_KEYS;
  s.n_chunks = (p->L + span - 1) / span;
  return s;
}

int score_chunks(const tsa_params* p) { return score_plan(p).n_chunks; }

// Workspace layout.  Stage part: status word (+ abort words), score scratch,
// per-head budget scratch.
// Forward part: scores, idx, k_head, k_seq and the compressed Q, K and V.
// (tsa_forward's attention writes its output in place, so no compressed
// output is stored.)
struct WsLayout {
  size_t status = 0, part_m = 0, part_z = 0, stats = 0, kh_scratch = 0, stage_end = 0;
  size_t scores = 0, idx = 0, k_head = 0, k_seq = 0, qc = 0, kc = 0, vc = 0, total = 0;
};

WsLayout layout_of(const tsa_params* p) {
  WsLayout w;
  const size_t bhq = static_cast<size_t>(p->B) * p->Hq;
  const size_t rows = bhq * static_cast<size_t>(p->w);
  const size_t nch = static_cast<size_t>(score_chunks(p));
  size_t off = 0;
  w.status = off;           off += kAlign;
  w.part_m = off;           off = align_up(off + rows * nch * sizeof(float));
  w.part_z = off;           off = align_up(off + rows * nch * sizeof(double));
  w.stats = off;            off = align_up(off + rows * sizeof(float2));
  w.kh_scratch = off;       off = align_up(off + bhq * sizeof(int32_t));
  w.stage_end = off;
  const size_t tok = bhq * static_cast<size_t>(p->L);
  w.scores = off;           off = align_up(off + tok * sizeof(float));
  w.idx = off;              off = align_up(off + tok * sizeof(int32_t));
  w.k_head = off;           off = align_up(off + bhq * sizeof(int32_t));
  w.k_seq = off;            off = align_up(off + static_cast<size_t>(p->B) * sizeof(int32_t));
  w.qc = off;               off = align_up(off + tok * static_cast<size_t>(p->d) * 2);
  w.kc = off;               off = align_up(off + tok * static_cast<size_t>(p->d) * 2);
  w.vc = off;               off = align_up(off + tok * static_cast<size_t>(p->d) * 2);
  w.total = off;
  return w;
}

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

bool per_head(const tsa_params* p) { return p->budget_mode == TSA_BUDGET_PER_HEAD; }

// The caller's q, k, v, o are token-major [B, L, H, d] (else head-major
// [B, H, L, d]); compressed buffers, scores and indices are always head-major.
bool token_major(const tsa_params* p) { return p->layout == TSA_LAYOUT_BLHD; }

tsa::RowStrides strides_of(bool tm, int heads, int L, int d) {
  const long long H = heads, Ll = L, dd = d;
  return tm ? tsa::RowStrides{Ll * H * dd, dd, H * dd, nullptr} : tsa::RowStrides{H * Ll * dd, Ll * dd, dd, nullptr};
}

// Packed varlen batch: the caller's q, k, v, o hold total_tokens tokens,
// sequence b at [cu_seqlens[b], cu_seqlens[b+1]).
bool packed(const tsa_params* p) { return p->cu_seqlens != nullptr; }

tsa::Seqs seqs_of(const tsa_params* p) { return tsa::Seqs{p->cu_seqlens, p->L, p->total_tokens}; }

// Row strides of the caller's tensors (with `heads` heads).
tsa::RowStrides caller_strides(const tsa_params* p, int heads) {
  tsa::RowStrides r = strides_of(token_major(p), heads, p->L, p->d);
  r.cu = p->cu_seqlens;
  return r;
}

// Kept-row counts as the kernels read them: per sequence [B], or per head
// [B, Hq] in the per-head budget mode.
tsa::Kept kept_of(const tsa_params* p, const int32_t* n) {
  return per_head(p) ? tsa::Kept{n, p->Hq, 1} : tsa::Kept{n, 1, 0};
}

float scale_of(const tsa_params* p) {
  return p->softmax_scale > 0.f ? p->softmax_scale : 1.0f / std::sqrt(static_cast<float>(p->d));
}

uint64_t limit_ns_of(const tsa_params* p) {
  const uint64_t ms = p->timeout_ms ? p->timeout_ms : 2000u;
  return ms * 1000000ull;
}

tsa_status cuda_ok(cudaError_t e) { return e == cudaSuccess ? TSA_OK : TSA_ERR_CUDA; }

tsa_status launch_ok() { return cuda_ok(cudaGetLastError()); }

// ---------------------------------------------------------------- TMA maps
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// bf16 rows of B sequences x `heads` heads x L tokens x d: dimensions
// (d, L, heads, B) for head-major memory, (d, heads, L, B) for token-major
// (strides ascend either way); box = box_rows tokens x 64 columns of one
// head, 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, int d, int L, int heads, int B, bool tm, int box_rows = 128) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t D = static_cast<cuuint64_t>(d), Ll = static_cast<cuuint64_t>(L),
                   H = static_cast<cuuint64_t>(heads), Bb = static_cast<cuuint64_t>(B);
  cuuint64_t dims[4] = {D, tm ? H : Ll, tm ? Ll : H, Bb};
  cuuint64_t strides[3] = {D * 2, D * 2 * dims[1], D * 2 * dims[1] * dims[2]};
  const cuuint32_t rows = static_cast<cuuint32_t>(box_rows);
  cuuint32_t box[4] = {64, tm ? 1u : rows, tm ? rows : 1u, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [rows, d] bf16 viewed as one 2D tensor; box = one row x 64 columns,
// 128-byte swizzle (the form tile::gather4 loads need).
bool make_row_map(CUtensorMap* m, const void* base, int d, long long rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(d) * 2};
  cuuint32_t box[2] = {64, 1};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ---------------------------------------------------------------- attributes
template <typename K>
bool ensure_smem(std::atomic<int> (&done)[kMaxDevices], K kernel, int bytes) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  if (done[dev].load(std::memory_order_acquire)) return true;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
    return false;
  done[dev].store(1, std::memory_order_release);
  return true;
}

std::atomic<int> g_attn64[kMaxDevices], g_attn128[kMaxDevices], g_gath64[kMaxDevices], g_gath128[kMaxDevices],
    g_gq64[kMaxDevices], g_gq128[kMaxDevices], g_st64[kMaxDevices],
    g_st128[kMaxDevices], g_sum64[kMaxDevices], g_sum128[kMaxDevices], g_budget[kMaxDevices],
    g_select[kMaxDevices], g_blk64[kMaxDevices], g_blk128[kMaxDevices], g_blks64[kMaxDevices],
    g_blks128[kMaxDevices];

constexpr int kBudgetSmem = tsa::BUD_SMEM;
constexpr int kSelectSmem = tsa::SEL_SMEM;

// ---------------------------------------------------------------- launchers
// Tensor map over the caller's q, k or v (`heads` heads): per-sequence
// batches in either layout, or packed sequences as one token-major sequence
// of total_tokens tokens.
bool make_caller_map(CUtensorMap* m, const tsa_params* p, const void* base, int heads, int box_rows = 128) {
  if (packed(p)) return make_map(m, base, p->d, p->total_tokens, heads, 1, true, box_rows);
  return make_map(m, base, p->d, p->L, heads, p->B, token_major(p), box_rows);
}

tsa_status run_score(const tsa_params* p, const void* q, const void* k, float* scores, void* ws,
                     cudaStream_t st) {
  const WsLayout w = layout_of(p);
  const ScorePlan sp = score_plan(p);
  CUtensorMap mq, mk;
  const bool tm = token_major(p);
  if (!make_caller_map(&mq, p, q, p->Hq, tsa::SC_QBOX) || !make_caller_map(&mk, p, k, p->Hkv, tsa::SC_KEYS))
    return TSA_ERR_CUDA;
  tsa::ScoreArgs a;
  a.scores = scores;
  a.part_m = at<float>(ws, w.part_m);
  a.part_z = at<double>(ws, w.part_z);
  a.stats = at<float2>(ws, w.stats);
  a.status = at<uint32_t>(ws, 0);
  a.abort_word = at<uint32_t>(ws, 8);
  a.L = p->L;
  a.w = p->w;
  a.Hq = p->Hq;
  a.Hkv = p->Hkv;
  a.G = p->Hq / p->Hkv;
  a.W32 = sp.W32;
  a.GH = sp.GH;
  a.n_hg = sp.n_hg;
  a.n_rp = sp.n_rp;
  a.MT = sp.MT;
  a.n_chunks = sp.n_chunks;
  a.chunk_tiles = sp.chunk_tiles;
  a.scale_log2 = scale_of(p) * 1.4426950408889634f;
  a.limit_ns = limit_ns_of(p);
  a.token_major = tm ? 1 : 0;
  a.test_stall = (p->flags & TSA_FLAG_TEST_STALL_SCORE) ? 1 : 0;
  a.seqs = seqs_of(p);
  const dim3 grid(sp.n_chunks, p->B * p->Hkv * sp.n_hg);
  const int rows = p->B * p->Hq * p->w;
  if (cudaMemsetAsync(a.abort_word, 0, sizeof(uint32_t), st) != cudaSuccess) return TSA_ERR_CUDA;
  if (p->d == 128) {
    constexpr int sm = tsa::ScoreLayout<128>::ALLOC;
    if (!ensure_smem(g_st128, tsa::score_kernel<128, false>, sm) ||
        !ensure_smem(g_sum128, tsa::score_kernel<128, true>, sm))
      return TSA_ERR_CUDA;
    tsa::score_kernel<128, false><<<grid, tsa::SC_THREADS, sm, st>>>(mq, mk, a);
    tsa::score_merge_kernel<<<(rows + 255) / 256, 256, 0, st>>>(a, rows);
    tsa::score_kernel<128, true><<<grid, tsa::SC_THREADS, sm, st>>>(mq, mk, a);
  } else {
    constexpr int sm = tsa::ScoreLayout<64>::ALLOC;
    if (!ensure_smem(g_st64, tsa::score_kernel<64, false>, sm) ||
        !ensure_smem(g_sum64, tsa::score_kernel<64, true>, sm))
      return TSA_ERR_CUDA;
    tsa::score_kernel<64, false><<<grid, tsa::SC_THREADS, sm, st>>>(mq, mk, a);
    tsa::score_merge_kernel<<<(rows + 255) / 256, 256, 0, st>>>(a, rows);
    tsa::score_kernel<64, true><<<grid, tsa::SC_THREADS, sm, st>>>(mq, mk, a);
  }
  return launch_ok();
}

// k_head receives every head's count (required); k_seq, when not null, the
// per-sequence budget of the mode (max, or ceiling of the mean; per-head
// mode reports the max).  partial: k_seq receives this device's share of a
// budget combined over devices instead (the sum of the counts in mean mode,
// the max otherwise).
tsa_status run_budget(const tsa_params* p, const float* scores, int32_t* k_head, int32_t* k_seq,
                      uint32_t* status, cudaStream_t st, bool partial = false) {
  if (!ensure_smem(g_budget, tsa::budget_kernel, kBudgetSmem)) return TSA_ERR_CUDA;
  tsa::BudgetArgs a{scores, k_head, status, p->L, p->Hq, p->keep_recent, static_cast<double>(p->tau), seqs_of(p)};
  tsa::budget_kernel<<<p->B * p->Hq * tsa::BS_CLUSTER, tsa::BS_THREADS, kBudgetSmem, st>>>(a);
  const bool mean = p->budget_mode == TSA_BUDGET_MEAN;
  if (k_seq) tsa::budget_finalize_kernel<<<p->B, 32, 0, st>>>(k_head, k_seq, p->Hq, mean ? (partial ? 2 : 1) : 0);
  return launch_ok();
}

tsa_status run_select(const tsa_params* p, const float* scores, const int32_t* kept, int32_t* idx,
                      cudaStream_t st) {
  if (!ensure_smem(g_select, tsa::select_kernel, kSelectSmem)) return TSA_ERR_CUDA;
  tsa::SelectArgs a{scores, kept_of(p, kept), idx, p->L, p->Hq, p->keep_recent, seqs_of(p)};
  tsa::select_kernel<<<p->B * p->Hq * tsa::BS_CLUSTER, tsa::BS_THREADS, kSelectSmem, st>>>(a);
  return launch_ok();
}

tsa_status run_gather(const tsa_params* p, const void* q, const void* k, const void* v, const int32_t* idx,
                      const int32_t* k_seq, void* qc, void* kc, void* vc, uint32_t* status, cudaStream_t st) {
  tsa::GatherArgs a;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.k = static_cast<const __nv_bfloat16*>(k);
  a.v = static_cast<const __nv_bfloat16*>(v);
  a.idx = idx;
  a.kept = kept_of(p, k_seq);
  a.seqs = seqs_of(p);
  a.qs = caller_strides(p, p->Hq);
  a.kvs = caller_strides(p, p->Hkv);
  a.qc = static_cast<__nv_bfloat16*>(qc);
  a.kc = static_cast<__nv_bfloat16*>(kc);
  a.vc = static_cast<__nv_bfloat16*>(vc);
  a.status = status;
  a.B = p->B;
  a.L = p->L;
  a.Hq = p->Hq;
  a.Hkv = p->Hkv;
  a.G = p->Hq / p->Hkv;
  // one resident wave of 4 CTAs per SM, each walking work items
  const long long items = static_cast<long long>(p->B) * p->Hkv * ((p->L + tsa::GT_ROWS - 1) / tsa::GT_ROWS);
  const int grid = static_cast<int>(items < 148LL * 4 ? items : 148LL * 4);
  if (p->d == 128)
    tsa::gather_kernel<128><<<grid, 256, 0, st>>>(a);
  else
    tsa::gather_kernel<64><<<grid, 256, 0, st>>>(a);
  return launch_ok();
}

tsa_status run_scatter(const tsa_params* p, const void* oc, const int32_t* idx, const int32_t* k_seq, void* o,
                       uint32_t* status, cudaStream_t st) {
  tsa::ScatterArgs a{static_cast<const __nv_bfloat16*>(oc), idx, kept_of(p, k_seq),
                     static_cast<__nv_bfloat16*>(o), caller_strides(p, p->Hq), status, p->L, p->Hq, seqs_of(p)};
  const dim3 g((p->L + tsa::SCAT_ROWS - 1) / tsa::SCAT_ROWS, p->B * p->Hq);
  if (p->d == 128)
    tsa::scatter_kernel<128><<<g, 256, 0, st>>>(a);
  else
    tsa::scatter_kernel<64><<<g, 256, 0, st>>>(a);
  return launch_ok();
}

// Attention over [B*Hq, L, d] queries against K/V with heads_kv heads
// (query head h of sequence b reads K/V head b*heads_kv + h/g_kv).  With idx,
// Q/K/V rows are gathered by index inside the kernel and output row i lands
// at row idx[i] of o (the rest of o is not touched).
// Attention over [B*Hq, L, d] queries against K/V with heads_kv heads
// (query head h of sequence b reads K/V head b*heads_kv + h/g_kv).
// idx (with scatter): output row i lands at row idx[i] of o (the rest of o is
// not touched).  idx with gather as well: Q/K/V rows are loaded by index from
// the uncompressed tensors instead of as compressed tiles.
// in_caller / out_caller: q, k, v / o are the caller's tensors (p->layout,
// possibly packed sequences) rather than head-major compressed buffers.
tsa_status run_attend(const tsa_params* p, const void* q, const void* k, const void* v, int heads_kv, int g_kv,
                      const int32_t* k_seq, void* o, float* lse, uint32_t* status, uint32_t* abort_word,
                      cudaStream_t st, bool in_caller, bool out_caller, const int32_t* idx = nullptr,
                      bool gather = false, const uint8_t* block_mask = nullptr) {
  CUtensorMap mq, mk, mv;
  const bool scatter = idx != nullptr;
  gather = gather && scatter;
  const long long tokens = (in_caller && packed(p)) ? p->total_tokens : static_cast<long long>(p->B) * p->L;
  const bool maps_ok =
      gather ? (make_row_map(&mq, q, p->d, tokens * p->Hq) && make_row_map(&mk, k, p->d, tokens * heads_kv) &&
                make_row_map(&mv, v, p->d, tokens * heads_kv))
      : in_caller ? (make_caller_map(&mq, p, q, p->Hq) && make_caller_map(&mk, p, k, heads_kv) &&
                     make_caller_map(&mv, p, v, heads_kv))
                  : (make_map(&mq, q, p->d, p->L, p->Hq, p->B, false) &&
                     make_map(&mk, k, p->d, p->L, heads_kv, p->B, false) &&
                     make_map(&mv, v, p->d, p->L, heads_kv, p->B, false));
  if (!maps_ok) return TSA_ERR_CUDA;
  if (cudaMemsetAsync(abort_word, 0, sizeof(uint32_t), st) != cudaSuccess) return TSA_ERR_CUDA;
  tsa::AttnArgs a;
  a.kept = kept_of(p, k_seq);
  a.o = static_cast<__nv_bfloat16*>(o);
  a.lse = lse;
  a.status = status;
  a.abort_word = abort_word;
  a.idx = idx;
  a.L = p->L;
  a.Hq = p->Hq;
  a.Hkv_map = heads_kv;
  a.G_map = g_kv;
  a.n_tiles = (p->L + 127) / 128;
  a.scale_log2 = scale_of(p) * 1.4426950408889634f;
  a.limit_ns = limit_ns_of(p);
  a.test_stall = (p->flags & TSA_FLAG_TEST_STALL) ? 1 : 0;
  a.token_major = (in_caller && token_major(p)) ? 1 : 0;
  a.in_packed = (in_caller && packed(p)) ? 1 : 0;
  a.seqs = seqs_of(p);
  a.os = out_caller ? caller_strides(p, p->Hq) : strides_of(false, p->Hq, p->L, p->d);
  a.block_mask = block_mask;
  const dim3 grid((a.n_tiles + 1) / 2, p->B * p->Hq);  // two query tiles per CTA
  auto launch = [&](auto kernel, std::atomic<int>(&attr)[kMaxDevices], int threads, int smem) -> tsa_status {
    if (!ensure_smem(attr, kernel, smem)) return TSA_ERR_CUDA;
    kernel<<<grid, threads, smem, st>>>(mq, mk, mv, a);
    return launch_ok();
  };
  if (p->d == 128) {
    using L = tsa::Attn2Layout<128>;
    if (block_mask) {
      if (!scatter) return launch(tsa::attend2_kernel<128, false, false, true>, g_blk128, L::THREADS, L::ALLOC);
      return launch(tsa::attend2_kernel<128, false, true, true>, g_blks128, L::THREADS, L::ALLOC);
    }
    if (!scatter) return launch(tsa::attend2_kernel<128, false, false>, g_attn128, L::THREADS, L::ALLOC);
    if (!gather) return launch(tsa::attend2_kernel<128, false, true>, g_gq128, L::THREADS, L::ALLOC);
    return launch(tsa::attend2_kernel<128, true, true>, g_gath128, L::THREADS, L::ALLOC);
  }
  using L = tsa::Attn2Layout<64>;
  if (block_mask) {
    if (!scatter) return launch(tsa::attend2_kernel<64, false, false, true>, g_blk64, L::THREADS, L::ALLOC);
    return launch(tsa::attend2_kernel<64, false, true, true>, g_blks64, L::THREADS, L::ALLOC);
  }
  if (!scatter) return launch(tsa::attend2_kernel<64, false, false>, g_attn64, L::THREADS, L::ALLOC);
  if (!gather) return launch(tsa::attend2_kernel<64, false, true>, g_gq64, L::THREADS, L::ALLOC);
  return launch(tsa::attend2_kernel<64, true, true>, g_gath64, L::THREADS, L::ALLOC);
}

// Zero the rows of o that no index selects (the selected rows are left as
// they are).
tsa_status run_zero_unselected(const tsa_params* p, const int32_t* idx, const int32_t* k_seq, void* o,
                               uint32_t* status, cudaStream_t st) {
  tsa::ScatterArgs a{nullptr, idx, kept_of(p, k_seq), static_cast<__nv_bfloat16*>(o), caller_strides(p, p->Hq),
                     status, p->L, p->Hq, seqs_of(p)};
  const dim3 g((p->L + tsa::SCAT_ROWS - 1) / tsa::SCAT_ROWS, p->B * p->Hq);
  if (p->d == 128)
    tsa::scatter_kernel<128, true><<<g, 256, 0, st>>>(a);
  else
    tsa::scatter_kernel<64, true><<<g, 256, 0, st>>>(a);
  return launch_ok();
}

tsa_status check_ws(const tsa_params* p, void* ws, size_t ws_bytes, bool full) {
  if (!ws) return TSA_ERR_WORKSPACE;
  if (!aligned(ws, kAlign)) return TSA_ERR_INVALID_ARG;
  const WsLayout w = layout_of(p);
  if (ws_bytes < (full ? w.total : w.stage_end)) return TSA_ERR_WORKSPACE;
  return TSA_OK;
}

bool tensors_ok(std::initializer_list<const void*> ptrs) {
  for (const void* q : ptrs)
    if (!q || !aligned(q, 16)) return false;
  return true;
}

uint32_t* status_of(void* ws) { return ws ? at<uint32_t>(ws, 0) : nullptr; }
uint32_t* abort_of(void* ws) { return at<uint32_t>(ws, 4); }   // attention; +8: score

}  // namespace

extern "C" {

int32_t tsa_abi_version(void) { return TSA_ABI_VERSION; }

const char* tsa_status_string(tsa_status s) {
  switch (s) {
    case TSA_OK: return "ok";
    case TSA_ERR_INVALID_ARG: return "invalid argument";
    case TSA_ERR_UNSUPPORTED: return "unsupported configuration";
    case TSA_ERR_WORKSPACE: return "workspace missing or too small";
    case TSA_ERR_CUDA: return "CUDA error";
    case TSA_ERR_NONFINITE: return "non-finite or negative score";
    case TSA_ERR_TIMEOUT: return "pipeline wait timed out";
    case TSA_ERR_BAD_INDEX: return "index outside [0, L)";
  }
  return "unknown status";
}

tsa_status tsa_check_params(const tsa_params* p) {
  if (!p) return TSA_ERR_INVALID_ARG;
  if (p->B < 1 || p->Hq < 1 || p->Hkv < 1 || p->L < 1 || p->d < 1 || p->w < 1) return TSA_ERR_INVALID_ARG;
  if (p->Hq % p->Hkv != 0) return TSA_ERR_INVALID_ARG;
  if (p->w > p->L) return TSA_ERR_INVALID_ARG;
  if (!(p->tau >= 0.f && p->tau < 1.f)) return TSA_ERR_INVALID_ARG;
  if (!(p->softmax_scale >= 0.f) || std::isinf(p->softmax_scale)) return TSA_ERR_INVALID_ARG;
  if ((p->flags & ~(TSA_FLAG_TEST_STALL | TSA_FLAG_TEST_STALL_SCORE)) != 0) return TSA_ERR_INVALID_ARG;
  if (p->budget_mode < TSA_BUDGET_MAX || p->budget_mode > TSA_BUDGET_PER_HEAD) return TSA_ERR_INVALID_ARG;
  if (p->keep_recent < 0 || p->keep_recent > p->L) return TSA_ERR_INVALID_ARG;
  if (p->layout != TSA_LAYOUT_BHLD && p->layout != TSA_LAYOUT_BLHD) return TSA_ERR_INVALID_ARG;
  if (p->cu_seqlens) {  // packed sequences: token-major, at least one token, offsets 4-byte aligned
    if (p->layout != TSA_LAYOUT_BLHD || p->total_tokens < 1 || !aligned(p->cu_seqlens, 4))
      return TSA_ERR_INVALID_ARG;
    if (static_cast<long long>(p->total_tokens) * (p->Hq > p->Hkv ? p->Hq : p->Hkv) >= (1LL << 31))
      return TSA_ERR_UNSUPPORTED;
  } else if (p->total_tokens != 0) {
    return TSA_ERR_INVALID_ARG;
  }
  if (p->d != 64 && p->d != 128) return TSA_ERR_UNSUPPORTED;
  if (p->w > 4096 || p->L > (1 << 22)) return TSA_ERR_UNSUPPORTED;
  if (static_cast<long long>(p->B) * p->Hq * p->L >= (1LL << 31)) return TSA_ERR_UNSUPPORTED;
  return TSA_OK;
}

tsa_status tsa_workspace_size(const tsa_params* p, size_t* bytes) {
  const tsa_status s = tsa_check_params(p);
  if (s != TSA_OK) return s;
  if (!bytes) return TSA_ERR_INVALID_ARG;
  *bytes = layout_of(p).total;
  return TSA_OK;
}

tsa_status tsa_stage_workspace_size(const tsa_params* p, size_t* bytes) {
  const tsa_status s = tsa_check_params(p);
  if (s != TSA_OK) return s;
  if (!bytes) return TSA_ERR_INVALID_ARG;
  *bytes = layout_of(p).stage_end;
  return TSA_OK;
}

tsa_status tsa_reset_device_status(void* ws, void* stream) {
  if (!ws || !aligned(ws, kAlign)) return TSA_ERR_INVALID_ARG;
  return cuda_ok(cudaMemsetAsync(ws, 0, 16, static_cast<cudaStream_t>(stream)));
}

tsa_status tsa_get_device_status(const void* ws, void* stream, uint32_t* flags) {
  if (!ws || !aligned(ws, kAlign)) return TSA_ERR_INVALID_ARG;
  uint32_t v = 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(&v, ws, sizeof(v), cudaMemcpyDeviceToHost, st) != cudaSuccess) return TSA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return TSA_ERR_CUDA;
  if (flags) *flags = v;
  if (v & TSA_DEVFLAG_TIMEOUT) return TSA_ERR_TIMEOUT;
  if (v & TSA_DEVFLAG_BAD_INDEX) return TSA_ERR_BAD_INDEX;
  if (v & TSA_DEVFLAG_NONFINITE) return TSA_ERR_NONFINITE;
  return TSA_OK;
}

tsa_status tsa_score(const tsa_params* p, const void* q, const void* k, float* scores, void* ws,
                     size_t ws_bytes, void* stream) {
  tsa_status s = tsa_check_params(p);
  if (s != TSA_OK) return s;
  if (!tensors_ok({q, k, scores})) return TSA_ERR_INVALID_ARG;
  if ((s = check_ws(p, ws, ws_bytes, false)) != TSA_OK) return s;
  return run_score(p, q, k, scores, ws, static_cast<cudaStream_t>(stream));
}

tsa_status tsa_budget(const tsa_params* p, const float* scores, int32_t* k_head, int32_t* k_seq, void* ws,
                      size_t ws_bytes, void* stream) {
  tsa_status s = tsa_check_params(p);
  if (s != TSA_OK) return s;
  if (!tensors_ok({scores, k_seq}) || (k_head && !aligned(k_head, 4))) return TSA_ERR_INVALID_ARG;
  if (per_head(p) && !k_head) return TSA_ERR_INVALID_ARG;  // the per-head counts are the budget
  if ((s = check_ws(p, ws, ws_bytes, false)) != TSA_OK) return s;
  int32_t* kh = k_head ? k_head : at<int32_t>(ws, layout_of(p).kh_scratch);
  return run_budget(p, scores, kh, k_seq, status_of(ws), static_cast<cudaStream_t>(stream));
}

tsa_status tsa_select(const tsa_params* p, const float* scores, const int32_t* k_seq, int32_t* idx, void* ws,
                      size_t ws_bytes, void* stream) {
  tsa_status s = tsa_check_params(p);
  if (s != TSA_OK) return s;
  if (!tensors_ok({scores, k_seq, idx})) return TSA_ERR_INVALID_ARG;
  if ((s = check_ws(p, ws, ws_bytes, false)) != TSA_OK) return s;
  return run_select(p, scores, k_seq, idx, static_cast<cudaStream_t>(stream));
}

tsa_status tsa_gather_qkv(const tsa_params* p, const void* q, const void* k, const void* v, const int32_t* idx,
                          const int32_t* k_seq, void* qc, void* kc, void* vc, void* ws, size_t ws_bytes,
                          void* stream) {
  tsa_status s = tsa_check_params(p);
  if (s != TSA_OK) return s;
  if (!tensors_ok({q, k, v, idx, k_seq, kc, vc}) || (qc && !aligned(qc, 16))) return TSA_ERR_INVALID_ARG;
  if (ws && (s = check_ws(p, ws, ws_bytes, false)) != TSA_OK) return s;
  return run_gather(p, q, k, v, idx, k_seq, qc, kc, vc, status_of(ws), static_cast<cudaStream_t>(stream));
}

tsa_status tsa_attend(const tsa_params* p, const void* qc, const void* kc, const void* vc, const int32_t* k_seq,
                      void* oc, float* lse, void* ws, size_t ws_bytes, void* stream) {
  tsa_status s = tsa_check_params(p);
  if (s != TSA_OK) return s;
  if (!tensors_ok({qc, kc, vc, k_seq, oc}) || (lse && !aligned(lse, 4))) return TSA_ERR_INVALID_ARG;
  if ((s = check_ws(p, ws, ws_bytes, false)) != TSA_OK) return s;
  return run_attend(p, qc, kc, vc, p->Hq, 1, k_seq, oc, lse, status_of(ws), abort_of(ws),
                    static_cast<cudaStream_t>(stream), false, false);
}

tsa_status tsa_attend_dense(const tsa_params* p, const void* q, const void* k, const void* v, void* o,
                            float* lse, void* ws, size_t ws_bytes, void* stream) {
  tsa_status s = tsa_check_params(p);
  if (s != TSA_OK) return s;
  if (!tensors_ok({q, k, v, o}) || (lse && !aligned(lse, 4))) return TSA_ERR_INVALID_ARG;
  if ((s = check_ws(p, ws, ws_bytes, false)) != TSA_OK) return s;
  return run_attend(p, q, k, v, p->Hkv, p->Hq / p->Hkv, nullptr, o, lse, status_of(ws), abort_of(ws),
                    static_cast<cudaStream_t>(stream), true, true);
}

tsa_status tsa_scatter(const tsa_params* p, const void* oc, const int32_t* idx, const int32_t* k_seq, void* o,
                       void* ws, size_t ws_bytes, void* stream) {
  tsa_status s = tsa_check_params(p);
  if (s != TSA_OK) return s;
  if (!tensors_ok({oc, idx, k_seq, o})) return TSA_ERR_INVALID_ARG;
  if (ws && (s = check_ws(p, ws, ws_bytes, false)) != TSA_OK) return s;
  return run_scatter(p, oc, idx, k_seq, o, status_of(ws), static_cast<cudaStream_t>(stream));
}

}  // extern "C"

namespace {

// Steps 3-6 of the forward from the scores and the kept counts: selection,
// gather, attention (output over qc in place) and scatter.
tsa_status forward_tail(const tsa_params* p, const void* q, const void* k, const void* v, void* o,
                        const float* scores, const int32_t* kseq, int32_t* idx, void* ws, cudaStream_t st) {
  const WsLayout w = layout_of(p);
  tsa_status s;
  if ((s = run_select(p, scores, kseq, idx, st)) != TSA_OK) return s;
  // gather once; attention on the compressed tensors with its output written
  // over qc in place (each CTA loads its own two query tiles into shared
  // memory before any of its output rows is stored, and no other CTA reads
  // them); then the scatter writes every row of o once
  // (tsa_gather_qkv + tsa_attend with oc = qc + tsa_scatter)
  void* qc = at<void>(ws, w.qc);
  void* kc = at<void>(ws, w.kc);
  void* vc = at<void>(ws, w.vc);
  if ((s = run_gather(p, q, k, v, idx, kseq, qc, kc, vc, status_of(ws), st)) != TSA_OK) return s;
  if ((s = run_attend(p, qc, kc, vc, p->Hq, 1, kseq, qc, nullptr, status_of(ws), abort_of(ws), st, false,
                      false)) != TSA_OK)
    return s;
  return run_scatter(p, qc, idx, kseq, o, status_of(ws), st);
}

bool out_ptrs_ok(const float* scores, const int32_t* idx, const int32_t* kvec, const int32_t* kseq) {
  return !(scores && !aligned(scores, 16)) && !(idx && !aligned(idx, 16)) && !(kvec && !aligned(kvec, 4)) &&
         !(kseq && !aligned(kseq, 4));
}

}  // namespace

extern "C" {

tsa_status tsa_forward(const tsa_params* p, const void* q, const void* k, const void* v, void* o,
                       float* scores_out, int32_t* idx_out, int32_t* k_seq_out, void* ws, size_t ws_bytes,
                       void* stream) {
  tsa_status s = tsa_check_params(p);
  if (s != TSA_OK) return s;
  if (!tensors_ok({q, k, v, o})) return TSA_ERR_INVALID_ARG;
  if (!out_ptrs_ok(scores_out, idx_out, nullptr, k_seq_out)) return TSA_ERR_INVALID_ARG;
  if ((s = check_ws(p, ws, ws_bytes, true)) != TSA_OK) return s;
  const WsLayout w = layout_of(p);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  float* scores = scores_out ? scores_out : at<float>(ws, w.scores);
  int32_t* idx = idx_out ? idx_out : at<int32_t>(ws, w.idx);
  // kept counts: k_seq [B] (max / mean), or the heads' own counts [B, Hq]
  int32_t* khead = (per_head(p) && k_seq_out) ? k_seq_out : at<int32_t>(ws, w.k_head);
  int32_t* kbud = (!per_head(p) && k_seq_out) ? k_seq_out : at<int32_t>(ws, w.k_seq);
  int32_t* kseq = per_head(p) ? khead : kbud;
  if ((s = run_score(p, q, k, scores, ws, st)) != TSA_OK) return s;
  if ((s = run_budget(p, scores, khead, kbud, status_of(ws), st)) != TSA_OK) return s;
  return forward_tail(p, q, k, v, o, scores, kseq, idx, ws, st);
}

tsa_status tsa_forward_begin(const tsa_params* p, const void* q, const void* k, float* scores_out,
                             int32_t* k_head_out, int32_t* k_part, void* ws, size_t ws_bytes, void* stream) {
  tsa_status s = tsa_check_params(p);
  if (s != TSA_OK) return s;
  if (!tensors_ok({q, k}) || !k_part || !aligned(k_part, 4)) return TSA_ERR_INVALID_ARG;
  if (!out_ptrs_ok(scores_out, nullptr, k_head_out, nullptr)) return TSA_ERR_INVALID_ARG;
  if ((s = check_ws(p, ws, ws_bytes, true)) != TSA_OK) return s;
  const WsLayout w = layout_of(p);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  float* scores = scores_out ? scores_out : at<float>(ws, w.scores);
  int32_t* khead = k_head_out ? k_head_out : at<int32_t>(ws, w.k_head);
  if ((s = run_score(p, q, k, scores, ws, st)) != TSA_OK) return s;
  return run_budget(p, scores, khead, k_part, status_of(ws), st, true);
}

tsa_status tsa_forward_end(const tsa_params* p, int32_t Hq_total, const void* q, const void* k, const void* v,
                           void* o, const float* scores, const int32_t* k_head, const int32_t* k_reduced,
                           int32_t* idx_out, int32_t* k_seq_out, void* ws, size_t ws_bytes, void* stream) {
  tsa_status s = tsa_check_params(p);
  if (s != TSA_OK) return s;
  if (Hq_total < p->Hq) return TSA_ERR_INVALID_ARG;
  if (static_cast<long long>(p->B) * Hq_total * p->L >= (1LL << 31)) return TSA_ERR_UNSUPPORTED;
  if (!tensors_ok({q, k, v, o})) return TSA_ERR_INVALID_ARG;
  if (!per_head(p) && (!k_reduced || !aligned(k_reduced, 4))) return TSA_ERR_INVALID_ARG;
  if (!out_ptrs_ok(scores, idx_out, k_head, k_seq_out)) return TSA_ERR_INVALID_ARG;
  if ((s = check_ws(p, ws, ws_bytes, true)) != TSA_OK) return s;
  const WsLayout w = layout_of(p);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const float* sc = scores ? scores : at<float>(ws, w.scores);
  int32_t* idx = idx_out ? idx_out : at<int32_t>(ws, w.idx);
  const int32_t* kseq = nullptr;
  if (per_head(p)) {  // nothing is combined over heads: each head keeps its own count
    const int32_t* kh = k_head ? k_head : at<int32_t>(ws, w.k_head);
    if (k_seq_out && cudaMemcpyAsync(k_seq_out, kh, static_cast<size_t>(p->B) * p->Hq * sizeof(int32_t),
                                     cudaMemcpyDeviceToDevice, st) != cudaSuccess)
      return TSA_ERR_CUDA;
    kseq = kh;
  } else if (p->budget_mode == TSA_BUDGET_MEAN) {  // the reduced value is the sum of every head's count
    int32_t* kb = k_seq_out ? k_seq_out : at<int32_t>(ws, w.k_seq);
    tsa::budget_mean_kernel<<<(p->B + 127) / 128, 128, 0, st>>>(k_reduced, kb, p->B, Hq_total);
    if ((s = launch_ok()) != TSA_OK) return s;
    kseq = kb;
  } else {  // the reduced value is the max over every head's count: the budget itself
    if (k_seq_out && k_seq_out != k_reduced &&
        cudaMemcpyAsync(k_seq_out, k_reduced, static_cast<size_t>(p->B) * sizeof(int32_t),
                        cudaMemcpyDeviceToDevice, st) != cudaSuccess)
      return TSA_ERR_CUDA;
    kseq = k_reduced;
  }
  return forward_tail(p, q, k, v, o, sc, kseq, idx, ws, st);
}

tsa_status tsa_attend_scatter(const tsa_params* p, const void* qc, const void* kc, const void* vc,
                              const int32_t* idx, const int32_t* k_seq, void* o, float* lse, void* ws,
                              size_t ws_bytes, void* stream) {
  tsa_status s = tsa_check_params(p);
  if (s != TSA_OK) return s;
  if (!tensors_ok({qc, kc, vc, idx, k_seq, o}) || (lse && !aligned(lse, 4))) return TSA_ERR_INVALID_ARG;
  if ((s = check_ws(p, ws, ws_bytes, false)) != TSA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((s = run_attend(p, qc, kc, vc, p->Hq, 1, k_seq, o, lse, status_of(ws), abort_of(ws), st, false, true,
                      idx)) != TSA_OK)
    return s;
  return run_zero_unselected(p, idx, k_seq, o, status_of(ws), st);
}

tsa_status tsa_attend_gathered(const tsa_params* p, const void* q, const void* k, const void* v,
                               const int32_t* idx, const int32_t* k_seq, void* o, float* lse, void* ws,
                               size_t ws_bytes, void* stream) {
  tsa_status s = tsa_check_params(p);
  if (s != TSA_OK) return s;
  if (!tensors_ok({q, k, v, idx, k_seq, o}) || (lse && !aligned(lse, 4))) return TSA_ERR_INVALID_ARG;
  if ((s = check_ws(p, ws, ws_bytes, false)) != TSA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((s = run_attend(p, q, k, v, p->Hkv, p->Hq / p->Hkv, k_seq, o, lse, status_of(ws), abort_of(ws), st, true,
                      true, idx, true)) != TSA_OK)
    return s;
  return run_zero_unselected(p, idx, k_seq, o, status_of(ws), st);
}

tsa_status tsa_attend_blocks(const tsa_params* p, const void* qc, const void* kc, const void* vc,
                             const int32_t* idx, const int32_t* k_seq, const uint8_t* block_mask, void* o,
                             float* lse, void* ws, size_t ws_bytes, void* stream) {
  tsa_status s = tsa_check_params(p);
  if (s != TSA_OK) return s;
  if (!tensors_ok({qc, kc, vc, k_seq, o}) || !block_mask || (idx && !aligned(idx, 16)) ||
      (lse && !aligned(lse, 4)))
    return TSA_ERR_INVALID_ARG;
  if ((s = check_ws(p, ws, ws_bytes, false)) != TSA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((s = run_attend(p, qc, kc, vc, p->Hq, 1, k_seq, o, lse, status_of(ws), abort_of(ws), st, false,
                      idx != nullptr, idx, false, block_mask)) != TSA_OK)
    return s;
  return idx ? run_zero_unselected(p, idx, k_seq, o, status_of(ws), st) : TSA_OK;
}

tsa_status tsa_layer_forward(const tsa_params* p, int32_t layer, const uint8_t* sparse_layers, int32_t n_layers,
                             const void* q, const void* k, const void* v, void* o, float* scores_out,
                             int32_t* idx_out, int32_t* k_seq_out, void* ws, size_t ws_bytes, void* stream) {
  tsa_status s = tsa_check_params(p);
  if (s != TSA_OK) return s;
  if (!sparse_layers || n_layers < 1 || layer < 0 || layer >= n_layers) return TSA_ERR_INVALID_ARG;
  if (sparse_layers[layer])
    return tsa_forward(p, q, k, v, o, scores_out, idx_out, k_seq_out, ws, ws_bytes, stream);
  return tsa_attend_dense(p, q, k, v, o, nullptr, ws, ws_bytes, stream);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Proxy scores without any device allocation.
//
// Some callers cannot call cudaMalloc: plug-ins whose host framework owns
// every device allocation through its own pool, code with a hard device
// memory budget, or plain C callers with no allocator for a workspace.  For
// them tsa_score_noalloc runs the same score kernels as tsa_score with their
// scratch (the per-chunk row statistics) in the fixed array below instead of
// a caller workspace.  The array lives in the library's device image, so
// every GPU that loads the library holds it until the process exits.
namespace {

static __device__ __align__(256) unsigned char g_score_scratch[TSA_NOALLOC_SCRATCH_BYTES];

std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_score_scratch on the current device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up once
// per device with that device current.
tsa_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return TSA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_score_scratch) != cudaSuccess || !ptr) return TSA_ERR_CUDA;
    g_scratch_ptr[dev] = ptr;
  }
  *out = g_scratch_ptr[dev];
  return TSA_OK;
}

}  // namespace

extern "C" tsa_status tsa_score_noalloc(const tsa_params* p, const void* q, const void* k, float* scores,
                                        void* stream) {
  tsa_status s = tsa_check_params(p);
  if (s != TSA_OK) return s;
  if (!tensors_ok({q, k, scores})) return TSA_ERR_INVALID_ARG;
  if (layout_of(p).stage_end > static_cast<size_t>(TSA_NOALLOC_SCRATCH_BYTES)) return TSA_ERR_WORKSPACE;
  void* scratch = nullptr;
  if ((s = scratch_address(&scratch)) != TSA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // The status and abort words at the start of the array describe this call
  // only: clear them first.  Every other scratch entry the kernels read is
  // written earlier in the same call when no CTA aborts; after an abort the
  // status word says so and the scores are not to be used.
  if (cudaMemsetAsync(scratch, 0, 16, st) != cudaSuccess) return TSA_ERR_CUDA;
  return run_score(p, q, k, scores, scratch, st);
}

extern "C" tsa_status tsa_score_noalloc_status(void* stream, uint32_t* flags) {
  void* scratch = nullptr;
  const tsa_status s = scratch_address(&scratch);
  if (s != TSA_OK) return s;
  return tsa_get_device_status(scratch, stream, flags);
}
