/*
 * tsa.h -- C ABI of the Token Sparse Attention prefill path on NVIDIA B200
 * (sm_100a).
 *
 * Method source, cited below as [GS]: the gist.science summary page
 * "Token Sparse Attention: Efficient Long-Context Inference with Interleaved
 * Token Selection" (arXiv 2602.03216), section 2 "Metodologia", with its
 * sub-sections "Arquitectura Central" (per-head compression of Q, K, V into
 * dense shorter tensors, ordinary attention on them, decompression of the
 * output into a zero-initialised full-length tensor) and "Cobertura Dinamica
 * de Tokens" (proxy scoring of recent queries against all keys, a coverage
 * budget from the ascending importance order, per-head top-k selection).
 * The abstract pages with the same title (chatpaper.ai, icml.cc poster 65647,
 * fugumt.com) describe the same compress / attend / decompress scheme.
 *
 * Notation: B sequences, Hq query heads, Hkv key/value heads, G = Hq/Hkv,
 * KV head of query head h is h / G (consecutive grouping), L tokens per
 * sequence, d head dimension, w proxy window, tau coverage threshold,
 * k_b keep budget of sequence b, S_h ascending index set of head h.
 *
 * Layouts (all row-major, contiguous, little-endian):
 *   q        bf16 [B, Hq,  L, d]      k, v   bf16 [B, Hkv, L, d]
 *   o        bf16 [B, Hq,  L, d]
 *            (head-major, p->layout == TSA_LAYOUT_BHLD, the default), or
 *            token-major with p->layout == TSA_LAYOUT_BLHD: q, o
 *            [B, L, Hq, d] and k, v [B, L, Hkv, d], the layout a prefill
 *            engine's projections produce.  Only the caller's q, k, v, o
 *            follow p->layout; every tensor below is always head-major.
 *            Varlen batches (p->cu_seqlens not NULL, token-major only):
 *            sequences of different lengths packed one after another, q, o
 *            [T, Hq, d] and k, v [T, Hkv, d] with T = p->total_tokens;
 *            sequence b is tokens [cu_seqlens[b], cu_seqlens[b+1]) and its
 *            length L_b is at most p->L, which then is the capacity of every
 *            per-head buffer below (entries past L_b are not meaningful).  A
 *            sequence shorter than w uses all its tokens as the window.
 *            Every call reads cu_seqlens on the device; a sequence that does
 *            not fit in [0, T] or is longer than L is treated as empty and
 *            sets TSA_DEVFLAG_BAD_INDEX (in tsa_budget).
 *   scores   fp32 [B, Hq, L]
 *   idx      int32 [B, Hq, L]: entries [0, k_b) hold S_h ascending, the rest -1
 *   k_head   int32 [B, Hq]            k_seq  int32 [B]
 *   kept     the rows kept by every head, argument of the calls after the
 *            budget (named k_seq there): k_seq [B] (one budget per sequence,
 *            budget modes MAX and MEAN), or the heads' own counts k_head
 *            [B, Hq] when p->budget_mode == TSA_BUDGET_PER_HEAD.  Below, k_b
 *            is the kept count of the head in question.
 *   qc, kc, vc, oc  bf16 [B, Hq, L, d]: compressed tensors, capacity L rows
 *            per head, rows [0, k_b) valid (K and V are gathered per query
 *            head, so a GQA group's heads each get their own compressed copy).
 *   lse      fp32 [B, Hq, L] (optional): natural-log sum of exp of the
 *            scaled logits of each valid compressed row.
 *
 * Conventions shared by every call:
 *   - Pointers named q, k, v, o, scores, idx, k_head, k_seq, qc, kc, vc, oc,
 *     lse and ws are DEVICE pointers on the current CUDA device.  The caller
 *     owns every buffer; the library allocates and frees nothing and keeps no
 *     state besides per-device cached attributes.
 *   - Tensor pointers must be 16-byte aligned; ws must be 256-byte aligned.
 *   - stream is a cudaStream_t (NULL = legacy default stream).  Every call is
 *     asynchronous on it and never synchronises the host, except
 *     tsa_get_device_status.  No call reads k_b back to the host: compressed
 *     buffers are sized at capacity L and kernels read k_seq on the device.
 *   - Argument errors are detected on the host and returned before any work
 *     is enqueued (TSA_ERR_INVALID_ARG, TSA_ERR_UNSUPPORTED,
 *     TSA_ERR_WORKSPACE).  A failed launch returns TSA_ERR_CUDA.
 *   - Errors found by kernels (non-finite scores, an index outside [0, L), a
 *     pipeline wait that ran past its time limit) are OR-ed into the device
 *     status word at the start of ws; read it with tsa_get_device_status.
 *     Kernels never trap; on such an error they finish or return early.
 *   - Supported: d in {64, 128}; Hq % Hkv == 0; 1 <= w <= min(L, 4096);
 *     0 <= tau < 1; L <= 2^22; B * Hq * L < 2^31.
 */
#ifndef TSA_H_
#define TSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define TSA_ABI_VERSION 3

typedef enum tsa_status {
  TSA_OK = 0,
  TSA_ERR_INVALID_ARG = 1,  /* null pointer, bad shape, misaligned pointer  */
  TSA_ERR_UNSUPPORTED = 2,  /* valid but unsupported (e.g. d = 96)           */
  TSA_ERR_WORKSPACE = 3,    /* workspace missing or smaller than required    */
  TSA_ERR_CUDA = 4,         /* a CUDA runtime/driver call or launch failed   */
  TSA_ERR_NONFINITE = 5,    /* device status: a score was NaN or infinite    */
  TSA_ERR_TIMEOUT = 6,      /* device status: a pipeline wait timed out      */
  TSA_ERR_BAD_INDEX = 7     /* device status: an index was outside [0, L)    */
} tsa_status;

/* tsa_params.flags: test hook for the failure path.  The attention kernels
 * (tsa_attend*, tsa_forward) first wait on a barrier that nothing completes;
 * the bounded wait runs out after timeout_ms, the kernel sets
 * TSA_DEVFLAG_TIMEOUT, lets its in-flight copies land, frees its tensor
 * memory and returns without writing outputs.  The context stays usable. */
#define TSA_FLAG_TEST_STALL 0x80000000u
/* The same test hook for the proxy-score kernels (tsa_score,
 * tsa_score_noalloc, the score step of tsa_forward): the first score pass
 * times out and sets TSA_DEVFLAG_TIMEOUT, every later score CTA of the call
 * stops early, and the scores are not written. */
#define TSA_FLAG_TEST_STALL_SCORE 0x40000000u

/* tsa_params.budget_mode: how the heads' coverage counts k_head combine into
 * the rows each head keeps.  [GS] calls the budget global without saying how
 * heads combine; MAX (every head of sequence b keeps k_b = max_h k_head) is
 * the default reading, MEAN (k_b = ceil(mean_h k_head)) and PER_HEAD (head h
 * keeps its own k_head, no shared budget) are the two other plain ones. */
/* tsa_params.layout: memory order of the caller's q, k, v and o. */
#define TSA_LAYOUT_BHLD 0
#define TSA_LAYOUT_BLHD 1

#define TSA_BUDGET_MAX 0
#define TSA_BUDGET_MEAN 1
#define TSA_BUDGET_PER_HEAD 2

/* Bits of the device status word (first 4 bytes of ws). */
#define TSA_DEVFLAG_NONFINITE 0x1u
#define TSA_DEVFLAG_TIMEOUT 0x2u
#define TSA_DEVFLAG_BAD_INDEX 0x4u

typedef struct tsa_params {
  int32_t B, Hq, Hkv, L, d;
  int32_t w;            /* proxy window: the last w query positions          */
  float tau;            /* coverage threshold, 0 <= tau < 1                  */
  float softmax_scale;  /* 0 selects 1/sqrt(d) (fp32)                        */
  uint32_t flags;       /* 0, or TSA_FLAG_TEST_STALL / _STALL_SCORE (tests)  */
  uint32_t timeout_ms;  /* limit of one pipeline wait; 0 selects 2000 ms     */
  int32_t budget_mode;  /* TSA_BUDGET_MAX (0), _MEAN or _PER_HEAD            */
  int32_t keep_recent;  /* 0 <= r <= L: the last r tokens of every sequence
                           are kept in every head (each k_head is raised to
                           at least r; the selection ranks them first)       */
  int32_t layout;       /* TSA_LAYOUT_BHLD (0) or TSA_LAYOUT_BLHD (1)        */
  int32_t total_tokens; /* varlen: T, the packed tensors' token count; else 0 */
  const int32_t* cu_seqlens; /* varlen: DEVICE int32 [B+1] token offsets,
                           non-decreasing from 0; NULL for B sequences of L  */
} tsa_params;

/* Version of this ABI (TSA_ABI_VERSION of the built library). */
int32_t tsa_abi_version(void);

/* Human-readable name of a status code.  Never NULL. */
const char* tsa_status_string(tsa_status s);

/* Host-only validation of p (the same checks every call makes). */
tsa_status tsa_check_params(const tsa_params* p);

/* Workspace bytes needed by tsa_forward (covers every stage call too): the
 * stage scratch, scores, indices, budgets and the compressed Q, K and V (the
 * compressed output overwrites the compressed Q, so it takes no space of its
 * own). */
tsa_status tsa_workspace_size(const tsa_params* p, size_t* bytes);

/* Workspace bytes needed by the single-stage calls below (status word and
 * the proxy-score row statistics; much smaller than tsa_workspace_size). */
tsa_status tsa_stage_workspace_size(const tsa_params* p, size_t* bytes);

/* Zero the device status word (enqueued on stream). */
tsa_status tsa_reset_device_status(void* ws, void* stream);

/* Synchronise stream, read the device status word into *flags (may be NULL)
 * and map it to a status: TSA_OK when no bit is set, else the first of
 * TSA_ERR_TIMEOUT, TSA_ERR_BAD_INDEX, TSA_ERR_NONFINITE that is set. */
tsa_status tsa_get_device_status(const void* ws, void* stream, uint32_t* flags);

/* Step 1 -- proxy scores.  [GS] "Cobertura Dinamica de Tokens", scoring:
 * for every (b, h) and window row i in [L-w, L), the causal softmax over keys
 * j <= i of scale * q[b,h,i].k[b,h/G,j]; scores[b,h,j] is the sum of those
 * weights over the w rows (fp32, accumulated in fp32/fp64).
 * In: q, k.  Out: scores.  ws: >= tsa_stage_workspace_size bytes. */
tsa_status tsa_score(const tsa_params* p, const void* q, const void* k, float* scores,
                     void* ws, size_t ws_bytes, void* stream);

/* Step 2 -- coverage budget.  [GS] "Cobertura Dinamica de Tokens", budget
 * allocation and per-head selection: per head, masses
 * q_j = ceil(score_j * 2^40) (int64), T = floor(tau * sum_j q_j) (fp64),
 * p_h = the largest count of least-important tokens whose mass sum is <= T,
 * k_head = max(L - p_h, keep_recent); the sequence's budget k_seq[b] =
 * max_h k_head (MAX and PER_HEAD modes) or ceil(mean_h k_head) (MEAN).
 * Bit-exact integer arithmetic.  Non-finite scores set TSA_DEVFLAG_NONFINITE.
 * In: scores.  Out: k_head (may be NULL except in PER_HEAD mode, where it is
 * the kept-count argument of the later calls), k_seq.  ws: stage size. */
tsa_status tsa_budget(const tsa_params* p, const float* scores, int32_t* k_head, int32_t* k_seq,
                      void* ws, size_t ws_bytes, void* stream);

/* Step 3 -- per-head top-k.  [GS] "Cobertura Dinamica de Tokens", per-head
 * selection: S_h = the k_b tokens of largest score (the last keep_recent
 * tokens first), equal scores going to the smaller index, written ascending
 * to idx[b,h,0..k_b); the rest of idx[b,h,:] is set to -1.  In: scores,
 * kept counts (see "kept" above).  Out: idx.  ws: stage size. */
tsa_status tsa_select(const tsa_params* p, const float* scores, const int32_t* k_seq, int32_t* idx,
                      void* ws, size_t ws_bytes, void* stream);

/* Step 4 -- gather.  [GS] "Arquitectura Central", compression:
 * qc[b,h,i] = q[b,h,S_h[i]], kc[b,h,i] = k[b,h/G,S_h[i]],
 * vc[b,h,i] = v[b,h/G,S_h[i]] for i < k_b.  Rows >= k_b are not written.
 * qc may be NULL: then only K and V are gathered.
 * An index outside [0, L) writes a zero row and sets TSA_DEVFLAG_BAD_INDEX
 * (when ws is not NULL).  ws: NULL or stage size. */
tsa_status tsa_gather_qkv(const tsa_params* p, const void* q, const void* k, const void* v,
                          const int32_t* idx, const int32_t* k_seq, void* qc, void* kc, void* vc,
                          void* ws, size_t ws_bytes, void* stream);

/* Step 5 -- causal attention on the compressed tensors.  [GS] "Arquitectura
 * Central": the compressed tensors stay dense, so an ordinary dense causal
 * kernel runs on them.  oc[b,h,i] = sum_{j<=i} softmax_j(scale *
 * qc[b,h,i].kc[b,h,j]) vc[b,h,j] for i < k_b (bf16 out, fp32
 * accumulation; tcgen05 tensor cores).  Rows >= k_b of oc are not written.
 * Rows of qc/kc/vc at or beyond k_b may hold any bits.  lse may be NULL.
 * ws: stage size (its status word receives timeouts). */
tsa_status tsa_attend(const tsa_params* p, const void* qc, const void* kc, const void* vc,
                      const int32_t* k_seq, void* oc, float* lse,
                      void* ws, size_t ws_bytes, void* stream);

/* Steps 5-6 fused -- attention on the compressed tensors with the scatter in
 * its epilogue.  [GS] "Arquitectura Central", decompression: compressed
 * output row i is written straight to o[b,h,S_h[i]] and every other row of o
 * is set to zero, so no compressed output is stored.  Same result as
 * tsa_attend followed by tsa_scatter.  In: qc, kc, vc (as tsa_attend), idx,
 * k_seq.  Out: o
 * [B,Hq,L,d]; lse (nullable) indexed by compressed row.  An index outside
 * [0, L) is skipped and sets TSA_DEVFLAG_BAD_INDEX.  ws: stage size. */
tsa_status tsa_attend_scatter(const tsa_params* p, const void* qc, const void* kc, const void* vc,
                              const int32_t* idx, const int32_t* k_seq, void* o, float* lse,
                              void* ws, size_t ws_bytes, void* stream);

/* Steps 4-6 fused -- gather, compressed attention and scatter in one kernel.
 * [GS] "Arquitectura Central": the same result as tsa_gather_qkv,
 * tsa_attend and tsa_scatter in sequence, without materialising the
 * compressed tensors: the attention kernel loads the rows S_h[i] of q and of
 * k, v (KV head h/G) by index with TMA row gathers, and writes compressed
 * output row i to o[b,h,S_h[i]]; every other row of o is set to zero.
 * In: q, k, v (original layouts), idx, k_seq.  Out: o [B,Hq,L,d]; lse
 * (nullable) indexed by compressed row as in tsa_attend.  An index outside
 * [0, L) is skipped and sets TSA_DEVFLAG_BAD_INDEX.  ws: stage size. */
tsa_status tsa_attend_gathered(const tsa_params* p, const void* q, const void* k, const void* v,
                               const int32_t* idx, const int32_t* k_seq, void* o, float* lse,
                               void* ws, size_t ws_bytes, void* stream);

/* Steps 5(-6) with a block-sparse mask over the compressed sequence.  [GS]
 * section 4 presents the method as complementary to block-sparse attention
 * kernels (e.g. FlexPrefill): those run on the compressed tensors.  Same as
 * tsa_attend (idx NULL: compressed output oc in o) or tsa_attend_scatter
 * (idx given: output scattered into o in p->layout, other rows zero), except
 * that compressed row i attends key j <= i only when j / 128 == i / 128 or
 * block_mask[b, h, i / 128, j / 128] is nonzero.  block_mask: DEVICE uint8
 * [B, Hq, NB, NB], NB = ceil(L / 128), caller-owned; entries above the
 * diagonal are ignored and diagonal blocks are always attended.  KV tiles
 * that neither query tile of a CTA's pair attends are skipped.
 * ws: stage size. */
tsa_status tsa_attend_blocks(const tsa_params* p, const void* qc, const void* kc, const void* vc,
                             const int32_t* idx, const int32_t* k_seq, const uint8_t* block_mask, void* o,
                             float* lse, void* ws, size_t ws_bytes, void* stream);

/* Dense causal GQA attention on the uncompressed tensors (the baseline the
 * method is measured against; the same kernel as tsa_attend with the
 * identity selection): o[b,h,i] = sum_{j<=i} softmax_j(scale *
 * q[b,h,i].k[b,h/G,j]) v[b,h/G,j].  lse may be NULL.  ws: stage size. */
tsa_status tsa_attend_dense(const tsa_params* p, const void* q, const void* k, const void* v,
                            void* o, float* lse, void* ws, size_t ws_bytes, void* stream);

/* Step 6 -- scatter.  [GS] "Arquitectura Central", decompression: o[b,h,:]
 * is zero except o[b,h,S_h[i]] = oc[b,h,i] for i < k_b.  idx[b,h,0..k_b)
 * must be strictly ascending, as tsa_select writes it: each CTA locates its
 * rows by binary search.  With such an idx every row of o is written exactly
 * once.  An entry outside [0, L_b) is not written and sets
 * TSA_DEVFLAG_BAD_INDEX (when ws is not NULL).  ws: NULL or stage size. */
tsa_status tsa_scatter(const tsa_params* p, const void* oc, const int32_t* idx, const int32_t* k_seq,
                       void* o, void* ws, size_t ws_bytes, void* stream);

/* The whole path: score -> budget -> select -> gather -> attention on the
 * compressed tensors (its output written over the compressed Q in the
 * workspace) -> scatter into o; enqueued on stream with no host
 * synchronisation.
 * scores_out, idx_out, k_seq_out may be NULL (then the workspace holds
 * them); when given they receive the intermediate results, k_seq_out the
 * kept counts in the mode's shape ([B], or [B, Hq] in PER_HEAD mode).
 * ws: >= tsa_workspace_size bytes. */
tsa_status tsa_forward(const tsa_params* p, const void* q, const void* k, const void* v, void* o,
                       float* scores_out, int32_t* idx_out, int32_t* k_seq_out,
                       void* ws, size_t ws_bytes, void* stream);

/* Head-sharded forward.  [GS] "Cobertura Dinamica de Tokens" makes the
 * budget global across the heads of a sequence; every other step is per
 * head.  When the query heads of one sequence are split over several devices
 * (each holding whole heads: its query heads and the key/value heads they
 * read), the forward runs in two halves around one exchange of B integers:
 *
 *   tsa_forward_begin   steps 1-2 on this device's heads: proxy scores and
 *                       the per-head coverage counts k_head, plus this
 *                       device's budget partial k_part [B]: the max of its
 *                       k_head (TSA_BUDGET_MAX, and TSA_BUDGET_PER_HEAD where
 *                       it is not used) or their sum (TSA_BUDGET_MEAN);
 *   (the caller)        reduces k_part over the devices of the sequence's
 *                       heads: MAX in MAX mode, SUM in MEAN mode, nothing in
 *                       PER_HEAD mode (e.g. ncclAllReduce on B int32);
 *   tsa_forward_end     the budget from the reduced value k_reduced (MAX: the
 *                       value itself; MEAN: ceil(k_reduced / Hq_total);
 *                       PER_HEAD: each head's own k_head), then steps 3-6.
 *
 * p describes this device's part (Hq, Hkv: its own head counts; every other
 * field as for the whole problem); q, k, v, o are its heads' tensors.
 * Hq_total is the number of query heads of a sequence over all devices
 * (p->Hq when nothing is split).  On one device, begin + end with k_reduced =
 * k_part compute exactly what tsa_forward computes.  Both halves take the
 * same ws (>= tsa_workspace_size), which must not be touched in between;
 * scores_out / scores and k_head_out / k_head may be NULL (the workspace
 * then holds them) and, when given, must be the same buffers in both calls.
 * k_part and k_reduced are DEVICE int32 [B] (k_reduced may be NULL in
 * PER_HEAD mode); idx_out and k_seq_out are as in tsa_forward. */
tsa_status tsa_forward_begin(const tsa_params* p, const void* q, const void* k, float* scores_out,
                             int32_t* k_head_out, int32_t* k_part, void* ws, size_t ws_bytes, void* stream);
tsa_status tsa_forward_end(const tsa_params* p, int32_t Hq_total, const void* q, const void* k, const void* v,
                           void* o, const float* scores, const int32_t* k_head, const int32_t* k_reduced,
                           int32_t* idx_out, int32_t* k_seq_out, void* ws, size_t ws_bytes, void* stream);

/* Layer-level switch.  [GS] section 2 "Seleccion de Capas Dispersas" applies
 * the method only in the layers chosen by a criterion on the model's hidden
 * states (inter-layer representation drift); that criterion needs a model
 * and is not computed here.  The caller supplies the choice instead:
 * sparse_layers is a HOST array of n_layers flags (nonzero = sparse), and
 * layer (0 <= layer < n_layers) selects this call's layer.  A sparse layer
 * runs tsa_forward (same arguments and workspace rules); a dense layer runs
 * tsa_attend_dense on q, k, v into o and leaves scores_out, idx_out and
 * k_seq_out untouched.  ws: >= tsa_workspace_size bytes. */
tsa_status tsa_layer_forward(const tsa_params* p, int32_t layer, const uint8_t* sparse_layers, int32_t n_layers,
                             const void* q, const void* k, const void* v, void* o, float* scores_out,
                             int32_t* idx_out, int32_t* k_seq_out, void* ws, size_t ws_bytes, void* stream);

/* Proxy scores with no device allocation at all.  No counterpart on the
 * pages: an addition for callers that cannot call cudaMalloc (a plug-in whose
 * host framework owns every device allocation, code under a hard device
 * memory budget, a C caller without an allocator for a workspace).
 *
 * Computes exactly what tsa_score computes, with the same kernels; the
 * scratch that tsa_score takes from ws lives instead in a fixed array of
 * TSA_NOALLOC_SCRATCH_BYTES inside the library, which every GPU that loads
 * the library holds until the process exits.  The caller still passes q, k
 * and scores.  Sizes whose scratch (tsa_stage_workspace_size) exceeds the
 * array are rejected with TSA_ERR_WORKSPACE before any work is enqueued.
 * The first call on a device looks up the array's device address (once per
 * device, with that device current); make that first call before any stream
 * capture.  All calls share the one array and it keeps the last call's
 * contents: calls whose kernels overlap on the GPU (different streams, or
 * different host threads on one device) race and must be serialised by the
 * caller.  Calls no cudaMalloc, cudaFree or allocating library routine.
 * Each call first clears the array's status word (enqueued on stream), so
 * after it the word describes that call alone: a bounded pipeline wait that
 * ran out (TSA_DEVFLAG_TIMEOUT, scores not written) or a sequence that did not
 * fit.  Read it with tsa_score_noalloc_status. */
#define TSA_NOALLOC_SCRATCH_BYTES (16u << 20)
tsa_status tsa_score_noalloc(const tsa_params* p, const void* q, const void* k, float* scores,
                             void* stream);

/* Status word of the most recent tsa_score_noalloc call on the current
 * device, read without a workspace: synchronises stream, writes the raw bits
 * to *flags (may be NULL) and maps them as tsa_get_device_status does.  No
 * counterpart on the pages; allocates nothing. */
tsa_status tsa_score_noalloc_status(void* stream, uint32_t* flags);

#ifdef __cplusplus
}
#endif

#endif /* TSA_H_ */
