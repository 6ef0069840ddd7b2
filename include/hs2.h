/*
 * hs2.h -- C ABI of libhs2: the KV-Reuse token-sparse attention of one HySparse2 hybrid block
 * on an NVIDIA B200 (sm_100a).
 *
 * The operation (HySparse2 pages):
 *  - "HySparse2: How Xiaomi Split the Transformer to Fix Agent Prefill Costs", section
 *    "KV Reuse and Token-Level Sparse Selection": a hybrid block of the cross-decoder is one
 *    full-attention layer followed by sparse-attention layers. The full layer attends over the
 *    whole context and produces both the KV cache and token selection indices; the sparse
 *    layers reuse the indices and the cache without recomputing them. Selection is per token:
 *    1,024 tokens from the whole context plus a forced window of the 128 most recent tokens,
 *    read from the full layer's cache.
 *  - "HySparse2: Hybrid Sparse Attention with Two-Level KV Sharing", bullets "KV Reuse
 *    refinements" and "Inference cost": token-level selection, forced local window, MQA (one
 *    K/V head for all query heads), FP8 KV cache.
 * Readings where the pages are silent: the importance score of cache position t for a query
 * row is s[t] = sum_h exp(c * q_h . k_t - lse_h), c = softmax_scale (1/sqrt(128) by default),
 * computed in a second pass from the full layer's log-sum-exp; ties go to the lower index;
 * the window is not part of the candidate set; the selected set is returned ascending.
 *
 * Conventions for every call:
 *  - Device pointers are CUDA global-memory pointers on the current device; "HOST" marks the
 *    few host pointers. The caller owns every buffer. The library allocates nothing, keeps no
 *    state between calls, and launches only on `stream` (a cudaStream_t; NULL = legacy default
 *    stream). Calls return after enqueueing; nothing synchronises.
 *  - Argument errors are detected on the host before anything is enqueued and returned as
 *    HS2_ERR_INVALID_ARG / HS2_ERR_UNSUPPORTED / HS2_ERR_WORKSPACE with a message in
 *    hs2_last_error(). A CUDA launch error returns HS2_ERR_CUDA. Errors found by the kernels
 *    themselves (a bounded wait that ran out) are recorded in the workspace and read back with
 *    hs2_read_device_status(). No C++ exception crosses this interface.
 *  - Shapes: B = batch, Nq = query tokens per sequence (1 for decode), H = query heads,
 *    d = 128. Query i of sequence b sits at cache position p = T_b - Nq + i and attends
 *    causally to positions [0, p] of its own sequence. Flat query row r = b * Nq + i.
 *  - Calls that overlap on the GPU must not share a workspace.
 */
#ifndef HS2_H_
#define HS2_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define HS2_VERSION 1
#define HS2_HEAD_DIM 128
#define HS2_MAX_BATCH 128     /* sequences per call */
#define HS2_MAX_TOPK 2048     /* global selection budget per query row */
#define HS2_MAX_WINDOW 4096   /* forced recent window per query row */
#define HS2_NOALLOC_SCRATCH_BYTES (4u << 20)  /* built-in scratch of hs2_topk_select_noalloc */

typedef enum {
  HS2_OK = 0,
  HS2_ERR_INVALID_ARG = 1,   /* null / misaligned pointer, bad shape, inconsistent sizes */
  HS2_ERR_UNSUPPORTED = 2,   /* valid but not implemented: head_dim != 128, H not 16/32, ... */
  HS2_ERR_WORKSPACE = 3,     /* workspace smaller than hs2_workspace_size() */
  HS2_ERR_CUDA = 4,          /* a CUDA runtime/driver call failed */
  HS2_ERR_DEVICE_CHECK = 5,  /* a kernel's own consistency check failed (device status) */
  HS2_ERR_TIMEOUT = 6        /* a kernel's bounded wait ran out (device status) */
} hs2_status;

typedef enum {
  HS2_KV_BF16 = 0,           /* K, V rows of 128 bf16 */
  HS2_KV_FP8_E4M3 = 1        /* K, V rows of 128 OCP e4m3fn codes; value = scale[row] * code */
} hs2_kv_dtype;

typedef enum { HS2_OUT_BF16 = 0, HS2_OUT_F32 = 1 } hs2_out_dtype;

/* The shared single-head (MQA) K/V cache of one full-attention layer, and the query shape.
 * Sequence b occupies cache rows [kv_start[b], kv_start[b] + kv_len[b]); its queries are its
 * last n_q tokens. Row-major [kv_rows, 128]; each row is one token's K (or V). */
typedef struct hs2_kv_view {
  int32_t batch;             /* B, 1..HS2_MAX_BATCH */
  int32_t n_q;               /* Nq >= 1; every kv_len[b] >= n_q */
  int32_t n_heads;           /* H: 16 or 32 query heads share the one K/V head */
  int32_t head_dim;          /* must be 128 */
  int32_t kv_dtype;          /* hs2_kv_dtype */
  int32_t reserved;          /* must be 0 */
  int64_t kv_rows;           /* rows of k / v / k_scale / v_scale (>= every sequence's end) */
  const void *k;             /* device, 16-byte aligned */
  const void *v;             /* device, 16-byte aligned */
  const float *k_scale;      /* device [kv_rows], 16-byte aligned, FP8 only (else NULL) */
  const float *v_scale;      /* device [kv_rows], 16-byte aligned, FP8 only (else NULL) */
  const int64_t *kv_start;   /* HOST [batch] */
  const int32_t *kv_len;     /* HOST [batch], T_b */
} hs2_kv_view;

/* Outputs of hs2_block_decode that the caller may leave to the library (pass NULL for them): the
 * flags of hs2_workspace_size that reserve room for them in the workspace. */
#define HS2_WS_SCORES 1u      /* scores == NULL: the [B*Nq, max p + 1] fp32 scores */
#define HS2_WS_SELECTION 2u   /* idx == count == NULL: the selected positions and their counts */

/* Bytes of device scratch the calls below need for this view and budget (same value for every
 * call on the view). flags: 0, or HS2_WS_SCORES and / or HS2_WS_SELECTION for an
 * hs2_block_decode call that leaves those outputs to the workspace. Any 256-byte-aligned device
 * buffer of at least this size works; its contents on entry do not matter. Host-only; does not
 * touch the GPU. Unknown flag bits: HS2_ERR_INVALID_ARG. */
hs2_status hs2_workspace_size(const hs2_kv_view *kv, int32_t topk, int32_t window,
                              uint32_t flags, size_t *bytes);

/* Step 1 -- the full-attention layer and its importance scores (pages: section "KV Reuse and
 * Token-Level Sparse Selection"; the full layer attends causally over the entire context).
 * For every query row r and head h:
 *   lse[r,h]  = log sum_{t<=p} exp(c q_h.k_t)
 *   out[r,h,:] = sum_{t<=p} exp(c q_h.k_t - lse[r,h]) v_t
 *   scores[r * score_stride + t] = sum_h exp(c q_h.k_t - lse[r,h])      for t in [0, p]
 * q: device bf16 [B, Nq, H, 128]. out: device [B, Nq, H, 128] of out_dtype. lse: device fp32
 * [B, Nq, H]. scores: device fp32, score_stride >= max p + 1 (entries past p are not written).
 * The scores are written by a second pass over K that uses the final lse. */
hs2_status hs2_full_attn_scores(const hs2_kv_view *kv, const void *q, float softmax_scale,
                                void *out, int32_t out_dtype, float *lse, float *scores,
                                int64_t score_stride, void *workspace, size_t workspace_bytes,
                                void *stream);

/* Step 2 -- token-level top-k plus forced window (pages: "KV Reuse and Token-Level Sparse
 * Selection"; "KV Reuse refinements"). For query row r at position p: candidates
 * C = [0, nc) with nc = max(0, p - window + 1), window W = [nc, p]. If nc <= topk the selection
 * is [0, p]; otherwise it is the topk candidates with the largest score (ties: lower index),
 * followed by W, all ascending. Scores are compared by their fp32 bit patterns, which for the
 * non-negative scores step 1 produces is the numeric order (an exact, deterministic radix
 * select). A candidate score that is negative (-0.0 included) or NaN breaks that order: the
 * call still completes and records HS2_ERR_DEVICE_CHECK in the device status.
 * idx: device int32 [B*Nq, idx_stride], idx_stride >= min(max p + 1, topk + window);
 * only the first count[r] entries of row r are written. count: device int32 [B*Nq]. */
hs2_status hs2_topk_select(const hs2_kv_view *kv, const float *scores, int64_t score_stride,
                           int32_t topk, int32_t window, int32_t *idx, int32_t idx_stride,
                           int32_t *count, void *workspace, size_t workspace_bytes,
                           void *stream);

/* Step 3 -- one sparse-attention layer with KV Reuse (pages: section "KV Reuse and Token-Level
 * Sparse Selection"; sparse layers take the full layer's indices as they are, and window tokens
 * come from the same cache the full layer wrote). Each query row
 * attends only to its selected positions; each gathered K/V row is loaded once for all heads:
 *   out[r,h,:] = sum_{j<count[r]} softmax_j(c q_h.k_{S_j}) v_{S_j},  S = idx[r, :count[r]]
 * q: device bf16 [B, Nq, H, 128] (this layer's own queries). Indices must lie in [0, p];
 * count[r] must be in [1, idx_stride] and at most topk + window of the workspace sizing. */
hs2_status hs2_sparse_gather_attn(const hs2_kv_view *kv, const void *q, const int32_t *idx,
                                  int32_t idx_stride, const int32_t *count,
                                  float softmax_scale, void *out, int32_t out_dtype,
                                  void *workspace, size_t workspace_bytes, void *stream);

/* The whole hybrid block: step 1, step 2, then n_sparse sparse layers that reuse the indices
 * and the cache, enqueued back to back on `stream`. q_sparse / out_sparse are HOST arrays of
 * n_sparse device pointers (layouts as in step 3). lse, scores, idx and count are outputs too
 * (layouts as above), each optional: a NULL lse, a NULL scores (score_stride is then ignored) or
 * NULL idx and count (idx_stride ignored; both or neither) are kept in the workspace instead,
 * which must then hold hs2_workspace_size(kv, topk, window, flags) bytes with HS2_WS_SCORES /
 * HS2_WS_SELECTION set for the NULL ones (the lse always fits). n_sparse may be 0. */
hs2_status hs2_block_decode(const hs2_kv_view *kv, const void *q_full,
                            const void *const *q_sparse, int32_t n_sparse, int32_t topk,
                            int32_t window, float softmax_scale, void *out_full,
                            void *const *out_sparse, int32_t out_dtype, float *lse,
                            float *scores, int64_t score_stride, int32_t *idx,
                            int32_t idx_stride, int32_t *count, void *workspace,
                            size_t workspace_bytes, void *stream);

/* hs2_block_decode, plus one cudaEvent_t (cast to void *) recorded on `stream` before the
 * first enqueued operation and after each step: events[0] before the workspace clear,
 * events[1] after it, events[2] after the full-attention pass 1 kernel, events[3] after the
 * merge of its partial results (no kernel for chunk/prefill queries, whose pass 1 merges
 * inside), events[4] after score pass 2, events[5] after the selection, events[6 + l] after
 * sparse layer l. n_events must be 6 + n_sparse. For timing individual kernels without a
 * profiler; results are identical. */
hs2_status hs2_block_decode_traced(const hs2_kv_view *kv, const void *q_full,
                                   const void *const *q_sparse, int32_t n_sparse, int32_t topk,
                                   int32_t window, float softmax_scale, void *out_full,
                                   void *const *out_sparse, int32_t out_dtype, float *lse,
                                   float *scores, int64_t score_stride, int32_t *idx,
                                   int32_t idx_stride, int32_t *count, void *workspace,
                                   size_t workspace_bytes, void *const *events,
                                   int32_t n_events, void *stream);

/* hs2_topk_select without a caller workspace. The pages have no counterpart to this call: it
 * is plumbing for callers that cannot allocate device memory -- for example a plugin hosted by
 * a runtime that has already reserved the whole device for its own memory pool, or a
 * latency-critical path that must not call cudaMalloc (which may synchronise the device).
 * Instead of a workspace it uses a scratch array of HS2_NOALLOC_SCRATCH_BYTES (4 MiB) that the
 * library declares as a static device variable: every GPU that loads libhs2 holds those 4 MiB
 * until the process exits. It calls no allocator (no cudaMalloc / cudaFree). Arguments, layouts
 * and results are those of hs2_topk_select.
 *  - The first call on each device looks up the scratch array's device address (with that
 *    device current) and caches it; make that first call before any stream capture.
 *  - Calls whose selection needs more scratch than the array holds (many long rows split over
 *    several CTAs) return HS2_ERR_WORKSPACE with the required size; use hs2_topk_select then.
 *  - All calls share the one array and it keeps the last call's contents (the parts that must
 *    start at zero are cleared on the stream at the start of each call). Calls that can
 *    overlap on the GPU -- on different streams, or from different host threads -- race on it
 *    and must be serialised by the caller.
 *  - The one error the selection kernels detect themselves (a negative or NaN candidate score,
 *    see hs2_topk_select; the selection has no waits that could run out) goes to a status word
 *    in the array: read it with hs2_noalloc_read_status (hs2_read_device_status needs a
 *    workspace). Each call clears it when it starts. */
hs2_status hs2_topk_select_noalloc(const hs2_kv_view *kv, const float *scores,
                                   int64_t score_stride, int32_t topk, int32_t window,
                                   int32_t *idx, int32_t idx_stride, int32_t *count,
                                   void *stream);

/* Synchronises `stream`, then returns the status the last hs2_topk_select_noalloc call on the
 * current device recorded in the built-in array (HS2_OK, or HS2_ERR_DEVICE_CHECK for a negative
 * or NaN candidate score) and clears it. HS2_ERR_CUDA if the read fails. Like the selection, it
 * calls no allocator; it races with a selection still running on another stream. */
hs2_status hs2_noalloc_read_status(void *stream);

/* Block-level variant of step 2: the granularity HySparse used and HySparse2 replaces
 * ("HySparse2: How Xiaomi Split the Transformer to Fix Agent Prefill Costs", section "KV Reuse and
 * Token-Level Sparse Selection": blocks of 64 tokens at the token variant's budget). For query
 * row r at position p, with C = [0, nc), nc = max(0, p - window + 1), and W = [nc, p] as in
 * hs2_topk_select: C is cut at multiples of block_size into blocks
 * [j * block_size, min((j + 1) * block_size, nc)); a block's score is the float32 sum of its
 * candidates' scores taken by folding the block in half (v[i] + v[i + n/2] for n = block_size,
 * ..., 2, zeros past nc), a fixed order; the topk / block_size blocks with the largest score
 * (ties: lower block index) are kept, their positions ascending, then W. If nc <= topk the
 * selection is [0, p]. block_size: 16, 32, 64 or 128, dividing topk. The output (idx, count,
 * idx_stride) has the layout of hs2_topk_select, so hs2_sparse_gather_attn consumes it as it
 * is; count[r] is topk + |W| unless the chosen blocks include a short last block. workspace:
 * device, 256-byte aligned, at least hs2_topk_select_blocks_workspace_size bytes (block scores
 * of every row); its contents on entry do not matter. Asynchronous on `stream`; argument errors
 * return before any launch. */
hs2_status hs2_topk_select_blocks_workspace_size(const hs2_kv_view *kv, int32_t block_size,
                                                 int32_t topk, int32_t window, size_t *bytes);
hs2_status hs2_topk_select_blocks(const hs2_kv_view *kv, const float *scores,
                                  int64_t score_stride, int32_t block_size, int32_t topk,
                                  int32_t window, int32_t *idx, int32_t idx_stride,
                                  int32_t *count, void *workspace, size_t workspace_bytes,
                                  void *stream);

/* Synchronises `stream` and returns the status the kernels of the last call on this workspace
 * recorded: HS2_OK, HS2_ERR_TIMEOUT or HS2_ERR_DEVICE_CHECK (HS2_ERR_CUDA if the read fails). */
hs2_status hs2_read_device_status(const void *workspace, void *stream);

/* Message for the last non-OK status returned on the calling thread ("" if none). */
const char *hs2_last_error(void);
const char *hs2_status_string(hs2_status status);
int32_t hs2_version(void);

/* Appends the n_q new tokens of every sequence to the shared cache ("HySparse2: Hybrid Sparse
 * Attention with Two-Level KV Sharing", "Inference cost": one FP8 K/V head shared by all query
 * heads; the step before the block, since the window and the sparse layers read this cache).
 * Cache row kv_start[b] + kv_len[b] - n_q + i (the sequence's last n_q rows, which kv_len
 * already counts) receives new_k[b][i][:] and new_v[b][i][:] (device, bf16 [batch, n_q, 128],
 * 16-byte aligned). bf16 cache: copied. e4m3 cache: per row and matrix, scale = max|x| / 448 in
 * float32 (1 for an all-zero row) is written to k_scale / v_scale and the codes are the
 * round-to-nearest-even e4m3 of the float32 quotient x / scale (IEEE division, correctly
 * rounded), saturated at 448. The view's K/V (and scale) buffers
 * are written: they are caller-owned device memory. Asynchronous on `stream`; argument errors
 * return before any launch. */
hs2_status hs2_kv_append(const hs2_kv_view *kv, const void *new_k, const void *new_v, void *stream);

/* ---- Context-parallel decode: one sequence's cache split by token range over ranks ----------
 * A rank holds rows [off, off + T_local) of a sequence whose decode query sits at global position
 * T_global - 1, as an ordinary view of T_local rows (n_q = 1; the local query position is then
 * its last row, and every local row precedes the query). One block step is:
 *   1. hs2_full_attn on the shard -> (O_r, lse_r); all-gather; hs2_lse_merge -> O, lse;
 *   2. hs2_score_pass on the shard with the merged lse -> the shard's scores (global scores of
 *      its positions); hs2_topk_select on the shard with the local window
 *      T_local - clamp(T_global - window - off, 0, T_local) -> its top-k;
 *      hs2_cp_pack_candidates -> its (score, global position) keys; all-gather;
 *      hs2_cp_merge_select -> the global selection S (the same on every rank);
 *   3. per sparse layer: hs2_cp_localize (S -> the shard's positions in S),
 *      hs2_sparse_gather_attn_partial -> (O_r, lse_r); all-gather; hs2_lse_merge -> O.
 * Attention over a union of disjoint position sets is the log-sum-exp merge of the parts, the
 * score of a position needs only the global lse, and the global top-k lies inside the union of
 * the shards' own top-k, so the result equals one GPU's over the whole context (up to the
 * float rounding of the merges; the selection is exact on the scores the ranks computed).
 * "HySparse2: Hybrid Sparse Attention with Two-Level KV Sharing", bullet "Inference cost" (1M-token
 * contexts). The collectives are the caller's (torch.distributed over NCCL). */

/* Step 1 alone (decode, n_q = 1): out and lse as hs2_full_attn_scores, no scores. */
hs2_status hs2_full_attn(const hs2_kv_view *kv, const void *q, float softmax_scale, void *out,
                         int32_t out_dtype, float *lse, void *workspace, size_t workspace_bytes,
                         void *stream);

/* The score pass alone (decode, n_q = 1) with a given lse (device fp32 [B, H], e.g. merged over
 * context shards): scores[b * score_stride + t] = sum_h exp(c q_h.k_t - lse[b, h]), t < kv_len[b]. */
hs2_status hs2_score_pass(const hs2_kv_view *kv, const void *q, float softmax_scale,
                          const float *lse, float *scores, int64_t score_stride, void *workspace,
                          size_t workspace_bytes, void *stream);

/* hs2_sparse_gather_attn with fp32 out and the log-sum-exp of the attended scores in lse
 * (device fp32 [B * n_q, H]); count[r] may be 0 (out = 0, lse = -inf). */
hs2_status hs2_sparse_gather_attn_partial(const hs2_kv_view *kv, const void *q,
                                          const int32_t *idx, int32_t idx_stride,
                                          const int32_t *count, float softmax_scale, float *out,
                                          float *lse, void *workspace, size_t workspace_bytes,
                                          void *stream);

/* Log-sum-exp merge of n_parts attention results over disjoint position sets:
 *   M = max_j lse_j, w_j = exp(lse_j - M), out = sum_j w_j out_j / sum_j w_j,
 *   lse = M + log sum_j w_j   (parts with lse = -inf contribute nothing; all empty: 0, -inf).
 * part_out: device fp32 [n_parts, rows, H, 128]; part_lse: device fp32 [n_parts, rows, H];
 * out: device [rows, H, 128] of out_dtype; lse: device fp32 [rows, H] or NULL. */
hs2_status hs2_lse_merge(int32_t n_parts, int64_t rows, int32_t n_heads, const float *part_out,
                         const float *part_lse, void *out, int32_t out_dtype, float *lse,
                         void *stream);

/* A shard's selected candidates as keys for the global merge: for entries j < count[b] of the
 * shard's own selection idx[b] (local positions), global position g = global_offset[b] + idx,
 * kept if g < global_len[b] - window (a global candidate); key = (fp32 bits of the score) << 32 |
 * (0xffffffff - g), so larger keys are higher scores, then lower positions. keys: device u64
 * [B, topk], unused slots 0. global_offset / global_len: HOST [B]. */
hs2_status hs2_cp_pack_candidates(const hs2_kv_view *kv, const int64_t *global_offset,
                                  const int32_t *global_len, const float *scores,
                                  int64_t score_stride, const int32_t *idx, int32_t idx_stride,
                                  const int32_t *count, int32_t topk, int32_t window,
                                  uint64_t *keys, void *stream);

/* The global selection from every shard's keys (device u64 [n_parts, batch, topk], n_parts x topk
 * <= 16384, part j being the shard that holds the j-th range of positions, each part's keys in
 * position order as hs2_cp_pack_candidates writes them): with p = global_len[b] - 1 and nc = max(0, p - window + 1), all of [0, p] if
 * nc <= topk, else the topk largest keys' positions ascending, then [nc, p] -- what
 * hs2_topk_select gives on the whole context's scores. idx: device int32 [batch, idx_stride]
 * (global positions), count: device int32 [batch]. global_len: HOST [batch]. */
hs2_status hs2_cp_merge_select(int32_t n_parts, int32_t batch, const int32_t *global_len,
                               const uint64_t *keys, int32_t topk, int32_t window, int32_t *idx,
                               int32_t idx_stride, int32_t *count, void *stream);

/* The shard's part of an ascending global selection: entries g in [global_offset[b],
 * global_offset[b] + local_len[b]) as local positions g - global_offset[b], in order (a
 * contiguous run), count_local[b] of them (possibly 0). global_offset / local_len: HOST [batch]. */
hs2_status hs2_cp_localize(int32_t batch, const int64_t *global_offset, const int32_t *local_len,
                           const int32_t *idx, int32_t idx_stride, const int32_t *count,
                           int32_t *idx_local, int32_t idx_local_stride, int32_t *count_local,
                           void *stream);

/* KV Bridging ("HySparse2: How Xiaomi Split the Transformer to Fix Agent Prefill Costs", section
 * "The Self-Decoder and Cross-Decoder Split": the cross-decoder full layer's cache is built from a
 * self-decoder full layer's hidden states, K_j = Proj_j^K(H_i^self), V_j = Proj_j^V(H_i^self);
 * the projections are taken as linear maps without bias). For the n_q last tokens of every
 * sequence (the rows hs2_kv_append writes):
 *   K = hidden . W_K^T,  V = hidden . W_V^T   (bf16 inputs, float32 accumulation on the tensor
 *   cores), rounded to bf16 and written to cache row kv_start[b] + kv_len[b] - n_q + i: as bf16,
 *   or, for an e4m3 cache, quantised from that bf16 row exactly as hs2_kv_append does.
 * hidden: device bf16 [batch, n_q, d_model], 16-byte aligned. w_kv: device bf16 [256, d_model],
 * rows 0..127 W_K and rows 128..255 W_V (output feature x input feature), 16-byte aligned.
 * d_model: a multiple of 64 in [64, 32768]. workspace: device, 256-byte aligned, >= 256 bytes
 * (the status word hs2_read_device_status reads). The view's K/V (and scale) buffers are
 * written. Asynchronous on `stream`; argument errors return before any launch. */
hs2_status hs2_kv_bridge(const hs2_kv_view *kv, const void *hidden, int32_t d_model,
                         const void *w_kv, void *workspace, size_t workspace_bytes, void *stream);

/* Exercises the bounded waits of the kernels: one thread waits on an mbarrier that nothing
 * arrives at, gives up after limit_us microseconds (1 .. 2e6) and records HS2_ERR_TIMEOUT in the
 * status word at the start of `workspace` (device, 256-byte aligned, >= 256 bytes), which the
 * call clears first; hs2_read_device_status then reports HS2_ERR_TIMEOUT and the context stays
 * usable. With workspace NULL and workspace_bytes 0 the status word is the one inside the
 * built-in array of hs2_topk_select_noalloc, which hs2_noalloc_read_status then reports (the
 * same end-to-end check for callers that cannot allocate). Not part of the method: a
 * failure-detection check. Returns HS2_ERR_WORKSPACE / HS2_ERR_INVALID_ARG on bad arguments
 * (nothing launched), HS2_ERR_CUDA on a launch error. */
hs2_status hs2_selftest_wait_timeout(uint32_t limit_us, void *workspace, size_t workspace_bytes,
                                     void *stream);

/* Evaluates, for the n device floats x (n >= 0), y[i] = the 2^x[i] that the tensor-core score
 * passes compute on the FMA pipe for part of their exponentials: x clamped at -125, split as
 * j + f with j = rint(x) and |f| <= 1/2, 2^f from a cubic fitted for minimal relative error on
 * [-1/2, 1/2] (Remez), 2^j added to the exponent. Relative error at most 7.5e-5 for
 * x in [-125, 0]. Not part of the method: a check of that approximation. Asynchronous on
 * `stream`; HS2_ERR_INVALID_ARG on NULL pointers or n out of range (nothing launched). */
hs2_status hs2_selftest_exp2(const float *x, float *y, int64_t n, void *stream);

/* Number of kernels this library has launched in the calling process since it was loaded
 * (successful launches only; the workspace clears done with cudaMemsetAsync are not counted).
 * Not part of the method: an accounting aid for callers that count launches per call. */
uint64_t hs2_launch_count(void);

#ifdef __cplusplus
}
#endif
#endif /* HS2_H_ */
