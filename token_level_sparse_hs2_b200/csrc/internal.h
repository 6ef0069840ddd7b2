// internal.h -- launch parameters shared by the C-ABI layer (hs2_api.cu) and the kernels.
// Everything a kernel needs travels by value in its parameter block (no device-side tables),
// so every launch is self-contained and capturable.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/hs2.h"

namespace hs2 {

constexpr int kHeadDim = 128;
constexpr int kTile = 64;             // cache rows per pipeline tile
constexpr int kHistBins = 2048;
// A split partial row: [max (log2 units), denominator, 2 pad, unnormalised output x 128];
// 132 floats keep the output 16-byte aligned.
constexpr int kPartRow = 4 + 128;
constexpr int kPartO = 4;       // top radix digit: bits [31:21] of the fp32 score
// decode pass 1: partial slots per (CTA, sequence) -- one per token group of consumer warps
constexpr int decode_slots_per_cta(int) { return 1; }   // warps merge in shared memory first

// device status bits (written into the workspace, read by hs2_read_device_status)
constexpr uint32_t kStatusTimeout = 1u;
constexpr uint32_t kStatusCheck = 2u;

// Per-sequence geometry. Work items (or partial slots) of sequence b are
// [item_begin[b], item_begin[b+1]); its 64-row tiles are [tile_begin[b], tile_begin[b+1]) of
// the concatenated tile list of all sequences.
struct SeqTable {
  int64_t start[HS2_MAX_BATCH];
  int32_t len[HS2_MAX_BATCH];
  int32_t item_begin[HS2_MAX_BATCH + 1];
  int32_t tile_begin[HS2_MAX_BATCH + 1];
};

// Decode (n_q == 1): full-attention pass 1 (PASS 0) and score pass 2 (PASS 1). A persistent
// grid of n_ctas CTAs; CTA i streams tiles [i*T/n_ctas, (i+1)*T/n_ctas) of the concatenated
// list (T = total_tiles). Pass-1 partial slots of sequence b start at seq.item_begin[b]: 4 per
// CTA that touches b.
struct DecodeParams {
  SeqTable seq;
  int32_t batch, n_heads;
  int32_t total_tiles;
  int32_t n_ctas;           // pass-1 grid (partial slots are laid out for it)
  int32_t n_ctas2;          // pass-2 grid
  int32_t window;           // pass 2: positions < p - window + 1 are top-k candidates
  float scale_log2;         // softmax_scale * log2(e)
  int64_t kv_rows;
  const float *k_scale;     // FP8 per-token scales (null for bf16)
  const float *v_scale;
  const void *q;            // bf16 [B, H, 128]
  void *out;                // [B, H, 128], bf16 or fp32 (pass 1)
  int32_t out_f32;
  float *lse;               // [B, H] (written by pass 1, read by pass 2)
  float *scores;            // pass 2: row b at scores + b * score_stride
  int64_t score_stride;
  uint32_t *hist;           // pass 2: [B, kHistBins] counts of candidate top digits, or null
  float *part;              // pass 1: [slots, H, kPartRow] partials
  uint32_t *status;
  uint4 *zero;              // pass 1: clears zero_n16 16-byte words here (the workspace's
  int32_t zero_n16;         // zero-initialised region) once the previous kernel has finished
  // tensor-core decode kernels: 128-row tiles of all sequences, concatenated like the 64-row
  // ones (sequence b's tiles are [tile128_begin[b], tile128_begin[b + 1]))
  int32_t tile128_begin[HS2_MAX_BATCH + 1];
  int32_t total_tiles128;
  // pass 1 with CTAs of each sequence's own (seq_split): sequence b owns CTAs
  // [cta_begin[b], cta_begin[b + 1]), which split its tiles equally, and the partial slot of a
  // CTA is its index; otherwise CTA i owns tiles [i T / G, (i + 1) T / G) of all sequences
  int32_t seq_split;
  int32_t cta_begin[HS2_MAX_BATCH + 1];
};

// Chunk / prefill (n_q > 1). Pass 1: blocks of 128 (query, head) rows (128 / H queries);
// pass 2: blocks of 8 queries. Each block's causal prefix is cut into n_chunks work items.
struct RowsParams {
  SeqTable seq;             // item_begin[b]: first block of sequence b
  int32_t batch, n_q, n_heads;
  int32_t q_per_block;      // queries per block
  int32_t n_chunks;         // kv chunks per block (1 = no split)
  int32_t n_items;          // blocks * n_chunks
  float scale_log2;
  int64_t kv_rows;
  const float *k_scale;     // FP8 per-token scales (null for bf16)
  const float *v_scale;
  const void *q;            // bf16 [B, n_q, H, 128]
  void *out;                // [B, n_q, H, 128]
  int32_t out_f32;
  float *lse;               // [B, n_q, H]
  float *scores;            // row (b * n_q + i) at scores + row * score_stride
  int64_t score_stride;
  float *part;              // pass 1, n_chunks > 1: [blocks, n_chunks, 128, 2 + 128]
  int32_t *counter;         // pass 1: [blocks] arrival counters (self-resetting)
  uint32_t *status;
};

// Sparse gather attention: one CTA per (query row, head group, split of the selected list).
struct SparseParams {
  SeqTable seq;
  int32_t batch, n_q, n_heads;
  int32_t n_tsplit;         // CTAs per row along the selected list (one thread-block cluster)
  int32_t head_groups;      // CTAs (clusters) per row across the heads: 1, or 2 of 16 heads
  int32_t split_len;        // selected entries per CTA (multiple of 64)
  float scale_log2;
  const void *q;            // bf16 [B, n_q, H, 128]
  const int32_t *idx;       // [B*n_q, idx_stride]
  int32_t idx_stride;
  const int32_t *count;     // [B*n_q]
  const void *k, *v;        // cache rows
  const float *k_scale, *v_scale;
  void *out;
  int32_t out_f32;
  uint32_t *status;
  int32_t idx_ready;        // idx / count were complete before the previous kernel started
  int32_t allow_empty;      // count 0 is valid (a context shard holding none of the selection)
  float *lse_out;           // [B*n_q, H] log-sum-exp of the attended scores, or null
};

// Cache append of n_q new rows per sequence (the last n_q rows of each sequence).
struct AppendParams {
  SeqTable seq;
  int32_t batch, n_q, fp8;
  const void *new_k, *new_v;  // bf16 [B, n_q, 128]
  void *k, *v;                // cache rows (bf16 or e4m3)
  float *k_scale, *v_scale;   // e4m3: per-row scales
};
cudaError_t launch_kv_append(const AppendParams &p, cudaStream_t s);

// KV Bridging: cache rows of each sequence's last n_q tokens projected from hidden states
// [B * n_q, d_model] by weights [256, d_model] (K rows 0..127, V rows 128..255).
struct BridgeParams {
  SeqTable seq;
  int32_t batch, n_q, m, d_model, fp8;
  void *k, *v;                // cache rows (bf16 or e4m3)
  float *k_scale, *v_scale;   // e4m3: per-row scales
  uint32_t *status;
};
struct BridgeMaps {
  CUtensorMap h, w;           // hidden [m, d_model], weights [256, d_model]; 64-wide boxes
};
cudaError_t launch_kv_bridge(const BridgeMaps &tm, const BridgeParams &p, int grid, cudaStream_t s);

// Largest thread-block cluster the sparse layer may use for this cache type and head count.
int sparse_max_cluster(int kv_dtype, int n_heads);

// Top-k + window selection: n_seg CTAs per query row, each over seg_len candidate positions.
struct TopkParams {
  SeqTable seq;
  int32_t batch, n_q;
  int32_t topk, window;
  const float *scores;
  int64_t score_stride;
  const uint32_t *hist;     // [B*n_q, kHistBins] top-digit counts from the score pass, or null
  uint32_t *hist_ws;        // [B*n_q, kHistBins] built here when hist is null and n_seg > 1
  int32_t n_seg, seg_len;
  int32_t cluster;          // 1: the n_seg (<= 8) segments of a row are one thread-block cluster
  uint32_t *cand_key;       // [B*n_q, cand_cap] (n_seg > 1)
  int32_t *cand_idx;
  int32_t cand_cap;
  int2 *seg_info;           // [B*n_q, n_seg] (first slot, count) of each segment's run
  int32_t *cand_count;      // [B*n_q] (self-resetting)
  int32_t *arrive;          // [B*n_q] (self-resetting)
  int32_t *idx;
  int32_t idx_stride;
  int32_t *count;
  uint32_t *status;
};

// Block-level selection: pooled block scores, then one CTA per query row.
struct BlockSelParams {
  SeqTable seq;
  int32_t batch, n_q;
  int32_t bs, kb, topk, window;    // block size (16 .. 128), blocks kept = topk / bs
  const float *scores;
  int64_t score_stride;
  float *blk;                      // [B*n_q, blk_stride] float32 block scores
  int64_t blk_stride;
  int32_t pool_ctas_per_row;       // pool grid = rows x this
  int32_t smem_keys;               // rows with at most this many blocks select in shared memory
  int32_t fused;                   // 1: one kernel, each CTA pools its own row (needs every
                                   // row's blocks to fit smem_keys)
  uint32_t *status;                // workspace status word (written 0)
  int32_t *idx;
  int32_t idx_stride;
  int32_t *count;
};
cudaError_t launch_block_select(const BlockSelParams &p, int n_rows, cudaStream_t s);
int block_pool_positions_per_cta();

// Merge of split partials into outputs: one CTA per (group, head). Group g owns partial slots
// [slot_begin(g), slot_begin(g) + n(g)): from seq.item_begin when by_seq, else g * n_fixed.
// Groups with a single slot were written directly by their CTA and are skipped.
struct MergeParams {
  SeqTable seq;
  int32_t by_seq;
  int32_t n_groups, n_fixed, n_heads;
  const float *part;        // [slots, H, kPartRow]
  void *out;                // [groups, H, 128]
  int32_t out_f32;
  float *lse;               // [groups, H] or null
};

// Context-parallel decode (a sequence's cache split by token range over ranks).
constexpr int kCpMaxKeys = 16384;   // parts x topk composites merged in shared memory
struct LseMergeParams {
  int32_t n_parts, n_heads;
  int64_t rows;
  const float *part_o;      // [n_parts, rows, H, 128]
  const float *part_lse;    // [n_parts, rows, H]
  void *out;                // [rows, H, 128]
  int32_t out_f32;
  float *lse;               // [rows, H] or null
};
struct CpParams {
  int32_t batch, n_parts, topk, window;
  int64_t offset[HS2_MAX_BATCH];   // global position of the shard's first row, per sequence
  int32_t local_len[HS2_MAX_BATCH];
  int32_t global_len[HS2_MAX_BATCH];
  const float *scores;
  int64_t score_stride;
  const int32_t *idx;       // [B, idx_stride]
  int32_t idx_stride;
  const int32_t *count;
  uint64_t *keys;           // pack: [B, topk]; select: [n_parts, B, topk] (const)
  int32_t *idx_out;         // select: [B, out_stride] global; localize: [B, out_stride] local
  int32_t out_stride;
  int32_t *count_out;
};
cudaError_t launch_lse_merge(const LseMergeParams &p, cudaStream_t s);
cudaError_t launch_cp_pack(const CpParams &p, cudaStream_t s);
cudaError_t launch_cp_select(const CpParams &p, cudaStream_t s);
cudaError_t launch_cp_localize(const CpParams &p, cudaStream_t s);

struct TensorMaps {
  CUtensorMap k, v;
  CUtensorMap ks, vs;         // e4m3 caches: the per-row scales as 1-D tensors (boxes of 128)
};

// launchers (return cudaGetLastError() of the launch)
cudaError_t launch_decode_pass(int pass, int kv_dtype, const TensorMaps &tm,
                               const DecodeParams &p, cudaStream_t s);
// Tiles per stage of the bf16 decode score pass (one CTA per SM when above 1, else two).
#ifndef HS2_PASS2_SUB
#define HS2_PASS2_SUB 1
#endif
// Score pass 2 at decode time for an e4m3 cache on tcgen05 (128-row tiles; grid p.n_ctas2
// persistent CTAs, one per SM; kv_dtype must be HS2_KV_FP8_E4M3).
cudaError_t launch_decode_score_tc(int kv_dtype, const TensorMaps &tm, const DecodeParams &p,
                                   cudaStream_t s);
cudaError_t launch_rows_pass(int pass, int kv_dtype, const TensorMaps &tm, const RowsParams &p,
                             cudaStream_t s);
cudaError_t launch_sparse(int kv_dtype, const SparseParams &p, cudaStream_t s);
cudaError_t launch_topk(const TopkParams &p, int n_rows, cudaStream_t s);
cudaError_t launch_merge(const MergeParams &p, cudaStream_t s);
// Score pass 2 of a bf16 cache for n_q > 1 on tcgen05 (blocks of rows_score_tc_queries(H)
// queries).
cudaError_t launch_rows_score_tc(const TensorMaps &tm, const RowsParams &p, cudaStream_t s);
int rows_score_tc_queries(int n_heads);
// Output pass 1 of a bf16 cache for n_q > 1 on tcgen05 (blocks of 128 / H queries, the chunk
// partials and counters of RowsParams).
cudaError_t launch_rows_attn_tc(const TensorMaps &tm, const RowsParams &p, cudaStream_t s);

// Counts one successful kernel launch (every launch of the library goes through launch_pdl).
void note_launch();
unsigned long long launches_so_far();

}  // namespace hs2
