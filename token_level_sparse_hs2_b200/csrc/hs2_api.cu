// hs2_api.cu -- the C ABI of libhs2 (declared in include/hs2.h): argument validation on the
// host, the work plan (how each step is split over CTAs), workspace carving, TMA descriptors
// and the launch sequence of one hybrid block:
//   full-attention pass 1 -> score pass 2 -> top-k + window -> sparse layer x n_sparse.
// Nothing here allocates, synchronises or keeps state between calls.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <functional>
#include <mutex>

#include "attn_tile.cuh"
#include "common.cuh"
#include "internal.h"

namespace hs2 {
namespace {
std::atomic<unsigned long long> g_launches{0};
}
void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }
unsigned long long launches_so_far() { return g_launches.load(std::memory_order_relaxed); }
}  // namespace hs2

namespace hs2 {

namespace {

thread_local char g_err[512] = "";

hs2_status fail(hs2_status st, const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof g_err, fmt, ap);
  va_end(ap);
  return st;
}

hs2_status ok() {
  g_err[0] = '\0';
  return HS2_OK;
}

constexpr int kTargetItems = 4 * 148;     // chunk work items per pass (~4 per SM)
constexpr int kMaxStreamCtas = 296;       // persistent decode grid, at most
constexpr int kSegLen = 16384;            // top-k candidates per CTA when rows are split
constexpr int kManyRows = 148;            // rows at least this many: one CTA per row
constexpr int kCandCapGlobal = 8192;
constexpr int kMaxSplit = 16;             // sparse-layer CTAs (one cluster) per query row, at most
constexpr int kRowsPerBlock = 128;        // (query, head) rows per pass-1 CTA for chunks
constexpr int kQueriesPass2 = 8;          // queries per pass-2 CTA for chunks
constexpr size_t kAlign = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }
bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Work plan and workspace layout for one view.
struct Plan {
  int B = 0, n_q = 0, H = 0, kv_dtype = 0;
  int64_t kv_rows = 0, max_p = 0;
  int n_rows = 0;
  // decode passes: concatenated 64-row tile list of all sequences
  int total_tiles = 0;
  int32_t tile_begin[HS2_MAX_BATCH + 1] = {};
  // multi-token chunks: pass-1 blocks of 128 / H queries, pass-2 blocks of 8 queries
  int32_t blk1_begin[HS2_MAX_BATCH + 1] = {}, blk2_begin[HS2_MAX_BATCH + 1] = {};
  int n_blk1 = 0, n_chunks1 = 1, n_blk2 = 0, n_chunks2 = 1;
  // top-k
  int n_seg = 1, seg_len = 0;
  // sparse layers: n_split chosen per call from the index capacity
  bool sparse_split = false;
  // workspace (byte offsets); [0, zero_end) is cleared at the start of every call
  size_t off_status = 0, off_cnt_rows = 0, off_hist = 0, off_cand_count = 0, off_arrive = 0,
         zero_end = 0;
  size_t off_part_p1 = 0, off_part_rows = 0, off_cand_key = 0, off_cand_idx = 0,
         off_seg_info = 0, total = 0;
};

hs2_status validate_view(const hs2_kv_view *kv) {
  if (!kv) return fail(HS2_ERR_INVALID_ARG, "kv view is NULL");
  if (kv->batch < 1 || kv->batch > HS2_MAX_BATCH)
    return fail(HS2_ERR_INVALID_ARG, "batch %d outside [1, %d]", kv->batch, HS2_MAX_BATCH);
  if (kv->n_q < 1) return fail(HS2_ERR_INVALID_ARG, "n_q %d < 1", kv->n_q);
  if (kv->head_dim != HS2_HEAD_DIM)
    return fail(HS2_ERR_UNSUPPORTED, "head_dim %d (only 128 is supported)", kv->head_dim);
  if (kv->n_heads != 16 && kv->n_heads != 32)
    return fail(HS2_ERR_UNSUPPORTED, "n_heads %d (16 or 32 query heads per K/V head)", kv->n_heads);
  if (kv->kv_dtype != HS2_KV_BF16 && kv->kv_dtype != HS2_KV_FP8_E4M3)
    return fail(HS2_ERR_INVALID_ARG, "kv_dtype %d", kv->kv_dtype);
  if (kv->reserved != 0) return fail(HS2_ERR_INVALID_ARG, "reserved field must be 0");
  if (kv->kv_rows < 1 || kv->kv_rows > (int64_t)INT32_MAX - 2 * 64)
    return fail(HS2_ERR_INVALID_ARG, "kv_rows %lld out of range", (long long)kv->kv_rows);
  if (!kv->k || !kv->v) return fail(HS2_ERR_INVALID_ARG, "k / v is NULL");
  if (!aligned16(kv->k) || !aligned16(kv->v))
    return fail(HS2_ERR_INVALID_ARG, "k / v must be 16-byte aligned");
  if (kv->kv_dtype == HS2_KV_FP8_E4M3) {
    if (!kv->k_scale || !kv->v_scale)
      return fail(HS2_ERR_INVALID_ARG, "FP8 cache needs k_scale and v_scale");
    if (!aligned16(kv->k_scale) || !aligned16(kv->v_scale))
      return fail(HS2_ERR_INVALID_ARG, "k_scale / v_scale must be 16-byte aligned");
  }
  if (!kv->kv_start || !kv->kv_len) return fail(HS2_ERR_INVALID_ARG, "kv_start / kv_len is NULL");
  for (int b = 0; b < kv->batch; ++b) {
    const int64_t s = kv->kv_start[b];
    const int32_t T = kv->kv_len[b];
    if (T < kv->n_q)
      return fail(HS2_ERR_INVALID_ARG, "kv_len[%d] = %d < n_q = %d", b, T, kv->n_q);
    if (s < 0 || s + T > kv->kv_rows)
      return fail(HS2_ERR_INVALID_ARG, "sequence %d rows [%lld, %lld) outside [0, %lld)", b,
                  (long long)s, (long long)(s + T), (long long)kv->kv_rows);
  }
  return HS2_OK;
}

void make_plan(const hs2_kv_view *kv, Plan &P) {
  P.B = kv->batch;
  P.n_q = kv->n_q;
  P.H = kv->n_heads;
  P.kv_dtype = kv->kv_dtype;
  P.kv_rows = kv->kv_rows;
  P.n_rows = P.B * P.n_q;
  P.max_p = 0;
  P.total_tiles = 0;
  for (int b = 0; b < P.B; ++b) {
    P.max_p = std::max<int64_t>(P.max_p, kv->kv_len[b] - 1);
    const int64_t r0 = kv->kv_start[b], r1 = r0 + kv->kv_len[b];
    P.tile_begin[b] = P.total_tiles;   // decode: tiles of every sequence, concatenated
    P.total_tiles += (int)((r1 + kTile - 1) / kTile - r0 / kTile);
  }
  P.tile_begin[P.B] = P.total_tiles;
  // multi-token chunks
  if (P.n_q > 1) {
    const int qpb1 = kRowsPerBlock / P.H;
    const int qpb2 = (P.kv_dtype == HS2_KV_BF16) ? rows_score_tc_queries(P.H) : kQueriesPass2;
    P.n_blk1 = P.n_blk2 = 0;
    for (int b = 0; b < P.B; ++b) {
      P.blk1_begin[b] = P.n_blk1;
      P.blk2_begin[b] = P.n_blk2;
      P.n_blk1 += (P.n_q + qpb1 - 1) / qpb1;
      P.n_blk2 += (P.n_q + qpb2 - 1) / qpb2;
    }
    P.blk1_begin[P.B] = P.n_blk1;
    P.blk2_begin[P.B] = P.n_blk2;
    P.n_chunks1 = std::max(1, std::min(64, (kTargetItems + P.n_blk1 - 1) / P.n_blk1));
    P.n_chunks2 = std::max(1, std::min(64, (kTargetItems + P.n_blk2 - 1) / P.n_blk2));
  }
  // top-k segments: split long rows when there are few of them
  const int64_t max_cand = P.max_p + 1;
  if (P.n_rows >= kManyRows) {
    P.n_seg = 1;
  } else {
    P.n_seg = (int)std::min<int64_t>(256, std::max<int64_t>(1, (max_cand + kSegLen - 1) / kSegLen));
  }
  P.seg_len = (int)((max_cand + P.n_seg - 1) / P.n_seg);
  P.sparse_split = P.n_rows < 2 * kManyRows;

  // workspace layout
  size_t o = 0;
  P.off_status = o; o = align_up(o + 4);
  P.off_cnt_rows = o; o = align_up(o + 4 * (size_t)P.n_blk1);
  P.off_hist = o; o = align_up(o + (P.n_seg > 1 ? 4 * (size_t)kHistBins * P.n_rows : 0));
  P.off_cand_count = o; o = align_up(o + 4 * (size_t)P.n_rows);
  P.off_arrive = o; o = align_up(o + 4 * (size_t)P.n_rows);
  P.zero_end = o;
  const size_t part_row = (size_t)P.H * kPartRow * 4;
  const size_t max_slots =
      (size_t)decode_slots_per_cta(P.H) * ((size_t)std::min(kMaxStreamCtas, P.total_tiles) + P.B);
  P.off_part_p1 = o; o = align_up(o + (P.n_q == 1 ? part_row * max_slots : 0));
  P.off_part_rows = o;
  o = align_up(o + (P.n_chunks1 > 1 ? (size_t)P.n_blk1 * P.n_chunks1 * kRowsPerBlock * kPartRow * 4 : 0));
  const size_t cand = (P.n_seg > 1) ? (size_t)P.n_rows * kCandCapGlobal * 4 : 0;
  P.off_cand_key = o; o = align_up(o + cand);
  P.off_cand_idx = o; o = align_up(o + cand);
  P.off_seg_info = o; o = align_up(o + (P.n_seg > 1 ? (size_t)P.n_rows * P.n_seg * 8 : 0));
  P.total = o;
}

void fill_seq(const hs2_kv_view *kv, const Plan &P, SeqTable &t) {
  memset(&t, 0, sizeof t);
  for (int b = 0; b < P.B; ++b) {
    t.start[b] = kv->kv_start[b];
    t.len[b] = kv->kv_len[b];
    t.tile_begin[b] = P.tile_begin[b];
  }
  t.tile_begin[P.B] = P.tile_begin[P.B];
}

hs2_status check_ws(const Plan &P, void *ws, size_t bytes) {
  if (!ws) return fail(HS2_ERR_INVALID_ARG, "workspace is NULL");
  if (reinterpret_cast<uintptr_t>(ws) % kAlign)
    return fail(HS2_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  if (bytes < P.total)
    return fail(HS2_ERR_WORKSPACE, "workspace %zu bytes < %zu required", bytes, P.total);
  return HS2_OK;
}

template <class T>
T *ws_at(void *ws, size_t off) {
  return reinterpret_cast<T *>(static_cast<uint8_t *>(ws) + off);
}

// ------------------------------------------------------------------ TMA descriptors

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

hs2_status get_encoder() {
  std::call_once(g_encode_once, [] {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  if (!g_encode) return fail(HS2_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  return HS2_OK;
}

hs2_status encode_maps(const hs2_kv_view *kv, TensorMaps &tm) {
  hs2_status st = get_encoder();
  if (st != HS2_OK) return st;
  memset(&tm, 0, sizeof tm);
  const cuuint32_t estr[2] = {1, 1};
  CUresult r;
  if (kv->kv_dtype == HS2_KV_BF16) {
    const cuuint64_t dims[2] = {128, (cuuint64_t)kv->kv_rows};
    const cuuint64_t strides[1] = {256};
    const cuuint32_t box[2] = {64, (cuuint32_t)kTile};
    for (int which = 0; which < 2; ++which) {
      r = g_encode(which ? &tm.v : &tm.k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                   const_cast<void *>(which ? kv->v : kv->k), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
      if (r != CUDA_SUCCESS) return fail(HS2_ERR_CUDA, "cuTensorMapEncodeTiled(K/V bf16) = %d", (int)r);
    }
  } else {
    const cuuint64_t dims[2] = {128, (cuuint64_t)kv->kv_rows};
    const cuuint64_t strides[1] = {128};
    const cuuint32_t box[2] = {128, (cuuint32_t)kTile};
    for (int which = 0; which < 2; ++which) {
      r = g_encode(which ? &tm.v : &tm.k, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
                   const_cast<void *>(which ? kv->v : kv->k), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
      if (r != CUDA_SUCCESS) return fail(HS2_ERR_CUDA, "cuTensorMapEncodeTiled(K/V e4m3) = %d", (int)r);
    }
    // the per-row scales, 128 rows per box (rows past kv_rows read as zero)
    const cuuint64_t sdims[1] = {(cuuint64_t)kv->kv_rows};
    const cuuint64_t sstrides[1] = {4};
    const cuuint32_t sbox[1] = {128};
    for (int which = 0; which < 2; ++which) {
      r = g_encode(which ? &tm.vs : &tm.ks, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 1,
                   const_cast<float *>(which ? kv->v_scale : kv->k_scale), sdims, sstrides, sbox,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
      if (r != CUDA_SUCCESS) return fail(HS2_ERR_CUDA, "cuTensorMapEncodeTiled(scales) = %d", (int)r);
    }
  }
  return HS2_OK;
}

hs2_status encode_bridge_maps(const void *hidden, int64_t m, int d_model, const void *w,
                              BridgeMaps &tm) {
  hs2_status st = get_encoder();
  if (st != HS2_OK) return st;
  memset(&tm, 0, sizeof tm);
  const cuuint32_t estr[2] = {1, 1};
  const cuuint64_t strides[1] = {(cuuint64_t)d_model * 2};
  const cuuint64_t hdims[2] = {(cuuint64_t)d_model, (cuuint64_t)m};
  const cuuint32_t hbox[2] = {64, 128};
  CUresult r = g_encode(&tm.h, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(hidden),
                        hdims, strides, hbox, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(HS2_ERR_CUDA, "cuTensorMapEncodeTiled(hidden) = %d", (int)r);
  const cuuint64_t wdims[2] = {(cuuint64_t)d_model, 256};
  const cuuint32_t wbox[2] = {64, 256};
  r = g_encode(&tm.w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(w), wdims, strides,
               wbox, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(HS2_ERR_CUDA, "cuTensorMapEncodeTiled(weights) = %d", (int)r);
  return HS2_OK;
}

hs2_status cuda_check(cudaError_t e, const char *what) {
  if (e != cudaSuccess) return fail(HS2_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return HS2_OK;
}

// ------------------------------------------------------------------ built-in selection scratch
// Backing store of hs2_topk_select_noalloc for callers that cannot allocate. In host code the
// name below is only a host-side stand-in for the device variable: a kernel must be given the
// device address that cudaGetSymbolAddress returns, looked up once per device (with that
// device current) and cached.

static __device__ __align__(256) uint8_t g_noalloc_scratch[HS2_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void *g_noalloc_ptr[kMaxDevices] = {};

hs2_status noalloc_scratch(void **out) {
  int dev = -1;
  hs2_status st = cuda_check(cudaGetDevice(&dev), "cudaGetDevice");
  if (st != HS2_OK) return st;
  if (dev < 0 || dev >= kMaxDevices) return fail(HS2_ERR_UNSUPPORTED, "device %d", dev);
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void *p = nullptr;
    st = cuda_check(cudaGetSymbolAddress(&p, g_noalloc_scratch), "cudaGetSymbolAddress(scratch)");
    if (st != HS2_OK) return st;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return HS2_OK;
}

// Compact layout of the selection's scratch: [status, counters, histograms] are cleared per
// call, candidate buffers are not.
struct NoallocLayout {
  size_t off_status, off_cand_count, off_arrive, off_hist, zero_end, off_cand_key, off_cand_idx,
      off_seg_info,
      total;
};

NoallocLayout noalloc_layout(const Plan &P) {
  NoallocLayout L;
  size_t o = 0;
  L.off_status = o; o = align_up(o + 4);
  L.off_cand_count = o; o = align_up(o + 4 * (size_t)P.n_rows);
  L.off_arrive = o; o = align_up(o + 4 * (size_t)P.n_rows);
  L.off_hist = o; o = align_up(o + (P.n_seg > 1 ? 4 * (size_t)kHistBins * P.n_rows : 0));
  L.zero_end = o;
  const size_t cand = (P.n_seg > 1) ? (size_t)P.n_rows * kCandCapGlobal * 4 : 0;
  L.off_cand_key = o; o = align_up(o + cand);
  L.off_cand_idx = o; o = align_up(o + cand);
  L.off_seg_info = o; o = align_up(o + (P.n_seg > 1 ? (size_t)P.n_rows * P.n_seg * 8 : 0));
  L.total = o;
  return L;
}

bool valid_scale(float s) { return std::isfinite(s) && s > 0.f; }

// largest sparse-layer cluster on the current device (cached per device, cache type, heads)
hs2_status sparse_cluster_limit(int kv_dtype, int n_heads, int *out) {
  static std::mutex mu;
  static int cache[64][2][2] = {};
  int dev = 0;
  hs2_status st = cuda_check(cudaGetDevice(&dev), "cudaGetDevice");
  if (st != HS2_OK) return st;
  const int kd = kv_dtype == HS2_KV_BF16 ? 0 : 1, hg = n_heads == 16 ? 0 : 1;
  std::lock_guard<std::mutex> lock(mu);
  if (dev < 0 || dev >= 64) {
    *out = 1;
    return HS2_OK;
  }
  if (cache[dev][kd][hg] == 0) cache[dev][kd][hg] = sparse_max_cluster(kv_dtype, n_heads);
  *out = cache[dev][kd][hg];
  return HS2_OK;
}

// multiprocessors of the current device (cached per device)
hs2_status sm_count(int *out) {
  static std::mutex mu;
  static int cache[64] = {};
  int dev = 0;
  hs2_status st = cuda_check(cudaGetDevice(&dev), "cudaGetDevice");
  if (st != HS2_OK) return st;
  std::lock_guard<std::mutex> lock(mu);
  if (dev >= 0 && dev < 64 && cache[dev] > 0) {
    *out = cache[dev];
    return HS2_OK;
  }
  int n = 0;
  st = cuda_check(cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev), "SM count");
  if (st != HS2_OK) return st;
  if (dev >= 0 && dev < 64) cache[dev] = n;
  *out = n;
  return HS2_OK;
}

// ------------------------------------------------------------------ steps

// Pass 1 can give every sequence of a batch CTAs of its own: a CTA whose tiles cross a sequence
// boundary stops all its warps for a mid-range flush of their partials and a new query, which
// measured about the time of seven tiles, so the split is taken whenever no CTA gets more than
// three tiles above the contiguous split's share. CTAs go to sequences by their tiles (at least
// one each, never more than the sequence has tiles, the rest by largest remainder); the grid
// is the number of CTAs handed out. cta_begin gets B + 1 prefix offsets.
static bool pass1_seq_split(int B, const int32_t *tb, int G, int32_t *cta_begin) {
  const int T = tb[B];
  if (B < 2 || B > G || T < 1) return false;
  int n[HS2_MAX_BATCH];
  double rem[HS2_MAX_BATCH];
  int used = 0;
  for (int b = 0; b < B; ++b) {
    const int nt = tb[b + 1] - tb[b];
    if (nt < 1) return false;
    const double share = (double)G * nt / T;
    n[b] = std::min(nt, std::max(1, (int)share));
    rem[b] = share - n[b];
    used += n[b];
  }
  if (used > G) return false;
  while (used < G) {
    int best = -1;
    for (int b = 0; b < B; ++b)
      if (n[b] < tb[b + 1] - tb[b] && (best < 0 || rem[b] > rem[best])) best = b;
    if (best < 0) break;
    ++n[best];
    rem[best] -= 1.0;
    ++used;
  }
  int most = 0;
  for (int b = 0; b < B; ++b) most = std::max(most, (tb[b + 1] - tb[b] + n[b] - 1) / n[b]);
  if (most > (T + G - 1) / G + 3) return false;
  cta_begin[0] = 0;
  for (int b = 0; b < B; ++b) cta_begin[b + 1] = cta_begin[b] + n[b];
  return true;
}

hs2_status run_full(const hs2_kv_view *kv, const Plan &P, const TensorMaps &tm, const void *q,
                    float scale, void *out, int out_f32, float *lse, float *scores,
                    int64_t score_stride, int window, bool with_hist, void *ws,
                    cudaStream_t stream, const std::function<hs2_status()> *mark = nullptr,
                    bool clear_in_pass1 = false, int passes = 3) {
  if (P.n_q != 1) {
    RowsParams rp;
    memset(&rp, 0, sizeof rp);
    rp.batch = P.B;
    rp.n_q = P.n_q;
    rp.n_heads = P.H;
    rp.scale_log2 = scale * 1.4426950408889634f;
    rp.kv_rows = kv->kv_rows;
    rp.k_scale = kv->k_scale;
    rp.v_scale = kv->v_scale;
    rp.q = q;
    rp.out = out;
    rp.out_f32 = out_f32;
    rp.lse = lse;
    rp.scores = scores;
    rp.score_stride = score_stride;
    rp.part = ws_at<float>(ws, P.off_part_rows);
    rp.counter = ws_at<int32_t>(ws, P.off_cnt_rows);
    rp.status = ws_at<uint32_t>(ws, P.off_status);
    for (int b = 0; b < P.B; ++b) {
      rp.seq.start[b] = kv->kv_start[b];
      rp.seq.len[b] = kv->kv_len[b];
    }
    RowsParams r1 = rp, r2 = rp;
    for (int b = 0; b <= P.B; ++b) {
      r1.seq.item_begin[b] = P.blk1_begin[b];
      r2.seq.item_begin[b] = P.blk2_begin[b];
    }
    r1.q_per_block = kRowsPerBlock / P.H;
    r1.n_chunks = P.n_chunks1;
    r1.n_items = P.n_blk1 * P.n_chunks1;
    r2.q_per_block = (P.kv_dtype == HS2_KV_BF16) ? rows_score_tc_queries(P.H) : kQueriesPass2;
    r2.n_chunks = P.n_chunks2;
    r2.n_items = P.n_blk2 * P.n_chunks2;
    hs2_status st = cuda_check(P.kv_dtype == HS2_KV_BF16 ? launch_rows_attn_tc(tm, r1, stream)
                                                         : launch_rows_pass(0, P.kv_dtype, tm, r1, stream),
                               "chunk pass 1");
    if (st != HS2_OK) return st;
    if (mark && (st = (*mark)()) != HS2_OK) return st;
    if (mark && (st = (*mark)()) != HS2_OK) return st;  // pass 1 merged its own partials
    st = cuda_check(P.kv_dtype == HS2_KV_BF16 ? launch_rows_score_tc(tm, r2, stream)
                                              : launch_rows_pass(1, P.kv_dtype, tm, r2, stream),
                    "chunk score pass 2");
    if (st != HS2_OK) return st;
    if (mark && (st = (*mark)()) != HS2_OK) return st;
    return HS2_OK;
  }
  DecodeParams dp;
  memset(&dp, 0, sizeof dp);
  fill_seq(kv, P, dp.seq);
  int sms = 0;
  hs2_status st = sm_count(&sms);
  if (st != HS2_OK) return st;
  // 128-row tiles for the tensor-core passes
  int t128 = 0;
  for (int b = 0; b < P.B; ++b) {
    dp.tile128_begin[b] = t128;
    const int64_t r0 = kv->kv_start[b], r1 = r0 + kv->kv_len[b];
    t128 += (int)((r1 + 127) / 128 - r0 / 128);
  }
  dp.tile128_begin[P.B] = t128;
  dp.total_tiles128 = t128;
  // pass 1: warp-level products over 64-row tiles (one CTA per SM for bf16, two for e4m3);
  // the score pass: the same for bf16, tcgen05 over 128-row tiles for e4m3 (one CTA per SM)
  const bool tc2 = P.kv_dtype == HS2_KV_FP8_E4M3;
  const int per_sm1 = P.kv_dtype == HS2_KV_BF16 ? 1 : 2;
  const int T = P.total_tiles;
  const int32_t *tb = P.tile_begin;
  int G = std::max(1, std::min({per_sm1 * sms, T, kMaxStreamCtas}));
  if (pass1_seq_split(P.B, tb, G, dp.cta_begin)) {
    // every CTA in one sequence: its partial slot is its index
    dp.seq_split = 1;
    G = dp.cta_begin[P.B];
    for (int b = 0; b <= P.B; ++b) dp.seq.item_begin[b] = dp.cta_begin[b];
  } else {
    // partial slots: one per (CTA, sequence) pair; CTA i owns tiles [i*T/G, (i+1)*T/G)
    auto cta_of = [&](int g) { return (int)(((int64_t)(g + 1) * G - 1) / T); };
    int slots = 0;
    for (int b = 0; b < P.B; ++b) {
      dp.seq.item_begin[b] = slots;
      slots += decode_slots_per_cta(P.H) * (cta_of(tb[b + 1] - 1) - cta_of(tb[b]) + 1);
    }
    dp.seq.item_begin[P.B] = slots;
  }
  dp.batch = P.B;
  dp.n_heads = P.H;
  dp.total_tiles = T;
  dp.n_ctas = G;
  dp.n_ctas2 = tc2 ? std::max(1, std::min(sms, t128))                 // one CTA per SM
                  : (HS2_PASS2_SUB > 1 ? std::max(1, std::min(sms, (P.total_tiles + 1) / 2))
                                       : std::max(1, std::min({2 * sms, P.total_tiles, kMaxStreamCtas})));
  dp.window = window;
  dp.scale_log2 = scale * 1.4426950408889634f;
  dp.kv_rows = kv->kv_rows;
  dp.k_scale = kv->k_scale;
  dp.v_scale = kv->v_scale;
  dp.q = q;
  dp.out = out;
  dp.out_f32 = out_f32;
  dp.lse = lse;
  dp.scores = scores;
  dp.score_stride = score_stride;
  dp.hist = with_hist ? ws_at<uint32_t>(ws, P.off_hist) : nullptr;
  dp.part = ws_at<float>(ws, P.off_part_p1);
  dp.status = ws_at<uint32_t>(ws, P.off_status);
  if (clear_in_pass1) {   // the caller skipped the workspace clear: pass 1 does it
    dp.zero = ws_at<uint4>(ws, 0);
    dp.zero_n16 = (int32_t)(P.zero_end / 16);
  }
  if (!(passes & 1)) {   // score pass only, with the caller's lse
    st = cuda_check(tc2 ? launch_decode_score_tc(P.kv_dtype, tm, dp, stream)
                        : launch_decode_pass(1, P.kv_dtype, tm, dp, stream),
                    "score pass 2");
    return st;
  }
  st = cuda_check(launch_decode_pass(0, P.kv_dtype, tm, dp, stream), "full-attention pass 1");
  if (st != HS2_OK) return st;
  if (mark && (st = (*mark)()) != HS2_OK) return st;
  {
    MergeParams mp;
    memset(&mp, 0, sizeof mp);
    mp.seq = dp.seq;
    mp.by_seq = 1;
    mp.n_groups = P.B;
    mp.n_heads = P.H;
    mp.part = dp.part;
    mp.out = out;
    mp.out_f32 = out_f32;
    mp.lse = lse;
    if ((st = cuda_check(launch_merge(mp, stream), "pass 1 merge")) != HS2_OK) return st;
  }
  if (mark && (st = (*mark)()) != HS2_OK) return st;
  if (!(passes & 2)) return HS2_OK;
  st = cuda_check(tc2 ? launch_decode_score_tc(P.kv_dtype, tm, dp, stream)
                      : launch_decode_pass(1, P.kv_dtype, tm, dp, stream),
                  "score pass 2");
  if (st != HS2_OK) return st;
  if (mark && (st = (*mark)()) != HS2_OK) return st;
  return HS2_OK;
}

// Device scratch the selection step uses (pointers into a workspace).
struct TopkScratch {
  uint32_t *status = nullptr, *hist = nullptr, *cand_key = nullptr;
  int32_t *cand_idx = nullptr, *cand_count = nullptr, *arrive = nullptr;
  int2 *seg_info = nullptr;
};

TopkScratch topk_scratch(const Plan &P, void *ws) {
  TopkScratch t;
  t.status = ws_at<uint32_t>(ws, P.off_status);
  t.hist = ws_at<uint32_t>(ws, P.off_hist);
  t.cand_key = ws_at<uint32_t>(ws, P.off_cand_key);
  t.cand_idx = ws_at<int32_t>(ws, P.off_cand_idx);
  t.cand_count = ws_at<int32_t>(ws, P.off_cand_count);
  t.arrive = ws_at<int32_t>(ws, P.off_arrive);
  t.seg_info = ws_at<int2>(ws, P.off_seg_info);
  return t;
}

hs2_status run_topk(const hs2_kv_view *kv, const Plan &P, const float *scores,
                    int64_t score_stride, int topk, int window, int32_t *idx, int idx_stride,
                    int32_t *count, bool hist_ready, const TopkScratch &sc, cudaStream_t stream) {
  TopkParams tp;
  memset(&tp, 0, sizeof tp);
  fill_seq(kv, P, tp.seq);
  tp.batch = P.B;
  tp.n_q = P.n_q;
  tp.topk = topk;
  tp.window = window;
  tp.scores = scores;
  tp.score_stride = score_stride;
  tp.n_seg = P.n_seg;
  tp.seg_len = P.seg_len;
  // rows split over at most 8 segments whose keys fit in registers: one cluster per row
  tp.cluster = (P.n_seg > 1 && P.n_seg <= 8 && P.seg_len <= 32 * 512) ? 1 : 0;
  if (P.n_seg > 1) {
    if (hist_ready) tp.hist = sc.hist;
    else tp.hist_ws = sc.hist;
  }
  tp.cand_key = sc.cand_key;
  tp.cand_idx = sc.cand_idx;
  tp.cand_cap = kCandCapGlobal;
  tp.seg_info = sc.seg_info;
  tp.cand_count = sc.cand_count;
  tp.arrive = sc.arrive;
  tp.idx = idx;
  tp.idx_stride = idx_stride;
  tp.count = count;
  tp.status = sc.status;
  return cuda_check(launch_topk(tp, P.n_rows, stream), "top-k selection");
}

hs2_status run_sparse(const hs2_kv_view *kv, const Plan &P, const void *q, const int32_t *idx,
                      int idx_stride, const int32_t *count, float scale, void *out, int out_f32,
                      void *ws, cudaStream_t stream, bool idx_ready = false,
                      float *lse_out = nullptr, bool allow_empty = false) {
  SparseParams sp;
  memset(&sp, 0, sizeof sp);
  fill_seq(kv, P, sp.seq);
  sp.batch = P.B;
  sp.n_q = P.n_q;
  sp.n_heads = P.H;
  const int64_t cap = std::min<int64_t>(idx_stride, P.max_p + 1);
  const int tiles = (int)((cap + kTile - 1) / kTile);
  int ts = 1;
  sp.head_groups = 1;
  if (P.sparse_split) {   // about one CTA per SM: spread the gather over the chip
    // few rows: the heads too are split, two 16-head CTAs (separate clusters) per row, each
    // gathering the row's selection for its heads (the second read of a row hits L2)
    sp.head_groups = P.H / 16;
    const int units = P.n_rows * sp.head_groups;
    int max_cluster = 1;
    hs2_status st = sparse_cluster_limit(P.kv_dtype, P.H / sp.head_groups, &max_cluster);
    if (st != HS2_OK) return st;
    ts = std::max(1, std::min({(kManyRows + units - 1) / units, tiles, kMaxSplit, max_cluster}));
  }
  const int tiles_per = (tiles + ts - 1) / ts;
  sp.split_len = tiles_per * kTile;
  sp.n_tsplit = (int)((cap + sp.split_len - 1) / sp.split_len);
  sp.scale_log2 = scale * 1.4426950408889634f;
  sp.idx_ready = idx_ready ? 1 : 0;
  sp.lse_out = lse_out;
  sp.allow_empty = allow_empty ? 1 : 0;
  sp.q = q;
  sp.idx = idx;
  sp.idx_stride = idx_stride;
  sp.count = count;
  sp.k = kv->k;
  sp.v = kv->v;
  sp.k_scale = kv->k_scale;
  sp.v_scale = kv->v_scale;
  sp.out = out;
  sp.out_f32 = out_f32;
  sp.status = ws_at<uint32_t>(ws, P.off_status);
  return cuda_check(launch_sparse(P.kv_dtype, sp, stream), "sparse gather attention");
}

hs2_status check_budget(int topk, int window) {
  if (topk < 1 || topk > HS2_MAX_TOPK)
    return fail(HS2_ERR_UNSUPPORTED, "topk %d outside [1, %d]", topk, HS2_MAX_TOPK);
  if (window < 0 || window > HS2_MAX_WINDOW)
    return fail(HS2_ERR_UNSUPPORTED, "window %d outside [0, %d]", window, HS2_MAX_WINDOW);
  return HS2_OK;
}

hs2_status check_idx(const Plan &P, int topk, int window, const int32_t *idx, int idx_stride,
                     const int32_t *count) {
  if (!idx || !count) return fail(HS2_ERR_INVALID_ARG, "idx / count is NULL");
  const int64_t need = std::min<int64_t>(P.max_p + 1, (int64_t)topk + window);
  if (idx_stride < need)
    return fail(HS2_ERR_INVALID_ARG, "idx_stride %d < %lld", idx_stride, (long long)need);
  return HS2_OK;
}

hs2_status check_full_args(const Plan &P, const void *q, float scale, const void *out,
                           int out_dtype, const float *lse, const float *scores,
                           int64_t score_stride) {
  if (!q || !out || !lse || !scores) return fail(HS2_ERR_INVALID_ARG, "q / out / lse / scores is NULL");
  if (!aligned16(q) || !aligned16(out)) return fail(HS2_ERR_INVALID_ARG, "q / out must be 16-byte aligned");
  if (!valid_scale(scale)) return fail(HS2_ERR_INVALID_ARG, "softmax_scale must be finite and > 0");
  if (out_dtype != HS2_OUT_BF16 && out_dtype != HS2_OUT_F32)
    return fail(HS2_ERR_INVALID_ARG, "out_dtype %d", out_dtype);
  if (score_stride < P.max_p + 1)
    return fail(HS2_ERR_INVALID_ARG, "score_stride %lld < %lld", (long long)score_stride,
                (long long)(P.max_p + 1));
  return HS2_OK;
}

// Block-level selection: the workspace holds the status word and the block scores.
constexpr int kBlockSelSmemKeys = 32768;   // block scores per row staged in shared memory

struct BlockPlan {
  int64_t blk_stride = 0;
  size_t off_blk = 0, total = 0;
  int pool_ctas_per_row = 0;
};

hs2_status check_block_args(int block_size, int topk) {
  if (block_size != 16 && block_size != 32 && block_size != 64 && block_size != 128)
    return fail(HS2_ERR_UNSUPPORTED, "block_size %d (16, 32, 64 or 128)", block_size);
  if (topk % block_size != 0)
    return fail(HS2_ERR_INVALID_ARG, "topk %d is not a multiple of block_size %d", topk, block_size);
  return HS2_OK;
}

BlockPlan block_plan(const Plan &P, int block_size) {
  BlockPlan B;
  const int64_t positions = P.max_p + 1;
  B.blk_stride = ((positions + block_size - 1) / block_size + 3) / 4 * 4;
  B.off_blk = align_up(4);
  B.total = align_up(B.off_blk + (size_t)P.n_rows * (size_t)B.blk_stride * 4);
  const int per = block_pool_positions_per_cta();
  B.pool_ctas_per_row = (int)((positions + per - 1) / per);
  return B;
}

// hs2_block_decode's own outputs that the caller may leave to the library: they follow the
// workspace regions of the plan (lse always; scores and the selection when asked for).
struct BlockExtra {
  size_t off_lse = 0, off_scores = 0, off_idx = 0, off_count = 0, total = 0;
  int64_t score_stride = 0;
  int32_t idx_stride = 0;
};

constexpr uint32_t kWsFlags = HS2_WS_SCORES | HS2_WS_SELECTION;

BlockExtra block_extra(const Plan &P, int topk, int window, uint32_t flags) {
  BlockExtra E;
  size_t o = P.total;
  E.off_lse = o; o = align_up(o + 4 * (size_t)P.n_rows * P.H);
  E.score_stride = (P.max_p + 1 + 63) / 64 * 64;
  E.idx_stride = (int32_t)std::min<int64_t>(P.max_p + 1, (int64_t)topk + window);
  E.off_scores = o;
  if (flags & HS2_WS_SCORES) o = align_up(o + 4 * (size_t)P.n_rows * (size_t)E.score_stride);
  E.off_idx = o;
  if (flags & HS2_WS_SELECTION) o = align_up(o + 4 * (size_t)P.n_rows * (size_t)E.idx_stride);
  E.off_count = o;
  if (flags & HS2_WS_SELECTION) o = align_up(o + 4 * (size_t)P.n_rows);
  E.total = o;
  return E;
}

hs2_status check_ws_bytes(void *ws, size_t bytes, size_t need, uint32_t flags) {
  if (!ws) return fail(HS2_ERR_INVALID_ARG, "workspace is NULL");
  if (reinterpret_cast<uintptr_t>(ws) % kAlign)
    return fail(HS2_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  if (bytes < need)
    return fail(HS2_ERR_WORKSPACE, "workspace %zu bytes < %zu required (hs2_workspace_size with flags %u)",
                bytes, need, flags);
  return HS2_OK;
}

}  // namespace
}  // namespace hs2

using namespace hs2;

extern "C" {

hs2_status hs2_workspace_size(const hs2_kv_view *kv, int32_t topk, int32_t window,
                              uint32_t flags, size_t *bytes) {
  hs2_status st = validate_view(kv);
  if (st != HS2_OK) return st;
  if ((st = check_budget(topk, window)) != HS2_OK) return st;
  if (!bytes) return fail(HS2_ERR_INVALID_ARG, "bytes is NULL");
  if (flags & ~kWsFlags) return fail(HS2_ERR_INVALID_ARG, "flags 0x%x: unknown bits", flags);
  Plan P;
  make_plan(kv, P);
  *bytes = block_extra(P, topk, window, flags).total;
  return ok();
}

hs2_status hs2_full_attn_scores(const hs2_kv_view *kv, const void *q, float softmax_scale,
                                void *out, int32_t out_dtype, float *lse, float *scores,
                                int64_t score_stride, void *workspace, size_t workspace_bytes,
                                void *stream) {
  hs2_status st = validate_view(kv);
  if (st != HS2_OK) return st;
  Plan P;
  make_plan(kv, P);
  if ((st = check_full_args(P, q, softmax_scale, out, out_dtype, lse, scores, score_stride)) != HS2_OK) return st;
  if ((st = check_ws(P, workspace, workspace_bytes)) != HS2_OK) return st;
  TensorMaps tm;
  if ((st = encode_maps(kv, tm)) != HS2_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((st = cuda_check(cudaMemsetAsync(workspace, 0, P.zero_end, s), "workspace clear")) != HS2_OK) return st;
  st = run_full(kv, P, tm, q, softmax_scale, out, out_dtype == HS2_OUT_F32, lse, scores,
                score_stride, 0, false, workspace, s);
  return st == HS2_OK ? ok() : st;
}

hs2_status hs2_topk_select(const hs2_kv_view *kv, const float *scores, int64_t score_stride,
                           int32_t topk, int32_t window, int32_t *idx, int32_t idx_stride,
                           int32_t *count, void *workspace, size_t workspace_bytes,
                           void *stream) {
  hs2_status st = validate_view(kv);
  if (st != HS2_OK) return st;
  if ((st = check_budget(topk, window)) != HS2_OK) return st;
  Plan P;
  make_plan(kv, P);
  if (!scores) return fail(HS2_ERR_INVALID_ARG, "scores is NULL");
  if (score_stride < P.max_p + 1)
    return fail(HS2_ERR_INVALID_ARG, "score_stride %lld < %lld", (long long)score_stride,
                (long long)(P.max_p + 1));
  if ((st = check_idx(P, topk, window, idx, idx_stride, count)) != HS2_OK) return st;
  if ((st = check_ws(P, workspace, workspace_bytes)) != HS2_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((st = cuda_check(cudaMemsetAsync(workspace, 0, P.zero_end, s), "workspace clear")) != HS2_OK) return st;
  st = run_topk(kv, P, scores, score_stride, topk, window, idx, idx_stride, count, false,
                topk_scratch(P, workspace), s);
  return st == HS2_OK ? ok() : st;
}

hs2_status hs2_topk_select_noalloc(const hs2_kv_view *kv, const float *scores,
                                   int64_t score_stride, int32_t topk, int32_t window,
                                   int32_t *idx, int32_t idx_stride, int32_t *count,
                                   void *stream) {
  hs2_status st = validate_view(kv);
  if (st != HS2_OK) return st;
  if ((st = check_budget(topk, window)) != HS2_OK) return st;
  Plan P;
  make_plan(kv, P);
  if (!scores) return fail(HS2_ERR_INVALID_ARG, "scores is NULL");
  if (score_stride < P.max_p + 1)
    return fail(HS2_ERR_INVALID_ARG, "score_stride %lld < %lld", (long long)score_stride,
                (long long)(P.max_p + 1));
  if ((st = check_idx(P, topk, window, idx, idx_stride, count)) != HS2_OK) return st;
  const NoallocLayout lay = noalloc_layout(P);
  if (lay.total > HS2_NOALLOC_SCRATCH_BYTES)
    return fail(HS2_ERR_WORKSPACE,
                "this selection needs %zu bytes of scratch; the built-in array holds %u "
                "(use hs2_topk_select with a workspace)", lay.total, HS2_NOALLOC_SCRATCH_BYTES);
  void *base = nullptr;
  if ((st = noalloc_scratch(&base)) != HS2_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((st = cuda_check(cudaMemsetAsync(base, 0, lay.zero_end, s), "scratch clear")) != HS2_OK) return st;
  TopkScratch sc;
  sc.status = ws_at<uint32_t>(base, lay.off_status);
  sc.cand_count = ws_at<int32_t>(base, lay.off_cand_count);
  sc.arrive = ws_at<int32_t>(base, lay.off_arrive);
  sc.hist = ws_at<uint32_t>(base, lay.off_hist);
  sc.cand_key = ws_at<uint32_t>(base, lay.off_cand_key);
  sc.cand_idx = ws_at<int32_t>(base, lay.off_cand_idx);
  sc.seg_info = ws_at<int2>(base, lay.off_seg_info);
  st = run_topk(kv, P, scores, score_stride, topk, window, idx, idx_stride, count, false, sc, s);
  return st == HS2_OK ? ok() : st;
}

hs2_status hs2_noalloc_read_status(void *stream) {
  void *base = nullptr;
  hs2_status st = noalloc_scratch(&base);
  if (st != HS2_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((st = cuda_check(cudaStreamSynchronize(s), "stream synchronize")) != HS2_OK) return st;
  uint32_t v = 0;
  // the status word sits at the start of the built-in array (noalloc_layout's off_status)
  if ((st = cuda_check(cudaMemcpy(&v, base, 4, cudaMemcpyDeviceToHost), "status read")) != HS2_OK)
    return st;
  if (v && (st = cuda_check(cudaMemset(base, 0, 4), "status clear")) != HS2_OK) return st;
  if (v & kStatusTimeout) return fail(HS2_ERR_TIMEOUT, "a kernel's bounded wait ran out");
  if (v & kStatusCheck)
    return fail(HS2_ERR_DEVICE_CHECK, "a candidate score was negative or NaN");
  return ok();
}

hs2_status hs2_topk_select_blocks_workspace_size(const hs2_kv_view *kv, int32_t block_size,
                                                 int32_t topk, int32_t window, size_t *bytes) {
  hs2_status st = validate_view(kv);
  if (st != HS2_OK) return st;
  if ((st = check_budget(topk, window)) != HS2_OK) return st;
  if ((st = check_block_args(block_size, topk)) != HS2_OK) return st;
  if (!bytes) return fail(HS2_ERR_INVALID_ARG, "bytes is NULL");
  Plan P;
  make_plan(kv, P);
  *bytes = block_plan(P, block_size).total;
  return ok();
}

hs2_status hs2_topk_select_blocks(const hs2_kv_view *kv, const float *scores,
                                  int64_t score_stride, int32_t block_size, int32_t topk,
                                  int32_t window, int32_t *idx, int32_t idx_stride,
                                  int32_t *count, void *workspace, size_t workspace_bytes,
                                  void *stream) {
  hs2_status st = validate_view(kv);
  if (st != HS2_OK) return st;
  if ((st = check_budget(topk, window)) != HS2_OK) return st;
  if ((st = check_block_args(block_size, topk)) != HS2_OK) return st;
  Plan P;
  make_plan(kv, P);
  if (!scores) return fail(HS2_ERR_INVALID_ARG, "scores is NULL");
  if (score_stride < P.max_p + 1)
    return fail(HS2_ERR_INVALID_ARG, "score_stride %lld < %lld", (long long)score_stride,
                (long long)(P.max_p + 1));
  if ((st = check_idx(P, topk, window, idx, idx_stride, count)) != HS2_OK) return st;
  const BlockPlan B = block_plan(P, block_size);
  if (!workspace) return fail(HS2_ERR_INVALID_ARG, "workspace is NULL");
  if (reinterpret_cast<uintptr_t>(workspace) % kAlign)
    return fail(HS2_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  if (workspace_bytes < B.total)
    return fail(HS2_ERR_WORKSPACE, "workspace %zu bytes < %zu required", workspace_bytes, B.total);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  BlockSelParams bp;
  memset(&bp, 0, sizeof bp);
  fill_seq(kv, P, bp.seq);
  bp.batch = P.B;
  bp.n_q = P.n_q;
  bp.bs = block_size;
  bp.kb = topk / block_size;
  bp.topk = topk;
  bp.window = window;
  bp.scores = scores;
  bp.score_stride = score_stride;
  bp.blk = ws_at<float>(workspace, B.off_blk);
  bp.blk_stride = B.blk_stride;
  bp.pool_ctas_per_row = B.pool_ctas_per_row;
  bp.smem_keys = (int)std::min<int64_t>(kBlockSelSmemKeys, B.blk_stride);
  // many rows: each CTA pools its own row (one launch, no block-score round trip); few long
  // rows: the pooling is spread over the chip first
  bp.fused = (P.n_rows >= kManyRows && B.blk_stride <= kBlockSelSmemKeys) ? 1 : 0;
  bp.status = ws_at<uint32_t>(workspace, 0);
  bp.idx = idx;
  bp.idx_stride = idx_stride;
  bp.count = count;
  st = cuda_check(launch_block_select(bp, P.n_rows, s), "block selection");
  return st == HS2_OK ? ok() : st;
}

hs2_status hs2_sparse_gather_attn(const hs2_kv_view *kv, const void *q, const int32_t *idx,
                                  int32_t idx_stride, const int32_t *count,
                                  float softmax_scale, void *out, int32_t out_dtype,
                                  void *workspace, size_t workspace_bytes, void *stream) {
  hs2_status st = validate_view(kv);
  if (st != HS2_OK) return st;
  Plan P;
  make_plan(kv, P);
  if (!q || !out) return fail(HS2_ERR_INVALID_ARG, "q / out is NULL");
  if (!aligned16(q) || !aligned16(out)) return fail(HS2_ERR_INVALID_ARG, "q / out must be 16-byte aligned");
  if (!idx || !count) return fail(HS2_ERR_INVALID_ARG, "idx / count is NULL");
  if (idx_stride < 1) return fail(HS2_ERR_INVALID_ARG, "idx_stride %d < 1", idx_stride);
  if (!valid_scale(softmax_scale)) return fail(HS2_ERR_INVALID_ARG, "softmax_scale must be finite and > 0");
  if (out_dtype != HS2_OUT_BF16 && out_dtype != HS2_OUT_F32)
    return fail(HS2_ERR_INVALID_ARG, "out_dtype %d", out_dtype);
  if ((st = check_ws(P, workspace, workspace_bytes)) != HS2_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((st = cuda_check(cudaMemsetAsync(workspace, 0, P.zero_end, s), "workspace clear")) != HS2_OK) return st;
  st = run_sparse(kv, P, q, idx, idx_stride, count, softmax_scale, out,
                  out_dtype == HS2_OUT_F32, workspace, s);
  return st == HS2_OK ? ok() : st;
}

static hs2_status block_impl(const hs2_kv_view *kv, const void *q_full,
                             const void *const *q_sparse, int32_t n_sparse, int32_t topk,
                             int32_t window, float softmax_scale, void *out_full,
                             void *const *out_sparse, int32_t out_dtype, float *lse,
                             float *scores, int64_t score_stride, int32_t *idx,
                             int32_t idx_stride, int32_t *count, void *workspace,
                             size_t workspace_bytes, void *const *events, int32_t n_events,
                             void *stream) {
  hs2_status st = validate_view(kv);
  if (st != HS2_OK) return st;
  if ((st = check_budget(topk, window)) != HS2_OK) return st;
  Plan P;
  make_plan(kv, P);
  // outputs left NULL live in the workspace (sized by hs2_workspace_size with the same flags)
  if ((idx == nullptr) != (count == nullptr))
    return fail(HS2_ERR_INVALID_ARG, "idx and count must both be given or both be NULL");
  const uint32_t flags = (scores ? 0u : (uint32_t)HS2_WS_SCORES) | (idx ? 0u : (uint32_t)HS2_WS_SELECTION);
  const BlockExtra E = block_extra(P, topk, window, flags);
  if ((st = check_ws_bytes(workspace, workspace_bytes, E.total, flags)) != HS2_OK) return st;
  if (!lse) lse = ws_at<float>(workspace, E.off_lse);
  if (!scores) {
    scores = ws_at<float>(workspace, E.off_scores);
    score_stride = E.score_stride;
  }
  if (!idx) {
    idx = ws_at<int32_t>(workspace, E.off_idx);
    count = ws_at<int32_t>(workspace, E.off_count);
    idx_stride = E.idx_stride;
  }
  if ((st = check_full_args(P, q_full, softmax_scale, out_full, out_dtype, lse, scores, score_stride)) != HS2_OK)
    return st;
  if ((st = check_idx(P, topk, window, idx, idx_stride, count)) != HS2_OK) return st;
  if (n_sparse < 0 || n_sparse > 64) return fail(HS2_ERR_INVALID_ARG, "n_sparse %d outside [0, 64]", n_sparse);
  if (n_sparse > 0 && (!q_sparse || !out_sparse))
    return fail(HS2_ERR_INVALID_ARG, "q_sparse / out_sparse is NULL");
  for (int l = 0; l < n_sparse; ++l) {
    if (!q_sparse[l] || !out_sparse[l]) return fail(HS2_ERR_INVALID_ARG, "sparse layer %d: NULL pointer", l);
    if (!aligned16(q_sparse[l]) || !aligned16(out_sparse[l]))
      return fail(HS2_ERR_INVALID_ARG, "sparse layer %d: q / out must be 16-byte aligned", l);
  }
  if (events) {
    if (n_events != 6 + n_sparse)
      return fail(HS2_ERR_INVALID_ARG, "n_events %d != 6 + n_sparse", n_events);
    for (int e = 0; e < n_events; ++e)
      if (!events[e]) return fail(HS2_ERR_INVALID_ARG, "event %d is NULL", e);
  }
  TensorMaps tm;
  if ((st = encode_maps(kv, tm)) != HS2_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int ev = 0;
  const std::function<hs2_status()> mark = [&]() -> hs2_status {
    if (!events) return HS2_OK;
    return cuda_check(cudaEventRecord(static_cast<cudaEvent_t>(events[ev++]), s), "event record");
  };
  if ((st = mark()) != HS2_OK) return st;
  // decode: the full layer's first kernel clears the workspace region itself (no separate
  // memset node between the previous call's last kernel and this call's first)
  const bool clear_in_pass1 = P.n_q == 1;
  if (!clear_in_pass1 &&
      (st = cuda_check(cudaMemsetAsync(workspace, 0, P.zero_end, s), "workspace clear")) != HS2_OK)
    return st;
  if ((st = mark()) != HS2_OK) return st;
  const bool hist = P.n_seg > 1;
  st = run_full(kv, P, tm, q_full, softmax_scale, out_full, out_dtype == HS2_OUT_F32, lse, scores,
                score_stride, window, hist, workspace, s, events ? &mark : nullptr, clear_in_pass1);
  if (st != HS2_OK) return st;
  st = run_topk(kv, P, scores, score_stride, topk, window, idx, idx_stride, count, hist,
                topk_scratch(P, workspace), s);
  if (st != HS2_OK) return st;
  if ((st = mark()) != HS2_OK) return st;
  for (int l = 0; l < n_sparse; ++l) {
    // layers after the first: the selection finished before the previous layer started
    st = run_sparse(kv, P, q_sparse[l], idx, idx_stride, count, softmax_scale, out_sparse[l],
                    out_dtype == HS2_OUT_F32, workspace, s, l > 0);
    if (st != HS2_OK) return st;
    if ((st = mark()) != HS2_OK) return st;
  }
  return ok();
}

hs2_status hs2_block_decode(const hs2_kv_view *kv, const void *q_full,
                            const void *const *q_sparse, int32_t n_sparse, int32_t topk,
                            int32_t window, float softmax_scale, void *out_full,
                            void *const *out_sparse, int32_t out_dtype, float *lse,
                            float *scores, int64_t score_stride, int32_t *idx,
                            int32_t idx_stride, int32_t *count, void *workspace,
                            size_t workspace_bytes, void *stream) {
  return block_impl(kv, q_full, q_sparse, n_sparse, topk, window, softmax_scale, out_full,
                    out_sparse, out_dtype, lse, scores, score_stride, idx, idx_stride, count,
                    workspace, workspace_bytes, nullptr, 0, stream);
}

hs2_status hs2_block_decode_traced(const hs2_kv_view *kv, const void *q_full,
                                   const void *const *q_sparse, int32_t n_sparse, int32_t topk,
                                   int32_t window, float softmax_scale, void *out_full,
                                   void *const *out_sparse, int32_t out_dtype, float *lse,
                                   float *scores, int64_t score_stride, int32_t *idx,
                                   int32_t idx_stride, int32_t *count, void *workspace,
                                   size_t workspace_bytes, void *const *events,
                                   int32_t n_events, void *stream) {
  if (!events) return fail(HS2_ERR_INVALID_ARG, "events is NULL");
  return block_impl(kv, q_full, q_sparse, n_sparse, topk, window, softmax_scale, out_full,
                    out_sparse, out_dtype, lse, scores, score_stride, idx, idx_stride, count,
                    workspace, workspace_bytes, events, n_events, stream);
}

hs2_status hs2_read_device_status(const void *workspace, void *stream) {
  if (!workspace) return fail(HS2_ERR_INVALID_ARG, "workspace is NULL");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t v = 0;
  hs2_status st = cuda_check(cudaStreamSynchronize(s), "stream synchronize");
  if (st != HS2_OK) return st;
  st = cuda_check(cudaMemcpy(&v, workspace, 4, cudaMemcpyDeviceToHost), "status read");
  if (st != HS2_OK) return st;
  if (v & kStatusTimeout) return fail(HS2_ERR_TIMEOUT, "a kernel's bounded wait ran out");
  if (v & kStatusCheck)
    return fail(HS2_ERR_DEVICE_CHECK,
                "a kernel's input check failed (an out-of-range index or count, or a negative or "
                "NaN candidate score)");
  return ok();
}

namespace hs2 {
namespace {
// One thread waits, bounded by limit_ns, on an mbarrier that expects one arrival and gets none,
// and records the timeout in the status word like every kernel of the library does.
__global__ void selftest_wait_kernel(uint32_t *status, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    fence_barrier_init();
    if (!mbar_wait_for(smem_u32(&bar), 0, limit_ns)) record_status(status, kStatusTimeout);
  }
}
}  // namespace
}  // namespace hs2

namespace hs2 {
namespace {
// y = exp2_poly2(x), the FMA-pipe 2^x of the tensor-core score passes, element by element
__global__ void selftest_exp2_kernel(const float *x, float *y, int64_t n) {
  const int64_t i = 2 * ((int64_t)blockIdx.x * blockDim.x + threadIdx.x);
  if (i + 1 < n) {
    const float2 r = exp2_poly2(make_float2(x[i], x[i + 1]));
    y[i] = r.x;
    y[i + 1] = r.y;
  } else if (i < n) {
    y[i] = exp2_poly2(make_float2(x[i], 0.f)).x;
  }
}
}  // namespace
}  // namespace hs2

hs2_status hs2_selftest_exp2(const float *x, float *y, int64_t n, void *stream) {
  if (!x || !y) return fail(HS2_ERR_INVALID_ARG, "x / y is NULL");
  if (n < 0 || n > ((int64_t)1 << 40)) return fail(HS2_ERR_INVALID_ARG, "n %lld out of range", (long long)n);
  if (n == 0) return ok();
  const int64_t pairs = (n + 1) / 2;
  const int64_t blocks = (pairs + 255) / 256;
  if (blocks > INT32_MAX) return fail(HS2_ERR_INVALID_ARG, "n too large");
  hs2::selftest_exp2_kernel<<<(unsigned)blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, y, n);
  hs2_status st = cuda_check(cudaGetLastError(), "exp2 self-test launch");
  if (st != HS2_OK) return st;
  hs2::note_launch();
  return ok();
}

hs2_status hs2_kv_append(const hs2_kv_view *kv, const void *new_k, const void *new_v, void *stream) {
  hs2_status st = validate_view(kv);
  if (st != HS2_OK) return st;
  if (!new_k || !new_v) return fail(HS2_ERR_INVALID_ARG, "new_k / new_v is NULL");
  if ((reinterpret_cast<uintptr_t>(new_k) | reinterpret_cast<uintptr_t>(new_v)) & 15)
    return fail(HS2_ERR_INVALID_ARG, "new_k / new_v must be 16-byte aligned");
  hs2::AppendParams ap;
  memset(&ap, 0, sizeof ap);
  for (int b = 0; b < kv->batch; ++b) {
    ap.seq.start[b] = kv->kv_start[b];
    ap.seq.len[b] = kv->kv_len[b];
  }
  ap.batch = kv->batch;
  ap.n_q = kv->n_q;
  ap.fp8 = kv->kv_dtype == HS2_KV_FP8_E4M3;
  ap.new_k = new_k;
  ap.new_v = new_v;
  ap.k = const_cast<void *>(kv->k);
  ap.v = const_cast<void *>(kv->v);
  ap.k_scale = const_cast<float *>(kv->k_scale);
  ap.v_scale = const_cast<float *>(kv->v_scale);
  st = cuda_check(hs2::launch_kv_append(ap, static_cast<cudaStream_t>(stream)), "kv append");
  return st == HS2_OK ? ok() : st;
}

// ------------------------------------------------------------------ context-parallel pieces

hs2_status hs2_full_attn(const hs2_kv_view *kv, const void *q, float softmax_scale, void *out,
                         int32_t out_dtype, float *lse, void *workspace, size_t workspace_bytes,
                         void *stream) {
  hs2_status st = validate_view(kv);
  if (st != HS2_OK) return st;
  if (kv->n_q != 1) return fail(HS2_ERR_UNSUPPORTED, "hs2_full_attn is for decode (n_q = 1)");
  Plan P;
  make_plan(kv, P);
  if (!q || !out || !lse) return fail(HS2_ERR_INVALID_ARG, "q / out / lse is NULL");
  if (!aligned16(q) || !aligned16(out)) return fail(HS2_ERR_INVALID_ARG, "q / out must be 16-byte aligned");
  if (!valid_scale(softmax_scale)) return fail(HS2_ERR_INVALID_ARG, "softmax_scale must be finite and > 0");
  if (out_dtype != HS2_OUT_BF16 && out_dtype != HS2_OUT_F32)
    return fail(HS2_ERR_INVALID_ARG, "out_dtype %d", out_dtype);
  if ((st = check_ws(P, workspace, workspace_bytes)) != HS2_OK) return st;
  TensorMaps tm;
  if ((st = encode_maps(kv, tm)) != HS2_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  st = run_full(kv, P, tm, q, softmax_scale, out, out_dtype == HS2_OUT_F32, lse, nullptr, 0, 0,
                false, workspace, s, nullptr, true, 1);
  return st == HS2_OK ? ok() : st;
}

hs2_status hs2_score_pass(const hs2_kv_view *kv, const void *q, float softmax_scale,
                          const float *lse, float *scores, int64_t score_stride, void *workspace,
                          size_t workspace_bytes, void *stream) {
  hs2_status st = validate_view(kv);
  if (st != HS2_OK) return st;
  if (kv->n_q != 1) return fail(HS2_ERR_UNSUPPORTED, "hs2_score_pass is for decode (n_q = 1)");
  Plan P;
  make_plan(kv, P);
  if (!q || !lse || !scores) return fail(HS2_ERR_INVALID_ARG, "q / lse / scores is NULL");
  if (!aligned16(q)) return fail(HS2_ERR_INVALID_ARG, "q must be 16-byte aligned");
  if (!valid_scale(softmax_scale)) return fail(HS2_ERR_INVALID_ARG, "softmax_scale must be finite and > 0");
  if (score_stride < P.max_p + 1)
    return fail(HS2_ERR_INVALID_ARG, "score_stride %lld < %lld", (long long)score_stride,
                (long long)(P.max_p + 1));
  if ((st = check_ws(P, workspace, workspace_bytes)) != HS2_OK) return st;
  TensorMaps tm;
  if ((st = encode_maps(kv, tm)) != HS2_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((st = cuda_check(cudaMemsetAsync(workspace, 0, P.zero_end, s), "workspace clear")) != HS2_OK) return st;
  st = run_full(kv, P, tm, q, softmax_scale, nullptr, 0, const_cast<float *>(lse), scores,
                score_stride, 0, false, workspace, s, nullptr, false, 2);
  return st == HS2_OK ? ok() : st;
}

hs2_status hs2_sparse_gather_attn_partial(const hs2_kv_view *kv, const void *q,
                                          const int32_t *idx, int32_t idx_stride,
                                          const int32_t *count, float softmax_scale, float *out,
                                          float *lse, void *workspace, size_t workspace_bytes,
                                          void *stream) {
  hs2_status st = validate_view(kv);
  if (st != HS2_OK) return st;
  Plan P;
  make_plan(kv, P);
  if (!q || !out || !lse) return fail(HS2_ERR_INVALID_ARG, "q / out / lse is NULL");
  if (!aligned16(q) || !aligned16(out)) return fail(HS2_ERR_INVALID_ARG, "q / out must be 16-byte aligned");
  if (!idx || !count) return fail(HS2_ERR_INVALID_ARG, "idx / count is NULL");
  if (idx_stride < 1) return fail(HS2_ERR_INVALID_ARG, "idx_stride %d < 1", idx_stride);
  if (!valid_scale(softmax_scale)) return fail(HS2_ERR_INVALID_ARG, "softmax_scale must be finite and > 0");
  if ((st = check_ws(P, workspace, workspace_bytes)) != HS2_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((st = cuda_check(cudaMemsetAsync(workspace, 0, P.zero_end, s), "workspace clear")) != HS2_OK) return st;
  st = run_sparse(kv, P, q, idx, idx_stride, count, softmax_scale, out, 1, workspace, s, false,
                  lse, true);
  return st == HS2_OK ? ok() : st;
}

hs2_status hs2_lse_merge(int32_t n_parts, int64_t rows, int32_t n_heads, const float *part_out,
                         const float *part_lse, void *out, int32_t out_dtype, float *lse,
                         void *stream) {
  if (n_parts < 1 || n_parts > 1024) return fail(HS2_ERR_INVALID_ARG, "n_parts %d outside [1, 1024]", n_parts);
  if (rows < 0 || n_heads < 1 || rows * n_heads > INT32_MAX)
    return fail(HS2_ERR_INVALID_ARG, "rows %lld x n_heads %d out of range", (long long)rows, n_heads);
  if (!part_out || !part_lse || !out) return fail(HS2_ERR_INVALID_ARG, "part_out / part_lse / out is NULL");
  if (out_dtype != HS2_OUT_BF16 && out_dtype != HS2_OUT_F32)
    return fail(HS2_ERR_INVALID_ARG, "out_dtype %d", out_dtype);
  LseMergeParams mp;
  memset(&mp, 0, sizeof mp);
  mp.n_parts = n_parts;
  mp.n_heads = n_heads;
  mp.rows = rows;
  mp.part_o = part_out;
  mp.part_lse = part_lse;
  mp.out = out;
  mp.out_f32 = out_dtype == HS2_OUT_F32;
  mp.lse = lse;
  hs2_status st = cuda_check(launch_lse_merge(mp, static_cast<cudaStream_t>(stream)), "lse merge");
  return st == HS2_OK ? ok() : st;
}

namespace {
hs2_status cp_fill(CpParams &cp, int32_t batch, const int64_t *offset, const int32_t *local_len,
                   const int32_t *global_len) {
  memset(&cp, 0, sizeof cp);
  if (batch < 1 || batch > HS2_MAX_BATCH)
    return fail(HS2_ERR_INVALID_ARG, "batch %d outside [1, %d]", batch, HS2_MAX_BATCH);
  cp.batch = batch;
  for (int b = 0; b < batch; ++b) {
    if (offset) cp.offset[b] = offset[b];
    if (local_len) cp.local_len[b] = local_len[b];
    if (global_len) cp.global_len[b] = global_len[b];
    if ((offset && offset[b] < 0) || (local_len && local_len[b] < 1) || (global_len && global_len[b] < 1))
      return fail(HS2_ERR_INVALID_ARG, "sequence %d: bad offset or length", b);
    if (offset && local_len && global_len && offset[b] + local_len[b] > global_len[b])
      return fail(HS2_ERR_INVALID_ARG, "sequence %d: shard [%lld, %lld) past the context (%d)", b,
                  (long long)offset[b], (long long)(offset[b] + local_len[b]), global_len[b]);
  }
  return HS2_OK;
}
}  // namespace

hs2_status hs2_cp_pack_candidates(const hs2_kv_view *kv, const int64_t *global_offset,
                                  const int32_t *global_len, const float *scores,
                                  int64_t score_stride, const int32_t *idx, int32_t idx_stride,
                                  const int32_t *count, int32_t topk, int32_t window,
                                  uint64_t *keys, void *stream) {
  hs2_status st = validate_view(kv);
  if (st != HS2_OK) return st;
  if (kv->n_q != 1) return fail(HS2_ERR_UNSUPPORTED, "context-parallel decode needs n_q = 1");
  if ((st = check_budget(topk, window)) != HS2_OK) return st;
  if (!global_offset || !global_len) return fail(HS2_ERR_INVALID_ARG, "global_offset / global_len is NULL");
  if (!scores || !idx || !count || !keys) return fail(HS2_ERR_INVALID_ARG, "scores / idx / count / keys is NULL");
  if (idx_stride < 1 || score_stride < 1) return fail(HS2_ERR_INVALID_ARG, "bad stride");
  CpParams cp;
  if ((st = cp_fill(cp, kv->batch, global_offset, kv->kv_len, global_len)) != HS2_OK) return st;
  for (int b = 0; b < kv->batch; ++b)
    if (score_stride < kv->kv_len[b]) return fail(HS2_ERR_INVALID_ARG, "score_stride < kv_len[%d]", b);
  cp.topk = topk;
  cp.window = window;
  cp.scores = scores;
  cp.score_stride = score_stride;
  cp.idx = idx;
  cp.idx_stride = idx_stride;
  cp.count = count;
  cp.keys = keys;
  st = cuda_check(launch_cp_pack(cp, static_cast<cudaStream_t>(stream)), "candidate pack");
  return st == HS2_OK ? ok() : st;
}

hs2_status hs2_cp_merge_select(int32_t n_parts, int32_t batch, const int32_t *global_len,
                               const uint64_t *keys, int32_t topk, int32_t window, int32_t *idx,
                               int32_t idx_stride, int32_t *count, void *stream) {
  hs2_status st = check_budget(topk, window);
  if (st != HS2_OK) return st;
  if (n_parts < 1 || (int64_t)n_parts * topk > kCpMaxKeys)
    return fail(HS2_ERR_UNSUPPORTED, "n_parts %d x topk %d above %d", n_parts, topk, kCpMaxKeys);
  if (!global_len || !keys || !idx || !count) return fail(HS2_ERR_INVALID_ARG, "NULL argument");
  CpParams cp;
  if ((st = cp_fill(cp, batch, nullptr, nullptr, global_len)) != HS2_OK) return st;
  for (int b = 0; b < batch; ++b)
    if (idx_stride < std::min<int64_t>(global_len[b], (int64_t)topk + window))
      return fail(HS2_ERR_INVALID_ARG, "idx_stride %d too small for sequence %d", idx_stride, b);
  cp.n_parts = n_parts;
  cp.topk = topk;
  cp.window = window;
  cp.keys = const_cast<uint64_t *>(keys);
  cp.idx_out = idx;
  cp.out_stride = idx_stride;
  cp.count_out = count;
  st = cuda_check(launch_cp_select(cp, static_cast<cudaStream_t>(stream)), "candidate merge");
  return st == HS2_OK ? ok() : st;
}

hs2_status hs2_cp_localize(int32_t batch, const int64_t *global_offset, const int32_t *local_len,
                           const int32_t *idx, int32_t idx_stride, const int32_t *count,
                           int32_t *idx_local, int32_t idx_local_stride, int32_t *count_local,
                           void *stream) {
  if (!global_offset || !local_len || !idx || !count || !idx_local || !count_local)
    return fail(HS2_ERR_INVALID_ARG, "NULL argument");
  if (idx_stride < 1 || idx_local_stride < idx_stride)
    return fail(HS2_ERR_INVALID_ARG, "idx_local_stride %d < idx_stride %d", idx_local_stride, idx_stride);
  CpParams cp;
  hs2_status st = cp_fill(cp, batch, global_offset, local_len, nullptr);
  if (st != HS2_OK) return st;
  cp.idx = idx;
  cp.idx_stride = idx_stride;
  cp.count = count;
  cp.idx_out = idx_local;
  cp.out_stride = idx_local_stride;
  cp.count_out = count_local;
  st = cuda_check(launch_cp_localize(cp, static_cast<cudaStream_t>(stream)), "selection localize");
  return st == HS2_OK ? ok() : st;
}

hs2_status hs2_kv_bridge(const hs2_kv_view *kv, const void *hidden, int32_t d_model,
                         const void *w_kv, void *workspace, size_t workspace_bytes, void *stream) {
  hs2_status st = validate_view(kv);
  if (st != HS2_OK) return st;
  if (d_model < 64 || d_model > 32768 || d_model % 64 != 0)
    return fail(HS2_ERR_UNSUPPORTED, "d_model %d (a multiple of 64 in [64, 32768])", d_model);
  if (!hidden || !w_kv) return fail(HS2_ERR_INVALID_ARG, "hidden / w_kv is NULL");
  if (!aligned16(hidden) || !aligned16(w_kv))
    return fail(HS2_ERR_INVALID_ARG, "hidden / w_kv must be 16-byte aligned");
  if (!workspace || reinterpret_cast<uintptr_t>(workspace) % kAlign)
    return fail(HS2_ERR_INVALID_ARG, "workspace must be a 256-byte aligned device buffer");
  if (workspace_bytes < 256)
    return fail(HS2_ERR_WORKSPACE, "workspace %zu bytes < 256 required", workspace_bytes);
  const int64_t m = (int64_t)kv->batch * kv->n_q;
  if (m > (int64_t)INT32_MAX - 128) return fail(HS2_ERR_UNSUPPORTED, "too many rows");
  Plan P;
  make_plan(kv, P);
  BridgeMaps tm;
  if ((st = encode_bridge_maps(hidden, m, d_model, w_kv, tm)) != HS2_OK) return st;
  BridgeParams bp;
  memset(&bp, 0, sizeof bp);
  fill_seq(kv, P, bp.seq);
  bp.batch = P.B;
  bp.n_q = P.n_q;
  bp.m = (int32_t)m;
  bp.d_model = d_model;
  bp.fp8 = kv->kv_dtype == HS2_KV_FP8_E4M3;
  bp.k = const_cast<void *>(kv->k);
  bp.v = const_cast<void *>(kv->v);
  bp.k_scale = const_cast<float *>(kv->k_scale);
  bp.v_scale = const_cast<float *>(kv->v_scale);
  bp.status = static_cast<uint32_t *>(workspace);
  int dev = 0, sms = 148;
  if ((st = cuda_check(cudaGetDevice(&dev), "cudaGetDevice")) != HS2_OK) return st;
  if ((st = cuda_check(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev),
                       "SM count")) != HS2_OK) return st;
  const int n_tiles = (int)((m + 255) / 256);   // units of two 128-row tiles
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((st = cuda_check(cudaMemsetAsync(workspace, 0, 4, s), "status clear")) != HS2_OK) return st;
  st = cuda_check(launch_kv_bridge(tm, bp, std::min(n_tiles, sms), s), "KV bridging");
  return st == HS2_OK ? ok() : st;
}

hs2_status hs2_selftest_wait_timeout(uint32_t limit_us, void *workspace, size_t workspace_bytes,
                                     void *stream) {
  if (limit_us < 1 || limit_us > 2000000) return fail(HS2_ERR_INVALID_ARG, "limit_us %u outside [1, 2e6]", limit_us);
  if (!workspace && workspace_bytes == 0) {   // the no-allocation selection's built-in status word
    hs2_status st = noalloc_scratch(&workspace);
    if (st != HS2_OK) return st;
    workspace_bytes = HS2_NOALLOC_SCRATCH_BYTES;
  }
  if (!workspace || workspace_bytes < 256 || (reinterpret_cast<uintptr_t>(workspace) & 255))
    return fail(HS2_ERR_WORKSPACE, "workspace must be 256-byte aligned and hold 256 bytes");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  hs2_status st = cuda_check(cudaMemsetAsync(workspace, 0, 4, s), "status clear");
  if (st != HS2_OK) return st;
  hs2::selftest_wait_kernel<<<1, 32, 0, s>>>(static_cast<uint32_t *>(workspace), (uint64_t)limit_us * 1000ull);
  if ((st = cuda_check(cudaGetLastError(), "self-test launch")) != HS2_OK) return st;
  hs2::note_launch();
  return ok();
}

const char *hs2_last_error(void) { return g_err; }

const char *hs2_status_string(hs2_status s) {
  switch (s) {
    case HS2_OK: return "HS2_OK";
    case HS2_ERR_INVALID_ARG: return "HS2_ERR_INVALID_ARG";
    case HS2_ERR_UNSUPPORTED: return "HS2_ERR_UNSUPPORTED";
    case HS2_ERR_WORKSPACE: return "HS2_ERR_WORKSPACE";
    case HS2_ERR_CUDA: return "HS2_ERR_CUDA";
    case HS2_ERR_DEVICE_CHECK: return "HS2_ERR_DEVICE_CHECK";
    case HS2_ERR_TIMEOUT: return "HS2_ERR_TIMEOUT";
  }
  return "HS2_ERR_UNKNOWN";
}

int32_t hs2_version(void) { return HS2_VERSION; }

uint64_t hs2_launch_count(void) { return hs2::launches_so_far(); }

}  // extern "C"
