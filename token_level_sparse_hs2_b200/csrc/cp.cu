// cp.cu -- context-parallel decode: one sequence's cache split by token range over several
// ranks, each running the hybrid block's kernels on its own shard, with three small exchanges
// per block between them (the collectives themselves are the caller's: NCCL all-gathers).
//
// The block's outputs are sums over cache positions (attention) or a selection from per-position
// scores, so a split by position composes exactly:
//  * attention over the union of shards = the log-sum-exp merge of each shard's (O, lse)
//    (lse_merge_kernel), for the full layer and for every sparse layer;
//  * the score of a position needs only the global lse, so after the first merge every rank
//    scores its own positions; the top-k of the whole context is contained in the union of the
//    shards' own top-k, so each rank packs its top-k (score, global position) pairs
//    (cp_pack_kernel) and every rank merges all of them (cp_select_kernel) to the same global
//    selection, ties to the lower position, window appended as on one GPU;
//  * each rank then attends to the selected positions it holds (cp_localize_kernel maps the
//    ascending global selection to its contiguous local run).
// "HySparse2: Hybrid Sparse Attention with Two-Level KV Sharing", bullet "Inference cost" (1M
// token contexts); "HySparse2: How Xiaomi Split the Transformer to Fix Agent Prefill Costs",
// section "KV Reuse and Token-Level Sparse Selection" (what each layer computes).
#include "common.cuh"
#include "internal.h"

namespace hs2 {

namespace {

// One CTA per (row, head), one thread per output dimension.
__global__ void __launch_bounds__(128) lse_merge_kernel(const __grid_constant__ LseMergeParams P) {
  griddep_launch_dependents();
  griddep_wait();
  const int64_t rh = blockIdx.x;                        // row * H + head
  const int d = threadIdx.x;
  const int64_t stride_lse = P.rows * P.n_heads;
  float M = -INFINITY;
  for (int j = 0; j < P.n_parts; ++j) M = fmaxf(M, __ldcg(P.part_lse + j * stride_lse + rh));
  float L = 0.f, O = 0.f;
  if (M != -INFINITY) {
    for (int j = 0; j < P.n_parts; ++j) {
      const float l = __ldcg(P.part_lse + j * stride_lse + rh);
      if (l == -INFINITY) continue;
      const float w = __expf(l - M);
      L += w;
      O += w * __ldcg(P.part_o + (j * stride_lse + rh) * kHeadDim + d);
    }
  }
  const float o = L > 0.f ? O / L : 0.f;
  if (P.out_f32) reinterpret_cast<float *>(P.out)[rh * kHeadDim + d] = o;
  else reinterpret_cast<__nv_bfloat16 *>(P.out)[rh * kHeadDim + d] = __float2bfloat16_rn(o);
  if (P.lse && d == 0) P.lse[rh] = L > 0.f ? M + __logf(L) : -INFINITY;
}

// (score, global position) packed so that the larger value is the higher score, then the lower
// position; 0 is below every packed pair and marks an empty slot.
__device__ __forceinline__ uint64_t cp_key(float score, int64_t g) {
  return ((uint64_t)__float_as_uint(score) << 32) | (uint64_t)(0xffffffffu - (uint32_t)g);
}

// One CTA per sequence: the shard's selected positions that are global candidates (position
// below the global window) as packed keys, then empty slots up to topk.
__global__ void __launch_bounds__(256) cp_pack_kernel(const __grid_constant__ CpParams P) {
  __shared__ int n_s;
  griddep_launch_dependents();
  griddep_wait();
  const int b = blockIdx.x;
  const int64_t wstart = (int64_t)P.global_len[b] - P.window;   // first window position
  const int cnt = min(__ldcg(P.count + b), P.idx_stride);
  const int32_t *idx = P.idx + (size_t)b * P.idx_stride;
  const float *s = P.scores + (size_t)b * P.score_stride;
  uint64_t *keys = P.keys + (size_t)b * P.topk;
  if (threadIdx.x == 0) n_s = 0;
  __syncthreads();
  for (int j = threadIdx.x; j < cnt; j += blockDim.x) {
    const int t = __ldcg(idx + j);
    const int64_t g = P.offset[b] + t;
    if (t >= 0 && t < P.local_len[b] && g < wstart) {
      const int slot = atomicAdd(&n_s, 1);
      if (slot < P.topk) keys[slot] = cp_key(__ldcg(s + t), g);
    }
  }
  __syncthreads();
  for (int j = n_s + threadIdx.x; j < P.topk; j += blockDim.x) keys[j] = 0;
}

constexpr int kCpThreads = 512;

// One CTA per sequence: the topk largest of the n_parts x topk packed keys (bitonic sort in
// shared memory), their positions in ascending order (a second bitonic sort), then the window.
__global__ void __launch_bounds__(kCpThreads) cp_select_kernel(const __grid_constant__ CpParams P) {
  extern __shared__ __align__(16) uint64_t cp_keys[];
  griddep_launch_dependents();
  griddep_wait();
  const int b = blockIdx.x;
  const int64_t p = (int64_t)P.global_len[b] - 1;
  const int64_t nc = max((int64_t)0, p - P.window + 1);
  int32_t *out = P.idx_out + (size_t)b * P.out_stride;
  if (nc <= P.topk) {
    for (int64_t t = threadIdx.x; t <= p; t += kCpThreads) out[t] = (int32_t)t;
    if (threadIdx.x == 0) P.count_out[b] = (int32_t)(p + 1);
    return;
  }
  const int n = P.n_parts * P.topk;
  int np = 1;
  while (np < n) np <<= 1;
  for (int i = threadIdx.x; i < np; i += kCpThreads) {
    uint64_t v = 0;
    if (i < n) {
      const int part = i / P.topk, j = i % P.topk;
      v = __ldcg(P.keys + ((size_t)part * P.batch + b) * P.topk + j);
    }
    cp_keys[i] = v;
  }
  __syncthreads();
  for (int k = 2; k <= np; k <<= 1) {           // ascending bitonic sort
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = threadIdx.x; i < np; i += kCpThreads) {
        const int x = i ^ j;
        if (x > i) {
          const uint64_t a = cp_keys[i], c = cp_keys[x];
          if (((i & k) == 0) == (a > c)) {
            cp_keys[i] = c;
            cp_keys[x] = a;
          }
        }
      }
      __syncthreads();
    }
  }
  // the topk largest are the last topk; their positions, padded to a power of two, sorted
  int kp = 1;
  while (kp < P.topk) kp <<= 1;
  uint32_t *pos = reinterpret_cast<uint32_t *>(cp_keys);   // reuses the front of the buffer
  uint32_t sel[HS2_MAX_TOPK / kCpThreads];
  int ns = 0;
  for (int i = threadIdx.x; i < kp; i += kCpThreads, ++ns)
    sel[ns] = (i < P.topk) ? 0xffffffffu - (uint32_t)cp_keys[np - 1 - i] : 0xffffffffu;
  __syncthreads();
  ns = 0;
  for (int i = threadIdx.x; i < kp; i += kCpThreads, ++ns) pos[i] = sel[ns];
  __syncthreads();
  for (int k = 2; k <= kp; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = threadIdx.x; i < kp; i += kCpThreads) {
        const int x = i ^ j;
        if (x > i) {
          const uint32_t a = pos[i], c = pos[x];
          if (((i & k) == 0) == (a > c)) {
            pos[i] = c;
            pos[x] = a;
          }
        }
      }
      __syncthreads();
    }
  }
  for (int i = threadIdx.x; i < P.topk; i += kCpThreads) out[i] = (int32_t)pos[i];
  for (int64_t t = nc + threadIdx.x; t <= p; t += kCpThreads) out[P.topk + (t - nc)] = (int32_t)t;
  if (threadIdx.x == 0) P.count_out[b] = (int32_t)(P.topk + (p - nc + 1));
}

// One CTA per sequence: the ascending global selection's positions inside this shard form one
// contiguous run; it is copied out shifted to local positions (possibly empty).
__global__ void __launch_bounds__(256) cp_localize_kernel(const __grid_constant__ CpParams P) {
  __shared__ int lo_s, hi_s;
  griddep_launch_dependents();
  griddep_wait();
  const int b = blockIdx.x;
  const int cnt = min(__ldcg(P.count + b), P.idx_stride);
  const int32_t *S = P.idx + (size_t)b * P.idx_stride;
  const int64_t g0 = P.offset[b], g1 = g0 + P.local_len[b];
  if (threadIdx.x == 0) {
    int lo = 0, hi = cnt;   // first entry >= g0
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (__ldcg(S + mid) < g0) lo = mid + 1;
      else hi = mid;
    }
    int lo2 = lo, hi2 = cnt;   // first entry >= g1
    while (lo2 < hi2) {
      const int mid = (lo2 + hi2) >> 1;
      if (__ldcg(S + mid) < g1) lo2 = mid + 1;
      else hi2 = mid;
    }
    lo_s = lo;
    hi_s = lo2;
  }
  __syncthreads();
  const int lo = lo_s, n = hi_s - lo_s;
  int32_t *out = P.idx_out + (size_t)b * P.out_stride;
  for (int j = threadIdx.x; j < n; j += blockDim.x) out[j] = (int32_t)(__ldcg(S + lo + j) - g0);
  if (threadIdx.x == 0) P.count_out[b] = n;
}

}  // namespace

cudaError_t launch_lse_merge(const LseMergeParams &p, cudaStream_t s) {
  if (p.rows * p.n_heads == 0) return cudaSuccess;
  cudaError_t e = launch_pdl(lse_merge_kernel, (int)(p.rows * p.n_heads), 128, 0, s, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_cp_pack(const CpParams &p, cudaStream_t s) {
  cudaError_t e = launch_pdl(cp_pack_kernel, p.batch, 256, 0, s, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_cp_select(const CpParams &p, cudaStream_t s) {
  const size_t smem = (size_t)kCpMaxKeys * 8;
  cudaError_t e = cudaFuncSetAttribute(cp_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  e = launch_pdl(cp_select_kernel, p.batch, kCpThreads, smem, s, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_cp_localize(const CpParams &p, cudaStream_t s) {
  cudaError_t e = launch_pdl(cp_localize_kernel, p.batch, 256, 0, s, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace hs2
