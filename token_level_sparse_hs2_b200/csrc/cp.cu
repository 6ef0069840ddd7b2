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
//    shards' own top-k, so each rank packs its top-k (score, global position) pairs in position
//    order (cp_pack_kernel) and every rank merges all of them (cp_select_kernel: a radix select
//    of the exact topk-th largest, then the keys above it in list order, which is position
//    order) to the same global selection, ties to the lower position, window appended as on
//    one GPU;
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

constexpr int kCpThreads = 512;
constexpr int kCpWarps = kCpThreads / 32;

// exclusive prefix sum over the CTA (kCpThreads threads) of one int per thread; *total = sum
__device__ int cp_block_scan(int v, int *warp_sums, int *total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int s = lane < kCpWarps ? warp_sums[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    if (lane < kCpWarps) warp_sums[lane] = s;
  }
  __syncthreads();
  const int before = (warp ? warp_sums[warp - 1] : 0) + x - v;
  *total = warp_sums[kCpWarps - 1];
  __syncthreads();
  return before;
}

// One CTA per sequence. The shard's selection idx is ascending and its global candidates
// (positions below the global window) come first, so they are packed in position order into the
// first slots; the remaining slots are empty (0).
__global__ void __launch_bounds__(kCpThreads) cp_pack_kernel(const __grid_constant__ CpParams P) {
  __shared__ int n_s;
  griddep_launch_dependents();
  griddep_wait();
  const int b = blockIdx.x;
  const int64_t wstart = (int64_t)P.global_len[b] - P.window;   // first window position
  const int cnt = min(min(__ldcg(P.count + b), P.idx_stride), P.topk + P.window);
  const int32_t *idx = P.idx + (size_t)b * P.idx_stride;
  const float *s = P.scores + (size_t)b * P.score_stride;
  uint64_t *keys = P.keys + (size_t)b * P.topk;
  if (threadIdx.x == 0) n_s = 0;
  __syncthreads();
  int mine = 0;
  for (int j = threadIdx.x; j < cnt; j += kCpThreads) {
    const int t = __ldcg(idx + j);
    const int64_t g = P.offset[b] + t;
    if (t >= 0 && t < P.local_len[b] && g < wstart && j < P.topk) {
      keys[j] = cp_key(__ldcg(s + t), g);
      ++mine;
    }
  }
  atomicAdd(&n_s, mine);
  __syncthreads();
  for (int j = n_s + threadIdx.x; j < P.topk; j += kCpThreads) keys[j] = 0;
}

// One CTA per sequence: the exact topk-th largest key tau of the n_parts x topk keys by a radix
// select on 8-bit digits from the top (stopping as soon as the bucket holds exactly the keys
// still needed), then the keys >= tau kept in list order -- shard by shard, each shard's keys in
// position order -- which is ascending position order; the window follows.
__global__ void __launch_bounds__(kCpThreads) cp_select_kernel(const __grid_constant__ CpParams P) {
  extern __shared__ __align__(16) uint64_t cp_keys[];
  __shared__ uint32_t hist[256];
  __shared__ int warp_sums[kCpWarps];
  __shared__ int bucket_s, above_s, inb_s;
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
  for (int i = threadIdx.x; i < n; i += kCpThreads) {
    const int part = i / P.topk, j = i % P.topk;
    cp_keys[i] = __ldcg(P.keys + ((size_t)part * P.batch + b) * P.topk + j);
  }
  __syncthreads();
  uint64_t prefix = 0, mask = 0;
  int need = P.topk;
  for (int shift = 56; shift >= 0; shift -= 8) {
    hist[threadIdx.x & 255] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += kCpThreads) {
      const uint64_t k = cp_keys[i];
      if ((k & mask) == prefix) atomicAdd(&hist[(k >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (threadIdx.x < 32) {   // bucket holding the need-th largest: one warp scans from the top
      const int lane = threadIdx.x;
      uint32_t c[8], sum = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        c[e] = hist[255 - (lane * 8 + e)];
        sum += c[e];
      }
      uint32_t incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      uint32_t run = incl - sum;
      if (run < (uint32_t)need && (uint32_t)need <= incl) {
        for (int e = 0; e < 8; ++e) {
          if (run + c[e] >= (uint32_t)need) {
            bucket_s = 255 - (lane * 8 + e);
            above_s = (int)run;
            inb_s = (int)c[e];
            break;
          }
          run += c[e];
        }
      }
    }
    __syncthreads();
    need -= above_s;
    prefix |= (uint64_t)bucket_s << shift;
    mask |= (uint64_t)0xff << shift;
    const bool whole = inb_s == need;   // every key of the bucket is kept
    __syncthreads();
    if (whole) break;
  }
  // keys with (key & mask) >= prefix are the topk largest; keep them in list order
  int run = 0;
  for (int i0 = 0; i0 < n; i0 += kCpThreads) {
    const int i = i0 + threadIdx.x;
    const bool take = i < n && (cp_keys[i] & mask) >= prefix;
    int tot;
    const int pos = cp_block_scan(take ? 1 : 0, warp_sums, &tot);
    if (take && run + pos < P.topk) out[run + pos] = (int32_t)(0xffffffffu - (uint32_t)cp_keys[i]);
    run += tot;
  }
  for (int64_t t = nc + threadIdx.x; t <= p; t += kCpThreads) out[P.topk + (t - nc)] = (int32_t)t;
  if (threadIdx.x == 0) P.count_out[b] = (int32_t)(P.topk + (p - nc + 1));
}

// One CTA per sequence: the ascending global selection's positions inside this shard form one
// contiguous run [lo, lo + n); it is copied out shifted to local positions (possibly empty).
__global__ void __launch_bounds__(kCpThreads) cp_localize_kernel(const __grid_constant__ CpParams P) {
  __shared__ int warp_sums[kCpWarps];
  griddep_launch_dependents();
  griddep_wait();
  const int b = blockIdx.x;
  const int cnt = min(__ldcg(P.count + b), P.idx_stride);
  const int32_t *S = P.idx + (size_t)b * P.idx_stride;
  const int64_t g0 = P.offset[b], g1 = g0 + P.local_len[b];
  int below = 0, inside = 0;
  for (int j = threadIdx.x; j < cnt; j += kCpThreads) {
    const int64_t g = __ldcg(S + j);
    below += g < g0;
    inside += g >= g0 && g < g1;
  }
  int lo, n;
  cp_block_scan(below, warp_sums, &lo);
  cp_block_scan(inside, warp_sums, &n);
  int32_t *out = P.idx_out + (size_t)b * P.out_stride;
  for (int j = threadIdx.x; j < n; j += kCpThreads) out[j] = (int32_t)(__ldcg(S + lo + j) - g0);
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
  cudaError_t e = launch_pdl(cp_pack_kernel, p.batch, kCpThreads, 0, s, p);
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
  cudaError_t e = launch_pdl(cp_localize_kernel, p.batch, kCpThreads, 0, s, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace hs2
