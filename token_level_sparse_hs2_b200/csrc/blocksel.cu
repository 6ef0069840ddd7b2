// blocksel.cu -- block-level selection: the granularity HySparse used and HySparse2 replaces.
//
// "HySparse2: How Xiaomi Split the Transformer to Fix Agent Prefill Costs", section "KV Reuse
// and Token-Level Sparse Selection": block-level selection spends the sparse budget on blocks of
// 64 tokens at once, the token-level variant spends the same 1,024 tokens one by one, plus the
// forced window of the 128 most recent tokens. For a query at position p the candidates
// C = [0, nc), nc = p - window + 1, are cut at multiples of the block size bs; a block's score
// is the sum of its candidates' scores; the topk / bs best blocks (ties: lower block index)
// are kept, their positions ascending, then the window [nc, p]. If nc <= topk every position
// is kept.
//
// Two kernels:
//  1. pool: every warp sums 128-token stretches of a score row into block scores. The float32
//     sum of a block folds it in half (v[i] + v[i + n/2], n = bs ... 2, zeros past nc), which is
//     what a shuffle butterfly computes when lane l holds positions l, l + 32, ...; the order
//     is fixed, so the block scores (and the selection) depend on the fp32 scores alone.
//  2. select: one CTA per query row; the keys (fp32 bit patterns of the block scores, ordered
//     like their values, packed with the negated block index so that all are distinct) are
//     staged in shared memory; a lower bound from the per-thread maxima filters them down to a
//     few candidates that are ranked exactly (below); the winners are put in ascending order
//     and expanded to positions.
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "internal.h"

namespace hs2 {

namespace {

constexpr int kPoolThreads = 256;
constexpr int kPoolSpan = 128;                       // positions a warp sums per step
constexpr int kPoolSteps = 4;                        // steps per warp per CTA
constexpr int kSelThreads = 256;
constexpr int kSelWarps = kSelThreads / 32;

__device__ __forceinline__ float warp_fold(float v, int from) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1)
    if (o <= from) v = __fadd_rn(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// One warp sums kPoolSteps 128-position stretches of a score row (stretches st0 + u * 8) into
// block scores out[j] (global or shared memory); positions at or past nc count as 0 and blocks
// that start at or past nc are not written. Lane l holds positions t0 + l + 32 m, m < 4.
template <int BS>
__device__ __forceinline__ void pool_stretches(const float *s, int64_t nc, int64_t st0, int lane,
                                               float *out) {
  float x[kPoolSteps][4];
#pragma unroll
  for (int u = 0; u < kPoolSteps; ++u) {
    const int64_t t0 = (st0 + (int64_t)u * (kPoolThreads / 32)) * kPoolSpan;
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const int64_t t = t0 + 32 * m + lane;
      x[u][m] = t < nc ? __ldg(s + t) : 0.0f;
    }
  }
#pragma unroll
  for (int u = 0; u < kPoolSteps; ++u) {
    const int64_t t0 = (st0 + (int64_t)u * (kPoolThreads / 32)) * kPoolSpan;
    if (t0 >= nc) continue;
    const int64_t j0 = t0 / BS;                      // first block of this stretch
    if constexpr (BS == 128) {
      // 128 -> 64: (l, l + 64) and (l + 32, l + 96); 64 -> 32: their sum; then the butterfly
      const float v = warp_fold(__fadd_rn(__fadd_rn(x[u][0], x[u][2]), __fadd_rn(x[u][1], x[u][3])), 16);
      if (lane == 0) out[j0] = v;
    } else if constexpr (BS == 64) {
      const float v0 = warp_fold(__fadd_rn(x[u][0], x[u][1]), 16);
      const float v1 = warp_fold(__fadd_rn(x[u][2], x[u][3]), 16);
      if (lane == 0) {
        out[j0] = v0;
        if (t0 + 64 < nc) out[j0 + 1] = v1;
      }
    } else {                                         // 32 or 16: lanes hold whole blocks
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const float v = warp_fold(x[u][m], BS / 2);
        const int64_t t = t0 + 32 * m + lane;        // block start when lane % BS == 0
        if ((lane & (BS - 1)) == 0 && t < nc) out[t / BS] = v;
      }
    }
  }
}

// Block scores of the long rows, spread over pool_ctas_per_row CTAs per row.
template <int BS>
__global__ void __launch_bounds__(kPoolThreads) block_pool_kernel(const __grid_constant__ BlockSelParams P) {
  griddep_launch_dependents();
  griddep_wait();
  const int r = blockIdx.x / P.pool_ctas_per_row, c = blockIdx.x % P.pool_ctas_per_row;
  const int b = r / P.n_q, i = r % P.n_q;
  const int64_t p = (int64_t)P.seq.len[b] - P.n_q + i;
  const int64_t nc = max((int64_t)0, p - P.window + 1);
  if (nc <= P.topk) return;                          // the row keeps every position
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t st0 = (int64_t)c * (kPoolThreads / 32) * kPoolSteps + warp;
  pool_stretches<BS>(P.scores + (size_t)r * P.score_stride, nc, st0, lane,
                     P.blk + (size_t)r * P.blk_stride);
}

// (key, block) packed so that the larger value is the higher score, then the lower block
__device__ __forceinline__ uint64_t pack_key(uint32_t key, int j) {
  return ((uint64_t)key << 32) | (uint64_t)(0xffffffffu - (uint32_t)j);
}

__device__ __forceinline__ uint64_t warp_max_u64(uint64_t v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    const uint64_t w = __shfl_xor_sync(0xffffffffu, v, o);
    v = w > v ? w : v;
  }
  return v;
}

// Exact top-kb of the composites (key, -block) of one row, all distinct:
//  a. every thread's best over its blocks j = tid, tid + 256, ...;
//  b. the bests of groups of blocks (j mod 64, or j mod 256 when kb >= 64); L = the kb-th
//     largest group best (a rank count over them). At least kb composites are >= L (the
//     kb best group bests), so the kb-th largest overall is >= L, and only the kb groups whose
//     best is >= L can hold such composites;
//  c. those groups compact their composites >= L into shared memory (at most kb x blocks
//     per group, typically a few dozen);
//  d. each candidate's rank is the number of larger candidates; ranks < kb are the winners.
// Rows whose candidates overflow the buffer take kb rounds of a block-wide arg-max instead.
constexpr int kCandMax = 2048;

// FUSED_BS > 0: the CTA computes its row's block scores itself (many short rows); 0: they come
// from block_pool_kernel.
template <int FUSED_BS>
__global__ void __launch_bounds__(kSelThreads) block_select_kernel(const __grid_constant__ BlockSelParams P) {
  extern __shared__ __align__(16) uint32_t bs_keys[];
  __shared__ uint64_t tbest[kSelThreads];
  __shared__ uint64_t gmax[kSelThreads];
  __shared__ uint64_t cand[kCandMax];
  __shared__ uint64_t red[kSelWarps];
  __shared__ uint64_t lim_s;
  __shared__ int32_t n_cand;
  __shared__ int32_t sel[HS2_MAX_TOPK / 16];
  __shared__ int32_t sorted_sel[HS2_MAX_TOPK / 16];
  griddep_launch_dependents();
  griddep_wait();
  const int r = blockIdx.x;
  const int b = r / P.n_q, i = r % P.n_q;
  const int64_t p = (int64_t)P.seq.len[b] - P.n_q + i;
  const int64_t nc = max((int64_t)0, p - P.window + 1);
  int32_t *out = P.idx + (size_t)r * P.idx_stride;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (r == 0 && tid == 0) *P.status = 0;             // nothing here records a device error
  if (nc <= P.topk) {
    for (int64_t t = tid; t <= p; t += kSelThreads) out[t] = (int32_t)t;
    if (tid == 0) P.count[r] = (int32_t)(p + 1);
    return;
  }
  const int bs = P.bs, kb = P.kb;
  const int nb = (int)((nc + bs - 1) / bs);
  const uint32_t *g = reinterpret_cast<const uint32_t *>(P.blk + (size_t)r * P.blk_stride);
  const uint32_t *key = g;
  if (tid == 0) n_cand = 0;
  if constexpr (FUSED_BS > 0) {      // pool this row into shared memory (nb <= smem_keys)
    const float *srow = P.scores + (size_t)r * P.score_stride;
    float *kf = reinterpret_cast<float *>(bs_keys);
    constexpr int kGroup = kSelWarps * kPoolSteps;   // stretches per CTA pass
    for (int64_t g0 = 0; g0 * kPoolSpan < nc; g0 += kGroup)
      pool_stretches<FUSED_BS>(srow, nc, g0 + warp, lane, kf);
    __syncthreads();
    key = bs_keys;
  } else if (nb <= P.smem_keys) {    // stage: 16-byte loads, eight in flight per thread
    const int n4 = (nb + 3) >> 2;
    const uint4 *g4 = reinterpret_cast<const uint4 *>(g);
    uint4 *s4 = reinterpret_cast<uint4 *>(bs_keys);
    for (int q0 = 0; q0 < n4; q0 += 8 * kSelThreads) {
      uint4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int q = q0 + u * kSelThreads + tid;
        if (q < n4) v[u] = __ldcg(g4 + q);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int q = q0 + u * kSelThreads + tid;
        if (q < n4) s4[q] = v[u];
      }
    }
    __syncthreads();
    key = bs_keys;
  }
  // a.
  uint64_t best = 0;
  for (int j = tid; j < nb; j += kSelThreads) {
    const uint64_t v = pack_key(key[j], j);
    best = v > best ? v : best;
  }
  // group g = the threads tid with tid % n_groups == g, i.e. the blocks j with
  // j % n_groups == g: every one of the first min(nb, n_groups) groups holds a block, and
  // nb > kb, so at least kb + 1 groups have one when n_groups > kb
  const int n_groups = kb < 64 ? 64 : kSelThreads;
  tbest[tid] = best;
  __syncthreads();
  if (tid < n_groups) {
    uint64_t g = 0;
    for (int u = tid; u < kSelThreads; u += n_groups) g = tbest[u] > g ? tbest[u] : g;
    gmax[tid] = g;
  }
  __syncthreads();
  const uint64_t gbest = gmax[tid % n_groups];
  // b. (groups without blocks hold 0 and rank below every real composite)
  if (tid < n_groups) {
    int rank = 0;
#pragma unroll 8
    for (int u = 0; u < n_groups; ++u) rank += gmax[u] > gbest;
    if (rank == kb - 1) lim_s = gbest;
  }
  __syncthreads();
  const uint64_t lim = lim_s;
  // c.
  if (gbest >= lim) {
    for (int j = tid; j < nb; j += kSelThreads) {
      const uint64_t v = pack_key(key[j], j);
      if (v >= lim) {
        const int slot = atomicAdd(&n_cand, 1);
        if (slot < kCandMax) cand[slot] = v;
      }
    }
  }
  __syncthreads();
  const int nC = n_cand;
  if (nC <= kCandMax) {
    // d.
    for (int c = tid; c < nC; c += kSelThreads) {
      const uint64_t v = cand[c];
      int rank = 0;
      for (int u = 0; u < nC; ++u) rank += cand[u] > v;
      if (rank < kb) sel[rank] = (int32_t)(0xffffffffu - (uint32_t)v);
    }
  } else {
    for (int round = 0; round < kb; ++round) {
      const uint64_t w = warp_max_u64(best);
      if (lane == 0) red[warp] = w;
      __syncthreads();
      if (warp == 0) {
        uint64_t v = lane < kSelWarps ? red[lane] : 0;
        v = warp_max_u64(v);
        if (lane == 0) {
          lim_s = v;
          sel[round] = (int32_t)(0xffffffffu - (uint32_t)v);
        }
      }
      __syncthreads();
      const uint64_t win = lim_s;
      const int jw = (int)(0xffffffffu - (uint32_t)win);
      if ((jw % kSelThreads) == tid) {              // the winner's owner: next best below it
        best = 0;
        for (int j = tid; j < nb; j += kSelThreads) {
          const uint64_t v = pack_key(key[j], j);
          if (v < win && v > best) best = v;
        }
      }
      __syncthreads();
    }
  }
  __syncthreads();
  if (tid < kb) {                                    // rank among the (distinct) winners
    const int x = sel[tid];
    int rank = 0;
    for (int u = 0; u < kb; ++u) rank += sel[u] < x;
    sorted_sel[rank] = x;
  }
  __syncthreads();
  // expand: winner k owns out[k * bs, (k + 1) * bs); only the last block of C can be short, and
  // if chosen it is the last winner in ascending order
  for (int e = tid; e < kb * bs; e += kSelThreads) {
    const int k = e / bs, u = e % bs;
    const int64_t t = (int64_t)sorted_sel[k] * bs + u;
    if (t < nc) out[e] = (int32_t)t;
  }
  const int64_t last_end = min(nc, ((int64_t)sorted_sel[kb - 1] + 1) * bs);
  const int64_t cnt = (int64_t)(kb - 1) * bs + (last_end - (int64_t)sorted_sel[kb - 1] * bs);
  for (int64_t t = nc + tid; t <= p; t += kSelThreads) out[cnt + (t - nc)] = (int32_t)t;
  if (tid == 0) P.count[r] = (int32_t)(cnt + (p - nc + 1));
}

}  // namespace

int block_pool_positions_per_cta() { return (kPoolThreads / 32) * kPoolSteps * kPoolSpan; }

template <class K>
cudaError_t set_smem(K kernel, size_t smem) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
}

cudaError_t launch_block_select(const BlockSelParams &p, int n_rows, cudaStream_t s) {
  const size_t smem = (size_t)p.smem_keys * 4;
  cudaError_t e;
  if (p.fused) {
    switch (p.bs) {
      case 16: if ((e = set_smem(block_select_kernel<16>, smem)) == cudaSuccess)
                 e = launch_pdl(block_select_kernel<16>, n_rows, kSelThreads, smem, s, p); break;
      case 32: if ((e = set_smem(block_select_kernel<32>, smem)) == cudaSuccess)
                 e = launch_pdl(block_select_kernel<32>, n_rows, kSelThreads, smem, s, p); break;
      case 64: if ((e = set_smem(block_select_kernel<64>, smem)) == cudaSuccess)
                 e = launch_pdl(block_select_kernel<64>, n_rows, kSelThreads, smem, s, p); break;
      case 128: if ((e = set_smem(block_select_kernel<128>, smem)) == cudaSuccess)
                 e = launch_pdl(block_select_kernel<128>, n_rows, kSelThreads, smem, s, p); break;
      default: return cudaErrorInvalidValue;
    }
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
  }
  const int pool_grid = n_rows * p.pool_ctas_per_row;
  switch (p.bs) {
    case 16: e = launch_pdl(block_pool_kernel<16>, pool_grid, kPoolThreads, 0, s, p); break;
    case 32: e = launch_pdl(block_pool_kernel<32>, pool_grid, kPoolThreads, 0, s, p); break;
    case 64: e = launch_pdl(block_pool_kernel<64>, pool_grid, kPoolThreads, 0, s, p); break;
    case 128: e = launch_pdl(block_pool_kernel<128>, pool_grid, kPoolThreads, 0, s, p); break;
    default: return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  if ((e = set_smem(block_select_kernel<0>, smem)) != cudaSuccess) return e;
  e = launch_pdl(block_select_kernel<0>, n_rows, kSelThreads, smem, s, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace hs2
