// topk.cu -- token-level selection: top-k of the candidate scores plus the forced window.
//
// "HySparse2: How Xiaomi Split the Transformer to Fix Agent Prefill Costs", section "KV Reuse
// and Token-Level Sparse Selection": the sparse budget is 1,024 individual tokens from the
// whole context plus a forced window of the 128 most recent tokens. For a query at position p
// the candidates are C = [0, nc), nc = p - window + 1, and the window is W = [nc, p]. If
// nc <= topk every position is kept; otherwise the topk candidates with the largest scores
// (ties: lower index) are kept, then W, in ascending order.
//
// Scores are non-negative fp32, so their bit patterns order like their values and the
// selection is an exact radix select on 32-bit keys:
//  1. top digit (bits 31..21) histogram: from the score pass (decode) or built here;
//  2. the bucket B1 holding the topk-th largest key; every candidate with digit >= B1 is
//     compacted (key, index) -- typically topk plus a few hundred;
//  3. in shared memory: the exact threshold key tau (digits 20..10, 9..0), how many keys equal
//     to tau are taken (the lowest indices: a radix select on the index), then the selected
//     indices are sorted (bitonic) and the window is appended.
// Long rows are split over several CTAs (segments) that compact into a global buffer; the last
// segment to arrive finishes the row. If the compacted set does not fit (many equal scores),
// the finishing CTA falls back to exact digit passes and an ordered scan over the whole row.
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "internal.h"

namespace hs2 {

namespace {

constexpr int kThreadsTk = 512;
constexpr int kWarpsTk = kThreadsTk / 32;
constexpr int kCandCap = 8192;     // candidates finished in shared memory

struct TkSmem {
  uint32_t hist[kHistBins];
  uint32_t key[kCandCap];
  int32_t idx[kCandCap];
  int32_t sel[HS2_MAX_TOPK];
  int32_t warp_sums[kWarpsTk];
  int32_t n_cand;
  int32_t n_sel;
  int32_t bucket;
  uint32_t above;
  int32_t last;
};

// One warp finds the bucket holding the `need`-th element counting from the top (desc) or
// the bottom (asc) of a histogram; result in sm.bucket / sm.above (count strictly before it).
__device__ void find_bucket(const uint32_t *hist, int nbins, uint32_t need, bool desc,
                            int32_t *out_bucket, uint32_t *out_before) {
  const int lane = threadIdx.x & 31;
  uint32_t run = 0;
  for (int base = 0; base < nbins; base += 32) {
    const int k = base + lane;
    const int bin = desc ? nbins - 1 - k : k;
    const uint32_t v = (k < nbins) ? hist[bin] : 0u;
    uint32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    const uint32_t tot = __shfl_sync(0xffffffffu, x, 31);
    if (run + tot >= need) {
      const unsigned ball = __ballot_sync(0xffffffffu, run + x >= need);
      const int first = __ffs(ball) - 1;
      const uint32_t before = __shfl_sync(0xffffffffu, x - v, first);
      if (lane == 0) {
        const int kk = base + first;
        *out_bucket = desc ? nbins - 1 - kk : kk;
        *out_before = run + before;
      }
      return;
    }
    run += tot;
  }
  if (lane == 0) {
    *out_bucket = desc ? 0 : nbins - 1;
    *out_before = run;
  }
}

// exclusive block-wide prefix sum of one int per thread; *total gets the block sum
__device__ int block_excl_scan(int v, int32_t *warp_sums, int *total) {
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
    int w = (lane < kWarpsTk) ? warp_sums[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < kWarpsTk) warp_sums[lane] = w;   // inclusive
  }
  __syncthreads();
  const int before = (warp > 0 ? warp_sums[warp - 1] : 0) + x - v;
  *total = warp_sums[kWarpsTk - 1];
  __syncthreads();
  return before;
}

__device__ __forceinline__ uint32_t load_key(const float *s, int64_t t) {
  return __float_as_uint(__ldg(s + t));
}

// Warp-aggregated append of (key, t) into a buffer of capacity cap; returns nothing, the
// counter keeps counting past cap so overflow is detectable.
template <bool kShared>
__device__ __forceinline__ void append(bool take, uint32_t key, int32_t t, int32_t *counter,
                                       uint32_t *kbuf, int32_t *ibuf, int cap) {
  const unsigned m = __ballot_sync(0xffffffffu, take);
  if (m == 0) return;
  const int lane = threadIdx.x & 31;
  const int leader = __ffs(m) - 1;
  int base = 0;
  if (lane == leader) base = atomicAdd(counter, __popc(m));
  base = __shfl_sync(0xffffffffu, base, leader);
  if (take) {
    const int slot = base + __popc(m & ((1u << lane) - 1u));
    if (slot < cap) {
      kbuf[slot] = key;
      ibuf[slot] = t;
    }
  }
}

// Exact finish on n <= kCandCap candidates in shared memory that contain every candidate with
// top digit >= B1 (above = how many have top digit > B1). Writes the ascending selection.
__device__ void finish_from_smem(TkSmem &sm, int n, int B1, uint32_t above, int topk,
                                 int32_t *out) {
  uint32_t prefix = (uint32_t)B1 << 21, mask = 0xffe00000u;
  uint32_t need = topk - above;
  const int shifts[2] = {10, 0};
  const int widths[2] = {11, 10};
  uint32_t n_eq = 0;
  for (int pass = 0; pass < 2; ++pass) {
    const int sh = shifts[pass], nb = 1 << widths[pass];
    for (int t = threadIdx.x; t < nb; t += kThreadsTk) sm.hist[t] = 0;
    __syncthreads();
    for (int t = threadIdx.x; t < n; t += kThreadsTk) {
      const uint32_t k = sm.key[t];
      if ((k & mask) == prefix) atomicAdd(&sm.hist[(k >> sh) & (nb - 1)], 1u);
    }
    __syncthreads();
    if (threadIdx.x < 32) find_bucket(sm.hist, nb, need, true, &sm.bucket, &sm.above);
    __syncthreads();
    const int bk = sm.bucket;
    need -= sm.above;
    prefix |= (uint32_t)bk << sh;
    mask |= (uint32_t)(nb - 1) << sh;
    if (pass == 1) n_eq = sm.hist[bk];
    __syncthreads();
  }
  const uint32_t tau = prefix;
  // index threshold among keys equal to tau: the need-th smallest index
  int32_t ithr = 0x7fffffff;
  if (need < n_eq) {
    uint32_t iprefix = 0, imask = 0, ineed = need;
    const int ish[3] = {21, 10, 0};
    const int iw[3] = {11, 11, 10};
    for (int pass = 0; pass < 3; ++pass) {
      const int sh = ish[pass], nb = 1 << iw[pass];
      for (int t = threadIdx.x; t < nb; t += kThreadsTk) sm.hist[t] = 0;
      __syncthreads();
      for (int t = threadIdx.x; t < n; t += kThreadsTk) {
        const uint32_t ix = (uint32_t)sm.idx[t];
        if (sm.key[t] == tau && (ix & imask) == iprefix) atomicAdd(&sm.hist[(ix >> sh) & (nb - 1)], 1u);
      }
      __syncthreads();
      if (threadIdx.x < 32) find_bucket(sm.hist, nb, ineed, false, &sm.bucket, &sm.above);
      __syncthreads();
      ineed -= sm.above;
      iprefix |= (uint32_t)sm.bucket << sh;
      imask |= (uint32_t)(nb - 1) << sh;
      __syncthreads();
    }
    ithr = (int32_t)iprefix;
  }
  // gather the selected indices
  if (threadIdx.x == 0) sm.n_sel = 0;
  __syncthreads();
  for (int t = threadIdx.x; t < ((n + 31) & ~31); t += kThreadsTk) {
    bool take = false;
    uint32_t k = 0;
    int32_t ix = 0;
    if (t < n) {
      k = sm.key[t];
      ix = sm.idx[t];
      take = k > tau || (k == tau && ix <= ithr);
    }
    const unsigned m = __ballot_sync(0xffffffffu, take);
    if (m) {
      const int lane = threadIdx.x & 31, leader = __ffs(m) - 1;
      int base = 0;
      if (lane == leader) base = atomicAdd(&sm.n_sel, __popc(m));
      base = __shfl_sync(0xffffffffu, base, leader);
      if (take) {
        const int slot = base + __popc(m & ((1u << lane) - 1u));
        if (slot < HS2_MAX_TOPK) sm.sel[slot] = ix;
      }
    }
  }
  __syncthreads();
  // bitonic sort of the topk selected indices (ascending), padded to a power of two
  int N = 2;
  while (N < topk) N <<= 1;
  for (int t = topk + threadIdx.x; t < N; t += kThreadsTk) sm.sel[t] = 0x7fffffff;
  __syncthreads();
  for (int k = 2; k <= N; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int t = threadIdx.x; t < N; t += kThreadsTk) {
        const int u = t ^ j;
        if (u > t) {
          const int a = sm.sel[t], c = sm.sel[u];
          const bool up = (t & k) == 0;
          if ((a > c) == up) {
            sm.sel[t] = c;
            sm.sel[u] = a;
          }
        }
      }
      __syncthreads();
    }
  }
  for (int t = threadIdx.x; t < topk; t += kThreadsTk) out[t] = sm.sel[t];
}

// Exact fallback over the whole candidate row in global memory (any number of equal keys):
// digit passes find tau, then one ordered scan writes the selection in index order.
__device__ void finish_from_global(TkSmem &sm, const float *s, int64_t nc, int B1,
                                   uint32_t above, int topk, int32_t *out) {
  uint32_t prefix = (uint32_t)B1 << 21, mask = 0xffe00000u;
  uint32_t need = topk - above;
  const int shifts[2] = {10, 0};
  const int widths[2] = {11, 10};
  for (int pass = 0; pass < 2; ++pass) {
    const int sh = shifts[pass], nb = 1 << widths[pass];
    for (int t = threadIdx.x; t < nb; t += kThreadsTk) sm.hist[t] = 0;
    __syncthreads();
    for (int64_t t = threadIdx.x; t < nc; t += kThreadsTk) {
      const uint32_t k = load_key(s, t);
      if ((k & mask) == prefix) atomicAdd(&sm.hist[(k >> sh) & (nb - 1)], 1u);
    }
    __syncthreads();
    if (threadIdx.x < 32) find_bucket(sm.hist, nb, need, true, &sm.bucket, &sm.above);
    __syncthreads();
    need -= sm.above;
    prefix |= (uint32_t)sm.bucket << sh;
    mask |= (uint32_t)(nb - 1) << sh;
    __syncthreads();
  }
  const uint32_t tau = prefix;
  const int need_eq = (int)need;
  int eq_run = 0, out_run = 0;
  for (int64_t base = 0; base < nc; base += kThreadsTk) {
    const int64_t t = base + threadIdx.x;
    uint32_t k = 0;
    if (t < nc) k = load_key(s, t);
    const int is_eq = (t < nc && k == tau) ? 1 : 0;
    int tot_eq;
    const int eq_before = block_excl_scan(is_eq, sm.warp_sums, &tot_eq);
    const bool take = (t < nc) && (k > tau || (is_eq && eq_run + eq_before < need_eq));
    int tot_sel;
    const int sel_before = block_excl_scan(take ? 1 : 0, sm.warp_sums, &tot_sel);
    if (take) out[out_run + sel_before] = (int32_t)t;
    eq_run += tot_eq;
    out_run += tot_sel;
  }
}

}  // namespace

// Global top-digit histogram of the candidates of each row (used when the score pass did not
// produce one and the row is split over several CTAs).
__global__ void __launch_bounds__(kThreadsTk) topk_hist_kernel(const __grid_constant__ TopkParams P) {
  __shared__ uint32_t hist[kHistBins];
  const int r = blockIdx.x / P.n_seg, sg = blockIdx.x % P.n_seg;
  const int b = r / P.n_q, i = r % P.n_q;
  const int64_t p = (int64_t)P.seq.len[b] - P.n_q + i;
  const int64_t nc = max((int64_t)0, p - P.window + 1);
  if (nc <= P.topk) return;
  for (int t = threadIdx.x; t < kHistBins; t += kThreadsTk) hist[t] = 0;
  __syncthreads();
  const float *s = P.scores + (size_t)r * P.score_stride;
  const int64_t s0 = (int64_t)sg * P.seg_len, s1 = min(nc, s0 + P.seg_len);
  for (int64_t t = s0 + threadIdx.x; t < s1; t += kThreadsTk)
    atomicAdd(&hist[load_key(s, t) >> 21], 1u);
  __syncthreads();
  uint32_t *gh = P.hist_ws + (size_t)r * kHistBins;
  for (int t = threadIdx.x; t < kHistBins; t += kThreadsTk)
    if (hist[t]) atomicAdd(&gh[t], hist[t]);
}

__global__ void __launch_bounds__(kThreadsTk) topk_select_kernel(const __grid_constant__ TopkParams P) {
  extern __shared__ __align__(16) uint8_t tk_raw[];
  TkSmem &sm = *reinterpret_cast<TkSmem *>(tk_raw);
  const int r = blockIdx.x / P.n_seg, sg = blockIdx.x % P.n_seg;
  const int b = r / P.n_q, i = r % P.n_q;
  const int64_t p = (int64_t)P.seq.len[b] - P.n_q + i;
  const int64_t nc = max((int64_t)0, p - P.window + 1);
  int32_t *out = P.idx + (size_t)r * P.idx_stride;
  if (nc <= P.topk) {
    if (sg == 0) {
      for (int64_t t = threadIdx.x; t <= p; t += kThreadsTk) out[t] = (int32_t)t;
      if (threadIdx.x == 0) P.count[r] = (int32_t)(p + 1);
    }
    return;
  }
  const float *s = P.scores + (size_t)r * P.score_stride;
  // 1. top-digit histogram
  const uint32_t *gh = P.hist ? P.hist + (size_t)r * kHistBins
                              : (P.hist_ws ? P.hist_ws + (size_t)r * kHistBins : nullptr);
  if (gh) {
    for (int t = threadIdx.x; t < kHistBins; t += kThreadsTk) sm.hist[t] = __ldcg(gh + t);
  } else {   // single segment: build it here
    for (int t = threadIdx.x; t < kHistBins; t += kThreadsTk) sm.hist[t] = 0;
    __syncthreads();
    for (int64_t t = threadIdx.x; t < nc; t += kThreadsTk) atomicAdd(&sm.hist[load_key(s, t) >> 21], 1u);
  }
  if (threadIdx.x == 0) sm.n_cand = 0;
  __syncthreads();
  // 2. bucket of the topk-th largest key
  if (threadIdx.x < 32) find_bucket(sm.hist, kHistBins, (uint32_t)P.topk, true, &sm.bucket, &sm.above);
  __syncthreads();
  const int B1 = sm.bucket;
  const uint32_t above = sm.above;
  // 3. compact every candidate of this segment with top digit >= B1
  const int64_t s0 = (int64_t)sg * P.seg_len, s1 = min(nc, s0 + P.seg_len);
  const int64_t span = s1 - s0;
  const int64_t steps = (span + kThreadsTk - 1) / kThreadsTk;
  int32_t *gcount = P.cand_count + r;
  uint32_t *gkey = P.cand_key + (size_t)r * P.cand_cap;
  int32_t *gidx = P.cand_idx + (size_t)r * P.cand_cap;
  for (int64_t it = 0; it < steps; ++it) {
    const int64_t t = s0 + it * kThreadsTk + threadIdx.x;
    uint32_t k = 0;
    bool take = false;
    if (t < s1) {
      k = load_key(s, t);
      take = (int)(k >> 21) >= B1;
    }
    if (P.n_seg == 1) append<true>(take, k, (int32_t)t, &sm.n_cand, sm.key, sm.idx, kCandCap);
    else append<false>(take, k, (int32_t)t, gcount, gkey, gidx, P.cand_cap);
  }
  int n;
  if (P.n_seg == 1) {
    __syncthreads();
    n = sm.n_cand;
  } else {
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
      const int prev = atomicAdd(P.arrive + r, 1);
      sm.last = (prev == P.n_seg - 1);
    }
    __syncthreads();
    if (!sm.last) return;
    __threadfence();
    n = __ldcg(gcount);
    if (n <= kCandCap) {
      for (int t = threadIdx.x; t < n; t += kThreadsTk) {
        sm.key[t] = __ldcg(gkey + t);
        sm.idx[t] = __ldcg(gidx + t);
      }
    }
    __syncthreads();
    if (threadIdx.x == 0) {   // ready for the next call
      P.arrive[r] = 0;
      *gcount = 0;
    }
  }
  // 4. finish
  const bool fits = (P.n_seg == 1) ? (n <= kCandCap) : (n <= kCandCap && n <= P.cand_cap);
  if (fits) finish_from_smem(sm, n, B1, above, P.topk, out);
  else finish_from_global(sm, s, nc, B1, above, P.topk, out);
  // 5. the forced window
  for (int64_t t = nc + threadIdx.x; t <= p; t += kThreadsTk) out[P.topk + (t - nc)] = (int32_t)t;
  if (threadIdx.x == 0) P.count[r] = (int32_t)(P.topk + (p - nc + 1));
}

size_t topk_smem_bytes() { return sizeof(TkSmem); }

cudaError_t launch_topk(const TopkParams &p, int n_rows, cudaStream_t s) {
  const size_t smem = sizeof(TkSmem);
  cudaError_t e = cudaFuncSetAttribute(topk_select_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int grid = n_rows * p.n_seg;
  if (!p.hist && p.n_seg > 1) {
    topk_hist_kernel<<<grid, kThreadsTk, 0, s>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  topk_select_kernel<<<grid, kThreadsTk, smem, s>>>(p);
  return cudaGetLastError();
}

}  // namespace hs2
