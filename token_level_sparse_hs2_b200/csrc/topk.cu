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
// selection is an exact radix select on 32-bit keys (a negative or NaN candidate score breaks
// that order: it is recorded in the status word as a device check):
//  1. top digit (bits 31..21) histogram: from the score pass (decode) or built here;
//  2. the bucket B1 holding the topk-th largest key; every candidate with digit >= B1 is
//     compacted (key, index) in position order (a ballot per warp and step and one block-wide
//     scan) -- typically topk plus a few hundred;
//  3. in shared memory: the exact threshold key tau (digits 20..10, 9..0), how many keys equal
//     to tau are taken (the lowest indices: a radix select on the index); one more ordered
//     compaction keeps the selected candidates in ascending order, and the window is appended.
// Long rows are split over several CTAs (segments). Up to 8 segments form a thread-block
// cluster and each stores its run into segment 0's shared memory; more segments compact
// into a global buffer and record where their run starts, and the last segment to arrive lays
// the runs out in segment order. Either way one CTA finishes the row. If the compacted set does not fit (many equal scores),
// the finishing CTA falls back to exact digit passes and an ordered scan over the whole row.
#include <cooperative_groups.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "internal.h"

namespace hs2 {

namespace {

constexpr int kThreadsTk = 512;
constexpr int kWarpsTk = kThreadsTk / 32;
constexpr int kCandCap = 8192;     // candidates finished in shared memory
constexpr int kUnroll = 8;         // independent score loads in flight per thread

struct TkSmem {
  uint32_t hist[kHistBins];
  uint32_t key[kCandCap];
  int32_t idx[kCandCap];
  int32_t scan[kThreadsTk];        // per (step, warp) counts of an ordered compaction
  int32_t seg_pre[kThreadsTk + 1]; // finishing CTA: candidates before each segment
  int32_t seg_src[kThreadsTk];     // finishing CTA: where each segment's candidates start
  int32_t warp_sums[kWarpsTk];
  int32_t bucket;
  uint32_t above;
  int32_t last;
};

// Finds the bucket holding the `need`-th element counting from the top (desc) or the bottom
// (asc) of a histogram, and how many elements come before it. Called by all threads
// (nbins = 1024 or 2048): each thread owns nbins / 512 consecutive positions of the scan
// order and one block scan finds the thread whose positions hold the target. The result is
// in *out_bucket / *out_before for every thread on return.
__device__ int block_excl_scan(int v, int32_t *warp_sums, int *total);

__device__ void find_bucket_block(const uint32_t *hist, int nbins, uint32_t need, bool desc,
                                  int32_t *warp_sums, int32_t *out_bucket, uint32_t *out_before) {
  const int E = nbins / kThreadsTk;
  const int k0 = threadIdx.x * E;
  if (threadIdx.x == 0) {   // only reached if need exceeds the total
    *out_bucket = desc ? 0 : nbins - 1;
    *out_before = 0;
  }
  uint32_t loc = 0;
  for (int e = 0; e < E; ++e) loc += hist[desc ? nbins - 1 - (k0 + e) : k0 + e];
  int tot;
  const uint32_t pre = (uint32_t)block_excl_scan((int)loc, warp_sums, &tot);
  if (pre < need && need <= pre + loc) {
    uint32_t run = pre;
    for (int e = 0; e < E; ++e) {
      const int bin = desc ? nbins - 1 - (k0 + e) : k0 + e;
      const uint32_t v = hist[bin];
      if (run + v >= need) {
        *out_bucket = bin;
        *out_before = run;
        break;
      }
      run += v;
    }
  }
  __syncthreads();
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

// Ordered compaction of one step of U elements per thread, element u of thread x standing at
// position u * kThreadsTk + x of the step (so consecutive threads read consecutive keys): the
// taken elements are numbered in that order, continuing from *run (the same in every thread),
// and emit(slot, u) is called for each. A ballot per (u, warp) and one block-wide scan over the
// U x kWarpsTk counts give every element its slot.
template <int U, class Emit>
__device__ __forceinline__ void ordered_append(uint32_t take_bits, TkSmem &sm, int &run, Emit emit) {
  static_assert(U * kWarpsTk <= kThreadsTk && U <= 32, "one scan entry per thread");
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  unsigned m[U];
  int mine = 0;   // lane u holds the count of step u
#pragma unroll
  for (int u = 0; u < U; ++u) {
    m[u] = __ballot_sync(0xffffffffu, (take_bits >> u) & 1u);
    if (lane == u) mine = __popc(m[u]);
  }
  if (lane < U) sm.scan[lane * kWarpsTk + warp] = mine;
  __syncthreads();
  const int v = threadIdx.x < U * kWarpsTk ? sm.scan[threadIdx.x] : 0;
  int tot;
  const int ex = block_excl_scan(v, sm.warp_sums, &tot);
  if (threadIdx.x < U * kWarpsTk) sm.scan[threadIdx.x] = ex;
  __syncthreads();
  const int base_mine = lane < U ? sm.scan[lane * kWarpsTk + warp] : 0;   // offset of step lane
  const unsigned below = (1u << lane) - 1u;
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int base = __shfl_sync(0xffffffffu, base_mine, u);
    if ((take_bits >> u) & 1u) emit(run + base + __popc(m[u] & below), u);
  }
  run += tot;
  __syncthreads();   // sm.scan is reused by the next step
}

// Writes, in order, the candidates among the first n <= U * kThreadsTk in shared memory (in
// ascending position order) whose key is above tau, or equal to it with an index <= ithr.
template <int U>
__device__ __forceinline__ void keep_ordered(TkSmem &sm, int n, uint32_t tau, int32_t ithr,
                                             int topk, int32_t *out) {
  uint32_t take = 0;
  int32_t ix[U];
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int j = u * kThreadsTk + threadIdx.x;
    ix[u] = 0;
    if (j < n) {
      const uint32_t k = sm.key[j];
      ix[u] = sm.idx[j];
      if (k > tau || (k == tau && ix[u] <= ithr)) take |= 1u << u;
    }
  }
  int run = 0;
  ordered_append<U>(take, sm, run, [&](int slot, int u) {
    if (slot < topk) out[slot] = ix[u];
  });
}

// Exact finish on n <= kCandCap candidates in shared memory, in ascending position order, that
// contain every candidate with top digit >= B1 (above = how many have top digit > B1). Writes
// the ascending selection.
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
    find_bucket_block(sm.hist, nb, need, true, sm.warp_sums, &sm.bucket, &sm.above);
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
      find_bucket_block(sm.hist, nb, ineed, false, sm.warp_sums, &sm.bucket, &sm.above);
      ineed -= sm.above;
      iprefix |= (uint32_t)sm.bucket << sh;
      imask |= (uint32_t)(nb - 1) << sh;
      __syncthreads();
    }
    ithr = (int32_t)iprefix;
  }
  // the candidates are in ascending position order: keep those above the threshold in that
  // order, with as many steps per thread as the candidates need
  static_assert(kCandCap == 16 * kThreadsTk, "one ordered step covers the candidates");
  if (n <= 4 * kThreadsTk) keep_ordered<4>(sm, n, tau, ithr, topk, out);
  else if (n <= 8 * kThreadsTk) keep_ordered<8>(sm, n, tau, ithr, topk, out);
  else keep_ordered<16>(sm, n, tau, ithr, topk, out);
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
    for (int64_t base = 0; base < nc; base += kThreadsTk * kUnroll) {
      uint32_t k[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int64_t t = base + u * kThreadsTk + threadIdx.x;
        k[u] = t < nc ? load_key(s, t) : 0u;
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u)
        if (base + u * kThreadsTk + threadIdx.x < nc && (k[u] & mask) == prefix)
          atomicAdd(&sm.hist[(k[u] >> sh) & (nb - 1)], 1u);
    }
    __syncthreads();
    find_bucket_block(sm.hist, nb, need, true, sm.warp_sums, &sm.bucket, &sm.above);
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
  griddep_launch_dependents();
  griddep_wait();
  const int r = blockIdx.x / P.n_seg, sg = blockIdx.x % P.n_seg;
  const int b = r / P.n_q, i = r % P.n_q;
  const int64_t p = (int64_t)P.seq.len[b] - P.n_q + i;
  const int64_t nc = max((int64_t)0, p - P.window + 1);
  if (nc <= P.topk) return;
  for (int t = threadIdx.x; t < kHistBins; t += kThreadsTk) hist[t] = 0;
  __syncthreads();
  const float *s = P.scores + (size_t)r * P.score_stride;
  const int64_t s0 = (int64_t)sg * P.seg_len, s1 = min(nc, s0 + P.seg_len);
  for (int64_t base = s0; base < s1; base += kThreadsTk * kUnroll) {
    uint32_t k[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t t = base + u * kThreadsTk + threadIdx.x;
      k[u] = t < s1 ? load_key(s, t) : 0xffffffffu;
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u)
      if (base + u * kThreadsTk + threadIdx.x < s1) atomicAdd(&hist[k[u] >> 21], 1u);
  }
  __syncthreads();
  uint32_t *gh = P.hist_ws + (size_t)r * kHistBins;
  for (int t = threadIdx.x; t < kHistBins; t += kThreadsTk)
    if (hist[t]) atomicAdd(&gh[t], hist[t]);
}

// kRegs: a segment of a split row is held in registers (decode rows, a few long rows); the
// variant without it (one CTA per row, many rows) keeps two CTAs resident per SM.
template <bool kRegs>
__global__ void __launch_bounds__(kThreadsTk, kRegs ? 1 : 2) topk_select_kernel(const __grid_constant__ TopkParams P) {
  extern __shared__ __align__(16) uint8_t tk_raw[];
  TkSmem &sm = *reinterpret_cast<TkSmem *>(tk_raw);
  griddep_launch_dependents();
  griddep_wait();
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
  const int64_t s0 = (int64_t)sg * P.seg_len, s1 = min(nc, s0 + P.seg_len);
  // a short segment (the usual split case) is read into registers together with the histogram
  constexpr int kRegKeys = 32;
  const bool in_regs = kRegs && gh && P.seg_len <= kRegKeys * kThreadsTk;
  uint32_t rk[kRegKeys];
  // largest key this thread reads: the bit patterns order like the values only for scores that
  // are not negative and not NaN (keys <= 0x7f800000, +inf); anything else is reported
  uint32_t kmax = 0;
  if (in_regs) {
#pragma unroll
    for (int u = 0; u < kRegKeys; ++u) {
      const int64_t t = s0 + u * kThreadsTk + threadIdx.x;
      rk[u] = t < s1 ? load_key(s, t) : 0u;
      kmax = max(kmax, rk[u]);
    }
  }
  if (gh) {
    uint32_t hv[kHistBins / kThreadsTk];   // all loads in flight before the first store
#pragma unroll
    for (int e = 0; e < kHistBins / kThreadsTk; ++e) hv[e] = __ldcg(gh + e * kThreadsTk + threadIdx.x);
#pragma unroll
    for (int e = 0; e < kHistBins / kThreadsTk; ++e) sm.hist[e * kThreadsTk + threadIdx.x] = hv[e];
  } else {   // single segment: build it here
    for (int t = threadIdx.x; t < kHistBins; t += kThreadsTk) sm.hist[t] = 0;
    __syncthreads();
    for (int64_t base = 0; base < nc; base += kThreadsTk * kUnroll) {
      uint32_t k[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int64_t t = base + u * kThreadsTk + threadIdx.x;
        k[u] = t < nc ? load_key(s, t) : 0u;
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u)
        if (base + u * kThreadsTk + threadIdx.x < nc) atomicAdd(&sm.hist[k[u] >> 21], 1u);
    }
  }
  __syncthreads();
  // 2. bucket of the topk-th largest key
  find_bucket_block(sm.hist, kHistBins, (uint32_t)P.topk, true, sm.warp_sums, &sm.bucket, &sm.above);
  const int B1 = sm.bucket;
  const uint32_t above = sm.above;
  // 3. compact, in position order, every candidate of this segment with top digit >= B1 (the
  // count keeps counting past the shared-memory capacity, which selects the exact fallback)
  int32_t *gcount = P.cand_count + r;
  uint32_t *gkey = P.cand_key + (size_t)r * P.cand_cap;
  int32_t *gidx = P.cand_idx + (size_t)r * P.cand_cap;
  int n_local = 0;
  if (in_regs) {
    uint32_t take = 0;
#pragma unroll
    for (int u = 0; u < kRegKeys; ++u) {
      const int64_t t = s0 + u * kThreadsTk + threadIdx.x;
      if (t < s1 && (int)(rk[u] >> 21) >= B1) take |= 1u << u;
    }
    ordered_append<kRegKeys>(take, sm, n_local, [&](int slot, int u) {
      if (slot < kCandCap) {
        sm.key[slot] = rk[u];
        sm.idx[slot] = (int32_t)(s0 + u * kThreadsTk + threadIdx.x);
      }
    });
  }
  if (!in_regs) {
    // Each warp walks its own contiguous range of the segment 32 positions at a time and
    // appends its candidates in order to its own share of the buffer (no CTA-wide barrier per
    // step); the shares are then closed up in warp order, which is position order.
    constexpr int kWarpCap = kCandCap / kWarpsTk;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t span = ((s1 - s0 + kWarpsTk * 32 - 1) / (kWarpsTk * 32)) * 32;
    const int64_t w0 = s0 + warp * span, w1 = min(s1, w0 + span);
    uint32_t *wkey = sm.key + warp * kWarpCap;
    int32_t *widx = sm.idx + warp * kWarpCap;
    int wcount = 0;
    const unsigned below = (1u << lane) - 1u;
    for (int64_t base = w0; base < w1; base += 32 * kUnroll) {
      uint32_t k[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int64_t t = base + u * 32 + lane;
        k[u] = t < w1 ? load_key(s, t) : 0u;
        kmax = max(kmax, k[u]);
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int64_t t = base + u * 32 + lane;
        const bool take = t < w1 && (int)(k[u] >> 21) >= B1;
        const unsigned m = __ballot_sync(0xffffffffu, take);
        if (take) {
          const int slot = wcount + __popc(m & below);
          if (slot < kWarpCap) {
            wkey[slot] = k[u];
            widx[slot] = (int32_t)t;
          }
        }
        wcount += __popc(m);
      }
    }
    if (lane == 0) sm.scan[warp] = wcount;
    __syncthreads();
    int pre = 0, tot = 0, over = 0;
    for (int w = 0; w < kWarpsTk; ++w) {
      const int c = sm.scan[w];
      if (w < warp) pre += c;
      tot += c;
      over |= c > kWarpCap;
    }
    __syncthreads();
    if (over) {
      n_local = kCandCap + 1;   // a share overflowed: the exact fallback reads the row again
    } else {
      // close up the shares in warp order: every share is read into registers before any is
      // written at its place
      constexpr int kPerLane = kWarpCap / 32;
      uint32_t kk[kPerLane];
      int32_t ii[kPerLane];
#pragma unroll
      for (int q = 0; q < kPerLane; ++q) {
        const int j = q * 32 + lane;
        kk[q] = j < wcount ? wkey[j] : 0u;
        ii[q] = j < wcount ? widx[j] : 0;
      }
      __syncthreads();
#pragma unroll
      for (int q = 0; q < kPerLane; ++q) {
        const int j = q * 32 + lane;
        if (j < wcount) {
          sm.key[pre + j] = kk[q];
          sm.idx[pre + j] = ii[q];
        }
      }
      n_local += tot;
    }
    __syncthreads();
  }
  if (kmax > 0x7f800000u) record_status(P.status, kStatusCheck);
  int n;
  if (P.n_seg == 1) {
    n = n_local;
  } else if (P.cluster) {
    // the row's segments form one thread-block cluster: every segment reads the counts of the
    // segments before it and stores its run at that offset into segment 0's shared memory
    // (remote stores, nothing waits on them), then segment 0 finishes with the runs in segment
    // order (its own is already in place)
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    if (threadIdx.x == 0) sm.last = n_local;          // this segment's count
    cluster.sync();
    const int ns = P.n_seg;
    int cnt = (threadIdx.x < 32 && (int)threadIdx.x < ns) ? *cluster.map_shared_rank(&sm.last, (int)threadIdx.x) : 0;
    int pre = (threadIdx.x < 32 && (int)threadIdx.x < sg) ? cnt : 0;
    if (threadIdx.x < 32) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
        pre += __shfl_xor_sync(0xffffffffu, pre, o);
      }
      if (threadIdx.x == 0) {
        sm.seg_pre[0] = pre;   // this segment's offset in segment 0's buffer
        sm.seg_pre[1] = cnt;   // the row's candidates
      }
    }
    __syncthreads();
    pre = sm.seg_pre[0];
    n = sm.seg_pre[1];
    if (sg != 0 && n <= kCandCap) {
      uint32_t *rkey = cluster.map_shared_rank(sm.key, 0);
      int32_t *ridx = cluster.map_shared_rank(sm.idx, 0);
      for (int j = threadIdx.x; j < n_local; j += kThreadsTk) {
        rkey[pre + j] = sm.key[j];
        ridx[pre + j] = sm.idx[j];
      }
    }
    cluster.sync();   // the runs are in segment 0's shared memory (release / acquire)
    if (sg != 0) return;
  } else {
    // publish this segment's candidates with one global reservation and record where they
    // went, so that the finishing CTA can lay the segments out in position order
    if (threadIdx.x == 0) sm.bucket = atomicAdd(gcount, n_local);
    __syncthreads();
    const int base = sm.bucket;
    const int ncopy = min(n_local, kCandCap);
    for (int t = threadIdx.x; t < ncopy; t += kThreadsTk) {
      if (base + t < P.cand_cap) {
        gkey[base + t] = sm.key[t];
        gidx[base + t] = sm.idx[t];
      }
    }
    if (threadIdx.x == 0) P.seg_info[(size_t)r * P.n_seg + sg] = make_int2(base, n_local);
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
    if (n <= kCandCap && n <= P.cand_cap) {
      const int ns = P.n_seg;
      int2 info = make_int2(0, 0);
      if (threadIdx.x < ns) info = __ldcg(&P.seg_info[(size_t)r * ns + threadIdx.x]);
      int tot;
      const int pre = block_excl_scan(info.y, sm.warp_sums, &tot);
      if (threadIdx.x < ns) {
        sm.seg_pre[threadIdx.x] = pre;
        sm.seg_src[threadIdx.x] = info.x;
      }
      __syncthreads();
      // every thread's loads in flight at once (up to kCandCap / kThreadsTk each), then stored
      // (the many-rows variant, held to 64 registers, keeps one load pair at a time)
      constexpr int kPer = kRegs ? kCandCap / kThreadsTk : 1;
      uint32_t kk[kPer];
      int32_t ii[kPer];
      for (int j0 = 0; j0 < n; j0 += kPer * kThreadsTk) {
#pragma unroll
        for (int q = 0; q < kPer; ++q) {
          const int j = j0 + q * kThreadsTk + threadIdx.x;
          if (j < n) {
            int lo = 0, hi = ns - 1;   // the last segment starting at or before j
            while (lo < hi) {
              const int mid = (lo + hi + 1) >> 1;
              if (sm.seg_pre[mid] <= j) lo = mid;
              else hi = mid - 1;
            }
            const int src = sm.seg_src[lo] + (j - sm.seg_pre[lo]);
            kk[q] = __ldcg(gkey + src);
            ii[q] = __ldcg(gidx + src);
          }
        }
#pragma unroll
        for (int q = 0; q < kPer; ++q) {
          const int j = j0 + q * kThreadsTk + threadIdx.x;
          if (j < n) {
            sm.key[j] = kk[q];
            sm.idx[j] = ii[q];
          }
        }
      }
    }
    __syncthreads();
    if (threadIdx.x == 0) {   // ready for the next call
      P.arrive[r] = 0;
      *gcount = 0;
    }
  }
  // 4. finish
  const bool fits = (P.n_seg == 1 || P.cluster) ? (n <= kCandCap) : (n <= kCandCap && n <= P.cand_cap);
  if (fits) finish_from_smem(sm, n, B1, above, P.topk, out);
  else finish_from_global(sm, s, nc, B1, above, P.topk, out);
  // 5. the forced window
  for (int64_t t = nc + threadIdx.x; t <= p; t += kThreadsTk) out[P.topk + (t - nc)] = (int32_t)t;
  if (threadIdx.x == 0) P.count[r] = (int32_t)(P.topk + (p - nc + 1));
}

size_t topk_smem_bytes() { return sizeof(TkSmem); }

cudaError_t launch_topk(const TopkParams &p, int n_rows, cudaStream_t s) {
  const size_t smem = sizeof(TkSmem);
  const bool regs = p.n_seg > 1;
  cudaError_t e = regs ? cudaFuncSetAttribute(topk_select_kernel<true>,
                                              cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)
                       : cudaFuncSetAttribute(topk_select_kernel<false>,
                                              cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int grid = n_rows * p.n_seg;
  if (!p.hist && p.n_seg > 1) {
    e = launch_pdl(topk_hist_kernel, grid, kThreadsTk, 0, s, p);
    if (e != cudaSuccess) return e;
  }
  if (p.cluster)
    e = launch_pdl_cluster(topk_select_kernel<true>, grid, kThreadsTk, smem, p.n_seg, s, p);
  else
    e = regs ? launch_pdl(topk_select_kernel<true>, grid, kThreadsTk, smem, s, p)
             : launch_pdl(topk_select_kernel<false>, grid, kThreadsTk, smem, s, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace hs2
