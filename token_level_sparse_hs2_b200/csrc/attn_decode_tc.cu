// attn_decode_tc.cu -- importance scores (score pass 2) of the full-attention layer at decode
// time (one query token per sequence) on the fifth-generation tensor cores.
//
// "HySparse2: How Xiaomi Split the Transformer to Fix Agent Prefill Costs", section "KV Reuse
// and Token-Level Sparse Selection": the full layer produces the selection indices the sparse
// layers reuse. The score of cached token t is the head-summed softmax probability
// s[t] = sum_h exp(c q_h . k_t - lse_h), lse_h from the output pass. With MQA ("HySparse2:
// Hybrid Sparse Attention with Two-Level KV Sharing", "Inference cost") every 128-row K tile
// meets all H query heads in one tensor-core product, D = K_tile . Q^T (M = 128 tokens,
// N = H heads), so one thread of the epilogue owns one token and sums its H exponentials
// without any exchange between threads.
//
// Cache formats:
//  * bf16: kind::f16 products over two 64-dim halves of the tile (8 steps of K = 16).
//  * e4m3 (value = k_scale[t] * code): kind::f8f6f4 products straight on the cached codes; no
//    widening. The query is split into two e4m3 terms per head, Q 2^-e_h = hi + lo, with e_h a
//    power of two that puts the head's largest |q| in [128, 256): hi is q rounded to e4m3 and
//    lo the remainder, which e4m3 holds exactly for every element of at least 2^-2 after the
//    scaling (a bf16 value has 8 significant bits, hi takes 4 and the remainder needs at most
//    4), so D = K.(hi + lo) equals K.Q 2^-e_h but for elements of magnitude below 2^-2
//    (2^-9 .. 2^-8 of the head's largest), whose remainder is rounded in e4m3's subnormal
//    range (error at most 2^-10 each). The logit is D k_scale[t] c 2^e_h.
//
// Persistent grid, one CTA per SM: CTA i walks an equal contiguous range of the concatenated
// 128-row tiles of all sequences, in reverse (pass 1 read those rows last; some are still in
// L2). Roles:
//   warp 9      producer: K tiles (and their scales) by TMA into a ring of stages;
//   warp 8      TMEM owner and MMA issuer (lane 0); its lanes also lay out each sequence's
//               query operand (one lane per head) in one of two shared-memory slots;
//   warps 0..7  epilogue in two groups of four taking alternate tiles, thread = token row:
//               s = sum_h exp2(D_h a_h - lse_h log2 e), the score store, and the top-digit count
//               of every candidate for the selection (shared-memory histograms for the range's
//               two lowest sequences, flushed once).
// Every wait is bounded; after a timeout the CTA records HS2_ERR_TIMEOUT, stops computing, waits
// for its own copies and products in flight and releases its tensor memory.
#include "attn_pipeline.cuh"
#include "internal.h"
#include "tc05.cuh"

namespace hs2 {

namespace {

constexpr int kDt = 128;                        // cache rows per tile (the MMA's M)
constexpr int kDtGroups = 2;                    // epilogue groups, alternate tiles
constexpr int kDtEpiWarps = 4 * kDtGroups;
constexpr int kDtWarpMma = kDtEpiWarps, kDtWarpTma = kDtEpiWarps + 1;
constexpr int kDtThreads = (kDtEpiWarps + 2) * 32;
constexpr int kDtAcc = 4;                       // accumulators of 32 columns
constexpr uint32_t kDtCols = 32 * kDtAcc;
constexpr int kDtQSlot = 32 * 256;              // a sequence's query operand (H <= 32 rows)

template <int KV>
struct DtCfg {
  static constexpr int kCodeBytes = (KV == kKvBf16) ? kDt * 256 : kDt * 128;
  static constexpr int kScaleBytes = (KV == kKvFp8) ? kDt * 4 : 0;
  static constexpr int kStageBytes = (kCodeBytes + kScaleBytes + 1023) / 1024 * 1024;
  static constexpr int kStages = (KV == kKvBf16) ? 5 : 8;
  static constexpr uint32_t kTx = kCodeBytes;
  // full: the TMA transaction (+ 32 lanes' scale copies); empty: the products (+ the scale
  // reads of the four epilogue warps of the tile's group)
  static constexpr uint32_t kFullCount = (KV == kKvFp8) ? 33 : 1;
  static constexpr uint32_t kEmptyCount = (KV == kKvFp8) ? 5 : 1;
  static constexpr size_t kBytes = 1024 + (size_t)kStages * kStageBytes + 2 * (size_t)kDtQSlot +
                                   2 * (size_t)kHistBins * 4 + kDtEpiWarps * 64 * 4 +
                                   (2 * kStages + 2 * kDtAcc + 2 + 1) * 8 + 16;
};

template <int KV>
struct DtSmem {
  using C = DtCfg<KV>;
  uint8_t *stages, *q;        // q: two slots of kDtQSlot bytes
  uint32_t *hist;             // [2][kHistBins]
  float *consts;              // [epilogue warp][64]: a_h, then lse_h log2 e
  uint64_t *full, *empty, *acc_full, *acc_empty, *qfree, *done;
  uint32_t *tmem_base;
  volatile int *abort_flag;
  __device__ explicit DtSmem(uint8_t *raw) {
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
    stages = base;
    q = stages + C::kStages * C::kStageBytes;
    hist = reinterpret_cast<uint32_t *>(q + 2 * kDtQSlot);
    consts = reinterpret_cast<float *>(hist + 2 * kHistBins);
    full = reinterpret_cast<uint64_t *>(consts + kDtEpiWarps * 64);
    empty = full + C::kStages;
    acc_full = empty + C::kStages;
    acc_empty = acc_full + kDtAcc;
    qfree = acc_empty + kDtAcc;
    done = qfree + 2;
    tmem_base = reinterpret_cast<uint32_t *>(done + 1);
    abort_flag = reinterpret_cast<volatile int *>(tmem_base + 1);
  }
};

__device__ __forceinline__ int dt_seq_of(const DecodeParams &P, int g) {
  int lo = 0, hi = P.batch - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (P.tile128_begin[mid] <= g) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// The CTA's 128-row tiles (CTA i of G owns [i T / G, (i + 1) T / G)), visited forward or in
// reverse; step() also tracks the sequence and its ordinal j among the sequences this CTA
// meets (0 for the first one visited).
struct DtWalk {
  int lo, hi, n, b, j;
  bool rev;
  __device__ DtWalk(const DecodeParams &P, bool reverse) {
    const int G = gridDim.x, T = P.total_tiles128;
    lo = (int)((int64_t)blockIdx.x * T / G);
    hi = (int)((int64_t)(blockIdx.x + 1) * T / G);
    n = hi - lo;
    rev = reverse;
    b = n > 0 ? dt_seq_of(P, rev ? hi - 1 : lo) : 0;
    j = 0;
  }
  __device__ __forceinline__ int step(const DecodeParams &P, int it) {
    const int g = rev ? hi - 1 - it : lo + it;
    if (rev) {
      while (g < P.tile128_begin[b]) {
        --b;
        ++j;
      }
    } else {
      while (g >= P.tile128_begin[b + 1]) {
        ++b;
        ++j;
      }
    }
    return g;
  }
  // the sequence the walk enters after sequence b, or -1
  __device__ __forceinline__ int next_seq(const DecodeParams &P) const {
    if (rev) return P.tile128_begin[b] > lo ? b - 1 : -1;
    return P.tile128_begin[b + 1] < hi ? b + 1 : -1;
  }
};

__device__ __forceinline__ int64_t dt_row0(const DecodeParams &P, int b, int g) {
  return (P.seq.start[b] / kDt + (g - P.tile128_begin[b])) * (int64_t)kDt;
}

__device__ __forceinline__ void dt_fail(const DecodeParams &P, volatile int *abort_flag) {
  record_status(P.status, kStatusTimeout);
  *abort_flag = 1;
}

// Bounded wait by lane 0 of the calling warp, shared with the warp; false after a timeout or
// once another warp has given up.
__device__ __forceinline__ bool dt_wait(const DecodeParams &P, volatile int *abort_flag,
                                        uint64_t *bar, uint32_t parity) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) {
    if (*abort_flag) {
      ok = false;
    } else if (!mbar_wait(smem_u32(bar), parity)) {
      dt_fail(P, abort_flag);
      ok = false;
    }
  }
  return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}

// kind::f8f6f4 instruction descriptor: fp32 accumulator, e4m3 A and B, both K-major.
__host__ __device__ constexpr uint32_t umma_idesc_e4m3(int m, int n) {
  return (1u << 4) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

__device__ __forceinline__ void umma_e4m3(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, bool accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n}\n"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"((uint32_t)accumulate));
}

// The query operand of sequence b in a slot, K-major with the 128-byte swizzle, one lane per
// head. bf16: two [32][128 B] halves (dims 0..63, 64..127). e4m3: hi [32][128 B], then lo.
template <int KV, int H>
__device__ void dt_prep_q(const DecodeParams &P, int b, uint8_t *slot) {
  const int h = threadIdx.x & 31;
  if (h < H) {
    const uint4 *q = reinterpret_cast<const uint4 *>(reinterpret_cast<const __nv_bfloat16 *>(P.q) +
                                                     ((size_t)b * H + h) * kHeadDim);
    if (KV == kKvBf16) {
#pragma unroll
      for (int c = 0; c < 16; ++c)
        *reinterpret_cast<uint4 *>(slot + (c >> 3) * (32 * 128) + sw128(h, (c & 7) * 16)) = q[c];
    } else {
      float amax = 0.f;
#pragma unroll 4
      for (int c = 0; c < 16; ++c) {
        const uint4 v = q[c];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[e]));
          amax = fmax3(amax, fabsf(f.x), fabsf(f.y));
        }
      }
      const int ex = amax > 0.f ? ilogbf(amax) - 7 : 0;   // largest |q 2^-ex| in [128, 256)
      const float down = ldexpf(1.f, -ex);
      uint8_t *hi_row = slot, *lo_row = slot + 32 * 128;
#pragma unroll 2
      for (int c = 0; c < 16; ++c) {   // 8 dims: 8 hi codes, 8 lo codes
        const uint4 v = q[c];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        uint32_t hc[2], lc[2];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[e]));
          f.x *= down;
          f.y *= down;
          const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(f, __NV_SATFINITE, __NV_E4M3);
          const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(hi, __NV_E4M3);
          const float2 hf = __half22float2(*reinterpret_cast<const __half2 *>(&hr));
          const __nv_fp8x2_storage_t lo =
              __nv_cvt_float2_to_fp8x2(make_float2(f.x - hf.x, f.y - hf.y), __NV_SATFINITE, __NV_E4M3);
          const int word = e >> 1, sh = (e & 1) * 16;
          if (sh == 0) {
            hc[word] = hi;
            lc[word] = lo;
          } else {
            hc[word] |= (uint32_t)hi << 16;
            lc[word] |= (uint32_t)lo << 16;
          }
        }
        *reinterpret_cast<uint2 *>(hi_row + sw128(h, c * 8)) = make_uint2(hc[0], hc[1]);
        *reinterpret_cast<uint2 *>(lo_row + sw128(h, c * 8)) = make_uint2(lc[0], lc[1]);
      }
    }
  }
  fence_proxy_async_smem();
  __syncwarp();
}

// This warp's per-sequence constants in cst[0..H) (a_h: the logit per unit of D, without the
// token's K scale) and cst[32..32+H) (lse_h log2 e), read back into registers by every lane.
template <int KV, int H, bool kLse = true>
__device__ void dt_seq_consts(const DecodeParams &P, int b, float *cst, float (&a)[H],
                              float (&l2)[H]) {
  const int h = threadIdx.x & 31;
  if (h < H) {
    float f = P.scale_log2;
    if (KV == kKvFp8) {   // the same power of two dt_prep_q takes out of the head
      const uint4 *q = reinterpret_cast<const uint4 *>(reinterpret_cast<const __nv_bfloat16 *>(P.q) +
                                                       ((size_t)b * H + h) * kHeadDim);
      float amax = 0.f;
#pragma unroll 4
      for (int c = 0; c < 16; ++c) {
        const uint4 v = q[c];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[e]));
          amax = fmax3(amax, fabsf(x.x), fabsf(x.y));
        }
      }
      f = ldexpf(P.scale_log2, amax > 0.f ? ilogbf(amax) - 7 : 0);
    }
    cst[h] = f;
    if (kLse) cst[32 + h] = P.lse[(size_t)b * H + h] * kLog2e;
  }
  __syncwarp();
#pragma unroll
  for (int i = 0; i < H; ++i) {
    a[i] = cst[i];
    l2[i] = kLse ? cst[32 + i] : 0.f;
  }
  __syncwarp();
}

template <int KV, int HG>
__global__ void __launch_bounds__(kDtThreads, 1)
    decode_score_tc_kernel(const __grid_constant__ TensorMaps tm, const __grid_constant__ DecodeParams P) {
  using C = DtCfg<KV>;
  constexpr int H = 16 * HG;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  DtSmem<KV> sm(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(smem_u32(&sm.full[s]), C::kFullCount);
      mbar_init(smem_u32(&sm.empty[s]), C::kEmptyCount);
    }
    for (int a = 0; a < kDtAcc; ++a) {
      mbar_init(smem_u32(&sm.acc_full[a]), 1);
      mbar_init(smem_u32(&sm.acc_empty[a]), 4);
    }
    mbar_init(smem_u32(&sm.qfree[0]), 1);
    mbar_init(smem_u32(&sm.qfree[1]), 1);
    mbar_init(smem_u32(&sm.done[0]), 1);
    *sm.abort_flag = 0;
    fence_barrier_init();
  }
  for (int t = threadIdx.x; t < 2 * kHistBins; t += kDtThreads) sm.hist[t] = 0;
  if (warp == kDtWarpMma) {
    tmem_alloc(smem_u32(sm.tmem_base), kDtCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  griddep_launch_dependents();
  const uint32_t tmem = *sm.tmem_base;
  DtWalk wk(P, true);
  const int b_lo = wk.n > 0 ? dt_seq_of(P, wk.lo) : 0;

  if (warp == kDtWarpTma) {
    // ------------------------------------------------------------ producer (K is not written
    // by any earlier kernel of the stream: it starts before they finish)
    int issued = 0;
    for (int it = 0; it < wk.n; ++it) {
      const int g = wk.step(P, it);
      const int s = it % C::kStages;
      if (it >= C::kStages && !dt_wait(P, sm.abort_flag, &sm.empty[s], ((it / C::kStages) & 1) ^ 1)) break;
      uint8_t *st = sm.stages + s * C::kStageBytes;
      const uint32_t bar = smem_u32(&sm.full[s]);
      const int64_t y64 = dt_row0(P, wk.b, g);
      const int y = (int)y64;
      if (lane == 0) {
        mbar_arrive_expect_tx(bar, C::kTx);
        if (KV == kKvBf16) {
#pragma unroll
          for (int half = 0; half < 2; ++half)
#pragma unroll
            for (int kb = 0; kb < 2; ++kb)
              tma_load_2d(smem_u32(st + kb * (kDt * 128) + half * (64 * 128)), &tm.k, bar, kb * 64,
                          y + half * 64);
        } else {
          tma_load_2d(smem_u32(st), &tm.k, bar, 0, y);
          tma_load_2d(smem_u32(st + 64 * 128), &tm.k, bar, 0, y + 64);
        }
      }
      if (KV == kKvFp8) {
        uint8_t *sc = st + C::kCodeBytes;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int rr = 4 * lane + u;
          const int64_t row = y64 + rr;
          const bool in = row < P.kv_rows;
          cp_async_4(smem_u32(sc + rr * 4), P.k_scale + (in ? row : 0), in ? 4u : 0u);
        }
        cp_async_mbar_arrive(bar);
      }
      ++issued;
    }
    // copies still in flight land before the CTA may exit
    for (int it = max(0, issued - C::kStages); it < issued; ++it)
      if (lane == 0) mbar_wait(smem_u32(&sm.full[it % C::kStages]), (it / C::kStages) & 1);
    __syncwarp();
  } else if (warp == kDtWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    griddep_wait();
    const uint32_t idesc = (KV == kKvBf16) ? umma_idesc_bf16(kDt, H) : umma_idesc_e4m3(kDt, H);
    int cur = -1, prepped = -1, last_seq_it = -1;
    if (wk.n > 0) {
      dt_prep_q<KV, H>(P, wk.b, sm.q);
      prepped = 0;
    }
    int b_next = -1;   // the sequence after the current one in the walk, if any
    for (int it = 0; it < wk.n; ++it) {
      const int g = wk.step(P, it);
      const int s = it % C::kStages, a = it % kDtAcc;
      if (wk.j != cur) {   // a new sequence: its slot was laid out earlier
        if (cur >= 0 && lane == 0) umma_commit(smem_u32(&sm.qfree[cur & 1]));   // cur's products
        cur = wk.j;
        last_seq_it = it;
        b_next = wk.next_seq(P);
      }
      if (!dt_wait(P, sm.abort_flag, &sm.full[s], (it / C::kStages) & 1)) break;
      if (it >= kDtAcc && !dt_wait(P, sm.abort_flag, &sm.acc_empty[a], ((it / kDtAcc) & 1) ^ 1)) break;
      tc_fence_after();
      if (lane == 0) {
        const uint32_t st = smem_u32(sm.stages + s * C::kStageBytes);
        const uint32_t qs = smem_u32(sm.q + (cur & 1) * kDtQSlot);
        const uint32_t d = tmem + a * 32;
        if (KV == kKvBf16) {
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint32_t off = (k >> 2) * (kDt * 128) + (k & 3) * 32;
            const uint32_t qoff = (k >> 2) * (32 * 128) + (k & 3) * 32;
            umma_bf16(d, umma_desc_sw128(st + off, 1024), umma_desc_sw128(qs + qoff, 1024), idesc, k > 0);
          }
        } else {
#pragma unroll
          for (int k = 0; k < 8; ++k) {   // hi terms, then lo terms
            const uint32_t off = (k & 3) * 32;
            const uint32_t qoff = (k >> 2) * (32 * 128) + (k & 3) * 32;
            umma_e4m3(d, umma_desc_sw128(st + off, 1024), umma_desc_sw128(qs + qoff, 1024), idesc, k > 0);
          }
        }
        umma_commit(smem_u32(&sm.empty[s]));
        umma_commit(smem_u32(&sm.acc_full[a]));
      }
      __syncwarp();
      // after the first tile of a sequence, lay out the next sequence's query in the other slot
      // once the products that read it last (two sequences back) have completed
      if (it == last_seq_it && b_next >= 0 && prepped < cur + 1) {
        if (cur >= 1 && !dt_wait(P, sm.abort_flag, &sm.qfree[(cur + 1) & 1], ((cur - 1) >> 1) & 1)) break;
        dt_prep_q<KV, H>(P, b_next, sm.q + ((cur + 1) & 1) * kDtQSlot);
        prepped = cur + 1;
      }
    }
    // every issued product has completed before the accumulators are released
    if (lane == 0) {
      umma_commit(smem_u32(&sm.done[0]));
      if (!mbar_wait(smem_u32(&sm.done[0]), 0)) dt_fail(P, sm.abort_flag);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3, grp = warp >> 2;
    const int tok = quarter * 32 + lane;   // TMEM lane = token row of the tile
    const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
    float *cst = sm.consts + warp * 64;
    float a_h[H], l2_h[H];
    int cur = -1;
    int64_t n_cand = 0, row0 = 0, row1 = 0;
    float *srow = nullptr;
    uint32_t *hrow = nullptr;
    griddep_wait();
    for (int it = 0; it < wk.n; ++it) {
      const int g = wk.step(P, it);
      if ((it & 1) != grp) continue;
      const int b = wk.b;
      if (b != cur) {
        cur = b;
        dt_seq_consts<KV, H>(P, b, cst, a_h, l2_h);
        row0 = P.seq.start[b];
        row1 = row0 + P.seq.len[b];
        n_cand = (int64_t)P.seq.len[b] - P.window;   // candidates: positions [0, p - window + 1)
        srow = P.scores + (size_t)b * P.score_stride;
        hrow = (b - b_lo < 2) ? sm.hist + (b - b_lo) * kHistBins
                              : (P.hist ? P.hist + (size_t)b * kHistBins : nullptr);
      }
      const int s = it % C::kStages, a = it % kDtAcc;
      if (!dt_wait(P, sm.abort_flag, &sm.acc_full[a], (it / kDtAcc) & 1)) break;
      tc_fence_after();
      float v[32];
      tmem_ld32(lane_addr + a * 32, v);
      float ks = 1.f;
      if (KV == kKvFp8)
        ks = reinterpret_cast<const float *>(sm.stages + s * C::kStageBytes + C::kCodeBytes)[tok];
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(smem_u32(&sm.acc_empty[a]));
        if (KV == kKvFp8) mbar_arrive(smem_u32(&sm.empty[s]));
      }
      // s = sum_h exp2(D_h a_h ks - lse_h log2 e), pairs of heads at a time
      float2 acc = make_float2(0.f, 0.f);
#pragma unroll
      for (int i = 0; i < H / 2; ++i) {
        float2 m = make_float2(a_h[2 * i], a_h[2 * i + 1]);
        if (KV == kKvFp8) m = fmul2(m, make_float2(ks, ks));
        const float2 x = ffma2(make_float2(v[2 * i], v[2 * i + 1]), m,
                               make_float2(-l2_h[2 * i], -l2_h[2 * i + 1]));
        acc = fadd2(acc, make_float2(fast_exp2(x.x), fast_exp2(x.y)));
      }
      const float sc = acc.x + acc.y;
      const int64_t row = dt_row0(P, b, g) + tok;
      if (row >= row0 && row < row1) {
        const int64_t pos = row - row0;
        srow[pos] = sc;
        if (hrow && pos < n_cand) atomicAdd(&hrow[__float_as_uint(sc) >> 21], 1u);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (P.hist && wk.n > 0 && !*sm.abort_flag) {
    const int b_hi = dt_seq_of(P, wk.hi - 1);
    for (int t = threadIdx.x; t < 2 * kHistBins; t += kDtThreads) {
      const int k = t / kHistBins;
      const uint32_t v = sm.hist[t];
      if (v && b_lo + k <= b_hi) atomicAdd(&P.hist[(size_t)(b_lo + k) * kHistBins + (t % kHistBins)], v);
    }
  }
  if (warp == kDtWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, kDtCols);
  }
}

// ============================================================================ pass 1, e4m3 cache
//
// Output pass of the full layer for an e4m3 cache (value = scale * code), per 128-row tile i:
//   S_i^T = K_i . (hi + lo)^T  kind::f8f6f4 on the cached codes (M = 128 tokens, N = H), into one
//                              of two TMEM buffers;
//   softmax (warps 0..3)       thread = token t: x_h = S_h k_scale[t] c 2^e_h (log2 units), the
//                              lazy reference max (moves only when some x_h exceeds it by more
//                              than 8: one barrier-reduced vote per tile, a transposing warp
//                              reduction and a TMEM rescale of O only then), p_h = 2^(x_h - m_h),
//                              the thread's share of each head's denominator, and
//                              P'_h = p_h v_scale[t] 2^100 as two bf16 terms (hi, and the
//                              remainder lo) into a [128 tokens][64 columns] tile: hi in columns
//                              [0, H), lo in [32, 32 + H), the rest zero;
//   converters (warps 4..7)    thread = token t: the V codes widened exactly to bf16 values
//                              times 2^-112 (one conversion and two logic operations per pair)
//                              into a [128 tokens][128 dims] tile, the 128-byte swizzled layout
//                              the tensor cores read as an MN-major operand; rows outside the
//                              sequence are written as zeros;
//   O^T += V_w^T . P'_i        kind::f16 (M = 128 dims, N = 64, K = 128 tokens) into TMEM; the
//                              output of head h is column h plus column 32 + h, times 2^12.
// The MMA warp issues S_{i+1} before O += P_i (the tensor cores work on the next scores while
// the softmax warps run). At every sequence boundary of the CTA's range the softmax warps write
// the CTA's partial (max, denominator, unnormalised output) in the layout the merge reads.
constexpr int kP1Stages = 4;
constexpr int kP1CodeBytes = kDt * 128;                      // K (or V) codes of a tile
constexpr int kP1StageBytes = 2 * kP1CodeBytes + 2 * kDt * 4; // K, V codes, then their scales
constexpr int kP1VwBytes = kDt * 256;                        // widened V: two [128][128 B] halves
constexpr int kP1PBytes = kDt * 128;                         // P': [128 tokens][64 heads] bf16
constexpr int kP1SoftWarps = 4, kP1ConvWarps = 4;
constexpr int kP1WarpMma = 8, kP1WarpTma = 9;
constexpr int kP1Threads = 10 * 32;
constexpr uint32_t kP1ColO = 64;                             // S buffers at 0 and 32
constexpr uint32_t kP1Cols = 128;
constexpr float kP1Lazy = 8.f;
// V is widened to bf16 times 2^-112 (e4m3x2_to_bf16x2_scaled) and P' carries 2^100, so the
// accumulator holds O 2^-12; the flush multiplies by 2^12.
constexpr float kP1PScale = 0x1p100f;
constexpr float kP1OScale = 0x1p12f;

// Two e4m3 codes (low byte first) to a bf16 pair holding their values times 2^-112, exactly:
// e4m3 -> f16 is exact and every e4m3 value is a normal f16 (or zero); the f16's magnitude
// bits shifted right by three form a bf16 whose 8-bit exponent field is the f16's 5-bit one,
// 112 below the value's own bf16 exponent (biases 127 and 15), with all three mantissa bits
// kept. One conversion and two logic operations per pair.
__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2_scaled(uint32_t two) {
  const uint32_t h = e4m3x2_to_f16x2(two);
  return ((h >> 3) & 0x0fff0fffu) | (h & 0x80008000u);
}

struct P1Smem {
  uint8_t *stages, *vw, *pp, *q;
  float *red;                 // [kP1SoftWarps][32] per-warp partials of head maxima / sums
  float *cst;                 // [kP1SoftWarps][96] per-warp scratch: factors, maxima, rescales
  uint64_t *full, *empty, *s_full, *s_free, *p_full, *p_free, *vw_full, *qfree, *done;
  uint32_t *tmem_base;
  volatile int *abort_flag;
  static constexpr size_t kBytes = 1024 + (size_t)kP1Stages * kP1StageBytes + kP1VwBytes +
                                   2 * (size_t)kP1PBytes + 2 * (size_t)kDtQSlot +
                                   kP1SoftWarps * 32 * 4 + kP1SoftWarps * 96 * 4 +
                                   (2 * kP1Stages + 12) * 8 + 16;
  __device__ explicit P1Smem(uint8_t *raw) {
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
    stages = base;
    vw = stages + kP1Stages * kP1StageBytes;
    pp = vw + kP1VwBytes;
    q = pp + 2 * kP1PBytes;
    red = reinterpret_cast<float *>(q + 2 * kDtQSlot);
    cst = red + kP1SoftWarps * 32;
    full = reinterpret_cast<uint64_t *>(cst + kP1SoftWarps * 96);
    empty = full + kP1Stages;
    s_full = empty + kP1Stages;
    s_free = s_full + 2;
    p_full = s_free + 2;
    p_free = p_full + 2;
    vw_full = p_free + 2;
    qfree = vw_full + 1;
    done = qfree + 2;
    tmem_base = reinterpret_cast<uint32_t *>(done + 1);
    abort_flag = reinterpret_cast<volatile int *>(tmem_base + 1);
  }
};

// all 128 softmax threads (named barrier 1): true if any of them passed true
__device__ __forceinline__ bool softmax_any(bool v) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 q, %1, 0;\n bar.red.or.pred p, 1, 128, q;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(r)
      : "r"((uint32_t)v)
      : "memory");
  return r != 0;
}

// Lane h of the warp ends with the maximum (kMax) or sum over the warp's lanes of v[h], h < H;
// v is overwritten. A transposing butterfly: at step s each lane keeps the half of its current
// head range selected by bit s of its lane index and combines it with its partner's.
template <int H, bool kMax>
__device__ __forceinline__ float warp_head_reduce(float (&v)[32]) {
  const int lane = threadIdx.x & 31;
  if (H == 16) {   // both half-warps end with all 16 heads
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float o = __shfl_xor_sync(0xffffffffu, v[i], 16);
      v[i] = kMax ? fmaxf(v[i], o) : v[i] + o;
    }
  }
#pragma unroll
  for (int s = H / 2; s >= 1; s >>= 1) {
    const bool up = (lane & s) != 0;
#pragma unroll
    for (int i = 0; i < s; ++i) {
      const float send = up ? v[i] : v[i + s];
      const float keep = up ? v[i + s] : v[i];
      const float o = __shfl_xor_sync(0xffffffffu, send, s);
      v[i] = kMax ? fmaxf(keep, o) : keep + o;
    }
  }
  return v[0];   // head lane % H
}

template <int HG>
__global__ void __launch_bounds__(kP1Threads, 1)
    decode_attn_fp8_tc_kernel(const __grid_constant__ TensorMaps tm, const __grid_constant__ DecodeParams P) {
  constexpr int H = 16 * HG;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  P1Smem sm(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kP1Stages; ++s) {
      mbar_init(smem_u32(&sm.full[s]), 33);                     // TMA + 32 scale-copy lanes
      mbar_init(smem_u32(&sm.empty[s]), 1 + kP1ConvWarps + kP1SoftWarps);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(&sm.s_full[a]), 1);
      mbar_init(smem_u32(&sm.s_free[a]), kP1SoftWarps);
      mbar_init(smem_u32(&sm.p_full[a]), kP1SoftWarps);
      mbar_init(smem_u32(&sm.p_free[a]), 1);
      mbar_init(smem_u32(&sm.qfree[a]), 1);
    }
    mbar_init(smem_u32(sm.vw_full), kP1ConvWarps);
    mbar_init(smem_u32(sm.done), 1);
    *sm.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp < kP1SoftWarps) {   // both P' tiles start zero: heads H..63 are never written
    for (int t = threadIdx.x; t < 2 * kP1PBytes / 16; t += kP1SoftWarps * 32)
      reinterpret_cast<uint4 *>(sm.pp)[t] = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
  }
  if (warp == kP1WarpMma) {
    tmem_alloc(smem_u32(sm.tmem_base), kP1Cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *sm.tmem_base;
  // the block's first kernel: the previous one may have appended cache rows; the next kernel
  // starts only after this wait (every later kernel of the block starts after it too)
  griddep_wait();
  griddep_launch_dependents();
  // the workspace's zero-initialised region (status word, histograms, selection counters): the
  // score pass and the selection read it only after this kernel has finished
  for (int t = blockIdx.x * kP1Threads + threadIdx.x; t < P.zero_n16; t += gridDim.x * kP1Threads)
    P.zero[t] = make_uint4(0, 0, 0, 0);
  DtWalk wk(P, false);

  if (warp == kP1WarpTma) {
    // ------------------------------------------------------------ producer
    int issued = 0;
    for (int it = 0; it < wk.n; ++it) {
      const int g = wk.step(P, it);
      const int s = it % kP1Stages;
      if (it >= kP1Stages && !dt_wait(P, sm.abort_flag, &sm.empty[s], ((it / kP1Stages) & 1) ^ 1)) break;
      uint8_t *st = sm.stages + s * kP1StageBytes;
      const uint32_t bar = smem_u32(&sm.full[s]);
      const int64_t y64 = dt_row0(P, wk.b, g);
      const int y = (int)y64;
      if (lane == 0) {
        mbar_arrive_expect_tx(bar, 2 * kP1CodeBytes);
        tma_load_2d(smem_u32(st), &tm.k, bar, 0, y);
        tma_load_2d(smem_u32(st + 64 * 128), &tm.k, bar, 0, y + 64);
        tma_load_2d(smem_u32(st + kP1CodeBytes), &tm.v, bar, 0, y);
        tma_load_2d(smem_u32(st + kP1CodeBytes + 64 * 128), &tm.v, bar, 0, y + 64);
      }
      uint8_t *sc = st + 2 * kP1CodeBytes;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int rr = 4 * lane + u;
        const int64_t row = y64 + rr;
        const bool in = row < P.kv_rows;
        cp_async_4(smem_u32(sc + rr * 4), P.k_scale + (in ? row : 0), in ? 4u : 0u);
        cp_async_4(smem_u32(sc + (kDt + rr) * 4), P.v_scale + (in ? row : 0), in ? 4u : 0u);
      }
      cp_async_mbar_arrive(bar);
      ++issued;
    }
    for (int it = max(0, issued - kP1Stages); it < issued; ++it)
      if (lane == 0) mbar_wait(smem_u32(&sm.full[it % kP1Stages]), (it / kP1Stages) & 1);
    __syncwarp();
  } else if (warp == kP1WarpMma) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t id_s = umma_idesc_e4m3(kDt, H);
    const uint32_t id_o = umma_idesc_bf16(kDt, 64) | (1u << 15) | (1u << 16);   // A, B MN-major
    int cur = -1, prepped = -1, first_it = -1, b_next = -1;
    bool prev_first = false;   // tile it - 1 was the first of its sequence
    if (wk.n > 0) {
      dt_prep_q<kKvFp8, H>(P, wk.b, sm.q);
      prepped = 0;
    }
    // O^T += V_w^T . P'_k for tile k (the first tile of a sequence starts the sum)
    auto pv = [&](int k, bool first) -> bool {
      if (!dt_wait(P, sm.abort_flag, &sm.p_full[k & 1], (k >> 1) & 1)) return false;
      if (!dt_wait(P, sm.abort_flag, sm.vw_full, k & 1)) return false;
      tc_fence_after();
      if (lane == 0) {
        const uint32_t vw = smem_u32(sm.vw), pp = smem_u32(sm.pp + (k & 1) * kP1PBytes);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_bf16(tmem + kP1ColO, umma_desc_sw128_mn(vw + kk * 2048, kDt * 128, 1024),
                    umma_desc_sw128_mn(pp + kk * 2048, kDt * 128, 1024), id_o, !first || kk > 0);
        umma_commit(smem_u32(&sm.p_free[k & 1]));
      }
      __syncwarp();
      return true;
    };
    bool ok = true;
    for (int it = 0; it < wk.n && ok; ++it) {
      wk.step(P, it);
      const int s = it % kP1Stages;
      bool first = false;
      if (wk.j != cur) {
        if (cur >= 0 && lane == 0) umma_commit(smem_u32(&sm.qfree[cur & 1]));
        cur = wk.j;
        first_it = it;
        first = true;
        b_next = wk.next_seq(P);
      }
      if (!dt_wait(P, sm.abort_flag, &sm.full[s], (it / kP1Stages) & 1)) break;
      if (it >= 2 && !dt_wait(P, sm.abort_flag, &sm.s_free[it & 1], ((it - 2) >> 1) & 1)) break;
      tc_fence_after();
      if (lane == 0) {
        const uint32_t st = smem_u32(sm.stages + s * kP1StageBytes);
        const uint32_t qs = smem_u32(sm.q + (cur & 1) * kDtQSlot);
#pragma unroll
        for (int k = 0; k < 8; ++k)   // hi terms, then lo terms
          umma_e4m3(tmem + (it & 1) * 32, umma_desc_sw128(st + (k & 3) * 32, 1024),
                    umma_desc_sw128(qs + (k >> 2) * (32 * 128) + (k & 3) * 32, 1024), id_s, k > 0);
        umma_commit(smem_u32(&sm.empty[s]));
        umma_commit(smem_u32(&sm.s_full[it & 1]));
      }
      __syncwarp();
      if (it >= 1 && !(ok = pv(it - 1, prev_first))) break;
      prev_first = first;
      if (it == first_it && b_next >= 0 && prepped < cur + 1) {
        if (cur >= 1 && !dt_wait(P, sm.abort_flag, &sm.qfree[(cur + 1) & 1], ((cur - 1) >> 1) & 1)) break;
        dt_prep_q<kKvFp8, H>(P, b_next, sm.q + ((cur + 1) & 1) * kDtQSlot);
        prepped = cur + 1;
      }
    }
    if (ok && wk.n > 0 && !*sm.abort_flag) pv(wk.n - 1, prev_first);
    if (lane == 0) {
      umma_commit(smem_u32(sm.done));
      if (!mbar_wait(smem_u32(sm.done), 0)) dt_fail(P, sm.abort_flag);
    }
    __syncwarp();
  } else if (warp >= kP1SoftWarps) {
    // ------------------------------------------------------------ converters: V -> bf16
    const int t = (warp - kP1SoftWarps) * 32 + lane;
    for (int it = 0; it < wk.n; ++it) {
      const int g = wk.step(P, it);
      const int s = it % kP1Stages;
      if (!dt_wait(P, sm.abort_flag, &sm.full[s], (it / kP1Stages) & 1)) break;
      if (it >= 1 && !dt_wait(P, sm.abort_flag, &sm.p_free[(it - 1) & 1], ((it - 1) >> 1) & 1)) break;
      const int64_t row = dt_row0(P, wk.b, g) + t;
      const bool valid = row >= P.seq.start[wk.b] && row < P.seq.start[wk.b] + P.seq.len[wk.b];
      const uint8_t *vc = sm.stages + s * kP1StageBytes + kP1CodeBytes;
#pragma unroll
      for (int c = 0; c < 8; ++c) {   // codes of dims 16c .. 16c + 15
        uint4 w = *reinterpret_cast<const uint4 *>(vc + sw128(t, c * 16));
        if (!valid) w = make_uint4(0, 0, 0, 0);
        const uint32_t in[4] = {w.x, w.y, w.z, w.w};
        uint32_t o[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          o[2 * e] = e4m3x2_to_bf16x2_scaled(in[e] & 0xffffu);
          o[2 * e + 1] = e4m3x2_to_bf16x2_scaled(in[e] >> 16);
        }
        uint8_t *half = sm.vw + (c >> 2) * (kDt * 128);
        const int k0 = 2 * (c & 3);
        *reinterpret_cast<uint4 *>(half + sw128(t, k0 * 16)) = make_uint4(o[0], o[1], o[2], o[3]);
        *reinterpret_cast<uint4 *>(half + sw128(t, (k0 + 1) * 16)) = make_uint4(o[4], o[5], o[6], o[7]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(smem_u32(sm.vw_full));
        mbar_arrive(smem_u32(&sm.empty[s]));
      }
    }
  } else {
    // ------------------------------------------------------------ softmax (thread = token)
    // Per-head values that every thread shares live in the warp's scratch (read as broadcasts):
    // cst[h] the logit factor c log2e 2^e_h of the sequence, cst[32 + h] the reference max m_h,
    // cst[64 + h] the last rescale factor (every warp computes the same values); the
    // denominator shares l[h] are per thread.
    const int t = warp * 32 + lane;
    const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
    float *cst = sm.cst + warp * 96;
    float l[H];
    int cur = -1, slot = 0;
    int64_t row0 = 0, row1 = 0;
    bool first_tile = true;
    // the CTA's partial of the current sequence, once its last product (tile it_end - 1) landed
    auto flush = [&](int it_end) -> bool {
      if (!dt_wait(P, sm.abort_flag, &sm.p_free[(it_end - 1) & 1], ((it_end - 1) >> 1) & 1)) return false;
      tc_fence_after();
      float o[32], o2[32];
      tmem_ld32(lane_addr + kP1ColO, o);
      tmem_ld32(lane_addr + kP1ColO + 32, o2);
      tmem_wait_ld();
      float *part = P.part + (size_t)slot * H * kPartRow;
#pragma unroll
      for (int h = 0; h < H; ++h)   // O[h][d = t]: the hi and lo columns
        part[h * kPartRow + kPartO + t] = (o[h] + o2[h]) * kP1OScale;
      float v[32];
#pragma unroll
      for (int h = 0; h < 32; ++h) v[h] = h < H ? l[h] : 0.f;
      const float ws = warp_head_reduce<H, false>(v);
      if (lane < H) sm.red[warp * 32 + lane] = ws;
      named_barrier_sync(2, kP1SoftWarps * 32);
      if (t < H) {
        float L = 0.f;
#pragma unroll
        for (int w = 0; w < kP1SoftWarps; ++w) L += sm.red[w * 32 + t];
        part[t * kPartRow + 0] = cst[32 + t];
        part[t * kPartRow + 1] = L;
      }
      named_barrier_sync(2, kP1SoftWarps * 32);   // sm.red is free again
      return true;
    };
    bool ok = true;
    for (int it = 0; it < wk.n; ++it) {
      const int g = wk.step(P, it);
      const int s = it % kP1Stages;
      const int b = wk.b;
      if (!dt_wait(P, sm.abort_flag, &sm.s_full[it & 1], (it >> 1) & 1)) { ok = false; break; }
      tc_fence_after();
      if (b != cur) {
        if (cur >= 0 && !(ok = flush(it))) break;
        cur = b;
        const int first_cta = (int)(((int64_t)(P.tile128_begin[b] + 1) * gridDim.x - 1) / P.total_tiles128);
        slot = P.seq.item_begin[b] + ((int)blockIdx.x - first_cta);
        float cq[H], unused[H];
        dt_seq_consts<kKvFp8, H, false>(P, b, cst, cq, unused);   // cst[h] = cq[h]
        if (lane < H) cst[32 + lane] = -INFINITY;
        __syncwarp();
#pragma unroll
        for (int h = 0; h < H; ++h) l[h] = 0.f;
        row0 = P.seq.start[b];
        row1 = row0 + P.seq.len[b];
        first_tile = true;
      }
      float x[32];
      tmem_ld32(lane_addr + (it & 1) * 32, x);
      const float *scl = reinterpret_cast<const float *>(sm.stages + s * kP1StageBytes + 2 * kP1CodeBytes);
      const float ks = scl[t], vs = scl[kDt + t];
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(smem_u32(&sm.s_free[it & 1]));
        mbar_arrive(smem_u32(&sm.empty[s]));
      }
      const int64_t row = dt_row0(P, b, g) + t;
      const bool valid = row >= row0 && row < row1;
      bool over = false;
#pragma unroll
      for (int h = 0; h < H; h += 4) {
        const float4 c4 = *reinterpret_cast<const float4 *>(cst + h);
        const float4 m4 = *reinterpret_cast<const float4 *>(cst + 32 + h);
        const float cc[4] = {c4.x, c4.y, c4.z, c4.w}, mm[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          x[h + e] = valid ? x[h + e] * (ks * cc[e]) : -INFINITY;
          over |= x[h + e] > mm[e] + kP1Lazy;
        }
      }
      if (softmax_any(over)) {
        // new reference maxima: the tile's head maxima over all 128 tokens (at most the old)
        float v[32];
#pragma unroll
        for (int h = 0; h < 32; ++h) v[h] = h < H ? x[h] : -INFINITY;
        const float wm = warp_head_reduce<H, true>(v);
        if (lane < H) sm.red[warp * 32 + lane] = wm;
        named_barrier_sync(2, kP1SoftWarps * 32);
#pragma unroll
        for (int h = 0; h < H; ++h) {
          const float mo = cst[32 + h];
          float mt = mo;
#pragma unroll
          for (int w = 0; w < kP1SoftWarps; ++w) mt = fmaxf(mt, sm.red[w * 32 + h]);
          const float alpha = (mo == -INFINITY) ? 0.f : fast_exp2(mo - mt);
          l[h] *= alpha;
          v[h] = mt;
          if (lane == 0) cst[64 + h] = alpha;
        }
        named_barrier_sync(2, kP1SoftWarps * 32);   // sm.red is free again
        __syncwarp();
        if (lane == 0) {   // every lane computed the same maxima
#pragma unroll
          for (int h = 0; h < H; ++h) cst[32 + h] = v[h];
        }
        __syncwarp();
        if (!first_tile) {   // O holds this sequence's earlier tiles: rescale it once they landed
          if (!dt_wait(P, sm.abort_flag, &sm.p_free[(it - 1) & 1], ((it - 1) >> 1) & 1)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int half = 0; half < 2; ++half) {   // hi columns, then lo columns
            float o[32];
            tmem_ld32(lane_addr + kP1ColO + 32 * half, o);
            tmem_wait_ld();
            uint32_t ou[32];
#pragma unroll
            for (int h = 0; h < 32; ++h) ou[h] = __float_as_uint(h < H ? o[h] * cst[64 + (h & (H - 1))] : 0.f);
            tmem_st32(lane_addr + kP1ColO + 32 * half, ou);
          }
          tmem_wait_st();
          tc_fence_before();
        }
      }
      // p = 2^(x - m), the denominator share, and P' = p v_scale 2^100 as two bf16 terms (hi
      // and the rounded remainder lo, 16 significant bits together): hi in heads [0, H) of the
      // tile, lo in heads [32, 32 + H); the product sums both halves into O's columns
      const float vsp = vs * kP1PScale;
      uint32_t phi[H / 2], plo[H / 2];
#pragma unroll
      for (int h = 0; h < H; h += 2) {
        const float2 m2 = *reinterpret_cast<const float2 *>(cst + 32 + h);
        const float p0 = fast_exp2(x[h] - m2.x), p1 = fast_exp2(x[h + 1] - m2.y);
        l[h] += p0;
        l[h + 1] += p1;
        const float a0 = p0 * vsp, a1 = p1 * vsp;
        const uint32_t hi = pack_bf16(a0, a1);
        phi[h / 2] = hi;
        plo[h / 2] = pack_bf16(a0 - __uint_as_float(hi << 16), a1 - __uint_as_float(hi & 0xffff0000u));
      }
      if (it >= 2 && !dt_wait(P, sm.abort_flag, &sm.p_free[it & 1], ((it - 2) >> 1) & 1)) { ok = false; break; }
      uint8_t *prow = sm.pp + (it & 1) * kP1PBytes;
#pragma unroll
      for (int c = 0; c < H / 8; ++c) {
        *reinterpret_cast<uint4 *>(prow + sw128(t, c * 16)) =
            make_uint4(phi[4 * c], phi[4 * c + 1], phi[4 * c + 2], phi[4 * c + 3]);
        *reinterpret_cast<uint4 *>(prow + sw128(t, 64 + c * 16)) =
            make_uint4(plo[4 * c], plo[4 * c + 1], plo[4 * c + 2], plo[4 * c + 3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&sm.p_full[it & 1]));
      first_tile = false;
    }
    if (ok && cur >= 0) flush(wk.n);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kP1WarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, kP1Cols);
  }
}

template <int HG>
cudaError_t launch_attn_fp8_t(const TensorMaps &tm, const DecodeParams &p, cudaStream_t s) {
  static_assert(P1Smem::kBytes <= 227 * 1024, "pass 1 shared memory");
  if (p.n_ctas < 1) return cudaSuccess;
  auto kern = decode_attn_fp8_tc_kernel<HG>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)P1Smem::kBytes);
  if (e != cudaSuccess) return e;
  e = launch_pdl(kern, p.n_ctas, kP1Threads, P1Smem::kBytes, s, tm, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int KV, int HG>
cudaError_t launch_score_t(const TensorMaps &tm, const DecodeParams &p, cudaStream_t s) {
  using C = DtCfg<KV>;
  static_assert(C::kBytes <= 227 * 1024, "score pass shared memory");
  if (p.n_ctas2 < 1) return cudaSuccess;
  auto kern = decode_score_tc_kernel<KV, HG>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::kBytes);
  if (e != cudaSuccess) return e;
  e = launch_pdl(kern, p.n_ctas2, kDtThreads, C::kBytes, s, tm, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_attn_fp8_tc(const TensorMaps &tm, const DecodeParams &p, cudaStream_t s) {
  if (p.n_heads == 16) return launch_attn_fp8_t<1>(tm, p, s);
  if (p.n_heads == 32) return launch_attn_fp8_t<2>(tm, p, s);
  return cudaErrorInvalidValue;
}

cudaError_t launch_decode_score_tc(int kv_dtype, const TensorMaps &tm, const DecodeParams &p,
                                   cudaStream_t s) {
  if (kv_dtype == HS2_KV_BF16) {
    if (p.n_heads == 16) return launch_score_t<kKvBf16, 1>(tm, p, s);
    if (p.n_heads == 32) return launch_score_t<kKvBf16, 2>(tm, p, s);
  } else {
    if (p.n_heads == 16) return launch_score_t<kKvFp8, 1>(tm, p, s);
    if (p.n_heads == 32) return launch_score_t<kKvFp8, 2>(tm, p, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace hs2
