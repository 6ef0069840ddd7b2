// attn_decode_tc.cu -- importance scores (score pass 2) of the full-attention layer at decode
// time (one query token per sequence) on the fifth-generation tensor cores.
//
// "HySparse2: How Xiaomi Split the Transformer to Fix Agent Prefill Costs", section "KV Reuse
// and Token-Level Sparse Selection": the full layer produces the selection indices the sparse
// layers reuse. The score of cached token t is the head-summed softmax probability
// s[t] = sum_h exp(c q_h . k_t - lse_h), lse_h from the output pass. With MQA ("HySparse2:
// Hybrid Sparse Attention with Two-Level KV Sharing", "Inference cost") every 128-row K tile
// meets all H query heads in one tensor-core product, D = K_tile . Q^T (M = 128 tokens,
// N = H heads, or 2H query terms for e4m3 below), so one thread of the epilogue owns one
// token and sums its H exponentials without any exchange between threads.
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
//    range (error at most 2^-10 each). The hi terms are the operand's rows [0, H) and the lo
//    terms its rows [H, 2H), so one product of N = 2H reads each K tile once and the epilogue
//    adds a head's two columns. The logit is (D_h + D_{H+h}) k_scale[t] c 2^e_h.
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
constexpr int kDtAcc = 4;                       // accumulators in TMEM
constexpr int kDtQSlot = 32 * 256;              // a sequence's query operand (2H <= 64 rows)

// The product's N (bf16: the H heads; e4m3: H hi rows, then H lo rows) and the TMEM columns
// one accumulator takes (at least 32, so that every allocation is a power of two).
template <int KV, int H>
struct DtCols {
  static constexpr int kN = (KV == kKvFp8) ? 2 * H : H;
  static constexpr uint32_t kAcc = kN < 32 ? 32 : kN;
  static constexpr uint32_t kAll = kAcc * kDtAcc;
};

template <int KV>
struct DtCfg {
  static constexpr int kCodeBytes = (KV == kKvBf16) ? kDt * 256 : kDt * 128;
  static constexpr int kScaleBytes = (KV == kKvFp8) ? kDt * 4 : 0;
  static constexpr int kStageBytes = (kCodeBytes + kScaleBytes + 1023) / 1024 * 1024;
  static constexpr int kStages = (KV == kKvBf16) ? 5 : 8;
  static constexpr uint32_t kTx = kCodeBytes + kScaleBytes;
  // full: the TMA transaction (codes, and for e4m3 the scales); empty: the products (+ the
  // scale reads of the four epilogue warps of the tile's group)
  static constexpr uint32_t kFullCount = 1;
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
// head. bf16: two [32][128 B] halves (dims 0..63, 64..127). e4m3: one [2H][128 B] block, hi in
// row h and lo in row H + h.
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
      // one lane works through its head's 128 dims alone: all loads in flight at once and the
      // loops unrolled, so that the chain is short
      uint4 qv[16];
#pragma unroll
      for (int c = 0; c < 16; ++c) qv[c] = q[c];
      float amax = 0.f;
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const uint32_t w[4] = {qv[c].x, qv[c].y, qv[c].z, qv[c].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[e]));
          amax = fmax3(amax, fabsf(f.x), fabsf(f.y));
        }
      }
      const int ex = amax > 0.f ? ilogbf(amax) - 7 : 0;   // largest |q 2^-ex| in [128, 256)
      const float down = ldexpf(1.f, -ex);
#pragma unroll
      for (int c = 0; c < 16; ++c) {   // 8 dims: 8 hi codes, 8 lo codes
        const uint32_t w[4] = {qv[c].x, qv[c].y, qv[c].z, qv[c].w};
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
        *reinterpret_cast<uint2 *>(slot + sw128(h, c * 8)) = make_uint2(hc[0], hc[1]);
        *reinterpret_cast<uint2 *>(slot + sw128(H + h, c * 8)) = make_uint2(lc[0], lc[1]);
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
      uint4 qv[16];
#pragma unroll
      for (int c = 0; c < 16; ++c) qv[c] = q[c];
      float amax = 0.f;
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const uint32_t w[4] = {qv[c].x, qv[c].y, qv[c].z, qv[c].w};
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
  using N = DtCols<KV, H>;
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
    tmem_alloc(smem_u32(sm.tmem_base), N::kAll);
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
      const int y = (int)dt_row0(P, wk.b, g);
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
          tma_load_1d(smem_u32(st + C::kCodeBytes), &tm.ks, bar, y);
        }
      }
      ++issued;
    }
    // copies still in flight land before the CTA may exit
    for (int it = max(0, issued - C::kStages); it < issued; ++it)
      if (lane == 0) mbar_wait(smem_u32(&sm.full[it % C::kStages]), (it / C::kStages) & 1);
    __syncwarp();
  } else if (warp == kDtWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    // The queries are an input of the block (no kernel before this one in the block writes
    // them, and the block's first kernel starts only after everything before the block has
    // ended), so the first operand is laid out while the previous kernel finishes; the lse
    // the epilogue reads is that kernel's output.
    const uint32_t idesc = (KV == kKvBf16) ? umma_idesc_bf16(kDt, N::kN) : umma_idesc_e4m3(kDt, N::kN);
    int cur = -1, prepped = -1, last_seq_it = -1;
    if (wk.n > 0) {
      dt_prep_q<KV, H>(P, wk.b, sm.q);
      prepped = 0;
    }
    griddep_wait();
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
        const uint32_t d = tmem + a * N::kAcc;
        if (KV == kKvBf16) {
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint32_t off = (k >> 2) * (kDt * 128) + (k & 3) * 32;
            const uint32_t qoff = (k >> 2) * (32 * 128) + (k & 3) * 32;
            umma_bf16(d, umma_desc_sw128(st + off, 1024), umma_desc_sw128(qs + qoff, 1024), idesc, k > 0);
          }
        } else {
#pragma unroll
          for (int k = 0; k < 4; ++k)   // 32 dims a step; hi and lo terms in one product
            umma_e4m3(d, umma_desc_sw128(st + k * 32, 1024), umma_desc_sw128(qs + k * 32, 1024), idesc, k > 0);
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
      float v[32], w[32];   // e4m3: v the hi columns, w the lo columns (H = 32); or v both (H = 16)
      tmem_ld32(lane_addr + a * N::kAcc, v);
      if (KV == kKvFp8 && H == 32) tmem_ld32(lane_addr + a * N::kAcc + 32, w);
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
        float2 d = make_float2(v[2 * i], v[2 * i + 1]);
        if (KV == kKvFp8) {
          m = fmul2(m, make_float2(ks, ks));
          d = fadd2(d, H == 32 ? make_float2(w[2 * i], w[2 * i + 1])
                               : make_float2(v[(H + 2 * i) & 31], v[(H + 2 * i + 1) & 31]));
        }
        const float2 x = ffma2(d, m, make_float2(-l2_h[2 * i], -l2_h[2 * i + 1]));
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
    tmem_dealloc(tmem, N::kAll);
  }
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

cudaError_t launch_decode_score_tc(int kv_dtype, const TensorMaps &tm, const DecodeParams &p,
                                   cudaStream_t s) {
  if (kv_dtype != HS2_KV_FP8_E4M3) return cudaErrorInvalidValue;
  if (p.n_heads == 16) return launch_score_t<kKvFp8, 1>(tm, p, s);
  if (p.n_heads == 32) return launch_score_t<kKvFp8, 2>(tm, p, s);
  return cudaErrorInvalidValue;
}

}  // namespace hs2
