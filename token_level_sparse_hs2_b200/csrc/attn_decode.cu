// attn_decode.cu -- the full-attention layer of a hybrid block at decode time (one query token
// per sequence): pass 1 (attention output + log-sum-exp) and pass 2 (importance scores).
//
// "HySparse2: How Xiaomi Split the Transformer to Fix Agent Prefill Costs", section "KV Reuse
// and Token-Level Sparse Selection": the full-attention layer attends over the whole context
// and produces the selection indices the sparse layers reuse. With MQA ("HySparse2: Hybrid
// Sparse Attention with Two-Level KV Sharing", "Inference cost") every K/V row serves all H
// query heads, so each 64-row tile is streamed from HBM once per pass and multiplied against
// all heads on the tensor cores.
//
// Work split (both passes): the 64-row tiles of all sequences (aligned to absolute row
// multiples of 64; rows of another sequence in a shared boundary tile are masked) are
// concatenated into one list, and a persistent grid of one CTA per SM takes equal contiguous
// ranges of it, crossing sequence boundaries. Warp `kConsumers` streams the range with TMA into
// a ring of stages; the consumer warps never stop between sequences. Pass 1: each consumer
// warp owns 16 heads x 16 rows of every tile and, when its sequence changes or the range
// ends, writes its partial softmax state (max, denominator, unnormalised output) to the
// workspace; merge_partials_kernel combines them into O and lse. Pass 2 walks its range in
// reverse, so it starts on the tiles pass 1 read last (still in L2), computes
// s[t] = sum_h exp2(x_h[t] - lse_h log2 e) and counts the top radix digit of every candidate.
#include "attn_pipeline.cuh"
#include "internal.h"

namespace hs2 {

namespace {

// Consumer warps come in groups that take turns on tiles (group i handles steps i, i + kGroups,
// ...); within a group, pass-1 warps split heads x rows, pass-2 warps split rows. Pass 1 runs
// 6 (bf16) or 8 (e4m3) consumer warps in one CTA per SM; pass 2 runs 4 in each of two CTAs
// per SM.
template <int KV, int HG, int PASS>
struct StreamCfg {
  // tile rows per pass-1 warp and pass-1 consumer warps: bf16 64 rows x 6 warps (registers
  // for a whole tile's scores); e4m3 32 rows x 8 warps (the widening wants more warps)
  static constexpr int kPass1Rows = (KV == kKvBf16) ? 64 : 32;
  static constexpr int kPass1Warps = (KV == kKvBf16) ? 6 : 4;
  static constexpr int kPass2Rows = 32;   // tile rows per pass-2 warp (all heads)
  // 64-row tiles per pipeline stage (kSub > 1: one CTA per SM moving kSub tiles a stage, with
  // 4 * kSub consumer warps; measured no faster than two CTAs per SM of single-tile stages)
#ifndef HS2_PASS2_SUB
#define HS2_PASS2_SUB 1
#endif
  static constexpr int kSub = (KV == kKvBf16 && PASS == 1) ? HS2_PASS2_SUB : 1;
  static constexpr int kPass2Warps = (kSub == 2) ? 8 : 4;
  static constexpr int kGroupWarps = (PASS == 0) ? (kTile / kPass1Rows) * HG : kSub * (kTile / kPass2Rows);
  static constexpr int kGroups = (PASS == 0) ? kPass1Warps / kGroupWarps : kPass2Warps / kGroupWarps;
  static constexpr int kConsumers = kGroupWarps * kGroups;
  static constexpr int kThreads = (kConsumers + 1) * 32;
  static constexpr int kKBytes = (KV == kKvBf16) ? 2 * kBoxBytes : kBoxBytes;
  static constexpr int kVBytes = (PASS == 0) ? kKBytes : 0;
  static constexpr int kScaleBytes = (KV == kKvFp8) ? (PASS == 0 ? 512 : 256) : 0;
  static constexpr int kTileBytes = kKBytes + kVBytes + kScaleBytes;   // one 64-row tile
  static constexpr int kStageBytes = (kSub * kTileBytes + 1023) / 1024 * 1024;
  static constexpr int kStages = (KV == kKvBf16) ? (PASS == 0 || kSub > 1 ? 6 : 4) : (PASS == 0 ? 4 : 6);
  // Stage s is refilled for steps s, s + kStages, ...; with kStages a multiple of kGroups all
  // of those steps belong to one group, so a group never waits on a stage whose previous fill
  // another group has not consumed yet (a parity wait cannot tell fill f from fill f + 2).
  static_assert(kStages % kGroups == 0, "stages must be a multiple of the consumer groups");
  static constexpr uint32_t kTxBytes = kKBytes + kVBytes;   // TMA bytes per 64-row tile
  static constexpr uint32_t kFullCount = (KV == kKvFp8) ? 33 : 1;
  // pass 1: the consumer warps' partials of a sequence merge in shared memory ([H][128] output
  // sums, then [8 warps][16 rows] max and denominator) before one partial per CTA is written
  static constexpr size_t kMergeBytes = (PASS == 0) ? (size_t)16 * HG * o_stride<KV>() * 4 + 8 * 16 * 2 * 4 : 0;
  static constexpr size_t kSmem = 1024 + (size_t)kStages * kStageBytes + 2 * kStages * 8 + 16 +
                                  (PASS == 1 ? 2 * (size_t)kHistBins * 4 : 0) + kMergeBytes;
};

__device__ __forceinline__ int seq_of_tile(const SeqTable &t, int batch, int g) {
  int lo = 0, hi = batch - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (t.tile_begin[mid] <= g) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// CTA i of G owns global tiles [i*T/G, (i+1)*T/G); cta_of_tile inverts that
__device__ __forceinline__ int range_lo(int i, int G, int T) { return (int)((int64_t)i * T / G); }
__device__ __forceinline__ int cta_of_tile(int g, int G, int T) {
  return (int)(((int64_t)(g + 1) * G - 1) / T);
}

// Walks a CTA's tiles (forward or reverse) and tracks the sequence of the current tile.
struct TileWalk {
  int lo, hi, n;
  bool reverse;
  int b;
  __device__ TileWalk(const DecodeParams &P, bool rev, bool per_seq = false) {
    if (per_seq) {   // the CTA's share of its own sequence's tiles
      int s0 = 0, s1 = P.batch - 1;
      while (s0 < s1) {
        const int mid = (s0 + s1 + 1) >> 1;
        if (P.cta_begin[mid] <= (int)blockIdx.x) s0 = mid; else s1 = mid - 1;
      }
      const int nc = P.cta_begin[s0 + 1] - P.cta_begin[s0], j = (int)blockIdx.x - P.cta_begin[s0];
      const int t0 = P.seq.tile_begin[s0], nt = P.seq.tile_begin[s0 + 1] - t0;
      lo = t0 + (int)((int64_t)j * nt / nc);
      hi = t0 + (int)((int64_t)(j + 1) * nt / nc);
    } else {
      const int G = gridDim.x, T = P.total_tiles;
      lo = range_lo(blockIdx.x, G, T);
      hi = range_lo(blockIdx.x + 1, G, T);
    }
    n = hi - lo;
    reverse = rev;
    b = (n > 0) ? seq_of_tile(P.seq, P.batch, reverse ? hi - 1 : lo) : 0;
  }
  // global tile of step it (steps are visited in order); updates b
  __device__ __forceinline__ int step(const DecodeParams &P, int it) {
    const int g = reverse ? hi - 1 - it : lo + it;
    if (reverse) {
      while (g < P.seq.tile_begin[b]) --b;
    } else {
      while (g >= P.seq.tile_begin[b + 1]) ++b;
    }
    return g;
  }
};

__device__ __forceinline__ int64_t tile_row0(const DecodeParams &P, int b, int g) {
  return (P.seq.start[b] / kTile + (g - P.seq.tile_begin[b])) * (int64_t)kTile;
}

template <int KV, int HG, int PASS>
__device__ void produce_stream(const TensorMaps &tm, const DecodeParams &P, uint8_t *stages,
                               uint64_t *full, uint64_t *empty, volatile int *abort_flag) {
  using C = StreamCfg<KV, HG, PASS>;
  const int lane = threadIdx.x & 31;
  TileWalk wk(P, PASS == 1, PASS == 0 && P.seq_split);
  // pass 1 is the block's first kernel: it waits for the previous kernel (which may have
  // appended rows to the cache) and only then lets the next kernel start, so every later kernel
  // of the block starts after that; pass 2 streams K without waiting
  if (PASS == 0) {
    griddep_wait();
    griddep_launch_dependents();
  }
  const int n_stages = (wk.n + C::kSub - 1) / C::kSub;
  for (int k = 0; k < n_stages; ++k) {
    const int s = k % C::kStages;
    const uint32_t par = ((k / C::kStages) & 1) ^ 1;
    if (k >= C::kStages) {
      bool ok = true;
      if (lane == 0) ok = mbar_wait(smem_u32(&empty[s]), par);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) {
        if (lane == 0) {
          record_status(P.status, kStatusTimeout);
          *abort_flag = 1;
        }
        return;
      }
    }
    if (*abort_flag) return;
    const uint32_t bar = smem_u32(&full[s]);
    const int nsub = min(C::kSub, wk.n - k * C::kSub);
    if (lane == 0) mbar_arrive_expect_tx(bar, nsub * C::kTxBytes);
    for (int u = 0; u < nsub; ++u) {
    const int g = wk.step(P, k * C::kSub + u);
    uint8_t *st = stages + s * C::kStageBytes + u * C::kTileBytes;
    const int64_t y64 = tile_row0(P, wk.b, g);
    const int y = (int)y64;
    if (lane == 0) {
      if (KV == kKvBf16) {
        tma_load_2d(smem_u32(st), &tm.k, bar, 0, y);
        tma_load_2d(smem_u32(st + kBoxBytes), &tm.k, bar, 64, y);
        if (PASS == 0) {
          tma_load_2d(smem_u32(st + C::kKBytes), &tm.v, bar, 0, y);
          tma_load_2d(smem_u32(st + C::kKBytes + kBoxBytes), &tm.v, bar, 64, y);
        }
      } else {
        tma_load_2d(smem_u32(st), &tm.k, bar, 0, y);
        if (PASS == 0) tma_load_2d(smem_u32(st + C::kKBytes), &tm.v, bar, 0, y);
      }
    }
    if (KV == kKvFp8) {
      uint8_t *sc = st + C::kKBytes + C::kVBytes;
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int rr = 2 * lane + u;
        const int64_t row = y64 + rr;
        const bool in = row < P.kv_rows;
        cp_async_4(smem_u32(sc + rr * 4), P.k_scale + (in ? row : 0), in ? 4u : 0u);
        if (PASS == 0)
          cp_async_4(smem_u32(sc + (kTile + rr) * 4), P.v_scale + (in ? row : 0), in ? 4u : 0u);
      }
      cp_async_mbar_arrive(bar);
    }
    }
  }
}

template <int KV, int HG, int PASS>
struct StreamSmem {
  using C = StreamCfg<KV, HG, PASS>;
  uint8_t *stages;
  uint64_t *full, *empty;
  volatile int *abort_flag;
  uint32_t *hist;
  float *merge_o, *merge_ml;
  __device__ explicit StreamSmem(uint8_t *raw) {
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
    stages = base;
    full = reinterpret_cast<uint64_t *>(stages + C::kStages * C::kStageBytes);
    empty = full + C::kStages;
    abort_flag = reinterpret_cast<volatile int *>(empty + C::kStages);
    hist = reinterpret_cast<uint32_t *>(empty + C::kStages + 2);
    merge_o = reinterpret_cast<float *>(empty + C::kStages + 2 + (PASS == 1 ? kHistBins : 0));
    merge_ml = merge_o + (PASS == 0 ? 16 * HG * o_stride<KV>() : 0);
  }
};

template <int KV>
__device__ __forceinline__ void load_q_rows(const __nv_bfloat16 *q, int row0, uint32_t (&qa)[8][4],
                                            float scale_log2, float (&rowf)[2]) {
  if (KV == kKvBf16) {
    load_q_frags_bf16_global(q, row0, qa);
    rowf[0] = rowf[1] = scale_log2;
  } else {
    float pw[2];
    load_q_frags_f16(q, row0, qa, pw);
    rowf[0] = scale_log2 * pw[0];
    rowf[1] = scale_log2 * pw[1];
  }
}

// ------------------------------------------------------------------ pass 1

// The CTA's partial for sequence b, written at slot = first slot of b + (CTA - first CTA of b).
// All consumer warps reach every flush together (they walk the same steps); they exchange their
// row maxima, add their outputs rescaled to the common maximum into shared memory in a fixed
// warp order (so results are bitwise reproducible), and the sum is written out once. Named
// barrier 1 spans the consumer warps only.
template <int KV, int HG>
__device__ void flush_partial(const DecodeParams &P, int b, int hg, const WarpSoftmax &st,
                              float *mo, float *mml) {
  using C = StreamCfg<KV, HG, 0>;
  constexpr int H = 16 * HG;
  constexpr int NT = C::kConsumers * 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
  float l[2] = {st.l[0], st.l[1]};
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    l[h] += __shfl_xor_sync(0xffffffffu, l[h], 1);
    l[h] += __shfl_xor_sync(0xffffffffu, l[h], 2);
  }
  if (c == 0) {
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      mml[(warp * 16 + g + 8 * hh) * 2 + 0] = st.m[hh];
      mml[(warp * 16 + g + 8 * hh) * 2 + 1] = l[hh];
    }
  }
  named_barrier_sync(1, NT);
  // common max of each of this warp's rows over the warps sharing its head group
  float f[2];
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    const int r = g + 8 * hh;
    float M = -INFINITY;
    for (int w = hg; w < C::kConsumers; w += HG) M = fmaxf(M, mml[(w * 16 + r) * 2]);
    f[hh] = (st.m[hh] == -INFINITY) ? 0.f : fast_exp2(st.m[hh] - M) * st.vref;
  }
  for (int k = 0; k < C::kConsumers / HG; ++k) {
    if (warp / HG == k) o_to_smem<KV>(mo + hg * 16 * o_stride<KV>(), st.o, f, k == 0);
    named_barrier_sync(1, NT);
  }
  const int first = P.seq_split ? P.cta_begin[b] : cta_of_tile(P.seq.tile_begin[b], gridDim.x, P.total_tiles);
  const int slot = P.seq.item_begin[b] + (blockIdx.x - first);
  float *part = P.part + (size_t)slot * H * kPartRow;
  for (int t = threadIdx.x; t < H * kHeadDim / 4; t += NT) {
    const int h = t / (kHeadDim / 4), d4 = t % (kHeadDim / 4);
    reinterpret_cast<float4 *>(part + h * kPartRow + kPartO)[d4] =
        reinterpret_cast<const float4 *>(mo + h * o_stride<KV>())[d4];
  }
  if (threadIdx.x < H) {
    const int h = threadIdx.x, hgh = h >> 4, r = h & 15;
    float M = -INFINITY, L = 0.f;
    for (int w = hgh; w < C::kConsumers; w += HG) M = fmaxf(M, mml[(w * 16 + r) * 2]);
    for (int w = hgh; w < C::kConsumers; w += HG) {
      const float m = mml[(w * 16 + r) * 2];
      if (m != -INFINITY) L += fast_exp2(m - M) * mml[(w * 16 + r) * 2 + 1];
    }
    part[h * kPartRow + 0] = M;
    part[h * kPartRow + 1] = L;
  }
  named_barrier_sync(1, NT);   // the buffers are clean before any warp's next flush
}

template <int KV, int HG>
__global__ void __launch_bounds__(StreamCfg<KV, HG, 0>::kThreads, (KV == kKvBf16) ? 1 : 2)
    decode_pass1_kernel(const __grid_constant__ TensorMaps tm, const __grid_constant__ DecodeParams P) {
  using C = StreamCfg<KV, HG, 0>;
  constexpr int H = 16 * HG;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  StreamSmem<KV, HG, 0> sm(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(smem_u32(&sm.full[s]), C::kFullCount);
      mbar_init(smem_u32(&sm.empty[s]), C::kGroupWarps);
    }
    *sm.abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (warp == C::kConsumers) {
    produce_stream<KV, HG, 0>(tm, P, sm.stages, sm.full, sm.empty, sm.abort_flag);
    return;
  }
  const int grp = warp / C::kGroupWarps, gw = warp % C::kGroupWarps;
  const int hg = gw % HG, tg = gw / HG;
  constexpr int NT = C::kPass1Rows / 8;
  const int tok0 = tg * C::kPass1Rows;
  const int c = lane & 3;
  TileWalk wk(P, false, P.seq_split != 0);
  int cur = -1;
  uint32_t qa[8][4];
  float rowf[2];
  WarpSoftmax st;
  st.init();
  griddep_wait();
  griddep_launch_dependents();
  // the workspace's zero-initialised region (status word, histograms, selection counters):
  // every earlier kernel of the stream has finished, and the score pass and the selection
  // read it only after this kernel has
  for (int t = blockIdx.x * (C::kConsumers * 32) + threadIdx.x; t < P.zero_n16;
       t += gridDim.x * (C::kConsumers * 32))
    P.zero[t] = make_uint4(0, 0, 0, 0);
  // every warp follows all steps of the CTA so that it flushes a partial for every sequence the
  // CTA touches, and computes only on its group's steps
  for (int it = 0; it < wk.n; ++it) {
    const int g = wk.step(P, it);
    const int b = wk.b;
    if (b != cur) {
      if (cur >= 0) flush_partial<KV, HG>(P, cur, hg, st, sm.merge_o, sm.merge_ml);
      cur = b;
      const __nv_bfloat16 *qb = reinterpret_cast<const __nv_bfloat16 *>(P.q) + (size_t)b * H * kHeadDim;
      load_q_rows<KV>(qb, hg * 16, qa, P.scale_log2, rowf);
      st.init();
    }
    if (it % C::kGroups != grp) continue;
    const int s = it % C::kStages;
    if (*sm.abort_flag) continue;   // after a timeout: keep walking, so every flush barrier is met
    if (!mbar_wait(smem_u32(&sm.full[s]), (it / C::kStages) & 1)) {
      record_status(P.status, kStatusTimeout);
      *sm.abort_flag = 1;
      continue;
    }
    const uint8_t *stg = sm.stages + s * C::kStageBytes;
    const int64_t trow = tile_row0(P, b, g);
    const int64_t row0 = P.seq.start[b], row1 = row0 + P.seq.len[b];
    bool valid[NT][2];
    float colk[NT][2], colv[NT][2];
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int rr = tok0 + n * 8 + 2 * c + e;
        const int64_t row = trow + rr;
        valid[n][e] = row >= row0 && row < row1;
        if (KV == kKvFp8) {
          const float *sc = reinterpret_cast<const float *>(stg + 2 * C::kKBytes);
          colk[n][e] = sc[rr];
          colv[n][e] = sc[kTile + rr];
        } else {
          colk[n][e] = 1.f;
          colv[n][e] = 1.f;
        }
      }
    float sacc[NT][4];
    qk_tile<KV, NT>(qa, smem_u32(stg), tok0, sacc);
    softmax_pv_tile<KV, NT>(st, sacc, rowf, colk, colv, valid, smem_u32(stg + C::kKBytes), tok0);
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&sm.empty[s]));
  }
  if (cur >= 0) flush_partial<KV, HG>(P, cur, hg, st, sm.merge_o, sm.merge_ml);
}

// ------------------------------------------------------------------ pass 2

template <int KV, int HG>
__global__ void __launch_bounds__(StreamCfg<KV, HG, 1>::kThreads, StreamCfg<KV, HG, 1>::kSub > 1 ? 1 : 2)
    decode_pass2_kernel(const __grid_constant__ TensorMaps tm, const __grid_constant__ DecodeParams P) {
  using C = StreamCfg<KV, HG, 1>;
  constexpr int H = 16 * HG;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  StreamSmem<KV, HG, 1> sm(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(smem_u32(&sm.full[s]), C::kFullCount);
      mbar_init(smem_u32(&sm.empty[s]), C::kGroupWarps);
    }
    *sm.abort_flag = 0;
    fence_barrier_init();
  }
  for (int t = threadIdx.x; t < 2 * kHistBins; t += C::kThreads) sm.hist[t] = 0;
  __syncthreads();
  griddep_launch_dependents();
  // Top-digit counts of the candidates: the first two sequences of this CTA's range count in
  // shared memory (flushed once at the end), any further ones straight into global memory.
  TileWalk wk(P, true);
  const int b_lo = (wk.n > 0) ? seq_of_tile(P.seq, P.batch, wk.lo) : 0;
  if (warp == C::kConsumers) {
    produce_stream<KV, HG, 1>(tm, P, sm.stages, sm.full, sm.empty, sm.abort_flag);
  } else {
    const int grp = warp / C::kGroupWarps, gw = warp % C::kGroupWarps;
    const int g8 = lane >> 2, c = lane & 3;
    constexpr int NT2 = C::kPass2Rows / 8;
    constexpr int kWarpsPerTile = kTile / C::kPass2Rows;
    const int sub = gw / kWarpsPerTile;                       // this warp's tile of each stage
    const int tok0 = (gw % kWarpsPerTile) * C::kPass2Rows;    // and its rows in that tile
    int cur = -1;
    int64_t n_cand = 0;
    uint32_t *hrow = nullptr;
    uint32_t qa[HG][8][4];
    float rowf[HG][2], lse2[HG][2];
    griddep_wait();
    const int n_stages = (wk.n + C::kSub - 1) / C::kSub;
    for (int k = grp; k < n_stages; k += C::kGroups) {
      const int it = k * C::kSub + sub;
      const int s = k % C::kStages;
      if (it >= wk.n) {   // the last stage holds fewer tiles: release it all the same
        if (!mbar_wait(smem_u32(&sm.full[s]), (k / C::kStages) & 1)) {
          record_status(P.status, kStatusTimeout);
          *sm.abort_flag = 1;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&sm.empty[s]));
        continue;
      }
      const int g = wk.step(P, it);
      const int b = wk.b;
      if (b != cur) {
        cur = b;
        const __nv_bfloat16 *qb = reinterpret_cast<const __nv_bfloat16 *>(P.q) + (size_t)b * H * kHeadDim;
#pragma unroll
        for (int mt = 0; mt < HG; ++mt) {
          load_q_rows<KV>(qb, mt * 16, qa[mt], P.scale_log2, rowf[mt]);
          lse2[mt][0] = P.lse[b * H + mt * 16 + g8] * kLog2e;
          lse2[mt][1] = P.lse[b * H + mt * 16 + g8 + 8] * kLog2e;
        }
        n_cand = (int64_t)P.seq.len[b] - P.window;   // candidates: positions [0, p - window + 1)
        hrow = (b - b_lo < 2) ? sm.hist + (b - b_lo) * kHistBins
                              : (P.hist ? P.hist + (size_t)b * kHistBins : nullptr);
      }
      if (!mbar_wait(smem_u32(&sm.full[s]), (k / C::kStages) & 1)) {
        record_status(P.status, kStatusTimeout);
        *sm.abort_flag = 1;
      }
      if (*sm.abort_flag) break;
      const uint8_t *stg = sm.stages + s * C::kStageBytes + sub * C::kTileBytes;
      const int64_t trow = tile_row0(P, b, g);
      const int64_t row0 = P.seq.start[b], row1 = row0 + P.seq.len[b];
      float colk[NT2][2];
#pragma unroll
      for (int n = 0; n < NT2; ++n)
#pragma unroll
        for (int e = 0; e < 2; ++e)
          colk[n][e] = (KV == kKvFp8)
                           ? reinterpret_cast<const float *>(stg + C::kKBytes)[tok0 + n * 8 + 2 * c + e]
                           : 1.f;
      float sacc[HG][NT2][4];
      qk_tile_mt<KV, HG, NT2>(qa, smem_u32(stg), tok0, sacc);
      // x = s * (rowf * colk) - lse2 and the sum over heads, two columns at a time
      float2 acc[NT2];
#pragma unroll
      for (int n = 0; n < NT2; ++n) acc[n] = make_float2(0.f, 0.f);
#pragma unroll
      for (int mt = 0; mt < HG; ++mt)
#pragma unroll
        for (int n = 0; n < NT2; ++n)
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const float2 a = make_float2(rowf[mt][h] * colk[n][0], rowf[mt][h] * colk[n][1]);
            const float2 x = ffma2(make_float2(sacc[mt][n][2 * h], sacc[mt][n][2 * h + 1]), a,
                                   make_float2(-lse2[mt][h], -lse2[mt][h]));
            acc[n] = fadd2(acc[n], make_float2(fast_exp2(x.x), fast_exp2(x.y)));
          }
      float cs[NT2][2];
#pragma unroll
      for (int n = 0; n < NT2; ++n) {
        cs[n][0] = acc[n].x;
        cs[n][1] = acc[n].y;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&sm.empty[s]));
#pragma unroll
      for (int n = 0; n < NT2; ++n)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          float v = cs[n][e];
          v += __shfl_xor_sync(0xffffffffu, v, 4);
          v += __shfl_xor_sync(0xffffffffu, v, 8);
          v += __shfl_xor_sync(0xffffffffu, v, 16);
          cs[n][e] = v;
        }
      if (g8 == 0) {
        float *srow = P.scores + (size_t)b * P.score_stride;
#pragma unroll
        for (int n = 0; n < NT2; ++n)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int64_t row = trow + tok0 + n * 8 + 2 * c + e;
            if (row >= row0 && row < row1) {
              const int64_t pos = row - row0;
              srow[pos] = cs[n][e];
              if (P.hist && pos < n_cand) atomicAdd(&hrow[__float_as_uint(cs[n][e]) >> 21], 1u);
            }
          }
      }
    }
  }
  __syncthreads();
  if (P.hist && wk.n > 0 && !*sm.abort_flag) {
    const int b_hi = seq_of_tile(P.seq, P.batch, wk.hi - 1);
    for (int t = threadIdx.x; t < 2 * kHistBins; t += C::kThreads) {
      const int k = t / kHistBins;
      const uint32_t v = sm.hist[t];
      if (v && b_lo + k <= b_hi) atomicAdd(&P.hist[(size_t)(b_lo + k) * kHistBins + (t % kHistBins)], v);
    }
  }
}

template <int KV, int HG>
cudaError_t launch_decode_t(int pass, const TensorMaps &tm, const DecodeParams &p,
                            cudaStream_t s) {
  static_assert(StreamCfg<KV, HG, 0>::kSmem <= 227 * 1024, "pass 1 shared memory");
  static_assert(StreamCfg<KV, HG, 1>::kSmem <= 227 * 1024, "pass 2 shared memory");
  if (p.n_ctas < 1) return cudaSuccess;
  if (pass == 0) {
    using C = StreamCfg<KV, HG, 0>;
    auto kern = decode_pass1_kernel<KV, HG>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::kSmem);
    if (e != cudaSuccess) return e;
    e = launch_pdl(kern, p.n_ctas, C::kThreads, C::kSmem, s, tm, p);
    if (e != cudaSuccess) return e;
  } else {
    using C = StreamCfg<KV, HG, 1>;
    auto kern = decode_pass2_kernel<KV, HG>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::kSmem);
    if (e != cudaSuccess) return e;
    e = launch_pdl(kern, p.n_ctas2, C::kThreads, C::kSmem, s, tm, p);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_pass(int pass, int kv_dtype, const TensorMaps &tm,
                               const DecodeParams &p, cudaStream_t s) {
  const int hg = p.n_heads / 16;
  if (kv_dtype == HS2_KV_BF16) {
    if (hg == 1) return launch_decode_t<kKvBf16, 1>(pass, tm, p, s);
    if (hg == 2) return launch_decode_t<kKvBf16, 2>(pass, tm, p, s);
  } else {
    if (hg == 1) return launch_decode_t<kKvFp8, 1>(pass, tm, p, s);
    if (hg == 2) return launch_decode_t<kKvFp8, 2>(pass, tm, p, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace hs2
