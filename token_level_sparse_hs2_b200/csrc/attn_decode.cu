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
// Work split: the cache rows of sequence b are cut into work items of `chunk_tiles` 64-row
// tiles aligned to absolute row multiples of 64 (rows of other sequences in a boundary tile are
// masked). One CTA per item: warp 4 issues TMA tile loads into a ring of stages; warps 0..3
// consume. Pass 1 writes (max, denominator, unnormalised output) per item and head; the last
// CTA of a sequence to finish (arrival counter) merges them into O and lse. Pass 2 re-reads K,
// computes s[t] = sum_h exp2(x_h[t] - lse_h * log2 e) and counts the top radix digit of every
// candidate score for the selection step.
#include "attn_pipeline.cuh"
#include "internal.h"

namespace hs2 {

namespace {

constexpr int kConsumerWarps = 4;
constexpr int kThreads = (kConsumerWarps + 1) * 32;

// ------------------------------------------------------------------ pass 1 + sparse layers

// Where a CTA's result goes. A group is the set of CTAs that share one output block (a
// sequence's items in pass 1, a query row's splits in a sparse layer). With one CTA per group
// the CTA writes the output directly; otherwise it writes its partial (max, denominator,
// unnormalised output per head) and the last CTA of the group to arrive merges all of them.
struct MergeTarget {
  int n_group;
  float *group_part;   // [n_group][H][2 + 128]
  int slot;            // this CTA's index in the group
  int *counter;
  void *out;           // [H][128] block of the output
  int out_f32;
  float *lse;          // [H] or null
};

// Merges the warps' softmax states (stashed in smem) and delivers the result.
template <int KV, int HG>
__device__ void finish_cta(const float *ws_o, const float *ws_ml, const MergeTarget &mt) {
  constexpr int H = 16 * HG;
  constexpr int TG = kConsumerWarps / HG;
  constexpr int PW = 2 + kHeadDim;
  __shared__ int s_last;
  if (mt.n_group == 1) {
    for (int t = threadIdx.x; t < H * kHeadDim; t += kThreads) {
      const int h = t / kHeadDim, d = t % kHeadDim;
      const int hg = h >> 4, r = h & 15;
      float M = -INFINITY;
      for (int tg = 0; tg < TG; ++tg) M = fmaxf(M, ws_ml[((tg * HG + hg) * 16 + r) * 2]);
      float L = 0.f, O = 0.f;
      for (int tg = 0; tg < TG; ++tg) {
        const int w = tg * HG + hg;
        const float m = ws_ml[(w * 16 + r) * 2];
        const float f = (m == -INFINITY) ? 0.f : fast_exp2(m - M);
        L += f * ws_ml[(w * 16 + r) * 2 + 1];
        O += f * ws_o[(w * 16 + r) * kHeadDim + d];
      }
      const float val = O / L;
      if (mt.out_f32) reinterpret_cast<float *>(mt.out)[t] = val;
      else reinterpret_cast<__nv_bfloat16 *>(mt.out)[t] = __float2bfloat16_rn(val);
      if (mt.lse && d == 0) mt.lse[h] = (M + __log2f(L)) * kLn2;
    }
    return;
  }
  float *part = mt.group_part + (size_t)mt.slot * H * PW;
  for (int t = threadIdx.x; t < H * PW; t += kThreads) {
    const int h = t / PW, col = t % PW;
    const int hg = h >> 4, r = h & 15;
    float M = -INFINITY;
    for (int tg = 0; tg < TG; ++tg) M = fmaxf(M, ws_ml[((tg * HG + hg) * 16 + r) * 2]);
    float acc = (col == 0) ? M : 0.f;
    if (col > 0) {
      for (int tg = 0; tg < TG; ++tg) {
        const int w = tg * HG + hg;
        const float m = ws_ml[(w * 16 + r) * 2];
        const float f = (m == -INFINITY) ? 0.f : fast_exp2(m - M);
        acc += f * (col == 1 ? ws_ml[(w * 16 + r) * 2 + 1] : ws_o[(w * 16 + r) * kHeadDim + col - 2]);
      }
    }
    part[t] = acc;
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const int prev = atomicAdd(mt.counter, 1);
    s_last = (prev == mt.n_group - 1);
    if (s_last) *mt.counter = 0;   // ready for the next call
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  for (int t = threadIdx.x; t < H * kHeadDim; t += kThreads) {
    const int h = t / kHeadDim, d = t % kHeadDim;
    float M = -INFINITY;
    for (int i = 0; i < mt.n_group; ++i) M = fmaxf(M, __ldcg(mt.group_part + ((size_t)i * H + h) * PW));
    float L = 0.f, O = 0.f;
    for (int i = 0; i < mt.n_group; ++i) {
      const float *pp = mt.group_part + ((size_t)i * H + h) * PW;
      const float m = __ldcg(pp);
      const float f = (m == -INFINITY) ? 0.f : fast_exp2(m - M);
      L += f * __ldcg(pp + 1);
      O += f * __ldcg(pp + 2 + d);
    }
    const float val = O / L;
    if (mt.out_f32) reinterpret_cast<float *>(mt.out)[t] = val;
    else reinterpret_cast<__nv_bfloat16 *>(mt.out)[t] = __float2bfloat16_rn(val);
    if (mt.lse && d == 0) mt.lse[h] = (M + __log2f(L)) * kLn2;
  }
}

// Consumer warps of pass 1 / sparse layers. Warp (hg, tg): heads [16 hg, 16 hg + 16), tile
// rows [tg * NTW, (tg+1) * NTW) with NTW = 16 * HG. `is_valid(it, rr)` says whether row rr
// of tile it holds a cache row this CTA attends to. The warp's state is stashed into
// ws_o / ws_ml (stage memory) at the end.
template <int KV, int HG, class Valid>
__device__ void consume_pv(const Valid &is_valid, uint8_t *stages, uint64_t *full,
                           uint64_t *empty, uint8_t *q_smem, const __nv_bfloat16 *qg,
                           float scale_log2, int n_tiles, volatile int *abort_flag,
                           uint32_t *status) {
  using C = DecodeCfg<KV, 0>;
  constexpr int H = 16 * HG;
  constexpr int NTW = 16 * HG;
  constexpr int NT = NTW / 8;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hg = warp % HG, tg = warp / HG;
  const int tok0 = tg * NTW;
  const int g = lane >> 2, c = lane & 3;
  uint32_t qa[8][4];
  float rowf[2];
  if (KV == kKvBf16) {
    load_q_frags_bf16(smem_u32(q_smem), H, hg * 16, qa);
    rowf[0] = rowf[1] = scale_log2;
  } else {
    float pw[2];
    load_q_frags_f16(qg, hg * 16, qa, pw);
    rowf[0] = scale_log2 * pw[0];
    rowf[1] = scale_log2 * pw[1];
  }
  WarpSoftmax st;
  st.init();
  for (int it = 0; it < n_tiles; ++it) {
    const int s = it % C::kStages;
    if (!mbar_wait(smem_u32(&full[s]), (it / C::kStages) & 1)) {
      record_status(status, kStatusTimeout);
      *abort_flag = 1;
    }
    if (*abort_flag) break;
    const uint8_t *stg = stages + s * C::kStageBytes;
    bool valid[NT][2];
    float colk[NT][2], colv[NT][2];
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int rr = tok0 + n * 8 + 2 * c + e;
        valid[n][e] = is_valid(it, rr);
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
    if (lane == 0) mbar_arrive(smem_u32(&empty[s]));
  }
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    st.l[h] += __shfl_xor_sync(0xffffffffu, st.l[h], 1);
    st.l[h] += __shfl_xor_sync(0xffffffffu, st.l[h], 2);
  }
  // every consumer is done with the stages before they are reused for the merge
  named_barrier_sync(1, kConsumerWarps * 32);
  float *ws_o = reinterpret_cast<float *>(stages);              // [warp][16][128]
  float *ws_ml = ws_o + kConsumerWarps * 16 * kHeadDim;         // [warp][16][2]
#pragma unroll
  for (int n = 0; n < 16; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int r = g + (e >> 1) * 8;
      ws_o[(warp * 16 + r) * kHeadDim + o_col<KV>(n, e & 1, c)] = st.o[n][e] * st.vref;
    }
  if (c == 0) {
    ws_ml[(warp * 16 + g) * 2 + 0] = st.m[0];
    ws_ml[(warp * 16 + g) * 2 + 1] = st.l[0];
    ws_ml[(warp * 16 + g + 8) * 2 + 0] = st.m[1];
    ws_ml[(warp * 16 + g + 8) * 2 + 1] = st.l[1];
  }
}

// Shared memory of a pass-1 / sparse CTA: stages | Q (bf16, H rows) | barriers | abort flag
template <int KV, int HG>
struct PvSmem {
  using C = DecodeCfg<KV, 0>;
  uint8_t *stages, *q;
  uint64_t *full, *empty;
  volatile int *abort_flag;
  __device__ explicit PvSmem(uint8_t *raw) {
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
    stages = base;
    q = stages + C::kStages * C::kStageBytes;
    full = reinterpret_cast<uint64_t *>(q + 16 * HG * 256);
    empty = full + C::kStages;
    abort_flag = reinterpret_cast<volatile int *>(empty + C::kStages);
  }
  static constexpr size_t bytes() {
    return 1024 + C::kStages * C::kStageBytes + 16 * HG * 256 + 2 * C::kStages * 8 + 16;
  }
};

template <int HG>
__device__ __forceinline__ void stage_q_bf16(uint8_t *q_smem, const __nv_bfloat16 *qg) {
  constexpr int H = 16 * HG;
  for (int t = threadIdx.x; t < H * 16; t += kThreads) {
    const int r = t >> 4, ch = t & 15;
    const uint4 v = *reinterpret_cast<const uint4 *>(qg + r * kHeadDim + ch * 8);
    *reinterpret_cast<uint4 *>(q_smem + tile_off(H, r, ch * 8)) = v;
  }
}

struct TileValid {
  int64_t tile_row0, row0, row1;   // absolute row of tile 0 row 0; the sequence's rows
  __device__ bool operator()(int it, int rr) const {
    const int64_t row = tile_row0 + (int64_t)it * kTile + rr;
    return row >= row0 && row < row1;
  }
};

template <int KV, int HG>
__global__ void __launch_bounds__(kThreads, 1)
    decode_pass1_kernel(const __grid_constant__ TensorMaps tm, const __grid_constant__ DecodeParams P) {
  using C = DecodeCfg<KV, 0>;
  constexpr int H = 16 * HG;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  PvSmem<KV, HG> sm(smem_raw);
  const int warp = threadIdx.x >> 5;
  const int item = blockIdx.x;
  const int b = find_item_seq(P.seq, P.batch, item);
  const int64_t row0 = P.seq.start[b], row1 = row0 + P.seq.len[b];
  const int seq_tile0 = static_cast<int>(row0 / kTile);
  const int seq_tiles = static_cast<int>((row1 + kTile - 1) / kTile) - seq_tile0;
  const int j = item - P.seq.item_begin[b];
  const int tile_begin = seq_tile0 + j * P.chunk_tiles;
  const int n_tiles = min(P.chunk_tiles, seq_tiles - j * P.chunk_tiles);
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(smem_u32(&sm.full[s]), C::kFullCount);
      mbar_init(smem_u32(&sm.empty[s]), kConsumerWarps);
    }
    *sm.abort_flag = 0;
    fence_barrier_init();
  }
  const __nv_bfloat16 *qg = reinterpret_cast<const __nv_bfloat16 *>(P.q) + (size_t)b * H * kHeadDim;
  if (KV == kKvBf16) stage_q_bf16<HG>(sm.q, qg);
  __syncthreads();
  if (warp == kConsumerWarps) {
    produce<KV, 0>(tm, P.k_scale, P.v_scale, P.kv_rows, sm.stages, sm.full, sm.empty, tile_begin,
                   n_tiles, sm.abort_flag, P.status);
  } else {
    const TileValid tv{(int64_t)tile_begin * kTile, row0, row1};
    consume_pv<KV, HG>(tv, sm.stages, sm.full, sm.empty, sm.q, qg, P.scale_log2, n_tiles,
                       sm.abort_flag, P.status);
  }
  __syncthreads();
  if (*sm.abort_flag) return;
  const float *ws_o = reinterpret_cast<const float *>(sm.stages);
  MergeTarget mt;
  mt.n_group = P.seq.item_begin[b + 1] - P.seq.item_begin[b];
  mt.group_part = P.part + (size_t)P.seq.item_begin[b] * H * (2 + kHeadDim);
  mt.slot = j;
  mt.counter = P.counter + b;
  mt.out_f32 = P.out_f32;
  mt.out = P.out_f32 ? (void *)(reinterpret_cast<float *>(P.out) + (size_t)b * H * kHeadDim)
                     : (void *)(reinterpret_cast<__nv_bfloat16 *>(P.out) + (size_t)b * H * kHeadDim);
  mt.lse = P.lse + (size_t)b * H;
  finish_cta<KV, HG>(ws_o, ws_o + kConsumerWarps * 16 * kHeadDim, mt);
}

// Sparse layer: gather producer. All 32 lanes of the producer warp copy two gathered rows
// each per tile with 16-byte cp.async, then arrive on the stage's barrier when they land.
template <int KV>
__device__ void produce_gather(const SparseParams &P, int r, int64_t seq_row0, int64_t p,
                               int e_begin, int cnt, uint8_t *stages, uint64_t *full,
                               uint64_t *empty, int n_tiles, volatile int *abort_flag) {
  using C = DecodeCfg<KV, 0>;
  const int lane = threadIdx.x & 31;
  const int32_t *idx = P.idx + (size_t)r * P.idx_stride;
  bool bad = false;
  for (int it = 0; it < n_tiles; ++it) {
    const int s = it % C::kStages;
    const uint32_t par = ((it / C::kStages) & 1) ^ 1;
    if (it >= C::kStages) {
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
    uint8_t *st = stages + s * C::kStageBytes;
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int rr = 2 * lane + u;
      const int e = e_begin + it * kTile + rr;
      const bool v = e < cnt;
      int64_t pos = v ? (int64_t)__ldg(idx + e) : 0;
      if (pos < 0 || pos > p) {   // out-of-range index: flag it and read row 0 instead
        bad = true;
        pos = 0;
      }
      const int64_t row = seq_row0 + pos;
      const uint32_t nb = v ? 16u : 0u;
      if (KV == kKvBf16) {
        const uint8_t *ksrc = reinterpret_cast<const uint8_t *>(P.k) + row * 256;
        const uint8_t *vsrc = reinterpret_cast<const uint8_t *>(P.v) + row * 256;
#pragma unroll
        for (int ch = 0; ch < 16; ++ch) {
          cp_async_16(smem_u32(st + tile_off(kTile, rr, ch * 8)), ksrc + ch * 16, nb);
          cp_async_16(smem_u32(st + C::kKBytes + tile_off(kTile, rr, ch * 8)), vsrc + ch * 16, nb);
        }
      } else {
        const uint8_t *ksrc = reinterpret_cast<const uint8_t *>(P.k) + row * 128;
        const uint8_t *vsrc = reinterpret_cast<const uint8_t *>(P.v) + row * 128;
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          cp_async_16(smem_u32(st + fp8_off(rr, ch * 16)), ksrc + ch * 16, nb);
          cp_async_16(smem_u32(st + C::kKBytes + fp8_off(rr, ch * 16)), vsrc + ch * 16, nb);
        }
        uint8_t *sc = st + 2 * C::kKBytes;
        cp_async_4(smem_u32(sc + rr * 4), P.k_scale + row, v ? 4u : 0u);
        cp_async_4(smem_u32(sc + (kTile + rr) * 4), P.v_scale + row, v ? 4u : 0u);
      }
    }
    cp_async_mbar_arrive(smem_u32(&full[s]));
  }
  if (bad) record_status(P.status, kStatusCheck);
}

struct CountValid {
  int e_begin, cnt;
  __device__ bool operator()(int it, int rr) const { return e_begin + it * kTile + rr < cnt; }
};

template <int KV, int HG>
__global__ void __launch_bounds__(kThreads, 1) sparse_gather_kernel(const __grid_constant__ SparseParams P) {
  using C = DecodeCfg<KV, 0>;
  constexpr int H = 16 * HG;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  PvSmem<KV, HG> sm(smem_raw);
  const int warp = threadIdx.x >> 5;
  const int r = blockIdx.x / P.n_split, j = blockIdx.x % P.n_split;
  const int b = r / P.n_q, i = r % P.n_q;
  const int64_t seq_row0 = P.seq.start[b];
  const int64_t p = (int64_t)P.seq.len[b] - P.n_q + i;
  int cnt = __ldg(P.count + r);
  if (cnt < 1 || cnt > P.idx_stride) {
    if (threadIdx.x == 0) record_status(P.status, kStatusCheck);
    cnt = max(1, min(cnt, P.idx_stride));
  }
  const int e_begin = j * P.split_len;
  const int n_tiles = max(0, min(P.split_len, cnt - e_begin) + kTile - 1) / kTile;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(smem_u32(&sm.full[s]), 32);
      mbar_init(smem_u32(&sm.empty[s]), kConsumerWarps);
    }
    *sm.abort_flag = 0;
    fence_barrier_init();
  }
  const __nv_bfloat16 *qg = reinterpret_cast<const __nv_bfloat16 *>(P.q) + (size_t)r * H * kHeadDim;
  if (KV == kKvBf16) stage_q_bf16<HG>(sm.q, qg);
  __syncthreads();
  if (warp == kConsumerWarps) {
    produce_gather<KV>(P, r, seq_row0, p, e_begin, cnt, sm.stages, sm.full, sm.empty, n_tiles,
                       sm.abort_flag);
  } else {
    const CountValid cv{e_begin, cnt};
    consume_pv<KV, HG>(cv, sm.stages, sm.full, sm.empty, sm.q, qg, P.scale_log2, n_tiles,
                       sm.abort_flag, P.status);
  }
  __syncthreads();
  if (*sm.abort_flag) return;
  const float *ws_o = reinterpret_cast<const float *>(sm.stages);
  MergeTarget mt;
  mt.n_group = P.n_split;
  mt.group_part = P.part + (size_t)r * P.n_split * H * (2 + kHeadDim);
  mt.slot = j;
  mt.counter = P.counter + r;
  mt.out_f32 = P.out_f32;
  mt.out = P.out_f32 ? (void *)(reinterpret_cast<float *>(P.out) + (size_t)r * H * kHeadDim)
                     : (void *)(reinterpret_cast<__nv_bfloat16 *>(P.out) + (size_t)r * H * kHeadDim);
  mt.lse = nullptr;
  finish_cta<KV, HG>(ws_o, ws_o + kConsumerWarps * 16 * kHeadDim, mt);
}

// ------------------------------------------------------------------ pass 2

// Warp w: all H heads (HG m-tiles), tile rows [16 w, 16 w + 16).
template <int KV, int HG>
__global__ void __launch_bounds__(kThreads, 1)
    decode_pass2_kernel(const __grid_constant__ TensorMaps tm, const __grid_constant__ DecodeParams P) {
  using C = DecodeCfg<KV, 1>;
  constexpr int H = 16 * HG;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *stages = smem;
  uint8_t *q_smem = stages + C::kStages * C::kStageBytes;
  uint32_t *hist = reinterpret_cast<uint32_t *>(q_smem + H * 256);   // kHistBins
  uint64_t *full = reinterpret_cast<uint64_t *>(hist + kHistBins);
  uint64_t *empty = full + C::kStages;
  volatile int *abort_flag = reinterpret_cast<volatile int *>(empty + C::kStages);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int item = blockIdx.x;
  const int b = find_item_seq(P.seq, P.batch, item);
  const int64_t row0 = P.seq.start[b], row1 = row0 + P.seq.len[b];
  const int seq_tile0 = static_cast<int>(row0 / kTile);
  const int seq_tiles = static_cast<int>((row1 + kTile - 1) / kTile) - seq_tile0;
  const int j = item - P.seq.item_begin[b];
  const int tile_begin = seq_tile0 + j * P.chunk_tiles;
  const int n_tiles = min(P.chunk_tiles, seq_tiles - j * P.chunk_tiles);
  const int64_t p = P.seq.len[b] - 1;
  const int64_t n_cand = p - P.window + 1;    // positions < n_cand are selection candidates

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(smem_u32(&full[s]), C::kFullCount);
      mbar_init(smem_u32(&empty[s]), kConsumerWarps);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  for (int t = threadIdx.x; t < kHistBins; t += kThreads) hist[t] = 0;
  const __nv_bfloat16 *qg = reinterpret_cast<const __nv_bfloat16 *>(P.q) + (size_t)b * H * kHeadDim;
  if (KV == kKvBf16) {
    for (int t = threadIdx.x; t < H * 16; t += kThreads) {
      const int r = t >> 4, ch = t & 15;
      const uint4 v = *reinterpret_cast<const uint4 *>(qg + r * kHeadDim + ch * 8);
      *reinterpret_cast<uint4 *>(q_smem + tile_off(H, r, ch * 8)) = v;
    }
  }
  __syncthreads();

  if (warp == kConsumerWarps) {
    produce<KV, 1>(tm, P.k_scale, P.v_scale, P.kv_rows, stages, full, empty, tile_begin, n_tiles,
                   abort_flag, P.status);
  } else {
    const int g = lane >> 2, c = lane & 3;
    const int tok0 = warp * 16;
    uint32_t qa[HG][8][4];
    float rowf[HG][2], lse2[HG][2];
#pragma unroll
    for (int mt = 0; mt < HG; ++mt) {
      if (KV == kKvBf16) {
        load_q_frags_bf16(smem_u32(q_smem), H, mt * 16, qa[mt]);
        rowf[mt][0] = rowf[mt][1] = P.scale_log2;
      } else {
        float pw[2];
        load_q_frags_f16(qg, mt * 16, qa[mt], pw);
        rowf[mt][0] = P.scale_log2 * pw[0];
        rowf[mt][1] = P.scale_log2 * pw[1];
      }
      lse2[mt][0] = P.lse[b * H + mt * 16 + g] * kLog2e;
      lse2[mt][1] = P.lse[b * H + mt * 16 + g + 8] * kLog2e;
    }
    float *srow = P.scores + (size_t)b * P.score_stride;
    for (int it = 0; it < n_tiles; ++it) {
      const int s = it % C::kStages;
      if (!mbar_wait(smem_u32(&full[s]), (it / C::kStages) & 1)) {
        record_status(P.status, kStatusTimeout);
        *abort_flag = 1;
      }
      if (*abort_flag) break;
      const uint8_t *stg = stages + s * C::kStageBytes;
      const int64_t tile_row = (int64_t)(tile_begin + it) * kTile;
      float colk[2][2];
#pragma unroll
      for (int n = 0; n < 2; ++n)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          if (KV == kKvFp8) {
            const float *sc = reinterpret_cast<const float *>(stg + C::kKBytes);
            colk[n][e] = sc[tok0 + n * 8 + 2 * c + e];
          } else {
            colk[n][e] = 1.f;
          }
        }
      float colsum[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
#pragma unroll
      for (int mt = 0; mt < HG; ++mt) {
        float sacc[2][4];
        qk_tile<KV, 2>(qa[mt], smem_u32(stg), tok0, sacc);
#pragma unroll
        for (int n = 0; n < 2; ++n)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float x = sacc[n][e] * rowf[mt][e >> 1] * colk[n][e & 1] - lse2[mt][e >> 1];
            colsum[n][e & 1] += fast_exp2(x);
          }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&empty[s]));
      // sum over the 8 row groups -> lanes 0..3 hold the 4 column sums
#pragma unroll
      for (int n = 0; n < 2; ++n)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          float v = colsum[n][e];
          v += __shfl_xor_sync(0xffffffffu, v, 4);
          v += __shfl_xor_sync(0xffffffffu, v, 8);
          v += __shfl_xor_sync(0xffffffffu, v, 16);
          colsum[n][e] = v;
        }
      if (g == 0) {
#pragma unroll
        for (int n = 0; n < 2; ++n)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int64_t row = tile_row + tok0 + n * 8 + 2 * c + e;
            if (row >= row0 && row < row1) {
              const int64_t pos = row - row0;
              const float sv = colsum[n][e];
              srow[pos] = sv;
              if (P.hist && pos < n_cand) atomicAdd(&hist[__float_as_uint(sv) >> 21], 1u);
            }
          }
      }
    }
  }
  __syncthreads();
  if (P.hist && !*abort_flag) {
    uint32_t *gh = P.hist + (size_t)b * kHistBins;
    for (int t = threadIdx.x; t < kHistBins; t += kThreads)
      if (hist[t]) atomicAdd(&gh[t], hist[t]);
  }
}

template <int KV, int HG>
constexpr size_t pass1_smem() {
  return PvSmem<KV, HG>::bytes();
}

template <int KV, int HG>
constexpr size_t pass2_smem() {
  using C = DecodeCfg<KV, 1>;
  return 1024 + C::kStages * C::kStageBytes + 16 * HG * 256 + kHistBins * 4 +
         2 * C::kStages * 8 + 16;
}

template <int KV, int HG>
cudaError_t launch_decode_t(int pass, const TensorMaps &tm, const DecodeParams &p,
                            cudaStream_t s) {
  static_assert(pass1_smem<KV, HG>() <= 227 * 1024, "pass 1 shared memory");
  static_assert(pass2_smem<KV, HG>() <= 227 * 1024, "pass 2 shared memory");
  if (pass == 0) {
    const size_t smem = pass1_smem<KV, HG>();
    auto kern = decode_pass1_kernel<KV, HG>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<p.n_items, kThreads, smem, s>>>(tm, p);
  } else {
    const size_t smem = pass2_smem<KV, HG>();
    auto kern = decode_pass2_kernel<KV, HG>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<p.n_items, kThreads, smem, s>>>(tm, p);
  }
  return cudaGetLastError();
}

template <int KV, int HG>
cudaError_t launch_sparse_t(const SparseParams &p, cudaStream_t s) {
  const size_t smem = pass1_smem<KV, HG>();
  auto kern = sparse_gather_kernel<KV, HG>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int grid = p.batch * p.n_q * p.n_split;
  kern<<<grid, kThreads, smem, s>>>(p);
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

cudaError_t launch_sparse(int kv_dtype, const SparseParams &p, cudaStream_t s) {
  const int hg = p.n_heads / 16;
  if (kv_dtype == HS2_KV_BF16) {
    if (hg == 1) return launch_sparse_t<kKvBf16, 1>(p, s);
    if (hg == 2) return launch_sparse_t<kKvBf16, 2>(p, s);
  } else {
    if (hg == 1) return launch_sparse_t<kKvFp8, 1>(p, s);
    if (hg == 2) return launch_sparse_t<kKvFp8, 2>(p, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace hs2
