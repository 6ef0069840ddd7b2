// attn_sparse.cu -- a sparse-attention layer of a hybrid block (KV Reuse): each query row's
// own queries attend only to the cache rows its full-attention layer selected, and every
// gathered K/V row serves all H heads.
//
// "HySparse2: How Xiaomi Split the Transformer to Fix Agent Prefill Costs", section "KV Reuse
// and Token-Level Sparse Selection": the sparse layers take the full layer's indices and cache
// as they are; the forced-window tokens are ordinary rows of that cache.
//
// One CTA per (query row, split of its selected list): warp 4 gathers 64 selected rows per
// tile with 16-byte cp.async into the swizzled tile layout; warps 0..3 run the same tensor-core
// online softmax as the full layer. Splits of one row are combined by merge_partials_kernel,
// which also serves the full layer's decode pass 1.
#include "attn_pipeline.cuh"
#include "internal.h"

namespace hs2 {

namespace {

constexpr int kConsumerWarps = 4;
constexpr int kThreads = (kConsumerWarps + 1) * 32;


// Where a CTA's result goes. A group is the set of CTAs that share one output block (a
// sequence's items in pass 1, a query row's splits in a sparse layer). With one CTA per group
// the CTA writes the output directly; otherwise it writes its partial (max, denominator,
// unnormalised output per head) and merge_partials_kernel combines the group afterwards.
struct MergeTarget {
  int n_group;
  float *group_part;   // [n_group][H][kPartRow]
  int slot;            // this CTA's index in the group
  void *out;           // [H][128] block of the output
  int out_f32;
  float *lse;          // [H] or null
};

// Merges the warps' softmax states (stashed in smem) and delivers the result.
template <int KV, int HG>
__device__ void finish_cta(const float *ws_o, const float *ws_ml, const MergeTarget &mt) {
  constexpr int H = 16 * HG;
  constexpr int TG = kConsumerWarps / HG;
  const bool direct = mt.n_group == 1;
  float *part = mt.group_part + (size_t)mt.slot * H * kPartRow;
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
    if (direct) {
      const float val = O / L;
      if (mt.out_f32) reinterpret_cast<float *>(mt.out)[t] = val;
      else reinterpret_cast<__nv_bfloat16 *>(mt.out)[t] = __float2bfloat16_rn(val);
      if (mt.lse && d == 0) mt.lse[h] = (M + __log2f(L)) * kLn2;
    } else {
      part[h * kPartRow + kPartO + d] = O;
      if (d == 0) {
        part[h * kPartRow] = M;
        part[h * kPartRow + 1] = L;
      }
    }
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
      int64_t pos = v ? (int64_t)__ldcg(idx + e) : 0;
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
  constexpr int NTW = 16 * HG;             // rows of a tile per warp
  constexpr int NT = NTW / 8;
  constexpr int TG = kConsumerWarps / HG;  // token groups per CTA
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  PvSmem<KV, HG> sm(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.x / P.n_split, j = blockIdx.x % P.n_split;
  const int b = r / P.n_q, i = r % P.n_q;
  const int64_t seq_row0 = P.seq.start[b];
  const int64_t p = (int64_t)P.seq.len[b] - P.n_q + i;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(smem_u32(&sm.full[s]), 32);
      mbar_init(smem_u32(&sm.empty[s]), kConsumerWarps);
    }
    *sm.abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  griddep_launch_dependents();
  griddep_wait();   // idx / count come from the selection kernel
  int cnt = __ldcg(P.count + r);
  if (cnt < 1 || cnt > P.idx_stride) {
    if (threadIdx.x == 0) record_status(P.status, kStatusCheck);
    cnt = max(1, min(cnt, P.idx_stride));
  }
  const int e_begin = j * P.split_len;
  const int n_tiles = max(0, min(P.split_len, cnt - e_begin) + kTile - 1) / kTile;
  const __nv_bfloat16 *qg = reinterpret_cast<const __nv_bfloat16 *>(P.q) + (size_t)r * H * kHeadDim;
  WarpSoftmax st;
  st.init();
  const int hg = warp % HG, tg = warp / HG;
  if (warp == kConsumerWarps) {
    produce_gather<KV>(P, r, seq_row0, p, e_begin, cnt, sm.stages, sm.full, sm.empty, n_tiles,
                       sm.abort_flag);
  } else {
    const int tok0 = tg * NTW;
    const int c = lane & 3;
    uint32_t qa[8][4];
    float rowf[2];
    if (KV == kKvBf16) {
      load_q_frags_bf16_global(qg, hg * 16, qa);
      rowf[0] = rowf[1] = P.scale_log2;
    } else {
      float pw[2];
      load_q_frags_f16(qg, hg * 16, qa, pw);
      rowf[0] = P.scale_log2 * pw[0];
      rowf[1] = P.scale_log2 * pw[1];
    }
    for (int it = 0; it < n_tiles; ++it) {
      const int s = it % C::kStages;
      if (!mbar_wait(smem_u32(&sm.full[s]), (it / C::kStages) & 1)) {
        record_status(P.status, kStatusTimeout);
        *sm.abort_flag = 1;
      }
      if (*sm.abort_flag) break;
      const uint8_t *stg = sm.stages + s * C::kStageBytes;
      bool valid[NT][2];
      float colk[NT][2], colv[NT][2];
#pragma unroll
      for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int rr = tok0 + n * 8 + 2 * c + e;
          valid[n][e] = e_begin + it * kTile + rr < cnt;
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
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      st.l[h] += __shfl_xor_sync(0xffffffffu, st.l[h], 1);
      st.l[h] += __shfl_xor_sync(0xffffffffu, st.l[h], 2);
    }
    if (P.n_split > 1) {
      // this warp's partial: slot j * TG + tg of row r, its 16 heads
      const int g = lane >> 2;
      const int slot = j * TG + tg;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        float *row = P.part + (((size_t)r * P.n_split * TG + slot) * H + hg * 16 + g + 8 * hh) * kPartRow;
#pragma unroll
        for (int n = 0; n < 16; ++n)
#pragma unroll
          for (int e = 0; e < 2; ++e) row[kPartO + o_col<KV>(n, e, c)] = st.o[n][2 * hh + e] * st.vref;
        if (c == 0) {
          row[0] = st.m[hh];
          row[1] = st.l[hh];
        }
      }
    } else {
      // one CTA per row: merge the token groups through shared memory (stages are free once
      // every consumer has finished its tiles)
      named_barrier_sync(1, kConsumerWarps * 32);
      float *ws_o = reinterpret_cast<float *>(sm.stages);
      float *ws_ml = ws_o + kConsumerWarps * 16 * kHeadDim;
      const int g = lane >> 2;
#pragma unroll
      for (int n = 0; n < 16; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e)
          ws_o[(warp * 16 + g + (e >> 1) * 8) * kHeadDim + o_col<KV>(n, e & 1, c)] = st.o[n][e] * st.vref;
      if (c == 0) {
        ws_ml[(warp * 16 + g) * 2 + 0] = st.m[0];
        ws_ml[(warp * 16 + g) * 2 + 1] = st.l[0];
        ws_ml[(warp * 16 + g + 8) * 2 + 0] = st.m[1];
        ws_ml[(warp * 16 + g + 8) * 2 + 1] = st.l[1];
      }
    }
  }
  if (P.n_split > 1) return;
  __syncthreads();
  if (*sm.abort_flag) return;
  const float *ws_o = reinterpret_cast<const float *>(sm.stages);
  MergeTarget mt;
  mt.n_group = 1;
  mt.group_part = nullptr;
  mt.slot = 0;
  mt.out_f32 = P.out_f32;
  mt.out = P.out_f32 ? (void *)(reinterpret_cast<float *>(P.out) + (size_t)r * H * kHeadDim)
                     : (void *)(reinterpret_cast<__nv_bfloat16 *>(P.out) + (size_t)r * H * kHeadDim);
  mt.lse = nullptr;
  finish_cta<KV, HG>(ws_o, ws_o + kConsumerWarps * 16 * kHeadDim, mt);
}

// One CTA per (group, head): 8 slot lanes x 32 lanes of 4 output dims; float4 loads.
constexpr int kMergeThreads = 256;

__global__ void __launch_bounds__(kMergeThreads) merge_partials_kernel(const __grid_constant__ MergeParams P) {
  __shared__ float red_m[kMergeThreads / 32];
  __shared__ float red_l[8];
  __shared__ float4 red_o[8][32];
  const int grp = blockIdx.x / P.n_heads, h = blockIdx.x % P.n_heads;
  int s0, n;
  if (P.by_seq) {
    s0 = P.seq.item_begin[grp];
    n = P.seq.item_begin[grp + 1] - s0;
  } else {
    s0 = grp * P.n_fixed;
    n = P.n_fixed;
  }
  if (n <= 1) return;
  griddep_launch_dependents();
  griddep_wait();   // partials come from the previous kernel
  const int H = P.n_heads;
  const int sl = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float m = -INFINITY;
  for (int i = threadIdx.x; i < n; i += kMergeThreads)
    m = fmaxf(m, __ldcg(P.part + ((size_t)(s0 + i) * H + h) * kPartRow));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) red_m[sl] = m;
  __syncthreads();
  float M = red_m[0];
#pragma unroll
  for (int i = 1; i < kMergeThreads / 32; ++i) M = fmaxf(M, red_m[i]);
  float L = 0.f;
  float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
  for (int i = sl; i < n; i += 8) {
    const float *row = P.part + ((size_t)(s0 + i) * H + h) * kPartRow;
    const float mi = __ldcg(row);
    const float f = (mi == -INFINITY) ? 0.f : fast_exp2(mi - M);
    L += f * __ldcg(row + 1);
    const float4 o = __ldcg(reinterpret_cast<const float4 *>(row + kPartO) + lane);
    O.x += f * o.x;
    O.y += f * o.y;
    O.z += f * o.z;
    O.w += f * o.w;
  }
  red_o[sl][lane] = O;
  if (lane == 0) red_l[sl] = L;
  __syncthreads();
  if (sl == 0) {
    float Lt = 0.f;
    float4 Ot = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      Lt += red_l[k];
      Ot.x += red_o[k][lane].x;
      Ot.y += red_o[k][lane].y;
      Ot.z += red_o[k][lane].z;
      Ot.w += red_o[k][lane].w;
    }
    const float inv = 1.f / Lt;
    const size_t oi = ((size_t)grp * H + h) * kHeadDim + 4 * lane;
    if (P.out_f32) {
      *reinterpret_cast<float4 *>(reinterpret_cast<float *>(P.out) + oi) =
          make_float4(Ot.x * inv, Ot.y * inv, Ot.z * inv, Ot.w * inv);
    } else {
      __nv_bfloat16 *o = reinterpret_cast<__nv_bfloat16 *>(P.out) + oi;
      *reinterpret_cast<uint2 *>(o) = make_uint2(pack_bf16(Ot.x * inv, Ot.y * inv),
                                                 pack_bf16(Ot.z * inv, Ot.w * inv));
    }
    if (P.lse && lane == 0) P.lse[(size_t)grp * H + h] = (M + __log2f(Lt)) * kLn2;
  }
}

template <int KV, int HG>
constexpr size_t sparse_smem() {
  return PvSmem<KV, HG>::bytes();
}

template <int KV, int HG>
cudaError_t launch_sparse_t(const SparseParams &p, cudaStream_t s) {
  const size_t smem = sparse_smem<KV, HG>();
  auto kern = sparse_gather_kernel<KV, HG>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int grid = p.batch * p.n_q * p.n_split;
  e = launch_pdl(kern, grid, kThreads, smem, s, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_merge(const MergeParams &p, cudaStream_t s) {
  cudaError_t e = launch_pdl(merge_partials_kernel, p.n_groups * p.n_heads, kMergeThreads, 0, s, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
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
