// attn_sparse.cu -- a sparse-attention layer of a hybrid block (KV Reuse): each query row's
// own queries attend only to the cache rows its full-attention layer selected, and every
// gathered K/V row serves all query heads of a 16-head group.
//
// "HySparse2: How Xiaomi Split the Transformer to Fix Agent Prefill Costs", section "KV Reuse
// and Token-Level Sparse Selection": the sparse layers take the full layer's indices and cache
// as they are; the forced-window tokens are ordinary rows of that cache.
//
// One CTA per (query row, split of the selected list): every warp gathers its share of each
// 64-row tile (16-byte cp.async into the swizzled tile layout, two stages) and runs the
// tensor-core online softmax on 16 heads x 16 rows of it. The token groups of a CTA merge in
// shared memory; the splits of a row form one thread-block cluster and merge through
// distributed shared memory: each CTA pushes its partial of head h into the CTA that finishes
// head h (one cluster barrier, then local reads), so no partial result goes through HBM.
// merge_partials_kernel (one CTA per output group and head) serves the decode full layer.
#include <algorithm>
#include <cooperative_groups.h>

#include "attn_pipeline.cuh"
#include "internal.h"

namespace hs2 {

namespace {

// One CTA per (query row, split of its selected list), no dedicated producer: the 4 * HG
// warps each gather 64 / (4 * HG) rows of every tile with 16-byte cp.async (so the copies are
// issued from all four SM sub-partitions at once) and each computes 16 heads x 16 rows of it.
constexpr int kPreTiles = 24;   // tiles whose indices are staged in shared memory up front

template <int KV, int HG>
struct SpCfg {
  static constexpr int kWarps = 4 * HG;
  static constexpr int kThreads = kWarps * 32;
  static constexpr int kRowsPerWarp = kTile / kWarps;
  static constexpr int kKBytes = (KV == kKvBf16) ? 2 * kBoxBytes : kBoxBytes;
  static constexpr int kStageBytes = (2 * kKBytes + (KV == kKvFp8 ? 512 : 0) + 1023) / 1024 * 1024;
  static constexpr int kStages = 2;
  // the stage ring doubles as the warp-merge area ([warp][16][128] outputs, [warp][16][2]
  // max / denominator) followed by the CTA's merged partial ([H][kPartRow]) for the cluster
  static constexpr size_t kMergeBytes = (size_t)kWarps * 16 * (o_stride<KV>() + 2) * 4 +
                                        (size_t)16 * HG * (kPartRow + 2) * 4;
  static constexpr size_t kRegion = ((size_t)kStages * kStageBytes > kMergeBytes)
                                        ? (size_t)kStages * kStageBytes : (kMergeBytes + 1023) / 1024 * 1024;
  static constexpr size_t kSmem = 1024 + kRegion + 2 * kStages * 8 + 16 + kPreTiles * kTile * 4;
  // split rows (a thread-block cluster per row): every CTA of the cluster pushes its (M, L, O) of
  // head h into the shared memory of CTA h % n_tsplit, at [h / n_tsplit][pusher][kPartRow]
  static constexpr size_t kRecvBytes = (size_t)(16 * HG + 15) * kPartRow * 4;
  static constexpr size_t kSmemSplit = kSmem + kRecvBytes;
};

// This warp's share of tile `it`: rows [w * RPW, (w+1) * RPW), cp.async into stage `st`, then
// one arrival per lane on `bar` once the copies land (entries past the list are zero-filled).
// Lane l owns one 16-byte column of the rows (bf16: chunk l % 16 of K (l < 16) or V; e4m3: chunk
// l % 8 of K or V of every other row), so a copy costs a shuffle of the row's position, one
// address multiply-add and the swizzled destination. Lanes < RPW hold the rows' positions.
template <int KV, int HG>
__device__ __forceinline__ void gather_rows(const SparseParams &P, int64_t seq_row0, int64_t p,
                                            int e_first, int cnt, int warp, uint8_t *st,
                                            uint32_t bar, int32_t pos_lane, bool &bad) {
  using C = SpCfg<KV, HG>;
  const int lane = threadIdx.x & 31;
  constexpr int RPW = C::kRowsPerWarp;
  int32_t mypos = -1;   // validated position of this lane's row, -1 past the list
  if (lane < RPW && e_first + warp * RPW + lane < cnt) {
    mypos = pos_lane;
    if (pos_lane < 0 || pos_lane > p) {
      bad = true;
      mypos = 0;
    }
  }
  if (KV == kKvBf16) {
    const int kv = lane >> 4, ch = lane & 15;
    const uint8_t *src0 = reinterpret_cast<const uint8_t *>(kv ? P.v : P.k) + seq_row0 * 256 + ch * 16;
    uint8_t *dst0 = st + kv * C::kKBytes + (ch >> 3) * (kTile * 128);
#pragma unroll
    for (int rl = 0; rl < RPW; ++rl) {
      const int rr = warp * RPW + rl;
      const int32_t pos = __shfl_sync(0xffffffffu, mypos, rl);
      cp_async_16(smem_u32(dst0 + rr * 128 + (((ch & 7) ^ (rr & 7)) << 4)),
                  src0 + (int64_t)max(pos, 0) * 256, pos >= 0 ? 16u : 0u);
    }
  } else {
    const int sub = lane >> 4, kv = (lane >> 3) & 1, ch = lane & 7;
    const uint8_t *src0 = reinterpret_cast<const uint8_t *>(kv ? P.v : P.k) + seq_row0 * 128 + ch * 16;
    uint8_t *dst0 = st + kv * C::kKBytes;
#pragma unroll
    for (int rl = 0; rl < RPW; rl += 2) {
      const int r2 = rl + sub, rr = warp * RPW + r2;
      const int32_t pos = __shfl_sync(0xffffffffu, mypos, r2);
      cp_async_16(smem_u32(dst0 + fp8_off(rr, ch * 16)), src0 + (int64_t)max(pos, 0) * 128,
                  pos >= 0 ? 16u : 0u);
    }
    if (lane < RPW) {
      const int rr = warp * RPW + lane;
      const int64_t row = seq_row0 + max(mypos, 0);
      uint8_t *sc = st + 2 * C::kKBytes;
      cp_async_4(smem_u32(sc + rr * 4), P.k_scale + row, mypos >= 0 ? 4u : 0u);
      cp_async_4(smem_u32(sc + (kTile + rr) * 4), P.v_scale + row, mypos >= 0 ? 4u : 0u);
    }
  }
  cp_async_mbar_arrive(bar);
}

template <int KV, int HG>
__global__ void __launch_bounds__(SpCfg<KV, HG>::kThreads, 2) sparse_gather_kernel(const __grid_constant__ SparseParams P) {
  using C = SpCfg<KV, HG>;
  constexpr int H = 16 * HG;
  constexpr int TG = 4;   // token groups: warp w covers rows [16 * (w / HG), +16) of a tile
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *stages = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(stages + C::kRegion);
  uint64_t *empty = full + C::kStages;
  volatile int *abort_flag = reinterpret_cast<volatile int *>(empty + C::kStages);
  int32_t *s_idx = const_cast<int32_t *>(reinterpret_cast<volatile int32_t *>(abort_flag + 4));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // CTA (row, head group, split): the row's head groups are separate clusters of n_tsplit CTAs
  const int rg = blockIdx.x / P.n_tsplit, ts = blockIdx.x % P.n_tsplit;
  const int r = rg / P.head_groups;
  const int hrow0 = r * P.n_heads + (rg % P.head_groups) * H;   // first (row, head) of this CTA
  const int b = r / P.n_q, i = r % P.n_q;
  const int64_t seq_row0 = P.seq.start[b];
  const int64_t p = (int64_t)P.seq.len[b] - P.n_q + i;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(smem_u32(&full[s]), C::kThreads);
      mbar_init(smem_u32(&empty[s]), C::kWarps);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  // split rows: announce this CTA to its cluster now; the matching wait comes just before the
  // first push into another CTA's shared memory, long after every CTA has started
  if (P.n_tsplit > 1) asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
  // idx / count come from the selection kernel. When it ran two or more launches earlier
  // (idx_ready: sparse layers after the first), the index staging and the first gathers are
  // issued before the wait for the previous layer, overlapping its tail. Every layer lets the
  // next one start only after its own wait has returned, so by then the selection kernel has
  // finished.
  if (!P.idx_ready) {
    griddep_wait();
    griddep_launch_dependents();
  }
  const int e_begin = ts * P.split_len;
  // the split's first kPreTiles tiles of row indices, staged in shared memory (coalesced)
  const int32_t *idx = P.idx + (size_t)r * P.idx_stride;
  const int n_pre = min(min(P.split_len, kPreTiles * kTile), P.idx_stride - e_begin);
  for (int t = threadIdx.x; t < n_pre; t += C::kThreads) s_idx[t] = __ldcg(idx + e_begin + t);
  int cnt = __ldcg(P.count + r);
  const int cmin = P.allow_empty ? 0 : 1;
  if (cnt < cmin || cnt > P.idx_stride) {
    if (threadIdx.x == 0) record_status(P.status, kStatusCheck);
    cnt = max(cmin, min(cnt, P.idx_stride));
  }
  const int n_tiles = max(0, min(P.split_len, cnt - e_begin) + kTile - 1) / kTile;
  __syncthreads();   // s_idx
  auto pos_of = [&](int it) -> int32_t {
    const int k = it * kTile + warp * C::kRowsPerWarp + lane;   // entry within the split
    if (lane >= C::kRowsPerWarp || e_begin + k >= cnt) return 0;
    return (k < n_pre) ? s_idx[k] : __ldcg(idx + e_begin + k);
  };
  bool bad = false;
  for (int it = 0; it < min(n_tiles, C::kStages); ++it)
    gather_rows<KV, HG>(P, seq_row0, p, e_begin + it * kTile, cnt, warp, stages + it * C::kStageBytes,
                        smem_u32(&full[it]), pos_of(it), bad);
  if (P.idx_ready) {
    griddep_wait();   // the queries may come from the previous layer
    griddep_launch_dependents();
  }

  const int hg = warp % HG, tg = warp / HG;
  const int tok0 = tg * 16;
  const int c = lane & 3, g = lane >> 2;
  const __nv_bfloat16 *qg = reinterpret_cast<const __nv_bfloat16 *>(P.q) + (size_t)hrow0 * kHeadDim;
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
  WarpSoftmax st;
  st.init();
  for (int it = 0; it < n_tiles; ++it) {
    const int s = it % C::kStages;
    if (!mbar_wait(smem_u32(&full[s]), (it / C::kStages) & 1)) {
      record_status(P.status, kStatusTimeout);
      *abort_flag = 1;
    }
    if (*abort_flag) break;
    const uint8_t *stg = stages + s * C::kStageBytes;
    bool valid[2][2];
    float colk[2][2], colv[2][2];
#pragma unroll
    for (int n = 0; n < 2; ++n)
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
    float sacc[2][4];
    qk_tile<KV, 2>(qa, smem_u32(stg), tok0, sacc);
    softmax_pv_tile<KV, 2>(st, sacc, rowf, colk, colv, valid, smem_u32(stg + C::kKBytes), tok0);
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&empty[s]));
    const int nxt = it + C::kStages;
    if (nxt < n_tiles) {   // refill this stage once every warp is done with it
      if (!mbar_wait(smem_u32(&empty[s]), (it / C::kStages) & 1)) {
        record_status(P.status, kStatusTimeout);
        *abort_flag = 1;
        break;
      }
      gather_rows<KV, HG>(P, seq_row0, p, e_begin + nxt * kTile, cnt, warp, stages + s * C::kStageBytes,
                          smem_u32(&full[s]), pos_of(nxt), bad);
    }
  }
  if (bad) record_status(P.status, kStatusCheck);
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    st.l[h] += __shfl_xor_sync(0xffffffffu, st.l[h], 1);
    st.l[h] += __shfl_xor_sync(0xffffffffu, st.l[h], 2);
  }
  // merge the token groups through shared memory (stages are free once every warp is past its
  // last tile). A CTA that gave up on a wait still takes every barrier below, so that the
  // cluster's other CTAs never wait for it; its status word already carries the error.
  __syncthreads();
  constexpr int OS = o_stride<KV>();
  float *ws_o = reinterpret_cast<float *>(stages);      // [warp][16][OS]
  float *ws_ml = ws_o + C::kWarps * 16 * OS;            // [warp][16][2]
  float *cpart = ws_ml + C::kWarps * 16 * 2;            // [H][kPartRow]: this CTA's (M, L, O)
  float *hml = cpart + H * kPartRow;                    // [H][2]: (M, L) of each head
  if (c == 0) {
    ws_ml[(warp * 16 + g) * 2 + 0] = st.m[0];
    ws_ml[(warp * 16 + g) * 2 + 1] = st.l[0];
    ws_ml[(warp * 16 + g + 8) * 2 + 0] = st.m[1];
    ws_ml[(warp * 16 + g + 8) * 2 + 1] = st.l[1];
  }
  __syncthreads();
  {  // each warp stores its output rows rescaled to the common maximum of their head
    float f[2];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int rw = g + 8 * hh;
      float M = -INFINITY;
#pragma unroll
      for (int k = 0; k < TG; ++k) M = fmaxf(M, ws_ml[((k * HG + hg) * 16 + rw) * 2]);
      f[hh] = (st.m[hh] == -INFINITY) ? 0.f : fast_exp2(st.m[hh] - M) * st.vref;
    }
    o_to_smem<KV>(ws_o + warp * 16 * OS, st.o, f, true);
    if (warp == 0) {   // (M, L) per head
      const int h = lane, hgh = h >> 4, rh = h & 15;
      if (h < H) {
        float M = -INFINITY, L = 0.f;
#pragma unroll
        for (int k = 0; k < TG; ++k) M = fmaxf(M, ws_ml[((k * HG + hgh) * 16 + rh) * 2]);
#pragma unroll
        for (int k = 0; k < TG; ++k) {
          const float m = ws_ml[((k * HG + hgh) * 16 + rh) * 2];
          if (m != -INFINITY) L += fast_exp2(m - M) * ws_ml[((k * HG + hgh) * 16 + rh) * 2 + 1];
        }
        hml[2 * h] = M;
        hml[2 * h + 1] = L;
      }
    }
  }
  __syncthreads();
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  const int ns = P.n_tsplit;
  float *recv = reinterpret_cast<float *>(smem_raw + C::kSmem);
  if (ns > 1) asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
  for (int t = threadIdx.x; t < H * kHeadDim / 4; t += C::kThreads) {   // sum of the token groups
    const int h = t / (kHeadDim / 4), d4 = t % (kHeadDim / 4);
    const int hgh = h >> 4, rh = h & 15;
    float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int k = 0; k < TG; ++k) {
      const float4 o = reinterpret_cast<const float4 *>(ws_o + ((k * HG + hgh) * 16 + rh) * OS)[d4];
      O.x += o.x;
      O.y += o.y;
      O.z += o.z;
      O.w += o.w;
    }
    if (P.n_tsplit == 1) {
      const float Lh = hml[2 * h + 1];
      const float inv = Lh > 0.f ? 1.f / Lh : 0.f;   // 0: a shard that holds none of the selection
      if (P.lse_out && d4 == 0)
        P.lse_out[(size_t)hrow0 + h] = Lh > 0.f ? (hml[2 * h] + __log2f(Lh)) * kLn2 : -INFINITY;
      const size_t oi = ((size_t)hrow0 + h) * kHeadDim + 4 * d4;
      if (P.out_f32) {
        *reinterpret_cast<float4 *>(reinterpret_cast<float *>(P.out) + oi) =
            make_float4(O.x * inv, O.y * inv, O.z * inv, O.w * inv);
      } else {
        *reinterpret_cast<uint2 *>(reinterpret_cast<__nv_bfloat16 *>(P.out) + oi) =
            make_uint2(pack_bf16(O.x * inv, O.y * inv), pack_bf16(O.z * inv, O.w * inv));
      }
    } else {   // push into the owner of head h
      float *row = cluster.map_shared_rank(recv, h % ns) + ((h / ns) * ns + ts) * kPartRow;
      reinterpret_cast<float4 *>(row + kPartO)[d4] = O;
      if (d4 == 0) {
        row[0] = hml[2 * h];
        row[1] = hml[2 * h + 1];
      }
    }
  }
  if (ns == 1) return;
  // cluster merge: CTA `ts` of the row finishes heads ts, ts + n_tsplit, ..., one warp per head,
  // from the (M, L, O) every CTA pushed into its shared memory. After this barrier no CTA touches
  // another's shared memory, so each may leave when done.
  cluster.sync();
  for (int h = ts + ns * warp; h < H; h += ns * C::kWarps) {
    const float *part = recv + (h / ns) * ns * kPartRow;   // [pusher][kPartRow]
    float mj = -INFINITY, lj = 0.f;
    if (lane < ns) {
      mj = part[lane * kPartRow];
      lj = part[lane * kPartRow + 1];
    }
    float M = mj;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    const float fj = (mj == -INFINITY) ? 0.f : fast_exp2(mj - M);
    float L = fj * lj;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
    float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < ns; ++j) {
      const float f = __shfl_sync(0xffffffffu, fj, j);
      const float4 o = reinterpret_cast<const float4 *>(part + j * kPartRow + kPartO)[lane];
      O.x += f * o.x;
      O.y += f * o.y;
      O.z += f * o.z;
      O.w += f * o.w;
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
    if (P.lse_out && lane == 0)
      P.lse_out[(size_t)hrow0 + h] = L > 0.f ? (M + __log2f(L)) * kLn2 : -INFINITY;
    const size_t oi = ((size_t)hrow0 + h) * kHeadDim + 4 * lane;
    if (P.out_f32) {
      *reinterpret_cast<float4 *>(reinterpret_cast<float *>(P.out) + oi) =
          make_float4(O.x * inv, O.y * inv, O.z * inv, O.w * inv);
    } else {
      *reinterpret_cast<uint2 *>(reinterpret_cast<__nv_bfloat16 *>(P.out) + oi) =
          make_uint2(pack_bf16(O.x * inv, O.y * inv), pack_bf16(O.z * inv, O.w * inv));
    }
  }
}

// CTAs per (group, head, part of head_dim): slot lanes x lanes of 4 output dims, float4 loads,
// so a group with many slots still spreads over several CTAs per head.
constexpr int kMergeThreads = 256;

// CHUNKS CTAs per (group, head), each owning 128 / CHUNKS output dims: 4 for a few partials per
// group (fewer CTAs), 8 for many (more slot lanes, shorter chains of loads per lane).
template <int CHUNKS>
__global__ void __launch_bounds__(kMergeThreads) merge_partials_kernel(const __grid_constant__ MergeParams P) {
  constexpr int kMergeChunks = CHUNKS;
  constexpr int kMergeQuads = 128 / 4 / kMergeChunks;        // float4 columns per CTA
  constexpr int kMergeLanes = kMergeThreads / kMergeQuads;   // slot lanes
  __shared__ float red_m[kMergeThreads / 32];
  __shared__ float red_l[kMergeLanes];
  __shared__ float4 red_o[kMergeLanes][kMergeQuads];
  const int ch = blockIdx.x % kMergeChunks;
  const int grp = blockIdx.x / kMergeChunks / P.n_heads, h = blockIdx.x / kMergeChunks % P.n_heads;
  int s0, n;
  if (P.by_seq) {
    s0 = P.seq.item_begin[grp];
    n = P.seq.item_begin[grp + 1] - s0;
  } else {
    s0 = grp * P.n_fixed;
    n = P.n_fixed;
  }
  griddep_launch_dependents();
  griddep_wait();   // partials come from the previous kernel
  const int H = P.n_heads;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float m = -INFINITY;
  for (int i = threadIdx.x; i < n; i += kMergeThreads)
    m = fmaxf(m, __ldcg(P.part + ((size_t)(s0 + i) * H + h) * kPartRow));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) red_m[w] = m;
  __syncthreads();
  float M = red_m[0];
#pragma unroll
  for (int i = 1; i < kMergeThreads / 32; ++i) M = fmaxf(M, red_m[i]);
  const int sl = threadIdx.x / kMergeQuads, dq = threadIdx.x % kMergeQuads;   // slot lane, dim quad
  float L = 0.f;
  float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 2
  for (int i = sl; i < n; i += kMergeLanes) {
    const float *row = P.part + ((size_t)(s0 + i) * H + h) * kPartRow;
    const float mi = __ldcg(row);
    const float f = (mi == -INFINITY) ? 0.f : fast_exp2(mi - M);
    L += f * __ldcg(row + 1);
    const float4 o = __ldcg(reinterpret_cast<const float4 *>(row + kPartO) + ch * kMergeQuads + dq);
    O.x += f * o.x;
    O.y += f * o.y;
    O.z += f * o.z;
    O.w += f * o.w;
  }
  red_o[sl][dq] = O;
  if (dq == 0) red_l[sl] = L;
  __syncthreads();
  if (threadIdx.x < kMergeQuads) {
    float Lt = 0.f;
    float4 Ot = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
    for (int k = 0; k < kMergeLanes; ++k) {
      Lt += red_l[k];
      Ot.x += red_o[k][threadIdx.x].x;
      Ot.y += red_o[k][threadIdx.x].y;
      Ot.z += red_o[k][threadIdx.x].z;
      Ot.w += red_o[k][threadIdx.x].w;
    }
    const float inv = 1.f / Lt;
    const size_t oi = ((size_t)grp * H + h) * kHeadDim + ch * (4 * kMergeQuads) + 4 * threadIdx.x;
    if (P.out_f32) {
      *reinterpret_cast<float4 *>(reinterpret_cast<float *>(P.out) + oi) =
          make_float4(Ot.x * inv, Ot.y * inv, Ot.z * inv, Ot.w * inv);
    } else {
      __nv_bfloat16 *o = reinterpret_cast<__nv_bfloat16 *>(P.out) + oi;
      *reinterpret_cast<uint2 *>(o) = make_uint2(pack_bf16(Ot.x * inv, Ot.y * inv),
                                                 pack_bf16(Ot.z * inv, Ot.w * inv));
    }
    if (P.lse && ch == 0 && threadIdx.x == 0) P.lse[(size_t)grp * H + h] = (M + __log2f(Lt)) * kLn2;
  }
}

template <int KV, int HG>
cudaError_t launch_sparse_t(const SparseParams &p, cudaStream_t s) {
  using C = SpCfg<KV, HG>;
  static_assert(C::kSmemSplit <= 227 * 1024, "sparse shared memory");
  auto kern = sparse_gather_kernel<KV, HG>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::kSmemSplit);
  if (e != cudaSuccess) return e;
  const int grid = p.batch * p.n_q * p.head_groups * p.n_tsplit;
  if (p.n_tsplit == 1) {
    e = launch_pdl(kern, grid, C::kThreads, C::kSmem, s, p);
  } else {
    if (p.n_tsplit > 8) {
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
      if (e != cudaSuccess) return e;
    }
    e = launch_pdl_cluster(kern, grid, C::kThreads, C::kSmemSplit, p.n_tsplit, s, p);
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// Largest cluster (<= 16) of which at least one can be resident at a time.
template <int KV, int HG>
int max_cluster_t() {
  using C = SpCfg<KV, HG>;
  auto kern = sparse_gather_kernel<KV, HG>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::kSmemSplit) != cudaSuccess ||
      cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) {
    cudaGetLastError();
    return 1;
  }
  for (int cs = 16; cs > 1; --cs) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(cs);
    cfg.blockDim = dim3(C::kThreads);
    cfg.dynamicSmemBytes = C::kSmemSplit;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cs;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) == cudaSuccess && n > 0) return cs;
    cudaGetLastError();
  }
  return 1;
}

}  // namespace


cudaError_t launch_merge(const MergeParams &p, cudaStream_t s) {
  int most = p.n_fixed;   // partials of the largest group
  if (p.by_seq)
    for (int g = 0; g < p.n_groups; ++g) most = std::max(most, p.seq.item_begin[g + 1] - p.seq.item_begin[g]);
  cudaError_t e = most > 64
      ? launch_pdl(merge_partials_kernel<8>, p.n_groups * p.n_heads * 8, kMergeThreads, 0, s, p)
      : launch_pdl(merge_partials_kernel<4>, p.n_groups * p.n_heads * 4, kMergeThreads, 0, s, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

int sparse_max_cluster(int kv_dtype, int n_heads) {
  const int hg = n_heads / 16;
  if (kv_dtype == HS2_KV_BF16) return hg == 1 ? max_cluster_t<kKvBf16, 1>() : max_cluster_t<kKvBf16, 2>();
  return hg == 1 ? max_cluster_t<kKvFp8, 1>() : max_cluster_t<kKvFp8, 2>();
}

cudaError_t launch_sparse(int kv_dtype, const SparseParams &p, cudaStream_t s) {
  const int hg = p.n_heads / 16 / p.head_groups;   // 16-head groups per CTA
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
