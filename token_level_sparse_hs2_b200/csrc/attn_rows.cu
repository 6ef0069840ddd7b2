// attn_rows.cu -- the full-attention layer of a hybrid block for multi-token query chunks
// (a short action appended to a long context, or a causal prefill): every query row attends
// causally to its own prefix and gets its own importance scores.
//
// "HySparse2: How Xiaomi Split the Transformer to Fix Agent Prefill Costs", section "KV Reuse
// and Token-Level Sparse Selection": the full layer attends over the whole context and
// produces the indices the sparse layers reuse; each query token selects its own tokens.
// With MQA all H heads of all queries in a block read the same K/V tile, so a CTA stages each
// 64-row tile once (TMA) and multiplies it against 128 (query, head) rows.
//
// Pass 1: CTA = 128 rows = 128 / H queries x H heads; 8 consumer warps own 16 rows each. The
// causal prefix of the block is cut into n_chunks work items; chunks of one block are merged
// by the last CTA to finish (arrival counter), or written directly when n_chunks == 1.
// Pass 2: CTA = 8 queries, one per consumer warp (all H heads), over one chunk of the block's
// prefix; scores of different chunks are independent, so nothing is merged.
#include "attn_pipeline.cuh"
#include "internal.h"

namespace hs2 {

namespace {

constexpr int kRowWarps = 8;
constexpr int kRowThreads = (kRowWarps + 1) * 32;
constexpr int kBlockRows = 128;

struct BlockGeom {
  int b, blk_global, j;
  int i0, nqb;            // first query of the block, queries in the block
  int64_t row0;           // first cache row of the sequence
  int64_t pfirst;         // position of the block's first query
  int tile_begin, n_tiles;
};

// item -> (sequence, block, chunk); blocks of a sequence run latest-first (longest prefixes)
__device__ __forceinline__ BlockGeom block_geom(const RowsParams &P, int item) {
  BlockGeom g;
  g.blk_global = item / P.n_chunks;
  g.j = item % P.n_chunks;
  g.b = find_item_seq(P.seq, P.batch, g.blk_global);
  const int nblk = P.seq.item_begin[g.b + 1] - P.seq.item_begin[g.b];
  const int blk = nblk - 1 - (g.blk_global - P.seq.item_begin[g.b]);
  g.i0 = blk * P.q_per_block;
  g.nqb = min(P.q_per_block, P.n_q - g.i0);
  g.row0 = P.seq.start[g.b];
  g.pfirst = (int64_t)P.seq.len[g.b] - P.n_q + g.i0;
  const int64_t plast = g.pfirst + g.nqb - 1;
  const int tile0 = (int)(g.row0 / kTile);
  const int ntl = (int)((g.row0 + plast) / kTile) - tile0 + 1;
  const int ch = (ntl + P.n_chunks - 1) / P.n_chunks;
  g.tile_begin = tile0 + g.j * ch;
  g.n_tiles = max(0, min(ch, ntl - g.j * ch));
  return g;
}

template <int KV>
struct RowsSmem {
  using C = DecodeCfg<KV, 0>;
  uint8_t *stages, *q;
  uint64_t *full, *empty;
  volatile int *abort_flag;
  __device__ explicit RowsSmem(uint8_t *raw) {
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
    stages = base;
    q = stages + C::kStages * C::kStageBytes;
    full = reinterpret_cast<uint64_t *>(q + kBlockRows * 256);
    empty = full + C::kStages;
    abort_flag = reinterpret_cast<volatile int *>(empty + C::kStages);
  }
  static constexpr size_t bytes() {
    return 1024 + C::kStages * C::kStageBytes + kBlockRows * 256 + 2 * C::kStages * 8 + 16;
  }
};

template <int KV, int HG>
__global__ void __launch_bounds__(kRowThreads, 1)
    rows_pass1_kernel(const __grid_constant__ TensorMaps tm, const __grid_constant__ RowsParams P) {
  using C = DecodeCfg<KV, 0>;
  constexpr int H = 16 * HG;
  constexpr int PW = kPartRow;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  RowsSmem<KV> sm(smem_raw);
  __shared__ int s_last;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const BlockGeom G = block_geom(P, blockIdx.x);
  const int nrows = G.nqb * H;   // valid (query, head) rows of the block
  const __nv_bfloat16 *qblk = reinterpret_cast<const __nv_bfloat16 *>(P.q) +
                              ((size_t)G.b * P.n_q + G.i0) * H * kHeadDim;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(smem_u32(&sm.full[s]), C::kFullCount);
      mbar_init(smem_u32(&sm.empty[s]), kRowWarps);
    }
    *sm.abort_flag = 0;
    fence_barrier_init();
  }
  griddep_launch_dependents();
  griddep_wait();
  if (KV == kKvBf16) {
    for (int t = threadIdx.x; t < kBlockRows * 16; t += kRowThreads) {
      const int r = t >> 4, ch = t & 15;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (r < nrows) v = *reinterpret_cast<const uint4 *>(qblk + r * kHeadDim + ch * 8);
      *reinterpret_cast<uint4 *>(sm.q + tile_off(kBlockRows, r, ch * 8)) = v;
    }
  }
  __syncthreads();

  const int g = lane >> 2, c = lane & 3;
  const int qq = (warp * 16) / H, h0 = (warp * 16) % H;
  const bool wq = warp < kRowWarps && qq < G.nqb;
  WarpSoftmax st;
  st.init();
  if (warp == kRowWarps) {
    produce<KV, 0>(tm, P.k_scale, P.v_scale, P.kv_rows, sm.stages, sm.full, sm.empty,
                   G.tile_begin, G.n_tiles, sm.abort_flag, P.status);
  } else {
    const int64_t plim = G.row0 + G.pfirst + qq;   // last cache row this warp's query sees
    uint32_t qa[8][4];
    float rowf[2];
    if (KV == kKvBf16) {
      load_q_frags_bf16(smem_u32(sm.q), kBlockRows, warp * 16, qa);
      rowf[0] = rowf[1] = P.scale_log2;
    } else {
      float pw[2] = {1.f, 1.f};
      if (wq) load_q_frags_f16(qblk, warp * 16, qa, pw);
      rowf[0] = P.scale_log2 * pw[0];
      rowf[1] = P.scale_log2 * pw[1];
    }
    for (int it = 0; it < G.n_tiles; ++it) {
      const int s = it % C::kStages;
      if (!mbar_wait(smem_u32(&sm.full[s]), (it / C::kStages) & 1)) {
        record_status(P.status, kStatusTimeout);
        *sm.abort_flag = 1;
      }
      if (*sm.abort_flag) break;
      const uint8_t *stg = sm.stages + s * C::kStageBytes;
      const int64_t trow = (int64_t)(G.tile_begin + it) * kTile;
      if (wq && trow <= plim) {
        bool valid[8][2];
        float colk[8][2], colv[8][2];
#pragma unroll
        for (int n = 0; n < 8; ++n)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int rr = n * 8 + 2 * c + e;
            const int64_t row = trow + rr;
            valid[n][e] = row >= G.row0 && row <= plim;
            if (KV == kKvFp8) {
              const float *sc = reinterpret_cast<const float *>(stg + 2 * C::kKBytes);
              colk[n][e] = sc[rr];
              colv[n][e] = sc[kTile + rr];
            } else {
              colk[n][e] = 1.f;
              colv[n][e] = 1.f;
            }
          }
        float sacc[8][4];
        qk_tile<KV, 8>(qa, smem_u32(stg), 0, sacc);
        softmax_pv_tile<KV, 8>(st, sacc, rowf, colk, colv, valid, smem_u32(stg + C::kKBytes), 0);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&sm.empty[s]));
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      st.l[h] += __shfl_xor_sync(0xffffffffu, st.l[h], 1);
      st.l[h] += __shfl_xor_sync(0xffffffffu, st.l[h], 2);
    }
  }
  __syncthreads();
  if (*sm.abort_flag) return;

  if (P.n_chunks == 1) {
    if (wq) {
      const size_t orow0 = ((size_t)G.b * P.n_q + G.i0 + qq) * H + h0;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const float inv = st.vref / st.l[hh];
        const size_t orow = orow0 + g + 8 * hh;
#pragma unroll
        for (int n = 0; n < 16; ++n)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const size_t oi = orow * kHeadDim + o_col<KV>(n, e, c);
            const float val = st.o[n][2 * hh + e] * inv;
            if (P.out_f32) reinterpret_cast<float *>(P.out)[oi] = val;
            else reinterpret_cast<__nv_bfloat16 *>(P.out)[oi] = __float2bfloat16_rn(val);
          }
        if (c == 0) P.lse[orow] = (st.m[hh] + __log2f(st.l[hh])) * kLn2;
      }
    }
    return;
  }
  // partial of this chunk: rows [warp*16, warp*16+16) of the block
  float *part = P.part + ((size_t)G.blk_global * P.n_chunks + G.j) * kBlockRows * PW;
  if (warp < kRowWarps) {
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      float *pr = part + (size_t)(warp * 16 + g + 8 * hh) * PW;
#pragma unroll
      for (int n = 0; n < 16; ++n)
#pragma unroll
        for (int e = 0; e < 2; ++e) pr[kPartO + o_col<KV>(n, e, c)] = st.o[n][2 * hh + e] * st.vref;
      if (c == 0) {
        pr[0] = st.m[hh];
        pr[1] = st.l[hh];
      }
    }
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const int prev = atomicAdd(&P.counter[G.blk_global], 1);
    s_last = (prev == P.n_chunks - 1);
    if (s_last) P.counter[G.blk_global] = 0;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const float *gp = P.part + (size_t)G.blk_global * P.n_chunks * kBlockRows * PW;
  for (int t = threadIdx.x; t < nrows * kHeadDim; t += kRowThreads) {
    const int r = t / kHeadDim, d = t % kHeadDim;
    float M = -INFINITY;
    for (int i = 0; i < P.n_chunks; ++i) M = fmaxf(M, __ldcg(gp + ((size_t)i * kBlockRows + r) * PW));
    float L = 0.f, O = 0.f;
    for (int i = 0; i < P.n_chunks; ++i) {
      const float *pp = gp + ((size_t)i * kBlockRows + r) * PW;
      const float m = __ldcg(pp);
      const float f = (m == -INFINITY) ? 0.f : fast_exp2(m - M);
      L += f * __ldcg(pp + 1);
      O += f * __ldcg(pp + kPartO + d);
    }
    const size_t orow = ((size_t)G.b * P.n_q + G.i0) * H + r;
    const float val = O / L;
    if (P.out_f32) reinterpret_cast<float *>(P.out)[orow * kHeadDim + d] = val;
    else reinterpret_cast<__nv_bfloat16 *>(P.out)[orow * kHeadDim + d] = __float2bfloat16_rn(val);
    if (d == 0) P.lse[orow] = (M + __log2f(L)) * kLn2;
  }
}

template <int KV>
struct RowsSmem2 {
  using C = DecodeCfg<KV, 1>;
  uint8_t *stages;
  uint64_t *full, *empty;
  volatile int *abort_flag;
  __device__ explicit RowsSmem2(uint8_t *raw) {
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
    stages = base;
    full = reinterpret_cast<uint64_t *>(stages + C::kStages * C::kStageBytes);
    empty = full + C::kStages;
    abort_flag = reinterpret_cast<volatile int *>(empty + C::kStages);
  }
  static constexpr size_t bytes() { return 1024 + C::kStages * C::kStageBytes + 2 * C::kStages * 8 + 16; }
};

template <int KV, int HG>
__global__ void __launch_bounds__(kRowThreads, 1)
    rows_pass2_kernel(const __grid_constant__ TensorMaps tm, const __grid_constant__ RowsParams P) {
  using C = DecodeCfg<KV, 1>;
  constexpr int H = 16 * HG;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  RowsSmem2<KV> sm(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const BlockGeom G = block_geom(P, blockIdx.x);
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(smem_u32(&sm.full[s]), C::kFullCount);
      mbar_init(smem_u32(&sm.empty[s]), kRowWarps);
    }
    *sm.abort_flag = 0;
    fence_barrier_init();
  }
  griddep_launch_dependents();
  griddep_wait();   // lse comes from pass 1
  __syncthreads();
  if (warp == kRowWarps) {
    produce<KV, 1>(tm, P.k_scale, P.v_scale, P.kv_rows, sm.stages, sm.full, sm.empty,
                   G.tile_begin, G.n_tiles, sm.abort_flag, P.status);
    return;
  }
  const int g = lane >> 2, c = lane & 3;
  const bool wq = warp < G.nqb;
  const int i = G.i0 + warp;
  const size_t qrow = (size_t)G.b * P.n_q + i;
  const int64_t plim = G.row0 + G.pfirst + warp;
  uint32_t qa[HG][8][4];
  float rowf[HG][2], lse2[HG][2];
  if (wq) {
    const __nv_bfloat16 *qg = reinterpret_cast<const __nv_bfloat16 *>(P.q) + qrow * H * kHeadDim;
#pragma unroll
    for (int mt = 0; mt < HG; ++mt) {
      if (KV == kKvBf16) {
        load_q_frags_bf16_global(qg, mt * 16, qa[mt]);
        rowf[mt][0] = rowf[mt][1] = P.scale_log2;
      } else {
        float pw[2];
        load_q_frags_f16(qg, mt * 16, qa[mt], pw);
        rowf[mt][0] = P.scale_log2 * pw[0];
        rowf[mt][1] = P.scale_log2 * pw[1];
      }
      lse2[mt][0] = P.lse[qrow * H + mt * 16 + g] * kLog2e;
      lse2[mt][1] = P.lse[qrow * H + mt * 16 + g + 8] * kLog2e;
    }
  }
  float *srow = P.scores + qrow * P.score_stride;
  for (int it = 0; it < G.n_tiles; ++it) {
    const int s = it % C::kStages;
    if (!mbar_wait(smem_u32(&sm.full[s]), (it / C::kStages) & 1)) {
      record_status(P.status, kStatusTimeout);
      *sm.abort_flag = 1;
    }
    if (*sm.abort_flag) break;
    const uint8_t *stg = sm.stages + s * C::kStageBytes;
    const int64_t trow = (int64_t)(G.tile_begin + it) * kTile;
    if (wq && trow <= plim) {
      float colk[8][2];
#pragma unroll
      for (int n = 0; n < 8; ++n)
#pragma unroll
        for (int e = 0; e < 2; ++e)
          colk[n][e] = (KV == kKvFp8) ? reinterpret_cast<const float *>(stg + C::kKBytes)[n * 8 + 2 * c + e] : 1.f;
      float cs[8][2];
#pragma unroll
      for (int n = 0; n < 8; ++n) cs[n][0] = cs[n][1] = 0.f;
#pragma unroll
      for (int mt = 0; mt < HG; ++mt) {
        float sacc[8][4];
        qk_tile<KV, 8>(qa[mt], smem_u32(stg), 0, sacc);
#pragma unroll
        for (int n = 0; n < 8; ++n)
#pragma unroll
          for (int e = 0; e < 4; ++e)
            cs[n][e & 1] += fast_exp2(sacc[n][e] * rowf[mt][e >> 1] * colk[n][e & 1] - lse2[mt][e >> 1]);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&sm.empty[s]));
#pragma unroll
      for (int n = 0; n < 8; ++n)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          float v = cs[n][e];
          v += __shfl_xor_sync(0xffffffffu, v, 4);
          v += __shfl_xor_sync(0xffffffffu, v, 8);
          v += __shfl_xor_sync(0xffffffffu, v, 16);
          cs[n][e] = v;
        }
      if (g == 0) {
#pragma unroll
        for (int n = 0; n < 8; ++n)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int64_t row = trow + n * 8 + 2 * c + e;
            if (row >= G.row0 && row <= plim) srow[row - G.row0] = cs[n][e];
          }
      }
    } else {
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&sm.empty[s]));
    }
  }
}

template <int KV, int HG>
cudaError_t launch_rows_t(int pass, const TensorMaps &tm, const RowsParams &p, cudaStream_t s) {
  if (pass == 0) {
    constexpr size_t smem = RowsSmem<KV>::bytes();
    static_assert(smem <= 227 * 1024, "rows pass 1 shared memory");
    auto kern = rows_pass1_kernel<KV, HG>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = launch_pdl(kern, p.n_items, kRowThreads, smem, s, tm, p);
    if (e != cudaSuccess) return e;
  } else {
    constexpr size_t smem = RowsSmem2<KV>::bytes();
    auto kern = rows_pass2_kernel<KV, HG>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = launch_pdl(kern, p.n_items, kRowThreads, smem, s, tm, p);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_rows_pass(int pass, int kv_dtype, const TensorMaps &tm, const RowsParams &p,
                             cudaStream_t s) {
  const int hg = p.n_heads / 16;
  if (kv_dtype == HS2_KV_BF16) {
    if (hg == 1) return launch_rows_t<kKvBf16, 1>(pass, tm, p, s);
    if (hg == 2) return launch_rows_t<kKvBf16, 2>(pass, tm, p, s);
  } else {
    if (hg == 1) return launch_rows_t<kKvFp8, 1>(pass, tm, p, s);
    if (hg == 2) return launch_rows_t<kKvFp8, 2>(pass, tm, p, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace hs2
