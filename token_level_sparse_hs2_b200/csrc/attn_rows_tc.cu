// attn_rows_tc.cu -- importance scores (score pass 2) of the full-attention layer for query
// chunks and prefill on the fifth-generation tensor cores (tcgen05, accumulators in TMEM).
//
// "HySparse2: How Xiaomi Split the Transformer to Fix Agent Prefill Costs", section "KV Reuse
// and Token-Level Sparse Selection": the full layer produces, for every query token, the
// scores from which that token's sparse selection is taken. The score of cache token t for
// a query at position p >= t is the softmax probability of t summed over the H query heads,
// s[t] = sum_h exp(c q_h . k_t - lse_h), with lse_h from the output pass.
//
// One CTA per (block of 256 / H queries, chunk of the block's causal prefix). For every
// 128-row K tile the product D = K_tile . Q_block^T - lse / (c log2 e) (M = 128 tokens,
// N = 256 (query, head) columns) is one chain of 9 tcgen05.mma into a TMEM accumulator: 8
// steps over head_dim, and a ninth whose A operand is a constant block with ones in its first
// three columns and whose B operand holds -lse_h log2 e / (c log2 e) of every column split
// into three bf16 terms (24 significant bits), so the accumulator already carries the
// log-sum-exp. Two accumulators alternate, so the tensor cores fill one while the epilogue
// drains the other:
//   warp 9      TMA producer: K tiles (two 64-row halves x two 64-dim boxes) into 3 stages;
//   warp 8      MMA issuer (one thread) and TMEM owner (512 columns);
//   warps 0..7  epilogue: warp w reads TMEM lanes 32 (w % 4) .. + 31 (one token each) and
//               columns 128 (w / 4) .. + 127, computes exp2(c log2e D) per column, sums the
//               H columns of each query and stores s for tokens t <= p.
// The exponentials (one per token, query and head) bound this pass. The special-function
// unit does most of them; kPolyCols of every 32 go to the FMA pipe instead (exp2_poly2).
#include "attn_pipeline.cuh"
#include "internal.h"
#include "tc05.cuh"

namespace hs2 {

namespace {

constexpr int kTcTile = 128;                  // cache rows per tile (the MMA's M)
constexpr int kTcN = 256;                     // (query, head) columns per block (the MMA's N)
constexpr int kTcStages = 3;
constexpr int kPolyCols = 12;                 // of every 32 columns, exponentiated by exp2_poly2
constexpr int kTcStageBytes = kTcTile * 256;  // two [128][128 B] swizzled dim blocks
constexpr int kTcEpiWarps = 8;
constexpr int kTcWarpMma = 8, kTcWarpTma = 9;
constexpr int kTcThreads = 10 * 32;
constexpr uint32_t kTcCols = 2 * kTcN;        // two accumulators

struct TcSmem {
  uint8_t *stages, *q;        // stages: kTcStages x 32 KB; q: two [256][128 B] dim blocks
  uint8_t *qx, *ones;         // ninth k-step: B [256][128 B] lse terms, A [128][128 B] ones
  uint64_t *full, *empty, *acc_full, *acc_empty, *done;
  uint32_t *tmem_base;
  volatile int *abort_flag;
  static constexpr size_t kBytes = 1024 + kTcStages * kTcStageBytes + 3 * kTcN * 128 +
                                   kTcTile * 128 + (2 * kTcStages + 5) * 8 + 16;
  __device__ explicit TcSmem(uint8_t *raw) {
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
    stages = base;
    q = stages + kTcStages * kTcStageBytes;
    qx = q + 2 * kTcN * 128;
    ones = qx + kTcN * 128;
    full = reinterpret_cast<uint64_t *>(ones + kTcTile * 128);
    empty = full + kTcStages;
    acc_full = empty + kTcStages;
    acc_empty = acc_full + 2;
    done = acc_empty + 2;
    tmem_base = reinterpret_cast<uint32_t *>(done + 1);
    abort_flag = reinterpret_cast<volatile int *>(tmem_base + 1);
  }
};

struct TcGeom {
  int b, i0, nqb;
  int64_t row0, pfirst;
  int tile_begin, n_tiles;   // absolute 128-row tiles
};

__device__ __forceinline__ TcGeom tc_geom(const RowsParams &P, int item) {
  TcGeom g;
  const int blk_global = item / P.n_chunks, j = item % P.n_chunks;
  g.b = find_item_seq(P.seq, P.batch, blk_global);
  const int nblk = P.seq.item_begin[g.b + 1] - P.seq.item_begin[g.b];
  const int blk = nblk - 1 - (blk_global - P.seq.item_begin[g.b]);   // latest blocks first
  g.i0 = blk * P.q_per_block;
  g.nqb = min(P.q_per_block, P.n_q - g.i0);
  g.row0 = P.seq.start[g.b];
  g.pfirst = (int64_t)P.seq.len[g.b] - P.n_q + g.i0;
  const int64_t plast = g.pfirst + g.nqb - 1;
  const int tile0 = (int)(g.row0 / kTcTile);
  const int ntl = (int)((g.row0 + plast) / kTcTile) - tile0 + 1;
  const int ch = (ntl + P.n_chunks - 1) / P.n_chunks;
  g.tile_begin = tile0 + j * ch;
  g.n_tiles = max(0, min(ch, ntl - j * ch));
  return g;
}

// hs[0] / hs[1] = sum of exp2(scale * v[i]) over i < 16 / i >= 16; the first kPolyCols / 2 of
// each half on the FMA pipe, the rest on the special-function unit.
__device__ __forceinline__ void exp2_sum16x2(const float (&v)[32], float scale, float (&hs)[2]) {
  const float2 sc = make_float2(scale, scale);
  float2 e[16];
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const int half = k >> 3, kk = k & 7;   // pair kk of half `half`: columns 16 half + 2 kk
    const float2 x = ffma2(make_float2(v[16 * half + 2 * kk], v[16 * half + 2 * kk + 1]), sc,
                           make_float2(0.f, 0.f));
    if (2 * kk < kPolyCols / 2) {
      e[k] = exp2_poly2(x);
    } else {
      e[k] = make_float2(fast_exp2(x.x), fast_exp2(x.y));
    }
  }
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    float2 s4[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) s4[k] = fadd2(e[8 * h + 2 * k], e[8 * h + 2 * k + 1]);
    const float2 s2a = fadd2(s4[0], s4[1]), s2b = fadd2(s4[2], s4[3]);
    const float2 s1 = fadd2(s2a, s2b);
    hs[h] = s1.x + s1.y;
  }
}

__device__ __forceinline__ void fail_timeout(const RowsParams &P, volatile int *abort_flag) {
  record_status(P.status, kStatusTimeout);
  *abort_flag = 1;
}

template <int HG>
__global__ void __launch_bounds__(kTcThreads, 1)
    rows_score_tc_kernel(const __grid_constant__ TensorMaps tm, const __grid_constant__ RowsParams P) {
  constexpr int H = 16 * HG;
  constexpr int NQ = kTcN / H;   // queries per block
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  TcSmem sm(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const TcGeom G = tc_geom(P, blockIdx.x);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kTcStages; ++s) {
      mbar_init(smem_u32(&sm.full[s]), 1);
      mbar_init(smem_u32(&sm.empty[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(&sm.acc_full[a]), 1);
      mbar_init(smem_u32(&sm.acc_empty[a]), kTcEpiWarps);
    }
    mbar_init(smem_u32(&sm.done[0]), 1);
    *sm.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kTcWarpMma) {
    tmem_alloc(smem_u32(sm.tmem_base), kTcCols);
    tmem_relinquish();
  }
  griddep_launch_dependents();
  griddep_wait();   // lse comes from pass 1

  // Q block -> shared memory (K-major, 128-byte swizzle), lse_h log2 e per column
  if (warp < kTcEpiWarps) {
    const __nv_bfloat16 *qg = reinterpret_cast<const __nv_bfloat16 *>(P.q) +
                              ((size_t)G.b * P.n_q + G.i0) * H * kHeadDim;
    const int nrows = G.nqb * H;
    for (int t = threadIdx.x; t < kTcN * 16; t += kTcEpiWarps * 32) {
      const int r = t >> 4, ch = t & 15;   // 16-byte chunk ch of row r
      uint4 v = make_uint4(0, 0, 0, 0);
      if (r < nrows) v = *reinterpret_cast<const uint4 *>(qg + (size_t)r * kHeadDim + ch * 8);
      *reinterpret_cast<uint4 *>(sm.q + (ch >> 3) * (kTcN * 128) + sw128(r, (ch & 7) * 16)) = v;
    }
    // ninth k-step operands: all 16-byte chunks zero, then the three terms of each row
    for (int t = threadIdx.x; t < (kTcN + kTcTile) * 8; t += kTcEpiWarps * 32)
      reinterpret_cast<uint4 *>(sm.qx)[t] = make_uint4(0, 0, 0, 0);   // qx and ones are adjacent
    named_barrier_sync(1, kTcEpiWarps * 32);
    for (int r = threadIdx.x; r < kTcN; r += kTcEpiWarps * 32) {
      float v = 0.f;
      if (r < nrows) v = -P.lse[((size_t)G.b * P.n_q + G.i0) * H + r] * kLog2e / P.scale_log2;
      const __nv_bfloat16 h1 = __float2bfloat16_rn(v);
      const float r1 = v - __bfloat162float(h1);
      const __nv_bfloat16 h2 = __float2bfloat16_rn(r1);
      const __nv_bfloat16 h3 = __float2bfloat16_rn(r1 - __bfloat162float(h2));
      __nv_bfloat16 *row = reinterpret_cast<__nv_bfloat16 *>(sm.qx + sw128(r, 0));
      row[0] = h1;
      row[1] = h2;
      row[2] = h3;
      if (r < kTcTile) {
        __nv_bfloat16 *one = reinterpret_cast<__nv_bfloat16 *>(sm.ones + sw128(r, 0));
        one[0] = one[1] = one[2] = __float2bfloat16_rn(1.f);
      }
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *sm.tmem_base;

  if (warp == kTcWarpTma) {
    // ------------------------------------------------------------ producer
    for (int it = 0; it < G.n_tiles; ++it) {
      const int s = it % kTcStages;
      if (it >= kTcStages) {
        bool ok = true;
        if (lane == 0) ok = mbar_wait(smem_u32(&sm.empty[s]), ((it / kTcStages) & 1) ^ 1);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) {
          if (lane == 0) fail_timeout(P, sm.abort_flag);
          break;
        }
      }
      if (*sm.abort_flag) break;
      if (lane == 0) {
        uint8_t *st = sm.stages + s * kTcStageBytes;
        const uint32_t bar = smem_u32(&sm.full[s]);
        const int y = (G.tile_begin + it) * kTcTile;
        mbar_arrive_expect_tx(bar, kTcStageBytes);
        for (int half = 0; half < 2; ++half)
          for (int kb = 0; kb < 2; ++kb)
            tma_load_2d(smem_u32(st + kb * (kTcTile * 128) + half * (64 * 128)), &tm.k, bar,
                        kb * 64, y + half * 64);
      }
    }
  } else if (warp == kTcWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t idesc = umma_idesc_bf16(kTcTile, kTcN);
    bool ok = true;
    for (int it = 0; it < G.n_tiles && ok; ++it) {
      const int s = it % kTcStages, a = it & 1;
      if (lane == 0) {
        ok = mbar_wait(smem_u32(&sm.full[s]), (it / kTcStages) & 1);
        if (ok && it >= 2) ok = mbar_wait(smem_u32(&sm.acc_empty[a]), ((it >> 1) & 1) ^ 1);
        if (!ok) fail_timeout(P, sm.abort_flag);
        if (*sm.abort_flag) ok = false;
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      if (lane == 0) {
        const uint32_t st = smem_u32(sm.stages + s * kTcStageBytes);
        const uint32_t qs = smem_u32(sm.q);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint32_t off = (k >> 2) * (kTcTile * 128) + (k & 3) * 32;
          const uint32_t qoff = (k >> 2) * (kTcN * 128) + (k & 3) * 32;
          umma_bf16(tmem + a * kTcN, umma_desc_sw128(st + off, 1024), umma_desc_sw128(qs + qoff, 1024),
                    idesc, k > 0);
        }
        umma_bf16(tmem + a * kTcN, umma_desc_sw128(smem_u32(sm.ones), 1024),
                  umma_desc_sw128(smem_u32(sm.qx), 1024), idesc, true);
        umma_commit(smem_u32(&sm.empty[s]));
        umma_commit(smem_u32(&sm.acc_full[a]));
      }
      __syncwarp();
    }
    // every issued product has completed before the accumulators are released
    if (lane == 0) {
      umma_commit(smem_u32(&sm.done[0]));
      if (!mbar_wait(smem_u32(&sm.done[0]), 0)) fail_timeout(P, sm.abort_flag);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3, half = warp >> 2;
    const int tok = quarter * 32 + lane;            // TMEM lane = token row of the tile
    const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
    constexpr int QH = NQ / 2;                      // queries of this half
    int64_t plim[QH];
#pragma unroll
    for (int j = 0; j < QH; ++j) plim[j] = G.pfirst + half * QH + j;   // last visible position
    for (int it = 0; it < G.n_tiles; ++it) {
      const int a = it & 1;
      bool ok = true;
      if (lane == 0) {
        ok = mbar_wait(smem_u32(&sm.acc_full[a]), (it >> 1) & 1);
        if (!ok) fail_timeout(P, sm.abort_flag);
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok || *sm.abort_flag) break;
      tc_fence_after();
      // 4 loads of 32 columns, each issued before the previous one is consumed
      float sum[QH];
#pragma unroll
      for (int j = 0; j < QH; ++j) sum[j] = 0.f;
      float va[32], vb[32];
      const uint32_t col0 = lane_addr + a * kTcN + half * 128;
      tmem_ld32(col0, va);
      tmem_wait_ld();
#pragma unroll
      for (int cb = 0; cb < 4; ++cb) {
        if (cb < 3) {
          if (cb & 1) tmem_ld32(col0 + (cb + 1) * 32, va);
          else tmem_ld32(col0 + (cb + 1) * 32, vb);
        }
        const float (&v)[32] = (cb & 1) ? vb : va;
        float hs[2];
        exp2_sum16x2(v, P.scale_log2, hs);
        const int c0 = cb * 32;
        if (H == 32) {
          sum[c0 / 32] += hs[0] + hs[1];
        } else {
          sum[c0 / 16] += hs[0];
          sum[c0 / 16 + 1] += hs[1];
        }
        if (cb < 3) tmem_wait_ld();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&sm.acc_empty[a]));
      const int64_t row = (int64_t)(G.tile_begin + it) * kTcTile + tok;
      const int64_t t = row - G.row0;
#pragma unroll
      for (int j = 0; j < QH; ++j) {
        const int qi = half * QH + j;
        if (qi < G.nqb && t >= 0 && t <= plim[j]) {
          float *srow = P.scores + ((size_t)G.b * P.n_q + G.i0 + qi) * P.score_stride;
          srow[t] = sum[j];
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kTcWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, kTcCols);
  }
}

template <int HG>
cudaError_t launch_t(const TensorMaps &tm, const RowsParams &p, cudaStream_t s) {
  static_assert(TcSmem::kBytes <= 227 * 1024, "score pass shared memory");
  auto kern = rows_score_tc_kernel<HG>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)TcSmem::kBytes);
  if (e != cudaSuccess) return e;
  e = launch_pdl(kern, p.n_items, kTcThreads, TcSmem::kBytes, s, tm, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

int rows_score_tc_queries(int n_heads) { return kTcN / n_heads; }

cudaError_t launch_rows_score_tc(const TensorMaps &tm, const RowsParams &p, cudaStream_t s) {
  if (p.n_heads == 16) return launch_t<1>(tm, p, s);
  if (p.n_heads == 32) return launch_t<2>(tm, p, s);
  return cudaErrorInvalidValue;
}

}  // namespace hs2
