// attn_rows_tc1.cu -- output pass (pass 1: O and lse) of the full-attention layer for query
// chunks and prefill on the fifth-generation tensor cores (tcgen05, S, P and O in TMEM).
//
// "HySparse2: How Xiaomi Split the Transformer to Fix Agent Prefill Costs", section "KV Reuse
// and Token-Level Sparse Selection": the full layer attends over the whole context; every query
// row sees its own causal prefix. With MQA every K/V tile serves all 128 (query, head) rows of
// a block (128 / H queries x H heads).
//
// One CTA per (block, chunk of the block's causal prefix); per 128-row K/V tile i:
//   S_i = Q . K_i^T      tcgen05.mma, A = Q block (smem), B = K tile (smem), D = S buffer i % 2
//   P_i = exp2(c log2e S_i - m)   eight softmax warps, two threads per (query, head) row (warps
//                        w and w + 4 read the same TMEM lanes, one half of the columns each):
//                        the row max (halves exchanged through shared memory), a lazy
//                        rescale, the exponentials (special-function unit and exp2_poly2), the
//                        row sum; P is written back over S as bf16 pairs
//   O += P_i . V_i       tcgen05.mma, A = P (TMEM), B = V tile (smem, MN-major), D = O
// The MMA warp issues S_{i+1} before O += P_i V_i, so the tensor cores compute the next scores
// while the softmax warps work. The reference max m only moves when a tile's row max exceeds
// it by more than 8 (P <= 2^8 in bf16); then the row's O is rescaled in TMEM once the previous
// P V product has landed. A block's chunks are merged by the last CTA to finish.
#include "attn_pipeline.cuh"
#include "internal.h"
#include "tc05.cuh"

namespace hs2 {

namespace {

constexpr int kA1Tile = 128;                    // cache rows per tile
constexpr int kA1Rows = 128;                    // (query, head) rows per block
constexpr int kA1KStages = 3, kA1VStages = 2;
constexpr int kA1TileBytes = kA1Tile * 256;     // two [128][128 B] swizzled dim blocks
constexpr int kA1SmWarps = 8;
constexpr int kA1WarpMma = 8, kA1WarpTma = 9;
constexpr int kA1Threads = 10 * 32;
constexpr uint32_t kA1Cols = 512;               // S/P buffers at 0 and 128, O at 256
constexpr uint32_t kA1ColO = 256;
constexpr float kA1Lazy = 8.f;
constexpr int kA1PolyPairs = 6;                 // of every 16 pairs, exponentiated by exp2_poly2

struct A1Smem {
  uint8_t *q, *k, *v;
  float *xm;                  // [2 buffers][2 halves][128 rows] partial row maxima / sums
  uint64_t *k_full, *k_empty, *v_full, *v_empty, *s_full, *p_full, *o_done, *done, *x_full;
  uint32_t *tmem_base;
  volatile int *abort_flag;
  static constexpr size_t kBytes = 1024 + (size_t)kA1Rows * 256 +
                                   (size_t)(kA1KStages + kA1VStages) * kA1TileBytes + 4 * kA1Rows * 4 +
                                   (2 * kA1KStages + 2 * kA1VStages + 8) * 8 + 16;
  __device__ explicit A1Smem(uint8_t *raw) {
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
    q = base;
    k = q + kA1Rows * 256;
    v = k + kA1KStages * kA1TileBytes;
    xm = reinterpret_cast<float *>(v + kA1VStages * kA1TileBytes);
    k_full = reinterpret_cast<uint64_t *>(xm + 4 * kA1Rows);
    k_empty = k_full + kA1KStages;
    v_full = k_empty + kA1KStages;
    v_empty = v_full + kA1VStages;
    s_full = v_empty + kA1VStages;
    p_full = s_full + 2;
    o_done = p_full + 2;
    done = o_done + 1;
    x_full = done + 1;
    tmem_base = reinterpret_cast<uint32_t *>(x_full + 2);
    abort_flag = reinterpret_cast<volatile int *>(tmem_base + 1);
  }
};

struct A1Geom {
  int b, blk_global, j, i0, nqb;
  int64_t row0, pfirst;
  int tile_begin, n_tiles;   // absolute 128-row tiles
};

// item -> (sequence, block, chunk); blocks of a sequence run latest-first (longest prefixes)
__device__ __forceinline__ A1Geom a1_geom(const RowsParams &P, int item) {
  A1Geom g;
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
  const int tile0 = (int)(g.row0 / kA1Tile);
  const int ntl = (int)((g.row0 + plast) / kA1Tile) - tile0 + 1;
  const int ch = (ntl + P.n_chunks - 1) / P.n_chunks;
  g.tile_begin = tile0 + g.j * ch;
  g.n_tiles = max(0, min(ch, ntl - g.j * ch));
  return g;
}

__device__ __forceinline__ void a1_fail(const RowsParams &P, volatile int *abort_flag) {
  record_status(P.status, kStatusTimeout);
  *abort_flag = 1;
}

// bounded wait by lane 0, result broadcast to the warp (records a timeout)
__device__ __forceinline__ bool warp_wait(const RowsParams &P, volatile int *abort_flag,
                                          uint64_t *bar, uint32_t parity) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) {
    ok = mbar_wait(smem_u32(bar), parity);
    if (!ok) a1_fail(P, abort_flag);
    if (*abort_flag) ok = false;
  }
  return __shfl_sync(0xffffffffu, ok, 0);
}

template <int HG>
__global__ void __launch_bounds__(kA1Threads, 1)
    rows_attn_tc_kernel(const __grid_constant__ TensorMaps tm, const __grid_constant__ RowsParams P) {
  constexpr int H = 16 * HG;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  A1Smem sm(smem_raw);
  __shared__ int s_last;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const A1Geom G = a1_geom(P, blockIdx.x);
  const int nrows = G.nqb * H;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kA1KStages; ++s) {
      mbar_init(smem_u32(&sm.k_full[s]), 1);
      mbar_init(smem_u32(&sm.k_empty[s]), 1);
    }
    for (int s = 0; s < kA1VStages; ++s) {
      mbar_init(smem_u32(&sm.v_full[s]), 1);
      mbar_init(smem_u32(&sm.v_empty[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(&sm.s_full[a]), 1);
      mbar_init(smem_u32(&sm.p_full[a]), kA1SmWarps);
    }
    mbar_init(smem_u32(&sm.o_done[0]), 1);
    mbar_init(smem_u32(&sm.done[0]), 1);
    mbar_init(smem_u32(&sm.x_full[0]), kA1SmWarps * 32);
    mbar_init(smem_u32(&sm.x_full[1]), kA1SmWarps * 32);
    *sm.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kA1WarpMma) {
    tmem_alloc(smem_u32(sm.tmem_base), kA1Cols);
    tmem_relinquish();
  }
  griddep_launch_dependents();
  griddep_wait();
  if (warp < kA1SmWarps) {   // Q block -> shared memory (K-major, 128-byte swizzle)
    const __nv_bfloat16 *qg = reinterpret_cast<const __nv_bfloat16 *>(P.q) +
                              ((size_t)G.b * P.n_q + G.i0) * H * kHeadDim;
    for (int t = threadIdx.x; t < kA1Rows * 16; t += kA1SmWarps * 32) {
      const int r = t >> 4, ch = t & 15;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (r < nrows) v = *reinterpret_cast<const uint4 *>(qg + (size_t)r * kHeadDim + ch * 8);
      *reinterpret_cast<uint4 *>(sm.q + (ch >> 3) * (kA1Rows * 128) + sw128(r, (ch & 7) * 16)) = v;
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *sm.tmem_base;
  const int n = G.n_tiles;

  float m_run = -INFINITY, l_run = 0.f;   // softmax threads: this row's state
  if (warp == kA1WarpTma) {
    // ------------------------------------------------------------ producer
    for (int it = 0; it < n; ++it) {
      const int sk = it % kA1KStages, sv = it % kA1VStages;
      if (it >= kA1KStages && !warp_wait(P, sm.abort_flag, &sm.k_empty[sk], ((it / kA1KStages) & 1) ^ 1)) break;
      const int y = (G.tile_begin + it) * kA1Tile;
      if (lane == 0) {
        uint8_t *st = sm.k + sk * kA1TileBytes;
        const uint32_t bar = smem_u32(&sm.k_full[sk]);
        mbar_arrive_expect_tx(bar, kA1TileBytes);
        for (int half = 0; half < 2; ++half)
          for (int kb = 0; kb < 2; ++kb)
            tma_load_2d(smem_u32(st + kb * (kA1Tile * 128) + half * (64 * 128)), &tm.k, bar, kb * 64, y + half * 64);
      }
      if (it >= kA1VStages && !warp_wait(P, sm.abort_flag, &sm.v_empty[sv], ((it / kA1VStages) & 1) ^ 1)) break;
      if (lane == 0) {
        uint8_t *st = sm.v + sv * kA1TileBytes;
        const uint32_t bar = smem_u32(&sm.v_full[sv]);
        mbar_arrive_expect_tx(bar, kA1TileBytes);
        for (int half = 0; half < 2; ++half)
          for (int kb = 0; kb < 2; ++kb)
            tma_load_2d(smem_u32(st + kb * (kA1Tile * 128) + half * (64 * 128)), &tm.v, bar, kb * 64, y + half * 64);
      }
    }
  } else if (warp == kA1WarpMma) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t id_s = umma_idesc_bf16(kA1Rows, kA1Tile);       // S: rows x tokens
    const uint32_t id_o = umma_idesc_bf16_bmn(kA1Rows, kHeadDim);  // O: rows x head_dim, V MN-major
    const uint32_t qs = smem_u32(sm.q);
    for (int it = 0; it <= n; ++it) {
      if (it < n) {   // S_it = Q . K_it^T
        const int sk = it % kA1KStages;
        if (!warp_wait(P, sm.abort_flag, &sm.k_full[sk], (it / kA1KStages) & 1)) break;
        tc_fence_after();
        if (lane == 0) {
          const uint32_t ks = smem_u32(sm.k + sk * kA1TileBytes);
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint32_t off = (k >> 2) * (kA1Tile * 128) + (k & 3) * 32;
            umma_bf16(tmem + (it & 1) * 128, umma_desc_sw128(qs + off, 1024),
                      umma_desc_sw128(ks + off, 1024), id_s, k > 0);
          }
          umma_commit(smem_u32(&sm.k_empty[sk]));
          umma_commit(smem_u32(&sm.s_full[it & 1]));
        }
        __syncwarp();
      }
      if (it >= 1) {  // O += P_j . V_j
        const int j = it - 1, sv = j % kA1VStages;
        if (!warp_wait(P, sm.abort_flag, &sm.p_full[j & 1], (j >> 1) & 1)) break;
        if (!warp_wait(P, sm.abort_flag, &sm.v_full[sv], (j / kA1VStages) & 1)) break;
        tc_fence_after();
        if (lane == 0) {
          const uint32_t vs = smem_u32(sm.v + sv * kA1TileBytes);
#pragma unroll
          for (int k = 0; k < 8; ++k)
            umma_bf16_ts(tmem + kA1ColO, tmem + (j & 1) * 128 + 8 * k,
                         umma_desc_sw128_mn(vs + k * 2048, kA1Tile * 128, 1024), id_o, j > 0 || k > 0);
          umma_commit(smem_u32(&sm.v_empty[sv]));
          umma_commit(smem_u32(&sm.o_done[0]));
        }
        __syncwarp();
      }
    }
    if (lane == 0) {   // every issued product has landed before TMEM is read or released
      umma_commit(smem_u32(&sm.done[0]));
      if (!mbar_wait(smem_u32(&sm.done[0]), 0)) a1_fail(P, sm.abort_flag);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax
    const int r = (warp & 3) * 32 + lane;            // TMEM lane = (query, head) row
    const int half = warp >> 2;                      // columns [64 half, 64 half + 64)
    const int qi = r / H;
    const int64_t plim = G.pfirst + qi;              // last visible position of this row
    const uint32_t lane_addr = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const float sc = P.scale_log2;
    for (int it = 0; it < n; ++it) {
      const int a = it & 1;
      if (!warp_wait(P, sm.abort_flag, &sm.s_full[a], (it >> 1) & 1)) break;
      tc_fence_after();
      float x[64];
      {
        float v[32];
        tmem_ld32(lane_addr + a * 128 + half * 64, v);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) x[i] = v[i];
        tmem_ld32(lane_addr + a * 128 + half * 64 + 32, v);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) x[32 + i] = v[i];
      }
      const int64_t tcol = (int64_t)(G.tile_begin + it) * kA1Tile + half * 64;   // row of column 0
      const bool full = tcol >= G.row0 && tcol + 63 - G.row0 <= G.pfirst;
      if (!__all_sync(0xffffffffu, full)) {
        const int64_t lo = G.row0 - tcol, hi = G.row0 + plim - tcol;   // valid columns [lo, hi]
#pragma unroll
        for (int i = 0; i < 64; ++i)
          if (i < lo || i > hi) x[i] = -INFINITY;
      }
      // partial max of raw scores (sc > 0), exchanged with the thread holding the other half
      float mh = fmax3(x[0], x[1], x[2]);
#pragma unroll
      for (int i = 3; i < 63; i += 2) mh = fmax3(mh, x[i], x[i + 1]);
      mh = fmaxf(mh, x[63]);
      sm.xm[(a * 2 + half) * kA1Rows + r] = mh;
      __syncwarp();
      if (lane == 0) mbar_arrive_cnt(smem_u32(&sm.x_full[a]), 32);
      if (!warp_wait(P, sm.abort_flag, &sm.x_full[a], (it >> 1) & 1)) break;
      const float mt = fmaxf(mh, sm.xm[(a * 2 + (half ^ 1)) * kA1Rows + r]) * sc;
      const bool move = mt > m_run + kA1Lazy;
      if (__any_sync(0xffffffffu, move)) {
        const float m_new = move ? mt : m_run;
        const float alpha = (m_run == -INFINITY) ? 0.f : fast_exp2(m_run - m_new);
        l_run *= alpha;
        m_run = m_new;
        if (it > 0) {   // rescale this half of O once the previous P V product has landed
          if (!warp_wait(P, sm.abort_flag, &sm.o_done[0], (it - 1) & 1)) break;
          tc_fence_after();
#pragma unroll
          for (int cb = 0; cb < 2; ++cb) {
            float v[32];
            tmem_ld32(lane_addr + kA1ColO + half * 64 + cb * 32, v);
            tmem_wait_ld();
            uint32_t u[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) u[i] = __float_as_uint(v[i] * alpha);
            tmem_st32(lane_addr + kA1ColO + half * 64 + cb * 32, u);
          }
          tmem_wait_st();
        }
      }
      const float mref = (m_run == -INFINITY) ? 0.f : m_run;
      const float2 sc2 = make_float2(sc, sc), neg = make_float2(-mref, -mref);
      float2 ls = make_float2(0.f, 0.f);
      uint32_t pk[32];
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        const float2 z = ffma2(make_float2(x[2 * k], x[2 * k + 1]), sc2, neg);
        float2 e;
        if ((k & 15) < kA1PolyPairs) e = exp2_poly2(z);
        else e = make_float2(fast_exp2(z.x), fast_exp2(z.y));
        ls = fadd2(ls, e);
        pk[k] = pack_bf16(e.x, e.y);
      }
      tmem_st32(lane_addr + a * 128 + half * 32, pk);
      l_run += ls.x + ls.y;
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&sm.p_full[a]));
    }
  }
  tc_fence_before();
  __syncthreads();   // the MMA warp has seen every product land (done barrier)
  tc_fence_after();
  const bool aborted = *sm.abort_flag != 0;
  if (warp < kA1SmWarps) sm.xm[(warp >> 2) * kA1Rows + (warp & 3) * 32 + lane] = l_run;
  __syncthreads();
  if (warp < kA1SmWarps && !aborted) {
    // ------------------------------------------------------------ output or chunk partial
    const int r = (warp & 3) * 32 + lane, half = warp >> 2;
    const float l_row = sm.xm[r] + sm.xm[kA1Rows + r];
    const uint32_t lane_addr = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const size_t orow = ((size_t)G.b * P.n_q + G.i0) * H + r;
    float *part = P.part + (((size_t)G.blk_global * P.n_chunks + G.j) * kA1Rows + r) * kPartRow;
    const float inv = (P.n_chunks == 1) ? 1.f / l_row : 1.f;
#pragma unroll
    for (int cb = 0; cb < 2; ++cb) {
      const int c0 = half * 64 + cb * 32;
      float v[32];
      tmem_ld32(lane_addr + kA1ColO + c0, v);
      tmem_wait_ld();
      if (n == 0) {
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = 0.f;
      }
      if (P.n_chunks > 1) {
#pragma unroll
        for (int i = 0; i < 32; i += 4)
          *reinterpret_cast<float4 *>(part + kPartO + c0 + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
      } else if (r < nrows) {
        if (P.out_f32) {
          float *o = reinterpret_cast<float *>(P.out) + orow * kHeadDim + c0;
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            *reinterpret_cast<float4 *>(o + i) = make_float4(v[i] * inv, v[i + 1] * inv, v[i + 2] * inv, v[i + 3] * inv);
        } else {
          __nv_bfloat16 *o = reinterpret_cast<__nv_bfloat16 *>(P.out) + orow * kHeadDim + c0;
#pragma unroll
          for (int i = 0; i < 32; i += 8)
            *reinterpret_cast<uint4 *>(o + i) =
                make_uint4(pack_bf16(v[i] * inv, v[i + 1] * inv), pack_bf16(v[i + 2] * inv, v[i + 3] * inv),
                           pack_bf16(v[i + 4] * inv, v[i + 5] * inv), pack_bf16(v[i + 6] * inv, v[i + 7] * inv));
        }
      }
    }
    if (half == 0) {
      if (P.n_chunks > 1) {
        part[0] = m_run;
        part[1] = l_row;
      } else if (r < nrows) {
        P.lse[orow] = (m_run + __log2f(l_row)) * kLn2;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kA1WarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, kA1Cols);
  }
  if (P.n_chunks == 1 || aborted) return;
  // ------------------------------------------------------------ chunk merge by the last CTA
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
  const float *gp = P.part + (size_t)G.blk_global * P.n_chunks * kA1Rows * kPartRow;
  for (int t = threadIdx.x; t < nrows * kHeadDim; t += kA1Threads) {
    const int r = t / kHeadDim, d = t % kHeadDim;
    float M = -INFINITY;
    for (int i = 0; i < P.n_chunks; ++i) M = fmaxf(M, __ldcg(gp + ((size_t)i * kA1Rows + r) * kPartRow));
    float L = 0.f, O = 0.f;
    for (int i = 0; i < P.n_chunks; ++i) {
      const float *pp = gp + ((size_t)i * kA1Rows + r) * kPartRow;
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

template <int HG>
cudaError_t launch_a1(const TensorMaps &tm, const RowsParams &p, cudaStream_t s) {
  static_assert(A1Smem::kBytes <= 227 * 1024, "output pass shared memory");
  auto kern = rows_attn_tc_kernel<HG>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)A1Smem::kBytes);
  if (e != cudaSuccess) return e;
  e = launch_pdl(kern, p.n_items, kA1Threads, A1Smem::kBytes, s, tm, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_rows_attn_tc(const TensorMaps &tm, const RowsParams &p, cudaStream_t s) {
  if (p.n_heads == 16) return launch_a1<1>(tm, p, s);
  if (p.n_heads == 32) return launch_a1<2>(tm, p, s);
  return cudaErrorInvalidValue;
}

}  // namespace hs2
