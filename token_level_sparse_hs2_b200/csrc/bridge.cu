// bridge.cu -- KV Bridging: the cross-decoder full layer's K and V projected from the hidden
// states of a self-decoder full layer and written into the shared cache.
//
// "HySparse2: How Xiaomi Split the Transformer to Fix Agent Prefill Costs", section "The
// Self-Decoder and Cross-Decoder Split": prefill runs only the self-decoder; the caches the
// cross-decoder's full layers read are built from self-decoder hidden states by learned
// projections, K_j = Proj_j^K(H_i^self), V_j = Proj_j^V(H_i^self) (here: linear maps, no bias).
//
// One dense GEMM [M, d] x [d, 256] -> [M, 256] (K and V side by side) on the fifth-generation
// tensor cores, persistent over units of two 128-row tiles that share each weight tile (the
// weights are re-read from L2 for every unit and k-block, so sharing them cuts the bytes per
// product by a third):
//   warp 5      TMA producer: two 128 x 64 tiles of the hidden states and the 256 x 64 tile of
//               the weights per k-block, kBrStages stages of 64 KB;
//   warp 4      MMA issuer (one thread, M = 128, N = 256, K = 16 per instruction, one
//               accumulator of 256 TMEM columns per tile of the unit) and TMEM owner;
//   warps 0..3  epilogue: warp w reads TMEM lanes 32 w .. + 31 (one output row per thread and
//               tile), rounds K and V to bf16 and writes the cache row of that token: bf16 as
//               is, or e4m3 codes plus the row's scale (the same quantiser as the cache append).
#include "common.cuh"
#include "internal.h"
#include "quant.cuh"
#include "tc05.cuh"

namespace hs2 {

namespace {

constexpr int kBrM = 128, kBrN = 256, kBrK = 64;
constexpr int kBrPair = 2;                            // 128-row tiles per unit, sharing the weights
constexpr int kBrStages = 3;
constexpr int kBrABytes = kBrM * 128;                 // [128 rows][64 bf16], 128-byte swizzle
constexpr int kBrBBytes = kBrN * 128;                 // [256 rows][64 bf16]
constexpr int kBrStageBytes = kBrPair * kBrABytes + kBrBBytes;
constexpr int kBrWarpMma = 4, kBrWarpTma = 5;
constexpr int kBrThreads = 6 * 32;
constexpr uint32_t kBrCols = kBrPair * kBrN;          // one accumulator per tile of the unit

struct BrSmem {
  uint8_t *stages;
  uint64_t *full, *empty, *acc_full, *acc_empty, *done;
  uint32_t *tmem_base;
  volatile int *abort_flag;
  static constexpr size_t kBytes = 1024 + kBrStages * kBrStageBytes + (2 * kBrStages + 5) * 8 + 16;
  __device__ explicit BrSmem(uint8_t *raw) {
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
    stages = base;
    full = reinterpret_cast<uint64_t *>(stages + kBrStages * kBrStageBytes);
    empty = full + kBrStages;
    acc_full = empty + kBrStages;
    acc_empty = acc_full + 2;
    done = acc_empty + 2;
    tmem_base = reinterpret_cast<uint32_t *>(done + 1);
    abort_flag = reinterpret_cast<volatile int *>(tmem_base + 1);
  }
};

__device__ __forceinline__ void br_fail(const BridgeParams &P, volatile int *abort_flag) {
  record_status(P.status, kStatusTimeout);
  *abort_flag = 1;
}

// Reads one matrix (128 accumulator columns from col) of this thread's row, rounds it to bf16
// and writes the cache row: 256 bytes of bf16, or 128 e4m3 codes and the row's scale.
__device__ __forceinline__ void store_row(uint32_t col, bool fp8, bool valid, uint8_t *dst,
                                         float *scale_dst) {
  uint32_t packed[64];
  float amax = 0.f;
#pragma unroll
  for (int c2 = 0; c2 < 2; ++c2) {
    float va[32], vb[32];
    tmem_ld32(col + c2 * 64, va);
    tmem_ld32(col + c2 * 64 + 32, vb);
    tmem_wait_ld();
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const __nv_bfloat162 pa = __floats2bfloat162_rn(va[2 * k], va[2 * k + 1]);
      const __nv_bfloat162 pb = __floats2bfloat162_rn(vb[2 * k], vb[2 * k + 1]);
      packed[c2 * 32 + k] = *reinterpret_cast<const uint32_t *>(&pa);
      packed[c2 * 32 + 16 + k] = *reinterpret_cast<const uint32_t *>(&pb);
      const float2 fa = __bfloat1622float2(pa), fb = __bfloat1622float2(pb);
      amax = fmax3(amax, fabsf(fa.x), fabsf(fa.y));
      amax = fmax3(amax, fabsf(fb.x), fabsf(fb.y));
    }
  }
  if (!valid) return;
  if (!fp8) {
    uint4 *d4 = reinterpret_cast<uint4 *>(dst);
#pragma unroll
    for (int j = 0; j < 16; ++j)
      d4[j] = make_uint4(packed[4 * j], packed[4 * j + 1], packed[4 * j + 2], packed[4 * j + 3]);
    return;
  }
  const float sc = fp8_row_scale(amax);
  const float rc = fp8_row_recip(sc);
  uint4 *d4 = reinterpret_cast<uint4 *>(dst);
#pragma unroll
  for (int j = 0; j < 8; ++j) {                      // 16 codes per store
    uint32_t w[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&packed[8 * j + 2 * q]));
      const float2 f1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&packed[8 * j + 2 * q + 1]));
      w[q] = (fp8_pair(f0.x, f0.y, sc, rc) & 0xffffu) | (fp8_pair(f1.x, f1.y, sc, rc) << 16);
    }
    d4[j] = make_uint4(w[0], w[1], w[2], w[3]);
  }
  *scale_dst = sc;
}

__global__ void __launch_bounds__(kBrThreads, 1)
    kv_bridge_kernel(const __grid_constant__ BridgeMaps tm, const __grid_constant__ BridgeParams P) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  BrSmem sm(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tiles = (P.m + kBrPair * kBrM - 1) / (kBrPair * kBrM);   // units of kBrPair tiles
  const int nk = P.d_model / kBrK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kBrStages; ++s) {
      mbar_init(smem_u32(&sm.full[s]), 1);
      mbar_init(smem_u32(&sm.empty[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(&sm.acc_full[a]), 1);
      mbar_init(smem_u32(&sm.acc_empty[a]), 4);
    }   // index 0 used: the unit's accumulators fill all of TMEM
    mbar_init(smem_u32(&sm.done[0]), 1);
    *sm.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kBrWarpTma && lane == 0) {
    prefetch_tensormap(&tm.h);
    prefetch_tensormap(&tm.w);
  }
  if (warp == kBrWarpMma) {
    tmem_alloc(smem_u32(sm.tmem_base), kBrCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *sm.tmem_base;
  griddep_launch_dependents();
  griddep_wait();   // the hidden states come from the previous kernel

  if (warp == kBrWarpTma) {
    // ------------------------------------------------------------ producer
    int it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x) {
      for (int kb = 0; kb < nk; ++kb, ++it) {
        const int s = it % kBrStages;
        if (lane == 0) {
          if (it >= kBrStages && !mbar_wait(smem_u32(&sm.empty[s]), ((it / kBrStages) & 1) ^ 1)) {
            br_fail(P, sm.abort_flag);
            ok = false;
          }
          if (*sm.abort_flag) ok = false;
          if (ok) {
            uint8_t *st = sm.stages + s * kBrStageBytes;
            const uint32_t bar = smem_u32(&sm.full[s]);
            mbar_arrive_expect_tx(bar, kBrStageBytes);
            for (int h = 0; h < kBrPair; ++h)
              tma_load_2d(smem_u32(st + h * kBrABytes), &tm.h, bar, kb * kBrK, (tile * kBrPair + h) * kBrM);
            tma_load_2d(smem_u32(st + kBrPair * kBrABytes), &tm.w, bar, kb * kBrK, 0);
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
      }
    }
  } else if (warp == kBrWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t idesc = umma_idesc_bf16(kBrM, kBrN);
    int it = 0, tl = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x, ++tl) {
      const int a = 0;
      if (lane == 0 && tl >= 1 && !mbar_wait(smem_u32(&sm.acc_empty[a]), (tl & 1) ^ 1)) {
        br_fail(P, sm.abort_flag);
        ok = false;
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      for (int kb = 0; kb < nk; ++kb, ++it) {
        const int s = it % kBrStages;
        if (lane == 0) {
          if (!mbar_wait(smem_u32(&sm.full[s]), (it / kBrStages) & 1)) {
            br_fail(P, sm.abort_flag);
            ok = false;
          }
          if (*sm.abort_flag) ok = false;
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        tc_fence_after();
        if (lane == 0) {
          const uint32_t st = smem_u32(sm.stages + s * kBrStageBytes);
#pragma unroll
          for (int k = 0; k < kBrK / 16; ++k)
#pragma unroll
            for (int h = 0; h < kBrPair; ++h)
              umma_bf16(tmem + h * kBrN, umma_desc_sw128(st + h * kBrABytes + k * 32, 1024),
                        umma_desc_sw128(st + kBrPair * kBrABytes + k * 32, 1024), idesc, (kb | k) != 0);
          umma_commit(smem_u32(&sm.empty[s]));
          if (kb == nk - 1) umma_commit(smem_u32(&sm.acc_full[a]));
        }
        __syncwarp();
      }
    }
    // every issued product has completed before the accumulators are released
    if (lane == 0) {
      umma_commit(smem_u32(&sm.done[0]));
      if (!mbar_wait(smem_u32(&sm.done[0]), 0)) br_fail(P, sm.abort_flag);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
    int tl = 0;
    for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++tl) {
      const int a = 0;
      bool ok = true;
      if (lane == 0 && !mbar_wait(smem_u32(&sm.acc_full[a]), tl & 1)) {
        br_fail(P, sm.abort_flag);
        ok = false;
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok || *sm.abort_flag) break;
      tc_fence_after();
      for (int h = 0; h < kBrPair; ++h) {
        const int r = (tile * kBrPair + h) * kBrM + warp * 32 + lane;   // row of the hidden states
        const bool valid = r < P.m;
        int64_t row = 0;
        if (valid) {
          const int b = r / P.n_q, i = r % P.n_q;
          row = P.seq.start[b] + (int64_t)P.seq.len[b] - P.n_q + i;
        }
        const size_t rb = P.fp8 ? kHeadDim : kHeadDim * 2;   // bytes per cache row
        store_row(lane_addr + h * kBrN, P.fp8, valid, static_cast<uint8_t *>(P.k) + row * rb,
                  P.k_scale + row);
        store_row(lane_addr + h * kBrN + 128, P.fp8, valid, static_cast<uint8_t *>(P.v) + row * rb,
                  P.v_scale + row);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&sm.acc_empty[a]));
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kBrWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, kBrCols);
  }
}

}  // namespace

cudaError_t launch_kv_bridge(const BridgeMaps &tm, const BridgeParams &p, int grid, cudaStream_t s) {
  static_assert(BrSmem::kBytes <= 227 * 1024, "bridge shared memory");
  cudaError_t e = cudaFuncSetAttribute(kv_bridge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)BrSmem::kBytes);
  if (e != cudaSuccess) return e;
  e = launch_pdl(kv_bridge_kernel, grid, kBrThreads, BrSmem::kBytes, s, tm, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace hs2
