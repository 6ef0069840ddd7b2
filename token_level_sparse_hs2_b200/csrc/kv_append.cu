// kv_append.cu -- writes the new tokens' K and V rows into the shared cache before the block
// runs (the step right before the hybrid block's full-attention layer).
//
// "HySparse2: Hybrid Sparse Attention with Two-Level KV Sharing" (academy.dair.ai), bullet
// "Inference cost": one K/V head serves every query head and the cache is stored in FP8.
// "HySparse2: How Xiaomi Split the Transformer to Fix Agent Prefill Costs", section "KV Reuse
// and Token-Level Sparse Selection": the sparse layers and the forced window read the full
// layer's cache, so every decode step appends its token there first.
//
// Each warp takes 16 (row, matrix) items, one per quarter warp per step, every load issued
// before any store: 128 bf16 values per row, 32 per lane. bf16 cache: a copy. e4m3 cache: the row's
// largest magnitude (quarter-warp max), scale = amax / 448 in float32 (1 for a zero row), codes =
// cvt.rn.satfinite of the float32 quotient x / scale (round to nearest even, saturating at 448),
// formed as in quant.cuh (a reciprocal per row, then Markstein's correction: one multiply and
// two fused multiply-adds per value).
#include "common.cuh"
#include "internal.h"
#include "quant.cuh"

namespace hs2 {

namespace {

constexpr int kLanesPerRow = 4;                        // 32 values (64 bytes of bf16) per lane
constexpr int kItemsPerStep = 32 / kLanesPerRow;       // (matrix, row) items per warp step
constexpr int kSteps = 2;                              // steps per warp, loads of both first

// Quarter warp q of a warp handles one (matrix, row) item per step; lane l of the quarter holds
// values [32 l, 32 l + 32) of the row. Every per-row scalar (the destination row and the scale)
// is computed once per 8 rows of the warp, and the row maximum takes two
// shuffles.
__global__ void __launch_bounds__(256) kv_append_kernel(const __grid_constant__ AppendParams P) {
  griddep_launch_dependents();
  griddep_wait();   // earlier kernels of the stream may still read the cache rows written here
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  const int q = lane / kLanesPerRow, ql = lane % kLanesPerRow;
  const int n_rows = P.batch * P.n_q, n_items = 2 * n_rows;   // (matrix, row) pairs
  uint4 raw[kSteps][4];
  int item[kSteps];
#pragma unroll
  for (int u = 0; u < kSteps; ++u) {   // all loads first
    item[u] = (warp * kSteps + u) * kItemsPerStep + q;
    if (item[u] < n_items) {
      const int kv = item[u] >= n_rows, r = item[u] - (kv ? n_rows : 0);
      const uint4 *src = reinterpret_cast<const uint4 *>(reinterpret_cast<const __nv_bfloat16 *>(kv ? P.new_v : P.new_k) +
                                                         (size_t)r * kHeadDim) + 4 * ql;
#pragma unroll
      for (int k = 0; k < 4; ++k) raw[u][k] = src[k];
    } else {
#pragma unroll
      for (int k = 0; k < 4; ++k) raw[u][k] = make_uint4(0, 0, 0, 0);
    }
  }
#pragma unroll
  for (int u = 0; u < kSteps; ++u) {
    const bool act = item[u] < n_items;
    const int kv = act && item[u] >= n_rows;
    const int r = act ? item[u] - (kv ? n_rows : 0) : 0;
    int b = r, i = 0;
    if (P.n_q != 1) {
      b = r / P.n_q;
      i = r - b * P.n_q;
    }
    const int64_t row = P.seq.start[b] + (int64_t)P.seq.len[b] - P.n_q + i;
    if (!P.fp8) {
      if (act) {
        uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<uint8_t *>(kv ? P.v : P.k) + row * (kHeadDim * 2)) + 4 * ql;
#pragma unroll
        for (int k = 0; k < 4; ++k) dst[k] = raw[u][k];
      }
      continue;
    }
    float amax = 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t w[4] = {raw[u][k].x, raw[u][k].y, raw[u][k].z, raw[u][k].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[e]));
        amax = fmax3(amax, fabsf(f.x), fabsf(f.y));
      }
    }
#pragma unroll
    for (int o = 1; o < kLanesPerRow; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float sc = fp8_row_scale(amax);
    const float rc = fp8_row_recip(sc);
    uint4 c[2];
#pragma unroll
    for (int k = 0; k < 4; ++k) {   // 8 values -> 8 codes (2 words)
      const uint32_t w[4] = {raw[u][k].x, raw[u][k].y, raw[u][k].z, raw[u][k].w};
      uint32_t cw[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[2 * h]));
        const float2 f1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[2 * h + 1]));
        cw[h] = (fp8_pair(f0.x, f0.y, sc, rc) & 0xffffu) | (fp8_pair(f1.x, f1.y, sc, rc) << 16);
      }
      if (k & 1) { c[k >> 1].z = cw[0]; c[k >> 1].w = cw[1]; }
      else { c[k >> 1].x = cw[0]; c[k >> 1].y = cw[1]; }
    }
    if (act) {
      uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<uint8_t *>(kv ? P.v : P.k) + row * kHeadDim + 32 * ql);
      dst[0] = c[0];
      dst[1] = c[1];
      if (ql == 0) (kv ? P.v_scale : P.k_scale)[row] = sc;
    }
  }
}

}  // namespace

cudaError_t launch_kv_append(const AppendParams &p, cudaStream_t s) {
  const int per_warp = kSteps * kItemsPerStep;
  const int warps = (2 * p.batch * p.n_q + per_warp - 1) / per_warp;
  const int grid = (warps * 32 + 255) / 256;
  cudaError_t e = launch_pdl(kv_append_kernel, grid, 256, 0, s, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace hs2
