// kv_append.cu -- writes the new tokens' K and V rows into the shared cache before the block
// runs (the step right before the hybrid block's full-attention layer).
//
// "HySparse2: Hybrid Sparse Attention with Two-Level KV Sharing" (academy.dair.ai), bullet
// "Inference cost": one K/V head serves every query head and the cache is stored in FP8.
// "HySparse2: How Xiaomi Split the Transformer to Fix Agent Prefill Costs", section "KV Reuse
// and Token-Level Sparse Selection": the sparse layers and the forced window read the full
// layer's cache, so every decode step appends its token there first.
//
// Each warp takes 8 (row, matrix) items, one per half warp per step, every load issued before
// any store: 128 bf16 values per row, 8 per lane. bf16 cache: a copy. e4m3 cache: the row's
// largest magnitude (half-warp max), scale = amax / 448 in float32 (1 for a zero row), codes =
// cvt.rn.satfinite of the float32 product x * (1 / scale), the reciprocal correctly rounded
// (round to nearest even, saturating at 448).
#include "common.cuh"
#include "internal.h"
#include "quant.cuh"

namespace hs2 {

namespace {

constexpr int kAppendRowsPerWarp = 8;   // two rows (one per half warp) per step, four steps

// Half warp h of a warp handles one (row, matrix) per step: 8 bf16 values per lane (16 bytes).
__global__ void __launch_bounds__(256) kv_append_kernel(const __grid_constant__ AppendParams P) {
  griddep_launch_dependents();
  griddep_wait();   // earlier kernels of the stream may still read the cache rows written here
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  const int half = lane >> 4, hl = lane & 15;
  const int n_rows = P.batch * P.n_q, n_items = 2 * n_rows;   // (matrix, row) pairs
  uint4 raw[kAppendRowsPerWarp / 2];
  int item[kAppendRowsPerWarp / 2];
#pragma unroll
  for (int u = 0; u < kAppendRowsPerWarp / 2; ++u) {   // all loads first
    item[u] = warp * kAppendRowsPerWarp + 2 * u + half;
    raw[u] = make_uint4(0, 0, 0, 0);
    if (item[u] < n_items) {
      const int kv = item[u] / n_rows, r = item[u] % n_rows;
      raw[u] = *(reinterpret_cast<const uint4 *>(reinterpret_cast<const __nv_bfloat16 *>(kv ? P.new_v : P.new_k) +
                                                (size_t)r * kHeadDim) + hl);
    }
  }
#pragma unroll
  for (int u = 0; u < kAppendRowsPerWarp / 2; ++u) {
    const bool act = item[u] < n_items;
    const int kv = act ? item[u] / n_rows : 0, r = act ? item[u] % n_rows : 0;
    const int b = r / P.n_q, i = r % P.n_q;
    const int64_t row = P.seq.start[b] + (int64_t)P.seq.len[b] - P.n_q + i;
    if (!P.fp8) {
      if (act) *(reinterpret_cast<uint4 *>(reinterpret_cast<uint8_t *>(kv ? P.v : P.k) + row * (kHeadDim * 2)) + hl) = raw[u];
      continue;
    }
    float x[8];
    const uint32_t w[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[k]));
      x[2 * k] = f.x;
      x[2 * k + 1] = f.y;
    }
    float amax = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) amax = fmaxf(amax, fabsf(x[k]));
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));   // within the half
    const float sc = fp8_row_scale(amax);
    const float inv = __frcp_rn(sc);
    uint32_t c[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) c[k] = fp8_pair(x[2 * k], x[2 * k + 1], inv);
    if (act) {
      uint8_t *dst = reinterpret_cast<uint8_t *>(kv ? P.v : P.k) + row * kHeadDim + 8 * hl;
      *reinterpret_cast<uint2 *>(dst) = make_uint2((c[0] & 0xffffu) | (c[1] << 16), (c[2] & 0xffffu) | (c[3] << 16));
      if (hl == 0) (kv ? P.v_scale : P.k_scale)[row] = sc;
    }
  }
}

}  // namespace

cudaError_t launch_kv_append(const AppendParams &p, cudaStream_t s) {
  const int warps = (2 * p.batch * p.n_q + kAppendRowsPerWarp - 1) / kAppendRowsPerWarp;
  const int grid = (warps * 32 + 255) / 256;
  cudaError_t e = launch_pdl(kv_append_kernel, grid, 256, 0, s, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace hs2
