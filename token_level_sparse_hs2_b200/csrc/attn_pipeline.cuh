// attn_pipeline.cuh -- the TMA tile pipeline shared by the full-attention kernels: stage
// layout per cache format and pass, and the producer warp that streams 64-row K (and V) tiles
// of the cache into a ring of shared-memory stages.
#pragma once

#include "attn_tile.cuh"
#include "internal.h"

namespace hs2 {

template <int KV, int PASS>
struct DecodeCfg {
  static constexpr int kKBytes = (KV == kKvBf16) ? 2 * kBoxBytes : kBoxBytes;
  static constexpr int kVBytes = (PASS == 0) ? kKBytes : 0;
  static constexpr int kScaleBytes = (KV == kKvFp8) ? (PASS == 0 ? 512 : 256) : 0;
  static constexpr int kStageRaw = kKBytes + kVBytes + kScaleBytes;
  static constexpr int kStageBytes = (kStageRaw + 1023) / 1024 * 1024;
  static constexpr int kStages = (KV == kKvBf16) ? (PASS == 0 ? 3 : 4) : (PASS == 0 ? 4 : 6);
  static constexpr uint32_t kTxBytes = kKBytes + kVBytes;          // TMA bytes per stage
  static constexpr uint32_t kFullCount = (KV == kKvFp8) ? 33 : 1;  // arrivals per stage
};

__device__ __forceinline__ int find_item_seq(const SeqTable &t, int batch, int item) {
  int lo = 0, hi = batch - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (t.item_begin[mid] <= item) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// ------------------------------------------------------------------ producer

// All 32 lanes run the loop: lane 0 waits for the slot and issues the TMA tile loads; for an
// FP8 cache every lane also copies two per-token scales (cp.async, bounds-checked) and arrives
// on the slot's barrier when they land. Full barriers expect 1 (bf16) or 33 (FP8) arrivals.
template <int KV, int PASS>
__device__ __forceinline__ void produce(const TensorMaps &tm, const float *k_scale,
                                        const float *v_scale, int64_t kv_rows, uint8_t *stages,
                                        uint64_t *full, uint64_t *empty, int tile_begin,
                                        int n_tiles, volatile int *abort_flag, uint32_t *status) {
  using C = DecodeCfg<KV, PASS>;
  const int lane = threadIdx.x & 31;
  for (int it = 0; it < n_tiles; ++it) {
    const int s = it % C::kStages;
    const uint32_t par = ((it / C::kStages) & 1) ^ 1;
    if (it >= C::kStages) {
      bool ok = true;
      if (lane == 0) ok = mbar_wait(smem_u32(&empty[s]), par);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) {
        if (lane == 0) {
          record_status(status, kStatusTimeout);
          *abort_flag = 1;
        }
        return;
      }
    }
    if (*abort_flag) return;
    uint8_t *st = stages + s * C::kStageBytes;
    const uint32_t bar = smem_u32(&full[s]);
    const int y = (tile_begin + it) * kTile;
    if (lane == 0) {
      mbar_arrive_expect_tx(bar, C::kTxBytes);
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
        const int64_t row = (int64_t)y + rr;
        const bool in = row < kv_rows;
        cp_async_4(smem_u32(sc + rr * 4), k_scale + (in ? row : 0), in ? 4u : 0u);
        if (PASS == 0)
          cp_async_4(smem_u32(sc + (kTile + rr) * 4), v_scale + (in ? row : 0), in ? 4u : 0u);
      }
      cp_async_mbar_arrive(bar);
    }
  }
}

}  // namespace hs2
