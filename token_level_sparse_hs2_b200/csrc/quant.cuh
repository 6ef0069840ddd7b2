// quant.cuh -- the FP8 (e4m3) cache row quantiser shared by every kernel that writes cache rows.
// Per row and matrix, from the format's definition value = scale * code: scale = max|x| / 448 in
// float32 (1 for an all-zero row); code of x = round-to-nearest-even e4m3 of the float32
// quotient x / scale (IEEE division, correctly rounded), saturated at the largest finite e4m3
// value (448).
#pragma once

#include <cuda_fp8.h>

namespace hs2 {

__device__ __forceinline__ float fp8_row_scale(float amax) {
  return amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
}

// two codes (low byte = a) of a row whose scale is sc
__device__ __forceinline__ uint32_t fp8_pair(float a, float b, float sc) {
  return __nv_cvt_float2_to_fp8x2(make_float2(__fdiv_rn(a, sc), __fdiv_rn(b, sc)),
                                  __NV_SATFINITE, __NV_E4M3);
}

}  // namespace hs2
