// quant.cuh -- the FP8 (e4m3) cache row quantiser shared by every kernel that writes cache rows.
// Per row and matrix, from the format's definition value = scale * code: scale = max|x| / 448 in
// float32 (1 for an all-zero row); code of x = round-to-nearest-even e4m3 of the float32
// quotient x / scale (IEEE division, correctly rounded), saturated at the largest finite e4m3
// value (448).
//
// The quotient is formed with Markstein's correction of the reciprocal product (P. Markstein,
// "Computation of elementary functions on the IBM RISC System/6000 processor", IBM J. Res. Dev.
// 34(1), 1990): r = RN(1 / scale) once per row, then per value q0 = RN(x r), e = RN(x - scale q0)
// (exact, one fused multiply-add) and q = RN(q0 + e r). Three rounded operations instead of a
// full division per value. For scales in [2^-100, 2^100] it equals the IEEE quotient for every
// bf16 x with |x| <= 448 scale whenever |x / scale| >= 2^-11, and gives a value of the same sign
// below 2^-11 in magnitude, where every such value has the code +-0 (an exhaustive check over
// all bf16 pairs is part of the tests); other scales divide directly.
#pragma once

#include <cuda_fp8.h>

namespace hs2 {

__device__ __forceinline__ float fp8_row_scale(float amax) {
  return amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
}

// The per-row constant of fp8_quotient: RN(1 / scale), or 0 to divide directly.
__device__ __forceinline__ float fp8_row_recip(float sc) {
  return (sc >= 0x1p-100f && sc <= 0x1p100f) ? __frcp_rn(sc) : 0.f;
}

// RN(x / sc), given rc = fp8_row_recip(sc)
__device__ __forceinline__ float fp8_quotient(float x, float sc, float rc) {
  if (rc == 0.f) return __fdiv_rn(x, sc);
  const float q0 = __fmul_rn(x, rc);
  const float e = __fmaf_rn(-sc, q0, x);
  return __fmaf_rn(e, rc, q0);
}

// two codes (low byte = a) of a row whose scale is sc (rc = fp8_row_recip(sc))
__device__ __forceinline__ uint32_t fp8_pair(float a, float b, float sc, float rc) {
  return __nv_cvt_float2_to_fp8x2(make_float2(fp8_quotient(a, sc, rc), fp8_quotient(b, sc, rc)),
                                  __NV_SATFINITE, __NV_E4M3);
}

}  // namespace hs2
