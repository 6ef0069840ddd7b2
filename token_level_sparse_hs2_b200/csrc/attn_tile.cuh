// attn_tile.cuh -- warp-level pieces of MQA attention over one shared-memory K/V tile.
//
// A warp owns 16 query-head rows and NT*8 cache rows of a 64-row tile. Tensor-core fragment
// conventions (mma.sync m16n8k16, g = lane / 4, c = lane % 4):
//   A (16 x 16, row):  a0a1 = A[g][2c..], a2a3 = A[g+8][2c..], a4a5 = A[g][2c+8..], a6a7 = A[g+8][2c+8..]
//   B (16 x 8, col):   b0 = B[2c..2c+1][g], b1 = B[2c+8..2c+9][g]
//   C (16 x 8):        c0,c1 = C[g][2c, 2c+1], c2,c3 = C[g+8][2c, 2c+1]
// S = Q . K^T has heads as rows and cache rows as columns; O += P . V has heads as rows and
// head_dim as columns, so two adjacent n8 tiles of S are directly one A fragment of P.
//
// Two cache formats:
//  * bf16: K/V tiles are [64][256 B] as two 128-byte swizzled boxes; bf16 MMAs; fragments
//    via ldmatrix (K) and ldmatrix.trans (V).
//  * e4m3: K/V tiles are [64][128 B], one swizzled box. Codes are widened exactly to f16 in
//    registers (cvt e4m3x2 -> f16x2) and f16 MMAs are used:
//      - K: ldmatrix on byte pairs gives lane (g,c) the 4 codes of dims 16*kb + 4c..4c+3 of
//        row g, so the K step's slots (2c, 2c+1, 2c+8, 2c+9) carry dims 4c..4c+3; Q's A
//        fragments are built with the same dim order.
//      - V: ldmatrix.trans on byte pairs gives lane (g,c) rows 2c, 2c+1 of dims 2g, 2g+1; a
//        byte permute splits them into an even-dim and an odd-dim B fragment, so output n8
//        tile 2*kb + parity holds dims 16*kb + 2*n + parity.
//      - Q is scaled by an exact power of two per head (2^-e_h) so its f16 copy keeps every
//        bf16 bit; the factor returns in the logit scale.
//      - The per-token V scale multiplies P; P is divided by the tile's largest V scale so
//        it stays in [0, 1] for f16, and the output accumulator is kept in units of the
//        current tile's reference scale (rescaled together with the softmax correction).
#pragma once

#include "common.cuh"

namespace hs2 {

enum KvType { kKvBf16 = 0, kKvFp8 = 1 };

__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);   // .x = lo
  return *reinterpret_cast<uint32_t *>(&v);
}

__device__ __forceinline__ void mma_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                        uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// two e4m3fn codes (low byte -> low half) to an exact f16 pair
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two) {
  uint32_t out;
  asm("{\n .reg .b16 t;\n cvt.u16.u32 t, %1;\n cvt.rn.f16x2.e4m3x2 %0, t;\n}\n"
      : "=r"(out)
      : "r"(two));
  return out;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// byte offset of (row r, byte b) in a [rows][128 B] swizzled FP8 tile
__device__ __forceinline__ uint32_t fp8_off(int r, int b) {
  return r * 128 + ((((b >> 4)) ^ (r & 7)) << 4) + (b & 15);
}

// Tile layouts. kSwz: TMA tiles with the 128-byte swizzle (tile_off / fp8_off). kPad: rows
// copied one by one (bulk copies) at a padded stride of 272 B (bf16) or 144 B (e4m3) -- 16
// bytes past the row, which spreads the 8 rows of an ldmatrix over distinct bank groups.
enum TileLayout { kSwz = 0, kPad = 1 };
constexpr int kPadRowBf16 = 272;
constexpr int kPadRowFp8 = 144;

template <int LAYOUT>
__device__ __forceinline__ uint32_t bf16_at(int r, int d) {
  if (LAYOUT == kSwz) return tile_off(kTile, r, d);
  return r * kPadRowBf16 + d * 2;
}

template <int LAYOUT>
__device__ __forceinline__ uint32_t fp8_at(int r, int b) {
  if (LAYOUT == kSwz) return fp8_off(r, b);
  return r * kPadRowFp8 + b;
}

// head_dim column of output fragment (n8 tile n, column element e&1) for lane c
template <int KV>
__device__ __forceinline__ int o_col(int n, int ecol, int c) {
  if (KV == kKvBf16) return n * 8 + 2 * c + ecol;
  return 16 * (n >> 1) + 4 * c + 2 * ecol + (n & 1);
}

// ------------------------------------------------------------------ Q fragments

// bf16: the 8 A fragments of head rows [row0, row0+16) from a swizzled bf16 block in smem.
__device__ __forceinline__ void load_q_frags_bf16(uint32_t q_smem, int rows, int row0,
                                                  uint32_t (&qa)[8][4]) {
  const int lane = threadIdx.x & 31;
  const int i = lane >> 3, j = lane & 7;
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
    const int r = row0 + (i & 1) * 8 + j;
    const int d = ks * 16 + (i >> 1) * 8;
    ldsm_x4(q_smem + tile_off(rows, r, d), qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3]);
  }
}

// bf16 A fragments straight from global memory (rows row0.. of a [*, 128] bf16 array)
__device__ __forceinline__ void load_q_frags_bf16_global(const __nv_bfloat16 *q, int row0,
                                                         uint32_t (&qa)[8][4]) {
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const uint32_t *r0 = reinterpret_cast<const uint32_t *>(q + (size_t)(row0 + g) * kHeadDim);
  const uint32_t *r1 = reinterpret_cast<const uint32_t *>(q + (size_t)(row0 + g + 8) * kHeadDim);
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
    qa[ks][0] = r0[ks * 8 + c];
    qa[ks][1] = r1[ks * 8 + c];
    qa[ks][2] = r0[ks * 8 + 4 + c];
    qa[ks][3] = r1[ks * 8 + 4 + c];
  }
}

// e4m3 path: f16 A fragments (dim order of the e4m3 K fragments) of head rows
// [row0, row0+16) of a bf16 [H][128] global array, each head scaled by 2^-e_h (exact).
// Returns the two per-row factors 2^e_h in pow_row.
__device__ __forceinline__ void load_q_frags_f16(const __nv_bfloat16 *q, int row0,
                                                 uint32_t (&qa)[8][4], float (&pow_row)[2]) {
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const __nv_bfloat16 *row = q + (size_t)(row0 + g + 8 * h) * kHeadDim;
    float amax = 0.f;
    for (int d = c; d < kHeadDim; d += 4) amax = fmaxf(amax, fabsf(__bfloat162float(row[d])));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    int e = 0;
    if (amax > 0.f) e = ilogbf(amax) - 13;   // largest |q'| in [2^13, 2^14)
    const float down = ldexpf(1.f, -e);
    pow_row[h] = ldexpf(1.f, e);
#pragma unroll
    for (int kb = 0; kb < 8; ++kb) {
      const int d = kb * 16 + 4 * c;
      const float x0 = __bfloat162float(row[d]) * down, x1 = __bfloat162float(row[d + 1]) * down;
      const float x2 = __bfloat162float(row[d + 2]) * down, x3 = __bfloat162float(row[d + 3]) * down;
      qa[kb][h] = pack_f16(x0, x1);        // a0a1 (row g) / a2a3 (row g+8)
      qa[kb][2 + h] = pack_f16(x2, x3);    // a4a5 / a6a7
    }
  }
}

// ------------------------------------------------------------------ S = Q . K^T

template <int KV, int NT, int LAYOUT = kSwz>
__device__ __forceinline__ void qk_tile(const uint32_t (&qa)[8][4], uint32_t k_smem, int tok0,
                                        float (&s)[NT][4]) {
  const int lane = threadIdx.x & 31;
  const int i = lane >> 3, j = lane & 7;
#pragma unroll
  for (int n = 0; n < NT; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) s[n][e] = 0.f;
  if (KV == kKvBf16) {
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
#pragma unroll
      for (int np = 0; np < NT / 2; ++np) {
        const int r = tok0 + np * 16 + (i >> 1) * 8 + j;
        const int d = ks * 16 + (i & 1) * 8;
        uint32_t b0, b1, b2, b3;
        ldsm_x4(k_smem + bf16_at<LAYOUT>(r, d), b0, b1, b2, b3);
        mma_bf16(s[2 * np], qa[ks], b0, b1);
        mma_bf16(s[2 * np + 1], qa[ks], b2, b3);
      }
    }
  } else {
#pragma unroll
    for (int n = 0; n < NT; ++n) {
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        // matrix i covers dims block kb = 4*half + i of rows tok0 + 8n + 0..7
        const int r = tok0 + n * 8 + j;
        const int kb = 4 * half + i;
        uint32_t w[4];
        ldsm_x4(k_smem + fp8_at<LAYOUT>(r, kb * 16), w[0], w[1], w[2], w[3]);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint32_t b0 = e4m3x2_to_f16x2(w[q] & 0xffffu);
          const uint32_t b1 = e4m3x2_to_f16x2(w[q] >> 16);
          mma_f16(s[n], qa[4 * half + q], b0, b1);
        }
      }
    }
  }
}

// S[mt] = Q[mt] . K^T for MT m-tiles (16 heads each) sharing every K fragment: each fragment
// is loaded (and, for e4m3, widened) once and fed to all MT tensor-core products.
template <int KV, int MT, int NT, int LAYOUT = kSwz>
__device__ __forceinline__ void qk_tile_mt(const uint32_t (&qa)[MT][8][4], uint32_t k_smem,
                                           int tok0, float (&s)[MT][NT][4]) {
  const int lane = threadIdx.x & 31;
  const int i = lane >> 3, j = lane & 7;
#pragma unroll
  for (int m = 0; m < MT; ++m)
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) s[m][n][e] = 0.f;
  if (KV == kKvBf16) {
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
#pragma unroll
      for (int np = 0; np < NT / 2; ++np) {
        const int r = tok0 + np * 16 + (i >> 1) * 8 + j;
        const int d = ks * 16 + (i & 1) * 8;
        uint32_t b0, b1, b2, b3;
        ldsm_x4(k_smem + bf16_at<LAYOUT>(r, d), b0, b1, b2, b3);
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          mma_bf16(s[m][2 * np], qa[m][ks], b0, b1);
          mma_bf16(s[m][2 * np + 1], qa[m][ks], b2, b3);
        }
      }
    }
  } else {
#pragma unroll
    for (int n = 0; n < NT; ++n) {
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int r = tok0 + n * 8 + j;
        const int kb = 4 * half + i;
        uint32_t w[4];
        ldsm_x4(k_smem + fp8_at<LAYOUT>(r, kb * 16), w[0], w[1], w[2], w[3]);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint32_t b0 = e4m3x2_to_f16x2(w[q] & 0xffffu);
          const uint32_t b1 = e4m3x2_to_f16x2(w[q] >> 16);
#pragma unroll
          for (int m = 0; m < MT; ++m) mma_f16(s[m][n], qa[m][4 * half + q], b0, b1);
        }
      }
    }
  }
}

// 2^x for x <= 0 on the FMA pipe (Cody-Waite split x = j + f, j = rint(x) by the 1.5 * 2^23
// rounding trick, |f| <= 1/2): 2^f from the cubic that minimises the relative error on
// [-1/2, 1/2] (Remez exchange, tests/exp2_poly_fit.py; max 7.5e-5), then j is added to the
// exponent field. x is clamped at -125 so the exponent cannot wrap; 2^-125 is far below any
// score's resolution.
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  constexpr float kMagic = 12582912.f;
  x.x = fmaxf(x.x, -125.f);
  x.y = fmaxf(x.y, -125.f);
  const float2 t = fadd2(x, make_float2(kMagic, kMagic));
  const float2 r = fadd2(t, make_float2(-kMagic, -kMagic));
  const float2 f = ffma2(r, make_float2(-1.f, -1.f), x);
  float2 p = ffma2(f, make_float2(0.0551716685f, 0.0551716685f), make_float2(0.2426111251f, 0.2426111251f));
  p = ffma2(p, f, make_float2(0.6932609677f, 0.6932609677f));
  p = ffma2(p, f, make_float2(0.9999280572f, 0.9999280572f));
  return make_float2(__int_as_float(__float_as_int(p.x) + (__float_as_int(t.x) << 23)),
                     __int_as_float(__float_as_int(p.y) + (__float_as_int(t.y) << 23)));
}

// ------------------------------------------------------------------ O += P . V

template <int KV, int NT, int LAYOUT = kSwz>
__device__ __forceinline__ void pv_tile(const uint32_t (&pa)[NT / 2][4], uint32_t v_smem,
                                        int tok0, float (&o)[16][4]) {
  const int lane = threadIdx.x & 31;
  const int i = lane >> 3, j = lane & 7;
#pragma unroll
  for (int kk = 0; kk < NT / 2; ++kk) {
    if (KV == kKvBf16) {
#pragma unroll
      for (int dp = 0; dp < 8; ++dp) {
        const int r = tok0 + kk * 16 + (i & 1) * 8 + j;
        const int d = dp * 16 + (i >> 1) * 8;
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(v_smem + bf16_at<LAYOUT>(r, d), b0, b1, b2, b3);
        mma_bf16(o[2 * dp], pa[kk], b0, b1);
        mma_bf16(o[2 * dp + 1], pa[kk], b2, b3);
      }
    } else {
#pragma unroll
      for (int kp = 0; kp < 4; ++kp) {
        // matrices: (rows +0..7, dim block 2kp), (rows +8..15, 2kp), (+0..7, 2kp+1), (+8..15, 2kp+1)
        const int r = tok0 + kk * 16 + (i & 1) * 8 + j;
        const int kb = 2 * kp + (i >> 1);
        uint32_t w[4];
        ldsm_x4_t(v_smem + fp8_at<LAYOUT>(r, kb * 16), w[0], w[1], w[2], w[3]);
#pragma unroll
        for (int hb = 0; hb < 2; ++hb) {
          const uint32_t lo = prmt(w[2 * hb], 0, 0x3120);       // rows 0..7:  (even | odd)
          const uint32_t hi = prmt(w[2 * hb + 1], 0, 0x3120);   // rows 8..15
          const uint32_t be0 = e4m3x2_to_f16x2(lo & 0xffffu), bo0 = e4m3x2_to_f16x2(lo >> 16);
          const uint32_t be1 = e4m3x2_to_f16x2(hi & 0xffffu), bo1 = e4m3x2_to_f16x2(hi >> 16);
          const int kb2 = 2 * kp + hb;
          mma_f16(o[2 * kb2], pa[kk], be0, be1);
          mma_f16(o[2 * kb2 + 1], pa[kk], bo0, bo1);
        }
      }
    }
  }
}

// Row stride (floats) of a shared-memory block holding output rows for o_to_smem: with it, the
// float2 (bf16 layout) or float4 (e4m3 layout) accesses of a warp hit every bank once.
template <int KV>
constexpr int o_stride() { return KV == kKvBf16 ? 136 : 144; }

// Stores (first) or adds this warp's output fragments, row hh scaled by f[hh], into rows
// g and g + 8 of a [16][o_stride<KV>()] float block at base, in head_dim order.
template <int KV>
__device__ __forceinline__ void o_to_smem(float *base, const float (&o)[16][4],
                                          const float (&f)[2], bool first) {
  const int lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    float *row = base + (g + 8 * hh) * o_stride<KV>();
    if (KV == kKvBf16) {
#pragma unroll
      for (int n = 0; n < 16; ++n) {
        float2 *p = reinterpret_cast<float2 *>(row + n * 8 + 2 * c);
        float2 v = make_float2(o[n][2 * hh] * f[hh], o[n][2 * hh + 1] * f[hh]);
        if (!first) {
          const float2 u = *p;
          v.x += u.x;
          v.y += u.y;
        }
        *p = v;
      }
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        float4 *p = reinterpret_cast<float4 *>(row + 16 * j + 4 * c);
        float4 v = make_float4(o[2 * j][2 * hh] * f[hh], o[2 * j + 1][2 * hh] * f[hh],
                               o[2 * j][2 * hh + 1] * f[hh], o[2 * j + 1][2 * hh + 1] * f[hh]);
        if (!first) {
          const float4 u = *p;
          v.x += u.x;
          v.y += u.y;
          v.z += u.z;
          v.w += u.w;
        }
        *p = v;
      }
    }
  }
}

// ------------------------------------------------------------------ online softmax

// State of one warp over its 16 head rows (this lane owns rows g and g+8).
struct WarpSoftmax {
  float m[2];       // running max of the log2-domain logits
  float l[2];       // this lane's part of the running denominator
  float vref;       // e4m3 path: V-scale unit of the accumulator (starts at 1; always 1 for bf16)
  float o[16][4];   // output accumulator fragments

  __device__ __forceinline__ void init() {
    m[0] = m[1] = -INFINITY;
    l[0] = l[1] = 0.f;
    vref = 1.f;
#pragma unroll
    for (int n = 0; n < 16; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) o[n][e] = 0.f;
  }
};

// One online-softmax step. s holds raw dot products; x = s * rowf[row] * colk[col] is the
// log2-domain logit; invalid columns are -inf. colv: per-column V scale (e4m3) or unused.
//
// st.m is a reference, not necessarily the running max: it only moves (and the accumulator is
// rescaled) when some row's tile max exceeds it by more than kLazy, so P = 2^(x - m) stays
// below 2^kLazy (bf16 P: 2^8; f16 P: 2^4). The result is unchanged: O and the denominator
// share the reference, and the final log-sum-exp is m + log2(l). For e4m3 caches the V-scale
// reference st.vref likewise only moves when the tile's largest scale leaves
// [vref * 2^-8, vref * 2^11], which keeps P * v_scale / vref within f16 range.
template <int KV, int NT, int LAYOUT = kSwz>
__device__ __forceinline__ void softmax_pv_tile(WarpSoftmax &st, float (&s)[NT][4],
                                                const float (&rowf)[2],
                                                const float (&colk)[NT][2],
                                                const float (&colv)[NT][2],
                                                const bool (&valid)[NT][2], uint32_t v_smem,
                                                int tok0) {
  constexpr float kLazy = (KV == kKvBf16) ? 8.f : 4.f;
  float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
  for (int n = 0; n < NT; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float x = s[n][e] * rowf[e >> 1] * colk[n][e & 1];
      x = valid[n][e & 1] ? x : -INFINITY;
      s[n][e] = x;
      mx[e >> 1] = fmaxf(mx[e >> 1], x);
    }
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 1));
    mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 2));
  }
  const bool keep = __all_sync(0xffffffffu, mx[0] <= st.m[0] + kLazy && mx[1] <= st.m[1] + kLazy);
  float alpha[2] = {1.f, 1.f};
  if (!keep) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const float mnew = fmaxf(st.m[h], mx[h]);
      const float mref = (mnew == -INFINITY) ? 0.f : mnew;   // nothing valid yet: p = 0 below
      alpha[h] = fast_exp2(st.m[h] - mref);                  // st.m = -inf gives 0
      st.m[h] = (mnew == -INFINITY) ? -INFINITY : mref;
    }
  }
  const float mref0 = (st.m[0] == -INFINITY) ? 0.f : st.m[0];
  const float mref1 = (st.m[1] == -INFINITY) ? 0.f : st.m[1];
  float vmul[NT][2];
  float ofix = 1.f;
  if (KV == kKvFp8) {
    float vmax = 0.f;
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int e = 0; e < 2; ++e) vmax = fmaxf(vmax, valid[n][e] ? colv[n][e] : 0.f);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
    if (vmax > 0.f && (vmax > st.vref * 2048.f || vmax < st.vref * (1.f / 256.f))) {
      ofix = st.vref / vmax;   // the accumulator moves to units of vmax
      st.vref = vmax;
    }
    const float inv = 1.f / st.vref;
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      vmul[n][0] = colv[n][0] * inv;
      vmul[n][1] = colv[n][1] * inv;
    }
  }
  uint32_t pa[NT / 2][4];
  float rs[2] = {0.f, 0.f};
#pragma unroll
  for (int n = 0; n < NT; ++n) {
    float p[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      p[e] = fast_exp2(s[n][e] - ((e >> 1) ? mref1 : mref0));
      rs[e >> 1] += p[e];
      if (KV == kKvFp8) p[e] *= vmul[n][e & 1];
    }
    if (KV == kKvBf16) {
      pa[n >> 1][(n & 1) * 2 + 0] = pack_bf16(p[0], p[1]);
      pa[n >> 1][(n & 1) * 2 + 1] = pack_bf16(p[2], p[3]);
    } else {
      pa[n >> 1][(n & 1) * 2 + 0] = pack_f16(p[0], p[1]);
      pa[n >> 1][(n & 1) * 2 + 1] = pack_f16(p[2], p[3]);
    }
  }
#pragma unroll
  for (int h = 0; h < 2; ++h) st.l[h] = st.l[h] * alpha[h] + rs[h];
  const float a0 = alpha[0] * ofix, a1 = alpha[1] * ofix;
  if (!__all_sync(0xffffffffu, a0 == 1.f && a1 == 1.f)) {
#pragma unroll
    for (int n = 0; n < 16; ++n) {
      st.o[n][0] *= a0;
      st.o[n][1] *= a0;
      st.o[n][2] *= a1;
      st.o[n][3] *= a1;
    }
  }
  pv_tile<KV, NT, LAYOUT>(pa, v_smem, tok0, st.o);
}

}  // namespace hs2
