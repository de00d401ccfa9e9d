// E4M3 encoding against a shared scale: q = e4m3_rn_satfinite(fl32(x / s)).
//
// Every element of a 1x128 group or a 128x128 block is divided by the same
// scale s = amax / 448. The quotient must be the IEEE round-to-nearest fp32
// quotient (one rounding, then one rounding to E4M3), so a plain multiply by
// 1/s is not enough. ScaleDivider uses Markstein's FMA correction (P.
// Markstein, "Computation of elementary functions on the IBM RISC System/6000
// processor", IBM J. Res. Dev. 34(1), 1990): with r = RN(1/s) and
// q0 = RN(x * r), the residual e = x - q0 * s is exact in one FMA and
// RN(q0 + e * r) is the correctly rounded x / s, as long as nothing
// underflows. The reciprocal is computed once per scale; elements that are
// zero or tiny (|x| < 2^-100), whose quotient is tiny (|x r| < 2^-100, where
// the quotient could be subnormal) or whose scale is subnormal take the IEEE
// division __fdiv_rn instead. tests/test_gpu_division.py checks the result
// bit for bit against __fdiv_rn for every bf16 amax and every bf16 x with
// |x| <= amax.
#pragma once

#include "common.cuh"

namespace fp8bs {

struct ScaleDivider {
  float s;
  float r;
  bool fast;      // Markstein allowed (per element checks still apply)
  bool fast_all;  // branch-free codes allowed for every element (see codes2)

  __device__ __forceinline__ explicit ScaleDivider(float scale) : s(scale) {
    r = __frcp_rn(scale);
    // s normal (>= 2^-126) keeps r finite and normal for every bf16 amax.
    fast = scale >= 1.17549435e-38f && scale <= 1.0e37f;
    fast_all = scale >= 8.27180613e-25f && scale <= 1.0e37f;  // s >= 2^-80
  }

  // Markstein's quotient without the range checks.
  __device__ __forceinline__ float quotient_unchecked(float x) const {
    const float q0 = __fmul_rn(x, r);
    const float e = __fmaf_rn(-q0, s, x);
    return __fmaf_rn(e, r, q0);
  }

  // E4M3 codes of two bf16 values packed as (lo, hi) halves of w, for s > 0.
  // With s >= 2^-80 every element goes through quotient_unchecked on its
  // magnitude and takes its sign bit from the input: the quotient is exact
  // where it can be nonzero in E4M3 (|x| >= 2^-100 and |x / s| >= 2^-100),
  // and everywhere else it is below 2^-20, far under the smallest E4M3
  // subnormal, so the code is the signed zero either way. Smaller scales take
  // the checked path.
  __device__ __forceinline__ uint32_t codes2(uint32_t w) const {
    const float x0 = __uint_as_float(w << 16), x1 = __uint_as_float(w & 0xFFFF0000u);
    if (fast_all) {
      const float q0 = quotient_unchecked(fabsf(x0)), q1 = quotient_unchecked(fabsf(x1));
      const uint32_t c = __nv_cvt_float2_to_fp8x2(make_float2(q0, q1), __NV_SATFINITE, __NV_E4M3);
      return c | ((w >> 8) & 0x80u) | ((w >> 16) & 0x8000u);
    }
    return __nv_cvt_float2_to_fp8x2(make_float2((*this)(x0), (*this)(x1)), __NV_SATFINITE,
                                    __NV_E4M3);
  }

  __device__ __forceinline__ float operator()(float x) const {
    const float q0 = __fmul_rn(x, r);
    // Markstein needs an exact residual (|x| >= 2^-100) and a normal quotient
    // (|q0| >= 2^-100); everything else (zeros, tiny values, tiny quotients,
    // subnormal scales) takes the IEEE division.
    if (fast && fabsf(x) >= 7.88860905e-31f && fabsf(q0) >= 7.88860905e-31f) {
      const float e = __fmaf_rn(-q0, s, x);
      return __fmaf_rn(e, r, q0);
    }
    return __fdiv_rn(x, s);
  }
};

// Two codes (x0 in the low byte) for a nonzero scale.
__device__ __forceinline__ uint32_t e4m3x2(const ScaleDivider& d, float x0, float x1) {
  return __nv_cvt_float2_to_fp8x2(make_float2(d(x0), d(x1)), __NV_SATFINITE, __NV_E4M3);
}

// One code; a zero scale (all-zero group or block) gives the element's signed zero.
__device__ __forceinline__ uint32_t e4m3_code_bf16(const ScaleDivider& d, uint32_t bf16_bits) {
  if (d.s == 0.0f) return (bf16_bits & 0x8000u) ? 0x80u : 0x00u;
  const float x = __uint_as_float(bf16_bits << 16);
  return static_cast<uint32_t>(__nv_cvt_float_to_fp8(d(x), __NV_SATFINITE, __NV_E4M3));
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Encode 8 bf16 values (a uint4) into 8 E4M3 bytes (a uint2).
__device__ __forceinline__ uint2 encode8(const uint4 v, const ScaleDivider& d) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t out[2] = {0u, 0u};
  if (d.s == 0.0f) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t lo = (w[i] & 0x8000u) ? 0x80u : 0u;
      const uint32_t hi = (w[i] & 0x80000000u) ? 0x80u : 0u;
      out[i >> 1] |= (lo | (hi << 8)) << ((i & 1) * 16);
    }
    return make_uint2(out[0], out[1]);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) out[i >> 1] |= d.codes2(w[i]) << ((i & 1) * 16);
  return make_uint2(out[0], out[1]);
}

// Largest |x| of 8 bf16 values.
__device__ __forceinline__ float amax8(const uint4 v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  float m = 0.0f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    m = fmaxf(m, fabsf(bf16_lo(w[i])));
    m = fmaxf(m, fabsf(bf16_hi(w[i])));
  }
  return m;
}

}  // namespace fp8bs
