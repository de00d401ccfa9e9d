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
// division __fdiv_rn instead. The scale itself, amax / 448, is formed the
// same way with the divisor 448. tests/cuda/div_check.cu checks all of it bit
// for bit against __fdiv_rn: the scale for every bf16 amax, and the quotient
// and codes (scalar and packed paths) for every bf16 amax and every bf16 x
// with |x| <= amax.
#pragma once

#include "common.cuh"

namespace fp8bs {

// Byte permute (PTX prmt.b32, default mode): selector nibble bits 0-2 pick one
// of the 8 bytes {b, a}; bit 3 set replicates that byte's sign bit instead.
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// Per 16-bit half: a bf16 whose magnitude is max(|a|, |b|). The sign bits of
// the result are meaningless (mask them before use).
__device__ __forceinline__ uint32_t bf16x2_absmax(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Largest magnitude (as fp32) of the two halves of a bf16x2 absmax word.
__device__ __forceinline__ float absmax_to_float(uint32_t m2) {
  const uint32_t m = m2 & 0x7FFF7FFFu;
  const uint32_t hi = m >> 16, lo = m & 0xFFFFu;
  return __uint_as_float((hi > lo ? hi : lo) << 16);
}

__device__ __forceinline__ uint64_t pack_f32x2(float lo, float hi) {
  uint64_t d;
  asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(lo), "f"(hi));
  return d;
}

// s = fl32(amax / 448), correctly rounded, for a finite amax >= 0.
__device__ __forceinline__ float scale_of_amax(float amax) {
  if (amax >= 7.88860905e-31f) {  // 2^-100: quotient and residual stay normal
    // 1/448 = 2^-9 * 8/7 rounded to nearest: mantissa 8/7 * 2^23 =
    // 9586980.57... -> 9586981 = 0x924925
    const float r = __uint_as_float(0x3B124925u);
    const float q0 = __fmul_rn(amax, r);
    const float e = __fmaf_rn(-q0, 448.0f, amax);
    return __fmaf_rn(e, r, q0);
  }
  return __fdiv_rn(amax, 448.0f);
}

struct ScaleDivider {
  float s;
  float r;
  bool fast;       // Markstein allowed (per element checks still apply)
  bool fast_all;   // branch-free codes allowed for every element (see codes2)
  uint64_t nr2;    // (-r, -r) packed for fp32x2 arithmetic
  uint64_t s2;     // (s, s)
  uint64_t r2;     // (r, r)
  uint64_t ns2;    // (-s, -s)

  __device__ __forceinline__ explicit ScaleDivider(float scale) : s(scale) {
    r = __frcp_rn(scale);
    // s normal (>= 2^-126) keeps r finite and normal for every bf16 amax.
    fast = scale >= 1.17549435e-38f && scale <= 1.0e37f;
    fast_all = scale >= 8.27180613e-25f && scale <= 1.0e37f;  // s >= 2^-80
    nr2 = pack_f32x2(-r, -r);
    s2 = pack_f32x2(scale, scale);
    r2 = pack_f32x2(r, r);
    ns2 = pack_f32x2(-scale, -scale);
  }

  // -(x / s) of two values at once, Markstein's steps on -r = -1/s (fp32x2
  // instructions): q' = RN(x * -r), e = RN(q' * s + x), RN(e * -r + q'). For
  // x != 0 every step is the exact negation of the scalar form's (round to
  // nearest is symmetric: q' = -q0, e is the same residual, the result -q).
  // For x = +-0 the result is the zero of the opposite sign as well: the
  // residual is +0 (opposite zeros add to +0) and the last sum, -0 + -0 for
  // x = +0 and -0 + +0 for x = -0, rounds to -0 and +0.
  __device__ __forceinline__ void neg_quotient2_unchecked(float x0, float x1, float& q0,
                                                         float& q1) const {
    asm("{\n\t.reg .b64 x, q, e;\n\t"
        "mov.b64 x, {%2, %3};\n\t"
        "mul.rn.f32x2 q, x, %4;\n\t"
        "fma.rn.f32x2 e, q, %5, x;\n\t"
        "fma.rn.f32x2 q, e, %4, q;\n\t"
        "mov.b64 {%0, %1}, q;\n\t}"
        : "=f"(q0), "=f"(q1)
        : "f"(x0), "f"(x1), "l"(nr2), "l"(s2));
  }

  // E4M3 codes of two bf16 values packed as (lo, hi) halves of w (lo -> byte
  // 0) with their sign bits inverted: the conversion of -(x / s) (E4M3
  // rounding and saturation are symmetric, so only the sign bit differs from
  // the code of x / s, zeros included). fast_all only.
  __device__ __forceinline__ uint32_t flipped_codes2(uint32_t w) const {
    float q0, q1;
    neg_quotient2_unchecked(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u), q0, q1);
    return __nv_cvt_float2_to_fp8x2(make_float2(q0, q1), __NV_SATFINITE, __NV_E4M3);
  }

  // E4M3 codes of two bf16 values packed as (lo, hi) halves of w, for s > 0
  // (x0 = lo -> byte 0). With s >= 2^-80 both elements take the branch-free
  // path: the quotient is exact where it can be nonzero in E4M3 (|x| >=
  // 2^-100 and |x / s| >= 2^-100), and everywhere else it is below 2^-20, far
  // under the smallest E4M3 subnormal, so the code is the zero of x's sign
  // either way. Smaller scales take the checked path.
  __device__ __forceinline__ uint32_t codes2(uint32_t w) const {
    if (fast_all) return flipped_codes2(w) ^ 0x8080u;
    const float x0 = __uint_as_float(w << 16), x1 = __uint_as_float(w & 0xFFFF0000u);
    return __nv_cvt_float2_to_fp8x2(make_float2((*this)(x0), (*this)(x1)), __NV_SATFINITE,
                                    __NV_E4M3);
  }

  // Four codes: the two of w0 in bytes 0-1, the two of w1 in bytes 2-3.
  __device__ __forceinline__ uint32_t codes4(uint32_t w0, uint32_t w1) const {
    if (fast_all) return prmt(flipped_codes2(w0), flipped_codes2(w1), 0x5410u) ^ 0x80808080u;
    return prmt(codes2(w0), codes2(w1), 0x5410u);
  }

  // x / s of the magnitudes of two values at once (Markstein's steps on r,
  // fp32x2 instructions; each lane rounds exactly like the scalar form, since
  // q0 * (-s) + x == -q0 * s + x).
  __device__ __forceinline__ void quotient2_unchecked(float x0, float x1, float& q0,
                                                      float& q1) const {
    asm("{\n\t.reg .b64 x, q, e;\n\t"
        "mov.b64 x, {%2, %3};\n\t"
        "mul.rn.f32x2 q, x, %4;\n\t"
        "fma.rn.f32x2 e, q, %5, x;\n\t"
        "fma.rn.f32x2 q, e, %4, q;\n\t"
        "mov.b64 {%0, %1}, q;\n\t}"
        : "=f"(q0), "=f"(q1)
        : "f"(x0), "f"(x1), "l"(r2), "l"(ns2));
  }

  // The same four codes as codes4, formed from the quotients of the
  // magnitudes with the four input sign bits merged back (one prmt in
  // sign-replicate mode and one lop3). The weight-block kernel streams
  // measurably faster with this form (28672 x 4096: 54.9 against 58.1 us),
  // the activation and 2:4 kernels with codes4.
  __device__ __forceinline__ uint32_t codes4_sign_merged(uint32_t w0, uint32_t w1) const {
    if (!fast_all) return codes4(w0, w1);
    auto mag2 = [this](uint32_t w) {
      const uint32_t a = w & 0x7FFF7FFFu;
      float q0, q1;
      quotient2_unchecked(__uint_as_float(a << 16), __uint_as_float(a & 0xFFFF0000u), q0, q1);
      return static_cast<uint32_t>(
          __nv_cvt_float2_to_fp8x2(make_float2(q0, q1), __NV_SATFINITE, __NV_E4M3));
    };
    return prmt(mag2(w0), mag2(w1), 0x5410u) | (prmt(w0, w1, 0xFDB9u) & 0x80808080u);
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

// Codes of two bf16 pairs (as codes4) for a zero scale (an all-zero group or
// block): each element's signed zero.
__device__ __forceinline__ uint32_t zero_codes4(uint32_t w0, uint32_t w1) {
  return prmt(w0, w1, 0xFDB9u) & 0x80808080u;
}

// Encode 8 bf16 values (a uint4) into 8 E4M3 bytes (a uint2).
__device__ __forceinline__ uint2 encode8(const uint4 v, const ScaleDivider& d) {
  if (d.s == 0.0f) return make_uint2(zero_codes4(v.x, v.y), zero_codes4(v.z, v.w));
  return make_uint2(d.codes4(v.x, v.y), d.codes4(v.z, v.w));
}

// The same bytes through codes4_sign_merged.
__device__ __forceinline__ uint2 encode8_sign_merged(const uint4 v, const ScaleDivider& d) {
  if (d.s == 0.0f) return make_uint2(zero_codes4(v.x, v.y), zero_codes4(v.z, v.w));
  return make_uint2(d.codes4_sign_merged(v.x, v.y), d.codes4_sign_merged(v.z, v.w));
}

// ----------------------------------------------------------- UE8M0 scales --
// "Format d'échelle UE8M0": a scale stored as float8_e8m0fnu, a bare power of
// two 2^(c - 127) (8 exponent bits, no sign, no mantissa). Chosen as the
// smallest power of two s with 448 * s >= amax, so no element saturates.
//
// For amax = 1.f * 2^(E - 127) (E its biased exponent) and 448 = 1.75 * 2^8:
// 448 * 2^e >= amax  <=>  e >= E - 135 + log2(1.f / 1.75), and since 1.f / 1.75
// lies in (0.57, 1.15), the smallest such e is E - 135 when 1.f <= 1.75
// (mantissa field <= 0x600000) and E - 134 otherwise; the code is e + 127,
// clamped to 0..254 (zero and subnormal amax give code 0).
__device__ __forceinline__ uint32_t ue8m0_code_of_amax(float amax) {
  const uint32_t b = __float_as_uint(amax);
  const int eb = static_cast<int>(b >> 23);
  const int code = eb - 8 + ((b & 0x7FFFFFu) > 0x600000u ? 1 : 0);
  return eb == 0 ? 0u : static_cast<uint32_t>(min(max(code, 0), 254));
}

// 1 / s = 2^(127 - c) as an fp32 value (normal for c <= 253; 2^-127 for 254).
__device__ __forceinline__ float ue8m0_inv_scale(uint32_t code) {
  return code >= 254u ? __uint_as_float(0x00400000u) : __uint_as_float((254u - code) << 23);
}

// E4M3 codes of 8 bf16 values against a power-of-two scale: x * (1 / s) is
// exact wherever it is a normal fp32 value and otherwise rounded once, so it
// equals the IEEE quotient x / s; the product keeps the sign (also of zero)
// and never exceeds 448 in magnitude (|x| <= amax <= 448 s).
__device__ __forceinline__ uint32_t pow2_codes2(uint32_t w, uint64_t r2) {
  float q0, q1;
  asm("{\n\t.reg .b64 x, q;\n\t"
      "mov.b64 x, {%2, %3};\n\t"
      "mul.rn.f32x2 q, x, %4;\n\t"
      "mov.b64 {%0, %1}, q;\n\t}"
      : "=f"(q0), "=f"(q1)
      : "f"(__uint_as_float(w << 16)), "f"(__uint_as_float(w & 0xFFFF0000u)), "l"(r2));
  return __nv_cvt_float2_to_fp8x2(make_float2(q0, q1), __NV_SATFINITE, __NV_E4M3);
}

__device__ __forceinline__ uint2 encode8_pow2(const uint4 v, float inv_scale) {
  const uint64_t r2 = pack_f32x2(inv_scale, inv_scale);
  return make_uint2(prmt(pow2_codes2(v.x, r2), pow2_codes2(v.y, r2), 0x5410u),
                    prmt(pow2_codes2(v.z, r2), pow2_codes2(v.w, r2), 0x5410u));
}

// silu(g) = g * sigmoid(g) = g / (1 + e^-g) in fp32 with the fast exponential
// and divide (relative error below 1e-6); the exponent's argument is clamped
// at 80 so that 1 + e^-g stays finite (for g < -80 the result is then about
// g e^-80 instead of g e^g, both negligible next to any GEMM tolerance).
__device__ __forceinline__ float silu_f32(float g) {
  return __fdividef(g, 1.0f + __expf(fminf(-g, 80.0f)));
}

// bf16x2 absmax word of 8 bf16 values (see absmax_to_float).
__device__ __forceinline__ uint32_t absmax8(const uint4 v) {
  return bf16x2_absmax(bf16x2_absmax(v.x, v.y), bf16x2_absmax(v.z, v.w));
}

}  // namespace fp8bs
