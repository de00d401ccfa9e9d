// Quantization kernels: dynamic 1x128 activation groups, 128x128 weight blocks.
//
// Rule ("FP8 à granularité fine", opening bullets): one fp32 scale per group of
// 128 input channels of a token (activations) or per 128x128 block (weights),
// s = amax / 448, code = e4m3(x / s) rounded to nearest-even and saturated to
// +-448; an all-zero group (s == 0) encodes signed zeros.
//
// Both kernels are HBM streaming kernels: 16-byte loads, one pass over the
// input, the scale written by the same kernel. Division is IEEE (__fdiv_rn)
// and conversion is the hardware cvt.rn.satfinite.e4m3x2.f32, so every byte is
// decided by a single fp32 division and a single rounding.
#include "common.cuh"
#include "kernels.h"

namespace fp8bs {

namespace {

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Encode 8 bf16 values (packed in a uint4) against scale s into 8 E4M3 bytes.
__device__ __forceinline__ uint2 encode8(const uint4 v, float s) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t out[2] = {0u, 0u};
  if (s == 0.0f) {
    // amax == 0: every element is +0 or -0; keep its sign.
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t lo = (w[i] & 0x8000u) ? 0x80u : 0u;
      const uint32_t hi = (w[i] & 0x80000000u) ? 0x80u : 0u;
      out[i >> 1] |= (lo | (hi << 8)) << ((i & 1) * 16);
    }
    return make_uint2(out[0], out[1]);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 r = make_float2(__fdiv_rn(bf16_lo(w[i]), s), __fdiv_rn(bf16_hi(w[i]), s));
    const uint32_t q = __nv_cvt_float2_to_fp8x2(r, __NV_SATFINITE, __NV_E4M3);
    out[i >> 1] |= q << ((i & 1) * 16);
  }
  return make_uint2(out[0], out[1]);
}

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

// X viewed flat: groups are consecutive runs of 128 elements (row-major
// [M][K] with K a multiple of 128), and the scale of flat group g is sa[g].
// A warp handles kUnits units of 4 groups (512 elements): lane i owns
// elements [8i, 8i+8) (group i/16) and [256+8i, 256+8i+8) (group 2+i/16), so
// each load and store instruction of the warp is contiguous.
template <int kUnits>
__global__ void __launch_bounds__(256) quant_act_group128_kernel(const uint4* __restrict__ x,
                                                                 uint2* __restrict__ qa,
                                                                 float* __restrict__ sa,
                                                                 int64_t n_groups) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t unit0 = warp * kUnits;

  uint4 v[kUnits][2];
  bool valid[kUnits][2];
#pragma unroll
  for (int u = 0; u < kUnits; ++u) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int64_t g = (unit0 + u) * 4 + 2 * h + (lane >> 4);
      valid[u][h] = g < n_groups;
      // element offset in uint4 (8 bf16) units: group g, 16-byte chunk lane % 16
      const int64_t idx = g * 16 + (lane & 15);
      v[u][h] = valid[u][h] ? __ldcs(x + idx) : make_uint4(0, 0, 0, 0);
    }
  }
#pragma unroll
  for (int u = 0; u < kUnits; ++u) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float m = amax8(v[u][h]);
#pragma unroll
      for (int off = 8; off >= 1; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
      const float s = __fdiv_rn(m, 448.0f);
      const int64_t g = (unit0 + u) * 4 + 2 * h + (lane >> 4);
      if (valid[u][h]) {
        qa[g * 16 + (lane & 15)] = encode8(v[u][h], s);
        if ((lane & 15) == 0) sa[g] = s;
      }
    }
  }
}

// One CTA of 256 threads per 128x128 block. Thread t owns the 16-byte chunk
// t % 16 of rows t/16 + 16 i (i = 0..7): 16 threads cover one 256-byte row.
__global__ void __launch_bounds__(256) quant_weight_block128_kernel(
    const __nv_bfloat16* __restrict__ w, uint8_t* __restrict__ qw, float* __restrict__ sw,
    int64_t N, int64_t K) {
  __shared__ float warp_max[8];
  const int t = threadIdx.x;
  const int64_t kb = blockIdx.x, nb = blockIdx.y;
  const int64_t KB = K / 128;
  const int chunk = t & 15;
  uint4 v[8];
  float m = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int64_t n = nb * 128 + i * 16 + (t >> 4);
    if (n < N) {
      v[i] = __ldcs(reinterpret_cast<const uint4*>(w + n * K + kb * 128) + chunk);
      m = fmaxf(m, amax8(v[i]));
    } else {
      v[i] = make_uint4(0, 0, 0, 0);
    }
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  if ((t & 31) == 0) warp_max[t >> 5] = m;
  __syncthreads();
  m = warp_max[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) m = fmaxf(m, warp_max[i]);
  const float s = __fdiv_rn(m, 448.0f);
  if (t == 0) sw[nb * KB + kb] = s;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int64_t n = nb * 128 + i * 16 + (t >> 4);
    if (n < N) {
      reinterpret_cast<uint2*>(qw + n * K + kb * 128)[chunk] = encode8(v[i], s);
    }
  }
}

}  // namespace

cudaError_t launch_quant_act_group128(const void* x, int64_t M, int64_t K, void* qa, float* sa,
                                      cudaStream_t stream) {
  constexpr int kUnits = 2;
  const int64_t n_groups = M * (K / 128);
  const int64_t units = (n_groups + 3) / 4;
  const int64_t warps = (units + kUnits - 1) / kUnits;
  const int64_t blocks = (warps + 7) / 8;
  if (blocks > 0x7FFFFFFF) return cudaErrorInvalidValue;
  quant_act_group128_kernel<kUnits><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
      static_cast<const uint4*>(x), static_cast<uint2*>(qa), sa, n_groups);
  return cudaGetLastError();
}

cudaError_t launch_quant_weight_block128(const void* w, int64_t N, int64_t K, void* qw, float* sw,
                                         cudaStream_t stream) {
  const int64_t NB = (N + 127) / 128, KB = K / 128;
  if (NB > 65535 || KB > 0x7FFFFFFF) return cudaErrorInvalidValue;
  dim3 grid(static_cast<unsigned>(KB), static_cast<unsigned>(NB));
  quant_weight_block128_kernel<<<grid, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(w),
                                                         static_cast<uint8_t*>(qw), sw, N, K);
  return cudaGetLastError();
}

}  // namespace fp8bs
