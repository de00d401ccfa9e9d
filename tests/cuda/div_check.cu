// Exhaustive check of the library's scale division (ScaleDivider) against
// CUDA's IEEE division __fdiv_rn, over the whole domain the quantizers use:
// s = fl32(amax / 448) for every positive finite bf16 amax, and every finite
// bf16 x with |x| <= amax (both signs). Also checks the E4M3 codes, both of
// the checked quotient and of the quantizers' branch-free pair path (both
// halves of the pair, the four-code forms), and the quantizers' scale
// amax / 448 for every amax.
#include <cstdint>

#include "../../fp8_block_scaled_group128_b200/csrc/e4m3_codec.cuh"

namespace {

struct Result {
  unsigned long long checked;
  unsigned long long quotient_mismatch;
  unsigned long long code_mismatch;
  uint32_t first_amax_bits;
  uint32_t first_x_bits;
};

__global__ void div_check_kernel(Result* res) {
  // blockIdx.x: amax bf16 pattern (1 .. 0x7F7F); threads: x patterns
  const uint32_t amax_bits = blockIdx.x + 1;
  const float amax = __uint_as_float(amax_bits << 16);
  const float s = __fdiv_rn(amax, 448.0f);
  const fp8bs::ScaleDivider d(s);
  unsigned long long n = 0, bad_q = 0, bad_c = 0;
  // the quantizers' scale amax / 448 (and the zero amax, once)
  if (threadIdx.x == 0) {
    bad_q += __float_as_uint(fp8bs::scale_of_amax(amax)) != __float_as_uint(s);
    if (blockIdx.x == 0) bad_q += __float_as_uint(fp8bs::scale_of_amax(0.0f)) != 0u;
  }
  for (uint32_t xb = threadIdx.x; xb < 0x10000u; xb += blockDim.x) {
    if ((xb & 0x7FFFu) > amax_bits) continue;   // |x| <= amax (same ordering as bits)
    const float x = __uint_as_float(xb << 16);
    const float q_ref = __fdiv_rn(x, s);
    const float q = d(x);
    ++n;
    if (__float_as_uint(q) != __float_as_uint(q_ref)) {
      ++bad_q;
      atomicCAS(&res->first_amax_bits, 0u, amax_bits);
      if (res->first_amax_bits == amax_bits) atomicCAS(&res->first_x_bits, 0u, xb | 0x10000u);
    }
    const uint32_t c = __nv_cvt_float_to_fp8(q, __NV_SATFINITE, __NV_E4M3);
    const uint32_t c_ref = __nv_cvt_float_to_fp8(q_ref, __NV_SATFINITE, __NV_E4M3);
    // the quantizers' pair path (x in the low half, +0 in the high half)
    const uint32_t c2 = d.codes2(xb) & 0xFFu;
    // both halves: x in the high half, -x in the low half
    const uint32_t c2p = d.codes2((xb << 16) | (xb ^ 0x8000u));
    // four at once: (x, -x) in the first word, (-x, x) in the second
    const uint32_t c4 = d.codes4((xb << 16) | (xb ^ 0x8000u), ((xb ^ 0x8000u) << 16) | xb);
    bad_c += (c4 != (c2p | ((((c2p & 0xFFu) << 8) | (c2p >> 8)) << 16)));
    // the weight-block kernel's form of the same four codes
    bad_c += (d.codes4_sign_merged((xb << 16) | (xb ^ 0x8000u), ((xb ^ 0x8000u) << 16) | xb) != c4);
    const uint32_t cn_ref =
        __nv_cvt_float_to_fp8(__fdiv_rn(-x, s), __NV_SATFINITE, __NV_E4M3);
    bad_c += (c != c_ref) + (c2 != c_ref) + ((c2p >> 8) != c_ref) + ((c2p & 0xFFu) != cn_ref);
  }
  atomicAdd(&res->checked, n);
  if (bad_q) atomicAdd(&res->quotient_mismatch, bad_q);
  if (bad_c) atomicAdd(&res->code_mismatch, bad_c);
}

}  // namespace

extern "C" int div_check(unsigned long long* out5) {
  Result* d = nullptr;
  if (cudaMalloc(&d, sizeof(Result)) != cudaSuccess) return 1;
  cudaMemset(d, 0, sizeof(Result));
  div_check_kernel<<<0x7F7F, 256>>>(d);
  Result h;
  const cudaError_t e = cudaMemcpy(&h, d, sizeof(Result), cudaMemcpyDeviceToHost);
  cudaFree(d);
  if (e != cudaSuccess || cudaGetLastError() != cudaSuccess) return 2;
  out5[0] = h.checked;
  out5[1] = h.quotient_mismatch;
  out5[2] = h.code_mismatch;
  out5[3] = h.first_amax_bits;
  out5[4] = h.first_x_bits;
  return 0;
}
