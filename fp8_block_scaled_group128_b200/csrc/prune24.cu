// 2:4 magnitude pruning along K, block quantization of the pruned weights and
// compression into (values, 2-bit metadata).
//
// Rule: in every group of 4 contiguous weights along K keep the two largest
// |w| ("Déployer la parcimonie 2:4 avec FP8 sur Hopper", steps 2 and 4 and
// the 2:4 mask example; "Combiner élagage et quantification ...", section on
// 2:4 sparsity); equal magnitudes go to the lower index; pruned weights
// become +0. Scales are then computed on the pruned 128x128 block (step 6 of
// the first page: prune, then recalibrate FP8).
//
// One CTA of 256 threads per 128x128 block, the same thread layout as the
// weight quantizer: thread t owns 8 consecutive weights (two groups of 4) of
// rows t/16 + 16 i. It writes 4 value bytes and 1 metadata byte per row.
#include "common.cuh"
#include "kernels.h"

namespace fp8bs {

namespace {

// Kept pair of a group of 4 bf16 magnitudes (sign cleared): rank each member
// by how many others beat it (larger magnitude, or equal magnitude at a lower
// index); ranks 0 and 1 are kept. Returns the nibble i0 | i1 << 2, i0 < i1.
__device__ __forceinline__ uint32_t select24(const uint32_t (&mag)[4]) {
  uint32_t keep = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    int beaten = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (j == i) continue;
      beaten += (mag[j] > mag[i]) || (mag[j] == mag[i] && j < i);
    }
    keep |= (beaten < 2 ? 1u : 0u) << i;
  }
  const uint32_t i0 = __ffs(keep) - 1;          // lowest kept position
  const uint32_t i1 = 31 - __clz(keep);         // highest kept position
  return i0 | (i1 << 2);
}

__device__ __forceinline__ uint32_t e4m3_code(uint32_t bf16_bits, float s) {
  if (s == 0.0f) return (bf16_bits & 0x8000u) ? 0x80u : 0x00u;
  const float x = __uint_as_float(bf16_bits << 16);
  const __nv_fp8_storage_t q = __nv_cvt_float_to_fp8(__fdiv_rn(x, s), __NV_SATFINITE, __NV_E4M3);
  return static_cast<uint32_t>(q);
}

__global__ void __launch_bounds__(256) prune24_compress_kernel(
    const __nv_bfloat16* __restrict__ w, int64_t N, int64_t K, uint8_t* __restrict__ vals,
    uint8_t* __restrict__ meta, float* __restrict__ sw, __nv_bfloat16* __restrict__ w_pruned) {
  __shared__ float warp_max[8];
  const int t = threadIdx.x;
  const int64_t kb = blockIdx.x, nb = blockIdx.y;
  const int64_t KB = K / 128;
  const int chunk = t & 15;

  uint32_t kept_bits[8][4];   // the 4 kept bf16 patterns (2 per group), per row
  uint32_t nibbles[8];
  float m = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int64_t n = nb * 128 + i * 16 + (t >> 4);
    uint4 v = make_uint4(0, 0, 0, 0);
    if (n < N) v = __ldcs(reinterpret_cast<const uint4*>(w + n * K + kb * 128) + chunk);
    const uint32_t words[4] = {v.x, v.y, v.z, v.w};
    uint32_t e[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      e[2 * j] = words[j] & 0xFFFFu;
      e[2 * j + 1] = words[j] >> 16;
    }
    uint32_t pruned[8];
    uint32_t nib2 = 0;
#pragma unroll
    for (int g = 0; g < 2; ++g) {
      const uint32_t mag[4] = {e[4 * g] & 0x7FFFu, e[4 * g + 1] & 0x7FFFu, e[4 * g + 2] & 0x7FFFu,
                               e[4 * g + 3] & 0x7FFFu};
      const uint32_t nib = select24(mag);
      const uint32_t i0 = nib & 3u, i1 = nib >> 2;
#pragma unroll
      for (int j = 0; j < 4; ++j) pruned[4 * g + j] = (j == i0 || j == i1) ? e[4 * g + j] : 0u;
      // kept values in position order; the block amax only sees kept values
      uint32_t k0 = 0, k1 = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (j == i0) k0 = e[4 * g + j];
        if (j == i1) k1 = e[4 * g + j];
      }
      kept_bits[i][2 * g] = k0;
      kept_bits[i][2 * g + 1] = k1;
      m = fmaxf(m, fabsf(__uint_as_float(k0 << 16)));
      m = fmaxf(m, fabsf(__uint_as_float(k1 << 16)));
      nib2 |= nib << (4 * g);
    }
    nibbles[i] = nib2;
    if (w_pruned != nullptr && n < N) {
      uint4 p;
      p.x = pruned[0] | (pruned[1] << 16);
      p.y = pruned[2] | (pruned[3] << 16);
      p.z = pruned[4] | (pruned[5] << 16);
      p.w = pruned[6] | (pruned[7] << 16);
      reinterpret_cast<uint4*>(w_pruned + n * K + kb * 128)[chunk] = p;
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
      uint32_t packed = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) packed |= e4m3_code(kept_bits[i][j], s) << (8 * j);
      // row n: 64 value bytes and 16 metadata bytes per 128-wide K-block
      reinterpret_cast<uint32_t*>(vals + n * (K / 2) + kb * 64)[chunk] = packed;
      meta[n * (K / 8) + kb * 16 + chunk] = static_cast<uint8_t>(nibbles[i]);
    }
  }
}

}  // namespace

cudaError_t launch_prune24_compress(const void* w, int64_t N, int64_t K, void* vals,
                                    uint8_t* meta, float* sw, void* w_pruned,
                                    cudaStream_t stream) {
  const int64_t NB = (N + 127) / 128, KB = K / 128;
  if (NB > 65535 || KB > 0x7FFFFFFF) return cudaErrorInvalidValue;
  dim3 grid(static_cast<unsigned>(KB), static_cast<unsigned>(NB));
  prune24_compress_kernel<<<grid, 256, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(w), N, K, static_cast<uint8_t*>(vals), meta, sw,
      static_cast<__nv_bfloat16*>(w_pruned));
  return cudaGetLastError();
}

}  // namespace fp8bs
