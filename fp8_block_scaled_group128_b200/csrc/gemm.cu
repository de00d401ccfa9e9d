// Dense block-scaled FP8 GEMM: shape dispatch onto the tcgen05 kernel of
// gemm_kernel.cuh ("FP8 à granularité fine": 1x128 activation groups against
// 128x128 weight blocks, fp32 scales, fp32 accumulation, bf16 output).
#include "gemm_kernel.cuh"

namespace fp8bs {

using namespace gemm_detail;

// Operand order of a dense GEMM. Up to 256 tokens the weights go on the MMA M
// side (decode order: the HBM-bound weight stream spread over the SMs, split
// over K where the tiles alone do not fill them). From 65 tokens on, a weight
// matrix wide enough to give the prefill-order kernel (128 tokens x 256 weight
// rows per tile) at least three quarters of a wave of tiles runs in prefill
// order instead: its promotion applies one scale per row, where the decode
// order's 128 x 128 tiles apply one per column, which paces them at 128 tokens
// (gate+up of Llama-3-8B at M = 128: 31.8 us in decode order, about 36 GB/s
// of weights per SM; 27.0 us in prefill order).
inline bool decode_order(int64_t M, int64_t N, int sm_count) {
  if (M > 256) return false;
  if (M <= 64) return true;
  const int64_t prefill_tiles = ((M + 127) / 128) * ((N + 255) / 256);
  return 4 * prefill_tiles < 3 * static_cast<int64_t>(sm_count);
}

int launch_block_gemm(const void* qa, const float* sa, const void* qw, const float* sw, void* y,
                      int64_t M, int64_t N, int64_t K, long long wait_limit, int* err,
                      cudaStream_t stream, void* qy, float* sy) {
  DeviceInfo dev;
  if (int st = current_device_info(&dev)) return st;
  GemmArgs a{};
  a.sa = sa;
  a.sw = sw;
  a.y = static_cast<__nv_bfloat16*>(y);
  a.M = static_cast<int>(M);
  a.N = static_cast<int>(N);
  a.KB = static_cast<int>(K / 128);
  a.NB = static_cast<int>((N + 127) / 128);
  a.wait_limit = wait_limit;
  a.err = err;
  a.qy = static_cast<uint8_t*>(qy);
  a.sy = sy;
  alignas(64) CUtensorMap ta, tb;

  const uint64_t KB = static_cast<uint64_t>(K / 128);
  // The next layer's quantization is fused into the epilogue for up to 16
  // tokens in decode order when the tiles are not split over K (a group of N
  // is a tile's 128 weight rows, staged per token for the Y stores), and above
  // 256 tokens in prefill order (a thread holds a group). In between, and with
  // a K split (a group spans the cluster), Y is written and then quantized by
  // the activation quantizer: timed on gate+up (28672 x 4096), the epilogue's
  // quantization sits on the last tile's critical path and cost more than the
  // second launch from 32 tokens on (64 tokens: 30.8 against 29.1 us; 128, in
  // prefill order: 30.2 against 29.5 us), and saved 0.6 us at 1 and 8.
  const bool decode = decode_order(M, N, dev.sm_count);
  const bool fuse_decode = decode && qy != nullptr && M <= 16 &&
                           choose_splits(static_cast<int>((N + 127) / 128), dev.sm_count,
                                         a.KB, 2) == 1;
  if (qy != nullptr && M <= 256 && !fuse_decode) {
    if (int st = launch_block_gemm(qa, sa, qw, sw, y, M, N, K, wait_limit, err, stream, nullptr,
                                   nullptr))
      return st;
    return launch_quant_act_group128(y, M, N, qy, sy, stream) == cudaSuccess ? FP8BS_OK
                                                                              : FP8BS_ERR_CUDA;
  }
  if (decode) {
    // Decode: weights on the MMA M side, tokens on the MMA N side; stages of
    // two K-blocks.
    constexpr int kKS = 2;
    const int BN = next_pow2_at_least16(M);
    a.row_tiles = static_cast<int>((N + 127) / 128);
    a.col_tiles = 1;
    const int tiles = a.row_tiles;
    const int S = choose_splits(tiles, dev.sm_count, a.KB, kKS);
    a.splits = S;
    const int grid_y = S > 1 ? tiles : (tiles < dev.sm_count ? tiles : dev.sm_count);
    if (int st = encode_tmap_kblocks(&ta, qw, 128, N, KB, K, 128, kKS, kSwizzle128B)) return st;
    if (int st = encode_tmap_kblocks(&tb, qa, 128, M, KB, K, BN, kKS, kSwizzle128B)) return st;
    if (fuse_decode)   // BN == 16 and S == 1 here
      return launch_cfg<16, true, false, 5, 1, kKS, true>(ta, tb, ta, a, grid_y, 1, stream);
    switch (BN) {
      case 16: return launch_cfg<16, true, false, 5, 1, kKS>(ta, tb, ta, a, grid_y, S, stream);
      case 32: return launch_cfg<32, true, false, 5, 1, kKS>(ta, tb, ta, a, grid_y, S, stream);
      case 64: return launch_cfg<64, true, false, 4, 1, kKS>(ta, tb, ta, a, grid_y, S, stream);
      case 128: return launch_cfg<128, true, false, 3, 2, kKS>(ta, tb, ta, a, grid_y, S, stream);
      default: return launch_cfg<256, true, false, 2, 2, kKS>(ta, tb, ta, a, grid_y, S, stream);
    }
  }
  // Prefill: tokens on the MMA M side, 256 weight rows on the MMA N side.
  constexpr int BN = 256;
  a.row_tiles = static_cast<int>((M + 127) / 128);
  a.col_tiles = static_cast<int>((N + BN - 1) / BN);
  a.splits = 1;
  const int64_t tiles = static_cast<int64_t>(a.row_tiles) * a.col_tiles;
  if (tiles > 0x7FFFFFFF) return FP8BS_ERR_SHAPE;
  const int grid_y = static_cast<int>(tiles < dev.sm_count ? tiles : dev.sm_count);
  if (int st = encode_tmap_kblocks(&ta, qa, 128, M, KB, K, 128, 1, kSwizzle128B)) return st;
  if (int st = encode_tmap_kblocks(&tb, qw, 128, N, KB, K, BN, 1, kSwizzle128B)) return st;
  if (qy != nullptr) return launch_cfg<BN, false, false, 3, 2, 1, true>(ta, tb, ta, a, grid_y, 1, stream);
  return launch_cfg<BN, false, false, 3, 2, 1>(ta, tb, ta, a, grid_y, 1, stream);
}

int launch_block_gemm_grouped(const void* qa, const float* sa, const void* qw, const float* sw,
                              const int* m_indices, void* y, int64_t M, int64_t N, int64_t K,
                              int64_t E, long long wait_limit, int* err, cudaStream_t stream) {
  // The prefill-order kernel for every M: tiles of 128 token rows (one
  // expert each) x 256 rows of that expert's weights.
  DeviceInfo dev;
  if (int st = current_device_info(&dev)) return st;
  GemmArgs a{};
  a.sa = sa;
  a.sw = sw;
  a.y = static_cast<__nv_bfloat16*>(y);
  a.M = static_cast<int>(M);
  a.N = static_cast<int>(N);
  a.KB = static_cast<int>(K / 128);
  a.NB = static_cast<int>((N + 127) / 128);
  a.wait_limit = wait_limit;
  a.err = err;
  a.m_indices = m_indices;
  a.E = static_cast<int>(E);
  constexpr int BN = 256;
  a.row_tiles = static_cast<int>((M + 127) / 128);
  a.col_tiles = static_cast<int>((N + BN - 1) / BN);
  a.splits = 1;
  const int64_t tiles = static_cast<int64_t>(a.row_tiles) * a.col_tiles;
  if (tiles > 0x7FFFFFFF) return FP8BS_ERR_SHAPE;
  const int grid_y = static_cast<int>(tiles < dev.sm_count ? tiles : dev.sm_count);
  const uint64_t KB = static_cast<uint64_t>(K / 128);
  alignas(64) CUtensorMap ta, tb;
  if (int st = encode_tmap_kblocks(&ta, qa, 128, M, KB, K, 128, 1, kSwizzle128B)) return st;
  if (int st = encode_tmap_kblocks(&tb, qw, 128, E * N, KB, K, BN, 1, kSwizzle128B)) return st;
  return launch_cfg<BN, false, false, 3, 2, 1>(ta, tb, ta, a, grid_y, 1, stream);
}

int launch_gemm_swiglu(const void* qa, const float* sa, const void* qw, const float* sw, void* h,
                       void* qh, float* sh, int64_t M, int64_t I, int64_t K, void* y_scratch,
                       long long wait_limit, int* err, cudaStream_t stream) {
  DeviceInfo dev;
  if (int st = current_device_info(&dev)) return st;
  if (M <= kSwiGLUDecodeMaxM && decode_order(M, 2 * I, dev.sm_count)) {
    // Decode-sized M: the decode-order GEMM of all 2I weight rows into the
    // scratch y [M][2I], then SwiGLU and the quantization per 1x128 group.
    if (int st = launch_block_gemm(qa, sa, qw, sw, y_scratch, M, 2 * I, K, wait_limit, err, stream))
      return st;
    return launch_swiglu_quant(y_scratch, M, I, h, qh, sh, stream) == cudaSuccess ? FP8BS_OK
                                                                                  : FP8BS_ERR_CUDA;
  }
  // The prefill-order kernel with the SwiGLU epilogue: a tile is 128 token
  // rows x 128 intermediate columns, i.e. gate rows [128 ct, +128) and up rows
  // [I + 128 ct, +128) of the [2I][K] weights (y_scratch unused).
  GemmArgs a{};
  a.sa = sa;
  a.sw = sw;
  a.y = static_cast<__nv_bfloat16*>(h);
  a.qy = static_cast<uint8_t*>(qh);
  a.sy = sh;
  a.M = static_cast<int>(M);
  a.N = static_cast<int>(2 * I);
  a.KB = static_cast<int>(K / 128);
  a.NB = static_cast<int>(2 * I / 128);
  a.swi = static_cast<int>(I);
  a.wait_limit = wait_limit;
  a.err = err;
  a.row_tiles = static_cast<int>((M + 127) / 128);
  a.col_tiles = static_cast<int>(I / 128);
  a.splits = 1;
  const int64_t tiles = static_cast<int64_t>(a.row_tiles) * a.col_tiles;
  if (tiles > 0x7FFFFFFF) return FP8BS_ERR_SHAPE;
  const int grid_y = static_cast<int>(tiles < dev.sm_count ? tiles : dev.sm_count);
  const uint64_t KB = static_cast<uint64_t>(K / 128);
  alignas(64) CUtensorMap ta, tb;
  if (int st = encode_tmap_kblocks(&ta, qa, 128, M, KB, K, 128, 1, kSwizzle128B)) return st;
  if (int st = encode_tmap_kblocks(&tb, qw, 128, 2 * I, KB, K, 128, 1, kSwizzle128B)) return st;
  return launch_cfg<256, false, false, 3, 2, 1, false, true>(ta, tb, ta, a, grid_y, 1, stream);
}

}  // namespace fp8bs
