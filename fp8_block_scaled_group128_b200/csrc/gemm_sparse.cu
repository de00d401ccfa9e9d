// 2:4 sparse block-scaled FP8 GEMM: the weight operand is given compressed
// (two kept E4M3 codes per group of 4 along K plus a 4-bit index nibble) as
// written by prune24_compress ("Déployer la parcimonie 2:4 avec FP8 sur
// Hopper": 2:4 groups along K; the result is defined as the dense block-scaled
// GEMM on the decompressed weights).
//
// The compressed weights always sit on the MMA M side (the 2:4 operand of
// tcgen05.mma.sp is A): tiles of 128 weight rows x BN tokens, BN <= 128 so that
// two partial buffers and the metadata fit the 512 TMEM columns. The metadata
// rows [n][K/8] are loaded as-is (16 bytes per row per 128-deep K-block) and
// copied into TMEM with tcgen05.cp, lane = weight row.
#include "gemm_kernel.cuh"

namespace fp8bs {

using namespace gemm_detail;

int launch_sparse24_gemm(const void* qa, const float* sa, const void* vals, const uint8_t* meta,
                         const float* sw, void* y, int64_t M, int64_t N, int64_t K,
                         long long wait_limit, int* err, cudaStream_t stream) {
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

  const int BN = M <= 128 ? next_pow2_at_least16(M) : 128;
  const int kKS = BN <= 32 ? 4 : 2;   // K-blocks per stage (bigger TMA copies)
  a.row_tiles = static_cast<int>((N + 127) / 128);
  a.col_tiles = static_cast<int>((M + BN - 1) / BN);
  const int64_t tiles64 = static_cast<int64_t>(a.row_tiles) * a.col_tiles;
  if (tiles64 > 65535LL * 148) return FP8BS_ERR_SHAPE;
  const int tiles = static_cast<int>(tiles64);
  const int S = choose_splits(tiles, dev.sm_count, a.KB, kKS);
  a.splits = S;
  const int grid_y = S > 1 ? tiles : (tiles < dev.sm_count ? tiles : dev.sm_count);

  const uint64_t KB = static_cast<uint64_t>(K / 128);
  alignas(64) CUtensorMap ta, tb, te;
  if (int st = encode_tmap_kblocks(&ta, vals, 64, N, KB, K / 2, 128, kKS, kSwizzle64B)) return st;
  if (int st = encode_tmap_kblocks(&te, meta, 16, N, KB, K / 8, 128, kKS, kSwizzleNone)) return st;
  if (int st = encode_tmap_kblocks(&tb, qa, 128, M, KB, K, BN, kKS, kSwizzle128B)) return st;
  switch (BN) {
    case 16: return launch_cfg<16, true, true, 4, 1, 4>(ta, tb, te, a, grid_y, S, stream);
    case 32: return launch_cfg<32, true, true, 3, 1, 4>(ta, tb, te, a, grid_y, S, stream);
    case 64: return launch_cfg<64, true, true, 5, 1, 2>(ta, tb, te, a, grid_y, S, stream);
    default: return launch_cfg<128, true, true, 3, 2, 2>(ta, tb, te, a, grid_y, S, stream);
  }
}

}  // namespace fp8bs
