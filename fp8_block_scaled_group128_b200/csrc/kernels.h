// Internal launchers behind the C ABI (validated arguments only).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace fp8bs {

cudaError_t launch_quant_act_group128(const void* x, int64_t M, int64_t K, void* qa, float* sa,
                                      cudaStream_t stream);
cudaError_t launch_quant_weight_block128(const void* w, int64_t N, int64_t K, void* qw, float* sw,
                                         cudaStream_t stream);
cudaError_t launch_prune24_compress(const void* w, int64_t N, int64_t K, void* vals,
                                    uint8_t* meta, float* sw, void* w_pruned,
                                    cudaStream_t stream);

// UE8M0 (power-of-two) scale variants: one code byte per group / block.
cudaError_t launch_quant_act_group128_ue8m0(const void* x, int64_t M, int64_t K, void* qa,
                                            uint8_t* sa8, cudaStream_t stream);
cudaError_t launch_quant_weight_block128_ue8m0(const void* w, int64_t N, int64_t K, void* qw,
                                               uint8_t* sw8, cudaStream_t stream);
int launch_block_gemm_ue8m0(const void* qa, const uint8_t* sa8, const void* qw, const uint8_t* sw8,
                            void* y, int64_t M, int64_t N, int64_t K, long long wait_limit,
                            int* err, cudaStream_t stream);

// Grouped (mixture-of-experts) block-scaled GEMMs: token row m uses the
// weights of expert m_indices[m] (weights [E][N][K]); every 128-row tile
// belongs to one expert. Return FP8BS_* status.
int launch_block_gemm_grouped(const void* qa, const float* sa, const void* qw, const float* sw,
                              const int* m_indices, void* y, int64_t M, int64_t N, int64_t K,
                              int64_t E, long long wait_limit, int* err, cudaStream_t stream);
int launch_block_gemm_grouped_ue8m0(const void* qa, const uint8_t* sa8, const void* qw,
                                    const uint8_t* sw8, const int* m_indices, void* y, int64_t M,
                                    int64_t N, int64_t K, int64_t E, long long wait_limit, int* err,
                                    cudaStream_t stream);

// The gate+up GEMM with SwiGLU and the next layer's 1x128 quantization in its
// epilogue: weights [W_gate; W_up] ([2I][K]); h = bf16(silu(gate) * up)
// ([M][I], h may be null), qh [M][I], sh [M][I/128]. Returns FP8BS_* status.
// Up to kSwiGLUDecodeMaxM tokens it may run as the decode GEMM into y_scratch
// ([M][2I] bf16, 16-byte aligned) followed by the SwiGLU quantization kernel
// (when the dense GEMM's dispatch picks the decode order for N = 2I);
// otherwise as one launch with the SwiGLU epilogue (y_scratch unused).
constexpr int64_t kSwiGLUDecodeMaxM = 256;
int launch_gemm_swiglu(const void* qa, const float* sa, const void* qw, const float* sw, void* h,
                       void* qh, float* sh, int64_t M, int64_t I, int64_t K, void* y_scratch,
                       long long wait_limit, int* err, cudaStream_t stream);

// The same with the decode path's y scratch in a fixed device array of
// kNoAllocScratchBytes (noalloc.cu): FP8BS_ERR_SCRATCH_LIMIT when M <= 256 and
// M * 2I * 2 bytes exceed it. swiglu_noalloc_setup looks up the array's
// address once per device (the current one) and returns it in *scratch.
constexpr int64_t kNoAllocScratchBytes = int64_t(16) << 20;
int swiglu_noalloc_setup(void** scratch);
bool swiglu_noalloc_fits(int64_t M, int64_t I);
int launch_gemm_swiglu_noalloc(const void* qa, const float* sa, const void* qw, const float* sw,
                               void* h, void* qh, float* sh, int64_t M, int64_t I, int64_t K,
                               long long wait_limit, int* err, cudaStream_t stream);

// Column shards gathered rank-major ([P][M][Np] bf16) -> full rows [M][P Np].
cudaError_t launch_interleave_columns(const void* src, int64_t P, int64_t M, int64_t Np, void* dst,
                                      cudaStream_t stream);

// SwiGLU + 1x128 quantization of a gate+up GEMM output y [M][2I] bf16.
cudaError_t launch_swiglu_quant(const void* y, int64_t M, int64_t I, void* h, void* qh, float* sh,
                                cudaStream_t stream);

// Dense block-scaled GEMM; with qy / sy also Y quantized in 1x128 groups along
// N for the next layer (y may then be null when M > 256). Returns FP8BS_* status.
int launch_block_gemm(const void* qa, const float* sa, const void* qw, const float* sw, void* y,
                      int64_t M, int64_t N, int64_t K, long long wait_limit, int* err,
                      cudaStream_t stream, void* qy = nullptr, float* sy = nullptr);

// 2:4 sparse block-scaled GEMM. Returns FP8BS_* status.
int launch_sparse24_gemm(const void* qa, const float* sa, const void* vals, const uint8_t* meta,
                         const float* sw, void* y, int64_t M, int64_t N, int64_t K,
                         long long wait_limit, int* err, cudaStream_t stream);

// Device address of the error word on the current device (cached per device).
int* device_error_word();

// Number of SMs and the sm major/minor of the current device (cached).
struct DeviceInfo {
  int device;
  int sm_count;
  int major;
  int minor;
};
int current_device_info(DeviceInfo* info);

// cuTensorMapEncodeTiled through the runtime's driver entry point: a 2-D
// tensor of bytes, `inner` contiguous x `outer` rows `row_stride_bytes` apart.
enum TmapSwizzle { kSwizzleNone = 0, kSwizzle64B = 64, kSwizzle128B = 128 };
int encode_tmap_2d(void* map_out, const void* base, int elem_bytes, uint64_t inner,
                   uint64_t outer, uint64_t row_stride_bytes, uint32_t box_inner,
                   uint32_t box_outer, TmapSwizzle swizzle);
inline int encode_tmap_2d_u8(void* map_out, const void* base, uint64_t inner, uint64_t outer,
                             uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer,
                             TmapSwizzle swizzle) {
  return encode_tmap_2d(map_out, base, 1, inner, outer, row_stride_bytes, box_inner, box_outer,
                        swizzle);
}

// A 3-D view of a row-major byte matrix [rows][row_stride_bytes] cut into
// K-blocks: dim 0 = `block_bytes` contiguous bytes of one K-block, dim 1 = the
// rows (`row_stride_bytes` apart), dim 2 = the K-blocks (`block_bytes` apart).
// A box {block_bytes, box_rows, box_blocks} lands in shared memory as
// box_blocks slabs of [box_rows][block_bytes].
int encode_tmap_kblocks(void* map_out, const void* base, uint64_t block_bytes, uint64_t rows,
                        uint64_t n_blocks, uint64_t row_stride_bytes, uint32_t box_rows,
                        uint32_t box_blocks, TmapSwizzle swizzle);

// Current bound of the kernels' mbarrier waits (SM cycles).
long long wait_limit();

}  // namespace fp8bs
