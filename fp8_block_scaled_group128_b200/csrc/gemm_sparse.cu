// 2:4 sparse block-scaled FP8 GEMM (placeholder until the sparse kernel lands).
#include "common.cuh"
#include "kernels.h"

namespace fp8bs {

int launch_sparse24_gemm(const void*, const float*, const void*, const uint8_t*, const float*,
                         void*, int64_t, int64_t, int64_t, long long, int*, cudaStream_t) {
  return FP8BS_ERR_CUDA;
}

}  // namespace fp8bs
