// The fused gate/up GEMM + SwiGLU + 1x128 quantization without any device
// allocation by the caller or by this library: for decode-sized M the [M][2I]
// bf16 intermediate between the GEMM and the SwiGLU kernel lives in a fixed
// file-scope device array instead of a caller-provided workspace.
//
// Setup: the first call on a device (with that device current) looks up the
// array's device address with cudaGetSymbolAddress and caches it per device;
// make that first call before any stream capture. Every later call only reads
// the cached pointer. All calls on one device share the one array, so calls
// that overlap in time (two streams, or two host threads, without ordering
// between them) race on it.
#include <atomic>
#include <mutex>

#include <cuda_bf16.h>

#include "fp8bs.h"
#include "kernels.h"

namespace fp8bs {

namespace {

constexpr int64_t kScratchElems = kNoAllocScratchBytes / 2;   // bf16 elements

// Nothing in the array must start at zero: in each call the GEMM writes every
// element of y [M][2I] before the SwiGLU kernel, next on the same stream,
// reads it.
static __device__ __align__(256) __nv_bfloat16 g_swiglu_scratch[kScratchElems];

constexpr int kMaxDevices = 64;
std::atomic<void*> g_scratch_ptr[kMaxDevices];
std::mutex g_scratch_mu;

}  // namespace

int swiglu_noalloc_setup(void** scratch) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FP8BS_ERR_CUDA;
  void* p = g_scratch_ptr[dev].load(std::memory_order_acquire);
  if (p == nullptr) {
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    p = g_scratch_ptr[dev].load(std::memory_order_relaxed);
    if (p == nullptr) {
      const cudaError_t e = cudaGetSymbolAddress(&p, g_swiglu_scratch);
      if (e != cudaSuccess || p == nullptr) {
        (void)cudaGetLastError();   // clear the (non-sticky) error for later calls
        return FP8BS_ERR_CUDA;
      }
      g_scratch_ptr[dev].store(p, std::memory_order_release);
    }
  }
  if (scratch != nullptr) *scratch = p;
  return FP8BS_OK;
}

bool swiglu_noalloc_fits(int64_t M, int64_t I) {
  return M > kSwiGLUDecodeMaxM || M * 2 * I <= kScratchElems;
}

int launch_gemm_swiglu_noalloc(const void* qa, const float* sa, const void* qw, const float* sw,
                               void* h, void* qh, float* sh, int64_t M, int64_t I, int64_t K,
                               long long wait_limit, int* err, cudaStream_t stream) {
  if (!swiglu_noalloc_fits(M, I)) return FP8BS_ERR_SCRATCH_LIMIT;
  void* scratch = nullptr;
  if (int st = swiglu_noalloc_setup(&scratch)) return st;
  // Above kSwiGLUDecodeMaxM the fused kernel needs no scratch; the pointer is
  // passed and left unused.
  return launch_gemm_swiglu(qa, sa, qw, sw, h, qh, sh, M, I, K, scratch, wait_limit, err, stream);
}

}  // namespace fp8bs
