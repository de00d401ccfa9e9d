// The C ABI of libfp8bs: argument validation, device checks, TMA descriptor
// encoding and the device error word. Every entry point validates its
// arguments before launching anything and returns an FP8BS_* status.
#include <atomic>
#include <cstdio>
#include <cstdlib>
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace fp8bs {

// The device error word: 0 = fine, otherwise an FP8BS_ERR_* code recorded by a
// kernel that gave up a bounded wait. Read and cleared by
// fp8bs_get_device_error().
__device__ int g_device_error = 0;

namespace {

std::atomic<long long> g_wait_limit{kDefaultWaitCycles};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Scale arrays (fp32 scales or UE8M0 codes) and expert indices are read with
// loads of at most 4 bytes.
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

int check_k(int64_t K) { return (K <= 0 || K % 128 != 0) ? FP8BS_ERR_SHAPE : FP8BS_OK; }

int from_cuda(cudaError_t e) { return e == cudaSuccess ? FP8BS_OK : FP8BS_ERR_CUDA; }

// Largest element count any single operand may have (int32 grid/TMA coordinates).
constexpr int64_t kMaxDim = (int64_t(1) << 31) - 1;

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

}  // namespace

int current_device_info(DeviceInfo* info) {
  static DeviceInfo cache[64];
  static std::once_flag flags[64];
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return FP8BS_ERR_CUDA;
  int st = FP8BS_OK;
  std::call_once(flags[dev], [&] {
    DeviceInfo d{dev, 0, 0, 0};
    if (cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      st = FP8BS_ERR_CUDA;
    cache[dev] = d;
  });
  if (st != FP8BS_OK) return st;
  *info = cache[dev];
  if (info->sm_count <= 0) return FP8BS_ERR_CUDA;
  if (info->major != 10 || info->minor != 0) return FP8BS_ERR_ARCH;
  return FP8BS_OK;
}

int encode_tmap_2d(void* map_out, const void* base, int elem_bytes, uint64_t inner,
                   uint64_t outer, uint64_t row_stride_bytes, uint32_t box_inner,
                   uint32_t box_outer, TmapSwizzle swizzle) {
  EncodeTiledFn fn = get_encode_fn();
  if (fn == nullptr) return FP8BS_ERR_CUDA;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_stride_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(static_cast<CUtensorMap*>(map_out),
                        elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_UINT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
                        const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE,
                        swizzle == kSwizzle128B  ? CU_TENSOR_MAP_SWIZZLE_128B
                        : swizzle == kSwizzle64B ? CU_TENSOR_MAP_SWIZZLE_64B
                                                 : CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FP8BS_OK : FP8BS_ERR_CUDA;
}

int encode_tmap_kblocks(void* map_out, const void* base, uint64_t block_bytes, uint64_t rows,
                        uint64_t n_blocks, uint64_t row_stride_bytes, uint32_t box_rows,
                        uint32_t box_blocks, TmapSwizzle swizzle) {
  EncodeTiledFn fn = get_encode_fn();
  if (fn == nullptr) return FP8BS_ERR_CUDA;
  const cuuint64_t dims[3] = {block_bytes, rows, n_blocks};
  const cuuint64_t strides[2] = {row_stride_bytes, block_bytes};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(block_bytes), box_rows, box_blocks};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(static_cast<CUtensorMap*>(map_out), CU_TENSOR_MAP_DATA_TYPE_UINT8, 3,
                        const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE,
                        swizzle == kSwizzle128B  ? CU_TENSOR_MAP_SWIZZLE_128B
                        : swizzle == kSwizzle64B ? CU_TENSOR_MAP_SWIZZLE_64B
                                                 : CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FP8BS_OK : FP8BS_ERR_CUDA;
}

long long wait_limit() { return g_wait_limit.load(); }

int* device_error_word() {
  static int* cache[64];
  static std::once_flag flags[64];
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::call_once(flags[dev], [&] {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_error) == cudaSuccess) cache[dev] = static_cast<int*>(p);
  });
  return cache[dev];
}

}  // namespace fp8bs

using namespace fp8bs;

extern "C" {

int fp8_quant_act_group128(const void* x_bf16, int64_t M, int64_t K, void* qa_e4m3, float* sa,
                           void* stream) {
  if (M < 0 || M > kMaxDim || K > kMaxDim) return FP8BS_ERR_SHAPE;
  if (int st = check_k(K)) return st;
  if (M == 0) return FP8BS_OK;
  if (!x_bf16 || !qa_e4m3 || !sa) return FP8BS_ERR_NULL;
  if (!aligned16(x_bf16) || !aligned16(qa_e4m3) || !aligned4(sa)) return FP8BS_ERR_ALIGN;
  DeviceInfo dev;
  if (int st = current_device_info(&dev)) return st;
  return from_cuda(launch_quant_act_group128(x_bf16, M, K, qa_e4m3, sa,
                                             static_cast<cudaStream_t>(stream)));
}

int fp8_quant_weight_block128(const void* w_bf16, int64_t N, int64_t K, void* qw_e4m3, float* sw,
                              void* stream) {
  if (N < 0 || N > 65535LL * 128 || K > kMaxDim) return FP8BS_ERR_SHAPE;
  if (int st = check_k(K)) return st;
  if (N == 0) return FP8BS_OK;
  if (!w_bf16 || !qw_e4m3 || !sw) return FP8BS_ERR_NULL;
  if (!aligned16(w_bf16) || !aligned16(qw_e4m3) || !aligned4(sw)) return FP8BS_ERR_ALIGN;
  DeviceInfo dev;
  if (int st = current_device_info(&dev)) return st;
  return from_cuda(launch_quant_weight_block128(w_bf16, N, K, qw_e4m3, sw,
                                                static_cast<cudaStream_t>(stream)));
}

int prune24_compress(const void* w_bf16, int64_t N, int64_t K, void* vals_e4m3, uint8_t* meta,
                     float* sw, void* w_pruned_bf16, void* stream) {
  if (N < 0 || N > 65535LL * 128 || K > kMaxDim) return FP8BS_ERR_SHAPE;
  if (int st = check_k(K)) return st;
  if (N == 0) return FP8BS_OK;
  if (!w_bf16 || !vals_e4m3 || !meta || !sw) return FP8BS_ERR_NULL;
  if (!aligned16(w_bf16) || !aligned16(vals_e4m3) || !aligned16(meta) || !aligned4(sw) ||
      (w_pruned_bf16 && !aligned16(w_pruned_bf16)))
    return FP8BS_ERR_ALIGN;
  DeviceInfo dev;
  if (int st = current_device_info(&dev)) return st;
  return from_cuda(launch_prune24_compress(w_bf16, N, K, vals_e4m3, meta, sw, w_pruned_bf16,
                                           static_cast<cudaStream_t>(stream)));
}

static int check_gemm_args(int64_t M, int64_t N, int64_t K) {
  if (M < 0 || N < 0 || M > kMaxDim || N > kMaxDim || K > kMaxDim) return FP8BS_ERR_SHAPE;
  if (int st = check_k(K)) return st;
  if (N % 8 != 0) return FP8BS_ERR_SHAPE;  // 16-byte rows of bf16 output
  return FP8BS_OK;
}

size_t fp8bs_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K, int sparse) {
  (void)M;
  (void)N;
  (void)K;
  (void)sparse;
  return 0;  // split-K partials are reduced in distributed shared memory
}

int fp8_block_gemm(const void* qa, const float* sa, const void* qw, const float* sw, void* y_bf16,
                   int64_t M, int64_t N, int64_t K, void* workspace, size_t workspace_bytes,
                   void* stream) {
  if (int st = check_gemm_args(M, N, K)) return st;
  if (M == 0 || N == 0) return FP8BS_OK;
  if (!qa || !sa || !qw || !sw || !y_bf16) return FP8BS_ERR_NULL;
  if (!aligned16(qa) || !aligned4(sa) || !aligned16(qw) || !aligned4(sw) || !aligned16(y_bf16))
    return FP8BS_ERR_ALIGN;
  if (workspace_bytes < fp8bs_gemm_workspace_bytes(M, N, K, 0)) return FP8BS_ERR_WORKSPACE;
  (void)workspace;
  int* err = device_error_word();
  if (err == nullptr) return FP8BS_ERR_CUDA;
  return launch_block_gemm(qa, sa, qw, sw, y_bf16, M, N, K, wait_limit(), err,
                           static_cast<cudaStream_t>(stream));
}

int fp8_block_gemm_quant(const void* qa, const float* sa, const void* qw, const float* sw,
                         void* y_bf16, void* qy_e4m3, float* sy, int64_t M, int64_t N, int64_t K,
                         void* workspace, size_t workspace_bytes, void* stream) {
  if (int st = check_gemm_args(M, N, K)) return st;
  if (N % 128 != 0) return FP8BS_ERR_SHAPE;  // whole 1x128 groups of Y
  if (M == 0 || N == 0) return FP8BS_OK;
  if (!qa || !sa || !qw || !sw || !qy_e4m3 || !sy) return FP8BS_ERR_NULL;
  if (M <= 256 && !y_bf16) return FP8BS_ERR_NULL;  // decode-sized M quantizes the stored Y
  if (!aligned16(qa) || !aligned4(sa) || !aligned16(qw) || !aligned4(sw) ||
      (y_bf16 && !aligned16(y_bf16)) || !aligned16(qy_e4m3) || !aligned4(sy))
    return FP8BS_ERR_ALIGN;
  if (workspace_bytes < fp8bs_gemm_workspace_bytes(M, N, K, 0)) return FP8BS_ERR_WORKSPACE;
  (void)workspace;
  int* err = device_error_word();
  if (err == nullptr) return FP8BS_ERR_CUDA;
  return launch_block_gemm(qa, sa, qw, sw, y_bf16, M, N, K, wait_limit(), err,
                           static_cast<cudaStream_t>(stream), qy_e4m3, sy);
}

int fp8_sparse24_gemm(const void* qa, const float* sa, const void* vals, const uint8_t* meta,
                      const float* sw, void* y_bf16, int64_t M, int64_t N, int64_t K,
                      void* workspace, size_t workspace_bytes, void* stream) {
  if (int st = check_gemm_args(M, N, K)) return st;
  if (M == 0 || N == 0) return FP8BS_OK;
  if (!qa || !sa || !vals || !meta || !sw || !y_bf16) return FP8BS_ERR_NULL;
  if (!aligned16(qa) || !aligned4(sa) || !aligned16(vals) || !aligned16(meta) ||
      !aligned4(sw) || !aligned16(y_bf16))
    return FP8BS_ERR_ALIGN;
  if (workspace_bytes < fp8bs_gemm_workspace_bytes(M, N, K, 1)) return FP8BS_ERR_WORKSPACE;
  (void)workspace;
  int* err = device_error_word();
  if (err == nullptr) return FP8BS_ERR_CUDA;
  return launch_sparse24_gemm(qa, sa, vals, meta, sw, y_bf16, M, N, K, wait_limit(), err,
                              static_cast<cudaStream_t>(stream));
}

int fp8_quant_act_group128_ue8m0(const void* x_bf16, int64_t M, int64_t K, void* qa_e4m3,
                                 uint8_t* sa_ue8m0, void* stream) {
  if (M < 0 || M > kMaxDim || K > kMaxDim) return FP8BS_ERR_SHAPE;
  if (int st = check_k(K)) return st;
  if (M == 0) return FP8BS_OK;
  if (!x_bf16 || !qa_e4m3 || !sa_ue8m0) return FP8BS_ERR_NULL;
  if (!aligned16(x_bf16) || !aligned16(qa_e4m3)) return FP8BS_ERR_ALIGN;
  DeviceInfo dev;
  if (int st = current_device_info(&dev)) return st;
  return from_cuda(launch_quant_act_group128_ue8m0(x_bf16, M, K, qa_e4m3, sa_ue8m0,
                                                   static_cast<cudaStream_t>(stream)));
}

int fp8_quant_weight_block128_ue8m0(const void* w_bf16, int64_t N, int64_t K, void* qw_e4m3,
                                    uint8_t* sw_ue8m0, void* stream) {
  if (N < 0 || N > 65535LL * 128 || K > kMaxDim) return FP8BS_ERR_SHAPE;
  if (int st = check_k(K)) return st;
  if (N == 0) return FP8BS_OK;
  if (!w_bf16 || !qw_e4m3 || !sw_ue8m0) return FP8BS_ERR_NULL;
  if (!aligned16(w_bf16) || !aligned16(qw_e4m3)) return FP8BS_ERR_ALIGN;
  DeviceInfo dev;
  if (int st = current_device_info(&dev)) return st;
  return from_cuda(launch_quant_weight_block128_ue8m0(w_bf16, N, K, qw_e4m3, sw_ue8m0,
                                                      static_cast<cudaStream_t>(stream)));
}

int fp8_block_gemm_ue8m0(const void* qa, const uint8_t* sa_ue8m0, const void* qw,
                         const uint8_t* sw_ue8m0, void* y_bf16, int64_t M, int64_t N, int64_t K,
                         void* workspace, size_t workspace_bytes, void* stream) {
  if (int st = check_gemm_args(M, N, K)) return st;
  if (M == 0 || N == 0) return FP8BS_OK;
  if (!qa || !sa_ue8m0 || !qw || !sw_ue8m0 || !y_bf16) return FP8BS_ERR_NULL;
  if (!aligned16(qa) || !aligned16(qw) ||
      !aligned16(y_bf16))
    return FP8BS_ERR_ALIGN;
  (void)workspace;
  (void)workspace_bytes;
  int* err = device_error_word();
  if (err == nullptr) return FP8BS_ERR_CUDA;
  return launch_block_gemm_ue8m0(qa, sa_ue8m0, qw, sw_ue8m0, y_bf16, M, N, K, wait_limit(), err,
                                 static_cast<cudaStream_t>(stream));
}

static int check_grouped_args(int64_t M, int64_t N, int64_t K, int64_t E) {
  if (int st = check_gemm_args(M, N, K)) return st;
  if (E < 1 || E > kMaxDim || (N > 0 && E > kMaxDim / N)) return FP8BS_ERR_SHAPE;
  return FP8BS_OK;
}

int fp8_grouped_gemm(const void* qa, const float* sa, const void* qw, const float* sw,
                     const int32_t* m_indices, void* y_bf16, int64_t M, int64_t N, int64_t K,
                     int64_t E, void* workspace, size_t workspace_bytes, void* stream) {
  if (int st = check_grouped_args(M, N, K, E)) return st;
  if (M == 0 || N == 0) return FP8BS_OK;
  if (!qa || !sa || !qw || !sw || !m_indices || !y_bf16) return FP8BS_ERR_NULL;
  if (!aligned16(qa) || !aligned4(sa) || !aligned16(qw) || !aligned4(sw) ||
      !aligned4(m_indices) || !aligned16(y_bf16))
    return FP8BS_ERR_ALIGN;
  (void)workspace;
  (void)workspace_bytes;
  int* err = device_error_word();
  if (err == nullptr) return FP8BS_ERR_CUDA;
  return launch_block_gemm_grouped(qa, sa, qw, sw, m_indices, y_bf16, M, N, K, E, wait_limit(),
                                   err, static_cast<cudaStream_t>(stream));
}

int fp8_grouped_gemm_ue8m0(const void* qa, const uint8_t* sa_ue8m0, const void* qw,
                           const uint8_t* sw_ue8m0, const int32_t* m_indices, void* y_bf16,
                           int64_t M, int64_t N, int64_t K, int64_t E, void* workspace,
                           size_t workspace_bytes, void* stream) {
  if (int st = check_grouped_args(M, N, K, E)) return st;
  if (M == 0 || N == 0) return FP8BS_OK;
  if (!qa || !sa_ue8m0 || !qw || !sw_ue8m0 || !m_indices || !y_bf16) return FP8BS_ERR_NULL;
  if (!aligned16(qa) || !aligned16(qw) ||
      !aligned4(m_indices) || !aligned16(y_bf16))
    return FP8BS_ERR_ALIGN;
  (void)workspace;
  (void)workspace_bytes;
  int* err = device_error_word();
  if (err == nullptr) return FP8BS_ERR_CUDA;
  return launch_block_gemm_grouped_ue8m0(qa, sa_ue8m0, qw, sw_ue8m0, m_indices, y_bf16, M, N, K,
                                         E, wait_limit(), err, static_cast<cudaStream_t>(stream));
}

size_t fp8bs_swiglu_workspace_bytes(int64_t M, int64_t I) {
  if (M <= 0 || I <= 0 || M > kSwiGLUDecodeMaxM) return 0;
  return static_cast<size_t>(M) * static_cast<size_t>(2 * I) * 2;   // y [M][2I] bf16
}

int fp8_gemm_swiglu_quant(const void* qa, const float* sa, const void* qw_gate_up,
                          const float* sw_gate_up, void* h_bf16, void* qh_e4m3, float* sh,
                          int64_t M, int64_t I, int64_t K, void* workspace,
                          size_t workspace_bytes, void* stream) {
  if (M < 0 || I < 0 || M > kMaxDim || I > kMaxDim / 2 || K > kMaxDim) return FP8BS_ERR_SHAPE;
  if (int st = check_k(K)) return st;
  if (I % 128 != 0) return FP8BS_ERR_SHAPE;   // whole 1x128 groups of h, whole weight blocks
  if (M == 0 || I == 0) return FP8BS_OK;
  if (!qa || !sa || !qw_gate_up || !sw_gate_up || !qh_e4m3 || !sh) return FP8BS_ERR_NULL;
  if (!aligned16(qa) || !aligned4(sa) || !aligned16(qw_gate_up) || !aligned4(sw_gate_up) ||
      (h_bf16 && !aligned16(h_bf16)) || !aligned16(qh_e4m3) || !aligned4(sh))
    return FP8BS_ERR_ALIGN;
  const size_t need = fp8bs_swiglu_workspace_bytes(M, I);
  if (workspace_bytes < need) return FP8BS_ERR_WORKSPACE;
  if (need > 0 && (workspace == nullptr || !aligned16(workspace))) return FP8BS_ERR_WORKSPACE;
  int* err = device_error_word();
  if (err == nullptr) return FP8BS_ERR_CUDA;
  return launch_gemm_swiglu(qa, sa, qw_gate_up, sw_gate_up, h_bf16, qh_e4m3, sh, M, I, K,
                            workspace, wait_limit(), err, static_cast<cudaStream_t>(stream));
}

int fp8_gemm_swiglu_quant_noalloc(const void* qa, const float* sa, const void* qw_gate_up,
                                  const float* sw_gate_up, void* h_bf16, void* qh_e4m3,
                                  float* sh, int64_t M, int64_t I, int64_t K, void* stream) {
  if (M < 0 || I < 0 || M > kMaxDim || I > kMaxDim / 2 || K > kMaxDim) return FP8BS_ERR_SHAPE;
  if (int st = check_k(K)) return st;
  if (I % 128 != 0) return FP8BS_ERR_SHAPE;
  if (!swiglu_noalloc_fits(M, I)) return FP8BS_ERR_SCRATCH_LIMIT;
  if (int st = swiglu_noalloc_setup(nullptr)) return st;   // once per device, then cached
  if (M == 0 || I == 0) return FP8BS_OK;
  if (!qa || !sa || !qw_gate_up || !sw_gate_up || !qh_e4m3 || !sh) return FP8BS_ERR_NULL;
  if (!aligned16(qa) || !aligned4(sa) || !aligned16(qw_gate_up) || !aligned4(sw_gate_up) ||
      (h_bf16 && !aligned16(h_bf16)) || !aligned16(qh_e4m3) || !aligned4(sh))
    return FP8BS_ERR_ALIGN;
  int* err = device_error_word();
  if (err == nullptr) return FP8BS_ERR_CUDA;
  return launch_gemm_swiglu_noalloc(qa, sa, qw_gate_up, sw_gate_up, h_bf16, qh_e4m3, sh, M, I, K,
                                    wait_limit(), err, static_cast<cudaStream_t>(stream));
}

int fp8_gather_columns(const void* src_bf16, int64_t P, int64_t M, int64_t Np, void* dst_bf16,
                       void* stream) {
  if (P < 1 || M < 0 || Np < 0 || P > kMaxDim || M > kMaxDim || Np > kMaxDim) return FP8BS_ERR_SHAPE;
  if (Np % 8 != 0) return FP8BS_ERR_SHAPE;   // 16-byte chunks of bf16
  if (M == 0 || Np == 0) return FP8BS_OK;
  if (!src_bf16 || !dst_bf16) return FP8BS_ERR_NULL;
  if (!aligned16(src_bf16) || !aligned16(dst_bf16)) return FP8BS_ERR_ALIGN;
  DeviceInfo dev;
  if (int st = current_device_info(&dev)) return st;
  return from_cuda(launch_interleave_columns(src_bf16, P, M, Np, dst_bf16,
                                             static_cast<cudaStream_t>(stream)));
}

int fp8bs_get_device_error(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return FP8BS_ERR_CUDA;
  int v = 0;
  const int zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(int)) != cudaSuccess) return FP8BS_ERR_CUDA;
  if (v != 0 && cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int)) != cudaSuccess)
    return FP8BS_ERR_CUDA;
  return v;
}

void fp8bs_set_wait_limit(long long cycles) {
  g_wait_limit.store(cycles > 0 ? cycles : kDefaultWaitCycles);
}

const char* fp8bs_status_string(int status) {
  switch (status) {
    case FP8BS_OK: return "ok";
    case FP8BS_ERR_NULL: return "a required pointer is NULL";
    case FP8BS_ERR_SHAPE: return "invalid shape (K must be a positive multiple of 128; N a multiple of 8 for GEMMs)";
    case FP8BS_ERR_ALIGN: return "a pointer is not aligned (16 bytes for matrices, 4 for fp32 scales and indices)";
    case FP8BS_ERR_WORKSPACE: return "workspace too small";
    case FP8BS_ERR_CUDA: return "CUDA call failed";
    case FP8BS_ERR_DEVICE_TIMEOUT: return "a kernel gave up a bounded wait";
    case FP8BS_ERR_ARCH: return "device is not sm_100 (B200)";
    case FP8BS_ERR_SCRATCH_LIMIT:
      return "problem exceeds the 16 MiB device scratch of fp8_gemm_swiglu_quant_noalloc "
             "(M <= 256 needs M * 2I * 2 bytes)";
    default: return "unknown status";
  }
}

int fp8bs_version(void) { return 200; }

}  // extern "C"
