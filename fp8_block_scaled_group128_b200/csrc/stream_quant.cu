// Streaming quantizers over 128x128 bf16 tiles: activation groups (S1),
// weight blocks (S2) and 2:4 prune + compress (S4).
//
// Rules: "FP8 à granularité fine", opening bullets (one fp32 scale per 1x128
// group of a token, or per 128x128 weight block; s = amax / 448, code =
// e4m3(x / s) rounded to nearest-even, saturating); "Déployer la parcimonie
// 2:4 avec FP8 sur Hopper", steps 2, 4, 6 and the 2:4 mask example, and
// "Combiner élagage et quantification ...", section on 2:4 sparsity (keep the
// two largest |w| of each 4 along K, ties to the lower index, pruned -> +0;
// scales from the pruned block).
//
// All three are HBM streaming kernels. CTAs are persistent (two per SM); thread
// 0 keeps a 3-deep ring of 32 KB tiles in flight with TMA
// (cp.async.bulk.tensor, no swizzle, out-of-range rows read as zero), and all
// 512 threads work from shared memory. Thread t owns the 16-byte chunk t % 16
// of rows t/16 + 32 i (i = 0..3): 16 threads cover one 256-byte row, so every
// global store of a warp is contiguous. The element quotient x / s is the IEEE
// fp32 quotient (ScaleDivider) and the conversion is the hardware
// cvt.rn.satfinite.e4m3x2.f32.
#include <mutex>

#include "e4m3_codec.cuh"
#include "kernels.h"

namespace fp8bs {

namespace {

enum class QMode { kAct, kWeight, kPrune };

constexpr int kTileBytes = 128 * 128 * 2;
constexpr int kQStages = 3;
constexpr int kQThreads = 512;
constexpr int kQWarps = kQThreads / 32;
constexpr int kRowsPerThread = 128 * 16 / kQThreads;   // 16 threads per 256-byte row
constexpr int kQSmemBytes = kQStages * kTileBytes + 1024 + 512;

struct QArgs {
  int64_t rows;            // M (activations) or N (weights)
  int64_t K;
  int64_t row_tiles;       // ceil(rows / 128)
  int64_t num_tiles;       // row_tiles * K / 128
  uint8_t* q;              // codes [rows][K] (act / weight) or vals [N][K/2] (prune)
  uint8_t* meta;           // prune: [N][K/8]
  float* scale;            // act: [M][K/128]; weight / prune: [NB][K/128]
  __nv_bfloat16* pruned;   // prune: optional [N][K]
  long long wait_limit;
  int* err;
};

// 2:4 selection of one group of 4 bf16 values held in a 64-bit word (value j
// in bits 16j..16j+15). Each member gets the key (|w| bits << 2) | (3 - j):
// a larger magnitude wins, and equal magnitudes go to the lower index. The two
// largest keys (a 4-input max / second-max network) are the kept pair.
// Returns i0 | i1 << 2 (i0 < i1) and the two kept bf16 patterns in position
// order.
__device__ __forceinline__ uint32_t select24(uint64_t g, uint32_t& k0, uint32_t& k1) {
  uint32_t key[4];
#pragma unroll
  for (int j = 0; j < 4; ++j)
    key[j] = ((static_cast<uint32_t>(g >> (16 * j)) & 0x7FFFu) << 2) | static_cast<uint32_t>(3 - j);
  const uint32_t a = max(key[0], key[1]), b = min(key[0], key[1]);
  const uint32_t c = max(key[2], key[3]), d = min(key[2], key[3]);
  const uint32_t top1 = max(a, c);
  const uint32_t top2 = max(min(a, c), max(b, d));
  const uint32_t p1 = 3u - (top1 & 3u), p2 = 3u - (top2 & 3u);
  const uint32_t i0 = min(p1, p2), i1 = max(p1, p2);
  k0 = static_cast<uint32_t>(g >> (16 * i0)) & 0xFFFFu;
  k1 = static_cast<uint32_t>(g >> (16 * i1)) & 0xFFFFu;
  return i0 | (i1 << 2);
}

// 2:4 selection and encoding of the 8 weights (two groups) of one thread-row:
// returns the 4 value bytes, sets the metadata byte and the pruned bf16 words.
__device__ __forceinline__ uint32_t prune8(const uint4 v, const ScaleDivider& d, uint32_t& nib2,
                                           uint4& pruned) {
  const uint64_t g0 = (static_cast<uint64_t>(v.y) << 32) | v.x;
  const uint64_t g1 = (static_cast<uint64_t>(v.w) << 32) | v.z;
  uint32_t a0, a1, b0, b1;
  const uint32_t n0 = select24(g0, a0, a1);
  const uint32_t n1 = select24(g1, b0, b1);
  nib2 = n0 | (n1 << 4);
  uint32_t packed;
  if (d.s == 0.0f) {
    packed = ((a0 & 0x8000u) ? 0x80u : 0u) | ((a1 & 0x8000u) ? 0x8000u : 0u) |
             ((b0 & 0x8000u) ? 0x800000u : 0u) | ((b1 & 0x8000u) ? 0x80000000u : 0u);
  } else {
    packed = d.codes2(a0 | (a1 << 16)) | (d.codes2(b0 | (b1 << 16)) << 16);
  }
  // pruned weights: keep positions i0, i1 of each group, +0 elsewhere
  const uint64_t m0 = (0xFFFFull << (16 * (n0 & 3u))) | (0xFFFFull << (16 * (n0 >> 2)));
  const uint64_t m1 = (0xFFFFull << (16 * (n1 & 3u))) | (0xFFFFull << (16 * (n1 >> 2)));
  const uint64_t p0 = g0 & m0, p1 = g1 & m1;
  pruned = make_uint4(static_cast<uint32_t>(p0), static_cast<uint32_t>(p0 >> 32),
                      static_cast<uint32_t>(p1), static_cast<uint32_t>(p1 >> 32));
  return packed;
}

template <QMode kMode>
__global__ void __launch_bounds__(kQThreads, 2)
    stream_quant_kernel(const __grid_constant__ CUtensorMap tmap_x, const QArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kQStages * kTileBytes);
  float* red = reinterpret_cast<float*>(full + kQStages);   // [2][kQWarps] block-max partials
  volatile int* abort_flag = reinterpret_cast<volatile int*>(red + 2 * kQWarps);

  const int t = threadIdx.x;
  const int chunk = t & 15;
  const int64_t KB = a.K / 128;
  const int64_t first = blockIdx.x, step = gridDim.x;

  if (t == 0) {
    for (int s = 0; s < kQStages; ++s) mbar_init(&full[s], 1);
    *abort_flag = 0;
    fence_mbarrier_init();
    tma_prefetch_desc(&tmap_x);
  }
  __syncthreads();
  // No global memory was touched so far; the input may come from the
  // previous kernel of the stream.
  grid_dependency_wait();
  grid_launch_dependents();
  int issued = 0;
  if (t == 0) {
    for (int s = 0; s < kQStages; ++s) {
      const int64_t tile = first + s * step;
      if (tile >= a.num_tiles) break;
      mbar_arrive_expect_tx(&full[s], kTileBytes);
      tma_load_2d(smem + s * kTileBytes, &tmap_x, &full[s], static_cast<int32_t>((tile % KB) * 128),
                  static_cast<int32_t>((tile / KB) * 128));
      ++issued;
    }
  }

  int it = 0;
  for (int64_t tile = first; tile < a.num_tiles; tile += step, ++it) {
    const int s = it % kQStages;
    const uint32_t parity = static_cast<uint32_t>(it / kQStages) & 1u;
    const int64_t kb = tile % KB, rb = tile / KB;
    if (!mbar_wait(&full[s], parity, a.wait_limit)) {
      record_device_error(a.err, FP8BS_ERR_DEVICE_TIMEOUT);
      *abort_flag = 1;
    }
    uint4 v[kRowsPerThread];
    const uint8_t* buf = smem + s * kTileBytes;
#pragma unroll
    for (int i = 0; i < kRowsPerThread; ++i)
      v[i] = *reinterpret_cast<const uint4*>(buf + (i * (kQThreads / 16) + (t >> 4)) * 256 +
                                             chunk * 16);

    float m = 0.0f;
    if constexpr (kMode != QMode::kAct) {
#pragma unroll
      for (int i = 0; i < kRowsPerThread; ++i) m = fmaxf(m, amax8(v[i]));
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
      if ((t & 31) == 0) red[(it & 1) * kQWarps + (t >> 5)] = m;
    }
    // Every thread has read stage s (and published its block-max partial);
    // the proxy fence orders those reads before the TMA that refills stage s.
    fence_proxy_async_smem();
    __syncthreads();
    if (*abort_flag) break;
    if (t == 0) {
      const int64_t nt = tile + kQStages * step;
      if (nt < a.num_tiles) {
        mbar_arrive_expect_tx(&full[s], kTileBytes);
        tma_load_2d(smem + s * kTileBytes, &tmap_x, &full[s], static_cast<int32_t>((nt % KB) * 128),
                    static_cast<int32_t>((nt / KB) * 128));
        ++issued;
      }
    }

    if constexpr (kMode == QMode::kAct) {
      // one 1x128 group per row: 16 threads hold a row
#pragma unroll
      for (int i = 0; i < kRowsPerThread; ++i) {
        float rm = amax8(v[i]);
#pragma unroll
        for (int off = 8; off >= 1; off >>= 1) rm = fmaxf(rm, __shfl_xor_sync(0xffffffffu, rm, off));
        const int64_t r = rb * 128 + i * (kQThreads / 16) + (t >> 4);
        const float sc = __fdiv_rn(rm, 448.0f);
        if (r < a.rows) {
          reinterpret_cast<uint2*>(a.q + r * a.K + kb * 128)[chunk] = encode8(v[i], ScaleDivider(sc));
          if (chunk == 0) a.scale[r * KB + kb] = sc;
        }
      }
    } else {
      m = red[(it & 1) * kQWarps];
#pragma unroll
      for (int w = 1; w < kQWarps; ++w) m = fmaxf(m, red[(it & 1) * kQWarps + w]);
      const float sc = __fdiv_rn(m, 448.0f);
      if (t == 0) a.scale[rb * KB + kb] = sc;
      const ScaleDivider d(sc);
#pragma unroll
      for (int i = 0; i < kRowsPerThread; ++i) {
        const int64_t r = rb * 128 + i * (kQThreads / 16) + (t >> 4);
        if (r >= a.rows) continue;
        if constexpr (kMode == QMode::kWeight) {
          reinterpret_cast<uint2*>(a.q + r * a.K + kb * 128)[chunk] = encode8(v[i], d);
        } else {
          uint32_t nib2;
          uint4 pr;
          const uint32_t packed = prune8(v[i], d, nib2, pr);
          // row r: 64 value bytes and 16 metadata bytes per 128-wide K-block
          reinterpret_cast<uint32_t*>(a.q + r * (a.K / 2) + kb * 64)[chunk] = packed;
          a.meta[r * (a.K / 8) + kb * 16 + chunk] = static_cast<uint8_t>(nib2);
          if (a.pruned != nullptr)
            reinterpret_cast<uint4*>(a.pruned + r * a.K + kb * 128)[chunk] = pr;
        }
      }
    }
  }
  // Copies still in flight (only after an early stop) must land before exit.
  if (t == 0 && *abort_flag) {
    for (int s = 0; s < kQStages; ++s) {
      // the most recent phase issued on stage s, if any
      const int n_on_s = issued / kQStages + (s < issued % kQStages ? 1 : 0);
      if (n_on_s > 0) mbar_wait(&full[s], static_cast<uint32_t>(n_on_s - 1) & 1u, kDefaultWaitCycles);
    }
  }
}

template <QMode kMode>
cudaError_t launch_stream(const void* x, int64_t rows, int64_t K, QArgs a, cudaStream_t stream) {
  DeviceInfo dev;
  if (current_device_info(&dev) != FP8BS_OK) return cudaErrorInvalidDevice;
  alignas(64) CUtensorMap map;
  if (encode_tmap_2d(&map, x, 2, K, rows, K * 2, 128, 128, kSwizzleNone) != FP8BS_OK)
    return cudaErrorInvalidValue;
  a.rows = rows;
  a.K = K;
  a.row_tiles = (rows + 127) / 128;
  a.num_tiles = a.row_tiles * (K / 128);
  a.wait_limit = wait_limit();
  a.err = device_error_word();
  auto kern = stream_quant_kernel<kMode>;
  static std::once_flag flags[64];
  cudaError_t attr = cudaSuccess;
  std::call_once(flags[dev.device], [&] {
    attr = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kQSmemBytes);
  });
  if (attr != cudaSuccess) return attr;
  const int64_t ctas = a.num_tiles < 2LL * dev.sm_count ? a.num_tiles : 2LL * dev.sm_count;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(ctas), 1, 1);
  cfg.blockDim = dim3(kQThreads, 1, 1);
  cfg.dynamicSmemBytes = kQSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute pdl;
  pdl.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl.val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = &pdl;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, map, a);
}

}  // namespace

cudaError_t launch_quant_act_group128(const void* x, int64_t M, int64_t K, void* qa, float* sa,
                                      cudaStream_t stream) {
  QArgs a{};
  a.q = static_cast<uint8_t*>(qa);
  a.scale = sa;
  return launch_stream<QMode::kAct>(x, M, K, a, stream);
}

cudaError_t launch_quant_weight_block128(const void* w, int64_t N, int64_t K, void* qw, float* sw,
                                         cudaStream_t stream) {
  QArgs a{};
  a.q = static_cast<uint8_t*>(qw);
  a.scale = sw;
  return launch_stream<QMode::kWeight>(w, N, K, a, stream);
}

cudaError_t launch_prune24_compress(const void* w, int64_t N, int64_t K, void* vals,
                                    uint8_t* meta, float* sw, void* w_pruned,
                                    cudaStream_t stream) {
  QArgs a{};
  a.q = static_cast<uint8_t*>(vals);
  a.meta = meta;
  a.scale = sw;
  a.pruned = static_cast<__nv_bfloat16*>(w_pruned);
  return launch_stream<QMode::kPrune>(w, N, K, a, stream);
}

}  // namespace fp8bs
