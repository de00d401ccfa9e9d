// The quantizers: activation groups (S1, act_quant_kernel), and, streaming
// 128x128 bf16 tiles, weight blocks (S2) and 2:4 prune + compress (S4).
//
// Rules: "FP8 à granularité fine", opening bullets (one fp32 scale per 1x128
// group of a token, or per 128x128 weight block; s = amax / 448, code =
// e4m3(x / s) rounded to nearest-even, saturating); "Déployer la parcimonie
// 2:4 avec FP8 sur Hopper", steps 2, 4, 6 and the 2:4 mask example, and
// "Combiner élagage et quantification ...", section on 2:4 sparsity (keep the
// two largest |w| of each 4 along K, ties to the lower index, pruned -> +0;
// scales from the pruned block).
//
// The tile kernel (S2, S4) streams HBM. CTAs are persistent (two per SM); thread
// 0 keeps a 3-deep ring of 32 KB tiles in flight with TMA
// (cp.async.bulk.tensor, no swizzle, out-of-range rows read as zero), and all
// T threads (512 for weight blocks, 256 for 2:4) work from shared memory.
// Thread t owns the 16-byte chunk t % 16 of rows t/16 + (T/16) i (i < 2048/T):
// 16 threads cover one 256-byte row, so every global store of a warp is
// contiguous. The element quotient x / s is the IEEE
// fp32 quotient (ScaleDivider) and the conversion is the hardware
// cvt.rn.satfinite.e4m3x2.f32.
#include <mutex>

#include "e4m3_codec.cuh"
#include "kernels.h"

namespace fp8bs {

namespace {

// kPruneOut: 2:4 prune + compress that also writes the pruned bf16 weights;
// kWeightE8: weight blocks with UE8M0 (power-of-two) scales.
enum class QMode { kWeight, kPrune, kPruneOut, kWeightE8 };

constexpr int kTileBytes = 128 * 128 * 2;
constexpr int kQStages = 3;
// Threads per CTA: 256 for the 2:4 modes (8 rows per thread, so the per-tile
// work -- the block max, the scale and its divider -- is spread over twice as
// many values: 28672 x 4096 59.8 -> 55.7 us), 512 for the weight blocks (4
// rows per thread; 56.2 against 58.4 us with 256).
template <QMode kMode>
struct QCfg {
  static constexpr int kThreads =
      (kMode == QMode::kPrune || kMode == QMode::kPruneOut) ? 256 : 512;
  static constexpr int kRowsPerThread = 128 * 16 / kThreads;   // 16 threads per 256-byte row
};
constexpr int kQSmemBytes = kQStages * kTileBytes + 1024 + 64;

struct QArgs {
  int64_t rows;            // M (activations) or N (weights)
  int64_t K;
  int64_t row_tiles;       // ceil(rows / 128)
  int64_t num_tiles;       // row_tiles * K / 128
  uint8_t* q;              // codes [rows][K] (act / weight) or vals [N][K/2] (prune)
  uint8_t* meta;           // prune: [N][K/8]
  float* scale;            // act: [M][K/128]; weight / prune: [NB][K/128]
  uint8_t* scale8;         // kWeightE8: UE8M0 codes [NB][K/128]
  __nv_bfloat16* pruned;   // prune: optional [N][K]
  long long wait_limit;
  int* err;
};

// |x| of both bf16 halves, and the lane mask of a >= b (0xFFFF per 16-bit
// lane where it holds), both on the half-precision pipe.
__device__ __forceinline__ uint32_t abs_bf16x2(uint32_t x) {
  uint32_t d;
  asm("abs.bf16x2 %0, %1;" : "=r"(d) : "r"(x));
  return d;
}

__device__ __forceinline__ uint32_t ge_bf16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("set.ge.u32.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// 2:4 selection, metadata and codes of the 8 weights (two groups of 4 along
// K) in one 16-byte chunk: group 0 in v.x (elements 0, 1) and v.y (2, 3),
// group 1 in v.z and v.w. Element j "beats" element i when |w_j| > |w_i|, or
// |w_j| == |w_i| and j < i; an element is kept when at most one other beats
// it, which keeps exactly two per group.
//
// Both groups are ranked at once in 16-bit lanes: E_j pairs element j of
// group 0 (low half) with element j of group 1 (high half); for i < j a
// packed bf16 comparison of the magnitudes (abs.bf16x2, set.ge.u32.bf16x2 on
// the half-precision pipe, which leaves the integer pipe to the rest) gives
// 0xFFFF in each lane where |w_i| >= |w_j|: for finite values the order of the
// magnitudes as numbers is that of their 15-bit patterns, and +0 and -0 tie.
// Each kept flag is then the majority of three such masks.
//
// Returns the 4 value bytes (kept codes of group 0 in position order, then
// group 1); sets the metadata byte (group 0 nibble in bits 0-3, group 1 in
// 4-7, nibble = i0 | i1 << 2) and, if kPruned, the pruned bf16 chunk.
template <bool kPruned>
__device__ __forceinline__ uint32_t prune8(const uint4 v, const ScaleDivider& d, uint32_t& meta,
                                           uint4& pruned) {
  const uint32_t e0 = prmt(v.x, v.z, 0x5410u), e1 = prmt(v.x, v.z, 0x7632u);
  const uint32_t e2 = prmt(v.y, v.w, 0x5410u), e3 = prmt(v.y, v.w, 0x7632u);
  const uint32_t g0 = abs_bf16x2(e0), g1 = abs_bf16x2(e1), g2 = abs_bf16x2(e2),
                 g3 = abs_bf16x2(e3);
  // c_ij (each lane all ones or zero): |w_i| >= |w_j|, i.e. i beats j (i < j)
  const uint32_t c01 = ge_bf16x2(g0, g1), c02 = ge_bf16x2(g0, g2), c03 = ge_bf16x2(g0, g3);
  const uint32_t c12 = ge_bf16x2(g1, g2), c13 = ge_bf16x2(g1, g3), c23 = ge_bf16x2(g2, g3);
  auto maj = [](uint32_t a, uint32_t b, uint32_t c) { return (a & b) | (a & c) | (b & c); };
  const uint32_t k0 = maj(c01, c02, c03);      // kept: beaten at most once
  const uint32_t k1 = maj(~c01, c12, c13);
  const uint32_t k2 = maj(~c02, ~c12, c23);
  const uint32_t k3 = maj(~c03, ~c13, ~c23);
  // i0 = 0 | 1 | 2 (first kept), i1 = 1 | 2 | 3 (last kept); the flags are
  // whole-lane masks, so each index bit is placed by its own constant: i0 and
  // i1 of group 0 in bits 0-1 and 8-9, of group 1 in bits 16-17 and 24-25
  const uint32_t sp = ((~k0 & k1 & 0x00010001u) | (~k0 & ~k1 & 0x00020002u)) |
                      (((k3 | ~k2) & 0x01000100u) | ((k3 | k2) & 0x02000200u));
  // metadata byte: nibbles i0 | i1 << 2 of group 0 in bits 0-3, of group 1 in
  // bits 4-7. sp * (1 + 2^6 + 2^12 + 2^18) adds four shifted copies of sp: the
  // fields at bits 0, 8, 16 and 24 land at bits 18, 20, 22 and 24, no two
  // partial sums overlap below bit 26 (so nothing carries into them), and the
  // byte is bits 18-25 (the caller stores the low 8 bits).
  meta = (sp * 0x41041u) >> 18;
  // kept bf16 values of each group in position order (halfwords i0 and i1):
  // byte selector 2i0 | (2i0 + 1) << 4 | 2i1 << 8 | (2i1 + 1) << 12, of which
  // prmt reads only the low 16 bits
  const uint32_t p0 = prmt(v.x, v.y, sp * 0x22u + 0x1010u);
  const uint32_t p1 = prmt(v.z, v.w, (sp >> 16) * 0x22u + 0x1010u);
  if constexpr (kPruned) {
    // 0xFFFF over kept halfwords: sign of bit 15 (group 0) or 31 (group 1)
    // of the kept flags, replicated
    pruned = make_uint4(v.x & prmt(k0, k1, 0xDD99u), v.y & prmt(k2, k3, 0xDD99u),
                        v.z & prmt(k0, k1, 0xFFBBu), v.w & prmt(k2, k3, 0xFFBBu));
  }
  if (d.s == 0.0f) return zero_codes4(p0, p1);
  return d.codes4(p0, p1);
}

template <QMode kMode>
__global__ void __launch_bounds__(QCfg<kMode>::kThreads, 2)
    stream_quant_kernel(const __grid_constant__ CUtensorMap tmap_x, const QArgs a) {
  constexpr int kQThreads = QCfg<kMode>::kThreads;
  constexpr int kRowsPerThread = QCfg<kMode>::kRowsPerThread;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kQStages * kTileBytes);
  // block max of tile `it` in slot it % 3, as the bits of a non-negative
  // float (ordered like the values): a slot is cleared two tiles ahead, after
  // everyone has read it
  unsigned* red = reinterpret_cast<unsigned*>(full + kQStages);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(red + 4);

  const int t = threadIdx.x;
  const int chunk = t & 15;
  const int KB = static_cast<int>(a.K / 128);
  // Tile index = rb * KB + kb; this CTA walks tiles blockIdx.x + j * gridDim.x.
  // The (rb, kb) of the current tile and of the next tile to load are
  // stepped without divisions.
  struct Cursor {
    int rb, kb;
  };
  const int step_rb = static_cast<int>(gridDim.x) / KB, step_kb = static_cast<int>(gridDim.x) % KB;
  auto advance = [&](Cursor& c) {
    c.kb += step_kb;
    c.rb += step_rb;
    if (c.kb >= KB) {
      c.kb -= KB;
      ++c.rb;
    }
  };
  const int64_t first = blockIdx.x, step = gridDim.x;
  Cursor cur{static_cast<int>(blockIdx.x) / KB, static_cast<int>(blockIdx.x) % KB};
  Cursor load = cur;

  if (t == 0) {
    for (int s = 0; s < kQStages; ++s) mbar_init(&full[s], 1);
    red[0] = red[1] = red[2] = 0u;
    *abort_flag = 0;
    fence_mbarrier_init();
    tma_prefetch_desc(&tmap_x);
  }
  __syncthreads();
  // No global memory was touched so far; the input may come from the
  // previous kernel of the stream. Its first tiles are prefetched into L2
  // meanwhile (a prefetch never changes what a later load reads).
  if (t == 0) {
    Cursor pf = load;
    for (int s = 0; s < kQStages; ++s) {
      if (first + s * step >= a.num_tiles) break;
      tma_prefetch_l2_2d(&tmap_x, pf.kb * 128, pf.rb * 128);
      advance(pf);
    }
  }
  grid_dependency_wait();
  grid_launch_dependents();
  int issued = 0;
  if (t == 0) {
    for (int s = 0; s < kQStages; ++s) {
      const int64_t tile = first + s * step;
      if (tile >= a.num_tiles) break;
      mbar_arrive_expect_tx(&full[s], kTileBytes);
      tma_load_2d(smem + s * kTileBytes, &tmap_x, &full[s], load.kb * 128, load.rb * 128);
      advance(load);
      ++issued;
    }
  }

  int it = 0;
  for (int64_t tile = first; tile < a.num_tiles; tile += step, ++it, advance(cur)) {
    const int s = it % kQStages;
    const uint32_t parity = static_cast<uint32_t>(it / kQStages) & 1u;
    const int64_t kb = cur.kb, rb = cur.rb;
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

    {
      uint32_t m2 = absmax8(v[0]);
#pragma unroll
      for (int i = 1; i < kRowsPerThread; ++i) m2 = bf16x2_absmax(m2, absmax8(v[i]));
      const unsigned mw = __reduce_max_sync(0xffffffffu, __float_as_uint(absmax_to_float(m2)));
      if ((t & 31) == 0) atomicMax(&red[it % 3], mw);
      if (t == 0) red[(it + 1) % 3] = 0u;   // read by everyone before the previous barrier
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
        tma_load_2d(smem + s * kTileBytes, &tmap_x, &full[s], load.kb * 128, load.rb * 128);
        advance(load);
        ++issued;
      }
    }

    if constexpr (kMode == QMode::kWeightE8) {
      const uint32_t code = ue8m0_code_of_amax(__uint_as_float(red[it % 3]));
      if (t == 0) a.scale8[rb * KB + kb] = static_cast<uint8_t>(code);
      const float inv = ue8m0_inv_scale(code);
      const int64_t r0 = rb * 128 + (t >> 4);
      const int rows_here = static_cast<int>(a.rows - r0 < 0 ? 0 : a.rows - r0);
#pragma unroll
      for (int i = 0; i < kRowsPerThread; ++i) {
        if (i * (kQThreads / 16) >= rows_here) break;
        const int64_t r = r0 + i * (kQThreads / 16);
        reinterpret_cast<uint2*>(a.q + r * a.K + kb * 128)[chunk] = encode8_pow2(v[i], inv);
      }
    } else {
      const float sc = scale_of_amax(__uint_as_float(red[it % 3]));
      if (t == 0) a.scale[rb * KB + kb] = sc;
      const ScaleDivider d(sc);
      // this thread's first row and its outputs; rows i step by kQThreads / 16
      const int64_t r0 = rb * 128 + (t >> 4);
      auto row = [&](int i) {
        const int64_t r = r0 + i * (kQThreads / 16);
        if constexpr (kMode == QMode::kWeight) {
          reinterpret_cast<uint2*>(a.q + r * a.K + kb * 128)[chunk] = encode8_sign_merged(v[i], d);
        } else {
          constexpr bool kOut = kMode == QMode::kPruneOut;
          uint32_t meta;
          uint4 pr;
          const uint32_t packed = prune8<kOut>(v[i], d, meta, pr);
          // row r: 64 value bytes and 16 metadata bytes per 128-wide K-block
          reinterpret_cast<uint32_t*>(a.q + r * (a.K / 2) + kb * 64)[chunk] = packed;
          a.meta[r * (a.K / 8) + kb * 16 + chunk] = static_cast<uint8_t>(meta);
          if constexpr (kOut) reinterpret_cast<uint4*>(a.pruned + r * a.K + kb * 128)[chunk] = pr;
        }
      };
      if ((rb + 1) * 128 <= a.rows) {
        // a whole row block (the same branch for the CTA): no row checks
#pragma unroll
        for (int i = 0; i < kRowsPerThread; ++i) row(i);
      } else {
        const int rows_here = static_cast<int>(a.rows - r0 < 0 ? 0 : a.rows - r0);
#pragma unroll
        for (int i = 0; i < kRowsPerThread; ++i) {
          if (i * (kQThreads / 16) >= rows_here) break;
          row(i);
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
  cfg.blockDim = dim3(QCfg<kMode>::kThreads, 1, 1);
  cfg.dynamicSmemBytes = kQSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute pdl;
  pdl.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl.val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = &pdl;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, map, a);
}

// Activation quantization (S1). A team of kTeam threads quantizes 1x128
// groups: each thread 128 / kTeam adjacent bf16 of a group (one or two
// 16-byte chunks), a kTeam-lane shuffle max, the encode of e4m3_codec.cuh,
// one store of its codes; the team's first thread writes the scale. A team
// takes kGroups groups spread over the grid (team, team + teams, ...) and
// issues all their loads before any arithmetic. Inputs that fill the GPU many
// times over use teams of 8 and 4 groups (128 bytes per thread in flight):
// with one chunk per thread the per-group work (the shuffle max, the scale
// and its divider) cost as many instructions as the codes and made the
// kernel ALU-bound (8192 x 14336: 62.1 -> 51.6 us); mid-sized inputs use
// teams of 8 with one group. Inputs of up to 8192 groups use teams of 16 and
// one group (the shortest path per thread, the lowest latency). Groups are
// contiguous in memory (row-major [M][K], K a multiple of 128) and the scale
// of group g is sa[g] (row-major [M][K/128]). No shared memory and no
// barrier: for decode-sized inputs the kernel costs one load round trip.
constexpr int kActThreads = 256;

template <int kGroups, int kTeam, bool kE8 = false>
__global__ void __launch_bounds__(kActThreads)
    act_quant_kernel(const __nv_bfloat16* __restrict__ x, int64_t groups,
                     uint8_t* __restrict__ q, void* __restrict__ scale) {
  static_assert(kTeam == 8 || kTeam == 16, "one or two 16-byte chunks per thread");
  constexpr int kChunks = 16 / kTeam;   // 16-byte chunks per thread
  // kE8: UE8M0 (power-of-two) scales, written as one code byte per group
  const int64_t teams = static_cast<int64_t>(gridDim.x) * (kActThreads / kTeam);
  const int64_t team =
      static_cast<int64_t>(blockIdx.x) * (kActThreads / kTeam) + (threadIdx.x / kTeam);
  const int part = threadIdx.x % kTeam;   // this thread's chunks: kChunks * part ...
  // While the previous kernel of the stream may still run, bring this
  // thread's input lines into L2 (one thread per 128-byte line): the
  // prefetch never changes what the loads below read, even if that kernel
  // writes x, and when it does not, the HBM latency overlaps the wait.
  if ((part * kChunks) % 8 == 0) {
#pragma unroll
    for (int j = 0; j < kGroups; ++j) {
      const int64_t g = team + j * teams;
      if (g < groups) prefetch_l2(reinterpret_cast<const uint4*>(x + g * 128) + kChunks * part);
    }
  }
  grid_dependency_wait();
  grid_launch_dependents();
  uint4 v[kGroups][kChunks];
#pragma unroll
  for (int j = 0; j < kGroups; ++j) {
    const int64_t g = team + j * teams;
    const uint4* src = reinterpret_cast<const uint4*>(x + g * 128) + kChunks * part;
#pragma unroll
    for (int c = 0; c < kChunks; ++c)
      v[j][c] = g < groups ? __ldg(src + c) : make_uint4(0u, 0u, 0u, 0u);
  }
#pragma unroll
  for (int j = 0; j < kGroups; ++j) {
    const int64_t g = team + j * teams;
    uint32_t m2 = absmax8(v[j][0]);
#pragma unroll
    for (int c = 1; c < kChunks; ++c) m2 = bf16x2_absmax(m2, absmax8(v[j][c]));
    float m = absmax_to_float(m2);
#pragma unroll
    for (int off = kTeam / 2; off >= 1; off >>= 1)
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    uint2 c8[kChunks];
    if constexpr (kE8) {
      const uint32_t code = ue8m0_code_of_amax(m);
      const float inv = ue8m0_inv_scale(code);
#pragma unroll
      for (int c = 0; c < kChunks; ++c) c8[c] = encode8_pow2(v[j][c], inv);
      if (g < groups && part == 0) static_cast<uint8_t*>(scale)[g] = static_cast<uint8_t>(code);
    } else {
      const float sc = scale_of_amax(m);
      const ScaleDivider d(sc);
#pragma unroll
      for (int c = 0; c < kChunks; ++c) c8[c] = encode8(v[j][c], d);
      if (g < groups && part == 0) static_cast<float*>(scale)[g] = sc;
    }
    if (g < groups) {
      if constexpr (kChunks == 2)
        reinterpret_cast<uint4*>(q + g * 128)[part] = make_uint4(c8[0].x, c8[0].y, c8[1].x, c8[1].y);
      else
        reinterpret_cast<uint2*>(q + g * 128)[part] = c8[0];
    }
  }
}

}  // namespace

namespace {

template <bool kE8>
cudaError_t launch_act(const void* x, int64_t M, int64_t K, void* qa, void* sa,
                       cudaStream_t stream) {
  DeviceInfo dev;
  if (current_device_info(&dev) != FP8BS_OK) return cudaErrorInvalidDevice;
  const int64_t groups = M * (K / 128);
  // teams of 16 with one group each for the smallest inputs (up to 8192
  // groups: the shortest path per thread); teams of 8, with four groups each
  // once teams of 8 would fill every SM (2048 threads) eight times over, else
  // with one
  const int form = groups <= 8192 ? 0 : groups >= 8LL * dev.sm_count * (2048 / 8) ? 2 : 1;
  const int64_t per_block = form == 0 ? kActThreads / 16 : form == 1 ? kActThreads / 8
                                                                     : (kActThreads / 8) * 4;
  const int64_t blocks = (groups + per_block - 1) / per_block;
  if (blocks > 0x7FFFFFFF) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(blocks), 1, 1);
  cfg.blockDim = dim3(kActThreads, 1, 1);
  cfg.stream = stream;
  cudaLaunchAttribute pdl;
  pdl.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl.val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = &pdl;
  cfg.numAttrs = 1;
  const auto* xp = static_cast<const __nv_bfloat16*>(x);
  auto* qp = static_cast<uint8_t*>(qa);
  if (form == 2) return cudaLaunchKernelEx(&cfg, act_quant_kernel<4, 8, kE8>, xp, groups, qp, sa);
  if (form == 1) return cudaLaunchKernelEx(&cfg, act_quant_kernel<1, 8, kE8>, xp, groups, qp, sa);
  return cudaLaunchKernelEx(&cfg, act_quant_kernel<1, 16, kE8>, xp, groups, qp, sa);
}

}  // namespace

cudaError_t launch_quant_act_group128(const void* x, int64_t M, int64_t K, void* qa, float* sa,
                                      cudaStream_t stream) {
  return launch_act<false>(x, M, K, qa, sa, stream);
}

cudaError_t launch_quant_act_group128_ue8m0(const void* x, int64_t M, int64_t K, void* qa,
                                            uint8_t* sa8, cudaStream_t stream) {
  return launch_act<true>(x, M, K, qa, sa8, stream);
}

cudaError_t launch_quant_weight_block128_ue8m0(const void* w, int64_t N, int64_t K, void* qw,
                                               uint8_t* sw8, cudaStream_t stream) {
  QArgs a{};
  a.q = static_cast<uint8_t*>(qw);
  a.scale8 = sw8;
  return launch_stream<QMode::kWeightE8>(w, N, K, a, stream);
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
  return w_pruned != nullptr ? launch_stream<QMode::kPruneOut>(w, N, K, a, stream)
                             : launch_stream<QMode::kPrune>(w, N, K, a, stream);
}

}  // namespace fp8bs

namespace fp8bs {

namespace {

// Gathered column shards -> full rows: src [P][M][Np] (rank p's columns
// [p Np, (p + 1) Np) of every row, as an all-gather leaves them) into
// dst [M][P Np], 16 bytes (8 bf16) per thread, both sides coalesced.
__global__ void __launch_bounds__(256)
    interleave_columns_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                              int64_t P, int64_t M, int64_t np16) {
  const int64_t total = P * M * np16;
  grid_dependency_wait();
  grid_launch_dependents();
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    // i enumerates dst: row m, rank p, chunk c of that rank's columns
    const int64_t c = i % np16;
    const int64_t p = (i / np16) % P;
    const int64_t m = i / (np16 * P);
    dst[i] = src[(p * M + m) * np16 + c];
  }
}

}  // namespace

cudaError_t launch_interleave_columns(const void* src, int64_t P, int64_t M, int64_t Np, void* dst,
                                      cudaStream_t stream) {
  DeviceInfo dev;
  if (current_device_info(&dev) != FP8BS_OK) return cudaErrorInvalidDevice;
  const int64_t np16 = Np / 8;
  const int64_t total = P * M * np16;
  const int64_t want = (total + 255) / 256;
  const int64_t blocks = want < 8LL * dev.sm_count ? want : 8LL * dev.sm_count;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(blocks > 0 ? blocks : 1), 1, 1);
  cfg.blockDim = dim3(256, 1, 1);
  cfg.stream = stream;
  cudaLaunchAttribute pdl;
  pdl.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl.val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = &pdl;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, interleave_columns_kernel, static_cast<const uint4*>(src),
                            static_cast<uint4*>(dst), P, M, np16);
}

}  // namespace fp8bs

namespace fp8bs {

namespace {

// SwiGLU and the next layer's 1x128 quantization on a gate+up GEMM output:
// y [M][2I] bf16 (gate columns [0, I), up columns [I, 2I)); per token m and
// group j of 128 intermediate columns, h = bf16(silu(gate) * up), and codes /
// scale of h with the activation quantizer's arithmetic. A team of 16
// threads per group, 8 columns per thread (one 16-byte load of gate and of
// up); no shared memory.
__global__ void __launch_bounds__(256)
    swiglu_quant_kernel(const __nv_bfloat16* __restrict__ y, int64_t M, int64_t I,
                        __nv_bfloat16* __restrict__ h, uint8_t* __restrict__ qh,
                        float* __restrict__ sh) {
  const int64_t groups_per_row = I / 128;
  const int64_t groups = M * groups_per_row;
  const int64_t team = static_cast<int64_t>(blockIdx.x) * 16 + (threadIdx.x >> 4);
  const int chunk = threadIdx.x & 15;
  grid_dependency_wait();
  grid_launch_dependents();
  const bool valid = team < groups;
  const int64_t m = valid ? team / groups_per_row : 0;
  const int64_t j = valid ? team - m * groups_per_row : 0;
  uint4 g4 = make_uint4(0u, 0u, 0u, 0u), u4 = g4;
  if (valid) {
    const __nv_bfloat16* row = y + m * 2 * I + j * 128 + chunk * 8;
    g4 = __ldg(reinterpret_cast<const uint4*>(row));
    u4 = __ldg(reinterpret_cast<const uint4*>(row + I));
  }
  const uint32_t gw[4] = {g4.x, g4.y, g4.z, g4.w}, uw[4] = {u4.x, u4.y, u4.z, u4.w};
  uint32_t hw[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float g0 = __uint_as_float(gw[i] << 16), g1 = __uint_as_float(gw[i] & 0xFFFF0000u);
    const float u0 = __uint_as_float(uw[i] << 16), u1 = __uint_as_float(uw[i] & 0xFFFF0000u);
    const __nv_bfloat162 p = __floats2bfloat162_rn(silu_f32(g0) * u0, silu_f32(g1) * u1);
    hw[i] = *reinterpret_cast<const uint32_t*>(&p);
  }
  const uint4 hv = make_uint4(hw[0], hw[1], hw[2], hw[3]);
  float mx = absmax_to_float(absmax8(hv));
#pragma unroll
  for (int off = 8; off >= 1; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  const float sc = scale_of_amax(mx);
  if (valid) {
    const int64_t off = m * I + j * 128 + chunk * 8;
    reinterpret_cast<uint2*>(qh + off)[0] = encode8(hv, ScaleDivider(sc));
    if (h != nullptr) *reinterpret_cast<uint4*>(h + off) = hv;
    if (chunk == 0) sh[m * groups_per_row + j] = sc;
  }
}

}  // namespace

cudaError_t launch_swiglu_quant(const void* y, int64_t M, int64_t I, void* h, void* qh, float* sh,
                                cudaStream_t stream) {
  const int64_t groups = M * (I / 128);
  const int64_t blocks = (groups + 15) / 16;
  if (blocks > 0x7FFFFFFF) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(blocks), 1, 1);
  cfg.blockDim = dim3(256, 1, 1);
  cfg.stream = stream;
  cudaLaunchAttribute pdl;
  pdl.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl.val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = &pdl;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, swiglu_quant_kernel, static_cast<const __nv_bfloat16*>(y), M, I,
                            static_cast<__nv_bfloat16*>(h), static_cast<uint8_t*>(qh), sh);
}

}  // namespace fp8bs
