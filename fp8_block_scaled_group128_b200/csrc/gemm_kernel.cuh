// The block-scaled FP8 GEMM kernel on tcgen05 tensor cores (shared by the
// dense and the 2:4 sparse entry points).
//
//   Y[m,n] = bf16_rn( sum_kb sA[m,kb] * sW[n/128,kb] * sum_{k in kb} qA[m,k] qW[n,k] )
//
// ("FP8 à granularité fine": 1x128 activation groups against 128x128 weight
// blocks, fp32 scales.) The scales change every 128-deep K-block, so the
// tensor cores cannot accumulate across K-blocks by themselves. Each K-block
// is one "partial" MMA chain written fresh into TMEM, and the epilogue warps
// promote it into fp32 register accumulators multiplied by sA * sW:
//
//   warp 0             TMA producer: K-block tiles -> shared memory, a
//                      kStages-deep ring of mbarriers.
//   warp 1 (and 2)     MMA issuer: per K-block, 4 x tcgen05.mma kind::f8f6f4
//                      (K = 32 each), or for 2:4 weights one tcgen05.cp of the
//                      metadata into TMEM and 2 x tcgen05.mma.sp (logical K =
//                      64 each), into one of kBufs TMEM partial buffers;
//                      commits free the smem stage and signal the partial. In
//                      decode order warps 1 and 2 issue alternate K-blocks.
//                      Both roles run their loops warp-wide and issue from one
//                      elected lane.
//   warps 4..          promotion / epilogue: tcgen05.ld the partial, FMA into
//                      registers with the K-block's scale product (staged per
//                      group of kG K-blocks in a shared table), hand the TMEM
//                      buffer back; at the end of a tile, round to bf16 and
//                      store through shared memory with TMA (or reduce split-K
//                      partials over the cluster).
//
// Operand orders:
//   kSwap = false (prefill, dense): MMA rows = tokens (128), MMA cols =
//     weight rows (BN = 256).
//   kSwap = true (decode, and every 2:4 launch): MMA rows = 128 weight rows,
//     MMA cols = tokens (BN = 16..256). When the weight tiles alone do not
//     fill the GPU, K is split over a thread-block cluster of `splits` CTAs
//     that sum their partial tiles through distributed shared memory in rank
//     order (pushed into the owner's receive buffer, or pulled from the other
//     CTAs' stage memory), so results are deterministic and no global scratch
//     is used.
// Without a K split the CTAs are persistent: CTA y walks tiles y, y+gridDim.y...
//
// Every mbarrier wait is bounded; a wait that runs out records
// FP8BS_ERR_DEVICE_TIMEOUT, and the CTA drains its own copies and MMAs in
// flight, frees TMEM and returns.
#pragma once

#include <map>
#include <mutex>
#include <tuple>

#include "common.cuh"
#include "e4m3_codec.cuh"
#include "kernels.h"

namespace fp8bs {

namespace gemm_detail {

constexpr int kBK = 128;               // K-block depth = one scale group, 128 bytes of E4M3
constexpr int kGroupRows = 16;         // tile raster: row tiles per group (L2 reuse)
constexpr int kEBytes = 128 * 16;      // sparse: metadata of one 128x128 block, 16 B per row
constexpr int kG = 8;                  // K-blocks per group of the epilogue's scale table

struct GemmArgs {
  const float* sa;      // [M][KB]
  const float* sw;      // [NB][KB]
  __nv_bfloat16* y;     // [M][N]
  int M, N, KB, NB;
  int row_tiles;        // tiles along the MMA M side (128 rows each)
  int col_tiles;        // tiles along the MMA N side (BN rows each)
  int splits;           // K splits = cluster size along x
  long long wait_limit; // bound of each mbarrier wait, SM cycles
  int* err;             // device error word
  uint8_t* qy;          // kQOut: Y quantized in 1x128 groups along N, [M][N] E4M3
  float* sy;            // kQOut: their scales, [M][N/128]
  // Grouped (mixture-of-experts) GEMM, prefill order only: the expert of
  // every token row ([M], null = one weight matrix); weights [E][N][K] and
  // scales [E][NB][KB]. Every 128-row tile takes the expert of its first row
  // (indices outside [0, E) count as expert 0).
  const int* m_indices;
  int E;
  // kSwiGLU: intermediate size I of a gate+up GEMM whose weights are
  // [W_gate; W_up] ([2I][K]); y, qy, sy then hold h = silu(gate) * up
  // ([M][I] bf16, may be null), its 1x128 codes [M][I] and scales [M][I/128].
  int swi;
};



// Expert of row tile `rt` of a grouped GEMM (0 when not grouped).
__device__ __forceinline__ int tile_expert(const GemmArgs& a, int rt) {
  if (a.m_indices == nullptr) return 0;
  const int e = __ldg(a.m_indices + static_cast<int64_t>(rt) * 128);
  return (e < 0 || e >= a.E) ? 0 : e;
}

// Split-K over a cluster of S CTAs: rank q reduces weight rows
// [recv_lo(q, S), recv_lo(q + 1, S)) of the 128-row tile (multiples of 4).
__host__ __device__ constexpr int recv_lo(int q, int S) { return 4 * (32 * q / S); }
__host__ __device__ constexpr int recv_rows(int q, int S) { return recv_lo(q + 1, S) - recv_lo(q, S); }
__host__ __device__ constexpr int recv_rows_max(int S) { return 4 * ((32 + S - 1) / S); }
static_assert(8 * recv_rows_max(8) <= 144 && 7 * recv_rows_max(7) <= 144 &&
                  6 * recv_rows_max(6) <= 144 && 5 * recv_rows_max(5) <= 144 &&
                  4 * recv_rows_max(4) <= 144 && 3 * recv_rows_max(3) <= 144 &&
                  2 * recv_rows_max(2) <= 144,
              "receive buffer: S slots of recv_rows_max(S) rows fit 144 rows");

template <int BN, bool kSwap, bool kSparse, int kStages, int kEpiWG, int kKS>
struct Cfg {
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N must be 16..256, step 16");
  static_assert((BN & (BN - 1)) == 0, "BN is a power of two (TMEM allocation)");
  static_assert(!kSparse || kSwap, "the 2:4 operand is the weight, on the MMA M side");
  // A stage holds kKS K-blocks (one 3-D TMA box per operand, so each copy is
  // large): A: kKS x 128 rows x 128 B (dense, 128 B swizzle) or kKS x 128 rows
  // x 64 B of compressed 2:4 values (64 B swizzle); B: kKS x BN rows x 128 B;
  // sparse metadata: kKS x 128 rows x 16 B.
  static constexpr int kAKb = kSparse ? 128 * kBK / 2 : 128 * kBK;  // A bytes per K-block
  static constexpr int kBKb = BN * kBK;                             // B bytes per K-block
  static constexpr int kABytes = kKS * kAKb;
  static constexpr int kBBytes = kKS * kBKb;
  static constexpr int kEStage = kSparse ? kKS * kEBytes : 0;
  static constexpr int kStageBytes = kABytes + kBBytes + kEStage;
  static constexpr int kThreads = 128 * (1 + kEpiWG);
  static constexpr int kCols = BN / kEpiWG;  // accumulator columns per epilogue thread
  static_assert(kCols % 16 == 0 && kCols <= 128, "epilogue column split");
  // Decode order: two warps issue the MMAs, alternating K-blocks (the
  // issue of a K-block's tcgen05 operations, ~300 cycles, paces the small
  // tiles otherwise).
  static constexpr bool kDualIssue = kSwap;
  // TMEM: kBufs partial buffers of BN columns (up to 8, so the MMA can run
  // ahead of the promotion), then (sparse) two metadata buffers of 4
  // columns per issuing warp; the allocation is a power of two >= 32.
  static constexpr int kMetaCols = kSparse ? 8 * (kDualIssue ? 2 : 1) : 0;
  static constexpr int kBufs = (512 - kMetaCols) / BN < 8 ? (512 - kMetaCols) / BN : 8;
  static_assert(kBufs >= 2, "at least two TMEM partial buffers");
  static constexpr int kTmemUsed = kBufs * BN + kMetaCols;
  static constexpr int kTmemCols =
      kTmemUsed <= 32 ? 32 : kTmemUsed <= 64 ? 64 : kTmemUsed <= 128 ? 128 : kTmemUsed <= 256 ? 256 : 512;
  static_assert(kTmemUsed <= 512, "TMEM has 512 columns");
  static constexpr uint32_t kIdesc = idesc_e4m3_f32(128, BN) | (kSparse ? (1u << 2) : 0u);
  static constexpr int kOffA = 0;
  static constexpr int kOffB = kStages * kABytes;
  static constexpr int kOffE = kOffB + kStages * kBBytes;
  static constexpr int kOffBar = kOffE + kStages * kEStage;
  static constexpr int kNumBars = 2 * kStages + 2 * kBufs + 1;
  static constexpr int kOffTmem = kOffBar + kNumBars * 8;
  static constexpr int kOffAbort = kOffTmem + 4;
  // scale table of the epilogue: 2 buffers x kG K-blocks x kSlots token
  // slots (row stride padded by 4 floats: conflict-free transposed stores,
  // 16-byte aligned rows)
  static constexpr int kEpiThreads = 128 * kEpiWG;
  static constexpr int kSlots = kSwap ? BN : 128 * kEpiWG;
  static constexpr int kTabStride = kSlots + 4;
  static constexpr int kPer = kG * kSlots / kEpiThreads;   // staged values per thread
  static_assert(kG * kSlots % kEpiThreads == 0, "scale table split");
  static constexpr int kOffTab = (kOffAbort + 4 + 15) / 16 * 16;
  static constexpr int kTabBytes = 2 * kG * kTabStride * 4;
  // prefill: the bf16 output tile [128][BN], staged for TMA stores as boxes
  // of 128 rows x 64 columns (128 bytes, 128-byte swizzle), 16 KB each
  static constexpr int kOffOut = (kOffTab + kTabBytes + 1023) / 1024 * 1024;
  static constexpr int kOutBytes = kSwap ? 0 : 128 * BN * 2;
  // decode order, one region used two ways: without a K split, the staging
  // buffers of the output TMA stores (per epilogue warpgroup, kChunk tokens x
  // 128 weight rows of bf16, token-major); with a K split, when it fits next
  // to the stages, the receive buffer of the push reduction (one slot of
  // recv_rows_max(S) weight rows x BN fp32 per CTA of the cluster, at most
  // 144 rows for S <= 8) and its mbarrier
  static constexpr int kChunk = kCols < 32 ? kCols : 32;
  static constexpr int kYstBytes = kSwap ? kEpiWG * kChunk * 256 : 0;
  static constexpr int kOffRecv = kOffOut + kOutBytes;
  static constexpr int kRecvBytes = 144 * BN * 4;
  static constexpr bool kPush =
      kSwap && kOffRecv + (kRecvBytes > kYstBytes ? kRecvBytes : kYstBytes) + 8 + 1024 <= 227 * 1024;
  static constexpr int kRegionBytes = kPush && kRecvBytes > kYstBytes ? kRecvBytes : kYstBytes;
  static constexpr int kOffRecvBar = kOffRecv + kRegionBytes;
  static constexpr int kSmemBytes =
      kOffRecvBar + (kPush ? 8 : 0) + 1024;  // + slack to align the base
  // split-K partial tile [BN][128] fp32 reuses the (drained) stage buffers
  static_assert(BN * 128 * 4 <= kStages * (kABytes + kBBytes), "split-K tile must fit the stages");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory");
  static_assert(kAKb % 1024 == 0 && kBKb % 1024 == 0, "stage buffers stay 1024-aligned");
};

__device__ __forceinline__ void tile_coords(int tile, int row_tiles, int col_tiles, int& rt,
                                            int& ct) {
  const int per_group = kGroupRows * col_tiles;
  const int g = tile / per_group;
  const int first = g * kGroupRows;
  const int rows = min(kGroupRows, row_tiles - first);
  const int local = tile - g * per_group;
  rt = first + local % rows;
  ct = local / rows;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

template <int BN, bool kSwap, bool kSparse, int kStages, int kEpiWG, int kKS, bool kQOut = false,
          bool kSwiGLU = false>
__global__ void __launch_bounds__(Cfg<BN, kSwap, kSparse, kStages, kEpiWG, kKS>::kThreads, 1)
    block_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a,
                      const __grid_constant__ CUtensorMap tmap_b,
                      const __grid_constant__ CUtensorMap tmap_e,
                      const __grid_constant__ CUtensorMap tmap_y, const GemmArgs args) {
  // tmap_e: the 2:4 metadata (sparse only); tmap_y: the output Y for the TMA
  // stores of the epilogue. kQOut: the epilogue also quantizes Y for the next
  // layer (args.qy, args.sy); in prefill order each thread holds one 1x128
  // group and Y itself is written only if args.y is set; in decode order
  // (unsplit tiles only) each token's group is the tile's 128 weight rows,
  // quantized from the staging buffer of the Y stores.
  using C = Cfg<BN, kSwap, kSparse, kStages, kEpiWG, kKS>;
  static_assert(!kQOut || (!kSparse && (kSwap || C::kCols == 128)),
                "fused quantization: one group per thread or per staged token");
  // kSwiGLU (prefill order): the 256 weight rows of a tile are gate rows
  // [128 ct, 128 ct + 128) and up rows [I + 128 ct, ...) (two TMA boxes of 128
  // rows); warpgroup 0 promotes the gate columns, warpgroup 1 the up columns of
  // the same token rows, and the epilogue combines them into
  // h = bf16(silu(gate) * up) and its 1x128 quantization along I.
  static_assert(!kSwiGLU || (!kSwap && !kQOut && BN == 256 && kEpiWG == 2), "SwiGLU epilogue");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sm_a = smem + C::kOffA;
  uint8_t* sm_b = smem + C::kOffB;
  uint8_t* sm_e = smem + C::kOffE;  // sparse only: metadata stages
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;
  uint64_t* tempty = tfull + C::kBufs;
  uint64_t* mma_done = tempty + C::kBufs;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffTmem);
  uint64_t* recv_bar = reinterpret_cast<uint64_t*>(smem + C::kOffRecvBar);   // kPush only
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffAbort);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int split = blockIdx.x;
  // K range of this split, boundaries rounded to whole stages (kKS K-blocks)
  const int kb0 = split == 0 ? 0
                             : static_cast<int>(static_cast<long long>(split) * args.KB /
                                                args.splits) / kKS * kKS;
  const int kb1 = split == args.splits - 1
                      ? args.KB
                      : static_cast<int>(static_cast<long long>(split + 1) * args.KB /
                                         args.splits) / kKS * kKS;
  const int num_tiles = args.row_tiles * args.col_tiles;
  const long long limit = args.wait_limit;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], C::kDualIssue ? 2 : 1);
    }
    for (int i = 0; i < C::kBufs; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 4 * kEpiWG);
    }
    mbar_init(mma_done, C::kDualIssue ? 2 : 1);
    if (C::kPush && args.splits > 1) {
      mbar_init(recv_bar, 1);
    }
    *abort_flag = 0;
    fence_mbarrier_init();
    if (C::kPush && args.splits > 1) {
      // phase 0 completes when every CTA of the cluster (this one included)
      // has stored this CTA's rows of its partial tile
      const int S = args.splits, rank = static_cast<int>(cluster_ctarank());
      const int rows = recv_rows(rank, S);
      mbar_arrive_expect_tx(recv_bar, static_cast<uint32_t>(S * rows * BN * 4));
    }
    tma_prefetch_desc(&tmap_a);
    tma_prefetch_desc(&tmap_b);
    if constexpr (kSparse) tma_prefetch_desc(&tmap_e);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // the receive barriers of the cluster are initialised before any CTA
  // stores into them (the matching wait precedes the stores)
  if (C::kPush && args.splits > 1) cluster_arrive_relaxed();
  const uint32_t tmem_base = *tmem_slot;
  // Decode order: the weight stages of the first tile (values and metadata
  // for 2:4) are prefetched into L2 while the previous kernel of the stream
  // may still run (an L2 prefetch never changes what a later load reads, so
  // this is safe even if that kernel writes the weights). Measured: 3-7 %
  // faster dense launches; 2:4 launches gain at 32 tokens and more (M = 128
  // four-linear sequence 75.3 -> 72.6 us, 2:4 prefill +4 %) and lose up to
  // 1 us at 16, so those do without.
  if constexpr (kSwap && (!kSparse || BN >= 32)) {
    if (threadIdx.x == 0 && static_cast<int>(blockIdx.y) < num_tiles) {
      int rt, ct;
      tile_coords(blockIdx.y, args.row_tiles, args.col_tiles, rt, ct);
      for (int kb = kb0, n = 0; kb < kb1 && n < kStages; kb += kKS, ++n) {
        tma_prefetch_l2_3d(&tmap_a, 0, rt * 128, kb);
        if constexpr (kSparse) tma_prefetch_l2_3d(&tmap_e, 0, rt * 128, kb);
      }
    }
  }
  // Everything else waits: inputs may come from the previous kernel.
  grid_dependency_wait();
  grid_launch_dependents();

  // Registers of the epilogue threads that outlive the role loop (split-K).
  float acc[C::kCols];

  // Prefill: 384 threads launched at 168 registers (64512); the producer / MMA
  // warpgroup drops to 40 and the two promotion warpgroups rise to 232
  // (128 x 40 + 256 x 232 = 64512).
  constexpr bool kRegSplit = !kSwap && kEpiWG == 2;
  static_assert(!kRegSplit || C::kThreads == 384, "register split assumes 3 warpgroups");

  if (warp < 4) {
   if constexpr (kRegSplit) setmaxnreg_dec<40>();
   if (warp == 0) {
    // -------------------------------------------------------- TMA producer --
    // The whole warp runs the loop; one elected lane issues.
    int stage = 0;
    uint32_t phase = 0;
    int issued = 0;
    for (int tile = blockIdx.y; tile < num_tiles && !*abort_flag; tile += gridDim.y) {
      int rt, ct;
      tile_coords(tile, args.row_tiles, args.col_tiles, rt, ct);
      // weight rows of this tile (of its expert, for a grouped GEMM)
      const int brow = ct * BN + (kSwap ? 0 : tile_expert(args, rt) * args.N);
      for (int kb = kb0; kb < kb1; kb += kKS) {
        if (!mbar_wait(&empty[stage], phase ^ 1u, limit)) {
          record_device_error(args.err, FP8BS_ERR_DEVICE_TIMEOUT);
          *abort_flag = 1;
          break;
        }
        // one box per operand covers K-blocks [kb, kb + kKS) (K-blocks past
        // the end of K read as zero and are not used)
        if (elect_one()) {
          mbar_arrive_expect_tx(&full[stage], C::kStageBytes);
          tma_load_3d(sm_a + stage * C::kABytes, &tmap_a, &full[stage], 0, rt * 128, kb);
          if constexpr (kSparse)
            tma_load_3d(sm_e + stage * C::kEStage, &tmap_e, &full[stage], 0, rt * 128, kb);
          if constexpr (kSwiGLU) {
            tma_load_3d(sm_b + stage * C::kBBytes, &tmap_b, &full[stage], 0, ct * 128, kb);
            tma_load_3d(sm_b + stage * C::kBBytes + 128 * kBK, &tmap_b, &full[stage], 0,
                        args.swi + ct * 128, kb);
          } else {
            tma_load_3d(sm_b + stage * C::kBBytes, &tmap_b, &full[stage], 0, brow, kb);
          }
        }
        __syncwarp();
        ++issued;
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    // Every copy issued must have landed before shared memory is reused or
    // the CTA exits (matters only when a consumer stopped early).
    const int pending = issued < kStages ? issued : kStages;
    for (int i = 0; i < pending; ++i) {
      int s = stage - 1 - i;
      uint32_t ph = phase;
      if (s < 0) {
        s += kStages;
        ph ^= 1u;
      }
      mbar_wait(&full[s], ph, kDefaultWaitCycles);
    }
   } else if (warp == 1 || (C::kDualIssue && warp == 2)) {
    // ---------------------------------------------------------- MMA issuer --
    // The whole warp runs the loop (warp-uniform operands); one elected lane
    // issues each tcgen05 operation. With two issuing warps, warp 1 + i
    // issues the K-blocks whose running index has parity i; both walk the
    // whole sequence (stages, partial buffers and their phases) and both
    // release each stage and the final barrier.
    const uint32_t me = static_cast<uint32_t>(warp - 1);
    int stage = 0;
    uint32_t phase = 0;
    int tb = 0;
    uint32_t tphase = 0;
    uint32_t kcount = 0;  // running K-block index of this CTA
    uint32_t e_buf = 0;   // sparse: this warp's TMEM metadata buffer, alternating
    bool ok = true;
    // Shared-memory descriptors of stage 0, K-block 0; every other operand
    // tile is an offset from them: the start-address field is address >> 4 in
    // the low 14 bits and shared addresses stay below 2^18, so adding
    // offset >> 4 moves it without touching the other fields.
    const uint64_t da0 = kSparse ? sw64_kmajor_desc(smem_u32(sm_a)) : sw128_kmajor_desc(smem_u32(sm_a));
    const uint64_t db0 = sw128_kmajor_desc(smem_u32(sm_b));
    const uint64_t de0 = kSparse ? noswizzle_kmajor_desc(smem_u32(sm_e), 128) : 0;
    for (int tile = blockIdx.y; ok && tile < num_tiles && !*abort_flag; tile += gridDim.y) {
      for (int kb = kb0; ok && kb < kb1; kb += kKS) {
        if (!mbar_wait(&full[stage], phase, limit)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int j = 0; j < kKS; ++j) {
          if (kb + j >= kb1) break;
          const bool mine = !C::kDualIssue || (kcount & 1u) == me;
          ++kcount;
          if (!mine) {
            if (++tb == C::kBufs) {
              tb = 0;
              tphase ^= 1u;
            }
            continue;
          }
          if (!mbar_wait(&tempty[tb], tphase ^ 1u, limit)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d = tmem_base + static_cast<uint32_t>(tb * BN);
          const uint64_t da = da0 + static_cast<uint32_t>((stage * C::kABytes + j * C::kAKb) >> 4);
          const uint64_t db = db0 + static_cast<uint32_t>((stage * C::kBBytes + j * C::kBKb) >> 4);
          if constexpr (kSparse) {
            // metadata of this K-block -> TMEM (4 columns, lane = weight
            // row), then two sparse MMAs of logical depth 64 (32 compressed
            // bytes of A and 64 bytes of B each), reading 2 metadata columns
            const uint32_t te =
                tmem_base + static_cast<uint32_t>(C::kBufs * BN) + 8u * me + 4u * e_buf;
            e_buf ^= 1u;
            const uint64_t de = de0 + static_cast<uint32_t>((stage * C::kEStage + j * kEBytes) >> 4);
            if (elect_one()) {
              tmem_cp_128x128b(te, de);
              mma_sp_f8f6f4_c<false>(d, da, db, te, C::kIdesc);
              mma_sp_f8f6f4_c<true>(d, da + (32 >> 4), db + (64 >> 4), te + 2, C::kIdesc);
              mma_commit(&tfull[tb]);
            }
          } else {
            if (elect_one()) {
              mma_f8f6f4_c<false>(d, da, db, C::kIdesc);
              mma_f8f6f4_c<true>(d, da + (32 >> 4), db + (32 >> 4), C::kIdesc);
              mma_f8f6f4_c<true>(d, da + (64 >> 4), db + (64 >> 4), C::kIdesc);
              mma_f8f6f4_c<true>(d, da + (96 >> 4), db + (96 >> 4), C::kIdesc);
              mma_commit(&tfull[tb]);
            }
          }
          __syncwarp();
          if (++tb == C::kBufs) {
            tb = 0;
            tphase ^= 1u;
          }
        }
        // the stage is free once every MMA that reads it has completed
        if (elect_one()) mma_commit(&empty[stage]);
        __syncwarp();
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    if (!ok) {
      record_device_error(args.err, FP8BS_ERR_DEVICE_TIMEOUT);
      *abort_flag = 1;
    }
    // All MMAs issued must be complete before TMEM is freed.
    if (elect_one()) mma_commit(mma_done);
    __syncwarp();
    mbar_wait(mma_done, 0, kDefaultWaitCycles);
   }
  } else {
    if constexpr (kRegSplit) setmaxnreg_inc<232>();
    // ------------------------------------------------- promotion / epilogue --
    const int wg = (warp - 4) >> 2;     // epilogue warpgroup
    const int quarter = warp & 3;       // TMEM lanes [32 quarter, 32 quarter + 32)
    const int row = quarter * 32 + lane;
    const int col0 = wg * C::kCols;
    const int64_t KB = args.KB;
    const int e = static_cast<int>(threadIdx.x) - 128;   // epilogue thread index
    float* tab = reinterpret_cast<float*>(smem + C::kOffTab);

    // Scale table. Every element of a K-block partial is scaled by
    // sA[token, kb] * sW[weight row block, kb]. Per group of kG K-blocks the
    // epilogue warps stage these products for every token slot of the tile in
    // a double-buffered shared table [kG][kSlots] (global loads run along kb,
    // one group ahead of its use), and the promotion reads them from shared
    // memory. Slots: decode order = the BN token columns; prefill order = the
    // 128 token rows, once per epilogue warpgroup (each has its own weight
    // block). The groups of this CTA are (tile, kbg) for its tiles in order and
    // kbg = kb0, kb0 + kG, ... < kb1.
    int g_tile = blockIdx.y, g_kb = kb0;   // next group to stage
    // coordinates of g_tile, recomputed only when it changes (the grouped
    // raster costs three integer divisions, a long dependency chain that
    // would otherwise stall every group boundary)
    int grt = 0, gct = 0;
    int64_t gsw = 0;   // prefill: offset of the staged tile's expert in sW
    // Thread e stages table entries (K-block sg of the group, slot s0 + i *
    // kSlotStep) for i < kPer: the same K-block for every i. In decode order
    // its first token and the scale pointers at K-block sg are fixed per
    // tile, so a group boundary only adds the group's first K-block to them
    // (prefill, short of registers, recomputes them per group).
    constexpr int kSlotStep = C::kEpiThreads / kG;
    static_assert(C::kEpiThreads % kG == 0 && (kSwap || 128 % kSlotStep == 0), "table slots");
    const int sg = e % kG, s0 = e / kG;
    int first = 0, nb0 = 0;                 // first token (decode) or row (prefill); weight block
    const float* a0 = args.sa;
    const float* w0 = args.sw;
    auto tile_bases = [&]() {
      tile_coords(g_tile, args.row_tiles, args.col_tiles, grt, gct);
      if constexpr (!kSwap)
        gsw = static_cast<int64_t>(tile_expert(args, grt)) * args.NB * args.KB;
      if constexpr (kSwap) {
        first = gct * BN + s0;
        nb0 = grt;
        a0 = args.sa + static_cast<int64_t>(first) * KB + sg;
        w0 = args.sw + static_cast<int64_t>(nb0) * KB + sg;
      }
    };
    if (g_tile < num_tiles) tile_bases();
    // raw loads of the next group; multiplied only when stored, a group
    // later, so that nothing waits on them
    float pre_a[C::kPer], pre_w[C::kPer];
    auto group_load = [&]() {
      if (g_tile >= num_tiles) return;
      const bool kb_ok = g_kb + sg < kb1;
#pragma unroll
      for (int i = 0; i < C::kPer; ++i) {
        const int d = i * kSlotStep;   // slot offset from s0
        float va = 0.0f, vw = 0.0f;
        if constexpr (kSwap) {
          if (kb_ok && first + d < args.M) {
            va = a0[static_cast<int64_t>(d) * KB + g_kb];
            vw = w0[g_kb];
          }
        } else {
          // slot s0 + d is token row s0 + (d & 127) of the tile, weight block
          // gct * BN / 128 + (d >> 7) * kCols / 128
          const int64_t m = static_cast<int64_t>(grt) * 128 + s0 + (d & 127);
          // weight block of warpgroup d >> 7 (SwiGLU: the gate block, then the
          // up block I / 128 blocks further)
          const int nb = kSwiGLU ? ((d >> 7) == 0 ? gct : args.swi / 128 + gct)
                                 : (gct * BN + (d >> 7) * C::kCols) / 128;
          const int kb = g_kb + sg;
          if (kb_ok && m < args.M && nb < args.NB) {
            va = args.sa[m * KB + kb];
            vw = args.sw[gsw + nb * KB + kb];
          }
        }
        pre_a[i] = va;
        pre_w[i] = vw;
      }
    };
    auto group_store = [&](int buf) {
#pragma unroll
      for (int i = 0; i < C::kPer; ++i)
        tab[(buf * kG + sg) * C::kTabStride + s0 + i * kSlotStep] = pre_a[i] * pre_w[i];
    };
    auto group_next = [&]() {
      g_kb += kG;
      if (g_kb >= kb1) {
        g_kb = kb0;
        g_tile += gridDim.y;
        if (g_tile < num_tiles) tile_bases();
      }
    };
    group_load();
    group_store(0);
    group_next();
    group_load();
    named_bar_sync(1, C::kEpiThreads);
    int buf = 0;

    int tb = 0;
    uint32_t tphase = 0;
    bool ok = true;
    // Every epilogue thread walks the same groups (the named barrier above
    // needs all of them); after a wait runs out, `ok` is false and the rest is
    // skipped.
    for (int tile = blockIdx.y; tile < num_tiles; tile += gridDim.y) {
      int rt, ct;
      tile_coords(tile, args.row_tiles, args.col_tiles, rt, ct);
#pragma unroll
      for (int i = 0; i < C::kCols; ++i) acc[i] = 0.0f;

      for (int kbg = kb0; kbg < kb1; kbg += kG) {
        const float* tg = tab + buf * kG * C::kTabStride;
        for (int j = 0; ok && j < kG; ++j) {
          const int kb = kbg + j;
          if (kb >= kb1) break;
          if (!mbar_wait(&tfull[tb], tphase, limit)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const float* trow = tg + j * C::kTabStride;
          const uint32_t tlane = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + tb * BN;
          const uint32_t taddr = tlane + col0;
          if constexpr (!kSwap && C::kCols % 64 == 0) {
            // prefill: 64 columns per TMEM round trip (two x32 loads, one wait).
            // SwiGLU: the tile's columns [0, 128) are gate, [128, 256) up (weight
            // blocks 0 and 1 of the scale table); warpgroup w promotes gate and
            // up columns [64 w, 64 w + 64) into acc[0, 64) and acc[64, 128), so a
            // thread holds both operands of each of its outputs.
#pragma unroll
            for (int c = 0; c < C::kCols; c += 64) {
              const float sc = trow[(kSwiGLU ? 2 * c : wg * 128) + row];
              const uint32_t ta = kSwiGLU ? tlane + 2 * c + wg * 64 : taddr + c;
              float v[64];
              tmem_ld32(ta, v);
              tmem_ld32(ta + 32, v + 32);
              tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 64; i += 2)
                fma2(acc[c + i], acc[c + i + 1], v[i], v[i + 1], sc, sc);
            }
          } else
#pragma unroll
          for (int c = 0; c < C::kCols; c += 32) {
            float v0[16], v1[16];
            tmem_ld16(taddr + c, v0);
            if (c + 16 < C::kCols) tmem_ld16(taddr + c + 16, v1);
            tmem_wait_ld();
            if constexpr (!kSwap) {
              const float sc = trow[wg * 128 + row];
#pragma unroll
              for (int i = 0; i < 16; ++i) acc[c + i] = fmaf(sc, v0[i], acc[c + i]);
              if (c + 16 < C::kCols) {
#pragma unroll
                for (int i = 0; i < 16; ++i) acc[c + 16 + i] = fmaf(sc, v1[i], acc[c + 16 + i]);
              }
            } else {
              // column scales of this K-block (the same for every lane)
              const float4* s4 = reinterpret_cast<const float4*>(trow + col0 + c);
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const float4 q = s4[i];
                fma2(acc[c + 4 * i], acc[c + 4 * i + 1], v0[4 * i], v0[4 * i + 1], q.x, q.y);
                fma2(acc[c + 4 * i + 2], acc[c + 4 * i + 3], v0[4 * i + 2], v0[4 * i + 3], q.z,
                     q.w);
              }
              if (c + 16 < C::kCols) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                  const float4 q = s4[4 + i];
                  float* a = acc + c + 16 + 4 * i;
                  fma2(a[0], a[1], v1[4 * i], v1[4 * i + 1], q.x, q.y);
                  fma2(a[2], a[3], v1[4 * i + 2], v1[4 * i + 3], q.z, q.w);
                }
              }
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty[tb]);
          if (++tb == C::kBufs) {
            tb = 0;
            tphase ^= 1u;
          }
        }
        // the group after this one goes into the other buffer (nobody reads it
        // any more: its last readers passed the previous barrier)
        group_store(buf ^ 1);
        group_next();
        group_load();
        named_bar_sync(1, C::kEpiThreads);
        buf ^= 1;
      }

      if constexpr (kSwiGLU) {
        // acc[c] = gate[m][j0 + 64 wg + c] and acc[64 + c] = up[m][j0 + 64 wg + c]
        // (c < 64) in fp32, token row m = 128 rt + row. Each thread forms its 64
        // h = bf16(silu(gate) * up); the scale of the 128-wide group comes from
        // the larger of the two warpgroups' half maxima, which cross through
        // [2][2][128] fp32 slots in the (here unused) output staging buffer. The
        // slots alternate between tiles, so one barrier per tile separates a
        // slot's writes from its reads and its reads from its next writes (two
        // tiles later, after the intervening tile's barrier). Each warpgroup then
        // encodes its 64 values with that scale (the activation quantizer's
        // arithmetic on the bf16 h).
        const int j0 = ct * 128;
        const int64_t m = static_cast<int64_t>(rt) * 128 + row;
        uint32_t hb[32];
#pragma unroll
        for (int c = 0; c < 64; c += 2)
          hb[c / 2] = pack_bf16x2(silu_f32(acc[c]) * acc[64 + c],
                                  silu_f32(acc[c + 1]) * acc[64 + c + 1]);
        uint32_t mx = 0u;
#pragma unroll
        for (int i = 0; i < 32; ++i) mx = bf16x2_absmax(mx, hb[i]);
        const float my_amax = absmax_to_float(mx);
        float* slots = reinterpret_cast<float*>(smem + C::kOffOut) +
                       (((tile - static_cast<int>(blockIdx.y)) / static_cast<int>(gridDim.y)) & 1) * 256;
        slots[wg * 128 + row] = my_amax;
        named_bar_sync(1, C::kEpiThreads);
        const float amax = fmaxf(my_amax, slots[(1 - wg) * 128 + row]);
        if (ok && m < args.M) {
          const float sc = scale_of_amax(amax);
          const ScaleDivider d(sc);
          const int64_t off = m * args.swi + j0 + wg * 64;
#pragma unroll
          for (int c = 0; c < 64; c += 16) {
            const uint4 v0 = make_uint4(hb[c / 2], hb[c / 2 + 1], hb[c / 2 + 2], hb[c / 2 + 3]);
            const uint4 v1 = make_uint4(hb[c / 2 + 4], hb[c / 2 + 5], hb[c / 2 + 6], hb[c / 2 + 7]);
            const uint2 e0 = encode8(v0, d), e1 = encode8(v1, d);
            *reinterpret_cast<uint4*>(args.qy + off + c) = make_uint4(e0.x, e0.y, e1.x, e1.y);
            if (args.y != nullptr) {
              *reinterpret_cast<uint4*>(args.y + off + c) = v0;
              *reinterpret_cast<uint4*>(args.y + off + c + 8) = v1;
            }
          }
          if (wg == 0) args.sy[m * (args.swi / 128) + j0 / 128] = sc;
        }
      } else if constexpr (!kSwap) {
        // This warpgroup's 128 columns = two 64-column boxes of the staged
        // tile. Its leader first waits until the previous tile's stores have
        // read the boxes; every thread then writes its row (16-byte chunk j
        // of row r at chunk position j ^ (r % 8): the 128-byte swizzle), and
        // the leader issues the two TMA stores, which run on while the next
        // tile is promoted. TMA leaves rows >= M and columns >= N unwritten.
        const bool leader = (warp & 3) == 0 && lane == 0;
        uint8_t* out = smem + C::kOffOut + wg * (C::kCols / 64) * 16384;
        if (leader) bulk_wait_group_read0();
        named_bar_sync(2 + wg, 128);
        if (ok) {
#pragma unroll
          for (int c = 0; c < C::kCols; c += 8) {
            uint4 pk;
            pk.x = pack_bf16x2(acc[c + 0], acc[c + 1]);
            pk.y = pack_bf16x2(acc[c + 2], acc[c + 3]);
            pk.z = pack_bf16x2(acc[c + 4], acc[c + 5]);
            pk.w = pack_bf16x2(acc[c + 6], acc[c + 7]);
            const int j = (c & 63) >> 3;
            *reinterpret_cast<uint4*>(out + (c >> 6) * 16384 + row * 128 +
                                      ((j ^ (row & 7)) << 4)) = pk;
          }
        }
        fence_proxy_async_smem();
        named_bar_sync(2 + wg, 128);
        if (leader && ok && (!kQOut || args.y != nullptr)) {
#pragma unroll
          for (int b = 0; b < C::kCols / 64; ++b)
            tma_store_2d(&tmap_y, out + b * 16384, ct * BN + col0 + b * 64, rt * 128);
          bulk_commit_group();
        }
        if constexpr (kQOut) {
          // The next layer's activation quantization, with the arithmetic of
          // the activation quantizer on the bf16 values just stored: this
          // thread's 128 columns of token row m are one 1x128 group of Y
          // along N (N is a multiple of 128).
          const int64_t m = static_cast<int64_t>(rt) * 128 + row;
          const int n0 = ct * BN + col0;
          if (ok && m < args.M && n0 < args.N) {
            auto chunk8 = [&](int c) {
              return make_uint4(pack_bf16x2(acc[c + 0], acc[c + 1]),
                                pack_bf16x2(acc[c + 2], acc[c + 3]),
                                pack_bf16x2(acc[c + 4], acc[c + 5]),
                                pack_bf16x2(acc[c + 6], acc[c + 7]));
            };
            uint32_t mx = absmax8(chunk8(0));
#pragma unroll
            for (int c = 8; c < C::kCols; c += 8) mx = bf16x2_absmax(mx, absmax8(chunk8(c)));
            const float sc = scale_of_amax(absmax_to_float(mx));
            const ScaleDivider d(sc);
            uint8_t* qrow = args.qy + m * args.N + n0;
#pragma unroll
            for (int c = 0; c < C::kCols; c += 8)
              *reinterpret_cast<uint2*>(qrow + c) = encode8(chunk8(c), d);
            args.sy[m * (args.N / 128) + n0 / 128] = sc;
          }
        }
      } else if (args.splits == 1) {
        // Column j of the tile is token ct*BN + col0 + j, the lane's row is
        // weight row rt*128 + row: the tile goes out transposed. Per chunk of
        // kChunk tokens, every thread writes its row's bf16 values into the
        // token-major staging buffer (256 bytes per token, a warp's 32 rows
        // are 64 contiguous bytes), and the leader issues one TMA store,
        // which clips tokens >= M and rows >= N; it runs on while the next
        // chunk or tile is computed.
        const bool leader = (warp & 3) == 0 && lane == 0;
        uint8_t* stage_y = smem + C::kOffRecv + wg * C::kChunk * 256;
#pragma unroll
        for (int c = 0; c < C::kCols; c += C::kChunk) {
          if (leader) bulk_wait_group_read0();
          named_bar_sync(2 + wg, 128);
          if (ok) {
#pragma unroll
            for (int j = 0; j < C::kChunk; ++j)
              *reinterpret_cast<__nv_bfloat16*>(stage_y + j * 256 + row * 2) =
                  __float2bfloat16_rn(acc[c + j]);
          }
          fence_proxy_async_smem();
          named_bar_sync(2 + wg, 128);
          if (leader && ok && (!kQOut || args.y != nullptr)) {
            tma_store_2d(&tmap_y, stage_y, rt * 128, ct * BN + col0 + c);
            bulk_commit_group();
          }
          if constexpr (kQOut) {
            // Each staged token holds one whole 1x128 group of Y (the tile's
            // 128 weight rows, 256 contiguous bytes): a team of 16 threads per
            // token quantizes it with the activation quantizer's arithmetic
            // (8 bf16 per thread, a 16-lane max) and writes 128 code bytes and
            // the scale. The staging buffer is rewritten only after the next
            // chunk's barrier, which every thread reaches after these reads.
            const int part = (warp & 3) * 32 + lane;
            const int team = part >> 4, sub = part & 15;
#pragma unroll
            for (int j = team; j < C::kChunk; j += 8) {
              const uint4 v = *reinterpret_cast<const uint4*>(stage_y + j * 256 + sub * 16);
              float am = absmax_to_float(absmax8(v));
#pragma unroll
              for (int off = 8; off >= 1; off >>= 1)
                am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, off));
              const float sc = scale_of_amax(am);
              const int64_t m = static_cast<int64_t>(ct) * BN + col0 + c + j;   // token
              if (ok && m < args.M) {
                *reinterpret_cast<uint2*>(args.qy + m * args.N + rt * 128 + sub * 8) =
                    encode8(v, ScaleDivider(sc));
                if (sub == 0) args.sy[m * (args.N / 128) + rt] = sc;
              }
            }
          }
        }
      }
    }
    // the last TMA stores have finished before the CTA exits
    if ((warp & 3) == 0 && lane == 0) bulk_wait_group0();
    if (!ok) {
      record_device_error(args.err, FP8BS_ERR_DEVICE_TIMEOUT);
      *abort_flag = 1;
    }
  }

  tc_fence_before();
  __syncthreads();

  if (C::kPush && args.splits > 1) {
    // ------------------------------- split-K reduction in the cluster, pushed --
    // Rank q of the cluster owns weight rows [recv_lo(q), recv_lo(q + 1)) of
    // the tile. Every epilogue thread stores its row of the fp32 partial tile
    // straight from registers into slot `rank` of the owner's receive buffer
    // (st.async, counted on the owner's receive barrier); each CTA then sums
    // its slots over ranks 0..S-1 in that order and writes its rows of Y.
    // No cluster-wide release barrier is needed: the receive barrier's
    // transaction count says when the data is there, and a CTA never reads
    // another CTA's memory.
    const int S = args.splits;
    const int rank = static_cast<int>(cluster_ctarank());
    const int slot_rows = recv_rows_max(S);
    float* recv = reinterpret_cast<float*>(smem + C::kOffRecv);
    cluster_wait();
    if (warp >= 4) {
      const int wg = (warp - 4) >> 2;
      const int row = (warp & 3) * 32 + lane;
      int q = 0;
      while (q + 1 < S && row >= recv_lo(q + 1, S)) ++q;
      const uint32_t dst = map_cluster(
          smem_u32(recv + (rank * slot_rows + row - recv_lo(q, S)) * BN + wg * C::kCols),
          static_cast<uint32_t>(q));
      const uint32_t bar = map_cluster(smem_u32(recv_bar), static_cast<uint32_t>(q));
#pragma unroll
      for (int j = 0; j < C::kCols; j += 4)
        st_async_v4(dst + 4 * j, acc[j], acc[j + 1], acc[j + 2], acc[j + 3], bar);
    }
    bool got = mbar_wait_cluster(recv_bar, 0, limit);
    if (!got) {
      record_device_error(args.err, FP8BS_ERR_DEVICE_TIMEOUT);
      // stores still in flight must land before this CTA's memory goes away
      mbar_wait_cluster(recv_bar, 0, kDefaultWaitCycles);
    }
    if (got && !*abort_flag) {
      int last_rt, last_ct;  // split-K CTAs own exactly one tile: blockIdx.y
      tile_coords(blockIdx.y, args.row_tiles, args.col_tiles, last_rt, last_ct);
      const int r_lo = recv_lo(rank, S);
      const int nr4 = recv_rows(rank, S) / 4;
      const int tok_left = args.M - last_ct * BN;
      const int n_tok = tok_left < BN ? tok_left : BN;
      // token index fastest: the threads of a warp read consecutive words
      for (int idx = threadIdx.x; idx < n_tok * nr4; idx += C::kThreads) {
        const int r4 = (idx / n_tok) * 4;
        const int j = idx - (idx / n_tok) * n_tok;
        float4 acc4 = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          if (q < S) {
            const float* p = recv + (q * slot_rows + r4) * BN + j;
            if (q == 0) {
              acc4 = make_float4(p[0], p[BN], p[2 * BN], p[3 * BN]);
            } else {
              acc4.x += p[0];
              acc4.y += p[BN];
              acc4.z += p[2 * BN];
              acc4.w += p[3 * BN];
            }
          }
        }
        const int out_row = last_ct * BN + j;            // token
        const int out_col = last_rt * 128 + r_lo + r4;   // weight row
        if (out_col < args.N) {
          uint2 pk;
          pk.x = pack_bf16x2(acc4.x, acc4.y);
          pk.y = pack_bf16x2(acc4.z, acc4.w);
          *reinterpret_cast<uint2*>(args.y + static_cast<int64_t>(out_row) * args.N + out_col) =
              pk;
        }
      }
    }
  } else if (kSwap && args.splits > 1) {
    // ---------------------------------------- split-K reduction in the cluster --
    // Each CTA publishes its fp32 partial tile [BN][128] (token-major, MMA row
    // index contiguous) in its own drained stage memory; rank r then sums, over
    // ranks 0..S-1 in that order, weight rows [4*(32r/S), 4*(32(r+1)/S)) of
    // every valid token and writes those Y elements. (Only the swapped, decode
    // order is ever split.)
    float* red = reinterpret_cast<float*>(smem);
    if (warp >= 4) {
      const int wg = (warp - 4) >> 2;
      const int row = (warp & 3) * 32 + lane;
#pragma unroll
      for (int j = 0; j < C::kCols; ++j) red[(wg * C::kCols + j) * 128 + row] = acc[j];
    }
    __syncwarp();
    cluster_sync();
    int last_rt, last_ct;  // split-K CTAs own exactly one tile: blockIdx.y
    tile_coords(blockIdx.y, args.row_tiles, args.col_tiles, last_rt, last_ct);
    if (kSwap && !*abort_flag) {
      const int S = args.splits;
      const int rank = static_cast<int>(cluster_ctarank());
      const int r_lo = 4 * (32 * rank / S), r_hi = 4 * (32 * (rank + 1) / S);
      const int nr4 = (r_hi - r_lo) / 4;
      const int tok_left = args.M - last_ct * BN;
      const int n_tok = tok_left < BN ? tok_left : BN;
      const int total4 = n_tok * nr4;
      for (int idx = threadIdx.x; idx < total4; idx += C::kThreads) {
        const int j = idx / nr4;
        const int r4 = r_lo + (idx - j * nr4) * 4;
        const uint32_t local = smem_u32(red + j * 128 + r4);
        float4 v[8];
#pragma unroll
        for (int q = 0; q < 8; ++q)
          if (q < S) v[q] = ld_cluster_f32x4(map_cluster(local, static_cast<uint32_t>(q)));
        float4 acc4 = v[0];
#pragma unroll
        for (int q = 1; q < 8; ++q) {
          if (q < S) {
            acc4.x += v[q].x;
            acc4.y += v[q].y;
            acc4.z += v[q].z;
            acc4.w += v[q].w;
          }
        }
        const int out_row = last_ct * BN + j;       // token
        const int out_col = last_rt * 128 + r4;     // weight row
        if (out_col < args.N) {
          uint2 pk;
          pk.x = pack_bf16x2(acc4.x, acc4.y);
          pk.y = pack_bf16x2(acc4.z, acc4.w);
          *reinterpret_cast<uint2*>(args.y + static_cast<int64_t>(out_row) * args.N + out_col) =
              pk;
        }
      }
    }
    __syncwarp();
    cluster_sync();
  }

  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

// ------------------------------------------------------------------ host side --

// How many clusters of `S` CTAs of `kern` can be resident at once (cached per
// kernel, device and S).
template <class Kern>
int max_active_clusters(Kern kern, int threads, int smem, int S, int dev) {
  static std::mutex mu;
  static std::map<std::tuple<const void*, int, int>, int> cache;
  const auto key = std::make_tuple(reinterpret_cast<const void*>(kern), dev, S);
  std::lock_guard<std::mutex> lock(mu);
  auto it = cache.find(key);
  if (it != cache.end()) return it->second;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(S), 1, 1);
  cfg.blockDim = dim3(static_cast<unsigned>(threads), 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = static_cast<unsigned>(S);
  attr.val.clusterDim.y = 1;
  attr.val.clusterDim.z = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;   // not cached: a later call may succeed
  }
  cache[key] = n;
  return n;
}

template <int BN, bool kSwap, bool kSparse, int kStages, int kEpiWG, int kKS, bool kQOut = false,
          bool kSwiGLU = false>
int launch_cfg(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& te,
               const GemmArgs& a, int grid_y, int splits, cudaStream_t stream) {
  // (grid_y, splits) as chosen by the shape heuristic; adjusted below.
  using C = Cfg<BN, kSwap, kSparse, kStages, kEpiWG, kKS>;
  // Y [M][N] bf16 for the epilogue's TMA stores: prefill boxes of 128 token
  // rows x 64 columns (128-byte swizzle), decode boxes of kChunk tokens x 128
  // weight rows (plain). Without Y (a fused quantization that writes only the
  // codes) the map stays zero and is never used.
  alignas(64) CUtensorMap ty{};
  if (a.y != nullptr && !kSwiGLU) {   // the SwiGLU epilogue stores h itself
    if (int st = kSwap ? encode_tmap_2d(&ty, a.y, 2, a.N, a.M, static_cast<uint64_t>(a.N) * 2,
                                        128, C::kChunk, kSwizzleNone)
                       : encode_tmap_2d(&ty, a.y, 2, a.N, a.M, static_cast<uint64_t>(a.N) * 2,
                                        64, 128, kSwizzle128B))
      return st;
  }
  auto kern = block_gemm_kernel<BN, kSwap, kSparse, kStages, kEpiWG, kKS, kQOut, kSwiGLU>;
  static std::once_flag flags[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return FP8BS_ERR_CUDA;
  cudaError_t attr_err = cudaSuccess;
  std::call_once(flags[dev], [&] {
    attr_err =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  });
  if (attr_err != cudaSuccess) return FP8BS_ERR_CUDA;

  // A split launch needs every cluster resident at once (a cluster of S CTAs
  // needs S free SMs of one GPC); shrink S until the clusters fit in one wave.
  GemmArgs args = a;
  while (splits > 1) {
    const int fit = max_active_clusters(kern, C::kThreads, C::kSmemBytes, splits, dev);
    if (fit >= grid_y) break;
    --splits;
    while (splits > 1 && args.KB / kKS < splits) --splits;
  }
  if (splits == 1 && args.splits > 1) {
    DeviceInfo info;
    if (current_device_info(&info) != FP8BS_OK) return FP8BS_ERR_CUDA;
    grid_y = grid_y < info.sm_count ? grid_y : info.sm_count;   // persistent
  }
  args.splits = splits;

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(splits), static_cast<unsigned>(grid_y), 1);
  cfg.blockDim = dim3(C::kThreads, 1, 1);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attrs[2];
  attrs[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attrs;
  cfg.numAttrs = 1;
  if (splits > 1) {
    attrs[1].id = cudaLaunchAttributeClusterDimension;
    attrs[1].val.clusterDim.x = static_cast<unsigned>(splits);
    attrs[1].val.clusterDim.y = 1;
    attrs[1].val.clusterDim.z = 1;
    cfg.numAttrs = 2;
  }
  if (cudaLaunchKernelEx(&cfg, kern, ta, tb, te, ty, args) != cudaSuccess) return FP8BS_ERR_CUDA;
  return FP8BS_OK;
}

inline int next_pow2_at_least16(int64_t v) {
  int b = 16;
  while (b < v) b <<= 1;
  return b;
}

// K split of a swapped (weights-on-M) launch: spread `tiles` units over the
// SMs with a cluster of up to 8 CTAs per tile when the tiles alone do not
// fill the GPU; at least one K-block per split.
inline int choose_splits(int tiles, int sm_count, int KB, int ks) {
  int S = 1;
  if (tiles < sm_count) {
    S = sm_count / tiles;
    if (S > 8) S = 8;
    if (S > KB / ks) S = KB / ks;
    if (S < 1) S = 1;
  }
  return S;
}

}  // namespace gemm_detail

}  // namespace fp8bs
