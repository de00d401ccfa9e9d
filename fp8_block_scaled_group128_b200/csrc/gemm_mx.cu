// The block-scaled FP8 GEMM with UE8M0 (power-of-two) scales, on the tensor
// cores' own block scaling ("FP8 à granularité fine", section "Format
// d'échelle UE8M0": scales stored as float8_e8m0fnu).
//
//   Y[m,n] = bf16_rn( sum_kb 2^(ea[m,kb]) * 2^(ew[n/128,kb]) * sum_{k in kb} qA[m,k] qW[n,k] )
//
// With power-of-two scales the product of a K-block can be scaled inside the
// MMA: tcgen05.mma ... kind::mxf8f6f4.block_scale multiplies every 32-deep
// slice of A rows and B columns by 2^(code - 127) read from TMEM, so the
// tensor core accumulates across all K-blocks of a tile in one fp32 TMEM
// accumulator and no per-K-block promotion on the CUDA cores is needed (the
// fp32-scale GEMM in gemm_kernel.cuh must promote every K-block). A 1x128
// activation group or a 128x128 weight block spans four 32-deep slices, which
// all take the group's (block's) code.
//
// Tiles of kP x 128 tokens (MMA M) x 256 weight rows (MMA N) over persistent
// CTAs (grouped raster). kP = 2 (the form used for M > 128): a cluster of two
// CTAs shares each MMA (tcgen05 cta_group::2, M = 256); each CTA loads 128
// token rows and 128 of the 256 weight rows per K-block (32 KB, six stages),
// its TMEM holds its 128 rows of the tile. kP = 1: one CTA, 48 KB per K-block,
// four stages. 384 threads per CTA:
//   warp 0        TMA producer (each CTA loads its own halves; in a pair both
//                 CTAs' copies complete on rank 0's barrier);
//   warp 1        MMA issuer (rank 0 only): per K-block four block-scaled MMAs
//                 (K = 32) and a commit that frees the stage in both CTAs; per
//                 group of four K-blocks three tcgen05.cp of the scale factors
//                 into TMEM, issued a group ahead; a commit per tile signals
//                 the accumulator;
//   warp 2        scale factors: per group of four K-blocks it writes the
//                 scale-factor chunks of a slot in shared memory (the layout
//                 of a 32x128b.warpx4 copy: row r of a chunk holds the words
//                 of rows r, r + 32, r + 64, r + 96; byte i of a word is the
//                 code of the group's K-block i, which the MMAs of that
//                 K-block select with the descriptor's scale-factor id): its
//                 CTA's 128 token rows and all 256 weight rows of the tile.
//                 The codes of the next group are loaded while the current
//                 one is written;
//   warps 4..11   epilogue: per tile, read this CTA's accumulator rows from
//                 TMEM into registers, release the accumulator, round to bf16
//                 and store (rows >= M and columns >= N are skipped).
// The accumulator (256 columns) and four scale-factor slots (16 columns each,
// one group each) share the 512 TMEM columns. A slot's shared memory is
// rewritten only after the copy that read it has completed (sf_empty), and
// its TMEM columns only after the MMAs of the group that last used them have
// completed (sf_tfree), so no copy overwrites scale factors still in use.
//
// Every mbarrier wait is bounded; a wait that runs out records
// FP8BS_ERR_DEVICE_TIMEOUT and the CTA drains what it can observe and winds
// down; in a pair both CTAs always meet at the same cluster barriers, so
// neither waits on a CTA that has left. No TMA load uses .multicast::cluster.
#include "gemm_kernel.cuh"

namespace fp8bs {

namespace mx_detail {

constexpr int kBM = 128;                 // token rows per CTA (MMA M per CTA)
constexpr int kBN = 256;                 // weight rows per tile (MMA N)
constexpr int kABytes = kBM * 128;       // one K-block of A per CTA: 16 KB
constexpr int kSFChunk = 512;            // 32 rows x 16 bytes
constexpr int kSFBytes = 3 * kSFChunk;   // A (128 rows), B (256 rows = two chunks)
constexpr int kThreads = 384;
constexpr int kTmemCols = 512;
constexpr int kSFCol0 = kBN;             // scale factors after the accumulator
constexpr int kSFColsPerSlot = 16;       // A: 4 columns, B: 8 columns (+4 unused)
constexpr int kSFSlots = 4;              // groups of four K-blocks in flight
constexpr int kGroupK = 4;               // K-blocks per scale-factor group (bytes of a word)
constexpr int kEpiWarps = 8;

template <int kP>
struct MxCfg {
  static_assert(kP == 1 || kP == 2, "one CTA or a CTA pair");
  static constexpr int kBNc = kBN / kP;               // weight rows loaded per CTA
  static constexpr int kBBytes = kBNc * 128;
  static constexpr int kStages = kP == 2 ? 6 : 4;
  static constexpr int kOffA = 0;
  static constexpr int kOffB = kOffA + kStages * kABytes;
  static constexpr int kOffSF = kOffB + kStages * kBBytes;
  static constexpr int kOffBar = kOffSF + kSFSlots * kSFBytes;
  // full_tma, empty per stage; sf_full, sf_empty, sf_tfree per slot;
  // acc_full, acc_empty, mma_done
  static constexpr int kNumBars = 2 * kStages + 3 * kSFSlots + 3;
  static constexpr int kOffTmem = kOffBar + kNumBars * 8;
  static constexpr int kOffAbort = kOffTmem + 4;
  static constexpr int kSmemBytes = kOffAbort + 4 + 1024;   // + slack to align to 1024
  static_assert(kSmemBytes <= 227 * 1024, "shared memory");
  static_assert(kABytes % 1024 == 0 && kBBytes % 1024 == 0, "swizzled stages stay 1024-aligned");
  static_assert(kSFCol0 + kSFSlots * kSFColsPerSlot <= kTmemCols, "TMEM columns");
  // A slot's TMEM columns are reused four groups later; the MMAs of that
  // group are waited for explicitly (sf_tfree), whatever the group sizes.
  static constexpr uint32_t kIdesc = idesc_mxf8_e4m3_ue8m0(kBM * kP, kBN);
};

struct MxArgs {
  const uint8_t* sa8;    // [M][KB] UE8M0 codes of the activation groups
  const uint8_t* sw8;    // [NB][KB] UE8M0 codes of the weight blocks
  __nv_bfloat16* y;      // [M][N]
  int M, N, KB, NB;
  int row_tiles, col_tiles;   // tiles of kP * 128 token rows and 256 weight rows
  long long wait_limit;
  int* err;
  // Grouped (mixture-of-experts) GEMM, kP = 1: the expert of every token row
  // ([M], null = one weight matrix); weights [E][N][K], codes [E][NB][KB].
  // Every 128-row tile takes the expert of its first row (indices outside
  // [0, E) count as expert 0).
  const int* m_indices;
  int E;
  bool words_ok;   // both code arrays 4-byte aligned: a group's codes load as one word
};

__device__ __forceinline__ int mx_tile_expert(const MxArgs& a, int rt) {
  if (a.m_indices == nullptr) return 0;
  const int e = __ldg(a.m_indices + static_cast<int64_t>(rt) * kBM);
  return (e < 0 || e >= a.E) ? 0 : e;
}

template <int kP>
__global__ void __launch_bounds__(kThreads, 1)
    mx_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a,
                   const __grid_constant__ CUtensorMap tmap_b, const MxArgs args) {
  using C = MxCfg<kP>;
  constexpr int kStages = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sm_a = smem + C::kOffA;
  uint8_t* sm_b = smem + C::kOffB;
  uint8_t* sm_sf = smem + C::kOffSF;
  uint64_t* full_tma = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* empty = full_tma + kStages;
  uint64_t* sf_full = empty + kStages;
  uint64_t* sf_empty = sf_full + kSFSlots;
  uint64_t* sf_tfree = sf_empty + kSFSlots;
  uint64_t* acc_full = sf_tfree + kSFSlots;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* mma_done = acc_empty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffTmem);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffAbort);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int rank = kP == 2 ? static_cast<int>(cluster_ctarank()) : 0;
  const bool leader = rank == 0;
  const int unit = static_cast<int>(blockIdx.x) / kP;     // this CTA's cluster
  const int units = static_cast<int>(gridDim.x) / kP;
  const int num_tiles = args.row_tiles * args.col_tiles;
  const int KB = args.KB;
  const long long limit = args.wait_limit;
  // the abort flag as one result for the whole warp (keeps role loops converged)
  auto aborted = [&]() { return __any_sync(0xffffffffu, *abort_flag != 0); };

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full_tma[i], 1);        // rank 0's expect_tx arrival (+ both CTAs' bytes)
      mbar_init(&empty[i], 1);           // the MMA commit
    }
    for (int i = 0; i < kSFSlots; ++i) {
      mbar_init(&sf_full[i], kP);        // every CTA's scale-factor writer
      mbar_init(&sf_empty[i], 1);        // the commit after the slot's copies
      mbar_init(&sf_tfree[i], 1);        // the commit after the group's MMAs
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, kEpiWarps * kP);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
    tma_prefetch_desc(&tmap_a);
    tma_prefetch_desc(&tmap_b);
  }
  if (warp == 1) {
    if constexpr (kP == 2) {
      tmem_alloc_pair(tmem_slot, kTmemCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, kTmemCols);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  // both CTAs' barriers are initialised before either CTA touches the other's
  if constexpr (kP == 2) cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // Inputs may come from the previous kernel of the stream.
  grid_dependency_wait();
  grid_launch_dependents();

  // shared::cluster addresses of rank 0's barriers (the pair's MMA side)
  auto leader_bar = [&](uint64_t* bar) -> uint32_t {
    return kP == 2 ? map_cluster(smem_u32(bar), 0u) : smem_u32(bar);
  };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer --
    int stage = 0;
    uint32_t phase = 0;
    int issued = 0;
    for (int tile = unit; tile < num_tiles && !aborted(); tile += units) {
      int rt, ct;
      gemm_detail::tile_coords(tile, args.row_tiles, args.col_tiles, rt, ct);
      // weight rows of this CTA's half of the tile (of its expert, if grouped)
      const int brow = ct * kBN + rank * C::kBNc + mx_tile_expert(args, rt) * args.N;
      const int arow = (rt * kP + rank) * kBM;
      bool ok = true;
      for (int kb = 0; kb < KB; ++kb) {
        if (!mbar_wait_warp(&empty[stage], phase ^ 1u, limit)) {
          record_device_error(args.err, FP8BS_ERR_DEVICE_TIMEOUT);
          *abort_flag = 1;
          ok = false;
          break;
        }
        if (elect_one()) {
          uint8_t* da = sm_a + stage * kABytes;
          uint8_t* db = sm_b + stage * C::kBBytes;
          if constexpr (kP == 2) {
            if (leader) mbar_arrive_expect_tx(&full_tma[stage], kP * (kABytes + C::kBBytes));
            const uint32_t bar = leader_bar(&full_tma[stage]);
            tma_load_3d_pair(da, &tmap_a, bar, 0, arow, kb);
            tma_load_3d_pair(db, &tmap_b, bar, 0, brow, kb);
          } else {
            mbar_arrive_expect_tx(&full_tma[stage], kABytes + C::kBBytes);
            tma_load_3d(da, &tmap_a, &full_tma[stage], 0, arow, kb);
            tma_load_3d(db, &tmap_b, &full_tma[stage], 0, brow, kb);
          }
        }
        __syncwarp();
        ++issued;
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
    }
    // Every copy issued must have landed before shared memory goes away. The
    // copies of both CTAs of a pair complete on rank 0's barriers, so rank 0
    // waits for them; rank 1 does not leave before rank 0 (the final cluster
    // barrier).
    if (leader) {
      const int pending = issued < kStages ? issued : kStages;
      for (int i = 0; i < pending; ++i) {
        int s = stage - 1 - i;
        uint32_t ph = phase;
        if (s < 0) {
          s += kStages;
          ph ^= 1u;
        }
        mbar_wait(&full_tma[s], ph, kDefaultWaitCycles);
      }
    }
  } else if (warp == 1) {
    // -------------------------------------------------------------- MMA issuer --
    // Scale-factor groups are numbered in this CTA's order of work: group q
    // covers K-blocks [4g, 4g + 4) (clipped to KB) of its q / ceil(KB/4)-th
    // tile, and lives in slot q % kSFSlots.
    if (leader) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      const int groups_per_tile = (KB + kGroupK - 1) / kGroupK;
      const int my_tiles = unit < num_tiles ? (num_tiles - 1 - unit) / units + 1 : 0;
      const int total_groups = my_tiles * groups_per_tile;
      const uint64_t da0 = sw128_kmajor_desc(smem_u32(sm_a));
      const uint64_t db0 = sw128_kmajor_desc(smem_u32(sm_b));
      const uint64_t dsf0 = noswizzle_kmajor_desc(smem_u32(sm_sf), 128);
      int q = 0;        // group of the K-block being issued
      int copied = 0;   // groups whose scale factors have been copied into TMEM
      // Copy group `copied` into its TMEM slot. Non-blocking: only if its
      // shared-memory chunks are already written. Returns false on a wait
      // that ran out.
      auto copy_next = [&](bool blocking) -> bool {
        const int g = copied;
        const int slot = g % kSFSlots;
        const uint32_t ph = static_cast<uint32_t>(g / kSFSlots) & 1u;
        if (blocking) {
          if (!(kP == 2 ? __all_sync(0xffffffffu, mbar_wait_cluster(&sf_full[slot], ph, limit))
                        : mbar_wait_warp(&sf_full[slot], ph, limit)))
            return false;
        } else if (!__all_sync(0xffffffffu, mbar_test_wait(&sf_full[slot], ph))) {
          return true;   // not written yet; try again later
        }
        // the MMAs that last read this slot's TMEM columns (group g - 4) are done
        if (g >= kSFSlots && !mbar_wait_warp(&sf_tfree[slot], ph ^ 1u, limit)) return false;
        tc_fence_after();
        const uint32_t t = tmem_base + static_cast<uint32_t>(kSFCol0 + slot * kSFColsPerSlot);
        const uint64_t d = dsf0 + static_cast<uint32_t>((slot * kSFBytes) >> 4);
        if (elect_one()) {
          if constexpr (kP == 2) {
            tmem_cp_32x128b_warpx4_pair(t, d);
            tmem_cp_32x128b_warpx4_pair(t + 4u, d + (kSFChunk >> 4));
            tmem_cp_32x128b_warpx4_pair(t + 8u, d + ((2 * kSFChunk) >> 4));
            mma_commit_pair_mc(&sf_empty[slot], 0x3);
          } else {
            tmem_cp_32x128b_warpx4(t, d);
            tmem_cp_32x128b_warpx4(t + 4u, d + (kSFChunk >> 4));
            tmem_cp_32x128b_warpx4(t + 8u, d + ((2 * kSFChunk) >> 4));
            mma_commit(&sf_empty[slot]);
          }
        }
        __syncwarp();
        ++copied;
        return true;
      };
      for (int tile = unit; ok && tile < num_tiles && !aborted(); tile += units) {
        // every epilogue of the pair has read the previous tile's accumulator
        if (!(kP == 2 ? __all_sync(0xffffffffu, mbar_wait_cluster(acc_empty, acc_phase ^ 1u, limit))
                      : mbar_wait_warp(acc_empty, acc_phase ^ 1u, limit))) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int kb = 0; kb < KB; ++kb) {
          // this group's scale factors must be in TMEM; the next group's are
          // copied as soon as they are written, a group ahead of their use
          if (copied <= q && !copy_next(true)) {
            ok = false;
            break;
          }
          if (copied == q + 1 && q + 1 < total_groups && !copy_next(false)) {
            ok = false;
            break;
          }
          if (!mbar_wait_warp(&full_tma[stage], phase, limit)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int slot = q % kSFSlots;
          const uint32_t sf = tmem_base + static_cast<uint32_t>(kSFCol0 + slot * kSFColsPerSlot);
          const uint32_t idesc = idesc_with_sf_id(C::kIdesc, static_cast<uint32_t>(kb % kGroupK));
          const uint64_t da = da0 + static_cast<uint32_t>((stage * kABytes) >> 4);
          const uint64_t db = db0 + static_cast<uint32_t>((stage * C::kBBytes) >> 4);
          const bool group_end = kb % kGroupK == kGroupK - 1 || kb == KB - 1;
          if (elect_one()) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const uint64_t aj = da + static_cast<uint32_t>((32 * j) >> 4);
              const uint64_t bj = db + static_cast<uint32_t>((32 * j) >> 4);
              const uint32_t acc = (kb | j) != 0 ? 1u : 0u;
              if constexpr (kP == 2) mma_mxf8f6f4_bs_pair(tmem_base, aj, bj, idesc, sf, sf + 4u, acc);
              else mma_mxf8f6f4_bs(tmem_base, aj, bj, idesc, sf, sf + 4u, acc);
            }
            if constexpr (kP == 2) {
              mma_commit_pair_mc(&empty[stage], 0x3);
              if (group_end) mma_commit_pair_mc(&sf_tfree[slot], 0x1);
            } else {
              mma_commit(&empty[stage]);
              if (group_end) mma_commit(&sf_tfree[slot]);
            }
          }
          __syncwarp();
          if (group_end) ++q;
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        if (elect_one()) {
          if constexpr (kP == 2) mma_commit_pair_mc(acc_full, 0x3);
          else mma_commit(acc_full);
        }
        __syncwarp();
        acc_phase ^= 1u;
      }
      if (!ok) {
        record_device_error(args.err, FP8BS_ERR_DEVICE_TIMEOUT);
        *abort_flag = 1;
      }
      // every MMA and copy issued must be complete before TMEM is freed (in
      // both CTAs of a pair)
      if (elect_one()) {
        if constexpr (kP == 2) mma_commit_pair_mc(mma_done, 0x3);
        else mma_commit(mma_done);
      }
      __syncwarp();
    }
    mbar_wait(mma_done, 0, kDefaultWaitCycles);
  } else if (warp == 2) {
    // ------------------------------------------------------------ scale factors --
    // Words of one group (four K-blocks from kg) of a tile: lane l holds those
    // of token rows l + 32 j of this CTA's rows and of the tile's two weight
    // blocks; byte i of a word is the code of K-block kg + i (0 past KB).
    struct Words {
      uint32_t a[4];
      uint32_t b[2];
    };
    // groups are whole, 4-byte aligned words
    const bool kb_aligned = KB % kGroupK == 0 && args.words_ok;
    auto word_of = [&](const uint8_t* row_codes, int kg) -> uint32_t {
      if (kb_aligned) return *reinterpret_cast<const uint32_t*>(row_codes + kg);
      uint32_t w = 0;
#pragma unroll
      for (int i = 0; i < kGroupK; ++i)
        if (kg + i < KB) w |= static_cast<uint32_t>(row_codes[kg + i]) << (8 * i);
      return w;
    };
    auto load_group = [&](int tile, int kg, Words& c) {
      c.a[0] = c.a[1] = c.a[2] = c.a[3] = 0u;
      c.b[0] = c.b[1] = 0u;
      if (tile >= num_tiles) return;
      int rt, ct;
      gemm_detail::tile_coords(tile, args.row_tiles, args.col_tiles, rt, ct);
      const int nb0 = ct * (kBN / 128);
      const uint8_t* sw8 = args.sw8 + static_cast<int64_t>(mx_tile_expert(args, rt)) * args.NB * KB;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int row = (rt * kP + rank) * kBM + lane + 32 * j;
        if (row < args.M) c.a[j] = word_of(args.sa8 + static_cast<int64_t>(row) * KB, kg);
      }
#pragma unroll
      for (int h = 0; h < 2; ++h)
        if (nb0 + h < args.NB) c.b[h] = word_of(sw8 + static_cast<int64_t>(nb0 + h) * KB, kg);
    };
    const uint32_t sf_full_leader0 = leader_bar(&sf_full[0]);
    int q = 0;
    Words cur, nxt;
    load_group(unit, 0, cur);
    bool ok = true;
    for (int tile = unit; ok && tile < num_tiles && !aborted(); tile += units) {
      for (int kg = 0; kg < KB; kg += kGroupK, ++q) {
        // the group after this one: prefetched while this one is written
        if (kg + kGroupK < KB) load_group(tile, kg + kGroupK, nxt);
        else load_group(tile + units, 0, nxt);
        const int slot = q % kSFSlots;
        const uint32_t ph = static_cast<uint32_t>(q / kSFSlots) & 1u;
        if (!mbar_wait_warp(&sf_empty[slot], ph ^ 1u, limit)) {
          record_device_error(args.err, FP8BS_ERR_DEVICE_TIMEOUT);
          *abort_flag = 1;
          ok = false;
          break;
        }
        uint8_t* sf = sm_sf + slot * kSFBytes + 16 * lane;
        *reinterpret_cast<uint4*>(sf) = make_uint4(cur.a[0], cur.a[1], cur.a[2], cur.a[3]);
        *reinterpret_cast<uint4*>(sf + kSFChunk) = make_uint4(cur.b[0], cur.b[0], cur.b[0], cur.b[0]);
        *reinterpret_cast<uint4*>(sf + 2 * kSFChunk) =
            make_uint4(cur.b[1], cur.b[1], cur.b[1], cur.b[1]);
        // the tensor core's copy reads these bytes through the async proxy
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          if constexpr (kP == 2) mbar_arrive_remote(sf_full_leader0 + 8u * slot);
          else mbar_arrive(&sf_full[slot]);
        }
        cur = nxt;
      }
    }
  } else if (warp >= 4) {
    // ---------------------------------------------------------------- epilogue --
    const int quarter = warp & 3;          // TMEM lanes [32 quarter, 32 quarter + 32)
    const int wg = (warp - 4) >> 2;        // columns [128 wg, 128 wg + 128)
    const int row = quarter * 32 + lane;
    const uint32_t acc_empty_leader = leader_bar(acc_empty);
    uint32_t acc_phase = 0;
    for (int tile = unit; tile < num_tiles; tile += units) {
      int rt, ct;
      gemm_detail::tile_coords(tile, args.row_tiles, args.col_tiles, rt, ct);
      if (!mbar_wait_warp(acc_full, acc_phase, limit)) {
        record_device_error(args.err, FP8BS_ERR_DEVICE_TIMEOUT);
        *abort_flag = 1;
        break;
      }
      acc_phase ^= 1u;
      tc_fence_after();
      float v[128];
      const uint32_t taddr =
          tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(wg * 128);
#pragma unroll
      for (int c = 0; c < 128; c += 32) tmem_ld32(taddr + c, v + c);
      tmem_wait_ld();
      // the accumulator is free for the next tile's MMAs
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if constexpr (kP == 2) mbar_arrive_remote(acc_empty_leader);
        else mbar_arrive(acc_empty);
      }
      const int64_t m = static_cast<int64_t>(rt * kP + rank) * kBM + row;
      const int n0 = ct * kBN + wg * 128;
      if (m < args.M) {
        __nv_bfloat16* yrow = args.y + m * args.N + n0;
#pragma unroll
        for (int c = 0; c < 128; c += 8) {
          if (n0 + c < args.N) {
            uint4 pk;
            pk.x = gemm_detail::pack_bf16x2(v[c + 0], v[c + 1]);
            pk.y = gemm_detail::pack_bf16x2(v[c + 2], v[c + 3]);
            pk.z = gemm_detail::pack_bf16x2(v[c + 4], v[c + 5]);
            pk.w = gemm_detail::pack_bf16x2(v[c + 6], v[c + 7]);
            *reinterpret_cast<uint4*>(yrow + c) = pk;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  // neither CTA of a pair frees its TMEM or leaves while the other may still
  // use it (MMAs of rank 0 write rank 1's TMEM; copies of rank 1 complete on
  // rank 0's barriers)
  if constexpr (kP == 2) cluster_sync();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    if constexpr (kP == 2) tmem_dealloc_pair(tmem_base, kTmemCols);
    else tmem_dealloc(tmem_base, kTmemCols);
  }
}

template <int kP>
int launch_mx(const void* qa, const void* qw, MxArgs a, int64_t M, int64_t N, int64_t K,
              const DeviceInfo& dev, cudaStream_t stream) {
  using C = MxCfg<kP>;
  a.words_ok = ((reinterpret_cast<uintptr_t>(a.sa8) | reinterpret_cast<uintptr_t>(a.sw8)) & 3u) == 0;
  a.row_tiles = static_cast<int>((M + kP * kBM - 1) / (kP * kBM));
  a.col_tiles = static_cast<int>((N + kBN - 1) / kBN);
  const int64_t tiles = static_cast<int64_t>(a.row_tiles) * a.col_tiles;
  if (tiles > 0x7FFFFFFF) return FP8BS_ERR_SHAPE;
  const uint64_t KB = static_cast<uint64_t>(K / 128);
  alignas(64) CUtensorMap ta, tb;
  if (int st = encode_tmap_kblocks(&ta, qa, 128, M, KB, K, kBM, 1, kSwizzle128B)) return st;
  const uint64_t b_rows = static_cast<uint64_t>(N) * (a.m_indices != nullptr ? a.E : 1);
  if (int st = encode_tmap_kblocks(&tb, qw, 128, b_rows, KB, K, C::kBNc, 1, kSwizzle128B))
    return st;
  auto kern = mx_gemm_kernel<kP>;
  static std::once_flag flags[64];
  cudaError_t attr_err = cudaSuccess;
  std::call_once(flags[dev.device], [&] {
    attr_err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    C::kSmemBytes);
  });
  if (attr_err != cudaSuccess) return FP8BS_ERR_CUDA;
  // persistent: as many CTAs (pairs) as can be resident at once, at most one
  // per tile
  int units = dev.sm_count / kP;
  if (kP == 2) {
    const int fit = gemm_detail::max_active_clusters(kern, kThreads, C::kSmemBytes, 2, dev.device);
    if (fit <= 0) return FP8BS_ERR_CUDA;
    units = fit;
  }
  if (tiles < units) units = static_cast<int>(tiles);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(units * kP), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attrs[2];
  attrs[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attrs;
  cfg.numAttrs = 1;
  if (kP == 2) {
    attrs[1].id = cudaLaunchAttributeClusterDimension;
    attrs[1].val.clusterDim.x = 2;
    attrs[1].val.clusterDim.y = 1;
    attrs[1].val.clusterDim.z = 1;
    cfg.numAttrs = 2;
  }
  if (cudaLaunchKernelEx(&cfg, kern, ta, tb, a) != cudaSuccess) return FP8BS_ERR_CUDA;
  return FP8BS_OK;
}

}  // namespace mx_detail

int launch_block_gemm_ue8m0(const void* qa, const uint8_t* sa8, const void* qw, const uint8_t* sw8,
                            void* y, int64_t M, int64_t N, int64_t K, long long wait_limit,
                            int* err, cudaStream_t stream) {
  using namespace mx_detail;
  DeviceInfo dev;
  if (int st = current_device_info(&dev)) return st;
  MxArgs a{};
  a.sa8 = sa8;
  a.sw8 = sw8;
  a.y = static_cast<__nv_bfloat16*>(y);
  a.M = static_cast<int>(M);
  a.N = static_cast<int>(N);
  a.KB = static_cast<int>(K / 128);
  a.NB = static_cast<int>((N + 127) / 128);
  a.wait_limit = wait_limit;
  a.err = err;
  // a pair needs two 128-row halves to fill its M = 256 MMA
  if (M > kBM) return launch_mx<2>(qa, qw, a, M, N, K, dev, stream);
  return launch_mx<1>(qa, qw, a, M, N, K, dev, stream);
}

int launch_block_gemm_grouped_ue8m0(const void* qa, const uint8_t* sa8, const void* qw,
                                    const uint8_t* sw8, const int* m_indices, void* y, int64_t M,
                                    int64_t N, int64_t K, int64_t E, long long wait_limit, int* err,
                                    cudaStream_t stream) {
  using namespace mx_detail;
  DeviceInfo dev;
  if (int st = current_device_info(&dev)) return st;
  MxArgs a{};
  a.sa8 = sa8;
  a.sw8 = sw8;
  a.y = static_cast<__nv_bfloat16*>(y);
  a.M = static_cast<int>(M);
  a.N = static_cast<int>(N);
  a.KB = static_cast<int>(K / 128);
  a.NB = static_cast<int>((N + 127) / 128);
  a.wait_limit = wait_limit;
  a.err = err;
  a.m_indices = m_indices;
  a.E = static_cast<int>(E);
  // single-CTA tiles of 128 token rows: one expert per tile
  return launch_mx<1>(qa, qw, a, M, N, K, dev, stream);
}

}  // namespace fp8bs
