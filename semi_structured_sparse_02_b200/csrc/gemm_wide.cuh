// gemm_wide.cuh -- the large-M GEMM: a CTA pair (cluster of two, tcgen05
// cta_group::2) computes a 256 x 256 output tile (256 x 240 when A carries
// sparsity metadata) with one MMA stream.
//
// Why a pair.  A single CTA's 128 x 128 tile needs about 195 bytes of operand
// per clock at the sparse tensor rate (A 16 KB + B 32 KB + metadata 2 KB per
// 128-deep bf16 stage), above what one SM can pull from L2, and the N = 128
// MMA itself issues at only ~62% of the N = 256 rate.  In a pair each CTA
// holds 128 rows of A (weights) and 128 rows of B (tokens); the pair's MMA is
// M = 256 (A rows of both CTAs) by N = 256 (B rows of both CTAs), so every
// CTA computes a 128 x 256 block while loading only half of B: 50 KB per
// 128 x 256 x 128 stage, ~98 bytes per clock at the sparse rate.
//
//   warp 0       both CTAs: TMA producer for the CTA's own A, B and metadata
//                halves; completion is counted on rank 0's stage barrier
//                (which expects both halves).  No multicast.
//   warp 1       both CTAs allocate tensor memory (pair allocation); rank 0,
//                lane 0 issues tcgen05.cp (metadata, both CTAs) and the pair
//                MMAs, then commits to the stage / accumulator barriers of
//                both CTAs.
//   warps 2..5   both CTAs: epilogue of the CTA's 128 accumulator rows.
//
// Tensor memory (512 columns per CTA).  Dense: two 256-column accumulators.
// Sparse and hybrid: the metadata needs columns too, so the tile is 240 B
// rows wide (the MMA's N = 240, 120 B rows per CTA): the accumulators start at
// columns 0 and 256 as in the dense kernel, and the metadata slots take the
// 16 columns after each (240..255 and 496..511).  Both kinds keep two whole
// accumulators, so a tile's MMAs start while the previous tile is drained.  (Two 256-column accumulators that share 32 columns with the
// metadata would make every tile's first MMA wait for the previous tile's
// last one and for the epilogue to drain the shared columns: a measured
// ~1.7 us per tile.)
//
// Work schedule: whole tiles, round-robin over the pairs.  By
// default the A tile index runs fastest (consecutive pairs share a B tile; A
// is re-read from L2 for every B tile).  When A is the larger operand and B
// fits comfortably in L2 (b_fastest, chosen on the host), the B index runs
// fastest instead, so that each A tile streams from HBM once and B is the
// operand re-read from L2.
//
// Hybrid weights (E4M3, a dense/sparse flag per 128 x 128 tile of A): the
// two CTAs of a pair hold two different 128-row blocks, and one pair MMA
// serves both, so each 128-deep K-step runs dense when either block's tile is
// dense there and sparse otherwise.  A dense step loads both halves from the
// dense-form copy of A (where a sparse tile is stored pruned), a sparse step
// the compressed values and metadata.  The producer warp reads the tile's
// flags into shared memory when it starts a tile; the stage kind goes to the
// MMA thread through shared memory, ordered by the stage barrier.
#pragma once

#include <type_traits>

#include "gemm.cuh"

namespace sp24 {

struct WideLaunch {
  CUtensorMap tm_a;     // A: dense [rows_a x K] or values [rows_a x K/2]; 128-byte box x 128 rows, SW128
  CUtensorMap tm_b;     // B: [rows_b x K]; 128-byte box x kBHalf rows (128, or 120 with metadata), SW128
  CUtensorMap tm_meta;  // metadata image viewed as [chunks * 8 rows x 256 B]; box 256 B x 8 * chunks rows
  CUtensorMap tm_a2;    // hybrid: values [rows_a x K/2]; 64-byte box x 128 rows, SW64 (tm_a: dense form)
  const uint8_t* tile_mask;  // hybrid: [ceil(rows_a/128) x K/128] dense flags
  int32_t rows_a, rows_b, K, num_kt;
  int32_t tiles_a, tiles_b;  // 256-row tiles of A, kBN-row tiles of B
  int32_t total_tiles, meta_blocks;  // metadata row blocks (128 rows) that exist
  int32_t b_fastest;                 // tile order: B tile index fastest (else A)
  int32_t out_f32, use_pdl;
  const float* scale_a;
  const float* scale_b;
  void* Y;
  int64_t ldy;
  uint64_t timeout_ns;
};

template <int kMode, bool kBf16>
struct WideCfg {
  static constexpr bool kSparse = kMode == kModeSparse;
  static constexpr bool kHybrid = kMode == kModeHybrid;  // E4M3 only
  static constexpr bool kUsesMeta = kSparse || kHybrid;
  static_assert(!kHybrid || !kBf16, "hybrid tiles are E4M3");
  // logical K per stage; a hybrid stage is one 128-deep tile column
  static constexpr int kKT = kSparse ? (kBf16 ? 128 : 256) : (kHybrid ? 128 : (kBf16 ? 64 : 128));
  static constexpr int kABytes = 128 * 128;  // hybrid: dense 128 x 128 B, or sparse 128 x 64 B
  static constexpr int kBBoxes = kSparse ? 2 : 1;
  static constexpr int kBN = kUsesMeta ? 240 : 256;  // B rows of a pair tile (the MMA's N)
  static constexpr int kBHalf = kBN / 2;             // B rows per CTA
  static constexpr int kBBoxBytes = kBHalf * 128;    // one 128-byte-wide box of B
  static constexpr int kBBytes = 128 * 128 * kBBoxes;  // boxes at 16 KB strides (1024-byte aligned)
  static constexpr int kMetaChunks = kSparse ? (kBf16 ? 1 : 2) : (kHybrid ? 1 : 0);
  static constexpr int kMetaBytes = kMetaChunks * 2048;
  static constexpr int kStageBytes = kABytes + kBBytes + kMetaBytes;  // per CTA
  static constexpr uint32_t kStageTx = kABytes + kBBoxes * kBBoxBytes + kMetaBytes;  // bytes a stage receives
  static constexpr int kStages = kSparse ? 4 : 6;
  static constexpr int kMetaCols = kMetaChunks * 4;
  static constexpr int kAcc1 = 256;  // first column of the second accumulator
  // metadata slots (sparse, hybrid): stage s in the gap after the first
  // accumulator, then in the gap after the second
  static constexpr int kSlotsPerGap = kUsesMeta ? (256 - kBN) / kMetaCols : 0;
  static_assert(!kUsesMeta || kStages <= 2 * kSlotsPerGap, "metadata slots overflow");
  __host__ __device__ static constexpr uint32_t meta_col(int s) {
    return s < kSlotsPerGap ? (uint32_t)(kBN + s * kMetaCols) : (uint32_t)(256 + kBN + (s - kSlotsPerGap) * kMetaCols);
  }
  static constexpr int kBarOffset = kStages * kStageBytes;
  static constexpr int kScaleOffset = kBarOffset + 256;
  static constexpr int kEpiOffset = kScaleOffset + 256 * 4;
  static constexpr int kMaxHybridKt = 2048;  // hybrid: K / 128 limit (one flag byte per K-step)
  static constexpr int kKindOffset = kEpiOffset + 4 * 2048;
  static constexpr int kSmemBytes = kKindOffset + (kHybrid ? kMaxHybridKt : 0) + 1024;  // + alignment slack
  static_assert(kSmemBytes <= 232448, "shared memory overflow");
};

template <int kMode, bool kBf16, bool kAIsW>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
k_gemm_wide(const __grid_constant__ WideLaunch g) {
  using C = WideCfg<kMode, kBf16>;
  constexpr int S = C::kStages;
  // programmatic dependent launch: every thread waits for the upstream grid
  // before it triggers the next launch, so a next GEMM that is independent of
  // this one may skip its own wait and still find this launch's inputs
  // complete
  if (!g.use_pdl) pdl_launch_dependents();
  auto wait_upstream = [&]() {
    if (g.use_pdl) {
      pdl_wait();
      pdl_launch_dependents();
    }
  };

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOffset);
  // bars[0..S): full (used in rank 0), [S..2S): empty, [2S..2S+2): acc_full,
  // [2S+2..2S+4): acc_empty (used in rank 0), [2S+4]: drain
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * S + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  // hybrid: the kind of each stage in flight (1 = dense), producer -> MMA
  volatile uint8_t* s_kind = reinterpret_cast<volatile uint8_t*>(tmem_slot + 2);
  // hybrid: the dense flag of every K-step of the producer's current tile
  volatile uint8_t* s_tile_kind = smem + C::kKindOffset;
  float* s_scale_b = reinterpret_cast<float*>(smem + C::kScaleOffset);
  uint8_t* s_epi = smem + C::kEpiOffset;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1;
  const int n_pairs = gridDim.x >> 1;

  auto bar_u32 = [&](int i) { return smem_u32(&bars[i]); };
  const int kFull = 0, kEmpty = S, kAccFull = 2 * S, kAccEmpty = 2 * S + 2, kDrain = 2 * S + 4;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(bar_u32(kFull + s), 1);
      mbar_init(bar_u32(kEmpty + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_u32(kAccFull + b), 1);
      mbar_init(bar_u32(kAccEmpty + b), 8);  // 4 epilogue warps in each of the 2 CTAs
    }
    mbar_init(bar_u32(kDrain), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), 512);
    tmem_relinquish_pair();
  }
  tc_fence_before_sync();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers initialized and tensor memory allocated
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;

  auto meta_chunks = [&](int kt) -> int {
    return (int)min((int64_t)C::kMetaChunks, (int64_t)(g.K / 128) - (int64_t)kt * C::kMetaChunks);
  };

  if (warp == 0 && C::kHybrid) {
    // ------------------------------------------------------------------ hybrid producer (both CTAs)
    // the whole warp reads a tile's dense flags; lane 0 issues the copies
    wait_upstream();
    const uint32_t full0 = mapa_shared(bar_u32(kFull), 0);
    const int num_kt = g.num_kt, total_tiles = g.total_tiles, tiles_a = g.tiles_a, meta_blocks = g.meta_blocks;
    const int tiles_b = g.tiles_b;
    const bool b_fastest = g.b_fastest != 0;
    const uint64_t timeout_ns = g.timeout_ns;
    const uint8_t* const mask = g.tile_mask;
    constexpr uint32_t kDenseTx = 2u * (128 * 128 + C::kBBoxBytes);          // A dense + B, both CTAs
    constexpr uint32_t kSparseTx = 2u * (128 * 64 + C::kBBoxBytes + 2048);   // A values + B + metadata
    int armed[S];
    for (int s = 0; s < S; ++s) armed[s] = -1;
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int tile = pair; tile < total_tiles; tile += n_pairs) {
      const int ta = b_fastest ? tile / tiles_b : tile % tiles_a;
      const int tb = b_fastest ? tile % tiles_b : tile / tiles_a;
      const int rb0 = ta * 2, rb1 = ta * 2 + 1;  // the pair's two 128-row blocks
      __syncwarp();  // lane 0 has finished with the previous tile's flags
      for (int kt = lane; kt < num_kt; kt += 32) {
        // a row block past the end of A counts as sparse (its rows are zero)
        const bool d = mask[(int64_t)rb0 * num_kt + kt] != 0 ||
                       (rb1 < meta_blocks && mask[(int64_t)rb1 * num_kt + kt] != 0);
        s_tile_kind[kt] = d ? 1 : 0;
      }
      __syncwarp();
      if (lane == 0) {
        const int ya = ta * 256 + (int)rank * 128;
        const int yb = tb * C::kBN + (int)rank * C::kBHalf;
        int rb = rb0 + (int)rank;
        if (rb >= meta_blocks) rb = 0;  // rows past the end: A is zero-filled; any valid metadata
        for (int kt = 0; kt < num_kt; ++kt) {
          if (!mbar_wait(bar_u32(kEmpty + stage), phase ^ 1, timeout_ns, kDevErrWaitEmpty)) {
            ok = false;
            *abort_flag = 1;
            break;
          }
          const bool dense = s_tile_kind[kt] != 0;
          if (rank == 0) {
            s_kind[stage] = dense ? 1 : 0;  // published by the arrive below (release)
            mbar_arrive_expect_tx(bar_u32(kFull + stage), dense ? kDenseTx : kSparseTx);
            armed[stage] = (int)phase;
          }
          const uint32_t sa = smem_u32(smem + stage * C::kStageBytes);
          const uint32_t fb = full0 + 8u * stage;
          if (dense) {
            tma_load_2d_pair(sa, &g.tm_a, fb, kt * 128, ya);
          } else {
            tma_load_2d_pair(sa, &g.tm_a2, fb, kt * 64, ya);
            tma_load_2d_pair(sa + C::kABytes + C::kBBytes, &g.tm_meta, fb, 0, (rb * num_kt + kt) * 8);
          }
          tma_load_2d_pair(sa + C::kABytes, &g.tm_b, fb, kt * 128, yb);
          if (++stage == S) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
    }
    // rank 0: wait (bounded) until every armed stage has landed
    if (lane == 0)
      for (int s = 0; s < S; ++s)
        if (armed[s] >= 0) mbar_wait(bar_u32(kFull + s), (uint32_t)armed[s], timeout_ns, kDevErrWaitFull);
    __syncwarp();
  } else if (warp == 0) {
    // ------------------------------------------------------------------ producer (both CTAs)
    if (lane != 0) wait_upstream();
    if (lane == 0) {
      wait_upstream();
      const uint32_t full0 = mapa_shared(bar_u32(kFull), 0);  // rank 0's stage barriers
      const int box_elems = kBf16 ? 64 : 128;                // 128 bytes of B per box row
      const int kc_total = g.K / 128;
      // parameter fields in registers (the asm below clobbers memory)
      const int num_kt = g.num_kt, total_tiles = g.total_tiles, tiles_a = g.tiles_a, meta_blocks = g.meta_blocks;
      const int tiles_b = g.tiles_b;
      const bool b_fastest = g.b_fastest != 0;
      const uint64_t timeout_ns = g.timeout_ns;
      int armed[S];
      for (int s = 0; s < S; ++s) armed[s] = -1;
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = pair; ok && tile < total_tiles; tile += n_pairs) {
        const int ta = b_fastest ? tile / tiles_b : tile % tiles_a;
        const int tb = b_fastest ? tile % tiles_b : tile / tiles_a;
        const int ya = ta * 256 + (int)rank * 128;
        const int yb = tb * C::kBN + (int)rank * C::kBHalf;
        int rb = ta * 2 + (int)rank;        // metadata row block of this CTA's A rows
        if (rb >= meta_blocks) rb = 0;    // rows past the end: A is zero-filled; any valid metadata
        for (int kt = 0; kt < num_kt; ++kt) {
          if (!mbar_wait(bar_u32(kEmpty + stage), phase ^ 1, timeout_ns, kDevErrWaitEmpty)) {
            ok = false;
            *abort_flag = 1;
            break;
          }
          if (rank == 0) {
            mbar_arrive_expect_tx(bar_u32(kFull + stage), 2u * C::kStageTx);
            armed[stage] = (int)phase;
          }
          const uint32_t sa = smem_u32(smem + stage * C::kStageBytes);
          const uint32_t fb = full0 + 8u * stage;
          const int ax = C::kSparse ? kt * (C::kKT / 2) : kt * C::kKT;
          tma_load_2d_pair(sa, &g.tm_a, fb, ax, ya);
#pragma unroll
          for (int bx = 0; bx < C::kBBoxes; ++bx)
            tma_load_2d_pair(sa + C::kABytes + bx * 16384, &g.tm_b, fb, kt * C::kKT + bx * box_elems, yb);
          if (C::kSparse)
            tma_load_2d_pair(sa + C::kABytes + C::kBBytes, &g.tm_meta, fb, 0,
                             (rb * kc_total + kt * C::kMetaChunks) * 8);
          if (++stage == S) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // rank 0: wait (bounded) until every armed stage has landed
      for (int s = 0; s < S; ++s)
        if (armed[s] >= 0) mbar_wait(bar_u32(kFull + s), (uint32_t)armed[s], timeout_ns, kDevErrWaitFull);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer (rank 0)
    wait_upstream();  // nothing to issue before the producer's loads anyway
    if (rank == 0 && lane == 0) {
      const uint32_t idesc = make_idesc(C::kSparse, kBf16, 256, C::kBN);
      const uint32_t idesc_dense = make_idesc(false, kBf16, 256, C::kBN);  // hybrid dense K-steps
      const uint32_t idesc_sp = make_idesc(true, kBf16, 256, C::kBN);      // hybrid sparse K-steps
      const uint32_t s0 = smem_u32(smem);
      const uint64_t da0 = smem_desc(s0, 16, 1024, kLayoutSw128);
      const uint64_t db0 = smem_desc(s0 + C::kABytes, 16, 1024, kLayoutSw128);
      const uint64_t dm0 = smem_desc(s0 + C::kABytes + C::kBBytes, 16, 128, kLayoutNone);
      // e4m3: the stage's two metadata chunks as one 128 x 256-bit copy
      const uint64_t dm2 = smem_desc(s0 + C::kABytes + C::kBBytes, 2048, 128, kLayoutNone);
      // hybrid sparse K-steps: A is 128 rows x 64 bytes, 64-byte swizzle
      const uint64_t dsp0 = smem_desc(s0, 16, 512, kLayoutSw64);
      const int num_kt = g.num_kt, total_tiles = g.total_tiles;
      const uint64_t timeout_ns = g.timeout_ns;
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int j = 0;
      for (int tile = pair; ok && tile < total_tiles; tile += n_pairs, ++j) {
        const int b = j & 1;
        // accumulator b is free once tile j-2 (the last one that used it) is drained
        if (j >= 2) {
          const int jr = j - 2;
          if (!mbar_wait(bar_u32(kAccEmpty + (jr & 1)), (uint32_t)((jr >> 1) & 1), timeout_ns,
                         kDevErrWaitAccEmpty)) {
            ok = false;
            *abort_flag = 1;
            break;
          }
        }
        tc_fence_after_sync();
        const uint32_t d = tmem_base + (b ? (uint32_t)C::kAcc1 : 0u);
        for (int kt = 0; kt < num_kt; ++kt) {
          if (!mbar_wait(bar_u32(kFull + stage), phase, timeout_ns, kDevErrWaitFull)) {
            ok = false;
            *abort_flag = 1;
            break;
          }
          tc_fence_after_sync();
          // this stage's descriptors: the stage-0 ones plus the stage offset
          // (the address field counts 16-byte units); the issuing thread is
          // on the critical path, so the loops below are fully unrolled
          const uint64_t so = (uint64_t)((uint32_t)stage * (uint32_t)(C::kStageBytes >> 4));
          const uint64_t da = da0 + so, db = db0 + so;
          const bool first = kt == 0;
          if (C::kHybrid) {
            const uint32_t mcol = C::meta_col(stage);
            if (s_kind[stage] != 0) {
#pragma unroll
              for (int q = 0; q < 4; ++q)
                mma_f8_pair(d, da + (uint64_t)(q * (32 >> 4)), db + (uint64_t)(q * (32 >> 4)), idesc_dense,
                            (first && q == 0) ? 0u : 1u);
            } else {
              tc_cp_128x128b_pair(tmem_base + mcol, dm0 + so);
#pragma unroll
              for (int q = 0; q < 2; ++q)
                mma_sp_f8_pair(d, dsp0 + so + (uint64_t)(q * (32 >> 4)), db + (uint64_t)(q * (64 >> 4)),
                               tmem_base + mcol + 2 * q, idesc_sp, (first && q == 0) ? 0u : 1u);
            }
          } else if (C::kSparse) {
            const uint32_t mcol = C::meta_col(stage);
            auto issue = [&](auto chunks_c) {
              constexpr int kChunks = decltype(chunks_c)::value;
              if (kChunks == 2) tc_cp_128x256b_pair(tmem_base + mcol, dm2 + so);
              else tc_cp_128x128b_pair(tmem_base + mcol, dm0 + so);
              constexpr int kMmas = kBf16 ? 4 : 2 * kChunks;
#pragma unroll
              for (int q = 0; q < kMmas; ++q) {
                const uint64_t a_d = da + (uint64_t)(q * (32 >> 4));
                const uint64_t b_d = db + (uint64_t)(((q >> 1) * 16384 + (q & 1) * 64) >> 4);
                const uint32_t acc = (first && q == 0) ? 0u : 1u;
                if (kBf16) {
                  const uint32_t col = mcol + q;
                  mma_sp_bf16_pair(d, a_d, b_d, tmem_base + (col & ~1u), idesc | (col & 1u), acc);
                } else {
                  const uint32_t col = mcol + 4 * (q >> 1) + 2 * (q & 1);
                  mma_sp_f8_pair(d, a_d, b_d, tmem_base + col, idesc, acc);
                }
              }
            };
            if (kBf16 || C::kMetaChunks == 1 || meta_chunks(kt) == C::kMetaChunks)
              issue(std::integral_constant<int, C::kMetaChunks>{});
            else
              issue(std::integral_constant<int, 1>{});
          } else {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint64_t a_d = da + (uint64_t)(q * (32 >> 4));
              const uint64_t b_d = db + (uint64_t)(q * (32 >> 4));
              if (kBf16) mma_bf16_pair(d, a_d, b_d, idesc, (first && q == 0) ? 0u : 1u);
              else mma_f8_pair(d, a_d, b_d, idesc, (first && q == 0) ? 0u : 1u);
            }
          }
          tc_commit_pair(bar_u32(kEmpty + stage), 0x3);  // frees the stage in both CTAs
          if (++stage == S) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        tc_commit_pair(bar_u32(kAccFull + b), 0x3);
      }
      tc_commit_pair(bar_u32(kDrain), 0x1);
      mbar_wait(bar_u32(kDrain), 0, g.timeout_ns, kDevErrWaitDrain);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ epilogue (both CTAs)
    wait_upstream();  // Y and the B scales may belong to the upstream grid
    const int lg = warp & 3;
    const int row = lg * 32 + lane;   // accumulator lane of this thread
    const int et = threadIdx.x - 64;  // 0..127
    const uint32_t acc_empty0 = mapa_shared(bar_u32(kAccEmpty), 0);
    uint8_t* wtile = s_epi + (warp - 2) * 2048;
    // values read once into registers (the asm statements below clobber
    // memory, which would force parameter fields to be re-read after each)
    const bool out_f32 = g.out_f32 != 0;
    const int rows_a = g.rows_a, rows_b = g.rows_b, tiles_a = g.tiles_a, total_tiles = g.total_tiles;
    const int tiles_b = g.tiles_b;
    const bool b_fastest = g.b_fastest != 0;
    uint8_t* const Yb = static_cast<uint8_t*>(g.Y);
    const int64_t ldy = g.ldy;
    const float* const scale_a = g.scale_a;
    const float* const scale_b = g.scale_b;
    int j = 0;
    for (int tile = pair; tile < total_tiles; tile += n_pairs, ++j) {
      const int ta = b_fastest ? tile / tiles_b : tile % tiles_a;
      const int tb = b_fastest ? tile % tiles_b : tile / tiles_a;
      const int b = j & 1;
      const int ga = ta * 256 + (int)rank * 128 + row;  // A row of this thread
      const float sa_v = (scale_a != nullptr && ga < rows_a) ? __ldg(scale_a + ga) : 1.0f;
      named_bar_sync(1, 128);  // the previous tile's stores are done with the B scales
      for (int i = et; i < C::kBN; i += 128) {
        const int gb = tb * C::kBN + i;
        s_scale_b[i] = (scale_b != nullptr && gb < rows_b) ? scale_b[gb] : 1.0f;
      }
      named_bar_sync(1, 128);
      bool ok = mbar_wait(bar_u32(kAccFull + b), (uint32_t)((j >> 1) & 1), g.timeout_ns, kDevErrWaitAccFull);
      __syncwarp();
      ok = named_bar_red_and(2, 128, ok);
      if (!ok) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after_sync();
      const uint32_t tbase = tmem_base + ((uint32_t)(lg * 32) << 16) + (b ? (uint32_t)C::kAcc1 : 0u);

      // scales and stores 16 accumulator columns starting at c0; EB (output
      // bytes) is a compile-time constant so the index arithmetic is shifts
      auto store16 = [&](auto eb_c, const float (&v)[16], int c0) {
        constexpr int EB = decltype(eb_c)::value;
        constexpr int PV = 16 / EB;  // elements per 16-byte vector
        const int gb0 = tb * C::kBN + c0;
        float sc[16];
#pragma unroll
        for (int i = 0; i < 16; i += 4) {
          const float4 t = *reinterpret_cast<const float4*>(s_scale_b + c0 + i);
          sc[i] = t.x * sa_v; sc[i + 1] = t.y * sa_v; sc[i + 2] = t.z * sa_v; sc[i + 3] = t.w * sa_v;
        }
        if (kAIsW) {
          // lane = output feature n, column = token m: stage the warp's
          // 32 n x 16 m block transposed, then write 16-byte vectors of n
          constexpr int VPR = 32 / PV;
          const int n0 = ta * 256 + (int)rank * 128 + lg * 32;
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float y = v[i] * sc[i];
            if (EB == 4) reinterpret_cast<float*>(wtile)[i * 32 + lane] = y;
            else reinterpret_cast<__nv_bfloat16*>(wtile)[i * 32 + lane] = __float2bfloat16_rn(y);
          }
          __syncwarp();
#pragma unroll
          for (int it = 0; it < 16 * VPR / 32; ++it) {
            const int q = lane + 32 * it;
            const int i = q / VPR, sg = q % VPR;
            const int m = gb0 + i;
            const int n = n0 + sg * PV;
            if (m < rows_b && n < rows_a) {
              uint8_t* dst = Yb + ((int64_t)m * ldy + n) * EB;
              const uint8_t* src = wtile + (i * 32 + sg * PV) * EB;
              if (n + PV <= rows_a) {
                *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(src);
              } else {
                for (int e = 0; e < (rows_a - n) * EB; ++e) dst[e] = src[e];
              }
            }
          }
          __syncwarp();
        } else {
          // lane = token m, column = output feature n: 16 consecutive n of row ga
          if (ga >= rows_a) return;
          constexpr int NW = 16 * EB / 4;
          uint32_t w[NW];
#pragma unroll
          for (int j = 0; j < NW; ++j) {
            if (EB == 4) {
              w[j] = __float_as_uint(v[j] * sc[j]);
            } else {
              const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * j] * sc[2 * j], v[2 * j + 1] * sc[2 * j + 1]);
              w[j] = *reinterpret_cast<const uint32_t*>(&h);
            }
          }
          uint8_t* dst = Yb + ((int64_t)ga * ldy + gb0) * EB;
          if (gb0 + 16 <= rows_b) {
#pragma unroll
            for (int q = 0; q < NW / 4; ++q)
              reinterpret_cast<uint4*>(dst)[q] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
          } else {
#pragma unroll
            for (int j = 0; j < NW; ++j) {
              const int e0 = j * 4 / EB;  // first output of word j
              if (e0 >= rows_b - gb0) break;
              if (EB == 4 || e0 + 1 < rows_b - gb0) reinterpret_cast<uint32_t*>(dst)[j] = w[j];
              else reinterpret_cast<uint16_t*>(dst)[2 * j] = (uint16_t)(w[j] & 0xFFFFu);
            }
          }
        }
      };
      auto store16_any = [&](const float (&v)[16], int c0) {
        if (out_f32) store16(std::integral_constant<int, 4>{}, v, c0);
        else store16(std::integral_constant<int, 2>{}, v, c0);
      };
      auto drain = [&](int c_begin, int c_end) {
#pragma unroll 1
        for (int c0 = c_begin; c0 < c_end; c0 += 16) {
          uint32_t r[16];
          tmem_ld_x16(tbase + c0, r);
          tmem_ld_wait();
          float v[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
          store16_any(v, c0);
        }
      };
      auto release = [&]() {
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(acc_empty0 + 8u * b);
      };
      drain(0, C::kBN);
      release();
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  cluster_sync();  // neither CTA leaves while its peer may still use its memory
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc_pair(tmem_base, 512);
  }
}

}  // namespace sp24
