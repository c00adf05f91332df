// gemm_wide_prune.cuh -- online activations pruned inside the GEMM: the
// CTA-pair GEMM with X (bf16) as the sparse operand, where X is pruned 2:4 and
// compressed in shared memory by the kernel itself, with no compressed copy
// of X in HBM (the 2:4-versus-quantization paper, paperpeel.com/paper/
// 2610.28947, sections 3.5 "Measuring speed" and 4.2: a dynamic operand pays
// for its own prune and compress every call).
//
//   warp 0        both CTAs: TMA producer.  Per stage, the CTA's 128 raw X rows
//                 x 128 positions (two 128-byte boxes, 128-byte swizzle) into the
//                 stage's staging area (counted on the CTA's own raw barrier),
//                 and the CTA's half of the W tile (counted on rank 0's stage
//                 barrier).  No multicast.
//   warp 1        tensor memory; rank 0, lane 0 issues the metadata copy and the
//                 pair MMAs (tcgen05.mma.sp.cta_group::2, M = 256, N = 256).
//   warps 2..5    epilogue (lane = token row of Y), as in k_gemm_wide.
//   warps 6..13   converters, both CTAs: thread t takes half t % 2 (64
//                 positions) of row t / 2; it reads its raw half-row, and once
//                 all converters have read (the compressed tile overwrites the
//                 staging area) writes the kept values in the swizzled sparse
//                 operand layout and its metadata nibbles; then the image rows
//                 are built from the nibbles, the writes are made visible to the
//                 tensor core (async proxy) and one converter arrives on rank
//                 0's stage barrier (3 arrivals complete a stage: rank 0's
//                 producer and the converters of both CTAs).
//
// Pruning an X tile in the producer repeats the prune for every W tile the X
// tile meets (N / 256 times), so this path trades HBM bytes for CUDA-core
// work; the two-kernel path (prune once, then the GEMM) stays available and
// the two are measured side by side.
#pragma once

#include <cuda_bf16.h>

#include "gemm.cuh"
#include "prune.cuh"

namespace sp24 {

constexpr int kPruneGemmThreads = 448;   // 6 warps as in k_gemm_wide + 8 converter warps

struct WidePruneLaunch {
  CUtensorMap tm_x;          // X: bf16 [rows_a x K]; box 64 elements x 128 rows, SW128
  CUtensorMap tm_b;          // W: bf16 [rows_b x K]; box 64 elements x 128 rows, SW128
  int32_t rows_a, rows_b, K, num_kt;
  int32_t tiles_a, tiles_b, total_tiles, b_fastest;
  int32_t out_f32, use_pdl;
  void* Y;
  int64_t ldy;
  uint16_t* x_values_out;    // NULL, or compressed X [rows_a x K/2] (written by the tiles of W block 0)
  uint8_t* x_meta_out;       // NULL, or the metadata image of X
  uint64_t timeout_ns;
};

struct WidePruneCfg {
  static constexpr int kStageBytes = 32768 + 32768 + 2048;  // raw X / compressed A, W half, metadata
  static constexpr int kStages = 3;
  static constexpr int kBOffset = 32768;
  static constexpr int kMetaOffset = 65536;
  static constexpr int kOverlap = 32;
  static constexpr int kAcc1 = 256 - kOverlap;
  static constexpr int kMetaCol0 = 512 - kOverlap;
  static constexpr int kBarOffset = kStages * kStageBytes;
  static constexpr int kCanonOffset = kBarOffset + 256;
  static constexpr int kEpiOffset = kCanonOffset + 2048;
  static constexpr int kSmemBytes = kEpiOffset + 4 * 2048 + 1024;
  static_assert(kStages * 4 <= kOverlap, "metadata slots overflow");
  static_assert(kSmemBytes <= 232448, "shared memory overflow");
};

template <bool kEmit>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPruneGemmThreads, 1)
k_gemm_wide_prune(const __grid_constant__ WidePruneLaunch g) {
  using C = WidePruneCfg;
  constexpr int S = C::kStages;
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
  // [0,S) full (rank 0), [S,2S) empty, [2S,3S) raw (own CTA), [3S,3S+2) acc full,
  // [3S+2,3S+4) acc empty (rank 0), [3S+4] drain
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3 * S + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint8_t (*canon)[16] = reinterpret_cast<uint8_t (*)[16]>(smem + C::kCanonOffset);
  uint8_t* s_epi = smem + C::kEpiOffset;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1;
  const int n_pairs = gridDim.x >> 1;
  auto bar_u32 = [&](int i) { return smem_u32(&bars[i]); };
  const int kFull = 0, kEmpty = S, kRaw = 2 * S, kAccFull = 3 * S, kAccEmpty = 3 * S + 2, kDrain = 3 * S + 4;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(bar_u32(kFull + s), 3);  // rank 0's producer + the converters of both CTAs
      mbar_init(bar_u32(kEmpty + s), 1);
      mbar_init(bar_u32(kRaw + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_u32(kAccFull + b), 1);
      mbar_init(bar_u32(kAccEmpty + b), 8);
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
  cluster_sync();
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;

  const int num_kt = g.num_kt, total_tiles = g.total_tiles, tiles_a = g.tiles_a, tiles_b = g.tiles_b;
  const bool b_fastest = g.b_fastest != 0;
  const uint64_t timeout_ns = g.timeout_ns;
  auto tile_coords = [&](int tile, int& ta, int& tb) {
    ta = b_fastest ? tile / tiles_b : tile % tiles_a;
    tb = b_fastest ? tile % tiles_b : tile / tiles_a;
  };

  if (warp == 0) {
    // ------------------------------------------------------------------ producer (both CTAs)
    wait_upstream();
    if (lane == 0) {
      const uint32_t full0 = mapa_shared(bar_u32(kFull), 0);
      const uint64_t pol_x = policy_evict_last();  // an X tile is read again for every W tile
      int armed_raw[S];
      for (int s = 0; s < S; ++s) armed_raw[s] = -1;
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = pair; ok && tile < total_tiles; tile += n_pairs) {
        int ta, tb;
        tile_coords(tile, ta, tb);
        const int ya = ta * 256 + (int)rank * 128;
        const int yb = tb * 256 + (int)rank * 128;
        for (int kt = 0; kt < num_kt; ++kt) {
          if (!mbar_wait(bar_u32(kEmpty + stage), phase ^ 1, timeout_ns, kDevErrWaitEmpty)) {
            ok = false;
            *abort_flag = 1;
            break;
          }
          const uint32_t sa = smem_u32(smem + stage * C::kStageBytes);
          mbar_arrive_expect_tx(bar_u32(kRaw + stage), 32768u);
          armed_raw[stage] = (int)phase;
#pragma unroll
          for (int bx = 0; bx < 2; ++bx)
            tma_load_2d(sa + bx * 16384, &g.tm_x, bar_u32(kRaw + stage), kt * 128 + bx * 64, ya, pol_x);
          if (rank == 0) mbar_arrive_expect_tx(bar_u32(kFull + stage), 2u * 32768u);
#pragma unroll
          for (int bx = 0; bx < 2; ++bx)
            tma_load_2d_pair(sa + C::kBOffset + bx * 16384, &g.tm_b, full0 + 8u * stage, kt * 128 + bx * 64, yb);
          if (++stage == S) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      for (int s = 0; s < S; ++s)
        if (armed_raw[s] >= 0) mbar_wait(bar_u32(kRaw + s), (uint32_t)armed_raw[s], timeout_ns, kDevErrWaitFull);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer (rank 0)
    wait_upstream();
    if (rank == 0 && lane == 0) {
      const uint32_t idesc = make_idesc(true, true, 256, 256);
      const uint32_t s0 = smem_u32(smem);
      const uint64_t da0 = smem_desc(s0, 16, 1024, kLayoutSw128);
      const uint64_t db0 = smem_desc(s0 + C::kBOffset, 16, 1024, kLayoutSw128);
      const uint64_t dm0 = smem_desc(s0 + C::kMetaOffset, 16, 128, kLayoutNone);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int j = 0;
      for (int tile = pair; ok && tile < total_tiles; tile += n_pairs, ++j) {
        const int b = j & 1;
        if (j >= 1) {
          const int jr = j - 1;
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
          const uint64_t so = (uint64_t)((uint32_t)stage * (uint32_t)(C::kStageBytes >> 4));
          const uint32_t mcol = C::kMetaCol0 + stage * 4;
          tc_cp_128x128b_pair(tmem_base + mcol, dm0 + so);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint64_t a_d = da0 + so + (uint64_t)(q * 2);
            const uint64_t b_d = db0 + so + (uint64_t)(((q >> 1) * 16384 + (q & 1) * 64) >> 4);
            const uint32_t col = mcol + q;
            mma_sp_bf16_pair(d, a_d, b_d, tmem_base + (col & ~1u), idesc | (col & 1u), (kt == 0 && q == 0) ? 0u : 1u);
          }
          tc_commit_pair(bar_u32(kEmpty + stage), 0x3);
          if (++stage == S) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        tc_commit_pair(bar_u32(kAccFull + b), 0x3);
      }
      tc_commit_pair(bar_u32(kDrain), 0x1);
      mbar_wait(bar_u32(kDrain), 0, timeout_ns, kDevErrWaitDrain);
    }
    __syncwarp();
  } else if (warp < 6) {
    // ------------------------------------------------------------------ epilogue (both CTAs)
    wait_upstream();
    const int lg = warp & 3;
    const int row = lg * 32 + lane;
    const uint32_t acc_empty0 = mapa_shared(bar_u32(kAccEmpty), 0);
    const bool out_f32 = g.out_f32 != 0;
    const int rows_a = g.rows_a, rows_b = g.rows_b;
    uint8_t* const Yb = static_cast<uint8_t*>(g.Y);
    const int64_t ldy = g.ldy;
    (void)s_epi;
    int j = 0;
    for (int tile = pair; tile < total_tiles; tile += n_pairs, ++j) {
      int ta, tb;
      tile_coords(tile, ta, tb);
      const int b = j & 1;
      const int ga = ta * 256 + (int)rank * 128 + row;  // token row of this thread
      bool ok = mbar_wait(bar_u32(kAccFull + b), (uint32_t)((j >> 1) & 1), timeout_ns, kDevErrWaitAccFull);
      __syncwarp();
      ok = named_bar_red_and(2, 128, ok);
      if (!ok) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after_sync();
      const uint32_t tbase = tmem_base + ((uint32_t)(lg * 32) << 16) + (b ? (uint32_t)C::kAcc1 : 0u);
      // 16 consecutive output features n of token row ga per call
      auto drain = [&](int c_begin, int c_end) {
#pragma unroll 1
        for (int c0 = c_begin; c0 < c_end; c0 += 16) {
          uint32_t r[16];
          tmem_ld_x16(tbase + c0, r);
          tmem_ld_wait();
          if (ga >= rows_a) continue;
          const int gb0 = tb * 256 + c0;
          uint8_t* dst = Yb + ((int64_t)ga * ldy + gb0) * (out_f32 ? 4 : 2);
          if (out_f32) {
            if (gb0 + 16 <= rows_b) {
#pragma unroll
              for (int q = 0; q < 4; ++q)
                reinterpret_cast<uint4*>(dst)[q] = make_uint4(r[4 * q], r[4 * q + 1], r[4 * q + 2], r[4 * q + 3]);
            } else {
              for (int e = 0; e < rows_b - gb0; ++e) reinterpret_cast<uint32_t*>(dst)[e] = r[e];
            }
          } else {
            uint32_t w[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const __nv_bfloat162 h = __floats2bfloat162_rn(__uint_as_float(r[2 * q]), __uint_as_float(r[2 * q + 1]));
              w[q] = *reinterpret_cast<const uint32_t*>(&h);
            }
            if (gb0 + 16 <= rows_b) {
              reinterpret_cast<uint4*>(dst)[0] = make_uint4(w[0], w[1], w[2], w[3]);
              reinterpret_cast<uint4*>(dst)[1] = make_uint4(w[4], w[5], w[6], w[7]);
            } else {
              for (int e = 0; e < rows_b - gb0; ++e)
                reinterpret_cast<uint16_t*>(dst)[e] = (uint16_t)((w[e >> 1] >> (16 * (e & 1))) & 0xFFFFu);
            }
          }
        }
      };
      auto release = [&]() {
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(acc_empty0 + 8u * b);
      };
      const int ov0 = b ? 0 : 256 - C::kOverlap;
      drain(ov0, ov0 + C::kOverlap);
      release();
      if (b) drain(C::kOverlap, 256);
      else drain(0, 256 - C::kOverlap);
    }
  } else {
    // ------------------------------------------------------------------ converters (both CTAs)
    wait_upstream();  // X may belong to the upstream grid (the TMA reads follow the producer's wait)
    const int t = threadIdx.x - 192;   // 0..255
    const int r = t >> 1, h = t & 1;   // row of the CTA's 128, half (64 positions) of the stage
    const uint32_t full0 = mapa_shared(bar_u32(kFull), 0);
    uint16_t* const xv_out = g.x_values_out;
    uint8_t* const xm_out = g.x_meta_out;
    const int rows_a = g.rows_a, K = g.K;
    const int meta_blocks = (rows_a + 127) / 128;
    int stage = 0;
    uint32_t phase = 0;
    for (int tile = pair; tile < total_tiles; tile += n_pairs) {
      int ta, tb;
      tile_coords(tile, ta, tb);
      const int rb = ta * 2 + (int)rank;  // 128-row block of X
      const bool emit = kEmit && tb == 0 && rb < meta_blocks;
      bool ok = true;
      for (int kt = 0; kt < num_kt; ++kt) {
        uint8_t* sa = smem + stage * C::kStageBytes;
        ok = mbar_wait(bar_u32(kRaw + stage), phase, timeout_ns, kDevErrWaitFull);
        ok = named_bar_red_and(3, 256, ok);  // every converter takes the same decision
        if (!ok) {
          *abort_flag = 1;
          break;
        }
        // this thread's 64 raw positions: the 8 16-byte chunks of row r in box h
        uint4 raw[8];
#pragma unroll
        for (int c = 0; c < 8; ++c)
          raw[c] = *reinterpret_cast<const uint4*>(sa + h * 16384 + r * 128 + ((c ^ (r & 7)) << 4));
        named_bar_sync(3, 256);  // all raw reads precede the compressed writes (same area)
        uint32_t kept[16];       // 32 kept bf16, two per word, ascending
        uint32_t nibs[2] = {0u, 0u};
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 v = raw[c];
          const uint32_t n0 = prune_pick4w(v.x, v.y, kept[2 * c]);
          const uint32_t n1 = prune_pick4w(v.z, v.w, kept[2 * c + 1]);
          nibs[c >> 2] |= (n0 | (n1 << 4)) << (8 * (c & 3));
        }
        // the compressed row: 128 bytes = 8 chunks, this half's 4 chunks
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int cc = h * 4 + i;
          *reinterpret_cast<uint4*>(sa + r * 128 + ((cc ^ (r & 7)) << 4)) =
              make_uint4(kept[4 * i], kept[4 * i + 1], kept[4 * i + 2], kept[4 * i + 3]);
        }
        *reinterpret_cast<uint2*>(&canon[r][h * 8]) = make_uint2(nibs[0], nibs[1]);
        if (emit) {
          const int64_t grow = (int64_t)rb * 128 + r;
          if (grow < rows_a) {
            uint4* dst = reinterpret_cast<uint4*>(xv_out + grow * (K / 2) + (int64_t)kt * 64 + h * 32);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[i] = make_uint4(kept[4 * i], kept[4 * i + 1], kept[4 * i + 2], kept[4 * i + 3]);
          }
        }
        named_bar_sync(3, 256);  // canon complete
        if (t < 128) {
          const uint4 w = image_row<false>(canon, t);
          *reinterpret_cast<uint4*>(sa + C::kMetaOffset + t * 16) = w;
          if (emit) *reinterpret_cast<uint4*>(xm_out + ((int64_t)rb * (K / 128) + kt) * 2048 + t * 16) = w;
        }
        fence_proxy_async_smem();  // the writes above feed the tensor core (async proxy)
        named_bar_sync(3, 256);    // every write and fence precedes the arrive; canon reusable
        if (t == 0) mbar_arrive_cluster(full0 + 8u * stage);
        if (++stage == S) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (!ok) break;
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc_pair(tmem_base, 512);
  }
}

}  // namespace sp24
