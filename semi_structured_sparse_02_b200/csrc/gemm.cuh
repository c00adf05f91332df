// gemm.cuh -- kernels 2 and 3: persistent, warp-specialized tcgen05 GEMM for
// sm_100a.  One template covers the dense MMA, the 2:4 sparse MMA
// (tcgen05.mma.sp, metadata in tensor memory) and the hybrid tile mix.
//
//   warp 0       TMA producer: A tile, B tile(s) and metadata chunk(s) of each
//                K-stage into a STAGES-deep shared-memory ring (mbarriers).
//   warp 1       tensor-memory allocator; lane 0 issues tcgen05.cp (metadata
//                shared -> tensor memory) and tcgen05.mma into one of two fp32
//                accumulators in tensor memory, then tcgen05.commit.
//   warps 2..5   epilogue: tcgen05.ld of the accumulator, scales, output
//                store, or split-K partial store + last-arriver reduction.
//
// The sparse operand is always MMA operand A ("Sparse tensor cores", section
// 2 of the 2:4-versus-quantization paper: the compressed first operand's
// indices pick the matching elements of the dense operand B).  For weights
// (W sparse) A = W and the accumulator holds Y^T (lane = output feature n,
// column = token m); for online activations A = X (lane = token m).
#pragma once

#include <cuda_bf16.h>

#include "sp24_device.cuh"

namespace sp24 {

enum GemmMode : int { kModeDense = 0, kModeSparse = 1, kModeHybrid = 2 };

constexpr int kGemmThreads = 192;
constexpr int kBlockA = 128;  // MMA M: rows of A per tile

struct GemmParams {
  int32_t rows_a, rows_b;     // A rows (tile_a dim), B rows (tile_b dim)
  int32_t K;                  // logical reduction length
  int32_t num_kt;             // K-stages per tile
  int32_t tiles_a, tiles_b;
  int32_t splits;             // split-K factor
  int32_t num_units;          // tiles_a * tiles_b * splits
  int32_t out_f32;            // 1: fp32 output, 0: bf16
  int32_t use_pdl;            // wait on the upstream grid before loading
  const uint8_t* meta;        // metadata image of A (sparse / hybrid)
  const uint8_t* tile_mask;   // hybrid: [tiles_a x K/128]
  const float* scale_a;       // per-A-row scale (E4M3) or null
  const float* scale_b;       // per-B-row scale (E4M3) or null
  void* Y;
  int64_t ldy;
  float* ws_partials;         // split-K partials [num_units][BN][128]
  unsigned int* ws_counters;  // split-K arrival counters [tiles]
  uint64_t timeout_ns;
};

// Compile-time geometry of one configuration.
template <int kMode, bool kBf16, int kBN>
struct GemmCfg {
  static constexpr bool kSparse = kMode == kModeSparse;
  static constexpr bool kHybrid = kMode == kModeHybrid;
  // logical K per stage
  static constexpr int kKT = kHybrid ? 128 : (kSparse ? (kBf16 ? 128 : 256) : (kBf16 ? 64 : 128));
  static constexpr int kABytes = kBlockA * 128;                 // A tile (dense or sparse)
  static constexpr int kBBoxes = kSparse ? 2 : 1;               // 128-byte-wide B boxes
  static constexpr int kBBytes = kBN * 128 * kBBoxes;
  static constexpr int kMetaChunks = kSparse ? (kBf16 ? 1 : 2) : (kHybrid ? 1 : 0);
  static constexpr int kMetaBytes = kMetaChunks * 2048;
  static constexpr int kStageBytes = kABytes + kBBytes + kMetaBytes;
  static constexpr int kSmemBudget = 225 * 1024;
  static constexpr int kStagesRaw = kSmemBudget / kStageBytes;
  static constexpr int kStages = kStagesRaw > 8 ? 8 : kStagesRaw;
  static_assert(kStages >= 2, "stage too large");
  static constexpr int kMetaCols = kMetaChunks * 4;              // tensor-memory columns per stage
  static constexpr int kAccCols = 2 * kBN;
  static constexpr int kColsNeeded = kAccCols + kStages * kMetaCols;
  static constexpr int kTmemCols = kColsNeeded <= 32 ? 32 : kColsNeeded <= 64 ? 64 :
                                   kColsNeeded <= 128 ? 128 : kColsNeeded <= 256 ? 256 : 512;
  static_assert(kColsNeeded <= 512, "tensor memory overflow");
  static constexpr int kMmasPerStage = 4;
  // bookkeeping after the stages
  static constexpr int kBarOffset = kStages * kStageBytes;
  static constexpr int kSmemBytes = kBarOffset + 256 + 1024;  // + barriers + alignment slack
};

// Byte counts the producer expects for one stage.
template <int kMode, bool kBf16, int kBN>
__device__ __forceinline__ uint32_t stage_tx_bytes(bool hybrid_dense, int meta_chunks) {
  using C = GemmCfg<kMode, kBf16, kBN>;
  if (C::kHybrid) return hybrid_dense ? (C::kABytes + kBN * 128) : (kBlockA * 64 + kBN * 128 + 2048);
  return C::kABytes + C::kBBytes + meta_chunks * 2048;
}

__device__ __forceinline__ void named_bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Named barrier with an AND reduction of a predicate over the participants.
__device__ __forceinline__ bool named_bar_red_and(int id, int count, bool pred) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 q, %1, 0;\n\t"
      "bar.red.and.pred p, %2, %3, q;\n\tselp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(out)
      : "r"((uint32_t)pred), "r"(id), "r"(count)
      : "memory");
  return out != 0;
}

template <int kMode, bool kBf16, int kBN, bool kAIsW>
__global__ void __launch_bounds__(kGemmThreads, 1)
k_gemm(const __grid_constant__ CUtensorMap tm_a,      // A: dense [rows_a x K] or values [rows_a x K/2]
       const __grid_constant__ CUtensorMap tm_a2,     // hybrid: values map (64-byte swizzle)
       const __grid_constant__ CUtensorMap tm_b,      // B: [rows_b x K]
       const GemmParams p) {
  using C = GemmCfg<kMode, kBf16, kBN>;
  constexpr int S = C::kStages;

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte alignment for the swizzled tiles
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOffset);
  // bars[0..S): full, [S..2S): empty, [2S..2S+2): acc_full, [2S+2..2S+4): acc_empty,
  // [2S+4]: drain
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * S + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* last_flag = reinterpret_cast<int*>(tmem_slot + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  auto full_bar = [&](int s) { return smem_u32(&bars[s]); };
  auto empty_bar = [&](int s) { return smem_u32(&bars[S + s]); };
  auto accf_bar = [&](int b) { return smem_u32(&bars[2 * S + b]); };
  auto acce_bar = [&](int b) { return smem_u32(&bars[2 * S + 2 + b]); };
  const uint32_t drain_bar = smem_u32(&bars[2 * S + 4]);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(accf_bar(b), 1);
      mbar_init(acce_bar(b), 128);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_b);
    if (C::kHybrid) tma_prefetch_desc(&tm_a2);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;

  if (p.use_pdl) pdl_wait();

  auto unit_coords = [&](int u, int& ta, int& tb, int& kb, int& ke) {
    const int tile = u / p.splits;
    const int s = u - tile * p.splits;
    ta = tile % p.tiles_a;
    tb = tile / p.tiles_a;
    kb = (int)(((int64_t)s * p.num_kt) / p.splits);
    ke = (int)(((int64_t)(s + 1) * p.num_kt) / p.splits);
  };
  auto is_dense_tile = [&](int ta, int kt) -> bool {
    return p.tile_mask[(int64_t)ta * p.num_kt + kt] != 0;
  };

  if (warp == 0) {
    // ------------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol_stream = policy_evict_first();  // A: read once
      const uint64_t pol_keep = policy_evict_last();     // B: re-read by many CTAs
      int stage = 0;
      uint32_t phase = 0;
      int armed[S];
      for (int s = 0; s < S; ++s) armed[s] = -1;
      bool ok = true;
      for (int u = blockIdx.x; u < p.num_units && ok; u += gridDim.x) {
        int ta, tb, kb, ke;
        unit_coords(u, ta, tb, kb, ke);
        for (int kt = kb; kt < ke; ++kt) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1, p.timeout_ns, kDevErrWaitEmpty)) {
            ok = false;
            *abort_flag = 1;
            break;
          }
          uint8_t* st = smem + stage * C::kStageBytes;
          const uint32_t sa = smem_u32(st);
          const uint32_t sb = sa + C::kABytes;
          const uint32_t sm = sb + C::kBBytes;
          const int32_t ya = ta * kBlockA, yb = tb * kBN;
          if (C::kHybrid) {
            const bool dense = is_dense_tile(ta, kt);
            mbar_arrive_expect_tx(full_bar(stage), stage_tx_bytes<kMode, kBf16, kBN>(dense, 1));
            if (dense) {
              tma_load_2d(sa, &tm_a, full_bar(stage), kt * 128, ya, pol_stream);
            } else {
              tma_load_2d(sa, &tm_a2, full_bar(stage), kt * 64, ya, pol_stream);
              bulk_load(sm, p.meta + ((int64_t)ta * p.num_kt + kt) * 2048, 2048, full_bar(stage),
                        pol_stream);
            }
            tma_load_2d(sb, &tm_b, full_bar(stage), kt * 128, yb, pol_keep);
          } else {
            int chunks = 0;
            if (C::kSparse) {
              const int kc_total = p.K / 128;
              const int kc0 = kt * C::kMetaChunks;
              chunks = min(C::kMetaChunks, kc_total - kc0);
            }
            mbar_arrive_expect_tx(full_bar(stage), stage_tx_bytes<kMode, kBf16, kBN>(false, chunks));
            // A: 128 bytes of each row per stage
            const int ax = C::kSparse ? kt * (C::kKT / 2) : kt * C::kKT;  // elements
            tma_load_2d(sa, &tm_a, full_bar(stage), ax, ya, pol_stream);
            // B: logical K range of the stage, in 128-byte boxes
            const int box_elems = kBf16 ? 64 : 128;
#pragma unroll
            for (int bx = 0; bx < C::kBBoxes; ++bx)
              tma_load_2d(sb + bx * kBN * 128, &tm_b, full_bar(stage), kt * C::kKT + bx * box_elems,
                          yb, pol_keep);
            if (C::kSparse) {
              const int64_t kc_total = p.K / 128;
              const uint8_t* src = p.meta + ((int64_t)ta * kc_total + (int64_t)kt * C::kMetaChunks) * 2048;
              bulk_load(sm, src, chunks * 2048, full_bar(stage), pol_stream);
            }
          }
          armed[stage] = (int)phase;
          if (++stage == S) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // wait (bounded) until every copy this thread started has landed
      for (int s = 0; s < S; ++s)
        if (armed[s] >= 0) mbar_wait(full_bar(s), (uint32_t)armed[s], p.timeout_ns, kDevErrWaitFull);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = make_idesc(C::kSparse, kBf16, kBlockA, kBN);
      const uint32_t idesc_dense = make_idesc(false, kBf16, kBlockA, kBN);
      const uint32_t idesc_sp = make_idesc(true, kBf16, kBlockA, kBN);
      const uint32_t meta_col0 = C::kAccCols;
      int stage = 0;
      uint32_t phase = 0;
      uint32_t acc_i = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < p.num_units && ok; u += gridDim.x) {
        int ta, tb, kb, ke;
        unit_coords(u, ta, tb, kb, ke);
        const int buf = acc_i & 1;
        const uint32_t acc_phase = (acc_i >> 1) & 1;
        if (!mbar_wait(acce_bar(buf), acc_phase ^ 1, p.timeout_ns, kDevErrWaitAccEmpty)) {
          ok = false;
          *abort_flag = 1;
          break;
        }
        tc_fence_after_sync();
        const uint32_t d = tmem_base + buf * kBN;
        for (int kt = kb; kt < ke; ++kt) {
          if (!mbar_wait(full_bar(stage), phase, p.timeout_ns, kDevErrWaitFull)) {
            ok = false;
            *abort_flag = 1;
            break;
          }
          tc_fence_after_sync();
          const uint32_t sa = smem_u32(smem + stage * C::kStageBytes);
          const uint32_t sb = sa + C::kABytes;
          const uint32_t sm = sb + C::kBBytes;
          const uint32_t mcol = meta_col0 + stage * C::kMetaCols;
          const bool first = kt == kb;
          if (C::kHybrid) {
            if (is_dense_tile(ta, kt)) {
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const uint64_t da = smem_desc(sa + j * 32, 16, 1024, kLayoutSw128);
                const uint64_t db = smem_desc(sb + j * 32, 16, 1024, kLayoutSw128);
                mma_f8(d, da, db, idesc_dense, (first && j == 0) ? 0u : 1u);
              }
            } else {
              tc_cp_128x128b(tmem_base + mcol, smem_desc(sm, 16, 128, kLayoutNone));
#pragma unroll
              for (int j = 0; j < 2; ++j) {
                const uint64_t da = smem_desc(sa + j * 32, 16, 512, kLayoutSw64);
                const uint64_t db = smem_desc(sb + j * 64, 16, 1024, kLayoutSw128);
                mma_sp_f8(d, da, db, tmem_base + mcol + 2 * j, idesc_sp, (first && j == 0) ? 0u : 1u);
              }
            }
          } else if (C::kSparse) {
            const int kc_total = p.K / 128;
            const int chunks = min(C::kMetaChunks, kc_total - kt * C::kMetaChunks);
            for (int c = 0; c < chunks; ++c)
              tc_cp_128x128b(tmem_base + mcol + 4 * c, smem_desc(sm + c * 2048, 16, 128, kLayoutNone));
            const int n_mma = kBf16 ? 4 : 2 * chunks;
            for (int j = 0; j < n_mma; ++j) {
              const uint64_t da = smem_desc(sa + j * 32, 16, 1024, kLayoutSw128);
              const uint64_t db = smem_desc(sb + (j >> 1) * kBN * 128 + (j & 1) * 64, 16, 1024,
                                            kLayoutSw128);
              const uint32_t acc = (first && j == 0) ? 0u : 1u;
              if (kBf16) {
                // one 32-bit metadata column per k-block; the selector picks
                // the odd column of an even-aligned pair
                const uint32_t col = mcol + j;
                mma_sp_bf16(d, da, db, tmem_base + (col & ~1u), idesc_sp | (col & 1u), acc);
              } else {
                // two metadata columns per k-block
                const uint32_t col = mcol + 4 * (j >> 1) + 2 * (j & 1);
                mma_sp_f8(d, da, db, tmem_base + col, idesc_sp, acc);
              }
            }
          } else {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const uint64_t da = smem_desc(sa + j * 32, 16, 1024, kLayoutSw128);
              const uint64_t db = smem_desc(sb + j * 32, 16, 1024, kLayoutSw128);
              if (kBf16) mma_bf16(d, da, db, idesc, (first && j == 0) ? 0u : 1u);
              else mma_f8(d, da, db, idesc, (first && j == 0) ? 0u : 1u);
            }
          }
          tc_commit(empty_bar(stage));  // frees the stage once these MMAs are done
          if (++stage == S) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        tc_commit(accf_bar(buf));
        ++acc_i;
      }
      // drain: every MMA and copy issued above has completed
      tc_commit(drain_bar);
      mbar_wait(drain_bar, 0, p.timeout_ns, kDevErrWaitDrain);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ epilogue
    const int lg = warp & 3;                   // tensor-memory lane group of this warp
    const int row = lg * 32 + lane;            // accumulator row (lane) within the tile
    const int et = threadIdx.x - 64;           // 0..127
    uint32_t acc_i = 0;
    for (int u = blockIdx.x; u < p.num_units; u += gridDim.x) {
      int ta, tb, kb, ke;
      unit_coords(u, ta, tb, kb, ke);
      const int buf = acc_i & 1;
      const uint32_t acc_phase = (acc_i >> 1) & 1;
      bool ok = mbar_wait(accf_bar(buf), acc_phase, p.timeout_ns, kDevErrWaitAccFull);
      __syncwarp();
      ok = named_bar_red_and(2, 128, ok);  // all epilogue threads agree
      if (!ok) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after_sync();
      const int ga = ta * kBlockA + row;     // global A row of this thread
      const bool a_live = ga < p.rows_a;
      const float sa_v = (p.scale_a != nullptr && a_live) ? p.scale_a[ga] : 1.0f;
      const uint32_t tbase = tmem_base + ((uint32_t)(lg * 32) << 16) + buf * kBN;
      float* part = p.splits > 1 ? p.ws_partials + (int64_t)u * kBN * 128 : nullptr;
#pragma unroll 1
      for (int c0 = 0; c0 < kBN; c0 += 16) {
        uint32_t r[16];
        tmem_ld_x16(tbase + c0, r);
        tmem_ld_wait();
        if (part != nullptr) {
#pragma unroll
          for (int i = 0; i < 16; ++i) __stcg(part + (c0 + i) * 128 + row, __uint_as_float(r[i]));
        } else {
          const int gb0 = tb * kBN + c0;
          if (kAIsW) {
            // lane = n (output feature), column = m (token)
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const int m = gb0 + i;
              if (m < p.rows_b && a_live) {
                float v = __uint_as_float(r[i]) * sa_v;
                if (p.scale_b != nullptr) v *= p.scale_b[m];
                if (p.out_f32) static_cast<float*>(p.Y)[(int64_t)m * p.ldy + ga] = v;
                else static_cast<__nv_bfloat16*>(p.Y)[(int64_t)m * p.ldy + ga] = __float2bfloat16_rn(v);
              }
            }
          } else {
            // lane = m (token), column = n (output feature)
            if (a_live) {
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const int n = gb0 + i;
                if (n < p.rows_b) {
                  float v = __uint_as_float(r[i]) * sa_v;
                  if (p.scale_b != nullptr) v *= p.scale_b[n];
                  if (p.out_f32) static_cast<float*>(p.Y)[(int64_t)ga * p.ldy + n] = v;
                  else static_cast<__nv_bfloat16*>(p.Y)[(int64_t)ga * p.ldy + n] = __float2bfloat16_rn(v);
                }
              }
            }
          }
        }
      }
      tc_fence_before_sync();
      mbar_arrive(acce_bar(buf));  // accumulator may be overwritten now
      ++acc_i;

      if (part != nullptr) {
        // split-K: the last unit of this tile to arrive sums all partials in
        // slot order (deterministic) and writes the output.
        const int tile = u / p.splits;
        __threadfence();
        named_bar_sync(1, 128);
        if (et == 0) {
          const unsigned int old = atomicAdd(&p.ws_counters[tile], 1u);
          *last_flag = (old == (unsigned int)(p.splits - 1)) ? 1 : 0;
        }
        named_bar_sync(1, 128);
        if (*last_flag) {
          __threadfence();
          const float* base = p.ws_partials + (int64_t)tile * p.splits * kBN * 128;
#pragma unroll 1
          for (int c = 0; c < kBN; ++c) {
            const int gb = tb * kBN + c;
            float v = 0.0f;
            for (int s = 0; s < p.splits; ++s) v += __ldcg(base + ((int64_t)s * kBN + c) * 128 + row);
            if (kAIsW) {
              if (gb < p.rows_b && a_live) {
                v *= sa_v;
                if (p.scale_b != nullptr) v *= p.scale_b[gb];
                if (p.out_f32) static_cast<float*>(p.Y)[(int64_t)gb * p.ldy + ga] = v;
                else static_cast<__nv_bfloat16*>(p.Y)[(int64_t)gb * p.ldy + ga] = __float2bfloat16_rn(v);
              }
            } else {
              if (gb < p.rows_b && a_live) {
                v *= sa_v;
                if (p.scale_b != nullptr) v *= p.scale_b[gb];
                if (p.out_f32) static_cast<float*>(p.Y)[(int64_t)ga * p.ldy + gb] = v;
                else static_cast<__nv_bfloat16*>(p.Y)[(int64_t)ga * p.ldy + gb] = __float2bfloat16_rn(v);
              }
            }
          }
          if (et == 0) p.ws_counters[tile] = 0u;  // ready for the next call
        }
        named_bar_sync(1, 128);
      }
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Bounded-wait self test: waits on a barrier that nothing completes.
// ---------------------------------------------------------------------------
__device__ int g_selftest_result = -1;

__global__ void k_selftest_bounded_wait(uint64_t timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const bool ok = mbar_wait(smem_u32(&bar), 0, timeout_ns, kDevErrSelftest);
    g_selftest_result = ok ? 1 : 0;
  }
}

}  // namespace sp24
