// gemm.cuh -- kernels 2 and 3: persistent, warp-specialized tcgen05 GEMM for
// sm_100a.  One template covers the dense MMA, the 2:4 sparse MMA
// (tcgen05.mma.sp, metadata in tensor memory) and the hybrid tile mix, for
// one problem or a group of up to kMaxGroup independent problems.
//
//   warp 0       TMA producer: A tile, B tile(s) and metadata chunk(s) of each
//                K-stage into a STAGES-deep shared-memory ring (mbarriers).
//   warp 1       tensor-memory allocator; lane 0 issues tcgen05.cp (metadata
//                shared -> tensor memory) and tcgen05.mma into one of two fp32
//                accumulators in tensor memory, then tcgen05.commit.
//   warps 2..5   epilogue: tcgen05.ld of the accumulator, scales, output
//                store; or a stream-K partial store / finish.
//
// Work schedule.  "Data-parallel": each CTA takes whole output tiles
// round-robin over the tiles of all problems.  "Stream-K" (few tiles, e.g.
// decode): the K-iterations of all tiles of all problems are laid end to end
// and every CTA streams one contiguous range of them (the host cuts the
// ranges by estimated cost and passes the boundaries), so a group streams
// without gaps between problems.  A tile split between CTAs is finished by
// the unit that holds its first K-iteration: that unit's range ends inside
// the tile, so the tile is its last segment, while every other contributor's
// segment lies at the start of (or spans) its own range.  The others store
// their fp32 partial tile with plain stores into their one slot and raise a
// flag; the finisher checks the flags before its own accumulator is ready,
// adds the partials as it drains tensor memory, stores Y and clears the
// flags for the next call.  The split, and with it the fp32 addition order,
// is fixed by the plan.
//
// Kernel chaining.  Every CTA triggers the dependent grid at once
// (programmatic dependent launch).  With w_static the producer starts
// streaming the A operand (weights + metadata) before waiting on the
// upstream grid; everything the upstream grid may write (B, scales of B,
// the output) is touched only after griddepcontrol.wait.
//
// The sparse operand is always MMA operand A ("Sparse tensor cores", section
// 2 of the 2:4-versus-quantization paper: the compressed first operand's
// indices pick the matching elements of the dense operand B).  For weights
// (W sparse) A = W and the accumulator holds Y^T (lane = output feature n,
// column = token m); for online activations A = X (lane = token m).
#pragma once

#include <cuda_bf16.h>

#include <type_traits>

#include "sp24_device.cuh"

namespace sp24 {

// kModeNvSparse / kModeNvDense: block-scaled NVFP4 operands (kind::mxf4nvf4):
// A pairwise 4:8 sparse (values, metadata image, scales per 32 positions) or
// dense (scales per 16), B dense NVFP4, one fp32 tensor scale per operand.
enum GemmMode : int { kModeDense = 0, kModeSparse = 1, kModeHybrid = 2, kModeNvSparse = 3, kModeNvDense = 4 };
enum GemmSched : int { kSchedDataParallel = 0, kSchedStreamK = 1 };

constexpr int kGemmThreads = 192;
constexpr int kBlockA = 128;  // MMA M: rows of A per tile
constexpr int kMaxGroup = 16; // problems per grouped launch
constexpr int kMaxSkUnits = 160;  // stream-K scheduling units (SMs or CTA pairs) a launch may have

// One problem of a (possibly grouped) launch.
struct GemmProblem {
  int32_t rows_a, rows_b;     // A rows (tile_a dim), B rows (tile_b dim)
  int32_t K;                  // logical reduction length
  int32_t num_kt;             // K-stages per tile
  int32_t tiles_a, tiles_b;
  int32_t tile_begin;         // first global tile index of this problem
  int32_t meta_blocks;        // 128-row blocks of the metadata image (pair tiles clamp to it)
  int32_t bn;                 // token-tile width of this problem (16..kBN, a multiple of 16; kBN in a pair)
  int64_t iter_begin;         // first global stream-K iteration of this problem
  const uint8_t* meta;        // metadata image of A (sparse / hybrid)
  const uint8_t* tile_mask;   // hybrid: [tiles_a x K/128]
  const float* scale_a;       // per-A-row scale (E4M3), tensor scale (NVFP4) or null
  const float* scale_b;       // per-B-row scale (E4M3), tensor scale (NVFP4) or null
  const uint8_t* sfa;         // NVFP4: scale image of A
  const uint8_t* sfb;         // NVFP4: scale image of B
  void* Y;
  int64_t ldy;
};

struct GemmParams {
  int32_t n_prob;
  int32_t sched;              // kSchedDataParallel / kSchedStreamK
  int64_t total_iters;        // stream-K: sum over problems of tiles * num_kt
  int32_t total_tiles;        // sum over problems of tiles
  int32_t out_f32;            // 1: fp32 output, 0: bf16
  int32_t use_pdl;            // wait on the upstream grid before dependent loads
  int32_t w_static;           // A operands are not written by the upstream grid
  int32_t after_independent;  // the upstream grid is an independent GEMM: wait for it only at the end
  uint64_t timeout_ns;
  float* sk_slots;            // stream-K partial tiles [units][pair half][128 rows][BN] fp32
  unsigned int* sk_flags;     // "partial stored" flags [units][pair half]
  // stream-K: unit u takes global K-stages [sk_bound[u], sk_bound[u + 1]),
  // ranges cut so that every unit gets the same weighted stage cost
  int64_t sk_bound[kMaxSkUnits + 1];
};

// Everything a launch needs, passed by value (tensor maps must live in
// parameter, constant or global memory for TMA).
template <int kMaxProb>
struct GemmLaunch {
  CUtensorMap tm_a[kMaxProb];   // A: dense [rows_a x K] or values [rows_a x K/2]
  CUtensorMap tm_a2[kMaxProb];  // hybrid: values map (64-byte boxes, 64-byte swizzle)
  CUtensorMap tm_a3[kMaxProb];  // hybrid: values map (128-byte boxes, 128-byte swizzle)
  CUtensorMap tm_b[kMaxProb];   // B: [rows_b x K]
  GemmProblem prob[kMaxProb];
  GemmParams p;
};

// Compile-time geometry of one configuration.  kPair: the tile's 256 A rows
// are split over a CTA pair (tcgen05 cta_group::2); each CTA holds 128 A rows
// and kBN/2 of the kBN B rows, and the pair's MMA is M = 256 by N = kBN.
template <int kMode, bool kBf16, int kBN, bool kPair = false>
struct GemmCfg {
  static constexpr bool kSparse = kMode == kModeSparse;
  static constexpr bool kHybrid = kMode == kModeHybrid;
  static constexpr bool kNvSparse = kMode == kModeNvSparse;
  static constexpr bool kNv = kNvSparse || kMode == kModeNvDense;
  static_assert(!(kPair && (kHybrid || kNv)), "hybrid and NVFP4 tiles run on single CTAs");
  static constexpr int kRowsA = kPair ? 2 * kBlockA : kBlockA;  // A rows per tile
  static constexpr int kBRows = kPair ? kBN / 2 : kBN;          // B rows per CTA
  // logical K per stage (NVFP4: 128 bytes of A per row, four MMAs)
  // (hybrid: two 128 x 128 tile columns per stage, each dense or sparse)
  static constexpr int kKT = kNv ? (kNvSparse ? 512 : 256)
                                 : kHybrid ? 256 : (kSparse ? (kBf16 ? 128 : 256) : (kBf16 ? 64 : 128));
  // A tile (dense or sparse); hybrid: two 16 KB slots, one per tile column
  static constexpr int kABytes = kBlockA * 128 * (kHybrid ? 2 : 1);
  static constexpr int kBBoxes = (kSparse || kNvSparse || kHybrid) ? 2 : 1;  // 128-byte-wide B boxes
  static constexpr int kBBytes = kBRows * 128 * kBBoxes;
  static constexpr int kMetaChunks = kSparse ? (kBf16 ? 1 : 2) : ((kHybrid || kNvSparse) ? 2 : 0);
  static constexpr int kMetaBytes = kMetaChunks * 2048;
  // NVFP4: four 512-byte scale chunks of A, then four of B (one per MMA)
  static constexpr int kSfBytes = kNv ? 4096 : 0;
  static constexpr int kSfChunkK = kNvSparse ? 128 : 64;        // logical K of one scale chunk
  static constexpr int kStageBytes = kABytes + kBBytes + kMetaBytes + kSfBytes;
  static constexpr int kSmemBudget = 212 * 1024;
  static constexpr int kStagesRaw = kSmemBudget / kStageBytes;
  static constexpr int kStages = kStagesRaw > 8 ? 8 : kStagesRaw;
  static_assert(kStages >= 2, "stage too large");
  // tensor-memory columns per stage: metadata, then (NVFP4) 16 of A scales
  // and 16 of B scales
  static constexpr int kMetaCols = kMetaChunks * 4 + (kNv ? 32 : 0);
  static constexpr int kAccCols = 2 * kBN;
  static constexpr int kColsNeeded = kAccCols + kStages * kMetaCols;
  static constexpr int kTmemCols = kColsNeeded <= 32 ? 32 : kColsNeeded <= 64 ? 64 :
                                   kColsNeeded <= 128 ? 128 : kColsNeeded <= 256 ? 256 : 512;
  static_assert(kColsNeeded <= 512, "tensor memory overflow");
  // bookkeeping after the stages: barriers, slots, the B-scale slice, and a
  // 2 KB output-staging tile per epilogue warp
  static constexpr int kBarOffset = kStages * kStageBytes;
  static constexpr int kScaleOffset = kBarOffset + 512;
  // NVFP4: a seventh warp issues each stage's scale and metadata copies into
  // tensor memory, so the MMA thread issues only the stage's four MMAs
  static constexpr int kThreads = kNv ? 224 : kGemmThreads;
  static constexpr int kEpiOffset = kScaleOffset + ((kBN * 4 + 127) / 128) * 128;
  static constexpr int kSmemBytes = kEpiOffset + 4 * 2048 + 1024;  // + alignment slack
  static_assert(kSmemBytes <= 232448, "shared memory overflow");
};

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

// fp32 vector atomic add (fire and forget).
__device__ __forceinline__ void red_add_v4(float* p, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}

__device__ __forceinline__ void st_release_gpu(unsigned int* p, unsigned int v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ unsigned int ld_acquire_gpu(const unsigned int* p) {
  unsigned int v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// GPU-scope acquire-release fetch-add: publishes (with the preceding CTA
// barrier) the CTA's partial adds and acquires the other contributors'.
__device__ __forceinline__ unsigned int atom_add_acq_rel_gpu(unsigned int* p, unsigned int v) {
  unsigned int old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

// ---------------------------------------------------------------------------
// Work segments: a (problem, tile, k-begin, k-end) range; seg numbers the
// segments of one CTA.  Every role of a CTA walks the same sequence.
// ---------------------------------------------------------------------------
template <int kMaxProb>
struct SegIter {
  int64_t it, it1;    // stream-K global iteration cursor and end
  int tile_g;         // data-parallel global tile cursor
  int pr;             // problem cursor (only moves forward)
  int j;
  __device__ __forceinline__ void init(const GemmLaunch<kMaxProb>& g, int cta, int grid) {
    j = 0;
    pr = 0;
    if (g.p.sched == kSchedStreamK) {
      it = g.p.sk_bound[cta];
      it1 = g.p.sk_bound[cta + 1];
    } else {
      tile_g = cta;
    }
  }
  __device__ __forceinline__ bool next(const GemmLaunch<kMaxProb>& g, int grid, int& prob, int& tile,
                                       int& kb, int& ke, int& seg) {
    if (g.p.sched == kSchedStreamK) {
      if (it >= it1) return false;
      while (pr + 1 < g.p.n_prob && it >= g.prob[pr + 1].iter_begin) ++pr;
      const GemmProblem& P = g.prob[pr];
      const int64_t local = it - P.iter_begin;
      tile = (int)(local / P.num_kt);
      kb = (int)(local - (int64_t)tile * P.num_kt);
      ke = (int)min((int64_t)P.num_kt, (int64_t)kb + (it1 - it));
      it += ke - kb;
    } else {
      if (tile_g >= g.p.total_tiles) return false;
      while (pr + 1 < g.p.n_prob && tile_g >= g.prob[pr + 1].tile_begin) ++pr;
      tile = tile_g - g.prob[pr].tile_begin;
      kb = 0;
      ke = g.prob[pr].num_kt;
      tile_g += grid;
    }
    prob = pr;
    seg = j++;
    return true;
  }
};

// The unit (CTA or CTA pair) whose stream-K range holds global iteration i:
// the last unit whose range starts at or before i (binary search).
__device__ __forceinline__ int sk_owner(const GemmParams& p, int units, int64_t i) {
  int lo = 0, hi = units - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.sk_bound[mid] <= i) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

template <int kMode, bool kBf16, int kBN, bool kAIsW, int kMaxProb, bool kPair = false>
__global__ void __launch_bounds__(GemmCfg<kMode, kBf16, kBN, kPair>::kThreads, 1)
k_gemm(const __grid_constant__ GemmLaunch<kMaxProb> g) {
  using C = GemmCfg<kMode, kBf16, kBN, kPair>;
  constexpr int S = C::kStages;
  static_assert(!kPair || kAIsW, "pairs split the weight rows");
  const GemmParams& p = g.p;

  // Programmatic dependent launch.  A launch that depends on its upstream
  // grid lets the next kernel launch only after every thread has seen the
  // upstream complete (wait, then trigger), so a next kernel that is
  // independent of this one may skip its own wait and still find this
  // launch's inputs complete.  A launch after an independent GEMM triggers at
  // once and waits only before exiting (its completion then implies the
  // upstream's).
  const bool wait_first = p.use_pdl && !p.after_independent;
  if (!wait_first) pdl_launch_dependents();

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte alignment for the swizzled tiles
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOffset);
  // bars[0..S): full, [S..2S): empty, [2S..2S+2): acc_full, [2S+2..2S+4): acc_empty,
  // [2S+4]: drain, [2S+5..3S+5): copies done (NVFP4), [3S+5]: copy drain (NVFP4).
  // In a pair the full, acc_empty and drain barriers of rank 0 are used.
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3 * S + 6);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* last_flag = reinterpret_cast<int*>(tmem_slot + 2);
  // hybrid: the kind of each stage in flight (1 = dense), producer -> MMA
  // thread, published by the stage barrier's arrive
  volatile uint8_t* s_kind = reinterpret_cast<volatile uint8_t*>(tmem_slot + 3);
  float* s_scale_b = reinterpret_cast<float*>(smem + C::kScaleOffset);
  uint8_t* s_epi = smem + C::kEpiOffset;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // scheduling units: CTAs, or CTA pairs
  const uint32_t rank = kPair ? cluster_ctarank() : 0u;
  const int unit = kPair ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int units = kPair ? (int)(gridDim.x >> 1) : (int)gridDim.x;

  auto full_bar = [&](int s) { return smem_u32(&bars[s]); };
  auto empty_bar = [&](int s) { return smem_u32(&bars[S + s]); };
  auto accf_bar = [&](int b) { return smem_u32(&bars[2 * S + b]); };
  auto acce_bar = [&](int b) { return smem_u32(&bars[2 * S + 2 + b]); };
  const uint32_t drain_bar = smem_u32(&bars[2 * S + 4]);
  auto cpd_bar = [&](int s) { return smem_u32(&bars[2 * S + 5 + s]); };
  const uint32_t cpdrain_bar = smem_u32(&bars[3 * S + 5]);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(accf_bar(b), 1);
      mbar_init(acce_bar(b), kPair ? 8 : 4);  // one arrive per epilogue warp (of both CTAs)
    }
    mbar_init(drain_bar, 1);
    if (C::kNv) {
      for (int s = 0; s < S; ++s) mbar_init(cpd_bar(s), 1);
      mbar_init(cpdrain_bar, 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    if (kPair) {
      tmem_alloc_pair(smem_u32(tmem_slot), C::kTmemCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
      tmem_relinquish();
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  if (kPair) cluster_sync();  // the peer's barriers and tensor memory are ready
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;

  // metadata chunks (128 K positions each) of stage kt of problem P
  auto meta_chunks = [&](const GemmProblem& P, int kt) -> int {
    return (int)min((int64_t)C::kMetaChunks, (int64_t)(P.K / 128) - (int64_t)kt * C::kMetaChunks);
  };
  // NVFP4: a last stage that covers only half of kKT (K % kKT == kKT / 2)
  auto nv_half = [&](const GemmProblem& P, int kt) -> bool {
    return (int64_t)P.K - (int64_t)kt * C::kKT < C::kKT;
  };

  if (warp == 0 && C::kHybrid) {
    // ------------------------------------------------------------------ hybrid producer
    // A stage covers two 128 x 128 tile columns of A.  Both sparse: one
    // 128-byte box of compressed values (128-byte swizzle) and both metadata
    // chunks, as in a plain 2:4 stage.  Otherwise each column separately: a
    // dense column from A's dense form (16 KB, 128-byte swizzle) into its
    // slot, a sparse one as a 64-byte box of values (64-byte swizzle) plus its
    // metadata chunk.  The stage's kind (bit c: column c dense; bit 2: no
    // second column, K / 128 odd) goes to the MMA thread in s_kind before the
    // stage's barrier is armed (the arrive releases it).  The whole warp walks
    // the segments; every 16 stages the lanes read the next 32 dense flags of
    // the tile row in parallel (one ballot), so no flag costs a dependent
    // global load.
    const uint64_t pol_stream = policy_evict_first();
    const uint64_t pol_keep = policy_evict_last();

    int armed[S];
    for (int s = 0; s < S; ++s) armed[s] = -1;
    auto flag_word = [&](const GemmProblem& P, int ta, int c0) -> uint32_t {
      const int kcols = P.K / 128;
      const int c = c0 + lane;
      const bool d = c < kcols && P.tile_mask[(int64_t)ta * kcols + c] != 0;
      return __ballot_sync(0xFFFFFFFFu, d);
    };
    auto stage_kind = [&](const GemmProblem& P, int kt, int i, uint32_t fl) -> uint32_t {
      const int b = (2 * i) & 31;
      return ((fl >> b) & 3u) | (2 * kt + 1 >= P.K / 128 ? 4u : 0u);
    };
    auto a_bytes = [&](uint32_t kind) -> uint32_t {
      if (kind == 0) return 16384u + 4096u;
      uint32_t b = (kind & 1u) ? 16384u : 8192u + 2048u;
      if (!(kind & 4u)) b += (kind & 2u) ? 16384u : 8192u + 2048u;
      return b;
    };
    auto load_a = [&](int stage, const GemmProblem& P, int pr, int ta, int kt, uint32_t kind) {
      const uint32_t sa = smem_u32(smem + stage * C::kStageBytes);
      const uint32_t sm = sa + C::kABytes + C::kBBytes;
      const int32_t ya = ta * kBlockA;
      const int64_t chunk0 = (int64_t)ta * (P.K / 128) + 2 * (int64_t)kt;
      if (kind == 0) {
        tma_load_2d(sa, &g.tm_a3[pr], full_bar(stage), kt * 128, ya, pol_stream);
        bulk_load(sm, P.meta + chunk0 * 2048, 4096, full_bar(stage), pol_stream);
        return;
      }
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        if (c == 1 && (kind & 4u)) break;
        const uint32_t slot = sa + c * 16384;
        if ((kind >> c) & 1u) {
          tma_load_2d(slot, &g.tm_a[pr], full_bar(stage), (2 * kt + c) * 128, ya, pol_stream);
        } else {
          tma_load_2d(slot, &g.tm_a2[pr], full_bar(stage), (2 * kt + c) * 64, ya, pol_stream);
          bulk_load(sm + c * 2048, P.meta + (chunk0 + c) * 2048, 2048, full_bar(stage), pol_stream);
        }
      }
    };
    auto arm = [&](int stage, uint32_t kind, int ph, int bn) {
      s_kind[stage] = (uint8_t)kind;
      mbar_arrive_expect_tx(full_bar(stage), a_bytes(kind) + (uint32_t)(bn * 128 * 2));
      armed[stage] = ph;
    };
    // 1. static weights: the first S stages' A copies before the dependency wait
    int pre = 0;
    if (p.w_static) {
      SegIter<kMaxProb> it;
      it.init(g, unit, units);
      int pr, tile, kb, ke, seg;
      while (pre < S && it.next(g, units, pr, tile, kb, ke, seg)) {
        const GemmProblem& P = g.prob[pr];
        const int ta = tile % P.tiles_a;
        const int take = min(ke - kb, S - pre);  // <= S <= 8 stages: one flag word
        const uint32_t fl = flag_word(P, ta, 2 * kb);
        if (lane == 0) {
          tma_prefetch_desc(&g.tm_a[pr]);
          tma_prefetch_desc(&g.tm_a2[pr]);
          tma_prefetch_desc(&g.tm_a3[pr]);
          for (int i = 0; i < take; ++i) {
            const uint32_t kind = stage_kind(P, kb + i, i, fl);
            arm(pre + i, kind, 0, P.bn);
            load_a(pre + i, P, pr, ta, kb + i, kind);
          }
        }
        pre += take;
      }
    }
    if (wait_first) {
      pdl_wait();
      pdl_launch_dependents();
    }
    // 2. the main stream
    int stage = 0;
    uint32_t phase = 0;
    int n = 0;
    bool ok = true;
    SegIter<kMaxProb> it;
    it.init(g, unit, units);
    int pr, tile, kb, ke, seg;
    while (ok && it.next(g, units, pr, tile, kb, ke, seg)) {
      const GemmProblem& P = g.prob[pr];
      const int ta = tile % P.tiles_a, tb = tile / P.tiles_a;
      if (lane == 0) {
        tma_prefetch_desc(&g.tm_a[pr]);
        tma_prefetch_desc(&g.tm_a2[pr]);
        tma_prefetch_desc(&g.tm_a3[pr]);
        tma_prefetch_desc(&g.tm_b[pr]);
      }
      uint32_t fl = 0;
      for (int kt = kb; kt < ke; ++kt) {
        const int i = kt - kb;
        if ((i & 15) == 0) fl = flag_word(P, ta, 2 * kt);
        if (lane == 0) {
          if (n >= pre) {
            if (!mbar_wait(empty_bar(stage), phase ^ 1, p.timeout_ns, kDevErrWaitEmpty)) {
              ok = false;
              *abort_flag = 1;
            } else {
              const uint32_t kind = stage_kind(P, kt, i & 15, fl);
              arm(stage, kind, (int)phase, P.bn);
              load_a(stage, P, pr, ta, kt, kind);
            }
          }
          if (ok) {
            const uint32_t sb = smem_u32(smem + stage * C::kStageBytes) + C::kABytes;
#pragma unroll
            for (int bx = 0; bx < 2; ++bx)
              tma_load_2d(sb + bx * kBN * 128, &g.tm_b[pr], full_bar(stage), kt * 256 + bx * 128, tb * P.bn, pol_keep);
            ++n;
            if (++stage == S) {
              stage = 0;
              phase ^= 1;
            }
          }
        }
        ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
      }
    }
    // wait (bounded) until every copy counted on this CTA's barriers has landed
    if (lane == 0)
      for (int s = 0; s < S; ++s)
        if (armed[s] >= 0) mbar_wait(full_bar(s), (uint32_t)armed[s], p.timeout_ns, kDevErrWaitFull);
    __syncwarp();
  } else if (warp == 0) {
    // ------------------------------------------------------------------ producer
    if (lane != 0 && wait_first) {
      pdl_wait();
      pdl_launch_dependents();
    }
    if (lane == 0) {
      const uint64_t pol_stream = policy_evict_first();  // A: read once
      const uint64_t pol_keep = policy_evict_last();     // B: re-read by many CTAs
      int armed[S];
      for (int s = 0; s < S; ++s) armed[s] = -1;
      // the barrier a copy completes on (rank 0's in a pair)
      auto fbar = [&](int stage) { return kPair ? mapa_shared(full_bar(stage), 0) : full_bar(stage); };
      auto load2d = [&](uint32_t dst, const CUtensorMap* map, int stage, int32_t x, int32_t y, uint64_t pol) {
        if (kPair) tma_load_2d_pair_hint(dst, map, fbar(stage), x, y, pol);
        else tma_load_2d(dst, map, full_bar(stage), x, y, pol);
      };

      // the A-operand (and metadata) part of one stage
      auto load_a = [&](int stage, int pr, int ta, int kt) {
        const GemmProblem& P = g.prob[pr];
        const uint32_t sa = smem_u32(smem + stage * C::kStageBytes);
        const uint32_t sm = sa + C::kABytes + C::kBBytes;
        const int32_t ya = ta * C::kRowsA + (int32_t)rank * kBlockA;
        if (C::kNv) {
          // 128 bytes of A per row; metadata chunks (sparse) and the four
          // scale chunks of A's 128-row block at this stage's K
          load2d(sa, &g.tm_a[pr], stage, kt * 128, ya, pol_stream);
          const int nsf = nv_half(P, kt) ? 2 : 4;
          if (C::kNvSparse)
            bulk_load(sm, P.meta + ((int64_t)ta * (P.K / 256) + 2 * (int64_t)kt) * 2048, (uint32_t)(nsf / 2) * 2048,
                      full_bar(stage), pol_stream);
          bulk_load(sm + C::kMetaBytes, P.sfa + ((int64_t)ta * (P.K / C::kSfChunkK) + 4 * (int64_t)kt) * 512,
                    (uint32_t)nsf * 512, full_bar(stage), pol_stream);
        } else {
          const int ax = C::kSparse ? kt * (C::kKT / 2) : kt * C::kKT;  // elements
          load2d(sa, &g.tm_a[pr], stage, ax, ya, pol_stream);
          if (C::kSparse) {
            const int64_t kc_total = P.K / 128;
            if (kPair) {
              // metadata through the 2-D map over the image (8 rows of 256 B per
              // chunk); rows past the end take block 0 (their A rows are zero)
              int rb = ta * 2 + (int)rank;
              if (rb >= P.meta_blocks) rb = 0;
              load2d(sm, &g.tm_a2[pr], stage, 0, (int32_t)((rb * kc_total + (int64_t)kt * C::kMetaChunks) * 8),
                     pol_stream);
            } else {
              const uint8_t* src = P.meta + ((int64_t)ta * kc_total + (int64_t)kt * C::kMetaChunks) * 2048;
              bulk_load(sm, src, meta_chunks(P, kt) * 2048, full_bar(stage), pol_stream);
            }
          }
        }
      };
      auto load_b = [&](int stage, int pr, int tb, int kt) {
        const uint32_t sb = smem_u32(smem + stage * C::kStageBytes) + C::kABytes;
        const int32_t yb = tb * g.prob[pr].bn + (int32_t)rank * C::kBRows;
        if (C::kNv) {
          // kKT / 2 bytes of B per row, then the four scale chunks of the
          // 128-row block of B that holds this tile (tiles of fewer than 128
          // rows are the only tile of their operand: the host checks)
          const GemmProblem& P = g.prob[pr];
#pragma unroll
          for (int bx = 0; bx < C::kBBoxes; ++bx)
            load2d(sb + bx * C::kBRows * 128, &g.tm_b[pr], stage, kt * (C::kKT / 2) + bx * 128, yb, pol_keep);
          const int nsf = nv_half(P, kt) ? 2 : 4;
          bulk_load(sb + C::kBBytes + C::kMetaBytes + 2048,
                    P.sfb + ((int64_t)((tb * P.bn) >> 7) * (P.K / C::kSfChunkK) + 4 * (int64_t)kt) * 512,
                    (uint32_t)nsf * 512, full_bar(stage), pol_keep);
        } else {
          const int box_elems = kBf16 ? 64 : 128;
#pragma unroll
          for (int bx = 0; bx < C::kBBoxes; ++bx)
            load2d(sb + bx * C::kBRows * 128, &g.tm_b[pr], stage, kt * C::kKT + bx * box_elems, yb, pol_keep);
        }
      };
      // bytes that complete one stage (both CTAs' halves in a pair)
      auto stage_bytes = [&](int pr, int ta, int kt) -> uint32_t {
        const GemmProblem& P = g.prob[pr];
        if (kPair) return 2u * (uint32_t)C::kStageBytes;  // metadata boxes are always whole
        // the B boxes hold this problem's bn rows
        const uint32_t bbytes = (uint32_t)(P.bn * 128 * C::kBBoxes);
        if (C::kNv) {
          const uint32_t nsf = nv_half(P, kt) ? 2u : 4u;
          return (uint32_t)C::kABytes + bbytes + (C::kNvSparse ? nsf / 2 * 2048u : 0u) + 2u * nsf * 512u;
        }
        uint32_t b = (uint32_t)C::kABytes + bbytes;
        if (C::kSparse) b += (uint32_t)meta_chunks(P, kt) * 2048;
        return b;
      };
      auto arm = [&](int stage, uint32_t bytes, int ph) {
        if (rank == 0) {
          mbar_arrive_expect_tx(full_bar(stage), bytes);
          armed[stage] = ph;
        }
      };

      // 1. weights first: arm the first S stages and start their A loads
      //    before the dependency wait when A is known not to be in flux
      int pre = 0;
      int last_pr = -1;
      if (p.w_static) {
        SegIter<kMaxProb> it;
        it.init(g, unit, units);
        int pr, tile, kb, ke, seg;
        while (pre < S && it.next(g, units, pr, tile, kb, ke, seg)) {
          if (pr != last_pr) {
            tma_prefetch_desc(&g.tm_a[pr]);
            if (kPair && C::kSparse) tma_prefetch_desc(&g.tm_a2[pr]);
            last_pr = pr;
          }
          const int ta = tile % g.prob[pr].tiles_a;
          for (int kt = kb; kt < ke && pre < S; ++kt, ++pre) {
            arm(pre, stage_bytes(pr, ta, kt), 0);
            load_a(pre, pr, ta, kt);
          }
        }
      }
      if (wait_first) {
        pdl_wait();
        pdl_launch_dependents();
      }

      // 2. the main stream
      int stage = 0;
      uint32_t phase = 0;
      int n = 0;
      bool ok = true;
      last_pr = -1;
      SegIter<kMaxProb> it;
      it.init(g, unit, units);
      int pr, tile, kb, ke, seg;
      while (ok && it.next(g, units, pr, tile, kb, ke, seg)) {
        if (pr != last_pr) {
          tma_prefetch_desc(&g.tm_a[pr]);
          tma_prefetch_desc(&g.tm_b[pr]);
          if (kPair && C::kSparse) tma_prefetch_desc(&g.tm_a2[pr]);
          last_pr = pr;
        }
        const int ta = tile % g.prob[pr].tiles_a, tb = tile / g.prob[pr].tiles_a;
        for (int kt = kb; kt < ke; ++kt, ++n) {
          if (n < pre) {
            load_b(stage, pr, tb, kt);  // A already in flight
          } else {
            if (!mbar_wait(empty_bar(stage), phase ^ 1, p.timeout_ns, kDevErrWaitEmpty)) {
              ok = false;
              *abort_flag = 1;
              break;
            }
            arm(stage, stage_bytes(pr, ta, kt), (int)phase);
            load_a(stage, pr, ta, kt);
            load_b(stage, pr, tb, kt);
          }
          if (++stage == S) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // wait (bounded) until every copy counted on this CTA's barriers has landed
      for (int s = 0; s < S; ++s)
        if (armed[s] >= 0) mbar_wait(full_bar(s), (uint32_t)armed[s], p.timeout_ns, kDevErrWaitFull);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer (rank 0 in a pair)
    if (wait_first) {  // nothing to issue before the producer's dependent loads anyway
      pdl_wait();
      pdl_launch_dependents();
    }
    if (lane == 0 && rank == 0) {
      // instruction descriptors for the current problem's token-tile width
      uint32_t idesc = 0, idesc_dense = 0, idesc_sp = 0;
      int idesc_bn = -1;
      auto set_idesc = [&](int bn) {
        if (bn == idesc_bn) return;
        idesc_bn = bn;
        idesc = C::kNv ? make_idesc_nvf4(C::kNvSparse, kBlockA, (uint32_t)bn)
                       : make_idesc(C::kSparse, kBf16, C::kRowsA, (uint32_t)bn);
        idesc_dense = make_idesc(false, kBf16, kBlockA, (uint32_t)bn);
        idesc_sp = make_idesc(true, kBf16, C::kRowsA, (uint32_t)bn);
      };
      const uint32_t meta_col0 = C::kAccCols;
      const uint32_t s0 = smem_u32(smem);
      const uint64_t da0 = smem_desc(s0, 16, 1024, kLayoutSw128);
      const uint64_t db0 = smem_desc(s0 + C::kABytes, 16, 1024, kLayoutSw128);
      const uint64_t dm0 = smem_desc(s0 + C::kABytes + C::kBBytes, 16, 128, kLayoutNone);
      // both chunks of an e4m3 stage as one 128 x 256-bit copy: the second
      // chunk is the second core matrix along the row, 2048 bytes on
      const uint64_t dm2 = smem_desc(s0 + C::kABytes + C::kBBytes, 2048, 128, kLayoutNone);
      // NVFP4: the first scale chunk of A (B's follow 2048 bytes on), one
      // 32-row x 128-bit matrix of 16-byte rows
      const uint64_t dsf0 = smem_desc(s0 + C::kABytes + C::kBBytes + C::kMetaBytes, 16, 128, kLayoutNone);
      // hybrid: a sparse tile column's 64-byte rows of values (64-byte swizzle)
      const uint64_t dsp0 = smem_desc(s0, 16, 512, kLayoutSw64);
      int stage = 0;
      uint32_t phase = 0;
      uint32_t acc_i = 0;
      bool ok = true;
      SegIter<kMaxProb> it;
      it.init(g, unit, units);
      int pr, tile, kb, ke, seg;
      while (ok && it.next(g, units, pr, tile, kb, ke, seg)) {
        const GemmProblem& P = g.prob[pr];
        set_idesc(kPair ? kBN : P.bn);
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
          // NVFP4: the copy warp's commit for this stage completes after the
          // stage's data arrived and its copies into tensor memory are done
          if (!mbar_wait(C::kNv ? cpd_bar(stage) : full_bar(stage), phase, p.timeout_ns, kDevErrWaitFull)) {
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
            const uint32_t kind = s_kind[stage];
            const uint64_t so = (uint64_t)((uint32_t)stage * (uint32_t)(C::kStageBytes >> 4));
            uint32_t acc = first ? 0u : 1u;
            if (kind == 0) {
              // both columns sparse: the plain 2:4 e4m3 stage
              tc_cp_128x256b(tmem_base + mcol, dm2 + so);
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const uint64_t a_d = da0 + so + (uint64_t)(j * 2);
                const uint64_t b_d = db0 + so + (uint64_t)(((j >> 1) * kBN * 128 + (j & 1) * 64) >> 4);
                mma_sp_f8(d, a_d, b_d, tmem_base + mcol + 2 * j, idesc_sp, acc);
                acc = 1u;
              }
            } else {
#pragma unroll
              for (int c = 0; c < 2; ++c) {
                if (c == 1 && (kind & 4u)) break;
                const uint64_t slot = so + (uint64_t)(c * (16384 >> 4));       // A slot of column c
                const uint64_t bbox = db0 + so + (uint64_t)((c * kBN * 128) >> 4);  // B box of column c
                if ((kind >> c) & 1u) {
#pragma unroll
                  for (int j = 0; j < 4; ++j) {
                    mma_f8(d, da0 + slot + (uint64_t)(j * 2), bbox + (uint64_t)(j * 2), idesc_dense, acc);
                    acc = 1u;
                  }
                } else {
                  tc_cp_128x128b(tmem_base + mcol + 4 * c, dm0 + so + (uint64_t)(c * (2048 >> 4)));
#pragma unroll
                  for (int j = 0; j < 2; ++j) {
                    mma_sp_f8(d, dsp0 + slot + (uint64_t)(j * 2), bbox + (uint64_t)(j * 4),
                              tmem_base + mcol + 4 * c + 2 * j, idesc_sp, acc);
                    acc = 1u;
                  }
                }
              }
            }
          } else if (C::kNv) {
            const uint64_t so = (uint64_t)((uint32_t)stage * (uint32_t)(C::kStageBytes >> 4));
            const uint64_t da = da0 + so, db = db0 + so;
            const uint32_t scol = mcol + C::kMetaChunks * 4;  // A scales; B scales 16 columns on
            auto issue = [&](auto mmas_c) {
              constexpr int kMmas = decltype(mmas_c)::value;
#pragma unroll
              for (int j = 0; j < kMmas; ++j) {
                const uint32_t acc = (first && j == 0) ? 0u : 1u;
                const uint32_t sfa = tmem_base + scol + 4 * j, sfb = tmem_base + scol + 16 + 4 * j;
                if (C::kNvSparse) {
                  // 32 bytes of A (128 logical positions) and 64 bytes of B per MMA
                  const uint64_t a_d = da + (uint64_t)(j * 2);
                  const uint64_t b_d = db + (uint64_t)(((j >> 1) * C::kBRows * 128 + (j & 1) * 64) >> 4);
                  mma_sp_nvf4(d, a_d, b_d, tmem_base + mcol + 2 * j, idesc, sfa, sfb, acc);
                } else {
                  mma_nvf4(d, da + (uint64_t)(j * 2), db + (uint64_t)(j * 2), idesc, sfa, sfb, acc);
                }
              }
            };
            if (nv_half(P, kt)) issue(std::integral_constant<int, 2>{});
            else issue(std::integral_constant<int, 4>{});
          } else if (C::kSparse) {
            // descriptors of this stage: the stage-0 descriptors plus the
            // stage offset (the address field counts 16-byte units)
            const uint64_t so = (uint64_t)((uint32_t)stage * (uint32_t)(C::kStageBytes >> 4));
            const uint64_t da = da0 + so, db = db0 + so;
            auto issue = [&](auto chunks_c) {
              constexpr int kChunks = decltype(chunks_c)::value;
              if (kChunks == 2) {
                if (kPair) tc_cp_128x256b_pair(tmem_base + mcol, dm2 + so);
                else tc_cp_128x256b(tmem_base + mcol, dm2 + so);
              } else {
                if (kPair) tc_cp_128x128b_pair(tmem_base + mcol, dm0 + so);
                else tc_cp_128x128b(tmem_base + mcol, dm0 + so);
              }
              constexpr int kMmas = kBf16 ? 4 : 2 * kChunks;
#pragma unroll
              for (int j = 0; j < kMmas; ++j) {
                const uint64_t a_d = da + (uint64_t)(j * (32 >> 4));
                const uint64_t b_d = db + (uint64_t)(((j >> 1) * C::kBRows * 128 + (j & 1) * 64) >> 4);
                const uint32_t acc = (first && j == 0) ? 0u : 1u;
                if (kBf16) {
                  // one 32-bit metadata column per k-block; the selector picks
                  // the odd column of an even-aligned pair
                  const uint32_t col = mcol + j;
                  if (kPair) mma_sp_bf16_pair(d, a_d, b_d, tmem_base + (col & ~1u), idesc_sp | (col & 1u), acc);
                  else mma_sp_bf16(d, a_d, b_d, tmem_base + (col & ~1u), idesc_sp | (col & 1u), acc);
                } else {
                  // two metadata columns per k-block
                  const uint32_t col = mcol + 4 * (j >> 1) + 2 * (j & 1);
                  if (kPair) mma_sp_f8_pair(d, a_d, b_d, tmem_base + col, idesc_sp, acc);
                  else mma_sp_f8(d, a_d, b_d, tmem_base + col, idesc_sp, acc);
                }
              }
            };
            // a stage is whole except, for e4m3, a last stage of one 128-deep chunk
            if (kBf16 || C::kMetaChunks == 1 || meta_chunks(P, kt) == C::kMetaChunks)
              issue(std::integral_constant<int, C::kMetaChunks>{});
            else
              issue(std::integral_constant<int, 1>{});
          } else {
            const uint64_t so = (uint64_t)((uint32_t)stage * (uint32_t)(C::kStageBytes >> 4));
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const uint64_t da = da0 + so + (uint64_t)(j * (32 >> 4));
              const uint64_t db = db0 + so + (uint64_t)(j * (32 >> 4));
              const uint32_t acc = (first && j == 0) ? 0u : 1u;
              if (kPair) {
                if (kBf16) mma_bf16_pair(d, da, db, idesc, acc);
                else mma_f8_pair(d, da, db, idesc, acc);
              } else {
                if (kBf16) mma_bf16(d, da, db, idesc, acc);
                else mma_f8(d, da, db, idesc, acc);
              }
            }
          }
          // frees the stage (in both CTAs of a pair) once these MMAs are done
          if (kPair) tc_commit_pair(empty_bar(stage), 0x3);
          else tc_commit(empty_bar(stage));
          if (++stage == S) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        if (kPair) tc_commit_pair(accf_bar(buf), 0x3);
        else tc_commit(accf_bar(buf));
        ++acc_i;
      }
      // drain: every MMA and copy issued above has completed
      if (kPair) tc_commit_pair(drain_bar, 0x1);
      else tc_commit(drain_bar);
      mbar_wait(drain_bar, 0, p.timeout_ns, kDevErrWaitDrain);
    }
    __syncwarp();
  } else if (C::kNv && warp == 6) {
    // ------------------------------------------------------------------ tensor-memory copies (NVFP4)
    // For every stage, once its data arrived: the metadata chunk(s) (sparse)
    // and each MMA's A and B scale chunks into the stage's tensor-memory slot,
    // then a commit to the stage's copies-done barrier, which the MMA thread
    // waits on instead of the data barrier.  A slot is refilled only after the
    // producer re-armed its stage, i.e. after the MMAs that read the slot's
    // previous contents completed.
    if (wait_first) {
      pdl_wait();
      pdl_launch_dependents();
    }
    if (lane == 0) {
      const uint32_t s0 = smem_u32(smem);
      const uint64_t dm0 = smem_desc(s0 + C::kABytes + C::kBBytes, 16, 128, kLayoutNone);
      const uint64_t dm2 = smem_desc(s0 + C::kABytes + C::kBBytes, 2048, 128, kLayoutNone);
      const uint64_t dsf0 = smem_desc(s0 + C::kABytes + C::kBBytes + C::kMetaBytes, 16, 128, kLayoutNone);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      SegIter<kMaxProb> it;
      it.init(g, unit, units);
      int pr, tile, kb, ke, seg;
      while (ok && it.next(g, units, pr, tile, kb, ke, seg)) {
        const GemmProblem& P = g.prob[pr];
        for (int kt = kb; kt < ke; ++kt) {
          if (!mbar_wait(full_bar(stage), phase, p.timeout_ns, kDevErrWaitFull)) {
            ok = false;
            *abort_flag = 1;
            break;
          }
          tc_fence_after_sync();
          const uint64_t so = (uint64_t)((uint32_t)stage * (uint32_t)(C::kStageBytes >> 4));
          const uint32_t mcol = C::kAccCols + stage * C::kMetaCols;
          const uint32_t scol = mcol + C::kMetaChunks * 4;  // A scales; B scales 16 columns on
          const uint64_t dsf = dsf0 + so;
          auto issue = [&](auto mmas_c) {
            constexpr int kMmas = decltype(mmas_c)::value;
            if (C::kNvSparse) {
              if (kMmas == 4) tc_cp_128x256b(tmem_base + mcol, dm2 + so);
              else tc_cp_128x128b(tmem_base + mcol, dm0 + so);
            }
#pragma unroll
            for (int j = 0; j < kMmas; ++j) {
              tc_cp_32x128b_x4(tmem_base + scol + 4 * j, dsf + (uint64_t)(32 * j));
              tc_cp_32x128b_x4(tmem_base + scol + 16 + 4 * j, dsf + (uint64_t)(128 + 32 * j));
            }
          };
          if (nv_half(P, kt)) issue(std::integral_constant<int, 2>{});
          else issue(std::integral_constant<int, 4>{});
          tc_commit(cpd_bar(stage));
          if (++stage == S) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // drain: every copy issued above has completed
      tc_commit(cpdrain_bar);
      mbar_wait(cpdrain_bar, 0, p.timeout_ns, kDevErrWaitDrain);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ epilogue
    if (wait_first) {                          // B scales and Y may belong to the upstream grid
      pdl_wait();
      pdl_launch_dependents();
    }
    const int lg = warp & 3;                   // tensor-memory lane group of this warp
    const int row = lg * 32 + lane;            // accumulator row (lane) within the CTA's half
    const int et = threadIdx.x - 64;           // 0..127
    uint32_t acc_i = 0;
    int cached_pr = -1, cached_tb = -1;
    uint8_t* wtile = s_epi + (warp - 2) * 2048;  // this warp's staging tile
    // values read once into registers: the tcgen05 and barrier asm statements
    // below clobber memory, which would otherwise force the parameter-struct
    // fields to be re-read after each of them
    const bool out_f32 = p.out_f32 != 0;
    float* const sk_slots = p.sk_slots;
    unsigned int* const sk_flags = p.sk_flags;
    SegIter<kMaxProb> it;
    it.init(g, unit, units);
    int pr, tile, kb, ke, seg;
    while (it.next(g, units, pr, tile, kb, ke, seg)) {
      const GemmProblem& P = g.prob[pr];
      const int ta = tile % P.tiles_a, tb = tile / P.tiles_a;
      const int bn = kPair ? kBN : P.bn;   // token-tile width of this problem
      const int buf = acc_i & 1;
      const uint32_t acc_phase = (acc_i >> 1) & 1;
      const int ga = ta * C::kRowsA + (int)rank * kBlockA + row;  // global A row of this thread
      const int rows_a = P.rows_a, rows_b = P.rows_b;
      uint8_t* const Yb = static_cast<uint8_t*>(P.Y);
      const int64_t ldy = P.ldy;
      const bool a_live = ga < rows_a;
      // scales: loaded before waiting for the accumulator so their latency hides
      const float sa_v = P.scale_a == nullptr ? 1.0f : C::kNv ? __ldg(P.scale_a) : a_live ? __ldg(P.scale_a + ga) : 1.0f;
      if (pr != cached_pr || tb != cached_tb) {
        named_bar_sync(1, 128);
        for (int i = et; i < bn; i += 128) {
          const int gb = tb * bn + i;
          s_scale_b[i] = P.scale_b == nullptr ? 1.0f : C::kNv ? P.scale_b[0] : gb < rows_b ? P.scale_b[gb] : 1.0f;
        }
        named_bar_sync(1, 128);
        cached_pr = pr;
        cached_tb = tb;
      }
      const bool full = (kb == 0 && ke == P.num_kt);
      // A split tile is finished by the unit that holds its first K-stage:
      // that unit's range ends inside the tile, so the tile is its last
      // segment, and every other contributor's segment of it lies at the
      // start of (or spans) that contributor's range.  The finisher waits
      // (bounded) for the others' partials before its own accumulator, so
      // the wait overlaps its last MMAs.
      const bool finisher = !full && kb == 0;
      int64_t i0 = 0;
      int c_first = 0, c_last = 0;
      if (!full) {
        i0 = P.iter_begin + (int64_t)tile * P.num_kt;
        c_first = sk_owner(p, units, i0);
        c_last = sk_owner(p, units, i0 + P.num_kt - 1);
      }
      // the partial slot of unit u (one per unit: a unit stores at most one
      // partial, for its first segment)
      auto slot_idx = [&](int u) { return (int64_t)u * (kPair ? 2 : 1) + (int64_t)rank; };
      // a unit with an empty range (possible when the ranges are cut by
      // cost) contributes nothing
      auto live = [&](int u) { return p.sk_bound[u] < p.sk_bound[u + 1]; };
      if (finisher && et == 0) {
        bool ok2 = true;
        for (int v = c_first + 1; v <= c_last && ok2; ++v) {
          if (!live(v)) continue;
          const unsigned int* f = sk_flags + slot_idx(v);
          if (ld_acquire_gpu(f) == 0u) {
            const uint64_t t0 = globaltimer_ns();
            while (ld_acquire_gpu(f) == 0u) {
              if (globaltimer_ns() - t0 > p.timeout_ns) {
                record_dev_error(kDevErrWaitCounter);
                ok2 = false;
                break;
              }
            }
          }
        }
        *last_flag = ok2 ? 1 : 2;
      }
      bool ok = mbar_wait(accf_bar(buf), acc_phase, p.timeout_ns, kDevErrWaitAccFull);
      __syncwarp();
      ok = named_bar_red_and(2, 128, ok);  // all epilogue threads agree (and see last_flag)
      if (!ok) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after_sync();
      const uint32_t tbase = tmem_base + ((uint32_t)(lg * 32) << 16) + buf * kBN;

      // Scales and stores 16 consecutive accumulator columns starting at c0
      // with 16-byte vector stores.  Rows of Y are 16-byte aligned (checked
      // on the host); a vector that crosses the end of a row is stored per
      // element.  EB (output bytes) is a compile-time constant so that the
      // index arithmetic is shifts and masks: this code runs on one warp per
      // sub-partition, where every dependent instruction shows in the time.
      auto store16 = [&](auto eb_c, const float (&v)[16], int c0) {
        constexpr int EB = decltype(eb_c)::value;
        constexpr int PV = 16 / EB;   // elements per 16-byte vector
        const int gb0 = tb * bn + c0;
        float sc[16];
#pragma unroll
        for (int i = 0; i < 16; i += 4) {
          const float4 t = *reinterpret_cast<const float4*>(s_scale_b + c0 + i);
          sc[i] = t.x * sa_v; sc[i + 1] = t.y * sa_v; sc[i + 2] = t.z * sa_v; sc[i + 3] = t.w * sa_v;
        }
        if (kAIsW) {
          // lane = n (output feature), column = m (token).  Stage the warp's
          // 32 n x 16 m block transposed, then write each output row's 32
          // consecutive n as 16-byte vectors.
          constexpr int VPR = 32 / PV;  // vectors per row of 32 n
          const int n0 = ta * C::kRowsA + (int)rank * kBlockA + lg * 32;
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
          // lane = m (token), column = n (output feature): this thread's 16
          // consecutive n of row ga
          if (!a_live) return;
          constexpr int NW = 16 * EB / 4;  // 32-bit words of output
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
              // whole 32-bit words inside the row (for bf16 a word holds two
              // outputs; a row of odd length ends in a half word)
              const int e0 = j * 4 / EB;  // first output of word j
              if (e0 >= rows_b - gb0) break;
              if (EB == 4 || e0 + 1 < rows_b - gb0) {
                reinterpret_cast<uint32_t*>(dst)[j] = w[j];
              } else {
                reinterpret_cast<uint16_t*>(dst)[2 * j] = (uint16_t)(w[j] & 0xFFFFu);
              }
            }
          }
        }
      };
      auto store16_any = [&](const float (&v)[16], int c0) {
        if (out_f32) store16(std::integral_constant<int, 4>{}, v, c0);
        else store16(std::integral_constant<int, 2>{}, v, c0);
      };

      // the accumulator may be overwritten now (one arrive per warp; rank
      // 0's barrier in a pair)
      auto release_acc = [&]() {
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) {
          if (kPair) mbar_arrive_cluster(mapa_shared(acce_bar(buf), 0));
          else mbar_arrive(acce_bar(buf));
        }
      };

      if (full) {
#pragma unroll 1
        for (int c0 = 0; c0 < bn; c0 += 16) {
          uint32_t r[16];
          tmem_ld_x16(tbase + c0, r);
          tmem_ld_wait();
          float v[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
          store16_any(v, c0);
        }
        release_acc();
      } else if (!finisher) {
        // store the partial tile (plain stores), then raise the flag
        // slot layout: float4 (col / 4) of row r at index (col / 4) * 128 + r,
        // so each warp store covers 512 contiguous bytes
        const int64_t my = slot_idx(unit);
        float4* dst = reinterpret_cast<float4*>(sk_slots + my * 128 * kBN) + row;
#pragma unroll 1
        for (int c0 = 0; c0 < bn; c0 += 16) {
          uint32_t r[16];
          tmem_ld_x16(tbase + c0, r);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 4; ++j)
            __stcg(dst + (c0 / 4 + j) * 128,
                   make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                               __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3])));
        }
        release_acc();
        named_bar_sync(1, 128);  // every store of the tile precedes the flag
        if (et == 0) {
          __threadfence();
          st_release_gpu(sk_flags + my, 1u);
        }
      } else {
        // the finisher: our accumulator plus the others' partials, 64
        // columns at a time
        const bool have = *last_flag == 1;
        constexpr int kFix = kBN < 64 ? kBN : 64;
#pragma unroll 1
        for (int cb = 0; cb < bn; cb += kFix) {
          float4 q[kFix / 4];
#pragma unroll
          for (int j = 0; j < kFix / 4; ++j) q[j] = make_float4(0.f, 0.f, 0.f, 0.f);
          if (have) {
            for (int v = c_first + 1; v <= c_last; ++v) {
              if (!live(v)) continue;
              const float4* src = reinterpret_cast<const float4*>(sk_slots + slot_idx(v) * 128 * kBN) + row;
              float4 t[kFix / 4];
#pragma unroll
              for (int j = 0; j < kFix / 4; ++j) t[j] = __ldcg(src + (cb / 4 + j) * 128);
#pragma unroll
              for (int j = 0; j < kFix / 4; ++j) {
                q[j].x += t[j].x; q[j].y += t[j].y; q[j].z += t[j].z; q[j].w += t[j].w;
              }
            }
          }
#pragma unroll
          for (int c0 = 0; c0 < kFix; c0 += 16) {
            if (cb + c0 >= bn) break;  // a problem narrower than the kernel's tile
            uint32_t r[16];
            tmem_ld_x16(tbase + cb + c0, r);
            tmem_ld_wait();
            float v[16];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const float4 t = q[c0 / 4 + j];
              v[4 * j] = __uint_as_float(r[4 * j]) + t.x;
              v[4 * j + 1] = __uint_as_float(r[4 * j + 1]) + t.y;
              v[4 * j + 2] = __uint_as_float(r[4 * j + 2]) + t.z;
              v[4 * j + 3] = __uint_as_float(r[4 * j + 3]) + t.w;
            }
            store16_any(v, cb + c0);
          }
        }
        release_acc();
        named_bar_sync(1, 128);  // every read of the partials precedes the reset
        if (et == 0)  // ready for the next call
          for (int v = c_first + 1; v <= c_last; ++v)
            if (live(v)) sk_flags[slot_idx(v)] = 0u;
        if (!have) *abort_flag = 1;
      }
      ++acc_i;
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  // after an independent GEMM: complete only once it has (stream order of
  // completion for whatever follows)
  if (p.use_pdl && p.after_independent) pdl_wait();
  if (kPair) cluster_sync();  // neither CTA leaves while its peer may still use its memory
  if (warp == 1) {
    tc_fence_after_sync();
    if (kPair) tmem_dealloc_pair(tmem_base, C::kTmemCols);
    else tmem_dealloc(tmem_base, C::kTmemCols);
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
