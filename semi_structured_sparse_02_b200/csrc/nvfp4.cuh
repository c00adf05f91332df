// nvfp4.cuh -- NVFP4 operands of the block-scaled tcgen05 MMA
// (kind::mxf4nvf4): the pairwise 4:8 sparse operand (prune + cast) and the
// dense NVFP4 operand (cast), written straight in the layouts the GEMM copies
// to shared and tensor memory.
//
// Format: E2M1 values (two per byte, the earlier element in the low nibble),
// one unsigned E4M3 scale per block of positions along K, one fp32 scale per
// tensor ("Quantization", section 2 of the 2:4-versus-quantization paper,
// paperpeel.com/paper/2610.28947).  The sparse operand keeps, in every group
// of eight along K, two of the four adjacent pairs, and carries one scale per
// 32 positions of K (section 6.2, "What pairwise 4:8 costs on Blackwell").
// Readings where the pages are silent (the same ones the oracle follows):
//   pairs: the two pairs of largest energy x0^2 + x1^2 (fp64, exact from
//          bf16) survive, ties to the lower pair index;
//   scales: s_t = amax_t / (448 * 6) (1 if amax_t = 0); block code
//          b = E4M3(amax_b / (6 * s_t)); code = E2M1(v / (decode(b) * s_t)),
//          each step one correctly rounded fp32 operation, E2M1 rounding to
//          nearest even and saturating at 6; a zero block scale gives code 0;
//   the amaxes of the sparse operand run over the kept values.
//
// Layouts:
//   values (sparse)  [rows x K/4] bytes: the kept elements in ascending position
//   codes (dense)    [rows x K/2] bytes
//   metadata image (sparse): 2048-byte chunks, one per (128-row block rb,
//          256 positions of K kc) at (rb * K/256 + kc) * 2048; image row L
//          (16 bytes at 16 L) holds row 128 rb + L's 32 group nibbles
//          p0 | p1 << 2 in order, the even group in the low nibble; rows past
//          the end hold 0x4 (pairs 0 and 1)
//   scale image: 512-byte chunks, one per (128-row block rb, four consecutive
//          scale blocks kq) at (rb * nblk/4 + kq) * 512; the code of row
//          r = 128 rb + 32 q + l, block 4 kq + j sits at byte 16 l + 4 q + j
//          (the order in which one tcgen05.cp.32x128b.warpx4 lands a chunk in
//          tensor memory for the MMA); rows past the end hold 0
//   tensor scale: one fp32 (during a call it first holds the amax bits).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "sp24_device.cuh"
#include "prune.cuh"

namespace sp24 {

constexpr int kNvThreads = 256;

// Byte offset of the scale code of (row r, block blk) in a scale image with
// nblk blocks per row (nblk % 4 == 0).
__host__ __device__ __forceinline__ int64_t sf_image_offset(int64_t r, int64_t blk, int64_t nblk) {
  const int64_t rb = r >> 7, rr = r & 127, kq = blk >> 2, j = blk & 3;
  return (rb * (nblk >> 2) + kq) * 512 + 16 * (rr & 31) + 4 * (rr >> 5) + j;
}

// Value of an E4M3 code with sign 0 (exact in fp32), from the format: bias 7,
// three mantissa bits, subnormal step 2^-9.
__device__ __forceinline__ float ue4m3_value(uint32_t c) {
  const uint32_t e = (c >> 3) & 15u, m = c & 7u;
  return e == 0 ? (float)m * 0x1p-9f : __uint_as_float(((e + 120u) << 23) | (m << 20));
}

// Eight fp32 values to eight E2M1 codes (round to nearest even, saturating),
// element i in nibble i.
__device__ __forceinline__ uint32_t e2m1x8(const float (&v)[8]) {
  uint32_t out;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(out)
      : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
  return out;
}

// The pair rule on one group of eight bf16 values (bit patterns): pair j
// (elements 2j, 2j+1) survives iff fewer than two pairs beat it, where i
// beats j when e_i > e_j or e_i == e_j and i < j.  Returns p0 | p1 << 2 and
// the four kept values in ascending position (by selects).
__device__ __forceinline__ uint32_t pick_pairs8(const uint32_t (&x)[8], uint32_t (&kept)[4]) {
  double e[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const double a = (double)bf16_bits_to_float(x[2 * j]), b = (double)bf16_bits_to_float(x[2 * j + 1]);
    e[j] = __dadd_rn(__dmul_rn(a, a), __dmul_rn(b, b));
  }
  const int l0 = (e[1] > e[0]) + (e[2] > e[0]) + (e[3] > e[0]);
  const int l1 = (e[0] >= e[1]) + (e[2] > e[1]) + (e[3] > e[1]);
  const int l2 = (e[0] >= e[2]) + (e[1] >= e[2]) + (e[3] > e[2]);
  const int l3 = (e[0] >= e[3]) + (e[1] >= e[3]) + (e[2] >= e[3]);
  const bool k0 = l0 < 2, k1 = l1 < 2, k2 = l2 < 2, k3 = l3 < 2;
  const uint32_t p0 = k0 ? 0u : (k1 ? 1u : 2u);
  const uint32_t p1 = k3 ? 3u : (k2 ? 2u : 1u);
  kept[0] = k0 ? x[0] : (k1 ? x[2] : x[4]);
  kept[1] = k0 ? x[1] : (k1 ? x[3] : x[5]);
  kept[2] = k3 ? x[6] : (k2 ? x[4] : x[2]);
  kept[3] = k3 ? x[7] : (k2 ? x[5] : x[3]);
  return p0 | (p1 << 2);
}

__device__ __forceinline__ void unpack8(const uint4 v, uint32_t (&x)[8]) {
  x[0] = v.x & 0xFFFFu; x[1] = v.x >> 16; x[2] = v.y & 0xFFFFu; x[3] = v.y >> 16;
  x[4] = v.z & 0xFFFFu; x[5] = v.z >> 16; x[6] = v.w & 0xFFFFu; x[7] = v.w >> 16;
}

// The tensor scale from the tensor amax (1 for amax 0).
__device__ __forceinline__ float nvfp4_tensor_scale(float amax) {
  return amax == 0.0f ? 1.0f : __fdiv_rn(amax, 2688.0f);
}

// Block code and effective scale S = decode(b) * s_t of one block.
__device__ __forceinline__ uint32_t nvfp4_block(float amax_b, float six_st, float s_t, float& S) {
  const uint32_t b = (uint32_t)e4m3_of(__fdiv_rn(amax_b, six_st));
  S = __fmul_rn(ue4m3_value(b), s_t);
  return b;
}

// Eight values to E2M1 codes under the effective scale S (code 0 if S == 0).
__device__ __forceinline__ uint32_t nvfp4_codes8(const float (&v)[8], float S) {
  if (S == 0.0f) return 0u;
  float q[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) q[i] = __fdiv_rn(v[i], S);
  return e2m1x8(q);
}

__device__ __forceinline__ void atomic_max_nonneg(unsigned int* p, float v) {
  atomicMax(p, __float_as_uint(v));  // non-negative floats order as their bits
}

// ---------------------------------------------------------------------------
// Tensor amax.  kKept: over the values the pair rule keeps (sparse operand);
// otherwise over every value.  One 16-byte load is one group of eight.
// ---------------------------------------------------------------------------
template <bool kKept>
__global__ void __launch_bounds__(kNvThreads)
k_nvfp4_amax(const uint16_t* __restrict__ src, int64_t rows, int64_t K, int64_t ld,
             unsigned int* __restrict__ amax_bits) {
  pdl_launch_dependents();
  pdl_wait();
  const int64_t gpr = K / 8;  // groups per row
  const int64_t total = rows * gpr;
  float m = 0.0f;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / gpr, g = i - r * gpr;
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(src + r * ld + g * 8));
    uint32_t x[8];
    unpack8(v, x);
    if (kKept) {
      uint32_t kept[4];
      pick_pairs8(x, kept);
#pragma unroll
      for (int j = 0; j < 4; ++j) m = fmaxf(m, fabsf(bf16_bits_to_float(kept[j])));
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) m = fmaxf(m, fabsf(bf16_bits_to_float(x[j])));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  if ((threadIdx.x & 31) == 0 && m > 0.0f) atomic_max_nonneg(amax_bits, m);
}

// amax bits -> tensor scale, in place.
__global__ void k_nvfp4_finalize(float* __restrict__ ts) {
  pdl_launch_dependents();
  pdl_wait();
  if (threadIdx.x == 0) ts[0] = nvfp4_tensor_scale(ts[0]);
}

// ---------------------------------------------------------------------------
// Sparse operand: prune (pairwise 4:8) + cast.  Grid-stride over chunks of
// 128 rows x 256 positions of K (one metadata chunk, two scale chunks);
// thread t takes row t / 2 and half t % 2 of the chunk: four scale blocks of
// 32 positions (four groups of eight each).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kNvThreads)
k_nvfp4_48_compress(const uint16_t* __restrict__ src, int64_t rows, int64_t K, int64_t ld,
                    uint8_t* __restrict__ values, uint8_t* __restrict__ meta, uint8_t* __restrict__ sf,
                    const unsigned int* __restrict__ amax_bits) {
  pdl_launch_dependents();
  pdl_wait();
  const float s_t = nvfp4_tensor_scale(__uint_as_float(*amax_bits));
  const float six_st = __fmul_rn(6.0f, s_t);
  const int64_t KC = K / 256;
  const int64_t RB = (rows + 127) / 128;
  const int64_t nblk = K / 32;
  const int rl = threadIdx.x >> 1, h = threadIdx.x & 1;
  for (int64_t c = blockIdx.x; c < RB * KC; c += gridDim.x) {
    const int64_t rb = c / KC, kc = c - rb * KC;
    const int64_t r = rb * 128 + rl;
    uint32_t nib_lo = 0x44444444u, nib_hi = 0x44444444u;  // rows past the end: pairs 0 and 1
    uint32_t sfw = 0;
    if (r < rows) {
      const uint4* p = reinterpret_cast<const uint4*>(src + r * ld + kc * 256 + h * 128);
      uint8_t* vrow = values + r * (K / 4) + kc * 64 + h * 32;
#pragma unroll 1
      for (int blk = 0; blk < 4; ++blk) {
        uint4 v[4];
#pragma unroll
        for (int gi = 0; gi < 4; ++gi) v[gi] = __ldg(p + blk * 4 + gi);
        float kept[16];
        uint32_t nibs = 0;
        float amax_b = 0.0f;
#pragma unroll
        for (int gi = 0; gi < 4; ++gi) {
          uint32_t x[8], k4[4];
          unpack8(v[gi], x);
          nibs |= pick_pairs8(x, k4) << (4 * gi);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            kept[4 * gi + j] = bf16_bits_to_float(k4[j]);
            amax_b = fmaxf(amax_b, fabsf(kept[4 * gi + j]));
          }
        }
        float S;
        const uint32_t b = nvfp4_block(amax_b, six_st, s_t, S);
        sfw |= b << (8 * blk);
        float lo[8], hi[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          lo[i] = kept[i];
          hi[i] = kept[8 + i];
        }
        *reinterpret_cast<uint2*>(vrow + blk * 8) = make_uint2(nvfp4_codes8(lo, S), nvfp4_codes8(hi, S));
        if (blk < 2) nib_lo = (blk == 0 ? (nib_lo & 0xFFFF0000u) | nibs : (nib_lo & 0x0000FFFFu) | (nibs << 16));
        else nib_hi = (blk == 2 ? (nib_hi & 0xFFFF0000u) | nibs : (nib_hi & 0x0000FFFFu) | (nibs << 16));
      }
    }
    *reinterpret_cast<uint2*>(meta + c * 2048 + rl * 16 + h * 8) = make_uint2(nib_lo, nib_hi);
    *reinterpret_cast<uint32_t*>(sf + (rb * (nblk / 4) + kc * 2 + h) * 512 + 16 * (rl & 31) + 4 * (rl >> 5)) = sfw;
  }
}

// ---------------------------------------------------------------------------
// Dense operand: cast with one scale per `block` (16 or 32) positions.  One
// thread per (row, four consecutive blocks): one 32-bit word of the scale
// image and 2 * block bytes of codes.  Rows from `rows` to the end of the last
// 128-row block only get zero scale words.
// ---------------------------------------------------------------------------
template <int kBlock>
__global__ void __launch_bounds__(kNvThreads)
k_nvfp4_quantize(const uint16_t* __restrict__ src, int64_t rows, int64_t K, int64_t ld,
                 uint8_t* __restrict__ codes, uint8_t* __restrict__ sf,
                 const unsigned int* __restrict__ amax_bits) {
  pdl_launch_dependents();
  pdl_wait();
  const float s_t = nvfp4_tensor_scale(__uint_as_float(*amax_bits));
  const float six_st = __fmul_rn(6.0f, s_t);
  const int64_t nblk = K / kBlock;
  const int64_t KQ = nblk / 4;
  const int64_t rows_pad = (rows + 127) / 128 * 128;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < rows_pad * KQ;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / KQ, kq = i - r * KQ;
    uint32_t sfw = 0;
    if (r < rows) {
      const uint4* p = reinterpret_cast<const uint4*>(src + r * ld + kq * 4 * kBlock);
      uint8_t* crow = codes + r * (K / 2) + kq * 2 * kBlock;
#pragma unroll 1
      for (int blk = 0; blk < 4; ++blk) {
        constexpr int kV = kBlock / 8;  // 16-byte loads per block
        uint4 raw[kV];
        uint32_t mb = 0;  // largest magnitude bits (the bf16 of the block amax)
#pragma unroll
        for (int q = 0; q < kV; ++q) {
          raw[q] = __ldg(p + blk * kV + q);
          mb = max(mb, amax_bits8(raw[q]));
        }
        float S;
        sfw |= nvfp4_block(bf16_bits_to_float(mb), six_st, s_t, S) << (8 * blk);
        uint32_t w[kV];
#pragma unroll
        for (int q = 0; q < kV; ++q) {
          uint32_t x[8];
          unpack8(raw[q], x);
          float e[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) e[j] = bf16_bits_to_float(x[j]);
          w[q] = nvfp4_codes8(e, S);
        }
        if (kV == 2) *reinterpret_cast<uint2*>(crow + blk * 8) = make_uint2(w[0], w[kV - 1]);
        else *reinterpret_cast<uint4*>(crow + blk * 16) = make_uint4(w[0], w[1 % kV], w[2 % kV], w[3 % kV]);
      }
    }
    const int64_t rr = r & 127;
    *reinterpret_cast<uint32_t*>(sf + ((r >> 7) * KQ + kq) * 512 + 16 * (rr & 31) + 4 * (rr >> 5)) = sfw;
  }
}

}  // namespace sp24
