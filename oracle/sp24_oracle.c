/*
 * sp24_oracle.c -- CPU oracle for 2:4 semi-structured sparsity (and, at the
 * end, the pairwise 4:8 sparse NVFP4 format that comes next).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load this file's library.  The CUDA
 * library never links, includes or calls it, and it never calls the CUDA
 * library: the two share no code, header, table or constant generator.
 *
 * Everything here is written to be checked by eye against the pages it
 * restates, so it is slow on purpose: plain loops, fp64 accumulation, no
 * blocking and no reordering beyond the definitions.
 *
 * Sources (page title, then section):
 *  [P1] "Production 2:4 Structured Sparsity for LLMs" (oh-bug.com),
 *       "Core Mechanisms and Production States of 2:4 Structured Sparsity",
 *       "Sparse Tactic Audit", "Dense Fallback and Hybrid Sparsity Design".
 *  [P3] "2:4 Structured Sparsity Explained" (tensorcore.si),
 *       "How 2:4 sparsity works" (format and storage table),
 *       "How to make a model 2:4 sparse" (keep the two largest magnitudes).
 *  [P4] the 2:4-versus-quantization paper (paperpeel.com/paper/2610.28947),
 *       section 2 "Sparse tensor cores" (compressed operand A, 2-bit index per
 *       kept value, groups along the reduction axis) and "Quantization"
 *       (FP8 E4M3 with one scale per row or channel), section 5.1 (magnitude
 *       pruning and round-to-nearest are the basic methods).
 *  [EXT] OCP 8-bit floating point specification, E4M3 encoding (bias 7,
 *       three mantissa bits, no infinities, largest finite 448).
 *
 * Readings where the pages are silent (each one is listed in the design notes):
 *  R1 ties between equal magnitudes go to the lower index;
 *  R2 a group always keeps exactly two positions, even when it holds fewer
 *     than two non-zeros (a kept zero is stored as zero);
 *  R3 metadata nibble of a group = i0 | (i1 << 2) with i0 < i1; the canonical
 *     byte order is row-major, two groups per byte, even group in the low
 *     nibble;
 *  R4 E4M3 scale = amax / 448 and inverse = 448 / amax, each a correctly
 *     rounded fp32 division; q = E4M3(round-to-nearest-even, saturating)
 *     of the fp32 product v * inverse; amax == 0 gives scale 1 and q = 0;
 *  R5 prune on bf16 magnitudes first, then quantize the kept values.
 *
 * Parity pins live in tests/test_oracle_pins.py.  The metadata image
 * permutation (orc_meta_image) is pinned only by its bijectivity and by
 * hand-derived positions from its written layout, and finally by the GPU
 * GEMM, which reads it through the tensor cores: it says "parity pinned by
 * layout spec" rather than by a page.
 */
#include <stdint.h>
#include <stddef.h>
#include <string.h>
#include <math.h>

/* ------------------------------------------------------------------ */
/* bf16 helpers                                                         */
/* ------------------------------------------------------------------ */

/* Exact value of a bf16 bit pattern (bf16 is the top half of an fp32). */
double orc_bf16_to_double(uint16_t b)
{
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static float bf16_to_float(uint16_t b)
{
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* Magnitude key: the bf16 bits without the sign.  For finite values the
 * integer order of these keys is the order of |v| (IEEE sign-magnitude),
 * and +0 / -0 compare equal. */
static int mag_key(uint16_t b) { return (int)(b & 0x7FFFu); }

/* ------------------------------------------------------------------ */
/* 1. Magnitude 2:4 prune of one group of four  [P3 "How to make a     */
/*    model 2:4 sparse"; P1 worked example]                             */
/* ------------------------------------------------------------------ */

/* Position i survives iff fewer than two other positions beat it, where j
 * beats i when |v_j| > |v_i|, or |v_j| == |v_i| and j < i (reading R1).
 * Exactly two positions survive for any input (reading R2).
 * Returns the metadata nibble i0 | (i1 << 2) and the two kept indices. */
int orc_prune_group(const uint16_t v[4], int *i0, int *i1)
{
    int kept[2];
    int nk = 0;
    for (int i = 0; i < 4; ++i) {
        int beaten_by = 0;
        for (int j = 0; j < 4; ++j) {
            if (j == i) continue;
            if (mag_key(v[j]) > mag_key(v[i])) beaten_by++;
            else if (mag_key(v[j]) == mag_key(v[i]) && j < i) beaten_by++;
        }
        if (beaten_by < 2) kept[nk++] = i;   /* i ascends, so kept[0] < kept[1] */
    }
    /* nk == 2 always: the "beats" relation is a strict total order. */
    *i0 = kept[0];
    *i1 = kept[1];
    return kept[0] | (kept[1] << 2);
}

/* ------------------------------------------------------------------ */
/* 2. Prune + compress whole rows (bf16 values)  [P3 "How 2:4 sparsity */
/*    works": half-size value array + 2-bit index per kept value]       */
/* ------------------------------------------------------------------ */

/* src: [rows x K] bf16 bits, row stride ld elements.  K % 4 == 0.
 * pruned:     [rows x K]   bf16 bits, the zeroed dense matrix (may be NULL)
 * values:     [rows x K/2] bf16 bits, kept values in ascending index order
 * meta_canon: [rows x K/8] bytes, canonical nibbles (reading R3)          */
void orc_prune_compress_bf16(const uint16_t *src, int64_t rows, int64_t K, int64_t ld,
                             uint16_t *pruned, uint16_t *values, uint8_t *meta_canon)
{
    if (rows <= 0 || K <= 0) return;
    for (int64_t r = 0; r < rows; ++r) {
        if (meta_canon) memset(meta_canon + r * (K / 8), 0, (size_t)(K / 8));
        for (int64_t g = 0; g < K / 4; ++g) {
            const uint16_t *v = src + r * ld + 4 * g;
            int i0, i1;
            int nib = orc_prune_group(v, &i0, &i1);
            if (values) {
                values[r * (K / 2) + 2 * g + 0] = v[i0];
                values[r * (K / 2) + 2 * g + 1] = v[i1];
            }
            if (pruned) {
                for (int i = 0; i < 4; ++i)
                    pruned[r * K + 4 * g + i] = (i == i0 || i == i1) ? v[i] : (uint16_t)0;
            }
            if (meta_canon) {
                uint8_t *byte = meta_canon + r * (K / 8) + g / 2;
                *byte |= (uint8_t)(nib << ((g % 2) * 4));
            }
        }
    }
}

/* ------------------------------------------------------------------ */
/* 3. Decompress: scatter kept values back into zeros  [P3 "How 2:4    */
/*    sparsity works"]                                                  */
/* ------------------------------------------------------------------ */

/* Element-size agnostic: elem_bytes is 2 (bf16) or 1 (e4m3 codes). */
void orc_decompress(const void *values, const uint8_t *meta_canon, int64_t rows, int64_t K,
                    int elem_bytes, void *dst)
{
    const uint8_t *vb = (const uint8_t *)values;
    uint8_t *db = (uint8_t *)dst;
    memset(dst, 0, (size_t)(rows * K * elem_bytes));
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t g = 0; g < K / 4; ++g) {
            int nib = (meta_canon[r * (K / 8) + g / 2] >> ((g % 2) * 4)) & 0xF;
            int i0 = nib & 3, i1 = (nib >> 2) & 3;
            memcpy(db + (r * K + 4 * g + i0) * elem_bytes,
                   vb + (r * (K / 2) + 2 * g + 0) * elem_bytes, (size_t)elem_bytes);
            memcpy(db + (r * K + 4 * g + i1) * elem_bytes,
                   vb + (r * (K / 2) + 2 * g + 1) * elem_bytes, (size_t)elem_bytes);
        }
    }
}

/* ------------------------------------------------------------------ */
/* 4. FP8 E4M3  [P4 "Quantization"; EXT: OCP FP8 spec]                  */
/* ------------------------------------------------------------------ */

/* Value of an E4M3 code: sign, 4-bit exponent (bias 7), 3-bit mantissa;
 * exponent field 0 is subnormal (m * 2^-9); S.1111.111 is NaN; there are no
 * infinities. */
double orc_e4m3_decode(uint8_t q)
{
    int s = (q >> 7) & 1;
    int e = (q >> 3) & 0xF;
    int m = q & 7;
    double mag;
    if (e == 0xF && m == 7) return NAN;
    if (e == 0) mag = ldexp((double)m, -9);
    else        mag = ldexp(1.0 + m / 8.0, e - 7);
    return s ? -mag : mag;
}

/* Round-to-nearest-even to E4M3 with saturation to +-448 (reading R4).
 * x is an fp32 value carried exactly in a double. */
uint8_t orc_e4m3_encode(double x)
{
    uint8_t sign = (x < 0.0 || (x == 0.0 && signbit(x))) ? 0x80 : 0x00;
    double a = fabs(x);
    if (a >= 448.0) return (uint8_t)(sign | 0x7E);        /* largest finite */
    /* quantum (spacing of representable values) of the binade holding a;
     * below the smallest normal 2^-6 the spacing is the subnormal step 2^-9 */
    int e;
    if (a < ldexp(1.0, -6)) {
        e = -6;
    } else {
        e = (int)floor(log2(a));
        /* guard log2 rounding at exact powers of two */
        if (ldexp(1.0, e) > a) e -= 1;
        if (ldexp(1.0, e + 1) <= a) e += 1;
    }
    double quantum = ldexp(1.0, e - 3);
    double t = a / quantum;              /* exact: quantum is a power of two */
    double fl = floor(t);
    double frac = t - fl;
    double n;
    if (frac > 0.5) n = fl + 1.0;
    else if (frac < 0.5) n = fl;
    else n = (fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;      /* tie: to even */
    double r = n * quantum;               /* the rounded magnitude */
    if (r > 448.0) r = 448.0;             /* cannot happen below 448, kept for clarity */
    if (r == 0.0) return sign;
    /* encode r */
    if (r < ldexp(1.0, -6)) {             /* subnormal: r = m * 2^-9 */
        int m = (int)(r / ldexp(1.0, -9));
        return (uint8_t)(sign | m);
    }
    int re = (int)floor(log2(r));
    if (ldexp(1.0, re) > r) re -= 1;
    if (ldexp(1.0, re + 1) <= r) re += 1;
    int m = (int)((r / ldexp(1.0, re) - 1.0) * 8.0);
    return (uint8_t)(sign | ((re + 7) << 3) | m);
}

/* fp32 correctly rounded quotient (the C compiler evaluates float / float in
 * fp32 round-to-nearest under the default environment). */
static float div_f32(float a, float b) { volatile float q = a / b; return q; }
static float mul_f32(float a, float b) { volatile float p = a * b; return p; }

/* Row scale and inverse from the row's amax (reading R4). */
void orc_e4m3_row_scale(float amax, float *scale, float *inv)
{
    if (amax == 0.0f) { *scale = 1.0f; *inv = 0.0f; return; }
    *scale = div_f32(amax, 448.0f);
    *inv = div_f32(448.0f, amax);
}

/* Per-row E4M3 quantization of a dense bf16 matrix (X per token).
 * q: [rows x K] codes; scales: [rows]. */
void orc_quantize_rows_e4m3(const uint16_t *src, int64_t rows, int64_t K, int64_t ld,
                            uint8_t *q, float *scales)
{
    for (int64_t r = 0; r < rows; ++r) {
        float amax = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            float a = fabsf(bf16_to_float(src[r * ld + k]));
            if (a > amax) amax = a;
        }
        float scale, inv;
        orc_e4m3_row_scale(amax, &scale, &inv);
        scales[r] = scale;
        for (int64_t k = 0; k < K; ++k)
            q[r * K + k] = orc_e4m3_encode((double)mul_f32(bf16_to_float(src[r * ld + k]), inv));
    }
}

/* Prune + compress with E4M3 output (reading R5: prune on bf16 magnitudes,
 * then quantize kept values with the row scale).  The row amax is taken over
 * the whole input row; for a sparse row it equals the pruned row's amax
 * because every group keeps its largest magnitude.
 *
 * Hybrid tiles [P1 "Dense Fallback and Hybrid Sparsity Design"; P2 Spense and
 * PATCH abstracts]: when tile_dense_mask is not NULL it holds one byte per
 * 128 x 128 tile (row-block major, ceil(rows/128) x K/128); a non-zero byte
 * keeps that tile dense.  A dense tile's values are quantized unpruned into
 * dense_q ([rows x K]); its slots in values are 0 and its canonical nibbles
 * are 0x4 (indices 0 and 1).  With a mask, dense_q is the whole hybrid matrix
 * in dense form: a sparse tile holds its kept codes at their positions and
 * zero bytes at the dropped ones (reading R11).  Without a mask dense_q is
 * not written.
 * values_q: [rows x K/2]; meta_canon: [rows x K/8]; scales: [rows]. */
void orc_prune_compress_e4m3(const uint16_t *src, int64_t rows, int64_t K, int64_t ld,
                             const uint8_t *tile_dense_mask,
                             uint8_t *values_q, uint8_t *meta_canon, float *scales,
                             uint8_t *dense_q)
{
    int64_t KT = K / 128;
    if (rows <= 0 || K <= 0) return;
    for (int64_t r = 0; r < rows; ++r) {
        float amax = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            float a = fabsf(bf16_to_float(src[r * ld + k]));
            if (a > amax) amax = a;
        }
        float scale, inv;
        orc_e4m3_row_scale(amax, &scale, &inv);
        scales[r] = scale;
        memset(meta_canon + r * (K / 8), 0, (size_t)(K / 8));
        for (int64_t g = 0; g < K / 4; ++g) {
            const uint16_t *v = src + r * ld + 4 * g;
            int dense_tile = tile_dense_mask &&
                             tile_dense_mask[(r / 128) * KT + (4 * g) / 128] != 0;
            int nib;
            if (dense_tile) {
                nib = 0x4;
                values_q[r * (K / 2) + 2 * g + 0] = 0;
                values_q[r * (K / 2) + 2 * g + 1] = 0;
                for (int i = 0; i < 4; ++i)
                    dense_q[r * K + 4 * g + i] =
                        orc_e4m3_encode((double)mul_f32(bf16_to_float(v[i]), inv));
            } else {
                int i0, i1;
                nib = orc_prune_group(v, &i0, &i1);
                values_q[r * (K / 2) + 2 * g + 0] =
                    orc_e4m3_encode((double)mul_f32(bf16_to_float(v[i0]), inv));
                values_q[r * (K / 2) + 2 * g + 1] =
                    orc_e4m3_encode((double)mul_f32(bf16_to_float(v[i1]), inv));
                if (tile_dense_mask) {
                    for (int i = 0; i < 4; ++i) dense_q[r * K + 4 * g + i] = 0;
                    dense_q[r * K + 4 * g + i0] = values_q[r * (K / 2) + 2 * g + 0];
                    dense_q[r * K + 4 * g + i1] = values_q[r * (K / 2) + 2 * g + 1];
                }
            }
            meta_canon[r * (K / 8) + g / 2] |= (uint8_t)(nib << ((g % 2) * 4));
        }
    }
}

/* Same hybrid treatment for bf16 output: dense tiles are copied unpruned
 * into dense_out ([rows x K]); their value slots are 0 and nibbles 0x4.
 * Sparse tiles appear in dense_out pruned: kept values at their positions,
 * +0 at the dropped ones (reading R11). */
void orc_prune_compress_bf16_hybrid(const uint16_t *src, int64_t rows, int64_t K, int64_t ld,
                                    const uint8_t *tile_dense_mask,
                                    uint16_t *values, uint8_t *meta_canon, uint16_t *dense_out)
{
    int64_t KT = K / 128;
    if (rows <= 0 || K <= 0) return;
    for (int64_t r = 0; r < rows; ++r) {
        memset(meta_canon + r * (K / 8), 0, (size_t)(K / 8));
        for (int64_t g = 0; g < K / 4; ++g) {
            const uint16_t *v = src + r * ld + 4 * g;
            int dense_tile = tile_dense_mask &&
                             tile_dense_mask[(r / 128) * KT + (4 * g) / 128] != 0;
            int nib;
            if (dense_tile) {
                nib = 0x4;
                values[r * (K / 2) + 2 * g + 0] = 0;
                values[r * (K / 2) + 2 * g + 1] = 0;
                for (int i = 0; i < 4; ++i) dense_out[r * K + 4 * g + i] = v[i];
            } else {
                int i0, i1;
                nib = orc_prune_group(v, &i0, &i1);
                values[r * (K / 2) + 2 * g + 0] = v[i0];
                values[r * (K / 2) + 2 * g + 1] = v[i1];
                for (int i = 0; i < 4; ++i) dense_out[r * K + 4 * g + i] = 0;
                dense_out[r * K + 4 * g + i0] = v[i0];
                dense_out[r * K + 4 * g + i1] = v[i1];
            }
            meta_canon[r * (K / 8) + g / 2] |= (uint8_t)(nib << ((g % 2) * 4));
        }
    }
}

/* ------------------------------------------------------------------ */
/* 5. Metadata image: the canonical nibbles rearranged into the order   */
/*    the sparse tensor-core instruction reads them from tensor memory. */
/*    Written from the layout specification in include/sp24.h, not from */
/*    the CUDA code.  Parity pinned by layout spec (see header).        */
/* ------------------------------------------------------------------ */

/* Image = sequence of 2048-byte chunks, chunk (rb, kc) at index
 * rb * (K/128) + kc, for row block rb (128 rows, rows past the end count as
 * all-zero rows whose groups keep indices 0 and 1, nibble 0x4) and K-chunk kc
 * (128 consecutive K positions = 32 groups).  A chunk is 128 image rows of 16
 * bytes; image row L is 4 little-endian 32-bit words w = 0..3.
 *
 * 16-bit operands (bf16): word w of image row L covers the 32 K positions
 * [32w, 32w+32) of the chunk, split in two 16-position halves h:
 *     h = (L / 8) % 2,  r = 16 * (L / 16) + (L % 8)
 *     bits  0..15 = nibbles of groups 8w + 4h + 0..3 of row r     (nibble j at bits 4j)
 *     bits 16..31 = nibbles of groups 8w + 4h + 0..3 of row r + 8
 * 8-bit operands (e4m3): image row L is row L; its 16 bytes are the row's 32
 * canonical nibbles of the chunk in order (group 2b in the low nibble of
 * byte b). */
static int canon_nib(const uint8_t *canon, int64_t rows, int64_t K, int64_t r, int64_t g)
{
    if (r >= rows) return 0x4;
    return (canon[r * (K / 8) + g / 2] >> ((g % 2) * 4)) & 0xF;
}

void orc_meta_image(const uint8_t *canon, int64_t rows, int64_t K, int is_8bit,
                    const uint8_t *tile_dense_mask, uint8_t *image)
{
    int64_t RB = (rows + 127) / 128, KC = K / 128;
    for (int64_t rb = 0; rb < RB; ++rb) {
        for (int64_t kc = 0; kc < KC; ++kc) {
            uint8_t *chunk = image + (rb * KC + kc) * 2048;
            int dense = tile_dense_mask && tile_dense_mask[rb * KC + kc] != 0;
            for (int L = 0; L < 128; ++L) {
                for (int w = 0; w < 4; ++w) {
                    uint32_t word = 0;
                    if (!is_8bit) {
                        int h = (L / 8) % 2;
                        int64_t r = rb * 128 + 16 * (L / 16) + (L % 8);
                        for (int j = 0; j < 4; ++j) {
                            int64_t g = kc * 32 + 8 * w + 4 * h + j;
                            uint32_t lo = dense ? 0x4u : (uint32_t)canon_nib(canon, rows, K, r, g);
                            uint32_t hi = dense ? 0x4u : (uint32_t)canon_nib(canon, rows, K, r + 8, g);
                            word |= lo << (4 * j);
                            word |= hi << (16 + 4 * j);
                        }
                    } else {
                        int64_t r = rb * 128 + L;
                        for (int j = 0; j < 8; ++j) {
                            int64_t g = kc * 32 + 8 * w + j;
                            uint32_t nib = dense ? 0x4u : (uint32_t)canon_nib(canon, rows, K, r, g);
                            word |= nib << (4 * j);
                        }
                    }
                    for (int b = 0; b < 4; ++b)
                        chunk[L * 16 + w * 4 + b] = (uint8_t)((word >> (8 * b)) & 0xFF);
                }
            }
        }
    }
}

/* ------------------------------------------------------------------ */
/* 6. GEMM in fp64 on dequantized operands  [P4 "Sparse tensor cores": */
/*    the sparse product equals the dense product of the pruned matrix] */
/* ------------------------------------------------------------------ */

/* Y[m][n] = sum_k X[m][k] * W[n][k];  A[m][n] = sum_k |X[m][k] * W[n][k]|.
 * X: [M x K], W: [N x K], both row-major fp64.  A may be NULL. */
void orc_gemm_f64(const double *X, const double *W, int64_t M, int64_t N, int64_t K,
                  double *Y, double *A)
{
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            double y = 0.0, a = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                double p = X[m * K + k] * W[n * K + k];
                y += p;
                a += fabs(p);
            }
            Y[m * N + n] = y;
            if (A) A[m * N + n] = a;
        }
    }
}

/* The same contraction evaluated only at listed (m, n) pairs, for sampled
 * checks at full problem sizes. */
void orc_gemm_f64_sampled(const double *X, const double *W, int64_t K,
                          const int64_t *ms, const int64_t *ns, int64_t count,
                          double *Y, double *A)
{
    for (int64_t i = 0; i < count; ++i) {
        double y = 0.0, a = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            double p = X[ms[i] * K + k] * W[ns[i] * K + k];
            y += p;
            a += fabs(p);
        }
        Y[i] = y;
        if (A) A[i] = a;
    }
}

/* Sparse-sum form: for each kept value of W's row, the index selects the
 * matching element of X's row [P4 "Sparse tensor cores"].
 * wvals: [N x K/2] dequantized kept values; meta_canon: [N x K/8]. */
void orc_gemm_sparse_f64(const double *X, int64_t M, int64_t K,
                         const double *wvals, const uint8_t *meta_canon, int64_t N,
                         double *Y)
{
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            double y = 0.0;
            for (int64_t g = 0; g < K / 4; ++g) {
                int nib = (meta_canon[n * (K / 8) + g / 2] >> ((g % 2) * 4)) & 0xF;
                int i0 = nib & 3, i1 = (nib >> 2) & 3;
                y += wvals[n * (K / 2) + 2 * g + 0] * X[m * K + 4 * g + i0];
                y += wvals[n * (K / 2) + 2 * g + 1] * X[m * K + 4 * g + i1];
            }
            Y[m * N + n] = y;
        }
    }
}

/* Array form of orc_e4m3_encode for the Python wrapper (x holds fp32 values
 * carried exactly in doubles). */
void orc_e4m3_encode_array(const double *x, int64_t n, uint8_t *q)
{
    for (int64_t i = 0; i < n; ++i) q[i] = orc_e4m3_encode(x[i]);
}

/* ------------------------------------------------------------------ */
/* 2:4 energy loss  [P4 section 1 and section 5, "The energy that 2:4  */
/*    removes": the share of a tensor's energy carried by the two      */
/*    values that 2:4 drops from each group of four]                   */
/* ------------------------------------------------------------------ */

/* For each row: the energy (sum of squares) of the values the 2:4 prune
 * drops, and the energy of the whole row, both in fp64 (a bf16 square is
 * exact in fp64).  The share is dropped / total, per row and summed over
 * rows for the tensor.  The dropped positions are those orc_prune_group
 * does not keep. */
void orc_energy_loss(const uint16_t *src, int64_t rows, int64_t K, int64_t ld,
                     double *row_dropped, double *row_total)
{
    for (int64_t r = 0; r < rows; ++r) {
        double dropped = 0.0, total = 0.0;
        for (int64_t g = 0; g < K / 4; ++g) {
            const uint16_t *v = src + r * ld + 4 * g;
            int i0, i1;
            orc_prune_group(v, &i0, &i1);
            for (int i = 0; i < 4; ++i) {
                const double x = orc_bf16_to_double(v[i]);
                total += x * x;
                if (i != i0 && i != i1) dropped += x * x;
            }
        }
        row_dropped[r] = dropped;
        row_total[r] = total;
    }
}

/* ================================================================== */
/* Pairwise 4:8 sparsity with NVFP4 values  [P4 section 2             */
/*    "Quantization" (NVFP4: E2M1 values, one E4M3 scale per 16        */
/*    elements, one per-tensor scale) and section 6.2 "What pairwise   */
/*    4:8 costs on Blackwell" (in each group of eight elements two of  */
/*    the four adjacent pairs are kept; the sparse block-scaled GEMM   */
/*    carries one scale per 32 positions of the reduction axis)]       */
/*  [EXT] OCP microscaling formats specification, E2M1 encoding (one   */
/*    sign bit, two exponent bits with bias 1, one mantissa bit, no    */
/*    infinities or NaN, largest finite 6).                            */
/* Readings (listed in the design notes): R14 a pair's weight is its   */
/* energy x0^2 + x1^2 (exact in fp64 from bf16), the two heaviest of   */
/* the four pairs are kept, ties to the lower pair index; R15 the      */
/* scale arithmetic below, each step one correctly rounded fp32        */
/* operation; R16 block and tensor scales of the sparse operand come   */
/* from the kept values; R17 the storage layout below.                 */
/* ================================================================== */

/* E2M1 code (low 4 bits): sign bit 3, exponent bits 2..1, mantissa bit 0. */
double orc_e2m1_decode(uint8_t q)
{
    int s = (q >> 3) & 1;
    int e = (q >> 1) & 3;
    int m = q & 1;
    double mag = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return s ? -mag : mag;
}

/* Round to nearest E2M1, ties to the even code (mantissa bit 0), magnitudes
 * above 6 saturate to 6; the sign is kept (a negative value that rounds to
 * zero gives the negative-zero code).  A plain scan of the eight magnitudes. */
uint8_t orc_e2m1_encode(double x)
{
    uint8_t sign = (x < 0.0 || (x == 0.0 && signbit(x))) ? 0x8 : 0x0;
    double a = fabs(x);
    int best = 0;
    double best_d = INFINITY;
    for (int c = 0; c < 8; ++c) {
        double d = fabs(a - orc_e2m1_decode((uint8_t)c));
        if (d < best_d || (d == best_d && (c & 1) == 0)) {
            best = c;
            best_d = d;
        }
    }
    if (a > 6.0) best = 7;
    return (uint8_t)(sign | best);
}

/* The pair rule on one group of eight bf16 values: pair j holds elements
 * 2j and 2j+1; pair j is kept iff fewer than two pairs beat it, where i
 * beats j when e_i > e_j, or e_i == e_j and i < j.  Returns the canonical
 * nibble p0 | p1 << 2 (p0 < p1). */
int orc_prune_pairs8(const uint16_t v[8], int *p0, int *p1)
{
    double e[4];
    for (int j = 0; j < 4; ++j) {
        double a = orc_bf16_to_double(v[2 * j]), b = orc_bf16_to_double(v[2 * j + 1]);
        e[j] = a * a + b * b;
    }
    int kept[2];
    int nk = 0;
    for (int j = 0; j < 4; ++j) {
        int beaten_by = 0;
        for (int i = 0; i < 4; ++i) {
            if (i == j) continue;
            if (e[i] > e[j] || (e[i] == e[j] && i < j)) beaten_by++;
        }
        if (beaten_by < 2) kept[nk++] = j;
    }
    *p0 = kept[0];
    *p1 = kept[1];
    return kept[0] | (kept[1] << 2);
}

/* The 4:8 pruned matrix in bf16 (dropped positions +0).  K % 8 == 0. */
void orc_prune_pairs_bf16(const uint16_t *src, int64_t rows, int64_t K, int64_t ld, uint16_t *pruned)
{
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t g = 0; g < K / 8; ++g) {
            const uint16_t *v = src + r * ld + 8 * g;
            int p0, p1;
            orc_prune_pairs8(v, &p0, &p1);
            for (int i = 0; i < 8; ++i)
                pruned[r * K + 8 * g + i] = (i / 2 == p0 || i / 2 == p1) ? v[i] : (uint16_t)0;
        }
}

/* Per-tensor scale from the tensor amax (R15): amax / (448 * 6), 1 for 0. */
float orc_nvfp4_tensor_scale(float amax)
{
    return amax == 0.0f ? 1.0f : div_f32(amax, 2688.0f);
}

/* Block scale code from the block amax (R15): E4M3(amax / (6 * s_t)). */
uint8_t orc_nvfp4_block_code(float amax_b, float s_t)
{
    return orc_e4m3_encode((double)div_f32(amax_b, mul_f32(6.0f, s_t)));
}

/* E2M1 code of v under block code b and tensor scale s_t (R15): the
 * effective scale is S = decode(b) * s_t in fp32 and the code rounds v / S
 * (one fp32 division); a zero scale gives code 0. */
uint8_t orc_nvfp4_code(float v, uint8_t b, float s_t)
{
    float S = mul_f32((float)orc_e4m3_decode(b), s_t);
    if (S == 0.0f) return 0;
    return orc_e2m1_encode((double)div_f32(v, S));
}

static void put_nibble(uint8_t *base, int64_t idx, uint8_t nib)
{
    if (idx % 2 == 0) base[idx / 2] = (uint8_t)((base[idx / 2] & 0xF0) | (nib & 0xF));
    else base[idx / 2] = (uint8_t)((base[idx / 2] & 0x0F) | ((nib & 0xF) << 4));
}

static uint8_t get_nibble(const uint8_t *base, int64_t idx)
{
    return (uint8_t)((base[idx / 2] >> ((idx % 2) * 4)) & 0xF);
}

/* Sparse operand, pairwise 4:8 with NVFP4 values (R16, R17).  K % 32 == 0.
 *   values:   [rows x K/4] bytes, the kept elements in ascending position,
 *             two E2M1 codes per byte (the earlier element in the low nibble)
 *   meta:     [rows x K/16] bytes, one canonical nibble p0 | p1 << 2 per
 *             group of eight, the even group in the low nibble
 *   scales:   [rows x K/32] E4M3 block codes, one per 32 positions of K
 *             (16 kept values)
 *   *tensor_scale: the fp32 per-tensor scale.
 * The tensor amax and each block amax run over the kept values. */
void orc_nvfp4_48_compress(const uint16_t *src, int64_t rows, int64_t K, int64_t ld,
                           uint8_t *values, uint8_t *meta, uint8_t *scales, float *tensor_scale)
{
    float amax_t = 0.0f;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t g = 0; g < K / 8; ++g) {
            const uint16_t *v = src + r * ld + 8 * g;
            int p0, p1;
            orc_prune_pairs8(v, &p0, &p1);
            const int pos[4] = {2 * p0, 2 * p0 + 1, 2 * p1, 2 * p1 + 1};
            for (int i = 0; i < 4; ++i) {
                float a = fabsf(bf16_to_float(v[pos[i]]));
                if (a > amax_t) amax_t = a;
            }
        }
    const float s_t = orc_nvfp4_tensor_scale(amax_t);
    *tensor_scale = s_t;
    memset(values, 0, (size_t)(rows * (K / 4)));
    memset(meta, 0, (size_t)(rows * (K / 16)));
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t blk = 0; blk < K / 32; ++blk) {
            float kept[16];
            int nk = 0;
            for (int64_t g = 4 * blk; g < 4 * blk + 4; ++g) {
                const uint16_t *v = src + r * ld + 8 * g;
                int p0, p1;
                int nib = orc_prune_pairs8(v, &p0, &p1);
                put_nibble(meta + r * (K / 16), g, (uint8_t)nib);
                const int pos[4] = {2 * p0, 2 * p0 + 1, 2 * p1, 2 * p1 + 1};
                for (int i = 0; i < 4; ++i) kept[nk++] = bf16_to_float(v[pos[i]]);
            }
            float amax_b = 0.0f;
            for (int i = 0; i < 16; ++i)
                if (fabsf(kept[i]) > amax_b) amax_b = fabsf(kept[i]);
            const uint8_t b = orc_nvfp4_block_code(amax_b, s_t);
            scales[r * (K / 32) + blk] = b;
            for (int i = 0; i < 16; ++i)
                put_nibble(values + r * (K / 4), 16 * blk + i, orc_nvfp4_code(kept[i], b, s_t));
        }
}

/* The dequantized dense matrix of a 4:8 NVFP4 operand (fp64, [rows x K]):
 * each kept code times its block scale times the tensor scale, zeros at
 * the dropped positions. */
void orc_nvfp4_48_dequant(const uint8_t *values, const uint8_t *meta, const uint8_t *scales,
                          float tensor_scale, int64_t rows, int64_t K, double *out)
{
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t k = 0; k < K; ++k) out[r * K + k] = 0.0;
        for (int64_t g = 0; g < K / 8; ++g) {
            const uint8_t nib = get_nibble(meta + r * (K / 16), g);
            const int p0 = nib & 3, p1 = (nib >> 2) & 3;
            const int pos[4] = {2 * p0, 2 * p0 + 1, 2 * p1, 2 * p1 + 1};
            const double sb = orc_e4m3_decode(scales[r * (K / 32) + g / 4]) * (double)tensor_scale;
            for (int i = 0; i < 4; ++i)
                out[r * K + 8 * g + pos[i]] = orc_e2m1_decode(get_nibble(values + r * (K / 4), 4 * g + i)) * sb;
        }
    }
}

/* Dense NVFP4 with one E4M3 block code per `block` elements along K (16: the
 * dense NVFP4 operand; 32: the dense operand of the sparse block-scaled GEMM,
 * which carries one scale per 32 positions of the reduction axis), the tensor
 * scale from the whole matrix (R15).  K % block == 0.
 *   codes: [rows x K/2] bytes, two E2M1 codes per byte; scales: [rows x K/block]. */
void orc_nvfp4_quantize_blocks(const uint16_t *src, int64_t rows, int64_t K, int64_t ld, int block,
                               uint8_t *codes, uint8_t *scales, float *tensor_scale)
{
    float amax_t = 0.0f;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t k = 0; k < K; ++k) {
            float a = fabsf(bf16_to_float(src[r * ld + k]));
            if (a > amax_t) amax_t = a;
        }
    const float s_t = orc_nvfp4_tensor_scale(amax_t);
    *tensor_scale = s_t;
    memset(codes, 0, (size_t)(rows * (K / 2)));
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t blk = 0; blk < K / block; ++blk) {
            float amax_b = 0.0f;
            for (int i = 0; i < block; ++i) {
                float a = fabsf(bf16_to_float(src[r * ld + block * blk + i]));
                if (a > amax_b) amax_b = a;
            }
            const uint8_t b = orc_nvfp4_block_code(amax_b, s_t);
            scales[r * (K / block) + blk] = b;
            for (int i = 0; i < block; ++i)
                put_nibble(codes + r * (K / 2), block * blk + i,
                           orc_nvfp4_code(bf16_to_float(src[r * ld + block * blk + i]), b, s_t));
        }
}

/* The dequantized matrix of a dense NVFP4 operand (fp64, [rows x K]). */
void orc_nvfp4_dequant_blocks(const uint8_t *codes, const uint8_t *scales, float tensor_scale,
                              int64_t rows, int64_t K, int block, double *out)
{
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t k = 0; k < K; ++k)
            out[r * K + k] = orc_e2m1_decode(get_nibble(codes + r * (K / 2), k)) *
                             orc_e4m3_decode(scales[r * (K / block) + k / block]) * (double)tensor_scale;
}

/* Device images of the NVFP4 operands for the block-scaled tensor-core MMA
 * (layout spec; parity pinned by layout spec and by the GPU GEMM that reads
 * them through the tensor cores, as for the 2:4 metadata image).
 *
 * 4:8 metadata image: 2048-byte chunks, one per (128-row block rb, 256
 * positions of K kc) at byte (rb * K/256 + kc) * 2048; image row L (16 bytes
 * at 16 L) is row 128 rb + L's canonical metadata bytes [16 kc, 16 kc + 16)
 * (32 group nibbles, the even group low); rows past the end hold 0x44 bytes
 * (pairs 0 and 1 in every group).  K % 256 == 0. */
void orc_nvfp4_48_meta_image(const uint8_t *meta, int64_t rows, int64_t K, uint8_t *image)
{
    int64_t RB = (rows + 127) / 128, KC = K / 256;
    for (int64_t rb = 0; rb < RB; ++rb)
        for (int64_t kc = 0; kc < KC; ++kc)
            for (int L = 0; L < 128; ++L) {
                uint8_t *dst = image + (rb * KC + kc) * 2048 + 16 * L;
                int64_t r = rb * 128 + L;
                for (int b = 0; b < 16; ++b)
                    dst[b] = r < rows ? meta[r * (K / 16) + 16 * kc + b] : (uint8_t)0x44;
            }
}

/* Scale image: 512-byte chunks, one per (128-row block rb, four consecutive
 * scale blocks kq) at byte (rb * nblk/4 + kq) * 512; the code of row
 * r = 128 rb + 32 q + l (0 <= l < 32), block 4 kq + j sits at byte
 * 16 l + 4 q + j of the chunk; rows past the end hold 0.  nblk % 4 == 0. */
void orc_nvfp4_scale_image(const uint8_t *scales, int64_t rows, int64_t nblk, uint8_t *image)
{
    int64_t RB = (rows + 127) / 128, KQ = nblk / 4;
    for (int64_t rb = 0; rb < RB; ++rb)
        for (int64_t kq = 0; kq < KQ; ++kq)
            for (int q = 0; q < 4; ++q)
                for (int l = 0; l < 32; ++l) {
                    int64_t r = rb * 128 + 32 * q + l;
                    for (int j = 0; j < 4; ++j)
                        image[(rb * KQ + kq) * 512 + 16 * l + 4 * q + j] =
                            r < rows ? scales[r * nblk + 4 * kq + j] : (uint8_t)0;
                }
}

/* 4:8 pairwise energy loss per row, as orc_energy_loss for 2:4: the energy
 * of the values the pair rule drops and of the whole row (fp64). */
void orc_energy_loss_48(const uint16_t *src, int64_t rows, int64_t K, int64_t ld,
                        double *row_dropped, double *row_total)
{
    for (int64_t r = 0; r < rows; ++r) {
        double dropped = 0.0, total = 0.0;
        for (int64_t g = 0; g < K / 8; ++g) {
            const uint16_t *v = src + r * ld + 8 * g;
            int p0, p1;
            orc_prune_pairs8(v, &p0, &p1);
            for (int i = 0; i < 8; ++i) {
                const double x = orc_bf16_to_double(v[i]);
                total += x * x;
                if (i / 2 != p0 && i / 2 != p1) dropped += x * x;
            }
        }
        row_dropped[r] = dropped;
        row_total[r] = total;
    }
}
