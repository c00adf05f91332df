/*
 * sp24.h -- C ABI of the B200 (sm_100a) 2:4 semi-structured sparse GEMM library.
 *
 * Y = X * W^T with X [M x K] and W [N x K], both row-major with K contiguous.
 * 2:4 sparsity: in every group of four consecutive elements along the
 * reduction axis K at most two are non-zero; the sparse operand is stored as
 * a half-size value array plus a 2-bit position index for each kept value.
 *   - "2:4 Structured Sparsity Explained" (tensorcore.si), section
 *     "How 2:4 sparsity works": the format, 36 bits per group of four FP16.
 *   - "Production 2:4 Structured Sparsity for LLMs" (oh-bug.com), section
 *     "Core Mechanisms and Production States of 2:4 Structured Sparsity":
 *     the worked example [0.42,-0.18,0.07,0.31] -> [0.42,0,0,0.31] and the
 *     pruned / eligible / selected states.
 *   - the 2:4-versus-quantization paper (paperpeel.com/paper/2610.28947),
 *     section 2, "Sparse tensor cores": the sparse MMA takes its first operand
 *     A compressed and uses the indices to select the matching elements of the
 *     dense operand B; only one operand is sparse; groups lie along K.
 *
 * Conventions for every call:
 *  - Pointers named *_dev are DEVICE pointers; the caller allocates and frees
 *    every buffer it passes.  The library's own device memory is limited to
 *    two documented items: the fixed scratch array of sp24_gemm_noalloc (a
 *    static array, held by every GPU that loads the library), and the L2
 *    flush buffer of sp24_select_tactic (twice the L2 size, allocated on the
 *    selector's first call on a device and kept until exit).  No other call
 *    allocates device memory.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Every call is asynchronous on that stream unless stated.
 *  - Argument errors are returned synchronously, before any launch.  A failed
 *    launch returns SP24_ERR_CUDA.  A device-side bounded wait that expires
 *    records a code in a device error word, read by sp24_last_device_error().
 *  - bf16 data are passed as 16-bit patterns, e4m3 data as bytes (OCP FP8
 *    E4M3: bias 7, 3 mantissa bits, no infinities, largest finite 448).
 *  - Leading dimensions (ld*) are in elements; every row pitch must be a
 *    multiple of 16 bytes and every base pointer 16-byte aligned
 *    (SP24_ERR_ALIGNMENT otherwise).
 *
 * Magnitude prune (reading where the pages are silent): in each group the
 * two positions with the largest |v| survive, comparing bf16 magnitude bits
 * as integers; equal magnitudes go to the lower index; a group always keeps
 * exactly two positions, so a group with fewer than two non-zeros keeps
 * zeros ("How to make a model 2:4 sparse": keep the two with the largest
 * magnitude).
 *
 * Metadata nibble of one group: i0 | (i1 << 2), i0 < i1 the kept positions.
 *
 * METADATA IMAGE LAYOUT (what sp24_prune_compress writes and sp24_gemm reads).
 * The nibbles are stored in the order the sparse tensor-core instruction reads
 * them from tensor memory, so the GEMM copies them to tensor memory with no
 * rearrangement.  The image is a sequence of 2048-byte chunks; chunk (rb, kc),
 * for row block rb (128 rows; rows past the end behave as all-zero rows whose
 * groups keep positions 0 and 1, nibble 0x4) and K-chunk kc (128 consecutive
 * K positions = 32 groups), sits at byte offset (rb * (K/128) + kc) * 2048.
 * A chunk is 128 image rows L of 16 bytes = four little-endian 32-bit words w.
 *  - 16-bit values (bf16): word w of image row L covers chunk positions
 *    [32w, 32w+32) in two halves h = (L/8) % 2 of 16 positions; with
 *    r = 16*(L/16) + L%8 (row within the block):
 *        bits  0..15: nibbles of groups 8w+4h+0..3 of row r   (nibble j at bit 4j)
 *        bits 16..31: nibbles of groups 8w+4h+0..3 of row r+8
 *  - 8-bit values (e4m3): image row L is row L; its 16 bytes hold the row's 32
 *    nibbles of the chunk in order, even group in the low nibble of a byte.
 * sp24_meta_bytes() returns the image size.
 */
#ifndef SP24_H
#define SP24_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum sp24_status {
    SP24_OK = 0,
    SP24_ERR_INVALID_ARG = 1,       /* a size or enum out of range              */
    SP24_ERR_NULL = 2,              /* a required pointer is NULL               */
    SP24_ERR_DTYPE = 3,             /* dtype combination not supported          */
    SP24_ERR_ALIGNMENT = 4,         /* pointer, pitch or shape misaligned       */
    SP24_ERR_NOT_2_4 = 5,           /* operand is not eligible for the sparse path */
    SP24_ERR_UNSUPPORTED_DEVICE = 6,/* current device is not sm_100             */
    SP24_ERR_CUDA = 7,              /* a CUDA runtime call failed               */
    SP24_ERR_DEVICE_TIMEOUT = 8,    /* a device-side bounded wait expired       */
    SP24_ERR_WORKSPACE = 9          /* workspace missing or too small           */
} sp24_status;

typedef enum sp24_dtype { SP24_BF16 = 0, SP24_E4M3 = 1, SP24_F32 = 2 } sp24_dtype;

typedef enum sp24_tactic { SP24_TACTIC_SPARSE = 0, SP24_TACTIC_DENSE = 1 } sp24_tactic;

/* ---------------------------------------------------------------------- */
/* Sizes                                                                   */
/* ---------------------------------------------------------------------- */

/* Bytes of the compressed value array [rows x K/2] of `dtype` (BF16 or E4M3). */
size_t sp24_values_bytes(int64_t rows, int64_t K, sp24_dtype dtype);

/* Bytes of the metadata image: ceil(rows/128) * (K/128) * 2048. */
size_t sp24_meta_bytes(int64_t rows, int64_t K);

/* ---------------------------------------------------------------------- */
/* Prune + compress (kernel 1)                                             */
/* ---------------------------------------------------------------------- */

/* Magnitude 2:4 prune of src along K and compression, in one pass over src
 * for BF16 output, and for E4M3 output without a tile mask on rows up to
 * 28672 wide (the row held in registers: amax, prune, cast and scale in one
 * launch); E4M3 with a tile mask or longer rows takes three stream-ordered
 * launches (row amax, prune, scale finalize).  Same results either way.
 *   src_dev     bf16 [rows x K], row pitch ld elements.
 *   out_dtype   SP24_BF16: values are the kept bf16 values.
 *               SP24_E4M3: kept values quantized per row: scale = amax/448,
 *               inv = 448/amax (both correctly rounded fp32 divisions, amax
 *               over the whole input row), q = E4M3 round-to-nearest-even
 *               saturating of the fp32 product v*inv; amax == 0 gives scale 1
 *               and q = 0 ("Quantization": FP8 E4M3 needs one scale per row;
 *               section 5.1: round-to-nearest is the basic quantizer; prune
 *               before quantize).
 *   values_dev  [rows x K/2] of out_dtype, contiguous (row pitch K/2).
 *   meta_dev    metadata image, sp24_meta_bytes(rows, K) bytes.
 *   row_scales_dev  fp32 [rows], required for E4M3, ignored for BF16.
 *   tile_dense_mask_dev  NULL, or one byte per 128 x 128 tile of src,
 *               [ceil(rows/128) x K/128] row-block major; non-zero keeps that
 *               tile dense (hybrid sparse-dense weights: "Dense Fallback and
 *               Hybrid Sparsity Design"; the Spense and PATCH abstracts on the
 *               SlideSparse page).  A dense tile is written unpruned (quantized
 *               with the row scale for E4M3) into dense_tiles_dev; its value
 *               slots are written as 0 and its metadata nibbles as 0x4.
 *   dense_tiles_dev  [rows x K] of out_dtype, contiguous: the hybrid matrix in
 *               dense form.  Dense tiles hold their values unpruned, sparse
 *               tiles their kept values in place and zeros at the dropped
 *               positions.  Required when the mask is given; not written
 *               without one.
 * Requirements: rows >= 1, K % 128 == 0, ld >= K, ld % 8 == 0.
 */
int sp24_prune_compress(const void *src_dev, int64_t rows, int64_t K, int64_t ld,
                        sp24_dtype out_dtype, void *values_dev, void *meta_dev,
                        float *row_scales_dev, const uint8_t *tile_dense_mask_dev,
                        void *dense_tiles_dev, void *stream);

/* Scatter compressed values back to a dense [rows x K] matrix of the same
 * element type (bf16 bits or e4m3 codes); zeros elsewhere.  Exact inverse of
 * the compression: decompress(compress(W)) == prune(W) bit for bit.
 *   values_dev [rows x K/2], meta_dev metadata image, dst_dev [rows x K]. */
int sp24_decompress(const void *values_dev, const void *meta_dev, int64_t rows, int64_t K,
                    sp24_dtype dtype, void *dst_dev, void *stream);

/* Per-row (per-token) E4M3 quantization of a dense bf16 matrix, same rule as
 * the E4M3 prune path: q [rows x K] (row pitch K), scales fp32 [rows]. */
int sp24_quantize_e4m3_rows(const void *src_dev, int64_t rows, int64_t K, int64_t ld,
                            void *q_dev, float *scales_dev, void *stream);

/* One matrix of a grouped per-token quantization (host struct; pointers are
 * device pointers, same meaning as in sp24_quantize_e4m3_rows). */
typedef struct sp24_quant_item {
    const void *src_dev;      /* bf16 [rows x K], row pitch ld elements          */
    int64_t rows, K, ld;
    void *q_dev;              /* e4m3 [rows x K], row pitch K                    */
    float *scales_dev;        /* fp32 [rows]                                     */
} sp24_quant_item;

/* The per-token quantization of up to 32 independent matrices in one launch
 * (same rule and results as sp24_quantize_e4m3_rows on each).  The item array
 * is read on the host during the call. */
int sp24_quantize_e4m3_rows_grouped(const sp24_quant_item *items, int n_items, void *stream);

/* ---------------------------------------------------------------------- */
/* GEMM (kernels 2 and 3)                                                  */
/* ---------------------------------------------------------------------- */

typedef struct sp24_gemm_args {
    int64_t M, N, K;          /* Y [M x N] = X [M x K] * W [N x K]^T            */
    sp24_dtype in_dtype;      /* SP24_BF16 or SP24_E4M3 (both operands)          */
    sp24_dtype out_dtype;     /* SP24_BF16 or SP24_F32                           */
    sp24_tactic tactic;       /* SPARSE: W given compressed; DENSE: W dense      */
    const void *X;            /* device, [M x K] row pitch ldx                   */
    int64_t ldx;
    const void *W;            /* device; DENSE: [N x K] pitch ldw; SPARSE: values
                                 [N x K/2] pitch ldw (elements of a values row)  */
    int64_t ldw;
    const void *W_meta;       /* device; SPARSE: metadata image of W             */
    const float *x_scales;    /* device fp32 [M]; E4M3 only (per token)          */
    const float *w_scales;    /* device fp32 [N]; E4M3 only (per output channel) */
    const uint8_t *tile_dense_mask; /* device; SPARSE E4M3 only: NULL or the
                                 [N/128 x K/128] hybrid tile mask                */
    const void *W_dense_tiles;/* device [N x K] pitch K: W in dense form as
                                 sp24_prune_compress writes it for a hybrid
                                 mask (sparse tiles pruned).  The one-CTA
                                 kernel reads dense tiles from it; a CTA pair
                                 (M, N >= 256) also reads a sparse tile from it
                                 at K-steps where the other half is dense    */
    void *Y;                  /* device, [M x N] row pitch ldy                   */
    int64_t ldy;
    void *workspace;          /* device stream-K workspace (see below) or NULL   */
    size_t workspace_bytes;
    uint32_t flags;           /* SP24_GEMM_* bits below, 0 for none              */
} sp24_gemm_args;

/* W, W_meta, w_scales, tile_dense_mask and W_dense_tiles are not written by
 * the kernel that precedes the call in the stream (static weights): the GEMM
 * starts streaming them before that kernel finishes (programmatic dependent
 * launch).  X, x_scales and Y are always ordered after it. */
#define SP24_GEMM_W_STATIC 1u

/* Shapes with M >= 256 tokens and N >= 256 output features run on CTA
 * pairs: one tcgen05 MMA over two SMs computes a 256 x 256 output tile (256
 * weight rows x 240 tokens when the weights are sparse or hybrid), each SM
 * loading half of both operands (no workspace).  With a hybrid mask they
 * do so only when those tiles are at least as many as the pairs that
 * fit on the device at once (a pair's K-step runs dense when either of its
 * two row blocks is dense there, which costs more than the one-CTA kernel's
 * per-tile choice unless the one-CTA kernel is short of tiles).  This flag
 * keeps such a call on the one-CTA kernel (128-row tiles); results agree to
 * the tolerance of the method, not bit for bit. */
#define SP24_GEMM_SINGLE_CTA 2u

/* For M <= 255 (and N >= 256, no hybrid mask): run 256-row weight tiles on
 * CTA pairs (M = 256 pair MMA, each SM loading half of the tile) instead of
 * 128-row tiles on single CTAs.  In a grouped call it applies when every
 * problem sets it.  With a hybrid mask and M, N >= 256: take the CTA-pair
 * kernel whatever the tile count.  Same results to the method's tolerance. */
#define SP24_GEMM_CTA_PAIR 4u

/* The kernel that precedes this call in the stream is an sp24 GEMM call that
 * is independent of it: neither call writes anything the other reads or
 * writes (inputs, outputs, workspace), and every input of this call was
 * complete when that preceding call began (it waited for its own upstream
 * kernel).  The call then starts its work as soon as SMs free up, without
 * waiting for the preceding GEMM to finish, and waits for it only before
 * exiting, so that its own completion still implies the preceding call's.
 * Ignored by the CTA-pair kernel, which always waits.  In a
 * grouped call it applies when every problem sets it.  Meant for chains of
 * independent GEMMs after one producer, such as a layer's projections after
 * one activation cast. */
#define SP24_GEMM_AFTER_INDEPENDENT 8u

/* Bytes of workspace the call would use for its stream-K schedule (0 if the
 * shape needs none).  Shapes with few output tiles per SM may split the
 * tiles' K range over all SMs (a cost model decides; the ranges are cut by
 * estimated cost, so SMs that stream wider token tiles get fewer K-stages);
 * a split tile is finished by the SM holding its first K-stage, which adds
 * the others' fp32 partial tiles (stored in the workspace) to its own.  The
 * split, and with it the fp32 summation order, is fixed by the shapes and the
 * device: repeated calls give identical results.  With a smaller or
 * missing workspace the call falls back to whole tiles per CTA (fewer SMs
 * busy on such shapes).  The workspace must be zero-filled once before its
 * first use; every call that returns SP24_OK leaves its state (the leading
 * sp24_gemm_workspace_state_bytes) zero again.  Calls that share a workspace
 * must not overlap on the GPU. */
size_t sp24_gemm_workspace_bytes(const sp24_gemm_args *args);

/* Y = s_x[m] * s_w[n] * sum_k x[m,k] * w[n,k] (scales only for E4M3), fp32
 * accumulation in tensor memory, one persistent tcgen05 kernel launch.
 * SPARSE (sparse operand = W, "Sparse tensor cores"): requires N % 128 == 0,
 * K % 128 == 0; SP24_ERR_NOT_2_4 otherwise.  DENSE: requires K % 16 == 0
 * (bf16) / K % 16 == 0 (e4m3); any M, N >= 1. */
int sp24_gemm(const sp24_gemm_args *args, void *stream);

/* Up to 16 independent GEMMs in one persistent launch (a grouped GEMM: the
 * projections that share an input, experts, or any batch of independent
 * problems).  Same results as sp24_gemm on each.  The work of all problems
 * is scheduled together, so the weights of the whole group stream without a
 * launch, ramp or tail between problems.  All problems must share in_dtype,
 * out_dtype and tactic, and either all carry a hybrid tile mask or none
 * does; otherwise SP24_ERR_INVALID_ARG.  Their token counts may differ: the
 * launch is built for the widest token tile of the group (16, 32, 64 or 128
 * tokens by M) and each problem runs its own width, so problems with small M
 * stream their weights next to wider ones (fewer pipeline stages than a
 * launch of small-M problems alone).  Hybrid problems run 128-row tiles on
 * single CTAs, each stage two tile columns, dense or sparse as their flags
 * say.  On the stream-K schedule, the first call with a given argument block
 * copies the problems' tile masks to the host (a small copy on `stream`,
 * waited for; skipped while `stream` is being captured) to cut the K ranges
 * by the bytes each step streams; the masks only steer that balance, the
 * kernel reads them itself.  The same holds for sp24_gemm.  Each args'
 * own workspace fields are ignored: the group uses `workspace` (size from
 * sp24_gemm_grouped_workspace_bytes, same zero-fill rule as sp24_gemm).
 * SP24_GEMM_W_STATIC applies when every problem sets it. */
int sp24_gemm_grouped(const sp24_gemm_args *args, int n, void *workspace_dev, size_t workspace_bytes,
                      void *stream);

/* Leading bytes of the workspace that hold the stream-K state (the
 * partial-tile flags): zero before the first call, and zero
 * again after every call that returns SP24_OK.  The rest of the workspace
 * holds partial tiles whose contents never matter between calls.  0 when the
 * call's schedule needs no workspace. */
size_t sp24_gemm_workspace_state_bytes(const sp24_gemm_args *args);
size_t sp24_gemm_grouped_workspace_state_bytes(const sp24_gemm_args *args, int n);

size_t sp24_gemm_grouped_workspace_bytes(const sp24_gemm_args *args, int n);

/* The GEMM for callers that cannot allocate device memory: code that runs
 * where cudaMalloc is unavailable or unwanted, for instance inside a stream
 * capture that must not allocate, in an allocator-free runtime, or under a
 * caller that owns every byte of device memory and has none to lend.  It
 * behaves like sp24_gemm but takes its stream-K scratch from a fixed 8 MiB
 * array inside this library (args->workspace and args->workspace_bytes are
 * ignored) and never allocates or frees device memory.
 * Not from the pages: they have no counterpart; this is an operational
 * variant of sp24_gemm.
 *  - The first call on each device looks up the array's device address (with
 *    that device current) and caches it; make that first call before any
 *    stream capture.  With hybrid weights on the stream-K schedule, the first
 *    call with a given argument block also reads the tile mask back to the
 *    host to balance the schedule (as sp24_gemm does; skipped while `stream`
 *    is being captured, which leaves the balance unweighted).
 *  - The schedule is the one sp24_gemm picks when given a workspace of
 *    sp24_gemm_noalloc_max_scratch_bytes(): a shape whose stream-K schedule
 *    would need more scratch than that runs whole tiles per CTA (no scratch),
 *    and shapes on the CTA-pair kernel (M, N >= 256) use none.  A plan that
 *    still needed more than the array would return SP24_ERR_WORKSPACE.
 *  - A call whose schedule uses scratch clears the part of the array that
 *    must start at zero (a memset on `stream`); every call shares the same
 *    array, so calls that overlap on the GPU race with each other (on one
 *    device, issue them on one stream or order them). */
int sp24_gemm_noalloc(const sp24_gemm_args *args, void *stream);

/* Size of the fixed scratch array sp24_gemm_noalloc draws on. */
size_t sp24_gemm_noalloc_max_scratch_bytes(void);

/* ---------------------------------------------------------------------- */
/* Online activation prune + compress fused ahead of the GEMM (kernel 4)   */
/* ---------------------------------------------------------------------- */

/* Bytes of workspace sp24_prune_compress_activations_fused needs when the
 * caller does not keep the compressed activations (values + image). */
size_t sp24_activations_workspace_bytes(int64_t M, int64_t K);

/* Every call: prune + compress X (bf16 [M x K], pitch ldx) along K, then
 * Y [M x N] = X_pruned * W^T with W dense bf16 [N x K] (pitch ldw), X as the
 * sparse operand ("Measuring speed": a dynamic operand pays for its own
 * prune and compress; section 4.2: a fused kernel reads the operand once and
 * writes the kept values and indices once).  The GEMM launch is chained to
 * the prune launch by programmatic dependent launch on `stream`.
 *   x_values_dev / x_meta_dev: where the compressed X goes ([M x K/2] bf16
 *   and the image of M rows); both NULL -> placed in workspace_dev, which must
 *   then hold sp24_activations_workspace_bytes(M, K) bytes.
 * Requirements: K % 128 == 0, ldx % 8 == 0, ldw % 8 == 0, N >= 1. */
int sp24_prune_compress_activations_fused(const void *X_dev, int64_t M, int64_t K, int64_t ldx,
                                          const void *W_dev, int64_t N, int64_t ldw,
                                          void *Y_dev, int64_t ldy, sp24_dtype out_dtype,
                                          void *x_values_dev, void *x_meta_dev,
                                          void *workspace_dev, size_t workspace_bytes,
                                          void *stream);

/* The online-activation path with the prune inside the GEMM: every call, a
 * CTA-pair GEMM loads raw bf16 X tiles with TMA and prunes + compresses them
 * in shared memory (converter warps of the GEMM kernel itself, same rule and
 * layouts as sp24_prune_compress), then Y [M x N] = X_pruned * W^T with W
 * dense bf16 [N x K], X as the sparse operand.  No compressed copy of X goes
 * through HBM ("Measuring speed", section 3.5 of the 2:4-versus-quantization
 * paper: a dynamic operand pays for its own prune; the two-kernel path of
 * sp24_prune_compress_activations_fused writes and re-reads it).  The prune of
 * an X tile is repeated for every 256-row block of W it meets.
 *   x_values_dev / x_meta_dev: NULL (both), or where the compressed X also
 *   goes ([M x K/2] bf16 and the image of M rows), for inspection.
 * Requirements: M >= 256, N >= 256, K % 128 == 0, ldx % 8 == 0, ldw % 8 == 0,
 * 16-byte aligned pointers.  Asynchronous on `stream`. */
int sp24_prune_activations_in_gemm(const void *X_dev, int64_t M, int64_t K, int64_t ldx, const void *W_dev,
                                   int64_t N, int64_t ldw, void *Y_dev, int64_t ldy, sp24_dtype out_dtype,
                                   void *x_values_dev, void *x_meta_dev, void *stream);

/* The online-activation path at the FP8 floor: per call, X (bf16 [M x K])
 * is pruned 2:4 along K on its bf16 magnitudes (same rule as
 * sp24_prune_compress), the kept values are cast to E4M3 with one fp32 scale
 * per token (row amax / 448, the rule of sp24_quantize_e4m3_rows), and then
 * Y [M x N] = X_sparse * Wq^T with Wq the dense E4M3 weights [N x K] and
 * their per-output-channel scales w_scales [N] (from sp24_quantize_e4m3_rows).
 * (The activation prune "optionally fuses FP8 or INT8 quantization":
 * 2:4-versus-quantization paper, section 3.5.)  x_values (E4M3 [M x K/2]),
 * x_meta (image, sp24_meta_bytes(M, K)) and x_scales ([M] fp32) receive the
 * compressed activations when given (all three or none); otherwise workspace
 * must hold sp24_activations_e4m3_workspace_bytes(M, K) bytes.  ldw is in
 * bytes and a multiple of 16.  Same errors as the bf16 path. */
size_t sp24_activations_e4m3_workspace_bytes(int64_t M, int64_t K);
int sp24_prune_compress_activations_fused_e4m3(const void *X_dev, int64_t M, int64_t K, int64_t ldx,
                                               const void *Wq_dev, const float *w_scales_dev, int64_t N,
                                               int64_t ldw, void *Y_dev, int64_t ldy, sp24_dtype out_dtype,
                                               void *x_values_dev, void *x_meta_dev, float *x_scales_dev,
                                               void *workspace_dev, size_t workspace_bytes, void *stream);

/* The 2:4 energy loss e_2:4 of a bf16 matrix [rows x K] (row-major, ld
 * elements): the share of the energy (sum of squares) carried by the two
 * values that the 2:4 prune of sp24_prune_compress drops from every group of
 * four along K ("the 2:4 energy loss": 2:4-versus-quantization paper,
 * section 1 and section 5, "The energy that 2:4 removes"), as a cheap
 * diagnostic next to the prune.  row_share_dev [rows] (fp64, may be NULL)
 * receives each row's share (0 for a row with no energy); sums_dev [2] (fp64,
 * may be NULL) receives the dropped and the total energy of the whole
 * tensor, so e_2:4 = sums[0] / sums[1] (the call zeroes sums first; the
 * atomic accumulation order varies, within fp64 rounding).  At least one
 * output is required.  K must be a multiple of 8, ld a multiple of 8, src
 * 16-byte aligned.  Asynchronous on `stream`. */
int sp24_energy_loss(const void *src_dev, int64_t rows, int64_t K, int64_t ld, double *row_share_dev,
                     double *sums_dev, void *stream);

/* ---------------------------------------------------------------------- */
/* Pairwise 4:8 sparse NVFP4 (the Blackwell sparse FP4 format)             */
/* ---------------------------------------------------------------------- */
/* NVFP4: E2M1 values (two per byte, the earlier element in the low nibble),
 * one unsigned E4M3 scale per block of positions along K, one fp32 scale per
 * tensor ("Quantization", section 2 of the 2:4-versus-quantization paper,
 * paperpeel.com/paper/2610.28947).  The pairwise 4:8 pattern keeps two of the
 * four adjacent pairs in every group of eight along K, and the sparse
 * block-scaled GEMM carries one scale per 32 positions of K (section 6.2,
 * "What pairwise 4:8 costs on Blackwell").
 * Readings where the pages are silent: the two pairs of largest energy
 * x0^2 + x1^2 survive (ties to the lower pair index); tensor scale
 * s_t = amax / 2688 (1 for amax 0); block code b = E4M3(amax_b / (6 s_t));
 * value code = E2M1(v / (decode(b) * s_t)), each step one correctly rounded
 * fp32 operation, E2M1 rounding to nearest even and saturating at 6 (a zero
 * block scale gives code 0); for the sparse operand both amaxes run over the
 * kept values.
 * Device layouts:
 *  - sparse values [rows x K/4] bytes (kept elements in ascending position);
 *    dense codes [rows x K/2] bytes;
 *  - 4:8 metadata image: 2048-byte chunks, one per (128-row block rb, 256
 *    positions kc) at (rb * K/256 + kc) * 2048; image row L (16 bytes at 16 L)
 *    holds row 128 rb + L's 32 group nibbles p0 | p1 << 2 (p0 < p1 the kept
 *    pairs) in order, the even group low; rows past the end hold 0x44;
 *  - scale image: 512-byte chunks, one per (128-row block rb, four
 *    consecutive scale blocks kq) at (rb * nblk/4 + kq) * 512, the code of row
 *    128 rb + 32 q + l, block 4 kq + j at byte 16 l + 4 q + j; rows past the
 *    end hold 0 (the order in which the tensor core reads scales from tensor
 *    memory after a 32 x 128-bit, four-quarter copy). */

size_t sp24_nvfp4_48_values_bytes(int64_t rows, int64_t K);      /* rows * K/4            */
size_t sp24_nvfp4_48_meta_bytes(int64_t rows, int64_t K);        /* ceil(rows/128)*K/256*2048 */
size_t sp24_nvfp4_codes_bytes(int64_t rows, int64_t K);          /* rows * K/2            */
size_t sp24_nvfp4_scales_bytes(int64_t rows, int64_t K, int block); /* ceil(rows/128)*128*K/block */

/* Pairwise 4:8 prune + NVFP4 cast of a bf16 matrix (weights, offline):
 * values, metadata image, scale image (one code per 32 positions) and the
 * tensor scale (device fp32; it holds the amax bits during the call).  Four
 * stream-ordered steps on `stream`: zero the tensor scale, tensor amax of the
 * kept values, prune + cast, amax -> scale.  Requirements: rows >= 1,
 * K % 256 == 0, ld >= K, ld % 8 == 0, all pointers 16-byte aligned. */
int sp24_prune_compress_nvfp4_48(const void *src_dev, int64_t rows, int64_t K, int64_t ld,
                                 void *values_dev, void *meta_dev, void *scales_dev, float *tensor_scale_dev,
                                 void *stream);

/* Dense NVFP4 cast of a bf16 matrix with one scale per `block` positions
 * (16: dense NVFP4; 32: the dense operand of the sparse 4:8 GEMM): codes,
 * scale image and tensor scale, as above (amax over every value).
 * Requirements: K % (4 * block) == 0, block in {16, 32}. */
int sp24_quantize_nvfp4(const void *src_dev, int64_t rows, int64_t K, int64_t ld, int block,
                        void *codes_dev, void *scales_dev, float *tensor_scale_dev, void *stream);

typedef struct sp24_nvfp4_gemm_args {
    int64_t M, N, K;          /* Y [M x N] = X [M x K] * W [N x K]^T           */
    sp24_tactic tactic;       /* SPARSE: W pairwise 4:8; DENSE: W dense NVFP4 */
    sp24_dtype out_dtype;     /* SP24_BF16 or SP24_F32                         */
    const void *X;            /* device, NVFP4 codes [M x K/2] (contiguous)    */
    const void *x_scales;     /* device, scale image of X: one code per 32
                                 positions (SPARSE) or per 16 (DENSE)          */
    const float *x_tensor_scale; /* device, 1 float                           */
    const void *W;            /* device; SPARSE: values [N x K/4]; DENSE: codes [N x K/2] */
    const void *W_meta;       /* device; SPARSE: 4:8 metadata image of W       */
    const void *w_scales;     /* device, scale image of W (per 32 / per 16)    */
    const float *w_tensor_scale; /* device, 1 float                           */
    void *Y;                  /* device, [M x N] row pitch ldy                 */
    int64_t ldy;
    void *workspace;          /* stream-K workspace (as sp24_gemm) or NULL     */
    size_t workspace_bytes;
    uint32_t flags;           /* SP24_GEMM_W_STATIC, SP24_GEMM_AFTER_INDEPENDENT */
} sp24_nvfp4_gemm_args;

/* Workspace of sp24_gemm_nvfp4's stream-K schedule (0 if none), with the
 * zero-fill rule of sp24_gemm_workspace_bytes. */
size_t sp24_gemm_nvfp4_workspace_bytes(const sp24_nvfp4_gemm_args *args);

/* Y = s_x * s_w * sum_k x[m,k] w[n,k] (block scales applied inside the
 * block-scaled tensor-core MMA, fp32 accumulation in tensor memory; tensor
 * scales in the epilogue).  SPARSE: tcgen05.mma.sp kind::mxf4nvf4 with the
 * 4:8 metadata; DENSE: the same kind, dense.  One persistent launch (128-row
 * weight tiles on single CTAs).  Requirements: K % 256 == 0, every pointer
 * 16-byte aligned, ldy * out bytes % 16 == 0. */
int sp24_gemm_nvfp4(const sp24_nvfp4_gemm_args *args, void *stream);

/* Up to 16 independent NVFP4 GEMMs in one launch (the decode regime, where
 * one launch per GEMM pays its ramp and tail every time): all problems share
 * the tactic (all 4:8 SPARSE or all DENSE) and the output type; each may have
 * its own M, N, K and buffers, and runs its own token-tile width inside the
 * widest problem's tile, with stream-K across problem boundaries as
 * sp24_gemm_grouped does.  Each args' own workspace fields are ignored: the
 * group uses `workspace` (size from sp24_gemm_nvfp4_grouped_workspace_bytes,
 * the zero-fill rule of sp24_gemm_workspace_bytes).  SP24_GEMM_W_STATIC and
 * SP24_GEMM_AFTER_INDEPENDENT apply when every problem sets them.  Errors:
 * SP24_ERR_INVALID_ARG for n outside 1..16 or mixed tactics,
 * SP24_ERR_DTYPE for mixed output types, and each problem's own checks. */
int sp24_gemm_nvfp4_grouped(const sp24_nvfp4_gemm_args *args, int n, void *workspace_dev, size_t workspace_bytes,
                            void *stream);
size_t sp24_gemm_nvfp4_grouped_workspace_bytes(const sp24_nvfp4_gemm_args *args, int n);

/* ---------------------------------------------------------------------- */
/* Tactic selection (kernel 5)                                             */
/* ---------------------------------------------------------------------- */

typedef struct sp24_tactic_record {
    double t_sparse_us;       /* median over iters (device time, CUDA events)   */
    double t_dense_us;
    double t_sparse_min_us;
    double t_dense_min_us;
    int32_t iters;
    int32_t eligible;         /* 1 if the sparse call passed eligibility         */
    int32_t selected;         /* sp24_tactic that the rule picked                */
    int32_t reserved;
    char reason[64];          /* why dense was chosen, "" if sparse was          */
} sp24_tactic_record;

/* Times the sparse call and the dense call of the same product on `stream`
 * with CUDA events (warmup untimed runs each, then iters timed runs each,
 * alternating), and selects SPARSE iff the sparse median is strictly below
 * the dense median; a tie or an ineligible sparse call selects DENSE
 * ("Sparse Tactic Audit": latency is the sole criterion; every fallback is
 * logged with its reason).  Synchronizes `stream`.  Both argument sets must
 * describe the same M, N, K and output buffer semantics.
 * Each timed call runs on a cold L2 (the library reads a buffer of twice the
 * L2 size before it; that buffer is allocated on the first call per device
 * and kept until exit), and the device is kept busy (a bounded spin kernel)
 * while the host enqueues the timed sequence, so host launch latency is not
 * timed. */
int sp24_select_tactic(const sp24_gemm_args *sparse_args, const sp24_gemm_args *dense_args,
                       int warmup, int iters, sp24_tactic_record *out, void *stream);

/* ---------------------------------------------------------------------- */
/* Status                                                                  */
/* ---------------------------------------------------------------------- */

const char *sp24_status_string(int status);

/* Reads (synchronously, on the current device) the device error word that a
 * bounded wait writes when it expires; SP24_OK if none.  Clears nothing. */
int sp24_last_device_error(void);

/* Clears the device error word of the current device (synchronous). */
int sp24_clear_device_error(void);

/* Upper bound, in nanoseconds of %globaltimer, of every device-side wait
 * (mbarrier waits in the GEMM).  Default 2 s.  Takes effect for launches
 * issued after the call. */
void sp24_set_wait_timeout_ns(uint64_t ns);

/* Launches a one-block kernel that waits (bounded by timeout_ns) on a
 * barrier that nothing completes, so that the bounded-wait path can be tested
 * without a fault.  Returns SP24_ERR_DEVICE_TIMEOUT when the wait expired as
 * designed (synchronizes the stream). */
int sp24_selftest_bounded_wait(uint64_t timeout_ns, void *stream);

/* Number of kernels this library has launched in this process. */
uint64_t sp24_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* SP24_H */
