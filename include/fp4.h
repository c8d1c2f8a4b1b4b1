/*
 * fp4.h -- C ABI of the B200 (sm_100a) fully-FP4 linear layer.
 *
 * The method follows three pages:
 *  [Q]   "Quartet: Native FP4 Training Can Be Optimal for Large Language
 *        Models" -- MXFP4 training (Hadamard-32 + QuEST forward, randomized
 *        Hadamard + SR(3/4) backward, clip-mask epilogue), Algorithm 1;
 *  [QII] "Quartet II: Accurate LLM Pre-Training in NVFP4 by Improved
 *        Unbiased Gradient Estimation" -- NVFP4 format and NVIDIA-style SR,
 *        Four-Over-Six, MS-EDEN (Algorithm 1) and its post hoc range
 *        alignment, the Quartet II computation graph;
 *  [BG]  "Bridging the Gap Between Promise and Performance for Microscaling
 *        FP4 Quantization" -- MXFP4 / NVFP4 formats, the MSE-optimal
 *        alternating scale search.
 *
 * Conventions for every call
 *  - All pointers named *_dev, and every pointer inside fp4_qtensor, are
 *    DEVICE pointers owned by the caller; the library allocates nothing and
 *    keeps no reference after the call returns.  Host pointers (structs
 *    passed by address) are read during the call only.
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *    default stream).  The returned int is a synchronous fp4_status for
 *    argument errors or launch failures.  Errors found on the device
 *    (non-finite input, bounded-wait timeout) are recorded in a device
 *    status word read (and cleared) by fp4_get_last_error().
 *  - Matrices are row-major.  A quantised tensor of shape rows x cols has
 *    its scale groups along cols (the GEMM's inner dimension).
 *  - FP4 codes: E2M1, 2 per byte, element 2j in bits 0-3 and element 2j+1
 *    in bits 4-7 of byte j of the row; code = sign << 3 | magnitude index of
 *    {0, 0.5, 1, 1.5, 2, 3, 4, 6}.
 *  - Linear scales: rows x (cols / g) bytes, row-major.  MXFP4: E8M0
 *    (2^(c-127)), g = 32.  NVFP4: E4M3, g = 16, times the fp32 tensor scale.
 *  - Swizzled scales (the tensor-core block-scale layout): 512-byte atoms
 *    covering 128 rows x 4 groups; byte (r, k) lives at
 *      ((r / 128) * nkb + k / 4) * 512 + (r % 32) * 16 + ((r % 128) / 32) * 4 + k % 4
 *    with nkb = ceil((cols / g) / 4); rows pad to 128 and groups to 4 with
 *    zeros.  Size: ceil(rows / 128) * nkb * 512 bytes.
 *  - QuEST clip mask: rows x (cols / 8) bytes, element 8b + j in bit j of
 *    byte b; 1 = the element was clipped.
 */
#ifndef FP4_B200_H
#define FP4_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *fp4_stream_t; /* == cudaStream_t */

enum fp4_status {
  FP4_OK = 0,
  FP4_ERR_INVALID_ARG = 1,      /* null pointer, bad size, bad enum value   */
  FP4_ERR_UNSUPPORTED = 2,      /* combination the pages do not define      */
  FP4_ERR_ALIGNMENT = 3,        /* pointer or dimension alignment violated  */
  FP4_ERR_WORKSPACE = 4,        /* workspace missing or too small           */
  FP4_ERR_CUDA = 5,             /* a CUDA runtime call or launch failed     */
  FP4_ERR_NONFINITE_INPUT = 6,  /* device: NaN or Inf seen in an input      */
  FP4_ERR_TIMEOUT = 7           /* device: a bounded wait gave up           */
};

enum fp4_format { FP4_MXFP4 = 0, FP4_NVFP4 = 1 };

enum fp4_rounding {
  FP4_RTN = 0,           /* AbsMax scale, round to nearest [Q]; [QII] Alg. 1 step 2 */
  FP4_QUEST = 1,         /* RMSE-optimal clipping + clip mask [Q] "QuEST in Detail" */
  FP4_FOUR_OVER_SIX = 2, /* NVFP4 only [QII] "Forward Pass Design"                  */
  FP4_SR = 3,            /* NVFP4: [QII] standard SR steps 1-3; MXFP4: SR(3/4 x) [Q] */
  FP4_MS_EDEN = 4,       /* NVFP4 only, needs a rotation [QII] MS-EDEN, post hoc     */
  FP4_RTN_SQUARE16 = 5   /* NVFP4 RTN, one scale per 16 x 16 block [QII] "The
                            square-block trade-off"; no rotation, rows a multiple
                            of 16, cols of 32; bf16 input only (not for
                            fp4_requantize); scales stored per 1 x 16 group, each
                            block's scale repeated on its 16 rows.  Quantising
                            x^T gives the transpose of quantising x.            */
};

/* Block Hadamard along the inner dimension [Q] "The Hadamard Transform".
 * block: 0 (none), 16, 32, 64, 128 or 256 (the sizes [BG] "Block-Wise
 * Hadamard Rotation" sweeps; 256 only for row-wise, non-transposed
 * quantisation).  randomized: 0 = H_g, 1 = H_g diag(d)
 * with d_j = +-1 drawn from Philox(seed, counter (j/4, 0, 3, sign_tag)), one
 * pattern for every block of the tensor; two operands of one GEMM must use
 * the same seed and sign_tag so the rotations cancel [QII] MS-EDEN step 1. */
typedef struct {
  int32_t block;
  int32_t randomized;
  uint32_t sign_tag;
} fp4_had;

/* Every pointer in fp4_qtensor except tensor_scale (4 bytes) must be 16-byte
 * aligned; otherwise the calls return FP4_ERR_ALIGNMENT. */
typedef struct {
  uint8_t *codes;      /* rows x cols/2, required                              */
  uint8_t *scales;     /* rows x cols/g linear; may be NULL if scales_swz set  */
  uint8_t *scales_swz; /* tensor-core layout; may be NULL if scales set        */
  float *tensor_scale; /* 1 float: NVFP4 fp32 scale; MXFP4 1.0 (4/3 for SR)    */
  uint8_t *mask;       /* rows x cols/8, QuEST only (else NULL)                */
  int64_t rows;        /* shape of the QUANTISED tensor                        */
  int64_t cols;
  int32_t fmt;         /* fp4_format                                           */
  int32_t reserved;
} fp4_qtensor;

/* Bytes of device workspace fp4_quantize / fp4_requantize need for a
 * quantised tensor of rows x cols (16-byte multiple; 0 for modes without a
 * global pass).  NVFP4 RTN/QuEST/4-6/SR: one amax word.  MS-EDEN: amax, the
 * bf16 E8M3 pseudo-scales (rows * cols/16 * 2) and the fp32 EDEN factors
 * (rows * cols/block * 4) of the post hoc range alignment [QII].  Square
 * blocks: amax and the fp32 maxima of the 16 x 16 blocks (rows/16 * cols/16
 * * 4 at byte 256).  MS-EDEN layout:
 * the amax bits (uint32) at byte 0; the pseudo-scales, row-major, at byte
 * 256; the EDEN factors, row-major, at byte 256 + the pseudo-scale bytes
 * rounded up to a multiple of 256.  After an MS-EDEN call the workspace
 * still holds these first-pass results. */
size_t fp4_quantize_workspace_size(int64_t rows, int64_t cols, int32_t fmt,
                                   int32_t rounding, int32_t had_block);

/* De-quantise a quantised tensor: D[r][c] = fp32(fp32(q * s_group) * s_tensor)
 * for the E2M1 value q of element (r, c), its group's scale s_group (E4M3 for
 * NVFP4, 2^(e-127) for MXFP4, from the LINEAR scales) and the tensor scale --
 * the dequantised value x_FP4 * x_FP8 * x_FP32 of [QII] "NVFP4 Format and
 * Standard Stochastic Rounding", rounded as the backward re-quantisation
 * reads a saved tensor ([QII] "The Complete Quartet II Computation Graph").
 * D_dev: rows x cols row-major, fp32 (out_dtype 0) or bf16 rounded to nearest
 * even (1), caller-owned, 16-byte aligned.  in: codes (16-byte aligned),
 * scales and tensor_scale required.  Asynchronous on `stream`; an empty tensor
 * launches nothing.  Errors: FP4_ERR_INVALID_ARG (null pointers, format,
 * out_dtype, cols not a multiple of the group), FP4_ERR_ALIGNMENT. */
int fp4_dequantize(const fp4_qtensor *in, void *D_dev, int32_t out_dtype, fp4_stream_t stream);

/* Transpose of a quantised tensor with 16 x 16 square-block scales
 * (FP4_RTN_SQUARE16): out = in^T, codes transposed and each block's scale
 * moved to the transposed block -- equal to quantising the transposed input
 * directly, which is how the NVIDIA recipe re-uses Q(W) for W^T ([QII] "The
 * square-block trade-off").  in: NVFP4, rows and cols multiples of 64 and
 * 16, codes, linear scales and tensor scale (device).  out: caller-owned,
 * codes (cols x rows/2), scales and/or scales_swz, tensor_scale; the call
 * writes rows, cols, fmt.  The result is the transpose only when `in` has
 * square-block scales.  Errors: FP4_ERR_INVALID_ARG, FP4_ERR_ALIGNMENT. */
int fp4_transpose_square16(const fp4_qtensor *in, fp4_qtensor *out, fp4_stream_t stream);

/* NVFP4 quantisation with MSE-optimal scales by alternating optimisation
 * ([BG] "MSE-Optimized Grid and Scale Selection", NVFP4 without rotation).
 *  1. s_T = amax / (6 * 256), the RTN tensor scale (1 for an all-zero x).
 *  2. Group step: each 16-element group takes the E4M3 scale code c in
 *     1..126 whose RTN codes of x * fp32(1 / d), d = fp32(E4M3(c) * s_T),
 *     give the smallest fp32 squared error (pairwise tree of
 *     fp32((x - fp32(q d))^2)); ties keep the larger c; a group whose
 *     maximum is zero takes c = 0 and zero codes.
 *  3. `iters` times: the tensor-scale step s_T = fp32(<x, u> / <u, u>) with
 *     u = E4M3(c_group) * q, the closed-form least-squares tensor scale for
 *     the codes held (both sums float64 pairwise trees over the row-major
 *     element order; s_T is kept when a sum is not positive or the quotient
 *     is not a finite positive fp32 value), then the group step again.
 * The squared error does not grow with `iters`.  x_dev: bf16 rows x cols,
 * row-major, 16-byte aligned; cols a multiple of 32.  iters: 0..64.  out:
 * as for fp4_quantize (codes, scales and/or scales_swz, tensor_scale = the
 * final s_T; mask unused); the call writes rows, cols and fmt = NVFP4.
 * ws_dev: fp4_quantize_mse_workspace_size bytes, 16-byte aligned: the amax
 * word at byte 0, then one float64 pair per 8192 elements at byte 256.
 * Launches 2 + 2 * iters kernels (plus one when the swizzled scales need
 * padding).  A non-finite input sets FP4_ERR_NONFINITE_INPUT on the device.
 * Errors: FP4_ERR_INVALID_ARG (shape, iters, null pointers),
 * FP4_ERR_ALIGNMENT, FP4_ERR_WORKSPACE, FP4_ERR_CUDA (a launch failed).
 * fp4_quantize_mse_workspace_size returns 0 for an invalid shape. */
size_t fp4_quantize_mse_workspace_size(int64_t rows, int64_t cols);
int fp4_quantize_mse(const void *x_dev, int64_t rows, int64_t cols, int32_t iters,
                     fp4_qtensor *out, void *ws_dev, size_t ws_bytes, fp4_stream_t stream);

/* Bytes of the swizzled scale buffer for rows x n_groups scales. */
size_t fp4_swizzled_scale_bytes(int64_t rows, int64_t n_groups);

/* Dense orthonormal block transforms of the forward pass, [BG] appendix on
 * linear transforms (Tables 13-14: Hadamard, DCT, DST and GSR at block sizes
 * 16 to 256).  GSR is named but not defined by the pages and has no value
 * here.
 *   FP4_XFORM_DCT2: C[i][j] = f_i cos(pi (2j+1) i / (2k)), f_0 = sqrt(1/k),
 *                   f_i = sqrt(2/k) (orthonormal DCT-II);
 *   FP4_XFORM_DST2: S[i][j] = g_i sin(pi (2j+1)(i+1) / (2k)),
 *                   g_{k-1} = sqrt(1/k), g_i = sqrt(2/k) (orthonormal DST-II).
 * fp4_block_transform: y = M x for every k-block of every row of x, k =
 * `block` in {16, 32, 64, 128, 256}.  x_dev: rows x cols bf16 row-major,
 * y_dev: rows x cols fp32, both 16-byte aligned, caller-owned; cols a
 * multiple of block, cols / block <= 65535.  y_i is the pairwise tree (level
 * 0 adds j = 2m and 2m + 1) of the fp32 products fp32(M[i][j] x_j), every
 * product and sum rounded to fp32; M's entries are fp64 values rounded once
 * to fp32 (the cosine of the reduced angle pi m / (2k), m in [0, k], times
 * the normalisation).  ws_dev: fp4_block_transform_workspace_size(block)
 * bytes (the k x k fp32 matrix, rebuilt by each call), 16-byte aligned.
 * Asynchronous on `stream`; 2 launches; an empty tensor launches nothing.
 * Errors: FP4_ERR_UNSUPPORTED (kind, block), FP4_ERR_INVALID_ARG (shape,
 * null pointers), FP4_ERR_ALIGNMENT, FP4_ERR_WORKSPACE, FP4_ERR_CUDA.  The
 * workspace query returns 0 for an unsupported block. */
enum fp4_transform_kind { FP4_XFORM_DCT2 = 1, FP4_XFORM_DST2 = 2 };
size_t fp4_block_transform_workspace_size(int32_t block);
int fp4_block_transform(const void *x_dev, float *y_dev, int64_t rows, int64_t cols, int32_t kind,
                        int32_t block, void *ws_dev, size_t ws_bytes, fp4_stream_t stream);

/* Quantise an fp32 matrix that is already transformed (e.g. the output of
 * fp4_block_transform): fp4_quantize's rules with no rotation and no
 * transpose.  y_dev: rows x cols fp32 row-major, 16-byte aligned, cols a
 * multiple of 32.  rounding: RTN, QuEST, Four-Over-Six (NVFP4) or SR;
 * MS-EDEN (its S lives on its own rotation blocks) and square blocks (bf16
 * block maxima) return FP4_ERR_UNSUPPORTED.  out, seed, tensor_tag and the
 * workspace (fp4_quantize_workspace_size(rows, cols, fmt, rounding, 0)) as
 * for fp4_quantize. */
int fp4_quantize_f32(const float *y_dev, int64_t rows, int64_t cols, int32_t fmt, int32_t rounding,
                     int32_t group, uint64_t seed, uint32_t tensor_tag, fp4_qtensor *out,
                     void *ws_dev, size_t ws_bytes, fp4_stream_t stream);

/* MXFP4 with fitted scales (MXFP4-dagger), [BG] "MXFP Scale Fitting"
 * (Appendix H, Table 11): the 8-bit scale of a 32-element group is a level q
 * in [0, 255] standing for 2^(alpha q + L_min), L_min / L_max = log2 of the
 * smallest / largest AbsMax group scale s = fp32(gmax / 6) of the tensor (over
 * groups with s > 0), alpha = (L_max - L_min) / 255 (the page's fractional
 * exponent step).  A group's level is the number of boundaries
 * fp32(2^(L_min + alpha (k + 0.5))), k = 0..254, not above s; its elements
 * are RTN_E2M1(x * fp32(1/d)), d = table[q] = fp32(2^(L_min + alpha q)),
 * saturating at 6.  Exponents are fp64 (log2 / exp2 of CUDA's math library,
 * each add and multiply rounded on its own), rounded once to fp32.  A group
 * with s = 0 (or a non-finite reciprocal scale) gets level 0 and zero codes;
 * with no s > 0 the table is all 1.  The scales are not powers of two, so the
 * tensor cores' E8M0 block scaling cannot apply them: there is no GEMM for
 * this format, only quantisation and de-quantisation (the page's accuracy
 * use).
 * fp4_quantize_mx_fit: x_dev bf16 rows x cols row-major (16-byte aligned),
 * cols a multiple of 32 and of had_block; had_block in {0, 16, ..., 256}: the
 * deterministic block Hadamard applied first (fp4_hadamard's transform).
 * codes_dev rows x cols/2 (16-byte aligned), levels_dev rows x cols/32,
 * table_dev 256 fp32: caller-owned outputs.  ws_dev:
 * fp4_quantize_mx_fit_workspace_size() bytes, 16-byte aligned.  3 launches
 * (+2 memsets); an empty tensor writes the all-1 table only.  A non-finite
 * input sets FP4_ERR_NONFINITE_INPUT on the device.
 * fp4_dequantize_mx_fit: out_dev[r][c] = fp32(E2M1(code) * table[level]),
 * rows x cols fp32, 16-byte aligned.
 * Errors: FP4_ERR_UNSUPPORTED (had_block), FP4_ERR_INVALID_ARG (shape, null
 * pointers), FP4_ERR_ALIGNMENT, FP4_ERR_WORKSPACE, FP4_ERR_CUDA. */
size_t fp4_quantize_mx_fit_workspace_size(void);
int fp4_quantize_mx_fit(const void *x_dev, int64_t rows, int64_t cols, int32_t had_block,
                        uint8_t *codes_dev, uint8_t *levels_dev, float *table_dev,
                        void *ws_dev, size_t ws_bytes, fp4_stream_t stream);
int fp4_dequantize_mx_fit(const uint8_t *codes_dev, const uint8_t *levels_dev, const float *table_dev,
                          int64_t rows, int64_t cols, float *out_dev, fp4_stream_t stream);

/* y = block (randomized) Hadamard of x along cols, fp32 out.
 * x_dev: rows x cols bf16; y_dev: rows x cols fp32; cols % block == 0.
 * [Q] "The Hadamard Transform": Sylvester order, 1/sqrt(g) normalisation. */
int fp4_hadamard(const void *x_dev, float *y_dev, int64_t rows, int64_t cols,
                 fp4_had had, uint64_t seed, fp4_stream_t stream);

/* Quantise a bf16 matrix.  x_dev is in_rows x in_cols; with transpose = 0 the
 * quantised tensor is x (rows = in_rows, cols = in_cols), with transpose = 1
 * it is x^T (rows = in_cols, cols = in_rows), i.e. the groups and the
 * rotation run along x's rows -- the backward operands of [QII] "The
 * Complete Quartet II Computation Graph".  group must equal the format's
 * group size (16 NVFP4, 32 MXFP4).  cols must be a multiple of
 * max(group, had.block); with transpose = 1, in_cols must be a multiple of 8
 * (FP4_ERR_ALIGNMENT otherwise).
 * seed/tensor_tag key the Philox streams of SR (element index in the output
 * layout) and MS-EDEN (group index).  out: caller fills the pointers; the
 * call writes rows, cols and fmt.  ws_dev: fp4_quantize_workspace_size bytes,
 * 16-byte aligned, contents need not be initialised. */
int fp4_quantize(const void *x_dev, int64_t in_rows, int64_t in_cols,
                 int32_t transpose, int32_t fmt, int32_t rounding, int32_t group,
                 fp4_had had, uint64_t seed, uint32_t tensor_tag,
                 fp4_qtensor *out, void *ws_dev, size_t ws_bytes,
                 fp4_stream_t stream);

/* fp4_quantize without a caller-provided workspace.  (This entry point has
 * no counterpart in the papers; it exists for library users.)
 *
 * Some callers cannot allocate device memory at the moment they quantise: a
 * host framework or serving engine that owns every byte of device memory and
 * hands none out after start-up, a plugin that is given only its inputs and
 * outputs, or a latency-critical loop where a cudaMalloc (which may
 * synchronise the device) is not acceptable.  This call needs no workspace:
 * the scratch that the global-amax and MS-EDEN modes need (amax word,
 * pseudo-scales, EDEN factors) lives in a fixed device array of
 * FP4_NOALLOC_SCRATCH_BYTES inside the library, which every GPU that loads
 * the library holds until the process exits.  The call allocates and frees
 * nothing (no cudaMalloc, no library allocator); the caller still provides x
 * and every output buffer of `out`, exactly as for fp4_quantize, and the
 * results are bit-identical to fp4_quantize's.
 *  - Limit: a quantised tensor whose fp4_quantize_workspace_size exceeds
 *    FP4_NOALLOC_SCRATCH_BYTES (4 MiB) returns FP4_ERR_WORKSPACE and launches
 *    nothing.  That is about 26.8 million elements for MS-EDEN with 128-blocks
 *    (16.7 million with 32-blocks, 11.1 million with 16-blocks) and about 268
 *    million for FP4_RTN_SQUARE16 (256 + rows * cols / 64 bytes: one fp32
 *    maximum per 16 x 16 block); the other NVFP4 modes (256 bytes) and all
 *    MXFP4 modes (none) fit at any size.  An invalid argument returns the
 *    same status as fp4_quantize, whatever the size.
 *  - All calls share the one array and it keeps the last call's contents; the
 *    part that must start at zero (the amax word) is cleared on `stream`
 *    inside the call.  Two calls whose work overlaps on the GPU (different
 *    streams, or different host threads on one device) race on the array and
 *    give wrong results: serialise them.
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current; make that first call
 *    before any stream capture. */
#define FP4_NOALLOC_SCRATCH_BYTES (4u << 20)
int fp4_quantize_noalloc(const void *x_dev, int64_t in_rows, int64_t in_cols,
                         int32_t transpose, int32_t fmt, int32_t rounding, int32_t group,
                         fp4_had had, uint64_t seed, uint32_t tensor_tag,
                         fp4_qtensor *out, fp4_stream_t stream);

/* Re-quantise a saved FP4 tensor [QII] computation graph backward steps 1-4:
 * de-quantise (fp32(fp32(q * s_group) * s_tensor)), optionally transpose,
 * rotate along the new inner dimension, quantise in `in->fmt` with
 * `rounding`.  in->scales (linear) is required. */
int fp4_requantize(const fp4_qtensor *in, int32_t transpose, int32_t rounding,
                   fp4_had had, uint64_t seed, uint32_t tensor_tag,
                   fp4_qtensor *out, void *ws_dev, size_t ws_bytes,
                   fp4_stream_t stream);

/* Linear (rows x n_groups) scales -> the swizzled tensor-core layout
 * (padding zeroed).  [Q] "Stage 2", scale factor layout. */
int fp4_swizzle_scales(const uint8_t *scales_dev, int64_t rows, int64_t n_groups,
                       uint8_t *scales_swz_dev, fp4_stream_t stream);

/* Block-scaled FP4 GEMM on the tcgen05 tensor cores [Q] "Stage 2":
 *   D = (A . SFA) (B . SFB)^T * (tA * tB)
 * A: M x K quantised tensor (A->rows = M, A->cols = K), B: N x K (B->rows = N),
 * same format; both K-major with swizzled scales (scales_swz required).
 * D_dev: M x N row-major, fp32 (out_dtype 0) or bf16 (out_dtype 1, rounded
 * to nearest even), FP32 accumulation.  K % 64 == 0, N % 8 == 0.
 * epi_inverse_had = 32 applies the Quartet backward epilogue
 * [Q] "Inverse Hadamard and clipping mask correction": every 32-column block
 * of the scaled product is multiplied by (1 - mask) (mask: M x N/8 bytes,
 * 1 = clipped in the forward pass; NULL = no mask) and then by H32^-1 = H32;
 * requires N % 32 == 0.  The 16/9 factor is the product of the operands'
 * tensor scales (4/3 each).  epi_inverse_had = 0 and a mask is an error. */
int fp4_gemm(const fp4_qtensor *A, const fp4_qtensor *B, void *D_dev, int32_t out_dtype,
             const uint8_t *epi_mask_dev, int32_t epi_inverse_had, fp4_stream_t stream);

/* ------------------------------------------------------- linear layer --
 * Y = X W^T forward and dX = dY W, dW = dY^T X backward, fully in FP4.
 * X: M x K bf16, W: N x K bf16, dY: M x N bf16 (row-major, device).
 *  FP4_RECIPE_QUARTET  [Q] Algorithm 1: MXFP4; forward H32 + QuEST (clip
 *      masks saved); backward RHT32 + SR(3/4) on dY / dY^T / W_q^T / X_q^T,
 *      epilogue 16/9 H32^-1( . (.) (1 - mask)).
 *  FP4_RECIPE_QUARTET2 [QII] computation graph: NVFP4; forward RTN +
 *      Four-Over-Six, no rotation; backward de-quantise, transpose, RHT128 on
 *      the inner dimension, MS-EDEN; no inverse transform.
 *  FP4_RECIPE_RTN      NVFP4 RTN on every operand, no rotation.
 *  FP4_RECIPE_TETRAJET2 the simplified (GPU-feasible) TetraJet-v2 the [QII]
 *      page compares against ("Comparison to TetraJet-v2 and the NVIDIA
 *      recipe"): NVFP4; forward RTN with native 1x16 scales, no rotation;
 *      backward de-quantise, transpose, RHT128 on the inner dimension and
 *      element-wise SR (the same graph as FP4_RECIPE_QUARTET2 with SR in
 *      place of MS-EDEN).
 *  FP4_RECIPE_NVIDIA   the NVIDIA recipe [QII] describes ("The square-block
 *      trade-off"): NVFP4; forward X with 1x16 RTN, W with 16x16
 *      square-block RTN, no rotation; backward SR; the dX GEMM re-uses the
 *      forward Q(W) transposed (fp4_transpose_square16) against SR(dY) without
 *      a rotation; the dW GEMM uses the 16-point RHT on dY^T and on the
 *      re-quantised X^T.
 * Seeds: every random draw of one backward step is keyed by step_seed; the
 * dX GEMM's operands share sign tag 0, the dW GEMM's sign tag 1; SR tensor
 * tags 1 (dY), 2 (W_q^T), 3 (dY^T), 4 (X_q^T); forward tags 5 (X), 6 (W). */
enum fp4_recipe_id {
  FP4_RECIPE_QUARTET = 0,
  FP4_RECIPE_QUARTET2 = 1,
  FP4_RECIPE_RTN = 2,
  FP4_RECIPE_TETRAJET2 = 3,
  FP4_RECIPE_NVIDIA = 4
};

typedef struct {
  int32_t fmt;            /* fp4_format of every operand                     */
  int32_t fwd_rounding;   /* fp4_rounding of X and W                         */
  int32_t fwd_had;        /* deterministic H block on K (0 = none)           */
  int32_t bwd_rounding;   /* fp4_rounding of the four backward operands      */
  int32_t bwd_had;        /* rotation block on each GEMM's inner dimension   */
  int32_t bwd_randomized; /* 1: RHT (random signs), 0: H                     */
  int32_t mask_epilogue;  /* 1: Quartet mask + H^-1 epilogue (fwd QuEST)     */
  int32_t out_y, out_dx, out_dw; /* 0 fp32, 1 bf16                           */
  int32_t w_rounding;     /* fp4_rounding of W in the forward pass, or -1 for
                             fwd_rounding (FP4_RTN_SQUARE16: square blocks)   */
  int32_t w_reuse;        /* 1: the dX GEMM multiplies by the forward Q(W),
                             transposed (needs w_rounding FP4_RTN_SQUARE16),
                             and dY is quantised for it without a rotation    */
} fp4_recipe;

/* Fill *r with a preset; returns FP4_ERR_INVALID_ARG for an unknown id. */
int fp4_recipe_preset(int32_t id, fp4_recipe *r);

/* Saved context of the forward pass, in caller-owned device memory:
 * xq is M x K (codes, linear scales, swizzled scales, tensor scale, and the
 * clip mask when the forward rounding is QuEST), wq is N x K likewise.
 * Sizes: codes rows*cols/2, scales rows*cols/g, swizzled
 * fp4_swizzled_scale_bytes(rows, cols/g), mask rows*cols/8, 4 bytes of scale. */
typedef struct {
  fp4_qtensor xq;
  fp4_qtensor wq;
} fp4_ctx;

/* Device workspace bytes of fp4_linear_fwd (is_bwd = 0) or fp4_linear_bwd
 * (is_bwd = 1): the quantiser scratch and, for the backward, the four
 * re-quantised operands. */
size_t fp4_linear_workspace_size(const fp4_recipe *r, int64_t M, int64_t N, int64_t K,
                                 int32_t is_bwd);

/* Forward: quantise X and W into ctx, Y_dev (M x N, r->out_y) = GEMM. */
int fp4_linear_fwd(const void *X_dev, const void *W_dev, int64_t M, int64_t N, int64_t K,
                   const fp4_recipe *r, uint64_t seed, void *Y_dev, fp4_ctx *ctx,
                   void *ws_dev, size_t ws_bytes, fp4_stream_t stream);

/* Backward: dX_dev (M x K, r->out_dx) and dW_dev (N x K, r->out_dw) from
 * dY and the saved context.  Either output may be NULL to skip its GEMM. */
int fp4_linear_bwd(const void *dY_dev, const fp4_ctx *ctx, int64_t M, int64_t N, int64_t K,
                   const fp4_recipe *r, uint64_t step_seed, void *dX_dev, void *dW_dev,
                   void *ws_dev, size_t ws_bytes, fp4_stream_t stream);

/* Read and clear the device status word after synchronising `stream`.
 * Returns FP4_OK or the first device-side fp4_status recorded. */
int fp4_get_last_error(fp4_stream_t stream);

/* Number of CUDA kernels this library has launched since it was loaded
 * (host-side counter, all devices and streams; no synchronisation). */
unsigned long long fp4_launch_count(void);

/* Device self-check of the E2M1 conversions: compares the hardware encoder
 * used by the quantisers with the per-element round-to-nearest-even rounding
 * over all 2^32 fp32 bit patterns (NaNs excluded), and the hardware decoder
 * (E2M1 pair -> f16x2 -> fp32) with the code table over all 256 code pairs.
 * ADDS the number of mismatching encoded words plus mismatching decoded
 * values to *mismatches_dev (caller zeroes it). */
int fp4_selftest_e2m1(unsigned long long *mismatches_dev, fp4_stream_t stream);

/* Device self-check of the exact shortcuts in the NVFP4 scale arithmetic
 * against CUDA's correctly rounded division and reciprocal and the E4M3
 * rounding.  ADDS mismatch counts to mismatches_dev[0..5] (6 counters, the
 * caller zeroes them): [0] the corrected division by 6 over every
 * non-negative finite fp32 dividend, [1] the reciprocal of every
 * non-negative E8M3 value, [2] the corrected division by a per-tensor
 * divisor on 2^32 hashed dividend/divisor pairs, [3] the hardware E4M3
 * decoder over every non-NaN code, [4] the hardware E4M3 encoder over every
 * non-negative finite fp32 value, [5] the MS-EDEN pseudo-scale rounding
 * E8M3(g / 6) taken from the product with fp32(1/6) over every non-negative
 * finite fp32 g and +inf. */
int fp4_selftest_arith(unsigned long long *mismatches_dev, fp4_stream_t stream);

/* Static description of a status code. */
const char *fp4_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* FP4_B200_H */
