/*
 * nvfp4.h -- C ABI of the B200 (sm_100a) NVFP4 quantised linear-layer library.
 *
 * The operation: the NVFP4 linear layer of 4-bit LLM pretraining, as described
 * on the page "Preentrenamiento de 4 bits con NVFP4 en un hibrido
 * Mamba-Transformer de 12B (10T tokens)" (NVIDIA method summary):
 *   - format passage: 4-bit E2M1 elements in blocks of 16, one E4M3 scale per
 *     block and one extra FP32 scale per tensor;
 *   - scope passage: NVFP4 is used only inside the GEMMs of linear layers;
 *   - recipe passage: 16x16 random Hadamard transforms on the weight-gradient
 *     operands, two-dimensional (16x16) block scaling for weights, stochastic
 *     rounding on gradients only;
 *   - performance passage: FP4 GEMMs run at twice FP8's rate and halve the
 *     operand memory.
 *
 * Conventions for every call
 *   - Pointers named "device" point to GPU global memory of the current device;
 *     everything else (structs, option blocks) is host memory read during the call.
 *   - The caller owns every buffer and the stream.  The library allocates no
 *     memory; calls that need scratch take a caller-supplied workspace.
 *   - Calls enqueue work on `stream` (a cudaStream_t passed as void*; NULL is the
 *     legacy default stream) and return without synchronising.  Stream order holds
 *     as usual: the GEMMs and the quantiser's second pass are launched as
 *     programmatic dependents of the kernel before them, so their set-up overlaps
 *     that kernel's last thread blocks, but each waits for it to complete before
 *     touching memory; the one exception, the second pass streaming its input
 *     early, reads a tensor that its own first pass only reads.  Every call may be
 *     captured into a CUDA graph.
 *   - Argument errors are reported synchronously by the return value, before
 *     anything is launched.  Device-side errors (a bounded wait that gave up)
 *     are reported by nvfp4_get_status().  No exception crosses the ABI.
 *   - nvfp4_last_error_string() describes the last non-OK status of the calling
 *     thread.
 *
 * Stored format (every nvfp4_tensor)
 *   - A logical [rows x cols] tensor blocked along cols (the contiguous axis).
 *   - codes: [rows][cols/2] bytes, two 4-bit E2M1 codes per byte, the element
 *     with the even column index in the low nibble.  Code = sign << 3 | index,
 *     index into the magnitudes {0, 0.5, 1, 1.5, 2, 3, 4, 6}.
 *   - scales: one unsigned E4M3 byte per 16-element block, in one of two layouts:
 *       NVFP4_SCALE_ROWMAJOR: [rows][cols/16], byte (r, j) at r*(cols/16) + j;
 *       NVFP4_SCALE_MMA: tiles of 128 rows x 4 block-columns (512 bytes); tile
 *         (r/128, j/4) at ((r/128) * ceil(cols/64) + j/4) * 512, and inside the
 *         tile byte (r%32)*16 + ((r%128)/32)*4 + j%4.  This is the order in
 *         which the tensor cores read block scales; nvfp4_gemm requires it.
 *   - tensor_scale: one FP32 decode scale S on the device.  The value of element
 *     (r, c) is E2M1(code) * E4M3(scale) * S.
 *   - A "col" layout of an [R x C] tensor is the [C x R] tensor of its transpose,
 *     blocked along R.
 */
#ifndef NVFP4_H
#define NVFP4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  NVFP4_OK = 0,
  NVFP4_ERR_INVALID_ARG = 1,       /* NULL where a buffer is needed, bad enum, bad option mix */
  NVFP4_ERR_UNSUPPORTED_SHAPE = 2, /* shape outside the documented multiples */
  NVFP4_ERR_MISALIGNED = 3,        /* pointer or leading dimension breaks 16-byte alignment */
  NVFP4_ERR_CUDA = 4,              /* a CUDA runtime call failed (launch, attribute, ...) */
  NVFP4_ERR_TIMEOUT = 5,           /* a device-side bounded wait gave up (nvfp4_get_status) */
  NVFP4_ERR_WORKSPACE = 6          /* workspace missing or smaller than nvfp4_workspace_size() */
} nvfp4_status;

enum { NVFP4_SCALE_ROWMAJOR = 0, NVFP4_SCALE_MMA = 1 };
enum { NVFP4_OUT_BF16 = 0, NVFP4_OUT_F32 = 1 };

/* One NVFP4 tensor: see "Stored format" above.  All three buffers are device
 * memory owned by the caller; sizes: codes rows*cols/2 bytes, scales
 * nvfp4_scales_bytes(rows, cols, scale_layout) bytes, tensor_scale 4 bytes.
 * An empty tensor (rows or cols 0) may leave codes and scales NULL. */
typedef struct {
  uint8_t* codes;
  uint8_t* scales;
  float* tensor_scale;
  int64_t rows;
  int64_t cols;
  int32_t scale_layout; /* NVFP4_SCALE_ROWMAJOR or NVFP4_SCALE_MMA */
  int32_t reserved;     /* must be 0 */
} nvfp4_tensor;

/* Quantiser options (recipe passage of the 12B NVFP4 page).
 *   stochastic : stochastic rounding of the elements of every emitted layout
 *                (gradients); otherwise round-to-nearest-even.  Element i of a
 *                layout (its linear index in the stored [rows x cols] order)
 *                draws a 16-bit random integer n from Philox4x32-10 with key
 *                (seed lo32, seed hi32):
 *                  g = i / 4 (groups of four consecutive elements), and group g
 *                  takes 32-bit word w = word g % 4 of the call with counter
 *                  (g/4 lo32, g/4 hi32, tag, offset), tag 0 for the row layout
 *                  and 1 for the col layout (one call per 16 elements);
 *                  with e = i % 4:  n(e=0) = w[23:16] * 256 + w[7:0],
 *                  n(e=1) = the 16-bit bit reversal of n(e=0),
 *                  n(e=2) = w[31:24] * 256 + w[15:8],
 *                  n(e=3) = the 16-bit bit reversal of n(e=2).
 *                With lo <= |y| < hi the neighbouring magnitudes of the scaled
 *                element y and f = (|y| - lo) / (hi - lo), the element rounds up
 *                iff floor(f * 2^16) + n >= 2^16; |y| >= 6 gives 6, the sign is
 *                kept.  The expected rounding error is below 2^-16 of a grid step
 *                (a slight bias towards lo, from the floor).
 *   rht_row    : 16x16 random Hadamard transform along the blocks of the row layout.
 *   rht_col    : the same along the blocks of the col layout (the token axis of
 *                the weight-gradient operands).
 *   block_2d   : one scale per 16x16 tile (weights); the row and col layouts then
 *                hold the same codes and scales, transposed.  Excludes stochastic
 *                and both RHT flags.
 *   seed       : Philox key.
 *   offset     : Philox counter word 3; must be < 2^32.
 *   rht_signs  : low 16 bits; bit j set negates element j of every 16-group
 *                before the transform.  Use the same value for both wgrad operands.
 *   amax_in    : NULL, or 3 device floats {raw amax, amax of the transformed col
 *                layout, amax of the transformed row layout} that replace the
 *                amax pass (delayed or externally fused scaling).
 *   amax_out   : NULL, or 3 device floats receiving the maxima used.
 * The tensor scale of a layout is S = amax / (6 * 448) (S = 1 when amax = 0),
 * with amax taken over the values that layout encodes (after its transform). */
typedef struct {
  int32_t stochastic;
  int32_t rht_row;
  int32_t rht_col;
  int32_t block_2d;
  uint64_t seed;
  uint64_t offset;
  uint32_t rht_signs;
  uint32_t reserved; /* must be 0 */
  const float* amax_in;
  float* amax_out;
} nvfp4_quant_opts;

/* Library version, major*10000 + minor*100 + patch. */
int nvfp4_version(void);

/* Bytes of caller workspace that nvfp4_quantize and the linear calls need
 * (device memory, 16-byte aligned; its contents need not be initialised). */
size_t nvfp4_workspace_size(void);

/* Bytes of the scale buffer of an NVFP4 tensor of logical shape [rows x cols]
 * in the given layout (the MMA layout pads rows to 128 and cols/16 to 4). */
size_t nvfp4_scales_bytes(int64_t rows, int64_t cols, int32_t scale_layout);

/* Quantise a BF16 tensor x [rows x cols] (device, row stride ld elements) to
 * NVFP4 (format and recipe passages of the 12B NVFP4 page).
 *   out_row : NULL, or the row layout, rows x cols (blocks along cols).
 *   out_col : NULL, or the col layout, cols x rows (blocks along rows).
 * At least one output.  Requires cols % 16 == 0; rows % 16 == 0 when out_col is
 * given or block_2d is set; x and ld*2 bytes 16-byte aligned; codes buffers
 * 16-byte aligned.  Work: one amax pass over x (skipped when amax_in is given)
 * and one quantise pass writing every requested layout and its tensor scale. */
nvfp4_status nvfp4_quantize(const void* x, int64_t rows, int64_t cols, int64_t ld,
                            const nvfp4_quant_opts* opts, nvfp4_tensor* out_row,
                            nvfp4_tensor* out_col, void* workspace, size_t workspace_bytes,
                            void* stream);

/* Dequantise q into out [rows x cols] (device, row stride ldo elements):
 * out = E2M1(code) * E4M3(scale) * S, rounded to BF16 (nearest even) or kept
 * in FP32.  Requires cols % 16 == 0 and 16-byte aligned out rows. */
nvfp4_status nvfp4_dequantize(const nvfp4_tensor* q, void* out, int64_t ldo, int32_t out_dtype,
                              void* stream);

/* Block-scaled NVFP4 GEMM on the sm_100a tensor cores (performance passage of
 * the 12B NVFP4 page; FP32 accumulation per the error-accumulation remark of
 * "Full-Stack FP4: Preentrenamiento Estable de LLM"):
 *   C[m][n] = alpha * S_A * S_B * sum_k A[m][k] * B[n][k]   (+ C[m][n] if accumulate)
 * with A [M x K] and B [N x K] NVFP4 tensors blocked along K (MMA scale layout),
 * C [M x N] device memory with row stride ldc elements, BF16 (nearest even) or FP32.
 * Requires M % 128 == 0, N % 128 == 0, K % 64 == 0, 16-byte aligned C rows. */
nvfp4_status nvfp4_gemm(const nvfp4_tensor* A, const nvfp4_tensor* B, void* C, int64_t ldc,
                        int32_t out_dtype, float alpha, int32_t accumulate, void* stream);

/* nvfp4_gemm with BF16 output that also reports, from its epilogue, the maxima the
 * next quantisation of C needs, so that quantisation can skip its amax pass (pass
 * amax_out as its nvfp4_quant_opts.amax_in).  The tensor scales of the format
 * passage of the 12B NVFP4 page come from these maxima; the page's recipe applies
 * the 16x16 random Hadamard transform to the weight-gradient operands, which for an
 * output that becomes the next linear's activations is its col layout.
 *   amax_out : 3 device floats, written by this call (stream-ordered):
 *              [0] max |C| over the stored BF16 values,
 *              [1] max |RHT16(C)| over C's col layout (16-row groups along M, sign
 *                  mask rht_signs, the transform of nvfp4_quantize's rht_col),
 *              [2] 0 (no row transform).
 * C is BF16 without accumulation; requires M >= 256 (the CTA-pair kernel) besides
 * the conditions of nvfp4_gemm.  Extends the hot path of the pages (the GEMM
 * epilogue feeding the next quantiser); the pages describe no such fusion. */
nvfp4_status nvfp4_gemm_amax(const nvfp4_tensor* A, const nvfp4_tensor* B, void* C, int64_t ldc,
                             float alpha, uint32_t rht_signs, float* amax_out, void* stream);

/* Several NVFP4 GEMMs in one persistent launch: C_i = S_Ai * S_Bi * A_i . B_i^T for
 * i < count (count <= 8), each as nvfp4_gemm with alpha 1 and no accumulation, all with
 * the same output type.  The output tiles of all problems form one queue that the CTA
 * pairs of a single grid work through, so the last, partial wave of one problem's tiles
 * overlaps the next problem's instead of leaving SMs idle between launches -- e.g. the
 * weight-gradient GEMMs of a layer's linears, deferred to the end of its backward pass
 * (whole-layer scheduling of the linears whose GEMMs the 12B NVFP4 page's recipe
 * quantises).  A[i], B[i]: host arrays of count tensor pointers; C[i], ldc[i]: outputs.
 * Requires per problem M, N, K > 0, M % 128 == 0, N % 128 == 0, K % 64 == 0, 16-byte
 * aligned C rows, and the CTA-pair kernel. */
nvfp4_status nvfp4_gemm_grouped(const nvfp4_tensor* const* A, const nvfp4_tensor* const* B, void* const* C,
                                const int64_t* ldc, int32_t count, int32_t out_dtype, void* stream);

/* Linear forward (fprop): Y [M x N] = Q(X) . Q(W)^T.
 *   X      : BF16 [M x K] activations (device, row stride ldx), quantised here
 *            row-wise with round-to-nearest-even into Xq_row (caller buffers,
 *            MMA scale layout).
 *   Wq_row : the row layout of the 2D-quantised weight W [N x K].
 *   Xq_col : NULL, or buffers for the col layout of X (K x M, 16x16 RHT along
 *            tokens with rht_signs, round-to-nearest-even) saved for wgrad,
 *            produced by the same pass over X.
 * Requires M % 128, N % 128, K % 64 == 0. */
nvfp4_status nvfp4_linear_fwd(const void* X, int64_t M, int64_t K, int64_t ldx,
                              const nvfp4_tensor* Wq_row, void* Y, int64_t ldy, int32_t out_dtype,
                              nvfp4_tensor* Xq_row, nvfp4_tensor* Xq_col, uint32_t rht_signs,
                              void* workspace, size_t workspace_bytes, void* stream);

/* Linear data gradient (dgrad): dX [M x K] = Q_sr(dY) . Q(W).
 *   dY     : BF16 [M x N] output gradient (device, row stride ldy), quantised
 *            row-wise with stochastic rounding (seed, offset) into dYq_row.
 *   Wq_col : the col layout of the 2D-quantised weight ([K x N], the exact
 *            transpose of Wq_row: no re-quantisation).
 *   dYq_col: NULL, or buffers for dY's col layout (N x M, RHT along tokens +
 *            stochastic rounding) saved for wgrad, from the same pass over dY.
 * Requires M % 128, K % 128, N % 64 == 0. */
nvfp4_status nvfp4_linear_dgrad(const void* dY, int64_t M, int64_t N, int64_t ldy,
                                const nvfp4_tensor* Wq_col, void* dX, int64_t ldx, int32_t out_dtype,
                                nvfp4_tensor* dYq_row, nvfp4_tensor* dYq_col, uint64_t seed,
                                uint64_t offset, uint32_t rht_signs, void* workspace,
                                size_t workspace_bytes, void* stream);

/* Linear weight gradient (wgrad): dW [N x K] = Q(H dY)^T . Q(H X), contracting
 * over the M tokens.  dYq_col [N x M] and Xq_col [K x M] are the col layouts
 * saved by nvfp4_linear_dgrad and nvfp4_linear_fwd with the same rht_signs, so
 * the transforms cancel in the product.  accumulate adds into dW (gradient
 * accumulation).  Requires N % 128, K % 128, M % 64 == 0. */
nvfp4_status nvfp4_linear_wgrad(const nvfp4_tensor* dYq_col, const nvfp4_tensor* Xq_col, void* dW,
                                int64_t ldw, int32_t out_dtype, int32_t accumulate, void* stream);

/* Bytes of device workspace that nvfp4_newton_schulz needs for an [m x n] matrix
 * (256-byte aligned; contents need not be initialised): the NVFP4 row and col
 * layouts of X, the BF16 residual R [m x m] and its row layout, and a few scalars.
 * 0 for a shape that nvfp4_newton_schulz rejects. */
size_t nvfp4_newton_schulz_workspace_size(int64_t m, int64_t n);

/* Newton-Schulz orthogonalisation with NVFP4 products.  The optimizer passage of
 * "Full-Stack FP4: Preentrenamiento Estable de LLM" runs the Newton-Schulz
 * iterations of the Muon optimizer natively in NVFP4 and gives no coefficients;
 * this is the coefficient-free cubic iteration for the orthogonal polar factor
 * (Bjorck and Bowie, SIAM J. Numer. Anal. 8, 1971), X <- 3/2 X - 1/2 X X^T X, in
 * residual form:
 *   X_0 = BF16(G / ||G||_F)     (normalize != 0; else X_0 = G)
 *   repeat iters times:
 *     Xr, Xc = nvfp4_quantize(X): row layout (blocks along n) and col layout
 *              (blocks along m), 1D, round-to-nearest-even, no transform
 *     R      = BF16(I - Xr . Xr^T)            an NVFP4 GEMM adding into I
 *     Rr     = nvfp4_quantize(R) row layout
 *     X      = BF16(X + 1/2 Rr . Xc^T)        an NVFP4 GEMM adding into X
 * Each GEMM that adds into a BF16 matrix rounds as BF16(fl32(fl32(product) + C)).
 * Singular values of G/||G||_F in (0, 1] converge towards 1; the 4-bit operands
 * leave them within about 10 % of 1.
 *   G        : BF16 [m x n] (device, row stride ldg elements).  Pass the wide
 *              orientation (m <= n): the work is 4 m^2 n FLOP per iteration.
 *   X        : BF16 [m x n] output (device, row stride ldx); may be G itself when
 *              ldx == ldg (in place); must not otherwise overlap G.
 *   iters    : number of iterations, >= 0.
 *   norm_out : NULL, or one device float receiving ||G||_F (normalize != 0): the
 *              square root of the FP64 sum of squares, rounded to FP32.
 *   workspace: nvfp4_newton_schulz_workspace_size(m, n) bytes of device memory,
 *              256-byte aligned.
 * Requires m % 128 == 0, n % 128 == 0, ldg and ldx multiples of 8, G and X
 * 16-byte aligned.  Extends the hot path of the pages (the optimizer step
 * around the linear layer); enqueues 2 + 7 * iters of this library's kernels
 * (sum of squares and normalisation; per iteration two quantiser passes over X,
 * the identity, two over R and the two GEMMs) and small memsets on `stream`. */
nvfp4_status nvfp4_newton_schulz(const void* G, int64_t m, int64_t n, int64_t ldg, void* X, int64_t ldx,
                                 int32_t iters, int32_t normalize, float* norm_out, void* workspace,
                                 size_t workspace_bytes, void* stream);

/* ---- LoRA-SVD linear.  "Full-Stack FP4: Preentrenamiento Estable de LLM" (linear-
 * projection passage) splits each projection's weight with a light LoRA-SVD
 * decomposition, W = W_res + L R, so that 4-bit quantisation noise falls on the
 * residual; the page gives neither the rank nor the refresh of the factors, so
 * L [N x r] and R [r x K] (BF16, e.g. the top-r singular triplets of W) are the
 * caller's.  The residual takes the NVFP4 path (2D weight blocks); the rank-r part
 * stays in BF16 and joins the NVFP4 GEMM's FP32 accumulator on the tensor cores
 * (nvfp4_gemm_lowrank); the building blocks below also serve it separately.
 * Every call here takes r in {16, 32, 48, 64}. */

/* W_res = BF16(fl32(W - s)), s = sum_j L[n][j] R[j][k] accumulated in FP32 in
 * increasing j (each product of BF16 values is exact in FP32 barring underflow).
 * W, W_res [N x K], L [N x r], R [r x K]: BF16 device matrices with row strides
 * ldw, ldo, ldl, ldr (elements).  Requires K % 8 == 0, W, R, W_res 16-byte aligned
 * with ldw, ldr, ldo multiples of 8.  Quantise W_res with 2D blocks for the
 * linear calls below. */
nvfp4_status nvfp4_lora_residual(const void* W, int64_t N, int64_t K, int64_t ldw, const void* L, int64_t ldl,
                                 const void* R, int64_t ldr, int32_t rank, void* W_res, int64_t ldo,
                                 void* stream);

/* U = BF16(A B^T): A [M x K] BF16 (row stride lda); B [r x K] (b_trans == 0, row
 * stride ldb) or given as its transpose [K x r] (b_trans != 0, row stride ldb);
 * U [M x r] BF16 (row stride ldu).  FP32 accumulation, one rounding to BF16.
 * Requires M % 16 == 0, K a positive multiple of 64, 16-byte aligned rows.
 * Enqueues one persistent kernel (one CTA per SM at most) on `stream`. */
nvfp4_status nvfp4_lowrank_project(const void* A, int64_t M, int64_t K, int64_t lda, const void* B, int64_t ldb,
                                   int32_t b_trans, int32_t rank, void* U, int64_t ldu, void* stream);

/* nvfp4_lowrank_project with the sums divided by g = fl32(*scale_a * *scale_b) before
 * the rounding: U' = BF16(fl32(fl32(A B^T) * fl32(1 / g))).  scale_a and scale_b are
 * device floats, typically the tensor scales of the two operands of the NVFP4 GEMM
 * that U' joins (nvfp4_gemm_lowrank multiplies its accumulator by that g). */
nvfp4_status nvfp4_lowrank_project_scaled(const void* A, int64_t M, int64_t K, int64_t lda, const void* B,
                                          int64_t ldb, int32_t b_trans, int32_t rank, const float* scale_a,
                                          const float* scale_b, void* U, int64_t ldu, void* stream);

/* NVFP4 GEMM with a rank-r BF16 term inside its accumulator (the LoRA-SVD linear
 * above, fused; "Full-Stack FP4", linear-projection passage):
 *   C[m][n] = BF16(g * (sum_k A[m][k] B[n][k] + sum_j U[m][j] V[n][j])),  g = fl32(S_A S_B)
 * where the first sum is the block-scaled NVFP4 product (as in nvfp4_gemm) and the
 * second a BF16 product on the tensor cores, both accumulated in the same FP32
 * accumulator; each output tile ends with one extra pipeline stage that loads its
 * U and V rows and issues r/16 BF16 MMAs.  A [M x K], B [N x K] as for nvfp4_gemm;
 * U [M x r], V [N x r] BF16 device matrices, row strides ldu, ldv (elements);
 * C [M x N] BF16, row stride ldc.  U is usually nvfp4_lowrank_project_scaled(...)
 * with the tensor scales of A and B, so that g U V^T is the plain low-rank product.
 * Requires the conditions of nvfp4_gemm, M >= 256, r in {16, 32, 48, 64}, 16-byte
 * aligned U and V rows. */
nvfp4_status nvfp4_gemm_lowrank(const nvfp4_tensor* A, const nvfp4_tensor* B, const void* U, int64_t ldu,
                                const void* V, int64_t ldv, int32_t rank, void* C, int64_t ldc, void* stream);

/* Y <- BF16(fl32(Y + U C^T)) in place: Y [M x N] BF16 (row stride ldy); U [M x r];
 * C [N x r] (c_trans == 0, row stride ldc) or given as its transpose [r x N]
 * (c_trans != 0).  FP32 accumulation of the product.  Requires M % 128 == 0,
 * N % 128 == 0, 16-byte aligned rows. */
nvfp4_status nvfp4_lowrank_expand_add(void* Y, int64_t M, int64_t N, int64_t ldy, const void* U, int64_t ldu,
                                      const void* C, int64_t ldc, int32_t c_trans, int32_t rank, void* stream);

/* LoRA-SVD fprop: X is quantised as in nvfp4_linear_fwd, U' = BF16(X R^T / g) with
 * g = fl32(S_X S_W) (nvfp4_lowrank_project_scaled), and
 *   Y = BF16(g * (Q(X) Q(W_res)^T + U' L^T))   in one nvfp4_gemm_lowrank.
 * Arguments as nvfp4_linear_fwd, plus L [N x r] and R [r x K] contiguous BF16 device
 * matrices and U, caller scratch of M * r BF16 (16-byte aligned).  Y is BF16.
 * Requires M >= 256 besides the conditions of nvfp4_linear_fwd.  Work: the
 * quantisation of X, one pass over X for U', and the GEMM. */
nvfp4_status nvfp4_lora_linear_fwd(const void* X, int64_t M, int64_t K, int64_t ldx, const nvfp4_tensor* Wq_res_row,
                                   const void* L, const void* R, int32_t rank, void* Y, int64_t ldy,
                                   nvfp4_tensor* Xq_row, nvfp4_tensor* Xq_col, uint32_t rht_signs, void* U,
                                   void* workspace, size_t workspace_bytes, void* stream);

/* LoRA-SVD dgrad: dY is quantised as in nvfp4_linear_dgrad, U' = BF16(dY L / g) with
 * g = fl32(S_dY S_W), and
 *   dX = BF16(g * (Q_sr(dY) Q(W_res) + U' R))   in one nvfp4_gemm_lowrank.
 * Arguments as nvfp4_linear_dgrad, plus L [N x r] contiguous, Rt = R^T [K x r]
 * contiguous (the tensor cores read R with its rank index contiguous), and U as for
 * nvfp4_lora_linear_fwd.  Requires M >= 256.  The weight gradient is that of W
 * itself: nvfp4_linear_wgrad, unchanged. */
nvfp4_status nvfp4_lora_linear_dgrad(const void* dY, int64_t M, int64_t N, int64_t ldy, const nvfp4_tensor* Wq_res_col,
                                     const void* L, const void* Rt, int32_t rank, void* dX, int64_t ldx,
                                     nvfp4_tensor* dYq_row, nvfp4_tensor* dYq_col, uint64_t seed, uint64_t offset,
                                     uint32_t rht_signs, void* U, void* workspace, size_t workspace_bytes,
                                     void* stream);

/* nvfp4_quantize without a workspace argument, for callers that cannot
 * allocate device memory at the point of the call -- for example a host thread
 * that must not take the allocator's device-wide locks or trigger its implicit
 * synchronisation, code that runs inside a fixed, pre-planned memory budget, or
 * a foreign-language caller that has no device allocator at hand.  No
 * counterpart on the source pages: it exists for how the library is called.
 *   Arguments, outputs and results are those of nvfp4_quantize.
 *   Scratch: a 256-byte array of device memory inside the library, held by
 *   every GPU that loads it until the process exits; this call allocates and
 *   frees nothing.  The quantiser needs 12 bytes of it for any tensor size;
 *   a scratch requirement above 256 bytes is rejected with
 *   NVFP4_ERR_WORKSPACE.
 *   Set-up: the first call on a device looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current and caches it; make that
 *   first call before any stream capture.
 *   Sharing: all calls on a device use the same array and leave their last
 *   values in it; each call clears what it needs.  Calls whose work overlaps
 *   on the GPU (different streams, no ordering between them) race on the
 *   array and may produce wrong tensor scales; order them on one stream or
 *   use nvfp4_quantize with a workspace per stream. */
nvfp4_status nvfp4_quantize_noalloc(const void* x, int64_t rows, int64_t cols, int64_t ld,
                                    const nvfp4_quant_opts* opts, nvfp4_tensor* out_row,
                                    nvfp4_tensor* out_col, void* stream);

/* Self-check of the conversions the quantiser encodes with.  The kernels use
 * the sm_100a conversion instructions for E2M1 round-to-nearest-even, E2M1
 * stochastic rounding (the rule stated for nvfp4_quant_opts.stochastic) and
 * E4M3 round-to-nearest-even; this call compares each with its definition on
 * the current device and writes mismatch counts to counts (3 device uint64,
 * 16-byte aligned): [0] E2M1 RNE over every float bit pattern, [1] E4M3 over
 * every non-negative finite float, [2] E2M1 stochastic rounding over n_sr
 * pseudo-random (value, random word) pairs.  All three are 0 on a conforming
 * GPU.  Asynchronous on `stream`; a few milliseconds of GPU time. */
nvfp4_status nvfp4_check_conversions(unsigned long long* counts, uint64_t n_sr, void* stream);

/* Synchronise `stream`, then report and clear any device-side error recorded
 * by this library's kernels on the current device since the last call
 * (NVFP4_ERR_TIMEOUT), or a pending CUDA error (NVFP4_ERR_CUDA).
 * A kernel whose bounded wait gives up (after 2 s) returns with its outputs
 * partly written; the only sign of it is this call's status.  So the outputs of
 * every call enqueued since the last clean status are valid only once this call
 * returns NVFP4_OK: check it at least once per training step, before the step's
 * results are used (for example before the optimizer update). */
nvfp4_status nvfp4_get_status(void* stream);

/* Text of the last non-OK status returned on the calling thread. */
const char* nvfp4_last_error_string(void);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4_H */
