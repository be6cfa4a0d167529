/*
 * fp4q.h -- C ABI of the B200 (sm_100a) block-scaled FP4 quantization library.
 *
 * Formats. A tensor is a row-major bf16 matrix [rows, cols]; blocks of
 * `block` consecutive elements along a row share one scale.
 *   NVFP4: E2M1 elements, one OCP E4M3 scale byte per block and one FP32
 *          per-tensor global scale s_g = amax / (448 * 6) (hierarchical
 *          scaling); block 16 is the hardware block, 4 / 8 / 32 are also
 *          provided ("Finer is Better (with the Right Scaling)", 手法 1-2).
 *   MXFP4: E2M1 elements, one E8M0 (power-of-two) scale byte per block of 32
 *          ("Bridging the Gap Between Promise and Performance for
 *          Microscaling FP4 Quantization", 技術概要 §1).
 *   UE5M3: E2M1 elements, one unsigned 5-exponent / 3-mantissa scale byte per
 *          block of 4 / 8 / 16 / 32 and no per-tensor scale (see
 *          fp4q_format for the encoding read here).
 *
 * Storage. codes: uint8 [rows, cols/2], element 2j in the low nibble of byte
 * j and element 2j+1 in the high nibble; 4-bit code = sign bit (bit 3) and
 * E2M1 magnitude index (bits 0-2). scales: uint8 [rows, cols/block]
 * row-major (E4M3 code, E8M0 byte = exponent + 127, or UE5M3 code). Per-block MSE:
 * float [rows, cols/block]. Dequantized values: [rows, cols] fp32 or bf16.
 *
 * Arithmetic. Every result except the GEMM's is bit-identical to the plain
 * CPU definition of the operation: one IEEE binary32 operation per step (a
 * fused multiply-add only where the definition has one, as in the GPTQ
 * updates), E2M1 / E4M3 / UE5M3 round-to-nearest-even with saturation, the
 * optional Hadamard rotation applied as a Walsh-Hadamard butterfly with
 * ascending stages, and block sums taken with the adjacent-pair tree. The
 * GEMM accumulates on the tensor cores in fp32 in the hardware's order.
 *
 * Conventions for every entry point:
 *  - All array pointers are DEVICE pointers owned by the caller, 16-byte
 *    aligned, dense row-major (leading dimension = cols). The library never
 *    allocates or frees memory and never synchronises (fp4q_device_errors
 *    aside): work is enqueued on `stream` (0 = legacy default stream) and
 *    the call returns before it completes.
 *  - State the library keeps between calls, all of it listed here:
 *      * a per-device error counter in device memory (fp4q_device_errors);
 *      * the CUDA error code of the last failed launch, per host thread
 *        (fp4q_last_cuda_error);
 *      * the 256-byte scratch array of fp4q_gemm_noalloc, one per device, and
 *        its device address, cached per device ordinal on first use;
 *      * host-side caches of launch facts that do not change while the
 *        process runs: the driver's tensor-map encoder entry point (TMA
 *        path) and the resident CTAs per SM of each persistent quantize
 *        kernel (queried once per kernel);
 *      * the test hook of fp4q_debug_fail_launches (process-wide);
 *      * the FP4Q_TMA environment switch, read at every quantize call
 *        (see fp4q_device_errors).
 *  - Arguments are validated on the host before anything is enqueued; on an
 *    error nothing is launched and outputs are untouched.
 *  - rows == 0 or cols == 0 is an empty tensor: its array pointers may be
 *    NULL, nothing is read or written except that NVFP4 global_scale_out
 *    receives 1.0 (and fp4q_global_amax writes 0).
 *  - Inputs must be finite, and so must their rotation (a blockwise Hadamard
 *    sum of inputs near the bf16 maximum can exceed the fp32 range; the
 *    codes of such a block are then unspecified). Outputs must not overlap
 *    inputs or each other
 *    (arrays an entry point documents as read and overwritten are the
 *    exception: they are updated in place).
 *  - FP4Q_ERR_CUDA means a launch was rejected by the CUDA runtime; the
 *    runtime's code is available from fp4q_last_cuda_error(). Faults that
 *    happen while the kernels run surface at the caller's next
 *    synchronisation, as for any CUDA work.
 */
#ifndef FP4Q_H
#define FP4Q_H

#include <stdint.h>

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FP4Q_OK = 0,
    FP4Q_ERR_NULL = 1,        /* a required pointer is NULL */
    FP4Q_ERR_SHAPE = 2,       /* negative sizes, or cols not a multiple of block / rot / sub */
    FP4Q_ERR_ALIGN = 3,       /* an array pointer is not 16-byte aligned (4 for scalars) */
    FP4Q_ERR_UNSUPPORTED = 4, /* format / block / strategy / rotation / sub not offered */
    FP4Q_ERR_ALIAS = 5,       /* global_amax_in and global_scale_out are the same address */
    FP4Q_ERR_CUDA = 6         /* the CUDA runtime rejected a launch */
} fp4q_status;

/* Block formats: FP4 (E2M1) elements with
 *   NVFP4  E4M3 block scales under an FP32 per-tensor scale s_g; blocks 4..32
 *   MXFP4  E8M0 (power-of-two) block scales; block 32
 *   UE5M3  unsigned 5-exponent / 3-mantissa block scales with no per-tensor
 *          scale; blocks 4..32. "Finer is Better (with the Right Scaling)"
 *          (意義と主張) compares this wide-range format with E4M3 +
 *          hierarchical scaling but gives no encoding; this library reads it
 *          as bias 15, subnormals at exponent field 0 (m * 2^-17), 0xFF the
 *          only NaN, largest 1.75 * 2^16 (0xFE), values above it saturating,
 *          round to nearest even. Quantize, dequantize and block MSE take it;
 *          FOCUS and the GEMM do not (FP4Q_ERR_UNSUPPORTED). */
typedef enum { FP4Q_FMT_NVFP4 = 0, FP4Q_FMT_MXFP4 = 1, FP4Q_FMT_UE5M3 = 2 } fp4q_format;

/* Block-scale selection ("Finer is Better (with the Right Scaling)", 手法 2).
 * MXFP4 offers FP4Q_ABSMAX (E8M0 byte floor(log2 amax) - 2 + 127) and
 * FP4Q_BRUTE_FORCE: the MSE-optimised scale of "Bridging the Gap Between
 * Promise and Performance for Microscaling FP4 Quantization" (技術概要 §2.2
 * item 1) over every E8M0 byte 0..254, ties -> lower byte. */
typedef enum {
    FP4Q_ABSMAX = 0,        /* code = RNE_E4M3(amax / (6 s_g)) */
    FP4Q_PREVENT_ZERO = 1,  /* abs-max code clipped below at 0x01 (2^-9) */
    FP4Q_FOUR_OVER_SIX = 2, /* targets 6 and 4; keep 4 only if its block SSE is lower */
    FP4Q_BRUTE_FORCE = 3    /* minimum block SSE over codes 0x01..0x7E; ties -> lower code */
} fp4q_strategy;

typedef enum { FP4Q_OUT_F32 = 0, FP4Q_OUT_BF16 = 1 } fp4q_dtype;

/* Optimizer of the FOCUS coefficient calibration ("FOCUS: ...", Metodologia
 * §1: the scales are learned by gradient descent through the STE; the page
 * names no optimizer). FP4Q_OPT_ADAM follows Kingma & Ba's algorithm. */
typedef enum { FP4Q_OPT_SGD = 0, FP4Q_OPT_ADAM = 1 } fp4q_optimizer;

/*
 * fp4q_quantize -- rotate (optional) -> per-block scale -> E2M1 RNE -> pack,
 * with optional dequantized values and per-block MSE.
 *
 * x                bf16 [rows, cols].
 * fmt, block       NVFP4 or UE5M3 with block in {4, 8, 16, 32}; MXFP4 with
 *                  block 32. UE5M3 candidate codes: RNE_UE5M3(amax / T), T = 6
 *                  (and 4 for 4-over-6); brute force over codes 0x01..0xFE.
 * strat            see fp4q_strategy.
 * rot              0 (none) or the blockwise Hadamard size 16, 32, 64, 128:
 *                  every rot-wide chunk of a row becomes H_rot x / sqrt(rot)
 *                  before scaling ("Bridging the Gap ...", 技術概要 §2.2
 *                  item 3); codes, dq and MSE are in the rotated domain.
 * global_amax_in   NVFP4: NULL to compute the abs-max of the (rotated)
 *                  tensor on the device (an extra read of x), or a device
 *                  float holding a calibrated abs-max (single pass). Ignored
 *                  for MXFP4 and UE5M3.
 * global_scale_out NVFP4: required device float, receives s_g. Ignored for
 *                  MXFP4 and UE5M3. When global_amax_in is NULL it is also used to
 *                  accumulate the abs-max before s_g replaces it.
 * codes            uint8 [rows, cols/2], required.
 * scales           uint8 [rows, cols/block], required.
 * block_mse        float [rows, cols/block] or NULL.
 * dq               [rows, cols] of dq_dtype, or NULL.
 * Errors: NULL, SHAPE (cols % block, cols % rot), ALIGN, UNSUPPORTED
 * (MXFP4 with PREVENT_ZERO or FOUR_OVER_SIX, unknown enum values), ALIAS, CUDA.
 */
fp4q_status fp4q_quantize(const void* x, int64_t rows, int64_t cols, fp4q_format fmt, int block,
                          fp4q_strategy strat, int rot, const float* global_amax_in,
                          float* global_scale_out, uint8_t* codes, uint8_t* scales,
                          float* block_mse, void* dq, fp4q_dtype dq_dtype, cudaStream_t stream);

/*
 * fp4q_dequantize -- value(code) * S with S = E4M3(scale) * s_g (NVFP4),
 * 2^(scale - 127) (MXFP4) or UE5M3(scale); only the dequantization scale is needed at
 * inference ("FOCUS: FP4 Optimization via Coupled-Relaxation and
 * Dual-Granularity Scaling", Metodologia §4).
 * global_scale: NVFP4 device float s_g (required); ignored for MXFP4 and UE5M3.
 * out: [rows, cols] of out_dtype (bf16 output is the RNE rounding of the fp32 value).
 */
fp4q_status fp4q_dequantize(const uint8_t* codes, const uint8_t* scales,
                            const float* global_scale, int64_t rows, int64_t cols,
                            fp4q_format fmt, int block, void* out, fp4q_dtype out_dtype,
                            cudaStream_t stream);

/*
 * fp4q_dequantize_unrotate -- fp4q_dequantize, then every rot-wide chunk of a
 * row taken back to the original domain by the normalised Walsh-Hadamard
 * transform (the blockwise rotation of "Bridging the Gap Between Promise and
 * Performance for Microscaling FP4 Quantization", 技術概要 §2.2 item 3; the
 * Sylvester matrix is symmetric with H H = n I, so the normalised transform
 * is its own inverse -- exactly for rot 16 and 64, up to the rounding of
 * 1/sqrt(rot) for 32 and 128). Same stage order and constant as the rotation
 * applied by fp4q_quantize. rot in {0, 16, 32, 64, 128}; 0 is plain
 * dequantization. Arguments, ownership and errors as fp4q_dequantize, plus
 * SHAPE when cols % rot != 0 and UNSUPPORTED for another rot.
 */
fp4q_status fp4q_dequantize_unrotate(const uint8_t* codes, const uint8_t* scales,
                                     const float* global_scale, int64_t rows, int64_t cols,
                                     fp4q_format fmt, int block, int rot, void* out,
                                     fp4q_dtype out_dtype, cudaStream_t stream);

/*
 * W4A4 FP4 GEMM on the tcgen05 block-scaled tensor cores -- the consumer of
 * the quantizer's output ("Bridging the Gap Between Promise and Performance
 * for Microscaling FP4 Quantization", 技術概要 §2.3: MXFP4 / NVFP4 matrix
 * multiplication on Blackwell SM100; §2.2 item 3: activations rotated and
 * quantized online in front of it).
 *
 * fp4q_mma_scale_bytes -- size in bytes of the scale buffer that
 * fp4q_scales_to_mma fills for a [rows, K] operand (rows padded to 128, blocks
 * to 4). 0 for invalid arguments (rows <= 0, K not a multiple of the block:
 * 16 for NVFP4, 32 for MXFP4). Host only; no GPU work.
 *
 * fp4q_scales_to_mma -- reorders the row-major block scales written by
 * fp4q_quantize (uint8 [rows, K/block]) into the block-scaled MMA's layout:
 * 512-byte atoms of 128 rows x 4 blocks, row r of an atom at byte
 * 16 (r % 32) + 4 (r / 32), block j at + j; atoms along K first; padding
 * bytes are zero. mma_scales: device, fp4q_mma_scale_bytes(rows, K, fmt)
 * bytes, caller-owned. Errors: UNSUPPORTED (fmt), SHAPE, NULL, CUDA.
 *
 * fp4q_gemm -- D[m, n] = alpha * sum_k A[m, k] * B[n, k], where A [M, K] and
 * B [N, K] (a weight in PyTorch's Linear layout) are packed E2M1 codes as
 * written by fp4q_quantize (uint8 [rows, K/2], K contiguous, element 2j in
 * the low nibble) with their block scales in MMA layout (fp4q_scales_to_mma
 * of the same rows and K). NVFP4: alpha = s_g(A) * s_g(B) from the two device
 * global scales; MXFP4: alpha = 1 (global scales ignored, may be NULL).
 * alpha_out: a caller-owned device float the library writes alpha into before
 * the GEMM reads it (so overlapping calls need distinct alpha_out). d: device
 * row-major [M, N] of d_dtype (fp32, or bf16 = RNE of the fp32 result).
 * Products are accumulated in fp32 on the tensor cores (order not specified).
 * K must be a multiple of 32 and N of 4 (fp32 output) or 8 (bf16); code,
 * scale and output pointers 16-byte aligned. Errors: UNSUPPORTED (fmt,
 * d_dtype), SHAPE, NULL, ALIGN, CUDA (also when the GEMM rejects the shape).
 */
/*
 * fp4q_gemm_noalloc -- fp4q_gemm without the alpha_out argument: alpha is
 * written into a 256-byte scratch array inside the library image (one float
 * of it is used) instead of a caller-owned device float. For callers that
 * cannot hand over memory on the call path. Limits: all calls on a device
 * share that one scratch float, so calls that overlap (in flight at the same
 * time on different streams or threads) race on it -- serialise them or use
 * fp4q_gemm; the first call on each device looks the scratch address up
 * (cudaGetSymbolAddress), so make that first call before any stream capture
 * begins. The address is cached for the life of the process: a process
 * that calls cudaDeviceReset on a device must not call this entry point on
 * that device afterwards. The pages have no counterpart: this is an
 * interface detail. Other arguments, results and errors as fp4q_gemm.
 */
fp4q_status fp4q_gemm_noalloc(const uint8_t* a_codes, const uint8_t* a_mma_scales,
                              const float* a_global_scale, const uint8_t* b_codes,
                              const uint8_t* b_mma_scales, const float* b_global_scale, int64_t M,
                              int64_t N, int64_t K, fp4q_format fmt, void* d, fp4q_dtype d_dtype,
                              cudaStream_t stream);

/*
 * fp4q_quantize_mma -- fp4q_quantize (block 16 for NVFP4, 32 for MXFP4; no MSE or
 * dq outputs) writing the scale bytes straight into the block-scaled MMA
 * layout of fp4q_scales_to_mma: the quantizer feeding fp4q_gemm in one launch
 * (rotation fused in front, "Bridging the Gap ...", 技術概要 §2.2 item 3).
 * mma_scales: fp4q_mma_scale_bytes(rows, cols, fmt) bytes whose padding bytes
 * (rows past rows, blocks past cols / block) must already be zero -- only the
 * real blocks are written. cols % 32 == 0 and rows * cols / 32 < 2^32.
 * Other arguments and errors as fp4q_quantize.
 */
fp4q_status fp4q_quantize_mma(const void* x, int64_t rows, int64_t cols, fp4q_format fmt,
                              fp4q_strategy strat, int rot, const float* global_amax_in,
                              float* global_scale_out, uint8_t* codes, uint8_t* mma_scales,
                              cudaStream_t stream);
size_t fp4q_mma_scale_bytes(int64_t rows, int64_t K, fp4q_format fmt);
fp4q_status fp4q_scales_to_mma(const uint8_t* scales, int64_t rows, int64_t K, fp4q_format fmt,
                               uint8_t* mma_scales, cudaStream_t stream);
fp4q_status fp4q_gemm(const uint8_t* a_codes, const uint8_t* a_mma_scales,
                      const float* a_global_scale, const uint8_t* b_codes,
                      const uint8_t* b_mma_scales, const float* b_global_scale, int64_t M,
                      int64_t N, int64_t K, fp4q_format fmt, float* alpha_out, void* d,
                      fp4q_dtype d_dtype, cudaStream_t stream);

/*
 * fp4q_block_mse -- per-block mean squared error of x (rotated by rot first)
 * against dequantize(codes, scales): tree sum of (y - yhat)^2 divided by
 * block ("Finer is Better (with the Right Scaling)", 手法 1: MSE per block
 * size). Equal bit for bit to fp4q_quantize's block_mse for its own codes.
 */
fp4q_status fp4q_block_mse(const void* x, const uint8_t* codes, const uint8_t* scales,
                           const float* global_scale, int64_t rows, int64_t cols,
                           fp4q_format fmt, int block, int rot, float* block_mse,
                           cudaStream_t stream);

/*
 * fp4q_focus_fwd -- FOCUS decoupled fake quantization (CRS + DGS):
 * W_hat = S_dq * Q(W / (S_dq * c_k)) where S_dq is the format's abs-max block
 * scale (shared by the hardware block) and c_k is the fp16 coefficient of
 * sub-block k ("FOCUS: ...", Metodologia §2 S_q = S_dq * c_i, §3 sub-block
 * formula). sub == block is CRS alone.
 * w        bf16 [rows, cols]; c: fp16 [rows, cols/sub]; sub in {2,4,8,16,32},
 *          dividing block.
 * global_amax_in / global_scale_out: as fp4q_quantize (NVFP4; abs-max of W).
 * w_hat    [rows, cols] of out_dtype, required.
 * codes, scales: optional deployable export (both or neither): the FP4 codes
 *          Q(W / (S_dq * c_k)) and the S_dq bytes; the coefficients are not
 *          part of it (Metodologia §4).
 */
fp4q_status fp4q_focus_fwd(const void* w, const void* c, int64_t rows, int64_t cols,
                           fp4q_format fmt, int block, int sub, const float* global_amax_in,
                           float* global_scale_out, void* w_hat, fp4q_dtype out_dtype,
                           uint8_t* codes, uint8_t* scales, cudaStream_t stream);

/*
 * fp4q_focus_bwd -- straight-through gradient of the coefficients
 * ("FOCUS: ...", Metodologia §1 STE): with dQ/du taken as 1,
 * dL/dc_k = -(sum over sub-block k of g_j * W_j) / (c_k * c_k), the sum in
 * fp32 with the adjacent-pair tree. S_dq receives no gradient.
 * w, g     bf16 [rows, cols] (g = dL/dW_hat); c: fp16 [rows, cols/sub];
 * dc       float [rows, cols/sub]; sub in {2,4,8,16,32}.
 */
fp4q_status fp4q_focus_bwd(const void* w, const void* g, const void* c, int64_t rows,
                           int64_t cols, int sub, float* dc, cudaStream_t stream);

/*
 * fp4q_focus_update -- one calibration step of the FOCUS coefficients from an
 * external gradient g = dL/dW_hat (the loss the caller differentiates: the
 * pages' distillation loss, or a layer-output loss such as
 * |X (W_hat - W)^T|^2 whose gradient 2 (W_hat - W) X^T X is a plain GEMM).
 * ("FOCUS: ...", Metodologia §1 STE and gradient descent, §2 c is an FP16
 * learnable parameter initialised to 1.)
 * Per sub-block k: c16 = fp16(c[k]) (round to nearest even; the value the
 * forward pass consumes), dc = -(tree_sum(g * W) / (c16 * c16)) as in
 * fp4q_focus_bwd, then the optimizer step on the fp32 master c[k]:
 *   SGD   c <- c - lr * dc
 *   Adam  m <- b1 m + (1 - b1) dc;  v <- b2 v + (1 - b2) (dc * dc);
 *         c <- c - alpha_t * (m / (sqrt(v) + eps)), the efficient ordering
 *         Kingma & Ba give beside their algorithm: the bias corrections sit
 *         in alpha_t = lr sqrt(1 - b2^t) / (1 - b1^t), computed in double on
 *         the host and rounded to fp32; every other step is one fp32
 *         operation, RNE.
 * w, g     bf16 [rows, cols].
 * c        fp32 [rows, cols/sub], read and overwritten (master coefficients).
 * c_half   nullable fp16 [rows, cols/sub]: fp16(c) after the step, ready for
 *          fp4q_focus_fwd.
 * m, v     fp32 [rows, cols/sub], Adam's moments, read and overwritten
 *          (start at zero); ignored (may be NULL) for SGD.
 * t        Adam's step number, >= 1. b1, b2, eps are ignored for SGD.
 * An unknown opt, or Adam with t < 1, returns FP4Q_ERR_UNSUPPORTED; Adam with
 * m or v NULL (with rows * cols > 0) returns FP4Q_ERR_NULL. c, c_half, m, v must not
 * overlap w or g.
 * Nothing keeps c positive: a coefficient driven to zero or below gives
 * unspecified codes in the next forward pass.
 */
fp4q_status fp4q_focus_update(const void* w, const void* g, float* c, void* c_half, float* m,
                              float* v, int64_t rows, int64_t cols, int sub, fp4q_optimizer opt,
                              float lr, float b1, float b2, float eps, int64_t t,
                              cudaStream_t stream);

/*
 * fp4q_focus_step -- one fused calibration step on the weight-reconstruction
 * loss L = sum (W_hat - W)^2: the FOCUS forward at c16 = fp16(c) (exactly
 * fp4q_focus_fwd's W_hat, kept in fp32), g = 2 (W_hat - W) in fp32, the
 * straight-through gradient dc = -(tree_sum(g * W) / (c16 * c16)) and the
 * optimizer step of fp4q_focus_update, in one pass over W
 * ("FOCUS: ...", Metodologia §1-§3). With c == 1 every element already lands
 * on its nearest point of the S_dq grid, so this loss is at its minimum there;
 * the step is the loop's fused building block, and losses that couple
 * elements go through fp4q_focus_update.
 * w, fmt, block, sub, global_amax_in, global_scale_out: as fp4q_focus_fwd.
 * c, c_half, m, v, opt, lr, b1, b2, eps, t: as fp4q_focus_update.
 * sse      nullable fp32 [rows, cols/sub]: tree_sum((W_hat - W)^2) per
 *          sub-block, at the coefficients before the step.
 */
fp4q_status fp4q_focus_step(const void* w, int64_t rows, int64_t cols, fp4q_format fmt, int block,
                            int sub, const float* global_amax_in, float* global_scale_out,
                            float* c, void* c_half, float* m, float* v, float* sse,
                            fp4q_optimizer opt, float lr, float b1, float b2, float eps,
                            int64_t t, cudaStream_t stream);

/*
 * fp4q_gptq -- GPTQ error feedback with static groups: the error-feedback part
 * of MR-GPTQ ("Bridging the Gap Between Promise and Performance for
 * Microscaling FP4 Quantization", 技術概要 §2.2: GPTQ with the MSE-optimised
 * grid, static activation reordering and rotations).
 * The block scales are fixed beforehand (static groups: `scales` and
 * `global_scale` as fp4q_quantize wrote them for the original weights, any
 * strategy -- FP4Q_BRUTE_FORCE is the MSE-optimised grid). The columns are
 * processed in the order perm (static activation reordering) against U, the
 * upper Cholesky factor of the inverse (damped) Hessian taken in that order
 * (H^-1 = U^T U); the codes are written in the original column order.
 * Per row, in batches of 128 positions: for each position j, q = E2M1 code
 * of w_j / S (code 0 where S == 0), e_j = (w_j - value(q) * S) / U[j][j],
 * and the later positions k of the batch take w_k = fma(-e_j, U[j][k], w_k);
 * after the batch every later column takes w_k -= (fma chain over the batch,
 * j ascending, of e_j * U[j][k]). All fp32, one rounding per operation.
 * w         bf16 [rows, cols], cols a multiple of 128.
 * fmt, block, scales [rows, cols/block], global_scale (NVFP4 s_g, device):
 *           the static block scales; any format.
 * rot       0, or 16 / 32 / 64 / 128: MR-GPTQ's rotation first -- every row
 *           is rotated chunk by chunk exactly as fp4q_quantize rotates it
 *           (blockwise normalised Walsh-Hadamard, fp32) and the feedback runs
 *           on the rotated weights; scales, global_scale, U and perm are then
 *           those of the rotated basis (scales from fp4q_quantize with the
 *           same rot; U from the Hessian of the rotated inputs, R H R). The
 *           codes are the rotated weights' (fp4q_dequantize_unrotate takes
 *           them back). With rot > 0 a row is staged in shared memory:
 *           cols * 4 bytes must not exceed 227 KB (else SHAPE).
 * U         fp32 [cols, cols] row-major (only the upper triangle is read).
 * perm      int32 [cols]: processing position -> original column, a
 *           permutation (entries outside 0..cols-1 are counted by
 *           fp4q_device_errors and read column 0); NULL = natural order.
 * work      fp32 [rows, cols] caller scratch (overwritten).
 * codes     uint8 [rows, cols/2] (zeroed, then written).
 * Launches: 1 memset + 2 * cols/128 - 1 kernels (2 when cols == 128): a
 * gather, one kernel per batch, and the trailing updates, each of which runs
 * beside the next batch's kernel in the same stream. Rows are independent.
 */
fp4q_status fp4q_gptq(const void* w, int64_t rows, int64_t cols, fp4q_format fmt, int block,
                      int rot, const uint8_t* scales, const float* global_scale, const float* U,
                      const int32_t* perm, float* work, uint8_t* codes, cudaStream_t stream);

/*
 * fp4q_global_amax -- abs-max of the (rotated) tensor into *amax_out (device
 * float): the per-tensor statistic of hierarchical scaling ("Finer is Better
 * (with the Right Scaling)", 手法 2). Feed it to global_amax_in of the calls
 * above to run them as a single pass.
 */
fp4q_status fp4q_global_amax(const void* x, int64_t rows, int64_t cols, int rot, float* amax_out,
                             cudaStream_t stream);

/*
 * Element-wise rounding primitives used by every kernel above, exposed so
 * that they can be checked exhaustively: one output byte per input float.
 * fp4q_e2m1_encode: 4-bit E2M1 code (sign kept, RNE, saturating at +-6).
 * fp4q_e4m3_encode: E4M3 code of a non-negative v with a clear sign bit
 *                   (RNE, saturating at 448); the kernels only round such
 *                   values (a block abs-max over a positive divisor).
 */
fp4q_status fp4q_e2m1_encode(const float* u, int64_t n, uint8_t* out, cudaStream_t stream);
fp4q_status fp4q_e4m3_encode(const float* v, int64_t n, uint8_t* out, cudaStream_t stream);

/* Human-readable name of a status code (static string). */
const char* fp4q_status_string(fp4q_status s);

/* The cudaError_t of the last FP4Q_ERR_CUDA returned on this host thread. */
int fp4q_last_cuda_error(void);

/*
 * Test hook for the CUDA-error path (the pages have no counterpart). While
 * cuda_error is nonzero, every entry point that would enqueue work validates
 * its arguments as usual and then, instead of enqueuing anything, returns
 * FP4Q_ERR_CUDA with cuda_error recorded for fp4q_last_cuda_error: no kernel,
 * memset or copy is issued and outputs are untouched. 0 restores normal
 * operation. Process-wide and not synchronised with calls in flight on other
 * threads; for tests only.
 */
void fp4q_debug_fail_launches(int cuda_error);

/*
 * Pipeline health. The TMA-fed quantize kernel waits on shared-memory
 * barriers with a bounded number of polls; a wait that runs out (which
 * correct operation never produces) makes the kernel leave early and adds
 * one to a per-device counter instead of hanging the GPU. This call
 * synchronises with the current device, returns the counter and clears it
 * (-1 if the read failed). Environment: by default the TMA-fed kernel takes
 * MXFP4 quantize calls behind a 64- or 128-wide rotation and the direct-load
 * kernel every other call; FP4Q_TMA=1 routes every call whose flattened
 * length is a multiple of 64 (all strategies but brute force) to the TMA-fed
 * kernel, FP4Q_TMA=0 none. Both kernels compute the same bits.
 */
int fp4q_device_errors(void);

#ifdef __cplusplus
}
#endif

#endif /* FP4Q_H */
