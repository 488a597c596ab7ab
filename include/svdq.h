/*
 * svdq.h -- C ABI of the SVDQuant W4A4 linear layer for NVIDIA B200 (sm_100a).
 *
 * The layer (SVDQuant; SOTA-314 practice page "Do this", NOTE-257 note page
 * "Contribution" and "Key results") computes
 *
 *     Y = Q(X diag(lam)^-1) Q(R) + (X diag(lam)^-1 L1) L2 + b
 *
 * where lam are per-input-channel smoothing factors, W_hat = diag(lam) W,
 * L1 = U Sigma[:, :r] and L2 = V^T[:r, :] are the top-r SVD factors of W_hat
 * (r = 32 at 4 bits), and R = W_hat - L1 L2 is the residual, quantized to NVFP4
 * (E2M1 values, groups of 16 along K, E4M3 scales, power-of-two FP32 tensor
 * scale) or INT4 (groups of 64, BF16 scales).
 *
 * Conventions shared by every entry point:
 *   - No exception or abort crosses this ABI; each call returns an svdq_status.
 *   - Matrices are row-major, BF16 values are passed as their uint16_t bit
 *     patterns, and "device" pointers are CUDA global-memory addresses of the
 *     current process on the layer's device.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Forward calls are stream-ordered and asynchronous: they enqueue kernels
 *     and return; they never synchronise (except with SVDQ_FWD_CHECK) and never
 *     allocate memory.  The caller owns X, Y and the workspace.
 *   - A layer owns its device buffers; svdq_destroy frees them.  A layer may be
 *     used by several streams only if their forward calls do not overlap in time
 *     on the device through a shared workspace.
 *   - Shape rules: K % 64 == 0, N % 16 == 0 (any N >= 1 for SVDQ_W4A16_INT4),
 *     M >= 1 (any M: tails are handled).
 *     Other shapes return SVDQ_EUNSUPPORTED.
 *   - Environment, read once when a layer is placed on its device:
 *     SVDQ_WAIT_BUDGET_MS -- wall-clock budget of every device wait (default
 *       2000): a wait that runs out records a timeout that svdq_check (or
 *       SVDQ_FWD_CHECK) reports as SVDQ_ETIMEOUT, and the kernel ends;
 *     SVDQ_K2_KERNEL=pair|single -- the W4A4 GEMM on CTA pairs (256 x 256
 *       tiles, clusters of two, tcgen05 cta_group::2) or on single CTAs
 *       (128 x 256 tiles, the default).  Both give bit-identical results.
 */
#ifndef SVDQ_H
#define SVDQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SVDQ_OK = 0,
  SVDQ_EINVAL = 1,          /* null pointer, bad enum, inconsistent sizes          */
  SVDQ_EUNSUPPORTED = 2,    /* shape or option this build does not implement       */
  SVDQ_ENOMEM = 3,          /* host or device allocation failed (prepare, set_lora,
                               deserialize; never a forward)                        */
  SVDQ_ECUDA = 4,           /* a CUDA runtime/driver call failed                   */
  SVDQ_ENOCONVERGE = 5,     /* the truncated SVD did not converge                  */
  SVDQ_ETIMEOUT = 6,        /* a bounded device wait expired (read with CHECK)     */
  SVDQ_ESTATE = 7           /* the layer has no device copy (prepared host-only)   */
} svdq_status;

typedef enum {
  SVDQ_NVFP4 = 0,           /* W4A4, E2M1 g16, E4M3 scales, FP32 tensor scales     */
  SVDQ_INT4 = 1,            /* W4A4, symmetric INT4 g64, BF16 scales               */
  SVDQ_W4A16_INT4 = 2,      /* weight-only INT4 g64 (adaptive-norm linears)        */
  SVDQ_W8A8_INT8 = 3        /* W8A8: INT8, one FP32 scale per token / output channel,
                               low-rank branch of rank 16                           */
} svdq_format;

/* Offline configuration.  rank: 32 for the 4-bit formats, 16 for SVDQ_W8A8_INT8
 * (SOTA-314 practice page, "Do this": rank 32 at 4 bits, 16 at 8 bits), or 0
 * = no low-rank branch; alpha:
 * smoothing migration strength (0.5).  flags: SVDQ_PREP_* bits (0 = the
 * round-to-nearest residual). */
typedef struct {
  int format;
  int rank;
  float alpha;
  unsigned flags;
} svdq_config;

/* Preparation flags.
 *
 * SVDQ_PREP_GPTQ quantizes the residual with GPTQ instead of round-to-nearest
 * (SOTA-314 practice page, "Do this": the residual is quantized with GPTQ, which
 * improves quality in most of the paper's settings).  The pages do not restate
 * GPTQ; this is the published algorithm (Frantar et al. 2022) in its plain
 * column-by-column form:
 *   H = X_hat^T X_hat over the calibration batch, X_hat = fp32(Xc / lam) (the
 *       smoothed activations the residual multiplies); a channel with H_kk = 0
 *       gets H_kk = 1; every H_kk then grows by 1% of the mean diagonal;
 *   U = the upper-triangular Cholesky factor of H^-1 (H^-1 = U^T U);
 *   the input channels k are visited in order: where k starts a group (16 for
 *       NVFP4, 64 for INT4) that group's scale is fixed from the current
 *       values, w_k is quantized with it exactly as round-to-nearest would,
 *       err = (w_k - deq_k) / U_kk, and every later channel j moves by
 *       -U_kj err.  Working values are float64; the quantizer sees their
 *       float32 rounding.  The NVFP4 tensor scale g_w still comes from R.
 * Only the W4A4 formats (it needs the calibration batch); the forward kernels
 * and the layout of the prepared codes are unchanged.  Host cost: a K x K
 * factorisation (about K^3 / 3 multiply-adds twice) and K^2 N / 2 updates.
 *
 * SVDQ_PREP_KEEP_GPTQ_FACTOR (with SVDQ_PREP_GPTQ) keeps U on the host for
 * svdq_export(SVDQ_T_GPTQ_U) -- K^2 doubles, e.g. 75 MB at K = 3072; without it
 * U is freed when svdq_prepare returns. */
#define SVDQ_PREP_GPTQ             0x1u
#define SVDQ_PREP_KEEP_GPTQ_FACTOR 0x2u

typedef struct svdq_layer svdq_layer;   /* opaque */

/* Read-only description of a prepared layer. */
typedef struct {
  int K, N, rank, format;
  int device;               /* CUDA ordinal, or -1 for a host-only layer           */
  int g_x_exp, g_w_exp;     /* NVFP4 tensor scales g = 2^exp (0 for INT4)          */
  int svd_iterations;       /* subspace steps the SVD took (on W_hat and, for a
                               flat spectrum, on its smaller Gram matrix)        */
  double svd_tail_energy;   /* ||W_hat||_F^2 - sum_{i<r} sigma_i^2                 */
} svdq_layer_info;

/* Forward flags. */
#define SVDQ_FWD_GELU      0x1u  /* tanh-GELU on the output (fc1 -> fc2 chains)      */
#define SVDQ_FWD_UNFUSED   0x2u  /* measurement variant: separate down-projection,
                                    quantize, bare GEMM and up-projection launches   */
#define SVDQ_FWD_NO_BRANCH 0x4u  /* measurement variant: bare W4A4 GEMM + bias,
                                    low-rank branch skipped (output is NOT the layer) */
#define SVDQ_FWD_CHECK     0x8u  /* synchronise the stream and report a device
                                    timeout as SVDQ_ETIMEOUT                          */

/* Tensors that svdq_export copies to the host (logical, unswizzled layouts). */
typedef enum {
  SVDQ_T_LAMBDA = 0,        /* float [K]       smoothing factors lam                */
  SVDQ_T_INV_LAMBDA = 1,    /* float [K]       fp32(1 / lam)                        */
  SVDQ_T_L1 = 2,            /* double [K][r]   U Sigma[:, :r] of W_hat              */
  SVDQ_T_L2 = 3,            /* double [r][N]   V^T[:r, :]                           */
  SVDQ_T_L1D = 4,           /* uint16 [K][r]   bf16(diag(1/lam) L1)  (BF16 bits)    */
  SVDQ_T_L2B = 5,           /* uint16 [r][N]   bf16(L2)                             */
  SVDQ_T_RESIDUAL = 6,      /* float [K][N]    R = fp32(W_hat - diag(lam) L1d L2b)  */
  SVDQ_T_SIGMA = 7,         /* double [r]      leading singular values of W_hat     */
  SVDQ_T_W_CODES = 8,       /* uint8 [N][K/2]  residual codes, K-major, even k low  */
  SVDQ_T_W_SCALES = 9,      /* NVFP4: uint8 [N][K/16] E4M3; INT4: uint16 [N][K/64] BF16;
                               W8A8: float [N] (W_CODES is then int8 [N][K])         */
  SVDQ_T_BIAS = 10,         /* float [N]                                            */
  SVDQ_T_GPTQ_U = 11,       /* double [K][K]   GPTQ factor U (upper, H^-1 = U^T U); only
                               with SVDQ_PREP_GPTQ | SVDQ_PREP_KEEP_GPTQ_FACTOR      */
  SVDQ_T_LORA_A = 12,       /* uint16 [K][r]   LoRA down factor A as attached (BF16)  */
  SVDQ_T_LORA_B = 13,       /* uint16 [r][N]   bf16(scale * B), the stored up factor  */
  SVDQ_T_COUNT = 14
} svdq_tensor;

/* ------------------------------------------------------------------ offline */

/* svdq_prepare -- smoothing, truncated SVD and residual quantization
 * (SOTA-314 "Do this": smooth, "compute the SVD of the smoothed weight, keep
 * the top r singular directions in 16 bits, and quantize only the residual").
 *
 *   cfg        format, rank (0 or 32), alpha (> 0 and < 1; 0.5 recommended),
 *              flags (SVDQ_PREP_*; unknown bits, or SVDQ_PREP_GPTQ with
 *              SVDQ_W4A16_INT4, or KEEP without GPTQ give SVDQ_EINVAL).
 *   K, N       input and output features.
 *   W_bf16     host, [K][N] row-major BF16 weight (Y = X W + b); read only.
 *   bias_bf16  host, [N] BF16, or NULL for no bias.
 *   calib_bf16 host, [M_calib][K] BF16 calibration activations (smoothing
 *              maxima and the activation tensor scale); required for the W4A4
 *              formats, ignored (may be NULL) for SVDQ_W4A16_INT4.
 *   device     CUDA ordinal that receives the prepared buffers, or -1 to keep
 *              the layer on the host (export only; forwards return SVDQ_ESTATE);
 *              below -1: SVDQ_EINVAL; a device the process cannot use:
 *              SVDQ_ECUDA.
 *   out        receives the new layer; owned by the caller, free with svdq_destroy.
 *
 * Runs on the host (multi-threaded), then copies the prepared buffers to
 * `device` with blocking copies.  Errors: SVDQ_EINVAL (also for a NaN or an
 * infinity in W, the bias or the calibration batch), SVDQ_EUNSUPPORTED (shape
 * rules; for SVDQ_NVFP4 also a calibration batch whose largest smoothed
 * magnitude puts the activation tensor-scale exponent outside [-40, 30], i.e.
 * below about 3e-10 or above about 7e11), SVDQ_ENOMEM, SVDQ_ECUDA,
 * SVDQ_ENOCONVERGE (the SVD's energy check failed, or the GPTQ Hessian was
 * not positive definite after damping).
 * On error *out is set to NULL and nothing leaks. */
svdq_status svdq_prepare(const svdq_config* cfg, int K, int N,
                         const uint16_t* W_bf16, const uint16_t* bias_bf16,
                         const uint16_t* calib_bf16, int M_calib,
                         int device, svdq_layer** out);

/* Frees the layer and its device buffers; NULL is a no-op. */
void svdq_destroy(svdq_layer* layer);

/* Fills *info; SVDQ_EINVAL for a NULL argument. */
svdq_status svdq_get_info(const svdq_layer* layer, svdq_layer_info* info);

/* Bytes of tensor `id` (0 if the layer's format has no such tensor, for an
 * unknown id or a NULL layer). */
size_t svdq_tensor_bytes(const svdq_layer* layer, int id);

/* Copy tensor `id` into host memory `dst` of `bytes` (must equal
 * svdq_tensor_bytes, which must not be 0; else SVDQ_EINVAL).  Host-side; no
 * GPU work. */
svdq_status svdq_export(const svdq_layer* layer, int id, void* dst, size_t bytes);

/* A short English description of `s`; never NULL ("unknown status" for a
 * value outside svdq_status). */
const char* svdq_status_string(svdq_status s);

/* svdq_set_lora -- attach a LoRA adapter (W -> W + scale A B) to the layer's
 * 16-bit low-rank branch without re-quantizing anything.  SOTA-314 practice
 * page, "Known implementations": the paper's engine loads off-the-shelf LoRA
 * adapters without re-quantization.  The branch becomes
 *     X L1d L2b + X A bf16(scale B),
 * i.e. L1d' = [L1d | A], L2b' = [L2b ; bf16(scale B)] (rank 32 + r); smoothing,
 * residual codes and scales are untouched.
 *
 *   r          adapter rank, 1..32; 0 removes the adapter (A, B ignored).
 *   A_bf16     host, [K][r] BF16 (acts on the unsmoothed input X); copied.
 *   B_bf16     host, [r][N] BF16; copied as bf16(scale * B), one rounding.
 *   scale      the adapter's scaling (e.g. alpha / r); finite.
 *
 * Forward cost: one more pass of the first kernel's down projection over X
 * (XL columns 32..63 = bf16(X A)), and one more pipeline stage per output tile
 * in the NVFP4 GEMM (XL_lora times bf16(scale B) into the same accumulator);
 * the INT4 GEMM reloads its branch buffer with the adapter's tiles within each
 * tile, into the same accumulator as well.  With an adapter attached, XL is [M][64]
 * BF16 (columns 32..63: X A, zero-padded past r) wherever the API exposes it,
 * and svdq_workspace_bytes grows accordingly.  Blocking: synchronizes the
 * device before replacing the adapter's device buffers, so no forward of this
 * layer may be pending on another thread.  Errors: SVDQ_EINVAL (r < 0, null
 * factors, non-finite scale), SVDQ_EUNSUPPORTED (r > 32, a SVDQ_W4A16_INT4 or
 * SVDQ_W8A8_INT8 layer), SVDQ_ENOMEM, SVDQ_ECUDA.  The fc1 -> fc2 chain (svdq_mlp_*) does not take
 * layers with an adapter (SVDQ_EUNSUPPORTED). */
svdq_status svdq_set_lora(svdq_layer* layer, int r, const uint16_t* A_bf16, const uint16_t* B_bf16,
                          float scale);

/* Checkpoints.  svdq_serialize writes a prepared layer (scalars, lam, 1/lam,
 * sigma, L1d, L2b, residual codes and scales, bias, and a LoRA adapter if one
 * is attached) into `bytes` == svdq_serialized_bytes(layer) bytes of host
 * memory `dst`; svdq_deserialize rebuilds the layer from such bytes, on
 * `device` (or host-only with -1), without repeating the SVD or the
 * quantization.  Preparation-only intermediates (the residual R, the float64
 * L1 and L2, the GPTQ factor) are not stored: their svdq_tensor_bytes are 0 on
 * a deserialized layer.  The byte layout is "SVDQ", a version (2), the scalar
 * fields, then each array as a 64-bit byte count and its bytes, then a 64-bit
 * FNV-1a checksum of all the bytes before it (host byte order throughout).
 * svdq_deserialize checks the checksum and every size against the shape and
 * format, and returns SVDQ_EINVAL on any mismatch, corruption or truncation;
 * SVDQ_ENOMEM, SVDQ_ECUDA as for svdq_prepare. */
size_t svdq_serialized_bytes(const svdq_layer* layer);
svdq_status svdq_serialize(const svdq_layer* layer, void* dst, size_t bytes);
svdq_status svdq_deserialize(const void* src, size_t bytes, int device, svdq_layer** out);

/* ------------------------------------------------------------------ forward */

/* Workspace bytes a forward over M tokens needs (activation codes, scales in the
 * tensor-core layout and the BF16 down projection X L1d).  0 on bad input. */
size_t svdq_workspace_bytes(const svdq_layer* layer, int M);

/* svdq_linear_forward -- the inference path.
 *   X          device, [M][K] BF16 row-major, 16-byte aligned.
 *   Y          device, [M][N] BF16 row-major, 16-byte aligned; fully overwritten.
 *   workspace  device, >= svdq_workspace_bytes(layer, M), 256-byte aligned.
 *   flags      SVDQ_FWD_* bits.
 * SVDQ_W8A8_INT8 enqueues three: a per-token scale pass over X (the largest
 * smoothed magnitude of each row), the first kernel (INT8 codes, rank-16 down
 * projection) and an INT8 tensor-core GEMM (exact int32 products, both scales
 * and the branch applied in the epilogue).
 * W4A4 formats enqueue two kernels: the fused down-projection + quantize pass
 * over X ("Down Projection with Quantize, because they read the same input")
 * and the block-scaled tensor-core GEMM whose epilogue adds the up-projection
 * and the bias ("Up Projection with the 4-bit compute, because they write the
 * same output"; SOTA-314 "Do this").  For SVDQ_INT4 the GEMM dequantizes each
 * group of 64 codes times its BF16 scale into FP16 on chip (exact: 3 + 8
 * significant bits) and multiplies on the FP16 tensor cores, since the B200
 * has no 4-bit integer MMA.  Exact for every group scale between 2^-24 of
 * the calibration batch's largest smoothed activation and about 220 times it;
 * a group whose smoothed activations exceed that upper limit is clamped to it
 * (its contribution shrinks by the ratio), and smaller scales are rounded to
 * FP16 subnormals (an absolute error below 2^-32 of the calibration maximum).
 * SVDQ_W4A16_INT4 (the adaptive-norm linears, "stay W4A16") enqueues one
 * weight-only GEMV kernel meant for a few
 * rows (M <= 16), needs no workspace (pass NULL, 0) and accepts only
 * SVDQ_FWD_CHECK among the flags.  The W4A4 kernels are programmatic dependent
 * launches: their prologues may overlap the preceding kernel on the stream,
 * but each waits for that kernel to complete before it reads its inputs or
 * writes anything, so stream order is kept. */
svdq_status svdq_linear_forward(const svdq_layer* layer, const void* X, int M, void* Y,
                                void* workspace, size_t workspace_bytes,
                                void* stream, unsigned flags);

/* The first kernel alone (NVFP4/INT4/W8A8).  Writes
 *   codes   device, svdq_act_code_bytes(layer, M) bytes: the 4-bit formats hold
 *           two codes per byte, the even k in the low nibble (INT4: 4-bit two's
 *           complement, row-major [M][K/2]; NVFP4: the GEMM's tiled layout, see
 *           svdq_act_codes_to_logical); W8A8 one int8 per byte in the tiled
 *           layout;
 *   scales  device, svdq_act_scale_bytes(layer, M) bytes: NVFP4 E4M3 in the
 *           tensor-core layout, INT4 BF16 [K/64][M rounded up to 128]
 *           (group-major), W8A8 FP32 [s_x | 1/s_x], each M rounded up to 128
 *           entries; padding rows zero;
 *   xl      when the layer has a branch, XL = bf16(X L1d): device [M][32] BF16
 *           whatever the rank (X L1d in the first `rank` columns, zeros after),
 *           [M][64] with a LoRA adapter (see svdq_set_lora); may be NULL for
 *           rank 0 without an adapter.
 * X and every output buffer 16-byte aligned (else SVDQ_EINVAL).  W8A8 runs its
 * per-token scale pass first (not in mode 2).  `mode` 0 = fused, 1 = quantize
 * only, 2 = down projection only. */
svdq_status svdq_quantize_act(const svdq_layer* layer, const void* X, int M,
                              void* codes, void* scales, void* xl,
                              void* stream, int mode);

/* The second kernel alone: Y from the first kernel's outputs (codes, scales,
 * xl and Y 16-byte aligned, else SVDQ_EINVAL).  flags: SVDQ_FWD_GELU,
 * SVDQ_FWD_NO_BRANCH, SVDQ_FWD_CHECK. */
svdq_status svdq_gemm(const svdq_layer* layer, const void* codes, const void* scales,
                      const void* xl, int M, void* Y, void* stream, unsigned flags);

/* Bytes of the activation codes for M tokens in the layout the GEMM reads:
 * INT4 M * K/2; NVFP4 ceil(M/128)*128 * ceil(K/256) * 128 (tiled); W8A8
 * ceil(M/128)*128 * ceil(K/128) * 128 (tiled, one byte per code). */
size_t svdq_act_code_bytes(const svdq_layer* layer, int M);

/* Host-side: convert a host copy of activation codes in the GEMM's layout
 * (svdq_act_code_bytes bytes) into the logical row-major [M][K/2] bytes.  The
 * NVFP4 layout stores, for each block of 128 rows and each stage of 256 codes
 * (128 bytes of a row), one contiguous 16 KiB block in which byte j of row r
 * sits at (r % 128) * 128 + (((j / 16) ^ (r % 8)) * 16) + j % 16: the order in
 * which the tensor core reads a 128-byte-swizzled operand tile, so the GEMM
 * fetches each stage with one contiguous copy.  W8A8 uses the same blocks for
 * stages of 128 one-byte codes and converts to int8 [M][K]. */
svdq_status svdq_act_codes_to_logical(const svdq_layer* layer, const void* device_layout,
                                      int M, void* logical);

/* Bytes of the activation scales for M tokens in the layout the GEMM reads. */
size_t svdq_act_scale_bytes(const svdq_layer* layer, int M);

/* Host-side: convert a host copy of activation scales in the GEMM's layout
 * (svdq_act_scale_bytes bytes) into the logical layout: NVFP4 uint8 [M][K/16],
 * INT4 uint16 [M][K/64] (BF16 bits), W8A8 float [M] (s_x). */
svdq_status svdq_act_scales_to_logical(const svdq_layer* layer, const void* device_layout,
                                       int M, void* logical);

/* Synchronise `stream` and report (and clear) the layer's device error word:
 * SVDQ_ETIMEOUT if a bounded device wait expired since the last check. */
svdq_status svdq_check(const svdq_layer* layer, void* stream);

/* ------------------------------------------------------------------ fc1 -> fc2 chain */

/* The transformer MLP fc1 -> tanh-GELU -> fc2 with fc2's input produced
 * already quantized by fc1's GEMM epilogue.  The pages fuse the down projection
 * with the quantizer "because they read the same input" (SOTA-314 practice
 * page, "Do this"; NOTE-257 note page, "Key results"); in the MLP that input
 * is fc1's output, so fc1's epilogue rounds y = [gelu](fc1 output) to BF16
 * -- the value fc2 would read -- and writes fc2's NVFP4 codes and scales from
 * it with fc2's own quantizer arithmetic, bit for bit what svdq_quantize_act
 * would write for that y, plus partial sums of fc2's down projection y L1d2
 * over the fc1 tiles each CTA owns.  A second small kernel adds the partials
 * of each row in a fixed order (deterministic; XL2 = bf16 of an FP32 sum whose
 * order differs from the first kernel's, so XL2 may differ from it by a BF16
 * rounding).  fc1's BF16 output and fc2's first kernel disappear from the path.
 *
 * Both layers: SVDQ_NVFP4, prepared on the same device, without a LoRA
 * adapter, fc1's N equal to fc2's K (else SVDQ_EUNSUPPORTED).  fc2's calibration batch (its lam and
 * activation tensor scale) is used as is.
 *
 * svdq_mlp_workspace_bytes: workspace of svdq_mlp_forward (and of
 *   svdq_mlp_fc1) for M tokens; flags as for svdq_mlp_forward (UNFUSED needs
 *   room for fc1's BF16 output).  0 on bad input.
 * svdq_mlp_fc1: fc1's first kernel, fc1's GEMM in chain mode and the partial
 *   sum.  codes2 / scales2 / xl2 (device, 16-byte aligned) receive fc2's
 *   activation codes (svdq_act_code_bytes(fc2, M)), scales
 *   (svdq_act_scale_bytes(fc2, M)) and XL2 ([M][32] BF16; may be NULL when fc2
 *   has rank 0) in the layouts svdq_quantize_act(fc2, ...) writes, ready for
 *   svdq_gemm(fc2, ...).  flags: SVDQ_FWD_GELU, SVDQ_FWD_CHECK.
 * svdq_mlp_forward: svdq_mlp_fc1, then fc2's GEMM: Y (device, [M][fc2 N]
 *   BF16).  flags: SVDQ_FWD_GELU (GELU after fc1; the MLP), SVDQ_FWD_CHECK, and
 *   SVDQ_FWD_UNFUSED (measurement variant: the two layers' forwards one after
 *   the other, fc1's BF16 output through HBM).
 * X, workspace: as for svdq_linear_forward.  Errors as for svdq_linear_forward;
 * a device timeout in either layer is reported with SVDQ_FWD_CHECK. */
size_t svdq_mlp_workspace_bytes(const svdq_layer* fc1, const svdq_layer* fc2, int M, unsigned flags);
svdq_status svdq_mlp_fc1(const svdq_layer* fc1, const svdq_layer* fc2, const void* X, int M,
                         void* codes2, void* scales2, void* xl2,
                         void* workspace, size_t workspace_bytes, void* stream, unsigned flags);
svdq_status svdq_mlp_forward(const svdq_layer* fc1, const svdq_layer* fc2, const void* X, int M, void* Y,
                             void* workspace, size_t workspace_bytes, void* stream, unsigned flags);

/* svdq_selftest_wait_timeout -- exercise the failure-detection path.
 *
 * Enqueues on `stream` a one-thread kernel that waits on a device barrier
 * nothing ever arrives at, with the same bounded wait every kernel of the
 * library uses.  After budget_us microseconds (1 .. 10,000,000) the wait gives
 * up, records a timeout in the layer's device error word and the kernel ends:
 * no fault, no trap, no hang, and the device stays usable.  The next
 * svdq_check on the layer then returns SVDQ_ETIMEOUT (and clears the word).
 * Errors: SVDQ_EINVAL (NULL layer, budget out of range), SVDQ_ESTATE (host-only
 * layer), SVDQ_ECUDA (launch failed). */
svdq_status svdq_selftest_wait_timeout(const svdq_layer* layer, unsigned budget_us, void* stream);

/* ------------------------------------------------------- allocation-free forward */

/* Size of the library's built-in device workspace (16 MiB). */
#define SVDQ_STATIC_WORKSPACE_BYTES (16u << 20)

/* svdq_linear_forward_static -- svdq_linear_forward without a caller workspace.
 *
 * (No counterpart on the method's pages: this is a deployment convenience.)
 * For callers that cannot allocate device memory when they run a layer -- code
 * inside a framework's memory pool or arena without access to its allocator,
 * runtimes that forbid allocation after start-up, plug-ins that only receive
 * input and output pointers -- the workspace is a fixed array of
 * SVDQ_STATIC_WORKSPACE_BYTES in the library's own device memory.  The CUDA
 * driver creates it on every device that loads the library and keeps it until
 * the process exits.  This call allocates and frees nothing.
 *
 *   X, M, Y, stream, flags  as for svdq_linear_forward.
 * A SVDQ_W4A16_INT4 layer needs no workspace and runs exactly as
 * svdq_linear_forward(layer, X, M, Y, NULL, 0, stream, flags).
 * Returns SVDQ_EUNSUPPORTED if svdq_workspace_bytes(layer, M) exceeds
 * SVDQ_STATIC_WORKSPACE_BYTES (for K = 3072: M above 9,349 tokens), and
 * SVDQ_ECUDA if the workspace address cannot be obtained.
 *
 * The first call on a device looks up the array's device address (once, with
 * that device made current); make that first call before any stream capture.
 * All calls share the one array, which keeps the last call's contents (the
 * forward needs no zeroed workspace): calls whose work overlaps on the GPU --
 * on different streams, or on different layers at once -- race and must not be
 * issued. */
svdq_status svdq_linear_forward_static(const svdq_layer* layer, const void* X, int M, void* Y,
                                       void* stream, unsigned flags);

#ifdef __cplusplus
}
#endif

#endif /* SVDQ_H */
