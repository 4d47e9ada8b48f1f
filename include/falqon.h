/*
 * falqon.h - C ABI of libfalqon, the B200 (sm_100a) hot path of FALQON's
 * melded FP8 linear layer: one training step of an FP8-quantized linear layer
 * whose LoRA adapter is merged into the quantized backbone.
 *
 * Method: "FALQON: Accelerating LoRA Fine-tuning with Low-Bit Floating-Point
 * Arithmetic" (NeurIPS 2025).  The paper's introduction states the problem
 * this interface follows: quantize activations and gradients per tensor,
 * run the forward and backward on the FP8 backbone alone (no separate LoRA
 * path), compute the adapter gradients, and fold the adapter update back
 * into the backbone with a row-wise proxy.
 *
 * Conventions shared by every call
 * --------------------------------
 *  - All matrices are row-major and contiguous.  bfloat16 tensors are passed
 *    as `void*` holding IEEE bfloat16 values; FP8 tensors as `uint8_t*`
 *    holding OCP E4M3 codes (E5M2 codes where a call's name ends in _e5m2);
 *    scales as `float*` (one float, on the device).
 *  - Every tensor pointer is a DEVICE pointer and must be 16-byte aligned.
 *    The caller owns every buffer; the library allocates no device memory.
 *  - `stream` is a cudaStream_t passed as `void*` (NULL = legacy default
 *    stream).  Every call is asynchronous on that stream and performs no
 *    host synchronisation; scales never leave the device.
 *  - Shape, null-pointer, alignment and workspace errors are reported by the
 *    return value BEFORE anything is launched.  FALQON_ERR_CUDA reports a
 *    failed launch.  Data-dependent conditions found while running
 *    (non-finite input, scale overflow, a bounded wait that ran out) are
 *    OR-ed into `*dev_status` (an int32 in device memory, nullable) as
 *    FALQON_DEV_* bits; the caller reads it after its own synchronisation.
 *  - `workspace` is caller-owned device memory of at least
 *    falqon_workspace_size(op, ...) bytes, 256-byte aligned; it may be NULL
 *    when that size is 0.  Calls that overlap on the GPU must not share a
 *    workspace.  No other aliasing between arguments is allowed except the
 *    documented in-place operands of falqon_proxy_update.
 *  - A workspace given to falqon_quantize or falqon_quantize_e5m2 must be
 *    initialised once, before its first use, by falqon_workspace_init (or
 *    filled with zero bytes by the caller).  Every quantize call leaves it
 *    initialised for the next, whatever the size of the tensor and
 *    whether or not a bounded wait ran out (FALQON_DEV_TIMEOUT): the calls
 *    keep a generation counter in it, and each call zeroes only the word
 *    the next call folds its maximum into, so no clearing step runs per
 *    call.  Other workspaces need no initialisation.
 *  - Every function is reentrant; the only global state is a per-device
 *    cache of device attributes and of the driver's tensor-map encoder.
 */
#ifndef FALQON_H_
#define FALQON_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FALQON_API __attribute__((visibility("default")))
#else
#define FALQON_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum falqon_status {
  FALQON_OK = 0,
  FALQON_ERR_INVALID_ARG = 1, /* null pointer, negative or zero size, bad flag */
  FALQON_ERR_UNSUPPORTED = 2, /* shape or alignment outside what the kernels take */
  FALQON_ERR_WORKSPACE = 3,   /* workspace too small or misaligned */
  FALQON_ERR_CUDA = 4         /* a CUDA runtime or driver call failed */
} falqon_status;

typedef enum falqon_dtype {
  FALQON_DTYPE_BF16 = 0,
  FALQON_DTYPE_F32 = 1
} falqon_dtype;

typedef enum falqon_op {
  FALQON_OP_QUANTIZE = 0,
  FALQON_OP_LINEAR_FWD = 1,
  FALQON_OP_LINEAR_BWD = 2,
  FALQON_OP_PROXY_UPDATE = 3,
  FALQON_OP_PROXY_UPDATE_TOPK = 4,
  FALQON_OP_FOLDED_T = 5,          /* the buffer T of the folded forward keeps for the backward */
  FALQON_OP_LINEAR_BWD_FOLDED = 6, /* workspace of falqon_linear_bwd_folded (U, when dA is wanted) */
  FALQON_OP_SEPARATE_SAVED_BF16 = 7, /* what falqon_lora_separate_fwd keeps for the backward, bf16 path */
  FALQON_OP_SEPARATE_SAVED_FP8 = 8,  /* the same, FP8 path */
  FALQON_OP_SEPARATE_FWD_FP8 = 9,    /* workspace of the FP8 separate forward (a quantize workspace) */
  FALQON_OP_SEPARATE_BWD_BF16 = 10,  /* workspace of falqon_lora_separate_bwd, bf16 path */
  FALQON_OP_SEPARATE_BWD_FP8 = 11    /* the same, FP8 path */
} falqon_op;

/* Precision of the separate LoRA paths (falqon_lora_separate_fwd / _bwd). */
typedef enum falqon_separate_precision {
  FALQON_SEPARATE_BF16 = 0, /* adapter products in bf16 */
  FALQON_SEPARATE_FP8 = 1   /* every adapter operand quantized to E4M3 per product */
} falqon_separate_precision;

/* Bits OR-ed into *dev_status by the kernels. */
#define FALQON_DEV_NONFINITE 1      /* amax of an input was NaN or infinite */
#define FALQON_DEV_SCALE_OVERFLOW 2 /* fmax/amax overflowed (fmax 448 for E4M3, 57344 for E5M2);
                                       the scale was clamped to FLT_MAX */
#define FALQON_DEV_TIMEOUT 4        /* a bounded on-chip wait ran out; outputs are invalid */

/* Flags of falqon_proxy_update. */
#define FALQON_PROXY_ACCUMULATE 1u /* P += dB_inc . A */
#define FALQON_PROXY_SELECT 2u     /* select rows, requantize them, clear their proxy */
#define FALQON_PROXY_KEEP_RESIDUAL 4u /* with SELECT: keep the unapplied residual, no clear */
#define FALQON_PROXY_STRICT 8u        /* the strict float32 FMA chain in index order (the default) */
#define FALQON_PROXY_TENSOR 16u       /* with ACCUMULATE: the accumulation on the tensor cores (see
                                         falqon_proxy_update); not with STRICT */
#define FALQON_PROXY_DEFER_CLEAR 32u  /* with ACCUMULATE | SELECT: selected rows' proxy cleared by the next call
                                         (row_mask carried between calls; see falqon_proxy_update) */

/*
 * falqon_quantize - per-tensor E4M3 quantization.
 *
 * Defined by the OpenReview rebuttal of the paper (reviewer 2, W2, rewrite
 * of the scaling sentence): a higher-precision tensor X is multiplied by a
 * per-tensor scaling factor s_X and the product is rounded to FP8 (E4M3).
 * The scale formula is not printed; this library uses current max-abs
 * scaling:
 *     amax = max |x|,  s = 448 / amax (IEEE float32 division; 1 if amax == 0),
 *     code = E4M3_satfinite_rne( fl32(x * s) ).
 * The optional residual is the paper's quantization error of Eq. 8
 * (rebuttal to reviewer 2, Q3): R = x - code/s, computed in float64 and
 * rounded to float32; it is the implicit initial adapter of melded LoRA.
 *
 *  x         [rows, cols] bfloat16 or float32 (dtype), device, read-only.
 *  codes     [rows, cols] uint8 E4M3 codes, device, written.
 *  scale     1 float, device, written (s).
 *  amax      1 float, device, written; nullable.
 *  residual  [rows, cols] float32, device, written; nullable.
 *  Requirements: rows >= 1, cols >= 1, cols % 16 == 0.
 *  Device status: NONFINITE (s is set to 1), SCALE_OVERFLOW.
 */
FALQON_API falqon_status falqon_quantize(const void* x, falqon_dtype dtype, int64_t rows, int64_t cols,
                              uint8_t* codes, float* scale, float* amax, float* residual,
                              int32_t* dev_status, void* workspace, size_t workspace_bytes,
                              void* stream);

/*
 * falqon_quantize_e5m2 - per-tensor E5M2 quantization, for gradients.
 *
 * The rebuttal (reviewer 2, W2) names E5M2 beside E4M3 as an FP8 format
 * under the same per-tensor scaling.  As falqon_quantize with the E5M2 format
 * (sign, 5 exponent bits of bias 15, 2 mantissa bits; largest finite value
 * 57344): amax = max|x|, s = 57344 / amax (one IEEE float32 division; the
 * same status bits), codes = E5M2(fl32(x * s)), nearest-even, saturating
 * (every magnitude above 57344, infinity included, encodes as +-57344), NaN
 * as 0x7F.  No residual.  Arguments, requirements and workspace as
 * falqon_quantize (workspace: falqon_workspace_size(FALQON_OP_QUANTIZE, ...)).
 */
FALQON_API falqon_status falqon_quantize_e5m2(const void* x, falqon_dtype dtype, int64_t rows, int64_t cols,
                                   uint8_t* codes, float* scale, float* amax, int32_t* dev_status,
                                   void* workspace, size_t workspace_bytes, void* stream);

/*
 * falqon_linear_fwd - forward GEMM on the FP8 backbone alone.
 *
 * The paper's introduction: adapters are merged into the FP8 backbone, so the
 * forward needs no separate LoRA path and no extra quantization:
 *     Y[m,n] = sum_k dec(Xq[m,k]) * dec(Wq[n,k]) / (s_X * s_W),
 * accumulated in float32 on the tensor cores, scaled and rounded to bf16.
 *
 *  xq [M, K] E4M3, s_x 1 float; wq [N, K] E4M3 (PyTorch Linear layout:
 *  out x in), s_w 1 float; y [M, N] bfloat16, written.
 *  Requirements: M >= 1; N, K >= 16 and multiples of 16.
 */
FALQON_API falqon_status falqon_linear_fwd(const uint8_t* xq, const float* s_x, const uint8_t* wq,
                                const float* s_w, int64_t M, int64_t N, int64_t K, void* y,
                                int32_t* dev_status, void* workspace, size_t workspace_bytes,
                                void* stream);

/*
 * falqon_linear_fwd_grouped - the forward of up to three layers that read the
 * same activation, in one launch.
 *
 * In a transformer block the query, key and value projections (and the MLP's
 * gate and up projections) read the same input; under FALQON each is the
 * FP8 backbone alone (as falqon_linear_fwd), so one quantized X serves all of
 * them:  Y_s = bf16( Xq . Wq_s^T / (s_X s_W_s) ),  s = 0 .. nseg-1.
 * One tcgen05 GEMM walks the concatenated output tiles of the segments; each
 * output equals falqon_linear_fwd's on the same operands, bit for bit.
 *
 *  xq [M, K], s_x as falqon_linear_fwd.  nseg: 1 to 3.  wq, s_w, N, y: HOST
 *  arrays of nseg entries: wq[s] [N[s], K] E4M3 (device), s_w[s] 1 float
 *  (device), y[s] [M, N[s]] bfloat16 (device), written.
 *  Requirements: M >= 1; K and every N[s] multiples of 16.
 */
FALQON_API falqon_status falqon_linear_fwd_grouped(const uint8_t* xq, const float* s_x, int nseg,
                                                   const uint8_t* const* wq, const float* const* s_w,
                                                   const int64_t* N, void* const* y, int64_t M, int64_t K,
                                                   int32_t* dev_status, void* stream);

/*
 * falqon_linear_bwd - backward of the melded layer.
 *
 *   dX = dYq . Wq / (s_dY s_W)                      (backbone only; [M, K])
 *   T  = bf16( Xq . A^T / s_X )                     ([M, r], kept in workspace)
 *   dB = dYq^T . T / s_dY                           ([N, r])
 *   U  = bf16( dYq . B / s_dY ),  dA = U^T . Xq / s_X   ([r, K])
 * dB follows the rebuttal to reviewer 4 (Q1): B's gradient only needs A x,
 * known at forward time.  dA is that answer's formula B^T dL/dO x^T; the
 * paper freezes A, so dA is optional (NULL skips U and dA).
 *
 *  dyq [M, N] E4M3, s_dy; wq [N, K] E4M3, s_w; xq [M, K] E4M3, s_x;
 *  A [r, K] bfloat16; B [N, r] bfloat16 (read only when dA != NULL).
 *  dx [M, K], dA [r, K], dB [N, r]: bfloat16 outputs, each nullable.
 *  Requirements: M >= 1; N, K multiples of 16; r >= 16 and a multiple of 16.
 *  Workspace (dA or dB wanted): falqon_workspace_size(FALQON_OP_LINEAR_BWD,
 *  M, N, K, r) bytes.  Up to r = 496 (or M not a multiple of 8) T and U are
 *  kept as bf16 hi/lo planes, 4 * align256(round_up(M, 8) * r * 2) bytes;
 *  from r = 512 the four products run as bf16 GEMMs on codes expanded once,
 *  and the workspace also holds the expanded codes and the float32
 *  intermediates (2M(K+N) + 4rM + 4r round_up(M, 8) + 8r max(N, K) bytes,
 *  each part padded to 256).
 */
FALQON_API falqon_status falqon_linear_bwd(const uint8_t* dyq, const float* s_dy, const uint8_t* wq,
                                const float* s_w, const uint8_t* xq, const float* s_x,
                                const void* A, const void* B, int64_t M, int64_t N, int64_t K,
                                int64_t r, void* dx, void* dA, void* dB, int32_t* dev_status,
                                void* workspace, size_t workspace_bytes, void* stream);

/*
 * falqon_linear_bwd_e5m2 - falqon_linear_bwd with the gradient in E5M2.
 *
 * Identical to falqon_linear_bwd (same arguments, outputs, requirements and
 * workspace) except that dyq holds E5M2 codes and s_dy is their scale, as
 * falqon_quantize_e5m2 writes them: dX is a mixed E5M2 x E4M3 tcgen05 GEMM,
 * and U and dB read dYq through the E5M2 decoding.
 */
FALQON_API falqon_status falqon_linear_bwd_e5m2(const uint8_t* dyq, const float* s_dy, const uint8_t* wq,
                                     const float* s_w, const uint8_t* xq, const float* s_x,
                                     const void* A, const void* B, int64_t M, int64_t N, int64_t K,
                                     int64_t r, void* dx, void* dA, void* dB, int32_t* dev_status,
                                     void* workspace, size_t workspace_bytes, void* stream);

/*
 * falqon_linear_fwd_folded - forward with quantized adapters folded into the
 * backbone GEMM.
 *
 * The paper's Fig. 2 (as the rebuttal to reviewer 2, W1/W9, describes it)
 * multiplies the activations with quantized weights W~, A~ and B~, and the
 * rebuttal to reviewer 3 (W3.1) has backbone and adapters in FP8; B's
 * gradient needs only A x, known at forward time (rebuttal to reviewer 4,
 * Q1).  With A~q = E4M3 codes of A and s_a its scale (falqon_quantize of A),
 * one tcgen05 GEMM computes
 *     [Y | T] = Xq . [Wq ; A~q]^T,   Y as falqon_linear_fwd (bit-identical),
 *     T[m,i] = sum_k dec(Xq[m,k]) * dec(A~q[i,k]) / (s_X * s_A),
 * accumulated in float32 and kept for falqon_linear_bwd_folded.
 *
 *  xq [M, K], s_x; wq [N, K], s_w; aq [r, K] E4M3, s_a 1 float; y [M, N]
 *  bfloat16, written.
 *  t_saved: caller-owned device buffer of falqon_workspace_size(
 *    FALQON_OP_FOLDED_T, M, 0, 0, r) bytes (256-byte aligned), written: T
 *    transposed as two bfloat16 planes, hi then lo, each [r][ld] with
 *    ld = M rounded up to a multiple of 8 and the plane padded to 256 bytes;
 *    T[m,i] = hi[i][m] + lo[i][m] (about 16 significant bits).
 *  Requirements: M >= 1; N, K multiples of 16; r a multiple of 16.
 */
FALQON_API falqon_status falqon_linear_fwd_folded(const uint8_t* xq, const float* s_x, const uint8_t* wq,
                                       const float* s_w, const uint8_t* aq, const float* s_a, int64_t M,
                                       int64_t N, int64_t K, int64_t r, void* y, void* t_saved,
                                       size_t t_saved_bytes, int32_t* dev_status, void* stream);

/*
 * falqon_linear_bwd_folded - backward with quantized adapters folded into
 * the backbone GEMM (the counterpart of falqon_linear_fwd_folded).
 *
 * With B~q the E4M3 codes of B [N, r] and s_b its scale, one tcgen05 GEMM
 * computes [dX | U] = dYq . [Wq | B~q]: dX as falqon_linear_bwd
 * (bit-identical), U[m,i] = sum_n dec(dYq[m,n]) * dec(B~q[n,i]) / (s_dY s_B);
 * then one launch computes
 *     dB = dYq^T . T / s_dY     (T from the forward's t_saved)   [N, r]
 *     dA = U^T . Xq / s_X                                        [r, K]
 *
 *  dyq [M, N], s_dy; wq [N, K], s_w (read when dx != NULL); bq [N, r],
 *  s_b, xq [M, K], s_x (read when dA != NULL); t_saved as the forward wrote
 *  it (read when dB != NULL).  dx, dA, dB: bfloat16 outputs, each nullable.
 *  workspace: falqon_workspace_size(FALQON_OP_LINEAR_BWD_FOLDED, M, N, K, r)
 *  bytes when dA != NULL (U), else unused.
 *  Requirements: as falqon_linear_fwd_folded.
 */
FALQON_API falqon_status falqon_linear_bwd_folded(const uint8_t* dyq, const float* s_dy, const uint8_t* wq,
                                       const float* s_w, const uint8_t* bq, const float* s_b,
                                       const uint8_t* xq, const float* s_x, const void* t_saved,
                                       size_t t_saved_bytes, int64_t M, int64_t N, int64_t K, int64_t r,
                                       void* dx, void* dA, void* dB, int32_t* dev_status, void* workspace,
                                       size_t workspace_bytes, void* stream);

/*
 * falqon_proxy_update - row-wise proxy update of the quantized backbone.
 *
 * The abstract and introduction: a row-wise proxy accumulates the adapter
 * updates and selectively applies substantial ones to the FP8 backbone,
 * skipping updates that would vanish under quantization.  This library's
 * rule (the pages' own rule, a top-k over the r rank components with k not
 * given, is falqon_proxy_update_topk):
 *   ACCUMULATE: D[n,k] = float32 FMA chain over i = 0..r-1 of
 *               dB_inc[n,i] * A[i,k], starting at +0; P = fl32(P + D).
 *   SELECT:     t = fl32( dec(Wq[n,k]) + fl32(s_W * P[n,k]) ), c' = E4M3(t);
 *               row n is selected iff some c' differs in value from Wq[n,k]
 *               (+0 equals -0).  Selected rows: every code whose value
 *               changes becomes c'[n,k], codes of unchanged value keep their
 *               bits (so a zero keeps its sign), and P[n,:] = +0.  Other
 *               rows: Wq bit-identical, P kept.  The decoded backbone is the
 *               same as with a verbatim rewrite of the row.
 *   KEEP_RESIDUAL (with SELECT): the error-feedback variant of the clear
 *               (the pages drop nothing explicitly; clearing drops the
 *               sub-step residual): a code whose value changes keeps
 *               P = fl32(P - fl32(fl32(dec(c') - dec(old)) / s_W)); every
 *               other code keeps its proxy.  Row mask and count as SELECT.
 *   STRICT:     the accumulation is the strict float32 chain above, which
 *               is also the default.
 *   TENSOR:     (with ACCUMULATE, not STRICT) P = fl32(P + D) with
 *               D = dB_inc . A formed on the tensor cores: bf16 products
 *               (exact) summed in float32 in the hardware's order, which no
 *               fixed sequence reproduces.  For large r the chain's r FMAs
 *               per element bound it by the float32 pipe (at r = 8192 and
 *               N = K = 4096, 275 GFLOP); the tensor cores take them at bf16
 *               tensor rate.  SELECT then runs on the resulting P as a pass
 *               of its own (with both flags, or in a later call), and it
 *               is that pass that reports a non-finite P.
 *               Requirements: r a multiple of 8.
 *   DEFER_CLEAR: (with ACCUMULATE and SELECT; not with KEEP_RESIDUAL or
 *               TENSOR) the same
 *               update with the clear of the selected rows carried to the
 *               next call instead of written into P: row_mask is read on
 *               entry, and rows n with row_mask[n] != 0 (the previous call's
 *               selection) read P[n,:] as +0; P' is written for every row,
 *               and row_mask (then n_selected) receives this call's
 *               selection on exit.  The proxy the caller holds is P with the
 *               rows marked in row_mask read as +0: it equals, bit for bit,
 *               the P the eager clear leaves, and a chain of DEFER_CLEAR
 *               calls updates Wq exactly as the eager calls do.  The pass
 *               that zeroes the selected rows (about all of P when most rows
 *               change) and the reads of those rows' proxy disappear.
 *               row_mask is required; before the first call it holds zeros
 *               (or the selection of a previous eager call, whose clear
 *               already happened: zeros are then also correct).
 * The default float32 chain is reproduced bit-for-bit.
 *
 *  wq [N, K] E4M3, in/out;  s_w 1 float (the backbone's fixed scale);
 *  proxy [N, K] float32, in/out;  dB_inc [N, r] bfloat16 (the increment of
 *  B this step: the caller folds in sign and learning rate);  A [r, K] bf16.
 *  row_mask [N] uint8 (0/1) and n_selected (1 int32): written when SELECT is
 *  set; nullable (row_mask is required, and also read, with DEFER_CLEAR).
 *  Requirements: N >= 1; K multiple of 16; r >= 1 (r unused without
 *  ACCUMULATE); flags: ACCUMULATE and/or SELECT, plus KEEP_RESIDUAL only
 *  with SELECT, TENSOR only with ACCUMULATE, DEFER_CLEAR only with both
 *  ACCUMULATE and SELECT and neither KEEP_RESIDUAL nor TENSOR.
 */
FALQON_API falqon_status falqon_proxy_update(uint8_t* wq, const float* s_w, float* proxy,
                                  const void* dB_inc, const void* A, int64_t N, int64_t K,
                                  int64_t r, uint32_t flags, uint8_t* row_mask,
                                  int32_t* n_selected, int32_t* dev_status, void* workspace,
                                  size_t workspace_bytes, void* stream);

/*
 * falqon_proxy_update_topk - proxy update with top-k selection over the r
 * rank components of the adapter.
 *
 * The OpenReview rebuttal (reviewer 3, Q1) has the top-k step run over r
 * rows, r much smaller than the layer dimension, and shrink the inner
 * dimension of the weight update from r to k; the rebuttal to reviewer 2
 * (W7) has the update merged into the weight by that selection, saving
 * memory and update cost.  Neither the score nor k is printed.  This
 * library's reading: the proxy of this rule is Q [r, N] float32, row i
 * holding the part of B's column i (rank component i, whose update to the
 * weight is Q[i,:]^T A[i,:]) not yet merged into the backbone.
 *   ACCUMULATE: Q[i,n] = fl32( Q[i,n] + dB_inc[n,i] ).
 *   SELECT:     score_i = max_n |Q[i,n]| * max_k |A[i,k]| (exact, float64);
 *               a component whose Q or A row holds a non-finite value
 *               scores +infinity and sets FALQON_DEV_NONFINITE.  The chosen
 *               set S is the k components of highest positive score, ties
 *               to the lower index.  Merge: D[n,k] = float32 FMA chain over
 *               i in S in increasing order from +0 of Q[i,n] * A[i,k];
 *               t = fl32( dec(Wq[n,k]) + fl32(s_W * D[n,k]) ); every code
 *               whose value changes becomes E4M3(t), the others keep their
 *               bits.  Clear: Q[i,:] = +0 for i in S.
 *   STRICT:     accepted, changes nothing.
 * Merging every component equals falqon_proxy_update (both flags) applied
 * to a proxy P = 0 with dB_inc = Q^T: the whole r-term update.  The cost is
 * 2 N K |S| flops and one pass over Wq; no per-weight proxy exists.
 *
 *  wq [N, K] E4M3, in/out (read and written when SELECT); s_w 1 float.
 *  proxy_q [r, N] float32, in/out.
 *  dB_inc [N, r] bfloat16 (the increment of B this step; read when
 *  ACCUMULATE).  A [r, K] bfloat16 (read when SELECT).
 *  k >= 0: the largest number of components to merge.
 *  comp_mask [r] uint8 (0/1) and n_selected (1 int32): written when SELECT;
 *  nullable.
 *  flags: ACCUMULATE and/or SELECT, optionally STRICT; KEEP_RESIDUAL is
 *  rejected (FALQON_ERR_INVALID_ARG): this rule keeps no per-weight proxy.
 *  workspace: falqon_workspace_size(FALQON_OP_PROXY_UPDATE_TOPK, 0, N, K, r)
 *  bytes when SELECT (per-CTA maxima, the chosen list).
 *  Requirements: N >= 1 and below 2^31; K a multiple of 16; 1 <= r <= 16384
 *  (FALQON_ERR_UNSUPPORTED beyond); k >= 0.
 *  Launches: one with ACCUMULATE alone; with SELECT four (maxima, choice,
 *  merge, clear), two when k == 0; nothing is synchronised with the host.
 */
FALQON_API falqon_status falqon_proxy_update_topk(uint8_t* wq, const float* s_w, float* proxy_q,
                                       const void* dB_inc, const void* A, int64_t N, int64_t K,
                                       int64_t r, int64_t k, uint32_t flags, uint8_t* comp_mask,
                                       int32_t* n_selected, int32_t* dev_status, void* workspace,
                                       size_t workspace_bytes, void* stream);

/*
 * falqon_linear_bwd_noalloc - falqon_linear_bwd for callers that cannot
 * allocate device memory.
 *
 * The paper has no counterpart to this call.  It serves callers that cannot
 * call cudaMalloc on the hot path (a host program that only holds device
 * pointers to its own tensors under a fixed memory budget, a plugin inside a
 * runtime that owns every allocation): it takes the same arguments as
 * falqon_linear_bwd minus the workspace, and keeps the adapter products'
 * intermediates in one scratch array compiled into the library.
 *
 *  - Limit: the scratch array is 16 MiB per device, held by every GPU that
 *    loads the library until the process exits.  A call asking for dA or dB
 *    needs falqon_workspace_size(FALQON_OP_LINEAR_BWD, M, N, K, r) bytes of
 *    it (the same with or without dA; up to r = 496, 4 * align256(
 *    round_up(M, 8) * r * 2));
 *    beyond 16 MiB it returns FALQON_ERR_WORKSPACE before launching
 *    anything.  Every other argument error is reported first, exactly as
 *    falqon_linear_bwd reports it.  A dX-only call needs no scratch.
 *  - Set-up: the first call on a device that needs scratch looks up the
 *    array's device address (cudaGetSymbolAddress) and caches it; make that
 *    first call before any stream capture on that device.  A failed lookup
 *    returns FALQON_ERR_CUDA and is not cached: a later call tries again.
 *  - Sharing: every call uses the same array, which keeps the last call's
 *    contents (nothing in it needs to start at zero).  Calls that overlap on
 *    the GPU race on it; serialise them.
 *  - Allocation: none (no cudaMalloc, cudaFree or allocating library call).
 */
FALQON_API falqon_status falqon_linear_bwd_noalloc(const uint8_t* dyq, const float* s_dy,
                                                   const uint8_t* wq, const float* s_w,
                                                   const uint8_t* xq, const float* s_x,
                                                   const void* A, const void* B, int64_t M,
                                                   int64_t N, int64_t K, int64_t r, void* dx,
                                                   void* dA, void* dB, int32_t* dev_status,
                                                   void* stream);

/*
 * falqon_lora_separate_fwd / falqon_lora_separate_bwd - LoRA kept as a
 * separate path beside the FP8 backbone: the comparison FALQON is measured
 * against, not FALQON's own path (which merges the adapter into Wq).
 *
 * The paper's introduction sets FALQON against separate LoRA paths on an FP8
 * backbone, whose small adapter products each pay a quantization; the
 * OpenReview rebuttals compare FP8 and FP16 adapters across ranks (reviewer
 * 2, W4, Table R1; reviewer 3, Q3, Table R6).  The adapter branch is a
 * separate layer; each of its products is rounded to bf16 and the branch is
 * added to the backbone's bf16 output as bf16 tensors add (a float32 sum
 * rounded once to bf16):
 *   forward   Ybb = the backbone product (falqon_linear_fwd),
 *             S = bf16(X . A^T), Y = bf16(fl32(Ybb + bf16(S . B^T)))
 *   backward  dXbb = the backbone product (falqon_linear_bwd's dX),
 *             G = bf16(dY . B), dX = bf16(fl32(dXbb + bf16(G . A))),
 *             dB = bf16(dY^T . S), dA = bf16(G^T . X)
 * FALQON_SEPARATE_BF16: the adapter products take X, dY, A and B as bf16.
 * FALQON_SEPARATE_FP8: every adapter operand is quantized per tensor to
 * E4M3 right before its product (as falqon_quantize): X and dY are the
 * backbone's codes xq and dyq, A and B are quantized each forward, S and G
 * once formed; each product divides by its two scales.
 *
 * Forward arguments: xq, s_x and wq, s_w as falqon_linear_fwd; x [M, K] bf16
 * (read by the bf16 path); A [r, K], B [N, r] bf16; y [M, N] bf16, written.
 * saved: caller-owned, falqon_workspace_size(FALQON_OP_SEPARATE_SAVED_BF16 or
 * _FP8, M, N, K, r) bytes, written (S, and in FP8 the codes and scales of S,
 * A and B), read by the backward.  workspace: FP8 path only,
 * falqon_workspace_size(FALQON_OP_SEPARATE_FWD_FP8, ...) bytes, a quantize
 * workspace (initialise it once with falqon_workspace_init).
 *
 * Backward arguments: dyq, s_dy as falqon_linear_bwd; dy [M, N] bf16 (bf16
 * path); wq, s_w (read when dx is wanted); xq, s_x (FP8 path, for dA); x
 * (bf16 path, for dA); A, B and saved as the forward left them.  dx [M, K],
 * dA [r, K], dB [N, r]: bf16 outputs, each nullable, not all null.
 * workspace: falqon_workspace_size(FALQON_OP_SEPARATE_BWD_BF16 or _FP8, M, N,
 * K, r) bytes; it holds a quantize workspace, so initialise it once with
 * falqon_workspace_init.
 * Requirements: M >= 1; N, K, r multiples of 16; r <= 65536.
 */
FALQON_API falqon_status falqon_lora_separate_fwd(int precision, const uint8_t* xq, const float* s_x,
                                                  const void* x, const uint8_t* wq, const float* s_w,
                                                  const void* A, const void* B, int64_t M, int64_t N, int64_t K,
                                                  int64_t r, void* y, void* saved, size_t saved_bytes,
                                                  int32_t* dev_status, void* workspace, size_t workspace_bytes,
                                                  void* stream);
FALQON_API falqon_status falqon_lora_separate_bwd(int precision, const uint8_t* dyq, const float* s_dy,
                                                  const void* dy, const uint8_t* wq, const float* s_w,
                                                  const uint8_t* xq, const float* s_x, const void* x,
                                                  const void* A, const void* B, const void* saved,
                                                  size_t saved_bytes, int64_t M, int64_t N, int64_t K, int64_t r,
                                                  void* dx, void* dA, void* dB, int32_t* dev_status,
                                                  void* workspace, size_t workspace_bytes, void* stream);

/*
 * falqon_selftest_bounded_waits - exercises the failure detection on the GPU
 * without a fault.
 *
 * Every wait inside the library's kernels is bounded (about one second of
 * clock cycles); when it runs out, the kernel ORs FALQON_DEV_TIMEOUT into
 * *dev_status and returns, and the context stays usable.  This call launches
 * one small kernel whose waits cannot complete: an mbarrier wait (the kind
 * the tcgen05 and quantize kernels use) on a phase nothing arrives on, and a
 * bounded poll (the kind the quantize kernel's grid exchange uses) of *flag.
 * Each wait that gives up sets FALQON_DEV_TIMEOUT and a bit in *which: 1 for
 * the mbarrier wait (always), 2 for the poll (only while *flag stays 0).
 * Takes about one second.
 *
 *  flag: 1 int32, device, read.  dev_status, which: 1 int32 each, device,
 *  OR-ed into.
 */
FALQON_API falqon_status falqon_selftest_bounded_waits(const int32_t* flag, int32_t* dev_status,
                                                       int32_t* which, void* stream);

/*
 * falqon_workspace_init - prepares a workspace for its first use: fills
 * `workspace_bytes` bytes with zeros on `stream` (asynchronous).  Required
 * once for a quantize workspace (see the conventions above); harmless for
 * any other.  Errors: NULL or 0 bytes -> FALQON_ERR_INVALID_ARG; not 256-byte
 * aligned -> FALQON_ERR_WORKSPACE; the fill failed -> FALQON_ERR_CUDA.
 */
FALQON_API falqon_status falqon_workspace_init(void* workspace, size_t workspace_bytes, void* stream);

/* Workspace bytes `op` needs for these sizes (arguments an op ignores may be 0). */
FALQON_API size_t falqon_workspace_size(falqon_op op, int64_t M, int64_t N, int64_t K, int64_t r);

/* Static description of a status code. */
FALQON_API const char* falqon_status_string(falqon_status status);

/* Library version string. */
FALQON_API const char* falqon_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FALQON_H_ */
