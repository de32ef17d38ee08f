/*
 * sbl.h — C ABI of the Sparse-BitLinear layer on NVIDIA B200 (sm_100a).
 *
 * The operator (Sparse-BitNet Guide: 1.58-Bit LLMs Meet 2:4 Sparsity, section
 * "Mathematical Formulation of Sparse-BitLinear"):
 *
 *     y = ( x_q . W_t^T ) * scale_o / s_t
 *
 * with W_t the N:M-masked ternary weights, x_q the per-token absmax int8
 * activations, scale_o the per-row absmean of the kept weights
 * (halo-sparse-bitnet-3:4-500m card, "Recipe") and s_t = 127 / max|x_t|.
 * sbl_linear_backward gives its straight-through gradients for training.
 *
 * Conventions every entry point follows
 *   - All pointers are DEVICE pointers unless stated, owned by the caller, and
 *     16-byte aligned.  The library allocates no device memory: scratch space
 *     is a caller-provided workspace (see sbl_linear_workspace_bytes).
 *   - `stream` is a cudaStream_t passed as void*; NULL means the legacy
 *     default stream.  Every call is asynchronous on `stream`; it returns once
 *     the work is enqueued.
 *   - Argument errors are detected on the host before anything is enqueued and
 *     returned synchronously; a CUDA launch failure returns SBL_ERR_CUDA.
 *   - Conditions only the device can see (non-finite inputs, a pipeline wait
 *     that ran out) set bits in a per-device status word that
 *     sbl_device_status() reads; kernels never trap.
 *   - Shapes: row-major, int64 sizes; O, T >= 0 (zero sizes are no-ops);
 *     K > 0 and K % 16 == 0.  (n, m) must be (2,4), (3,4), (6,8) or (4,8).
 *   - Nothing throws across this boundary.
 */
#ifndef SBL_H
#define SBL_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SBL_OK = 0,
    SBL_ERR_INVALID_ARG = 1,   /* null/unaligned pointer, negative or bad size      */
    SBL_ERR_UNSUPPORTED = 2,   /* N:M pattern or shape outside what the kernels do  */
    SBL_ERR_NONFINITE = 3,     /* device saw NaN/Inf in W or x (sbl_device_status)  */
    SBL_ERR_CUDA = 4,          /* a CUDA runtime/driver call failed                 */
    SBL_ERR_TIMEOUT = 5,       /* a bounded device-side wait ran out                */
    SBL_ERR_WORKSPACE = 6      /* workspace missing, too small or unaligned         */
} sbl_status;

/* Most weight matrices one grouped call takes (sbl_prepare_weights_grouped,
 * sbl_linear_grouped). */
#define SBL_MAX_GROUP 8

/* Output element types of sbl_linear. */
enum { SBL_F32 = 0, SBL_BF16 = 1 };

/* Contraction paths of sbl_linear_path.  SBL_PATH_PREFILL lets the library
 * pick the tensor-core kernel; the others force one of them (tests, tuning):
 * one CTA per 128-token tile, a pair of CTAs on two SMs per 256-token tile,
 * or (2:4 weights only) the structured-sparse MMA on compressed weights. */
enum { SBL_PATH_AUTO = 0, SBL_PATH_DECODE = 1, SBL_PATH_PREFILL = 2,
       SBL_PATH_PREFILL_1CTA = 3, SBL_PATH_PREFILL_PAIR = 4, SBL_PATH_PREFILL_SPARSE = 5 };

/*
 * sbl_prepare_weights — N:M mask, per-row scale, ternarise and 2-bit pack.
 *
 * Follows the Sparse-BitNet Guide, "Mathematical Formulation of
 * Sparse-BitLinear" (mask equation: Top-N |W| of every M contiguous input-dim
 * weights; joint sparse-ternary equation W_t = mask * clip(round(W/scale),-1,1)),
 * the Sparse-BitNet README, "How It Works / Sparse-BitNet" (mask first, then
 * quantise what remains), and the halo-sparse-bitnet-3:4-500m card
 * ("Recipe": per-row absmean; "Packed vs raw": 2 bits per weight,
 * 00 = 0, 01 = +1, 10 = -1, four codes per byte).
 *
 *   W          fp32 [O, K] latent weights (input).
 *   O, K, n, m shape and N:M pattern; K % 16 == 0, K % m == 0.
 *   packed     uint8 [O, K/4] (output).  Weight k of a row is byte k/4,
 *              bits 2(k%4)..2(k%4)+1 (least significant code first).
 *   row_scale  fp32 [O] (output): mean of |W| over the kept weights of the
 *              row — the exact sum rounded once to double, divided by the
 *              kept count in double, rounded to float — clamped below at 1e-5.
 *   mask_bits  uint8 [O, K/8] (output, may be NULL): bit k%8 of byte k/8 is
 *              set when weight k is kept.  Ties in |W| keep the lower index.
 *   round(W/scale) is round-half-to-even; a weight is nonzero exactly when it
 *   is kept and |W| > scale/2.
 *   Non-finite W sets SBL_ERR_NONFINITE in the device status word; the
 *   outputs of such a row are unspecified.
 */
sbl_status sbl_prepare_weights(const float* W, int64_t O, int64_t K, int n, int m,
                               uint8_t* packed, float* row_scale, uint8_t* mask_bits,
                               void* stream);

/*
 * sbl_prepare_weights_ex — sbl_prepare_weights with convention flags.
 *
 *   flags  0, or SBL_PREP_SCALE_BF16: the row scale is stored as the halo
 *          card's "Packed vs raw" format keeps it, one bf16 row_scale per row:
 *          the fp32 scale above (after the 1e-5 clamp) is rounded to nearest
 *          even bf16, and that value ternarises the row and is written to
 *          row_scale (as fp32, exactly).
 *          SBL_PREP_SCALE_GLOBAL: one scale for the whole matrix, as the
 *          Sparse-BitNet Guide's module listing computes gamma: the mean of |W|
 *          over all O*K weights (masked ones included) — the exact sum rounded
 *          once to double, divided by O*K in double, rounded to float, clamped
 *          below at 1e-5 (then rounded to bf16 with SBL_PREP_SCALE_BF16) — used
 *          for every row and written to every row_scale entry.  Needs
 *          O*K < 2^32 (else SBL_ERR_UNSUPPORTED); calls with this flag on one
 *          device must be ordered, as they share a small static scratch.
 *          Other bits: SBL_ERR_INVALID_ARG.
 */
#define SBL_PREP_SCALE_BF16 1
#define SBL_PREP_SCALE_GLOBAL 2
sbl_status sbl_prepare_weights_ex(const float* W, int64_t O, int64_t K, int n, int m,
                                  uint8_t* packed, float* row_scale, uint8_t* mask_bits,
                                  int flags, void* stream);

/*
 * sbl_prepare_weights_grouped — sbl_prepare_weights for G weight matrices of
 * the same K in one call (the projections of one layer), with the per-row
 * scale and no flags.  W, O, packed, row_scale: HOST arrays of G entries
 * (device pointers, row counts O[g] >= 0); mask_bits: NULL or a host array of
 * G device pointers (entries may be NULL).  Each matrix's results are exactly
 * sbl_prepare_weights'; rows up to K = 8192 are prepared by one launch over
 * the stacked rows.  1 <= G <= SBL_MAX_GROUP, else SBL_ERR_INVALID_ARG.
 */
sbl_status sbl_prepare_weights_grouped(int G, const float* const* W, const int64_t* O, int64_t K, int n, int m,
                                       uint8_t* const* packed, float* const* row_scale, uint8_t* const* mask_bits,
                                       void* stream);

/*
 * sbl_quant_act — per-token absmax int8 activation quantisation.
 *
 * Follows the activation equation of the Sparse-BitNet Guide, "Mathematical
 * Formulation of Sparse-BitLinear" (beta = max_j |x_j| per token,
 * clip(round(x * 127 / beta), -128, 127)) and the BitNet-TinyDialogues card
 * (W1.58A8: 8-bit per-token activations).
 *
 *   x_bf16  bf16 bit patterns [T, K] (input).
 *   x_q     int8 [T, K] (output), natural column order.
 *   s_tok   fp32 [T] (output): s_t = 127 / max(max_k |x_tk|, 1e-5) in IEEE
 *           float division; x_q = clamp(round_half_even(x * s_t), -128, 127)
 *           with the product rounded to float.
 *   Non-finite x sets SBL_ERR_NONFINITE in the device status word; x_q and
 *   s_tok of that token are then unspecified.
 */
sbl_status sbl_quant_act(const uint16_t* x_bf16, int64_t T, int64_t K,
                         int8_t* x_q, float* s_tok, void* stream);

/*
 * sbl_rmsnorm_quant_act — RMSNorm, then per-token absmax int8 quantisation.
 *
 * The activation step of the Sparse-BitNet Guide, "Mathematical Formulation of
 * Sparse-BitLinear" (activations are normalised by RMSNorm before the absmax),
 * in the form of the guide's SparseBitLinear module listing (torch RMSNorm
 * over the K input features with an elementwise weight):
 *   x_norm = (x * (1 / sqrt(sum_k x_k^2 / K + eps))) * g
 * in float32, every step IEEE-rounded (the pages give no order; the sum of
 * squares is formed in a fixed one: lane l of 32 adds, in increasing k, the
 * squares of the 16-element blocks b with b % 32 == l, and the lane sums are
 * combined by an xor butterfly at offsets 16, 8, 4, 2, 1), then x_q and s_tok
 * exactly as sbl_quant_act computes them from x_norm.
 *
 *   x_bf16  bf16 bit patterns [T, K] (input), K % 16 == 0 like every entry
 *           point (else SBL_ERR_INVALID_ARG).
 *   g       fp32 [K] (input): the RMSNorm weight, 16-byte aligned.
 *   eps     finite, >= 0 (torch's default for float32 is 2^-23); else
 *           SBL_ERR_INVALID_ARG.
 *   x_q     int8 [T, K] (output), natural column order.
 *   s_tok   fp32 [T] (output): 127 / max(max_k |x_norm|, 1e-5).
 *   Non-finite x or a non-finite normalised value sets SBL_ERR_NONFINITE in
 *   the device status word; that token's outputs are then unspecified.
 */
sbl_status sbl_rmsnorm_quant_act(const uint16_t* x_bf16, const float* g, float eps, int64_t T, int64_t K,
                                 int8_t* x_q, float* s_tok, void* stream);

/*
 * sbl_mask_monitor — mask change rate and mask verification.
 *
 * The Sparse-BitNet README ("Features": dynamic mask monitoring during
 * training; its CLI monitors the mask change rate every N steps) and the
 * halo-sparse-bitnet-3:4-500m card ("Recipe": mask-verify every 500 steps).
 * Compares two mask bitmaps as sbl_prepare_weights writes them (uint8
 * [O, K/8], bit k % 8 of byte k / 8 set when weight k is kept, 16-byte
 * aligned):
 *   totals       uint64 [2] on the device (output, 8-byte aligned):
 *                totals[0] = positions whose kept state differs between
 *                old_bits and new_bits (the change rate is totals[0] / (O*K));
 *                totals[1] = M-groups of new_bits that do not keep exactly N.
 *   row_changed  uint32 [O] on the device (output, may be NULL): the changed
 *                positions of each row.
 * (n, m) as for sbl_prepare_weights.  Asynchronous on `stream`; totals are
 * overwritten (not accumulated).
 */
sbl_status sbl_mask_monitor(const uint8_t* old_bits, const uint8_t* new_bits, int64_t O, int64_t K, int n, int m,
                            uint64_t* totals, uint32_t* row_changed, void* stream);

/* Flags of sbl_linear_backward. */
enum { SBL_BWD_DW_TERNARY = 1 };

/*
 * sbl_linear_backward — straight-through (STE) gradients of sbl_linear, the
 * training path.
 *
 * The Sparse-BitNet Guide, "Training Stability & The Straight-Through
 * Estimator": the backward passes the N:M mask and the ternary rounding
 * unchanged to the latent weights (masked positions included, so a pruned
 * weight can re-enter the mask); the Sparse-BitNet README, "How It Works /
 * BitLinear": gradients pass the quantiser by straight-through estimation.
 * With the activation quantiser passed through too, the forward reads
 * y = x_hat . W_hat^T, x_hat[t,k] = x_q[t,k] / s_t, W_hat[o,k] = scale_o * W_t[o,k]:
 *
 *   dY         fp32 [T, O]: gradient of the loss with respect to y.
 *   x_q, s_tok the forward's int8 [T, K] activations in natural column order
 *              and fp32 [T] scales (sbl_quant_act / sbl_rmsnorm_quant_act).
 *   packed, row_scale  the prepared weights (sbl_prepare_weights), [O, K/4], [O].
 *   dX         fp32 [T, K] (output, may be NULL):
 *              dX[t,k] = sum_o dY[t,o] * scale_o * W_t[o,k] — the gradient at
 *              the quantiser's input (after the RMSNorm, for the fused front end).
 *   dW         fp32 [O, K] (output, may be NULL):
 *              dW[o,k] = sum_t dY[t,o] * x_q[t,k] / s_t; with
 *              SBL_BWD_DW_TERNARY each row is multiplied by scale_o once more
 *              (the gradient at the ternary matrix of the guide's equation
 *              y = (x~ . W~^T) * beta * gamma / 127, as its module returns it).
 * fp32 arithmetic with fused multiply-adds in an unspecified order: each
 * output is within (n + 2) * 2^-24 * sum |terms| of the exact value, n the
 * reduction length (O for dX, T for dW; n + 3 for SBL_BWD_DW_TERNARY).
 * Empty reductions write zeros (dW for T == 0, dX for O == 0).  Only the
 * pointers the requested outputs read must be valid.  At least one of dX, dW
 * must be non-NULL.
 * K % 16 == 0; any T, O >= 0.  Asynchronous on `stream`; no workspace.
 */
sbl_status sbl_linear_backward(const float* dY, int64_t T, int64_t O, const int8_t* x_q, const float* s_tok,
                               int64_t K, const uint8_t* packed, const float* row_scale, float* dX, float* dW,
                               int flags, void* stream);

/*
 * sbl_linear_backward_ws — the gradients of sbl_linear_backward on the tcgen05
 * tensor cores, with a caller-provided workspace.
 *
 * Same operation, arguments, flags and results as sbl_linear_backward (the
 * Sparse-BitNet Guide, "Training Stability & The Straight-Through
 * Estimator"), plus:
 *   workspace        device scratch of at least
 *                    sbl_linear_backward_workspace_bytes(T, O, K, dX != NULL,
 *                    dW != NULL) bytes, 256-byte aligned; contents on entry
 *                    do not matter (else SBL_ERR_WORKSPACE).  Calls that share
 *                    it must be ordered on one stream.
 * How: the fp32 factor of each product (dY * scale_o for dX, dY / s_t for dW,
 * each one IEEE rounding) is split exactly into three bf16 parts (hi, mid,
 * lo: its 24 significand bits in three 8-bit pieces); the other factor
 * (ternary W_t, or x_q with |x_q| <= 127) is exact in bf16; the workspace
 * holds both operands in bf16, K-major, and a kind::f16 tensor-core GEMM with
 * fp32 accumulation sums the 3n exact products.  Error: within
 * (n + 2) * 2^-24 * sum |terms| of the exact value for the tensor cores' fp32
 * accumulation as measured on B200 (n + 3 with SBL_BWD_DW_TERNARY); exact
 * where every partial sum is a float.  T and O up to 2^21, else
 * SBL_ERR_UNSUPPORTED.  Empty reductions (T == 0 or O == 0) write zeros and
 * need no workspace.
 */
size_t sbl_linear_backward_workspace_bytes(int64_t T, int64_t O, int64_t K, int need_dx, int need_dw);
sbl_status sbl_linear_backward_ws(const float* dY, int64_t T, int64_t O, const int8_t* x_q, const float* s_tok,
                                  int64_t K, const uint8_t* packed, const float* row_scale, float* dX, float* dW,
                                  int flags, void* workspace, size_t workspace_bytes, void* stream);

/*
 * sbl_linear_workspace_bytes — bytes of device workspace sbl_linear needs for
 * these sizes: the quantised activations and their scales, in the kernels'
 * internal layout (T*K + 4*T bytes, each rounded up to 256), plus, for 2:4
 * weights (K % 64 == 0) at sizes that take a prefill path, the weights'
 * compressed form for the sparse tensor cores (O*K/2 + O*32*ceil(K/256)
 * bytes, each rounded up to 256) or, when the one-CTA tensor-core kernel is
 * split along k (few output tiles facing a long K, small T), its int32
 * accumulator tiles (64 KiB per 128 x 128 output tile), whichever is larger.
 * Depends on the current device's SM count.  Never 0 for T > 0.  A smaller
 * workspace that still holds the first part is accepted; sbl_linear then
 * stays on the dense, unsplit paths.
 */
size_t sbl_linear_workspace_bytes(int64_t T, int64_t K, int64_t O, int n, int m);

/*
 * sbl_linear — y = dequant(int8(x) . W_t^T) on prepared weights.
 *
 * Follows the linear-evaluation equation of the Sparse-BitNet Guide,
 * "Mathematical Formulation of Sparse-BitLinear": the integer product of the
 * int8 activations and the ternary weights, rescaled by beta * gamma / 127,
 * here scale_o / s_t with int32 accumulation.
 *
 *   x_bf16     bf16 bit patterns [T, K] (input).
 *   packed     uint8 [O, K/4] and row_scale fp32 [O] from sbl_prepare_weights.
 *   n, m       the N:M pattern the weights were prepared with.
 *   y          [T, O] (output), fp32 (y_dtype SBL_F32) or bf16 (SBL_BF16,
 *              round to nearest even of the fp32 value).
 *   acc_out    int32 [T, O] (output, may be NULL): the integer accumulators.
 *   workspace  device scratch of at least sbl_linear_workspace_bytes(), 256-byte
 *              aligned; its contents on entry do not matter and are
 *              overwritten.  Calls that share a workspace must be ordered on
 *              one stream.
 *   Chooses the decode path for T <= sbl_decode_max_tokens() (CUDA-core dp4a
 *   for one or two tokens, the warp-level int8 MMA for more when K % 64 == 0)
 *   and the tcgen05 tensor-core prefill path above it (the latter needs
 *   K % 64 == 0; other K always take the decode path).
 */
sbl_status sbl_linear(const uint16_t* x_bf16, int64_t T, int64_t K,
                      const uint8_t* packed, const float* row_scale, int64_t O, int n, int m,
                      void* y, int y_dtype, int32_t* acc_out,
                      void* workspace, size_t workspace_bytes, void* stream);

/*
 * sbl_copy_to_device, sbl_copy_to_host — the host<->device transfers of a
 * pass that starts and ends in host memory (x and the latent weights in, y
 * out), enqueued on `stream` as one asynchronous copy each; they return
 * before the copy has finished.
 *
 *   device_dst / device_src  device memory of the caller.
 *   host_src / host_dst      host memory of the caller; page-locked memory
 *                            (cudaHostAlloc, torch pin_memory) lets the copy
 *                            overlap kernels and the other direction, pageable
 *                            memory is staged by the runtime.
 *   bytes                    0 is a no-op (the pointers are not read).
 * Errors: SBL_ERR_INVALID_ARG for a NULL pointer with bytes > 0 (checked on
 * the host before anything is enqueued); SBL_ERR_CUDA if the runtime rejects
 * the copy.
 */
sbl_status sbl_copy_to_device(void* device_dst, const void* host_src, size_t bytes, void* stream);
sbl_status sbl_copy_to_host(void* host_dst, const void* device_src, size_t bytes, void* stream);

/*
 * sbl_linear_hostio — sbl_linear on activations and outputs in host memory
 * (the Sparse-BitNet Guide, "Mathematical Formulation of Sparse-BitLinear",
 * as sbl_linear): copies x_host into x_dev, runs sbl_linear(x_dev, ..., y_dev,
 * ...) and copies y_dev into y_host, all three enqueued on `stream` in that
 * order; the call returns before they finish, so synchronise the stream
 * before reading y_host.
 *
 *   x_host   bf16 bit patterns [T, K] in host memory (page-locked for overlap).
 *   x_dev    device staging for x, T*K*2 bytes, 16-byte aligned.
 *   y_dev    device staging for y, T*O*4 (SBL_F32) or T*O*2 (SBL_BF16) bytes,
 *            16-byte aligned.
 *   y_host   host memory for y, the same size.
 *   Other arguments as sbl_linear (no acc_out).
 * Errors: the argument checks of sbl_linear, and SBL_ERR_INVALID_ARG for a
 * NULL host or staging pointer, all made on the host before anything is
 * enqueued; SBL_ERR_CUDA if a copy or kernel launch fails.
 */
sbl_status sbl_linear_hostio(const uint16_t* x_host, int64_t T, int64_t K, uint16_t* x_dev,
                             const uint8_t* packed, const float* row_scale, int64_t O, int n, int m,
                             void* y_dev, void* y_host, int y_dtype,
                             void* workspace, size_t workspace_bytes, void* stream);

/*
 * sbl_linear_path — sbl_linear with the contraction path forced
 * (SBL_PATH_DECODE, or one of the SBL_PATH_PREFILL* tensor-core paths;
 * SBL_PATH_AUTO is sbl_linear).  Every path gives the same results.
 * A prefill path with K % 64 != 0 returns SBL_ERR_UNSUPPORTED.
 * SBL_PATH_PREFILL_SPARSE (the Sparse-BitNet Guide, "The Hardware Mechanics
 * of 2:4 Sparsity": two kept values and their 2-bit positions per group of
 * four feed the structured-sparse MMA) needs (n, m) = (2, 4), else
 * SBL_ERR_UNSUPPORTED, and a workspace that also holds the compressed weights,
 * else SBL_ERR_WORKSPACE.  Packed codes with more than two nonzeros in a group
 * of four are not 2:4 weights: the call then sets SBL_ERR_INVALID_ARG in the
 * device status word and its results are unspecified.
 */
sbl_status sbl_linear_path(const uint16_t* x_bf16, int64_t T, int64_t K,
                           const uint8_t* packed, const float* row_scale, int64_t O, int n, int m,
                           void* y, int y_dtype, int32_t* acc_out,
                           void* workspace, size_t workspace_bytes, int path, void* stream);

/*
 * sbl_linear_rmsnorm — the whole forward of the Sparse-BitNet Guide's
 * SparseBitLinear module on prepared weights: RMSNorm of x (as in
 * sbl_rmsnorm_quant_act, weight g, epsilon eps), per-token absmax int8, the
 * integer product with the ternary weights and the rescale, y as sbl_linear
 * returns it.  Arguments and `path` as sbl_linear_path, plus g (fp32 [K],
 * 16-byte aligned, not NULL) and eps (finite, >= 0).  Needs K % 64 == 0 at
 * the sizes that take the decode path (there the activations are normalised
 * and quantised by one kernel and contracted on the warp-level MMA), else
 * SBL_ERR_UNSUPPORTED.  The workspace is sized by sbl_linear_workspace_bytes().
 */
sbl_status sbl_linear_rmsnorm(const uint16_t* x_bf16, const float* g, float eps, int64_t T, int64_t K,
                              const uint8_t* packed, const float* row_scale, int64_t O, int n, int m,
                              void* y, int y_dtype, int32_t* acc_out,
                              void* workspace, size_t workspace_bytes, int path, void* stream);

/*
 * sbl_linear_q — sbl_linear on activations that are already quantised.
 *
 * Sparse-BitNet Guide, "Mathematical Formulation of Sparse-BitLinear": the
 * integer product of the int8 activations with the ternary weights, rescaled
 * by row_scale[o] / s_tok[t].  Here the activation step (the x̃ equation) is
 * the caller's: x_q (int8 [T, K], column order, 16-byte aligned) and s_tok
 * (fp32 [T], 16-byte aligned) exactly as sbl_quant_act writes them.  A
 * training forward keeps them for the backward; a layer split along K
 * across GPUs quantises the whole row once and contracts its slice.
 * packed, row_scale, O, n, m, y, y_dtype and acc_out are as for sbl_linear;
 * y and acc_out equal sbl_linear's on the x that x_q came from.
 *   - Needs K % 64 == 0, else SBL_ERR_UNSUPPORTED.  T <= 16 (with K <= 24576)
 *     runs on the warp-MMA decode kernel, larger sizes on the tensor cores.
 *   - The workspace is sized by sbl_linear_workspace_bytes().  The dense
 *     tensor-core GEMMs and the decode kernel read x_q in the weight codes'
 *     pairing order, written into the workspace by one permutation kernel
 *     (T * K bytes read and written); the 2:4 sparse GEMM reads x_q in place.
 *   - x_q and s_tok are read only; the library keeps no reference to them.
 * Errors as sbl_linear; asynchronous on `stream`.
 */
sbl_status sbl_linear_q(const int8_t* x_q, const float* s_tok, int64_t T, int64_t K,
                        const uint8_t* packed, const float* row_scale, int64_t O, int n, int m,
                        void* y, int y_dtype, int32_t* acc_out,
                        void* workspace, size_t workspace_bytes, void* stream);

/*
 * sbl_linear_noalloc — sbl_linear for callers that cannot allocate device memory.
 *
 * The pages have no counterpart for this entry point; it serves callers that
 * cannot provide a workspace: a plugin whose host application owns the whole
 * device-memory budget, a plain C caller with no allocator of its own, or a
 * latency-critical path where an allocation could synchronise the device.
 *
 * Same arguments and results as sbl_linear, minus the workspace.  The scratch
 * (quantised activations and per-token scales) lives in one array of
 * SBL_NOALLOC_SCRATCH_BYTES of static device memory inside the library, which
 * every GPU that loads the library holds until the process exits.  The call
 * allocates nothing.
 *   - Calls whose quantised activations and scales (T * K + 4 * T bytes, each
 *     rounded up to 256: T = 1024 fits at K = 7168 but not at K = 8192) do
 *     not fit in the array return SBL_ERR_WORKSPACE and enqueue nothing.  2:4
 *     calls use the sparse tensor cores only when the compressed weights fit
 *     in the rest of the array.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress); make that first call before any stream capture.
 *   - All calls on a device share the one array: calls that may overlap on the
 *     GPU (different streams without ordering between them) race on it and
 *     give wrong results.  Order them on one stream.
 */
#define SBL_NOALLOC_SCRATCH_BYTES (8u << 20)

sbl_status sbl_linear_noalloc(const uint16_t* x_bf16, int64_t T, int64_t K,
                              const uint8_t* packed, const float* row_scale, int64_t O, int n, int m,
                              void* y, int y_dtype, int32_t* acc_out, void* stream);

/*
 * sbl_linear_grouped — G layers that read the same activations (the q, k and v
 * projections of an attention block; the gate and up projections of an FFN)
 * in one call.
 *
 * Each result is exactly sbl_linear's for that layer (the Sparse-BitNet
 * Guide, "Mathematical Formulation of Sparse-BitLinear", applied per weight
 * matrix; the activations' int8 codes and scales depend on x alone, so one
 * quantisation serves every layer).
 *   packed, row_scale, O, y   HOST arrays of G entries: layer g's prepared
 *                             weights (device pointers), its row count
 *                             (O[g] >= 0; 0 skips it) and its [T, O[g]]
 *                             output (device pointer); acc_out: NULL, or a
 *                             host array of G device pointers (entries may
 *                             be NULL).
 *   x_bf16, T, K, n, m, y_dtype  as sbl_linear; one pattern for all layers.
 *   workspace   for prefill sizes, sbl_linear_grouped_workspace_bytes(T, K)
 *               bytes, 256-byte aligned (else SBL_ERR_WORKSPACE); decode
 *               sizes use none (NULL allowed).
 * One or two tokens: one launch streams all G weight matrices (one pass of
 * their stacked rows).  Three to 16 tokens: the warp-level MMA decode per
 * layer.  Prefill: x is quantised once, then one launch of the tensor-core
 * GEMM schedules the output tiles of up to four layers together (CTA pairs or
 * one CTA, as for one layer of their combined size; the 2:4 sparse kernel and
 * the split along k are not used).
 * 1 <= G <= SBL_MAX_GROUP, else SBL_ERR_INVALID_ARG.
 */
size_t sbl_linear_grouped_workspace_bytes(int64_t T, int64_t K);
sbl_status sbl_linear_grouped(const uint16_t* x_bf16, int64_t T, int64_t K, int G, const uint8_t* const* packed,
                              const float* const* row_scale, const int64_t* O, int n, int m, void* const* y,
                              int y_dtype, int32_t* const* acc_out, void* workspace, size_t workspace_bytes,
                              void* stream);

/*
 * sbl_linear_plan — the contraction path sbl_linear takes for these sizes on
 * the current device with a workspace of `workspace_bytes`: SBL_PATH_DECODE,
 * SBL_PATH_PREFILL_1CTA, SBL_PATH_PREFILL_PAIR or SBL_PATH_PREFILL_SPARSE.
 * Enqueues nothing.  Invalid sizes or patterns return the negated status
 * (e.g. -SBL_ERR_UNSUPPORTED); a workspace too small for any path returns
 * -SBL_ERR_WORKSPACE.
 */
int sbl_linear_plan(int64_t T, int64_t K, int64_t O, int n, int m, size_t workspace_bytes);

/* Largest T that sbl_linear sends to the decode path. */
int64_t sbl_decode_max_tokens(void);

/*
 * sbl_device_status — synchronises `stream`, then returns and clears the
 * current device's status word: SBL_OK, or the first of SBL_ERR_TIMEOUT /
 * SBL_ERR_NONFINITE / SBL_ERR_INVALID_ARG (weights given as 2:4 that are not)
 * that any kernel raised since the last call.
 */
sbl_status sbl_device_status(void* stream);

/*
 * sbl_selftest_bounded_wait — launches one block that waits on a barrier that
 * nothing ever completes, with the same bounded wait the pipelines use but a
 * short limit of `max_polls` polls.  The kernel records SBL_ERR_TIMEOUT in the
 * status word and returns; the call then reports sbl_device_status().
 * Exists so that the timeout path is tested without hanging a GPU.
 */
sbl_status sbl_selftest_bounded_wait(uint32_t max_polls, void* stream);

/* Human-readable name of a status code (static storage). */
const char* sbl_status_string(sbl_status s);

/* Library version string (static storage). */
const char* sbl_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SBL_H */
