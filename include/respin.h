/*
 * respin.h -- C ABI of the ReSpinQuant block-boundary library (B200, sm_100a).
 *
 * The library implements the inference-time hot path of "ReSpinQuant:
 * Efficient Layer-Wise LLM Quantization via Subspace Residual Rotation
 * Approximation" (arXiv 2604.11080, as explained on the gist.science pages in
 * zh, it, nl, es and fr; cited below by language and section):
 *
 *   1. the per-token basis fix at a block boundary,
 *        h' = residual * (I + U_r V_r^T) + x,
 *      the rank-r form of the residual-path transition T = R_out^T R_in
 *      (zh §2.1-§2.2; nl §2B-§2C; fr §2B-§2C), fused with
 *   2. per-token symmetric INT4 quantization of h' (W4A4, zh §3-§4), and
 *   3. the W4A4 GEMM that consumes those codes (zh §2.2: the linears stay
 *      ordinary linears once the rotations are fused into their weights).
 *
 * Conventions for every call:
 *   - Tokens are rows; tensors are row-major and contiguous.
 *   - bf16 means IEEE bfloat16 (raw 16-bit storage), fp32 means IEEE binary32.
 *   - INT4 codes are packed two per byte: element 2j in the low nibble of byte
 *     j, element 2j+1 in the high nibble, two's complement (value & 0xF).
 *   - All tensor pointers are DEVICE pointers owned by the caller, on the
 *     device that is current when the call is made, 16-byte aligned unless
 *     stated otherwise. The library never allocates per call.
 *   - `stream` is a cudaStream_t handle (NULL = legacy default stream). Calls
 *     are asynchronous: they validate, enqueue their kernels and return.
 *   - Every call returns a respin_status_t. Validation errors are returned
 *     before anything is enqueued; respin_last_error() then holds a message.
 *     Kernels never trap: a kernel that gives up on a bounded wait records a
 *     code in a device status word that respin_device_status() reads.
 *   - No call is thread-safe with respect to the same plan being destroyed.
 */
#ifndef RESPIN_H_
#define RESPIN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  RESPIN_OK = 0,
  RESPIN_ERR_INVALID_ARG = 1,   /* null/negative/unknown argument          */
  RESPIN_ERR_ALIGNMENT = 2,     /* a pointer is not suitably aligned        */
  RESPIN_ERR_UNSUPPORTED = 3,   /* a size outside what the kernels support  */
  RESPIN_ERR_CUDA = 4,          /* a CUDA runtime call failed               */
  RESPIN_ERR_OOM = 5,           /* device allocation failed (plan creation) */
  RESPIN_ERR_DEVICE_CHECK = 6   /* a kernel recorded a device-side failure  */
} respin_status_t;

typedef struct respin_plan_s* respin_plan_t;

/* Plan flag: respin_boundary_forward writes h' as fp32 (the value before the
 * bfloat16 rounding) instead of bf16. The codes are still computed from the
 * bfloat16-rounded h'. Used to check the arithmetic of the fix directly. */
#define RESPIN_H_FP32_DEBUG 1u

/* Plan flag: 3-bit activation codes (W3A3, named beside W4A4 on the
 * explainer pages: zh §3-§4, it §3-§4, nl §3-§4, es §3-§4, fr §4; no
 * quantizer is given there). The quantizer bound becomes 3 instead of 7:
 * inv = 3 / amax, scale = amax / 3, codes in [-3, 3], stored in the same
 * two's-complement nibbles, so w4a4_gemm consumes them (and 3-bit weight
 * codes) unchanged. */
#define RESPIN_ACT_INT3 2u

/*
 * respin_plan_create -- prepare the rank-r fix of one block boundary.
 *
 * Passage: the top-r SVD of Delta T = T - I gives the subspace in which the
 * residual is rotated (it §2C; nl §2C; es §2B; fr §2C); with row vectors the
 * fix is h (I + U_r V_r^T), which is the zh §2.2 form x + Q (M Q^T x) with
 * U_r = Q and V_r = Q M.
 *
 *   out    : receives the plan handle.
 *   D      : hidden size; D % 128 == 0, 128 <= D <= 65536.
 *   r      : rank; 0 <= r <= 128 and r % 8 == 0. r == 0 gives plain
 *            residual + x followed by quantization.
 *   U_r    : HOST fp32 [D, r] row-major (may be NULL iff r == 0).
 *   V_r    : HOST fp32 [D, r] row-major (may be NULL iff r == 0).
 *   flags  : 0, or RESPIN_H_FP32_DEBUG and/or RESPIN_ACT_INT3.
 *
 * The plan rounds U_r and V_r to bfloat16 (round to nearest even), copies
 * them to the current device (owned by the plan) and picks the launch
 * configuration. Synchronous. Errors: INVALID_ARG, UNSUPPORTED (e.g. D*r too
 * large for the on-chip factor slices), OOM, CUDA.
 */
respin_status_t respin_plan_create(respin_plan_t* out, int D, int r,
                                   const float* U_r, const float* V_r,
                                   unsigned flags);

/*
 * respin_plan_create_subspace -- prepare a boundary from the stored
 * subspace form.
 *
 * Passage: zh §2.2 steps 1-3 keep, per boundary, one D x r basis Q and one
 * r x r rotation R_sub and apply the fix as projection y = Q^T x, transform
 * z = (R_sub - I) y inside the subspace, re-projection x + Q z; the online
 * parameter count of zh §4 (64 D r) is this form. In the row convention of
 * respin_boundary_forward the same fix is
 *     y = residual Q,  z = y M^T,  h = residual + x + z Q^T,  M = R_sub - I,
 * i.e. the factor form with U_r = Q and V_r = Q M, stored in half the bytes.
 *
 *   out    : receives the plan handle.
 *   D      : hidden size; 2048 or 4096 (CTA pairs split the columns;
 *            short calls at D = 4096 use clusters of four).
 *   r      : rank, 1 <= r <= 32.
 *   Q      : HOST fp32 [D, r] row-major.
 *   R_sub  : HOST fp32 [r, r] row-major.
 *   flags  : 0, or RESPIN_H_FP32_DEBUG and/or RESPIN_ACT_INT3.
 *
 * The plan rounds Q to bfloat16 (round to nearest even) and forms
 * M = R_sub - I exactly, rounded once to fp32; respin_boundary_forward then
 * computes y and z in fp32 (z_i = sum_j y_j M_ij in j order) and h in fp32
 * as for factor plans. Synchronous. Errors: INVALID_ARG, UNSUPPORTED, OOM,
 * CUDA.
 */
respin_status_t respin_plan_create_subspace(respin_plan_t* out, int D, int r,
                                            const float* Q, const float* R_sub,
                                            unsigned flags);

/* respin_plan_destroy -- free the plan's device factors. Waits for the device
 * to finish outstanding work first. Unknown or already destroyed handles give
 * INVALID_ARG. NULL is a no-op. */
respin_status_t respin_plan_destroy(respin_plan_t plan);

/*
 * respin_boundary_forward -- fused block-boundary step for N tokens.
 *
 * Passage: the residual connection in the rotated basis needs the transition
 * T before the addition (fr §2B; zh §2.2 "x_out = T x_in + ..."), applied in
 * the rank-r subspace as projection, transform, re-projection and residual
 * (zh §2.2 steps 1-3). Per token (row) n, in fp32 with the plan's bf16
 * factors:
 *     y      = residual[n] U_r                       (r values)
 *     h[n]   = residual[n] + x[n] + y V_r^T
 *     h'[n]  = bf16(h[n])                            (round to nearest even)
 *     amax   = max_i |h'[n, i]|
 *     inv    = B / amax, scale[n] = amax / B         (binary32, RN)
 *     q[n,i] = clamp(rint(h'[n,i] * inv), -B-1, B)   (ties to even)
 * with B = 7 (INT4), or B = 3 for a plan made with RESPIN_ACT_INT3.
 * A token with amax < 2^-125 gets scale 0 and all-zero codes.
 *
 *   plan      : from respin_plan_create or respin_plan_create_subspace;
 *               its device must be current.
 *   x         : bf16 [N, D] block output (device).
 *   residual  : bf16 [N, D] residual stream (device), or NULL for zero (then
 *               h' = x and the factors are not used).
 *   N         : tokens; N == 0 is a no-op; N < 0 is INVALID_ARG.
 *   h_out     : bf16 [N, D] (fp32 [N, D] with RESPIN_H_FP32_DEBUG), or NULL
 *               to skip writing h'.
 *   q_packed  : uint8 [N, D/2] packed codes (device).
 *   scale     : fp32 [N] per-token scales (device, 4-byte aligned).
 *   stream    : cudaStream_t.
 * No input may overlap an output. Errors: INVALID_ARG, ALIGNMENT, CUDA.
 *
 * Large calls of plans with padded rank 64 / 128 (from 256 tokens) and of
 * rank-16 / 32 plans at D = 8192 (from 4096 tokens) with an h_out buffer run
 * as three kernels on the stream (projection, re-projection, codes); until
 * the last one, q_packed holds partial projections and scale the per-token
 * amax, so, like every output, they are final only once the call's work on
 * the stream is complete. Nothing is allocated.
 */
respin_status_t respin_boundary_forward(respin_plan_t plan, const void* x,
                                        const void* residual, int N,
                                        void* h_out, uint8_t* q_packed,
                                        float* scale, void* stream);

/*
 * w4a4_gemm -- out = bf16((float(acc) * scale_act[n]) * scale_w[o]) with
 * acc[n, o] = sum_k a[n, k] w[o, k] exactly in int32 (W4A4 linear, zh §3-§4,
 * fr §4; the weights already carry the fused rotations, zh §2.2).
 *
 *   q_act     : uint8 [N, K/2] packed activation codes (device).
 *   scale_act : fp32 [N] per-token scales (device, 4-byte aligned).
 *   q_w       : uint8 [O, K/2] packed weight codes, one row per output
 *               channel (device).
 *   scale_w   : fp32 [O] per-channel scales (device, 16-byte aligned).
 *   N         : tokens (N == 0 is a no-op).
 *   K         : reduction size; K % 128 == 0, 128 <= K <= 65536.
 *   O         : output channels; O % 16 == 0, O >= 16.
 *   out       : bf16 [N, O] (device).
 * Both products of the epilogue round to nearest even in binary32; the
 * integer sum is exact, so the result does not depend on which kernel runs
 * (N <= 128: weight-streaming kernel; above: tensor-memory tiles).
 * Errors: INVALID_ARG, UNSUPPORTED, ALIGNMENT, CUDA.
 */
respin_status_t w4a4_gemm(const uint8_t* q_act, const float* scale_act,
                          const uint8_t* q_w, const float* scale_w, int N,
                          int K, int O, void* out, void* stream);

/* w4a4_gemm_i32 -- same contraction, writes the exact int32 accumulators
 * acc_out [N, O] (device) instead of the scaled bf16 output. For tests. */
respin_status_t w4a4_gemm_i32(const uint8_t* q_act, const uint8_t* q_w,
                              int N, int K, int O, int32_t* acc_out,
                              void* stream);

/*
 * w4a4_gemm_rowmax -- w4a4_gemm, and in the same pass the maxima of |out|
 * (out as stored, bf16) per token and 256-channel tile:
 *     rowmax[n, t] = max_{o in [256 t, 256 t + 256) and o < O} |out[n, o]|
 * for a following per-token quantization of out (the input of the next
 * linear, e.g. the up projection's output feeding the down projection in
 * the quantized linears of zh §3-§4), so that pass needs no reduction of its
 * own.
 *
 *   rowmax : fp32 [N, ceil(O / 256)] (device, 4-byte aligned, caller-owned;
 *            every entry is written).
 *   Other arguments as w4a4_gemm. Needs N > 128 (the tensor-memory kernel);
 *   smaller N gives UNSUPPORTED. Errors: as w4a4_gemm.
 */
respin_status_t w4a4_gemm_rowmax(const uint8_t* q_act, const float* scale_act,
                                 const uint8_t* q_w, const float* scale_w,
                                 int N, int K, int O, void* out,
                                 float* rowmax, void* stream);

/*
 * respin_quantize_rowmax -- per-token codes and scales of a bf16 matrix u
 * [N, D] whose per-token maxima of |u| are given as partial maxima (rowmax
 * [N, D / 256], as written by w4a4_gemm_rowmax): amax = max over the row's
 * partials, then the quantizer of respin_boundary_forward (inv = B / amax,
 * scale = amax / B, q = rint(u inv), B = 7, or 3 with RESPIN_ACT_INT3;
 * amax < 2^-125 gives scale 0 and zero codes). The codes equal those of
 * respin_boundary_forward with an r = 0 plan and no residual on the same u.
 *
 *   u        : bf16 [N, D] (device, 16-byte aligned).
 *   rowmax   : fp32 [N, D / 256] (device).
 *   N, D     : D % 256 == 0, 256 <= D <= 65536.
 *   q_packed : uint8 [N, D/2]; scale : fp32 [N] (device).
 *   flags    : 0 or RESPIN_ACT_INT3.
 * Launched as a programmatic dependent of the previous kernel of the stream
 * (it waits for that kernel before reading u). Errors: INVALID_ARG,
 * UNSUPPORTED, ALIGNMENT, CUDA.
 */
respin_status_t respin_quantize_rowmax(const void* u, const float* rowmax,
                                       int N, int D, uint8_t* q_packed,
                                       float* scale, unsigned flags,
                                       void* stream);

/*
 * respin_factors_from_subspace -- plan factors from the subspace form.
 *
 * Passage: zh §2.2 steps 1-3 store one D x r basis Q and an r x r rotation
 * R_sub per boundary and apply x + Q ((R_sub - I) (Q^T x)) to a column
 * vector. For a row vector h the same map is h + (h U_r) V_r^T with
 *     U_r = Q,   V_r = Q (R_sub - I)
 * (computed in float64, rounded to float).
 *
 *   D, r   : 0 < r <= D.
 *   Q      : HOST fp32 [D, r] row-major.
 *   R_sub  : HOST fp32 [r, r] row-major.
 *   U_r    : HOST fp32 [D, r] output (caller-owned).
 *   V_r    : HOST fp32 [D, r] output (caller-owned).
 * Host only (no device, no allocation). Errors: INVALID_ARG.
 */
respin_status_t respin_factors_from_subspace(int D, int r, const float* Q,
                                            const float* R_sub, float* U_r,
                                            float* V_r);

/*
 * respin_factors_from_transition -- plan factors from a dense transition.
 *
 * Passage: the top-r SVD of Delta T = T - I gives the subspace (it §2C,
 * nl §2C, es §2B, fr §2C). Row convention h' = h T: with
 * Delta T = sum_i s_i u_i v_i^T (s_1 >= s_2 >= ...),
 *     U_r = [u_1 .. u_r],   V_r = [s_1 v_1 .. s_r v_r],
 * so h (I + U_r V_r^T) is the best rank-r fix in the Frobenius norm. Float64
 * block subspace iteration (block max(2r, r + 8), deterministic start) with
 * Rayleigh-Ritz steps until the top-r subspace stops moving.
 *
 *   D, r    : 0 < r < D, r <= 128.
 *   T       : HOST fp32 [D, D] row-major.
 *   gap_tol : the truncation is refused (UNSUPPORTED) unless
 *             s_r - s_(r+1) > gap_tol * s_1; without a gap the top-r subspace
 *             is not unique (e.g. r splitting a pair of equal singular values).
 *   U_r,V_r : HOST fp32 [D, r] outputs (caller-owned).
 *   sigma   : HOST fp64 [r + 1] output s_1 .. s_(r+1), or NULL. Also written
 *             when the gap check refuses.
 * Host only; O(D^2 r) work per iteration, 8 D^2 bytes of host memory for
 * the float64 copy of T. Errors: INVALID_ARG, UNSUPPORTED, OOM.
 */
respin_status_t respin_factors_from_transition(int D, int r, const float* T,
                                               double gap_tol, float* U_r,
                                               float* V_r, double* sigma);

/*
 * respin_fuse_weight -- fold the block rotations into a linear's weight.
 *
 * Passage: the rotations are merged into the weights offline so that the
 * linears stay ordinary linears (zh §2.2, e.g. W~ = R^T W R; fr §2A,
 * W~ = W R). For y = W x with the input arriving as x~ = R_in^T x and the
 * output wanted as y~ = R_out^T y:
 *     W_fused = R_out^T W R_in        (W_fused x~ = R_out^T W x),
 * or W R_in when R_out is NULL.
 *
 *   O, K    : output and input size (O, K > 0).
 *   W       : HOST fp32 [O, K] row-major (one row per output channel).
 *   R_in    : HOST fp32 [K, K] row-major.
 *   R_out   : HOST fp32 [O, O] row-major, or NULL.
 *   W_fused : HOST fp32 [O, K] output (caller-owned).
 * Host only: float64 products over the host's threads, each element one sum
 * in a fixed order. Errors: INVALID_ARG, OOM.
 */
respin_status_t respin_fuse_weight(int O, int K, const float* W,
                                   const float* R_in, const float* R_out,
                                   float* W_fused);

/*
 * respin_quantize_weight -- per-output-channel symmetric INT4 (or INT3)
 * weight codes for w4a4_gemm (the explainers evaluate W4A4 and W3A3, zh
 * §3-§4; they give no weight quantizer). Per row o, in binary32 as for the
 * activations: amax = max_k |W[o,k]|, inv = qmax / amax,
 * q = clamp(rint(W[o,k] inv), -qmax-1, qmax) (ties to even),
 * scale_w[o] = amax / qmax; a row with amax < 2^-125 gets scale 0 and zero
 * codes.
 *
 *   O, K    : rows and columns (K even).
 *   W       : HOST fp32 [O, K] row-major.
 *   qmax    : 7 (INT4) or 3 (INT3).
 *   q_w     : HOST uint8 [O, K/2] packed codes (element 2j in the low nibble).
 *   scale_w : HOST fp32 [O].
 * Host only. Errors: INVALID_ARG.
 */
respin_status_t respin_quantize_weight(int O, int K, const float* W, int qmax,
                                       uint8_t* q_w, float* scale_w);

/* respin_device_status -- synchronizes the current device, then returns and
 * clears the device status word through *code (0 = no kernel gave up; else
 * the site of the first wait that gave up since the last clear). Returns
 * DEVICE_CHECK if *code != 0. The outputs of a launch in which a wait gave up
 * are invalid (the kernel skips its stores after the failure); the status
 * word itself never changes what a later launch computes. */
respin_status_t respin_device_status(int* code);

/* respin_selftest_wait_limit -- failure-detection self test (for tests).
 * Enqueues a one-thread kernel whose bounded mbarrier wait has nothing to
 * wait for: after limit_us microseconds (1 .. 2,000,000) it gives up,
 * records site 901 in the device status word (unless an earlier failure is
 * recorded there) and returns. Nothing is copied or stored. The next
 * respin_device_status() then reports DEVICE_CHECK with code 901 and clears
 * the word. Errors: INVALID_ARG, CUDA. */
respin_status_t respin_selftest_wait_limit(unsigned limit_us, void* stream);

/* respin_last_error -- message of the last failed call on this thread (empty
 * string if none). The pointer stays valid until the next call on this
 * thread. */
const char* respin_last_error(void);

/* respin_version -- library version string. */
const char* respin_version(void);

#ifdef __cplusplus
}
#endif

#endif /* RESPIN_H_ */
