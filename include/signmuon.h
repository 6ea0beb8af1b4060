/*
 * signmuon.h -- C ABI of libsignmuon.so, a B200 (sm_100a) implementation of
 * one Sign-Muon optimizer step for M workers simulated on one GPU.
 *
 * Sources, by page title:
 *   [paper] "SignMuon: 通信高效的分布式Muon优化" (a rendering of arXiv 2605.16311)
 *   [blog]  "SignMuon: Matrix Directions, Majority Votes, and the Actual Bytes Sent"
 *
 * Conventions shared by every entry point
 *   - Every call returns an int status (SIGNMUON_OK or an error below) and
 *     never aborts the process.  signmuon_last_error() gives the text of the
 *     handle's last error.
 *   - "device" pointers are CUDA device allocations of the calling process on
 *     the handle's device (for example torch tensors); "host" pointers are
 *     ordinary (ideally pinned) host memory.  Pointers passed as float/uint8
 *     arrays must be 16-byte aligned.
 *   - The parameter vector is flat: the matrices of `shapes` concatenated in
 *     order, each row-major, d = sum(rows*cols) elements.  Convolution weights
 *     are flattened to out x (in*kh*kw) by the caller.
 *   - Work is enqueued on the CUDA stream given at init.  Calls return without
 *     waiting for the GPU, except where a call says otherwise.
 *   - A handle belongs to the device that was current at signmuon_init.  A
 *     call on it makes that device current while it runs and gives the
 *     caller's current device back before it returns.
 *   - The caller owns W, G, signs, sums, majority and every buffer it passes;
 *     the library owns the momentum, the Newton-Schulz workspace and the
 *     packed sign buffers of the step.
 */
#ifndef SIGNMUON_H
#define SIGNMUON_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct signmuon_ctx* signmuon_t;

/* status codes */
#define SIGNMUON_OK            0
#define SIGNMUON_E_INVALID     1  /* bad argument: shape, M, K, beta, lambda, eps, P, null or misaligned pointer */
#define SIGNMUON_E_OVERFLOW    2  /* int8 vote accumulator requested with M > 127 */
#define SIGNMUON_E_NONFINITE   3  /* a momentum norm was NaN/Inf: W was not updated */
#define SIGNMUON_E_CUDA        4  /* a CUDA runtime/driver call failed */
#define SIGNMUON_E_NOMEM       5  /* device allocation failed */
#define SIGNMUON_E_TIMEOUT     6  /* a kernel's bounded wait expired; results are invalid */
#define SIGNMUON_E_UNSUPPORTED 7  /* call not available for this handle (e.g. step on a vote-only handle) */

/* scale step of PolarNS ([paper] Algorithm 1 input "scale") */
#define SIGNMUON_SCALE_FRO      0  /* X0 = Mom / (||Mom||_F + eps) */
#define SIGNMUON_SCALE_SPECTRAL 1  /* X0 = Mom / (sigma + eps), sigma by P power iterations */

/* flags for signmuon_init */
#define SIGNMUON_NS_FP32     (1u << 0) /* fp32 Newton-Schulz (SIMT) instead of bf16 tcgen05 tensor cores */
#define SIGNMUON_NS_QUINTIC  (1u << 1) /* quintic NS X(15/8 I - 10/8 X^T X + 3/8 (X^T X)^2) */
#define SIGNMUON_POST_POLAR  (1u << 2) /* post-vote local polar step: D = PolarNS(majority) */
#define SIGNMUON_ACC_INT8    (1u << 3) /* int8 vote sums: signmuon_vote / signmuon_vote_ternary write
                                          them and signmuon_sums_step reads them (M <= 127) */
#define SIGNMUON_ASYNC       (1u << 4) /* step, polar, local_signs, vote_step and sums_step do not
                                          wait; signmuon_sync reports their status.  Such a step
                                          makes no host synchronisation and no allocation, so it
                                          can be captured into a CUDA graph on the handle's stream
                                          (its pointers and eta are then fixed by the capture) */
#define SIGNMUON_VOTE_ONLY   (1u << 5) /* allocate no step workspace: vote/pack/update calls only */
#define SIGNMUON_KEEP_POLAR  (1u << 6) /* signmuon_step also writes U for signmuon_get_polar; without it
                                          the last Newton-Schulz GEMM of a bf16 step (K > 0) writes
                                          only the signs (one-bit, or int8 with SIGNMUON_TERNARY) */
/* Named variants ([paper] "SignMuon: 通信高效的分布式Muon优化" Algorithm 2, §4, Table 1):
 * TIE_PLUS           a tied vote (sum 0, even M) gives +1 instead of 0 (Algorithm 2's sign
 *                    default on the {-1, +1} wire); applies to signmuon_vote's majority and
 *                    to the step.
 * POLAR_AFTER_ONLY   the step signs the momentum itself and orthogonalises only after the
 *                    vote (§4 "where to orthogonalise"); requires SIGNMUON_POST_POLAR.
 * MUON_MEAN          the Muon baseline instead of Sign-Muon: D = PolarNS(mean of the M
 *                    workers' momenta), W <- fl32(W - eta D); no signs, no vote; cannot be
 *                    combined with POST_POLAR, POLAR_AFTER_ONLY, TERNARY or NORMALIZED_SIGN.
 * TERNARY            the step sends sign(U) in {-1, 0, +1} as one int8 per entry (d bytes
 *                    per worker: §3's sign with sign(0) = 0, the payload of Algorithm 2's
 *                    int8 SUM all-reduce) instead of one bit, and votes on the integer
 *                    sums of those; U is always kept.  The handle holds M*d more bytes.
 * NORMALIZED_SIGN    D = majority / (s + eps) per matrix, s the handle's scale estimate of
 *                    the majority matrix (spectral: the P-step power-iteration estimate of
 *                    ||majority||_2; fro: ||majority||_F) -- the explicitly normalised sign
 *                    step of §4's analysis.  Cannot be combined with POST_POLAR (it is the
 *                    post-vote step with no Newton-Schulz iteration).
 * PI_WARM            each power iteration (spectral scale) starts from the iterate the same
 *                    problem ended with in the previous call instead of ones/sqrt(m): one
 *                    state per (worker, matrix) for the M-worker PolarNS (signmuon_step and
 *                    signmuon_polar share it) and one per matrix for the post-vote,
 *                    normalised-sign and Muon-baseline PolarNS.  A zero or non-finite state
 *                    (the first call, a zero matrix, a failed step) starts cold.  A
 *                    checkpoint saves the state with signmuon_get/set_pi_state (it is not
 *                    part of get/set_momentum).  No effect with SIGNMUON_SCALE_FRO. */
#define SIGNMUON_TIE_PLUS          (1u << 7)
#define SIGNMUON_POLAR_AFTER_ONLY  (1u << 8)
#define SIGNMUON_MUON_MEAN         (1u << 9)
#define SIGNMUON_TERNARY           (1u << 10)
#define SIGNMUON_NORMALIZED_SIGN   (1u << 11)
#define SIGNMUON_PI_WARM           (1u << 12)
/* NS_GRAM: run the bf16 cubic Newton-Schulz iteration in Gram space when that
 * needs at least 15 % fewer tensor-core flops (every matrix with m >= 256, n
 * well above m, K >= 2): A0 = X0 X0^T, then per iteration the m x m products
 * A_{k+1} = P_k A_k P_k and Q_{k+1} = P_k Q_k with P_k = a I + b A_k (all
 * polynomials in A0, so they commute), and one final X_K = Q_K X0.  In exact
 * arithmetic both give the same X_K.  In bf16 the Gram-space iterates carry the
 * squared spectrum and the iteration does not correct its own rounding: the
 * polar error stays within 1.2x of the iteration on X, but the signs of the
 * smallest entries flip several times more often, so the default iterates on X. */
#define SIGNMUON_NS_GRAM           (1u << 13)

/* ------------------------------------------------------------------------
 * signmuon_init -- plan the step and allocate its device state.
 *
 * Defines the problem of [paper] Algorithm 1 and Algorithm 2 (their input
 * lists: beta, lambda, K, eps, scale, P, and M workers).
 *   out     host out-pointer; receives the handle (NULL on error).
 *   shapes  host array of n_mats (rows, cols) pairs, each >= 1.
 *   M       number of workers, 1..256.
 *   beta    momentum in [0, 1).      lambda  coupled weight decay >= 0.
 *   K       Newton-Schulz iterations >= 0 (0: U = X0, the scaled momentum).
 *   eps     stability constant > 0, added to the scale: X0 = Mom/(s+eps).
 *   scale   SIGNMUON_SCALE_FRO or SIGNMUON_SCALE_SPECTRAL.
 *   P       power iterations (>= 1 when scale is spectral; ignored for fro).
 *   flags   SIGNMUON_* flags above.
 *   stream  cudaStream_t to enqueue on (NULL = the legacy default stream).
 * Momentum starts at zero ([paper] Algorithm 2 initialisation).  Errors:
 * E_INVALID, E_OVERFLOW (ACC_INT8 with M > 127), E_NOMEM, E_CUDA.
 * ---------------------------------------------------------------------- */
int signmuon_init(signmuon_t* out, const int64_t* shapes, int n_mats, int M,
                  float beta, float lambda, int K, float eps, int scale, int P,
                  unsigned flags, void* stream);

/* ------------------------------------------------------------------------
 * signmuon_step -- one distributed Sign-Muon step ([paper] Algorithm 2 with
 * the tie-to-zero vote of [blog] "A tiny aggregation calculation", and the
 * optional post-vote polar step of [paper] §4).
 *   W    device float[d], updated in place: W <- fl32(W - eta*D).
 *   G    host array of M device pointers, each float[d]: worker gradients.
 *   eta  step size.
 * Per worker: Mom_m <- beta*Mom_m + (1-beta)(G_m + lambda*W); U_m =
 * PolarNS(Mom_m) per matrix; bits_m = (U_m >= 0) packed LSB-first (with
 * SIGNMUON_TERNARY: t_m = sign(U_m) in {-1, 0, +1}, one int8 each).  Then
 * sums = sum_m (2 bits_m - 1) (or sum_m t_m), majority = sign(sums) (0 on a
 * tie), D = majority, PolarNS(majority) or majority / (s + eps) per matrix
 * (SIGNMUON_POST_POLAR / SIGNMUON_NORMALIZED_SIGN).  Unless SIGNMUON_ASYNC, waits for
 * the GPU and returns E_NONFINITE when a momentum norm is NaN/Inf; W is then
 * left unchanged (the momentum keeps the non-finite values: restore it with
 * signmuon_set_momentum).
 * ---------------------------------------------------------------------- */
int signmuon_step(signmuon_t h, float* W, const float* const* G, float eta);

/* ------------------------------------------------------------------------
 * signmuon_local_signs / signmuon_vote_step -- signmuon_step in two halves,
 * so that the signs can cross a collective in between: each GPU holds some
 * of the workers, all-gathers their signs, and every GPU votes and updates its
 * own replica of W ([paper] Algorithm 2: local polar and sign, one exchange
 * of the signs, local majority and update; [blog] "the actual bytes sent").
 * signmuon_step(W, G) is signmuon_local_signs into the handle's own buffers
 * followed by signmuon_vote_step over them, kernel for kernel.
 *
 * signmuon_local_signs: momentum, scale, PolarNS and signs of the handle's M
 * workers; W is read (weight decay), not written.
 *   W       device float[d].     G  host array of M device pointers, float[d].
 *   signs   device buffer; worker m's signs at signs + m*stride: ceil(d/8)
 *           packed bytes (LSB-first, as signmuon_pack), or d int8 ternary
 *           signs with SIGNMUON_TERNARY.
 *   stride  bytes between workers: a multiple of 16, at least one worker's
 *           signs.  The call may zero the whole M*stride bytes (packed signs
 *           of matrices whose column counts are not multiples of 32 are OR-ed
 *           into a zeroed buffer).
 * Unless SIGNMUON_ASYNC, waits and returns E_NONFINITE when a momentum norm is
 * NaN/Inf (the signs are then not valid: do not vote on them).  Not for
 * MUON_MEAN handles (E_UNSUPPORTED).
 *
 * signmuon_vote_step: majority of M sign buffers at signs + j*stride (any M in
 * 1..256, e.g. the all-gathered signs of every GPU's workers, in worker
 * order), then the post-vote step the handle's flags ask for and W <-
 * fl32(W - eta*D).  Vote-only handles may call it when they ask for no
 * post-vote step.  Waits like signmuon_step.  After it, signmuon_get_direction
 * gives D only for the post-vote steps (E_UNSUPPORTED when the vote was fused
 * with the update).
 * ---------------------------------------------------------------------- */
int signmuon_local_signs(signmuon_t h, const float* W, const float* const* G, uint8_t* signs,
                         int64_t stride);
int signmuon_vote_step(signmuon_t h, float* W, const uint8_t* signs, int64_t stride, int M,
                       float eta);

/* ------------------------------------------------------------------------
 * signmuon_vote_step_ptrs -- signmuon_vote_step with worker j's signs at
 * signs[j] instead of signs + j*stride: on a node of GPUs each rank maps the
 * other ranks' sign buffers into its address space (signmuon_ipc_open) and
 * the vote kernel reads their packed bits over NVLink directly, with no
 * all-gather copy in between ([paper] Algorithm 2's one exchange of the
 * signs; [blog] "One bit of information is not automatically a one-bit
 * all-reduce").
 *   signs  host array of M device pointers (this GPU's memory or a peer's
 *          mapped by signmuon_ipc_open), each 16-byte aligned, each holding
 *          one worker's ceil(d/8) packed bytes (d int8 signs with
 *          SIGNMUON_TERNARY) padded to a multiple of 16; every buffer must
 *          hold its signs when the call's kernels run (the caller orders the
 *          writers and this call, e.g. by a collective in between).
 *   M      1..256 workers, in worker order.
 * Otherwise as signmuon_vote_step.  Errors: E_INVALID (null or misaligned),
 * E_UNSUPPORTED (MUON_MEAN, or a vote-only handle with a post-vote step).
 * ---------------------------------------------------------------------- */
int signmuon_vote_step_ptrs(signmuon_t h, float* W, const uint8_t* const* signs, int M, float eta);

/* ------------------------------------------------------------------------
 * CUDA IPC for the exchange between GPUs (no counterpart on the pages: the
 * plumbing that lets signmuon_vote_step_ptrs read a peer's sign buffer).
 * signmuon_ipc_get_handle: the IPC handle (SIGNMUON_IPC_HANDLE_BYTES bytes,
 *   written to `handle`) of the device allocation that contains dev_ptr, and
 *   dev_ptr's byte offset in it (to *offset); send both to the peer.
 * signmuon_ipc_open: map a peer's allocation (handle from another process)
 *   into this process on the current device; *base receives its address here
 *   (add the offset).  Peer access is enabled as needed.
 * signmuon_ipc_close: unmap a base pointer returned by signmuon_ipc_open.
 * Errors: E_INVALID (null pointers, not a device allocation), E_CUDA (the
 * runtime refused: see signmuon_last_error(NULL)).
 * ---------------------------------------------------------------------- */
#define SIGNMUON_IPC_HANDLE_BYTES 64
int signmuon_ipc_get_handle(const void* dev_ptr, void* handle, int64_t* offset);
int signmuon_ipc_open(const void* handle, void** base);
int signmuon_ipc_close(void* base);

/* ------------------------------------------------------------------------
 * signmuon_sums_step -- the second half of the step when the vote sums arrive
 * already added up: [paper] Algorithm 2's integer SUM all-reduce of the
 * workers' signs (each GPU sums its own workers with signmuon_vote or
 * signmuon_vote_ternary, an all-reduce adds the GPUs' sums).  majority =
 * sign(sums) with the handle's tie rule, then the post-vote step the flags
 * ask for and W <- fl32(W - eta*D).
 *   W     device float[d].
 *   sums  device int32[d], or int8[d] with SIGNMUON_ACC_INT8 (then at most 127
 *         workers in all, so that no partial or total sum overflows); 16-byte
 *         aligned.
 * Waits like signmuon_step; signmuon_get_direction then gives D.
 * ---------------------------------------------------------------------- */
int signmuon_sums_step(signmuon_t h, float* W, const void* sums, float eta);

/* ------------------------------------------------------------------------
 * signmuon_step_host -- signmuon_step on HOST buffers: copies W and the M
 * gradients to library-owned device buffers (allocated on first use: W and
 * two sets of M gradients), runs the step and copies W back.  Pinned host
 * memory gives full copy bandwidth.
 *   W_host     float[d], read and then overwritten with the updated weights.
 *   G_host     host array of M pointers, each float[d]; only read.
 * The gradients come in on a second stream of the library's, alternating
 * between the two device sets.  Without SIGNMUON_ASYNC the call waits and
 * returns the step's status.  With it the call returns once the copies and
 * the step are queued, and the next call's gradients come in while this
 * step runs and W goes back; W_host and every G_host[m] must then stay
 * valid and unchanged until signmuon_sync (a W_host shared by consecutive
 * calls is fine: each call reads it after the call before has written it).
 * ---------------------------------------------------------------------- */
int signmuon_step_host(signmuon_t h, float* W_host, const float* const* G_host, float eta);

/* ------------------------------------------------------------------------
 * signmuon_vote -- majority vote over M packed one-bit sign buffers
 * ([paper] Algorithm 2: integer SUM of signs, then sign(); [blog]: ties map
 * to 0, sums range over [-M, M]).
 *   signs     host array of M device pointers, each ceil(d/8) bytes; bit j of
 *             byte b is element 8b+j, a set bit means +1.
 *   d         number of entries (>= 0).
 *   sums      device int32[d] (int8[d] when SIGNMUON_ACC_INT8), may be NULL.
 *   majority  device int8[d] in {-1, 0, +1}, may be NULL.
 * Results are bit-exact integers.
 * ---------------------------------------------------------------------- */
int signmuon_vote(signmuon_t h, const uint8_t* const* signs, int64_t d, void* sums,
                  int8_t* majority);

/* ------------------------------------------------------------------------
 * signmuon_pack -- entrywise one-bit sign of a flat float vector ([paper] §3
 * entrywise sign; [blog] d/8-byte payload): bit = (U >= 0), so 0 and -0 send
 * +1 and NaN sends 0.  U device float[d]; out device uint8[ceil(d/8)], pad
 * bits 0.
 * ---------------------------------------------------------------------- */
int signmuon_pack(signmuon_t h, const float* U, int64_t d, uint8_t* out);

/* ------------------------------------------------------------------------
 * signmuon_sign_ternary -- entrywise ternary sign of a flat float vector
 * ([paper] §3: sign(0) = 0): out[i] = +1 if U[i] > 0, -1 if U[i] < 0, else 0
 * (0, -0 and NaN give 0).  U device float[d]; out device int8[d]; both
 * 16-byte aligned.  d >= 0.  Errors: E_INVALID.
 * ---------------------------------------------------------------------- */
int signmuon_sign_ternary(signmuon_t h, const float* U, int64_t d, int8_t* out);

/* ------------------------------------------------------------------------
 * signmuon_vote_ternary -- majority vote over M int8 ternary sign buffers
 * ([paper] Algorithm 2's integer SUM of the workers' signs, d bytes per
 * worker; [blog] "A tiny aggregation calculation": sums in [-M, M], ties to 0,
 * or to +1 with SIGNMUON_TIE_PLUS).
 *   signs     host array of M device pointers, each int8[d] with entries -1,
 *             0 or +1 (other values give unspecified sums, never a fault),
 *             16-byte aligned.
 *   d         number of entries (>= 0).
 *   sums      device int32[d] (int8[d] when SIGNMUON_ACC_INT8), may be NULL.
 *   majority  device int8[d] in {-1, 0, +1}, may be NULL.
 * Results are bit-exact integers.  Errors: E_INVALID (null or misaligned).
 * ---------------------------------------------------------------------- */
int signmuon_vote_ternary(signmuon_t h, const int8_t* const* signs, int64_t d, void* sums,
                          int8_t* majority);

/* ------------------------------------------------------------------------
 * signmuon_apply_update -- W <- fl32(W - eta*D), one rounding (fused
 * multiply-add), [paper] Algorithm 1/2 update.  W, D device float[d].
 * ---------------------------------------------------------------------- */
int signmuon_apply_update(signmuon_t h, float* W, const float* D, int64_t d, float eta);

/* ------------------------------------------------------------------------
 * signmuon_polar -- PolarNS of every matrix of the plan for M independent
 * inputs ([paper] §3 Muon polar factor, §4 Newton-Schulz), with the handle's
 * K, eps, scale, P and precision flags.
 *   X  host array of M device pointers, each float[d] (flat matrices).
 *   U  host array of M device pointers, each float[d] (output).
 * ---------------------------------------------------------------------- */
int signmuon_polar(signmuon_t h, const float* const* X, float* const* U);

/* ------------------------------------------------------------------------
 * State access (device float[d] / uint8[ceil(d/8)] buffers of the caller).
 * get/set_momentum: worker m's momentum (checkpoint / resume).
 * get_polar: worker m's U from the last step (or signmuon_polar call);
 * SIGNMUON_E_UNSUPPORTED when the step did not keep it (handle made without
 * SIGNMUON_KEEP_POLAR on shapes whose signs are packed inside the last
 * Newton-Schulz GEMM, and always with POLAR_AFTER_ONLY or MUON_MEAN).
 * get_signs: worker m's packed bits from the last step (SIGNMUON_E_UNSUPPORTED
 * with MUON_MEAN or TERNARY).  get_ternary_signs: worker m's int8[d] ternary
 * signs from the last step (SIGNMUON_E_UNSUPPORTED unless TERNARY).
 * get_direction: the last step's D (E_UNSUPPORTED before the first step, and
 * after a signmuon_vote_step whose vote was fused with the update).
 * get_scales: host float[M*n_mats]: the last step's scale s per (worker,
 * matrix), worker-major (waits for the GPU).  A post-vote step (POST_POLAR,
 * NORMALIZED_SIGN, MUON_MEAN) writes its own scales, those of the majority
 * (or mean) matrices, into worker 0's row.
 * ---------------------------------------------------------------------- */
int signmuon_get_momentum(signmuon_t h, int m, float* dst);
int signmuon_set_momentum(signmuon_t h, int m, const float* src);
/* The warm power-iteration state of a SIGNMUON_PI_WARM handle, the rest of
 * what a checkpoint needs besides W and the momentum: which = 0 for the
 * M-worker problems (signmuon_info out[6] floats), 1 for the one-problem-set
 * PolarNS (out[7] floats).  dst / src are device float buffers of that size.
 * A zero state makes the next power iteration start cold.  E_UNSUPPORTED
 * without SIGNMUON_PI_WARM. */
int signmuon_get_pi_state(signmuon_t h, int which, float* dst);
int signmuon_set_pi_state(signmuon_t h, int which, const float* src);
int signmuon_get_polar(signmuon_t h, int m, float* dst);
int signmuon_get_signs(signmuon_t h, int m, uint8_t* dst);
int signmuon_get_ternary_signs(signmuon_t h, int m, int8_t* dst);
int signmuon_get_direction(signmuon_t h, float* dst);
int signmuon_get_scales(signmuon_t h, float* dst_host);
/* get_gram: the Gram matrix (g x g, g = min(rows, cols), row-major floats on
 * the host) that the last Newton-Schulz iteration of worker m used for
 * matrix `mat`: X X^T of the wide orientation; after one iteration it is the
 * unscaled Gram of the staged momentum (waits for the GPU).  On the bf16 path
 * with the cubic polynomial, iterations after the first store the apply's
 * whole operator a I + b X X^T there instead (the a X term folded into it);
 * a handle that iterates in Gram space (SIGNMUON_NS_GRAM)
 * leaves one of the iteration's m x m iterates A_k there.  After a post-vote
 * step, worker 0's slot holds the post-vote step's. */
int signmuon_get_gram(signmuon_t h, int m, int mat, float* dst_host);

/* Newton-Schulz coefficients: n=2 (a, b) for X <- aX + b(XX^T)X ([paper] §3
 * two-coefficient form), n=3 (a, b, c) for the quintic flag.  Defaults:
 * (1.5, -0.5) and (15/8, -10/8, 3/8). */
int signmuon_set_ns_coeffs(signmuon_t h, const float* coeffs, int n);

/* Wait for the handle's stream; returns the first deferred error
 * (E_NONFINITE, E_TIMEOUT, E_CUDA) since the last sync, and clears it.  Until
 * then a deferred error stays set: later SIGNMUON_ASYNC calls on the handle
 * run but leave W unchanged. */
int signmuon_sync(signmuon_t h);

/* Sizes: out[0]=d, out[1]=packed bytes per worker, out[2]=device bytes owned
 * by the handle, out[3]=number of shape groups, out[4]=M, out[5]=n_mats,
 * out[6]=power-iteration state floats of the M-worker problems,
 * out[7]=those of one problem set (n <= 8 values are written). */
int signmuon_info(signmuon_t h, int64_t* out, int n);

/* Host-only planning (no GPU needed): same outputs as signmuon_info for a
 * would-be handle; validates like signmuon_init. */
int signmuon_plan(const int64_t* shapes, int n_mats, int M, int K, int scale, int P,
                  unsigned flags, int64_t* out, int n);

/* Host-only: the plan's tables as JSON text, for inspection and for checking
 * the planner without a GPU.  The tables are the shape groups and their
 * buffer bases, the matrices, the 4096-entry chunks of the elementwise
 * kernels, the GEMM tile lists per op (Gram, quintic square, apply) for M
 * workers and for one, each with its tensor-core schedule for a 148-SM B200
 * (empty for round robin) and both makespans, the power-iteration tiles (the 128 x 128 tiles on and
 * above each Gram's diagonal), row slices, vector and partial-sum offsets, and
 * the buffer sizes.  *need receives the text's size in bytes, with the
 * terminating NUL.  buf may be NULL to ask for the size; a non-NULL buf
 * shorter than that returns E_INVALID.  Validates like signmuon_init. */
int signmuon_plan_tables(const int64_t* shapes, int n_mats, int M, int K, int scale, int P,
                         unsigned flags, char* buf, int64_t cap, int64_t* need);

/* Per-kernel timing.  signmuon_profile(h, 1) makes the following calls record
 * a CUDA event pair around every kernel they launch on the handle's stream;
 * signmuon_profile_read() waits for the stream, adds up the elapsed times per
 * kind (ms[k], launches[k] for k < n) since the last read, and resets them.
 * Kinds: 0 momentum pass, 1 norm finalisation, 2/3/4 Newton-Schulz GEMMs
 * (Gram, quintic square, apply), 5 power iteration, 6 one-bit pack (only
 * when the signs are not packed inside the last GEMM) or ternary sign, 7 vote
 * (fused with the update, or with the staging of the majority for the
 * post-vote step), 8 staging of the mean momentum (MUON_MEAN), 9/10/11
 * post-vote Newton-Schulz GEMMs (Gram, square, apply), 12 update, 13 K=0
 * scaling. */
#define SIGNMUON_PROF_KINDS 14
int signmuon_profile(signmuon_t h, int enable);
int signmuon_profile_read(signmuon_t h, double* ms, int64_t* launches, int n);

/* ------------------------------------------------------------------------
 * signmuon_spectral_norm_noalloc -- power-iteration estimate of the largest
 * singular value of one matrix, for callers that cannot allocate device
 * memory (code running under CUDA graph capture, frameworks that own all
 * device memory through their own allocator, real-time paths that must not
 * enter the driver's allocator).  It needs no handle and allocates nothing:
 * its working vectors live in one static device array of 1,048,576 floats
 * (4 MiB) that every GPU loading this library holds until the process exits.
 * The paper has no counterpart to this call; it is the step's spectral scale
 * made available on its own.
 *   X       device float[rows*cols], row-major.
 *   rows, cols >= 1 with max(rows,cols) + 2*min(rows,cols) <= 1048576;
 *           larger sizes return SIGNMUON_E_INVALID (see signmuon_last_error(NULL)).
 *   P       power iterations >= 1.
 *   sigma   device float[1], receives the estimate.
 *   stream  cudaStream_t (NULL = the legacy default stream).
 * Same estimate as the step's spectral scale: on the orientation whose small
 * side is m, u0 = ones/sqrt(m), u <- X(X^T u)/||X(X^T u)||, P times, then
 * sigma = ||X^T u||; computed in fp32 from X directly.
 * The first call on a device looks up the static array's device address
 * (and may load the library's device code); make that first call before any
 * stream capture.  All calls share the array and every call rewrites what it
 * reads; calls that overlap on the same GPU (for example on different
 * streams) race on it -- serialize them.  Enqueued on
 * `stream`; returns without waiting.
 * ---------------------------------------------------------------------- */
int signmuon_spectral_norm_noalloc(const float* X, int64_t rows, int64_t cols, int P, float* sigma,
                                   void* stream);

/* Number of kernels this library has launched in this process (all handles). */
int64_t signmuon_kernel_launches(void);

const char* signmuon_last_error(signmuon_t h);
const char* signmuon_status_string(int status);
void signmuon_destroy(signmuon_t h);

#ifdef __cplusplus
}
#endif
#endif /* SIGNMUON_H */
