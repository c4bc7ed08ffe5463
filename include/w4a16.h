/*
 * w4a16.h -- C ABI of libw4a16.so: per-group INT4 round-to-nearest weight
 * quantization and the W4A16 linear layer on NVIDIA B200 (sm_100a).
 *
 * Method sources (cited by page title and section):
 *   [LQ]  "LLM quantization methods: principles and implementation"
 *         (zhiyuanblog.org/blog/llm-quantization): §1 (0.5 byte per INT4
 *         parameter), §2.2 (symmetric and asymmetric integer quantization,
 *         scale and zero point, round, clamp, dequantize), §2.3 (per-group
 *         granularity along in_features, in_features % group == 0),
 *         §4.1 (GPTQ: H = 2XX^T, column-wise quantization with the error
 *         pushed through the inverse Hessian),
 *         §4.2 (AWQ: weights multiplied by a per-input-channel factor before
 *         quantizing; the factor (a/w)^alpha from mean activation and weight
 *         magnitudes, alpha chosen by a grid search on the layer's output
 *         error).
 *   [PTQ] "PTQ weight quantization: from GPTQ to AWQ" (jonathanding.github.io),
 *         sections "Round-to-Nearest" and "AWQ".
 *   [MF]  "Quantization method families" (inference-learning-path.pages.dev),
 *         §2: W4A16 keeps activations in 16-bit floats and dequantizes the
 *         weights in front of the matmul; decode is bound by weight bandwidth,
 *         prefill by compute.
 *
 * Conventions shared by every entry point:
 *   - All array arguments are DEVICE pointers of the current CUDA device,
 *     allocated and owned by the caller; the library allocates no memory
 *     (exception: the first w4_awq_search on a device creates a cuBLAS
 *     handle there, which allocates its own workspace).
 *     Base pointers must be 16-byte aligned (else W4_ERR_UNSUPPORTED).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Every call only enqueues work and returns: results are ready once the
 *     caller synchronizes that stream.  Launch failures return W4_ERR_CUDA;
 *     faults inside a kernel surface at the caller's synchronization.
 *   - Arguments are validated on the host before anything is enqueued; an
 *     invalid call returns its status and touches no memory.
 *   - Matrices are row-major.  W is [N][K] = (out_features x in_features); X is
 *     [M][K]; Y is [M][N].  Groups run along K (in_features).
 *   - Inputs must be finite; results for NaN or Inf inputs are unspecified.
 *   - Thread safety: calls on different streams may run concurrently; the
 *     library keeps no per-call host state beyond a per-device cache of
 *     attributes (SM count, kernel attributes) filled on first use.
 */
#ifndef W4A16_H
#define W4A16_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    W4_OK = 0,
    W4_ERR_INVALID_ARG = 1, /* bad shape, null pointer, K % group != 0, ... */
    W4_ERR_UNSUPPORTED = 2, /* valid but not implemented (group size, alignment, dtype) */
    W4_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed while enqueueing */
    W4_ERR_TIMEOUT = 4,     /* a bounded device-side wait ran out (see w4_device_status) */
    W4_ERR_BOUNDS = 5       /* an in-kernel bounds check of the W4_DEBUG build failed */
} w4_status;

typedef enum { W4_F16 = 0, W4_BF16 = 1 } w4_dtype;

/*
 * w4_quantize -- per-group INT4 round-to-nearest quantization and packing.
 * [LQ] §2.2 + §2.3 (+ §4.2 for col_scale); [PTQ] "Round-to-Nearest".
 *
 *   W          [N][K] fp16 or bf16 (wt), the weight (out x in).
 *   col_scale  nullable [K] fp32: AWQ per-input-channel factor; when given,
 *              every weight is first replaced by fl32(w * col_scale[k]).
 *   group      elements per group along K: 32, 64, 128 or 256; K % group == 0
 *              (W4_ERR_INVALID_ARG otherwise).
 *   sym != 0   symmetric:  s = fl(amax / 7), q = clamp(rne(fl(w / s)), -7, 7),
 *              stored code u = q + 8, zeros[] = 8.0f.
 *   sym == 0   asymmetric: s = fl(fl(max - min) / 15),
 *              zp = clamp(rne(fl(-min / s)), 0, 15),
 *              u = clamp(rne(fl(fl(w / s) + zp)), 0, 15), zeros[] = zp.
 *   All arithmetic is IEEE fp32 with round-to-nearest-even; rne() rounds
 *   half to even.  A group whose scale is 0 stores s = 0, zero = 8 (sym) or
 *   0 (asym) and every code equal to that zero, so it dequantizes to 0.
 *   Outputs (caller-allocated):
 *     packed   [N][K/2] bytes.  The codes of k = 8j..8j+7 of a row form the
 *              little-endian 32-bit word j; nibble i (bits 4i..4i+3) of that
 *              word holds k = 8j + {0,2,4,6,1,3,5,7}[i].
 *     scales   [N][K/group] fp32.
 *     zeros    [N][K/group] fp32 (integer values 0..15).
 *   Dequantization of any code: w_hat = (u - zero) * scale.
 *   Requires K % 8 == 0, N >= 1, K >= 1.
 */
int w4_quantize(const void *W, int wt, int64_t K, int64_t N, int group, int sym,
                const float *col_scale, uint8_t *packed, float *scales, float *zeros,
                void *stream);

/*
 * w4a16_workspace_bytes -- scratch bytes w4a16_gemm needs for this shape
 * (0 when it needs none: 1 <= M <= 8 with K <= 4096, and shapes whose row
 * blocks are not split).  The workspace holds per-tile arrival counters
 * (a fixed area at its start) and split-K partial sums.  It must be
 * zero-filled once before its first use; every w4a16_gemm call leaves the
 * counter area zero again when its work completes and fully rewrites the
 * partials it reads, so one workspace serves any number of calls of any
 * shapes issued one after another on ONE stream.  Calls that may overlap on
 * the GPU (other streams) need separate workspaces.  A call whose bounded
 * wait ran out, or (W4_DEBUG build) whose bounds check failed
 * (w4_device_status reports W4_ERR_TIMEOUT or W4_ERR_BOUNDS), may stop
 * partway and leave counters armed: zero-fill the workspace again before
 * reusing it.
 */
size_t w4a16_workspace_bytes(int64_t M, int64_t K, int64_t N, int group);

/*
 * w4a16_gemm -- Y = X * dequant(packed, scales, zeros)^T, the W4A16 linear layer.
 * [MF] §2 (dequant -> 16-bit matmul); dequantization as in [LQ] §2.2.
 *
 *   X        [M][K] fp16 or bf16 (xt); Y [M][N] in the same dtype.
 *   packed, scales, zeros: the layout w4_quantize writes; zeros may be NULL,
 *            which means every zero point is 8 (the symmetric storage).
 *   group    must be 128 (W4_ERR_UNSUPPORTED otherwise).
 *   Each Y[m][n] = sum_k X[m][k] * ((u[n][k] - zero) * scale) is accumulated in
 *   fp32 (the integer (u - zero) is exact in the 16-bit operand type; the
 *   group scale multiplies the fp32 partial sum of its group) and rounded
 *   once to the output dtype.
 *   M = 1 with K % 512 == 0 and K <= 4096 runs the CUDA-core GEMV (three
 *   CTAs of four warps per SM, whole rows streamed per warp, no workspace);
 *   other 1 <= M <= 8
 *   with K <= 4096 the small-M GEMV on warp-level tensor-core MMAs (whole
 *   rows, no workspace); other M <= 32 the persistent stream-K decode path
 *   on tcgen05; larger M runs the
 *   tcgen05 prefill path (TMA-staged X, dequantized W tiles in shared
 *   memory, accumulators in tensor memory).
 *   The decode paths are launched with programmatic dependent launch: they
 *   may start while the preceding kernel of the stream finishes, and they
 *   start streaming the weights before that kernel has completed (the
 *   tcgen05 decode path `packed` only; the GEMVs `packed`, `scales` and
 *   `zeros`).  X, Y and the workspace are touched only after.  So the
 *   weights must not be written by the immediately preceding kernel if that
 *   kernel itself allows early dependent launch (the kernels of this library
 *   that write them do not).
 *   workspace / workspace_bytes: at least w4a16_workspace_bytes(M, K, N, group)
 *   bytes of device memory prepared as described there (may be NULL when
 *   that size is 0); a smaller workspace returns W4_ERR_INVALID_ARG.
 */
int w4a16_gemm(const void *X, int xt, int64_t M, const uint8_t *packed, const float *scales,
               const float *zeros, int64_t K, int64_t N, int group, void *Y, void *workspace,
               size_t workspace_bytes, void *stream);

/*
 * w4a16_gemm_noalloc -- the decode path of w4a16_gemm (M <= 32) for callers
 * that cannot allocate device memory, such as a plugin inside a host
 * application that owns every device allocation, or a latency-critical path
 * where cudaMalloc and the synchronization it may imply are not allowed.  The
 * source pages have no counterpart to this entry point: it is a property of
 * this library's interface, not of the method.
 *
 *   Arguments and result as w4a16_gemm, without the workspace: the scratch
 *   space lives in a 4 MiB device array inside the library, which every GPU
 *   that loads the library holds until the process exits.  The call allocates
 *   nothing (no cudaMalloc, cudaFree or allocating library routine); it clears
 *   the counter area of the array with cudaMemsetAsync on `stream` first.
 *   M > 32 returns W4_ERR_UNSUPPORTED (that path of w4a16_gemm needs no
 *   workspace); a shape whose workspace would exceed 4 MiB returns
 *   W4_ERR_UNSUPPORTED, with the reason in w4_last_error().
 *   All calls on a device share the one array: calls that may overlap on the
 *   GPU (other streams, other host threads) race and give wrong results.
 *   The first call on each device looks up the array's device address with
 *   that device current, which may also load the library's device code and
 *   the 4 MiB array onto the device (CUDA loads modules lazily) -- a step
 *   that can allocate device memory and synchronize.  Make that first call
 *   as a warm-up, outside any latency-critical path and before any stream
 *   capture.  Shapes whose decode kernel uses no scratch space (see
 *   w4a16_workspace_bytes) never touch the array.
 */
int w4a16_gemm_noalloc(const void *X, int xt, int64_t M, const uint8_t *packed,
                       const float *scales, const float *zeros, int64_t K, int64_t N, int group,
                       void *Y, void *stream);

/*
 * w4_awq_search_workspace_bytes -- device scratch bytes w4_awq_search needs
 * for Mc calibration rows and a K-in, N-out layer (0 for a shape it rejects).
 * About 0.57 N K + 6 Mc N + 2 Mc K bytes, plus 8 K bytes of fp64 column
 * partial sums per 256 rows of max(Mc, N) and the decode path's workspace
 * when Mc <= 32.
 */
size_t w4_awq_search_workspace_bytes(int64_t Mc, int64_t K, int64_t N, int group);

/*
 * w4_awq_search -- AWQ per-input-channel scale search for one linear layer.
 * [LQ] §4.2: minimise || Q(W * s)(X / s) - W X || over s_j = (a_j / w_j)^alpha,
 * a_j = mean_i |X_ij| over the calibration rows, w_j = mean_n |W_nj|, alpha
 * grid-searched; [PTQ] "AWQ": XW = (X diag(s)^-1)(diag(s) W).
 *
 *   W          [N][K] fp16 or bf16 (xt): the unquantized weight.
 *   X          [Mc][K] same dtype: calibration activations of the layer.
 *   group, sym the quantizer Q (w4_quantize); group must be 128.
 *   alphas     HOST array of n_alpha (1 .. 64) values in [0, 1]; read during
 *              the call only.
 *   Outputs (device, caller-allocated):
 *     err        [n_alpha] fp64: err[t] = sum_{i,n} (Yq - Yref)^2, the squared
 *                Frobenius norm of the layer's output error at alphas[t];
 *     best_scale [K] fp32: s at the best alpha (all ones if every err is NaN);
 *     best_index [1] int32: the first t with the smallest err (-1 if all NaN);
 *     packed_out, scales_out, zeros_out: nullable (all three or none); when
 *                given, Q(W * best_scale) in the w4_quantize layout, ready for
 *                w4a16_gemm with activations divided by best_scale.
 *   For each alpha:
 *     s_j  = fl32(pow(a_j / w_j, alpha)) in fp64 (s_j = 1 where a_j or w_j is 0);
 *            a_j and w_j are fp64 sums rounded once to fp32 after the division;
 *     Q    = w4_quantize(W, col_scale = s);
 *     Xs   = X / s: fl32 division rounded once to the 16-bit dtype;
 *     Yq   = w4a16_gemm(Xs, Q), the 16-bit output of the W4A16 layer;
 *     Yref = X W^T accumulated and kept in fp32 (cuBLAS GEMM);
 *     err  = fixed-order fp64 sum of (Yq - Yref)^2: repeated calls on the same
 *            device give bit-identical results.
 *   workspace / workspace_bytes: at least w4_awq_search_workspace_bytes(...)
 *   bytes, 256-byte aligned, contents irrelevant (clobbered).  One workspace
 *   per concurrently running search.
 *   Returns W4_ERR_INVALID_ARG for a bad shape, count, alpha, pointer or
 *   workspace; W4_ERR_UNSUPPORTED for group != 128, misaligned pointers or
 *   a missing libcublas.so.12; W4_ERR_CUDA if an enqueue fails.
 *   Besides the stream's work this call takes a process-wide lock around
 *   its cuBLAS call; the first call on a device opens libcublas.so.12 (the
 *   process's copy if already loaded) and creates a cuBLAS handle for that
 *   device, kept until the process exits, so make the first call outside any
 *   stream capture.
 */
int w4_awq_search(const void *W, const void *X, int xt, int64_t Mc, int64_t K, int64_t N,
                  int group, int sym, const float *alphas, int n_alpha, double *err,
                  float *best_scale, int *best_index, uint8_t *packed_out, float *scales_out,
                  float *zeros_out, void *workspace, size_t workspace_bytes, void *stream);

/*
 * w4_gptq_workspace_bytes / w4_gptq_quantize_workspace_bytes -- device
 * scratch bytes of w4_gptq and w4_gptq_quantize (0 for a shape they reject):
 * about 9 K^2 + 4 N K + 512 N bytes (w4_gptq) and 4 N K + 512 N (the loop).
 */
size_t w4_gptq_workspace_bytes(int64_t Mc, int64_t K, int64_t N, int group);
size_t w4_gptq_quantize_workspace_bytes(int64_t K, int64_t N, int group);

/*
 * w4_gptq -- GPTQ quantization of one layer ([LQ] §4.1; [PTQ] "GPTQ"):
 * minimise ||W X^T - W^ X^T|| column by column, pushing each column's
 * rounding error onto the columns not yet quantized through the inverse
 * Hessian, with lazy updates every 128 columns.
 *
 *   W          [N][K] fp16 or bf16 (xt), the weight; X [Mc][K] the same dtype,
 *              the layer's calibration activations.
 *   group      must be 128 (the GPTQ block); K % 128 == 0, K <= 65536,
 *              N <= 8388480; sym as w4_quantize.
 *   percdamp   damping in [0, 1]: H = 2 X^T X + percdamp * mean(diag) * I
 *              (the usual 0.01; the pages give none).
 *   Outputs: packed / scales / zeros in the w4_quantize layout (w4a16_gemm
 *   consumes them unchanged); U_out nullable [K][K] fp32: the factor used
 *   (row-major, upper triangular, zeros below the diagonal).
 *   Steps, all this library's kernels in fp32 with IEEE division and square
 *   root: H = 2 X^T X (tiled GEMM, fp32 accumulation); U = the upper
 *   Cholesky factor of H^-1 without forming H^-1 (the blocked Cholesky
 *   factor Lr of the index-reversed H, a blocked triangular inverse, then
 *   U = reversed(Lr^-1)); then the column loop of w4_gptq_quantize.  The call
 *   synchronizes `stream` once, after the factorization, to read its status:
 *   W4_ERR_INVALID_ARG if the damped Hessian is not positive definite (e.g. X
 *   all zero with damping).  No library is called.
 *   workspace: w4_gptq_workspace_bytes bytes, 256-byte aligned, clobbered.
 */
int w4_gptq(const void *W, const void *X, int xt, int64_t Mc, int64_t K, int64_t N, int group,
            int sym, float percdamp, uint8_t *packed, float *scales, float *zeros, float *U_out,
            void *workspace, size_t workspace_bytes, void *stream);

/*
 * w4_gptq_quantize -- the GPTQ column loop alone, given U.
 *   W [N][K] (wt), U [K][K] fp32 row-major, upper triangle read (U^T U is the
 *   damped inverse Hessian; U[j][j] > 0).  For every row, for each block of
 *   128 columns: the group's scale and zero point from the row's current
 *   weights (w4_quantize's formulas, fp32); then for each column j in order:
 *   code u_j (w4_quantize's rounding), err_j = (w_j - (u_j - z) s) / U[j][j],
 *   w_k = fma(-err_j, U[j][k], w_k) for the block's k > j; after the block,
 *   for every later column k: w_k = w_k - acc with acc the fp32 fma chain of
 *   err_j U[j][k] over the block's j in order.  All fp32, IEEE division, so
 *   the codes are a fixed function of W and U.  Asynchronous; no library.
 */
int w4_gptq_quantize(const void *W, int wt, int64_t K, int64_t N, int group, int sym,
                     const float *U, uint8_t *packed, float *scales, float *zeros,
                     void *workspace, size_t workspace_bytes, void *stream);

/*
 * w4_device_status -- reads (and, if reset != 0, clears) the current device's
 * status word that kernels set when a bounded wait runs out or, in the
 * W4_DEBUG build, when a bounds check fails.  Synchronizes the device first.
 * Returns W4_OK, W4_ERR_BOUNDS (a check failed; takes precedence),
 * W4_ERR_TIMEOUT, or W4_ERR_CUDA if the read fails.
 */
int w4_device_status(int reset);

/*
 * W4_DEBUG build (the pages have no counterpart; it stands in for a memory
 * checker).  Built with -DW4_DEBUG (python -m weight_only_int4_pack_b200.build
 * --debug, which writes libw4a16_debug.so), the decode, GEMV, prefill and
 * quantizer kernels check every global and shared-memory index and every
 * bulk / tensor copy they issue against the extents of their buffers.  A
 * failed check does not trap: it sets the status word (W4_ERR_BOUNDS, read
 * by w4_device_status) with the file and source line of the first failure,
 * and the thread skips the access, so the context stays usable and the
 * results of that call are undefined.  The normal build has no checks.
 *
 * w4_debug_build -- 1 if this library was built with W4_DEBUG, else 0.
 * w4_debug_first_failure -- synchronizes the device and writes the file id
 *   and line of the first failed check since the status word was last
 *   cleared (0 and 0 if none); does not clear it.  File ids: 1 w4_quantize.cu,
 *   2 w4_decode.cu, 3 w4_prefill.cu, 4 w4_gemv.cu, 5 w4_gemv1.cu.  Returns
 *   W4_OK, W4_ERR_INVALID_ARG for a null pointer, or W4_ERR_CUDA.
 */
int w4_debug_build(void);
int w4_debug_first_failure(int *file_id, int *line);

/*
 * w4_selftest_wait_timeout -- failure-detection self-test (the pages have no
 * counterpart).  Enqueues on `stream` one small kernel whose only mbarrier
 * wait can never complete (nothing arrives on the barrier).  The wait is
 * bounded by timeout_us microseconds (1 .. 1000000), exactly as every wait
 * of the library's kernels is bounded by its own limit: when it runs out the
 * kernel sets the device status word and returns, and the CUDA context stays
 * usable.  A caller (or a test) checks the mechanism with
 * w4_device_status(1) == W4_ERR_TIMEOUT afterwards.
 * Returns W4_OK once the kernel is enqueued, W4_ERR_INVALID_ARG for a
 * timeout out of range, W4_ERR_CUDA if the launch fails.
 */
int w4_selftest_wait_timeout(unsigned timeout_us, void *stream);

/*
 * w4_last_error -- text describing the most recent failure on the calling
 * thread: which check or which CUDA call failed, and why ("" if none yet).
 * Thread-local storage owned by the library, valid until the thread's next
 * failing call; never NULL.
 */
const char *w4_last_error(void);

/* Human-readable name of a status code (static storage; never NULL). */
const char *w4_status_string(int status);

/* ABI version of this header: (major << 16) | minor. */
int w4_abi_version(void);

#define W4A16_ABI_VERSION 0x00010003

#ifdef __cplusplus
}
#endif

#endif /* W4A16_H */
