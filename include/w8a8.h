/*
 * w8a8.h -- C ABI of libw4a16.so, second workload: the W8A8 linear layer with
 * per-tensor INT8 (SmoothQuant) or FP8 E4M3 weights and activations on NVIDIA
 * B200 (sm_100a, tcgen05.mma kind::i8 / kind::f8f6f4).
 *
 * Method sources (cited by page title and section):
 *   [LQ]  "LLM quantization methods: principles and implementation"
 *         (zhiyuanblog.org/blog/llm-quantization): §2.2 symmetric integer
 *         quantization (scale = max|x| / (2^(b-1) - 1), round, clamp);
 *         §4.3 SmoothQuant (s_j = max|X_j|^alpha / max|W_j|^(1-alpha), clamped
 *         below at 1e-5; X' = X / s, W' = W * s, X'W' = XW; W8A8 with both
 *         operands INT8 per tensor, activations quantized at inference);
 *         §4.6 FP8 E4M3 (scale = max|x| / 448, x / scale cast to E4M3).
 *   [MF]  "Quantization method families" (inference-learning-path.pages.dev),
 *         §3.3 SmoothQuant and §3.4 FP8: W8A8 runs the matmul on 8-bit
 *         tensor cores; FP8 activations are scaled per tensor at run time.
 *
 * Conventions are those of w4a16.h (device pointers owned by the caller,
 * 16-byte aligned; `stream` a cudaStream_t as void*; calls only enqueue;
 * arguments validated on the host before anything is enqueued; row-major;
 * status codes w4_status; w4_last_error() describes a failure).
 * Quantized matrices are [rows][K] bytes: int8 two's complement (W8_INT8) or
 * E4M3 codes (W8_E4M3: 1 sign, 4 exponent bits with bias 7, 3 fraction bits;
 * largest finite 448, no infinities).  K must be a multiple of 16.
 */
#ifndef W8A8_H
#define W8A8_H

#include <stddef.h>
#include <stdint.h>

#include "w4a16.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { W8_INT8 = 0, W8_E4M3 = 1 } w8_format;

/* Column operations of w8_quantize. */
typedef enum { W8_COL_NONE = 0, W8_COL_MUL = 1, W8_COL_DIV = 2 } w8_col_op;

/*
 * w8_smooth_scales -- SmoothQuant factors of one layer ([LQ] §4.3).
 *   X [Mc][K] calibration activations and W [N][K] weights, fp16 or bf16 (xt).
 *   s [K] fp32 out: a_j = max_i |X_ij|, w_j = max_n |W_nj| (exact);
 *     s_j = max(fl32(fl32(a_j^alpha) / fl32(w_j^(1 - alpha))), 1e-5), each power
 *     computed in fp64 and rounded once to fp32; s_j = 1 where a_j or w_j is 0.
 *   alpha in [0, 1] (the pages use 0.5).
 *   workspace: at least 8 * K bytes (contents clobbered).
 */
int w8_smooth_scales(const void *X, const void *W, int xt, int64_t Mc, int64_t K, int64_t N,
                     float alpha, float *s, void *workspace, size_t workspace_bytes,
                     void *stream);

/*
 * w8_quantize -- per-tensor symmetric 8-bit quantization of A [rows][K].
 *   at         fp16 or bf16.
 *   col, col_op: nullable [K] fp32 column factor; W8_COL_MUL replaces each
 *              element by fl32(a * col[k]) (the weight side, W * s), W8_COL_DIV
 *              by fl32(a / col[k]) (the activation side, X / s); W8_COL_NONE
 *              ignores col.
 *   fmt        W8_INT8: scale = fl32(amax / 127), q = clamp(rne(fl32(v / scale)),
 *              -127, 127); W8_E4M3: scale = fl32(amax / 448), q = E4M3 nearest
 *              (ties to even, saturating) of fl32(v / scale).  amax = max |v|
 *              over the whole tensor; amax = 0 gives scale 0 and every q = 0.
 *   q          [rows][K] bytes out.
 *   scale      device float[2] out: scale[0] = the scale, scale[1] = amax.
 *   Two kernels (the amax reduction, then the codes); division is IEEE fp32.
 */
int w8_quantize(const void *A, int at, int64_t rows, int64_t K, const float *col, int col_op,
                int fmt, void *q, float *scale, void *stream);

/*
 * w8_gemm -- the 8-bit layer on quantized operands:
 *   Y[m][n] = (sum_k Xq[m][k] * Wq[n][k]) * fl32(x_scale[0] * w_scale[0]).
 *   Xq [M][K], Wq [N][K] in format fmt; x_scale, w_scale device floats (the
 *   scale[0] written by w8_quantize).  Y [M][N] fp16 or bf16 (yt).
 *   W8_INT8: exact int32 accumulation (|sum| < 2^31 for K < 133000), then
 *     fl32(acc) * fl32(sx * sw) in fp32, rounded once to yt.
 *   W8_E4M3: fp32 accumulation on the tensor cores, then the same epilogue.
 *   One persistent tcgen05 kernel: TMA-staged operands (128-byte swizzle),
 *   tcgen05.mma kind::i8 / kind::f8f6f4, 128 weight rows x 256 activation
 *   rows per tile, two accumulators in tensor memory.
 */
int w8_gemm(const void *Xq, const float *x_scale, const void *Wq, const float *w_scale, int fmt,
            int64_t M, int64_t K, int64_t N, void *Y, int yt, void *stream);

/* w8a8_workspace_bytes -- scratch bytes of w8a8_linear: M * K + 256, rounded up. */
size_t w8a8_workspace_bytes(int64_t M, int64_t K);

/*
 * w8a8_linear -- the W8A8 layer on 16-bit activations, quantized on the fly:
 *   Xq = w8_quantize(X, col = s, W8_COL_DIV, fmt) into the workspace (with
 *   s = NULL: no smoothing), then Y = w8_gemm(Xq, Wq).  X [M][K] fp16 or bf16
 *   (xt); Y [M][N] in the same dtype.  Wq / w_scale come from
 *   w8_quantize(W, col = s, W8_COL_MUL, fmt).
 */
int w8a8_linear(const void *X, int xt, int64_t M, int64_t K, const float *s, int fmt,
                const void *Wq, const float *w_scale, int64_t N, void *Y, void *workspace,
                size_t workspace_bytes, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* W8A8_H */
