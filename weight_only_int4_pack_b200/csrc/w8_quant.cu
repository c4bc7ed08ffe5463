// w8_quant.cu -- the 8-bit side of the W8A8 layer: SmoothQuant factors,
// per-tensor symmetric INT8 / FP8 E4M3 quantization, and w8a8_linear (the
// activations quantized on the fly, then the 8-bit GEMM of w8_gemm.cu).
//
// Method: "LLM quantization methods: principles and implementation"
// (zhiyuanblog.org/blog/llm-quantization) §2.2 (symmetric: scale = max|x| /
// (2^(b-1) - 1), q = clamp(round(x / scale), -qmax, qmax)), §4.3 SmoothQuant
// (s_j = max|X_j|^alpha / max|W_j|^(1-alpha), clamped below at 1e-5;
// X' = X / s, W' = W * s; both INT8 per tensor, the activations at run time)
// and §4.6 FP8 (scale = max|x| / 448, cast to E4M3).
//
// Per-tensor quantization is two passes over the tensor: amax_kernel (a
// max-reduction of |v| -- per-column maxima of |a|, the column op applied once
// per column -- with one atomicMax on the float's bits per CTA -- the
// bits of non-negative floats order like the values, and max does not depend
// on the order, so the result is exact and deterministic), then quant8_kernel
// (every thread derives the scale from amax; CTA 0 publishes it).  Column
// maxima for the smoothing factors work the same way, one word per column.

#include <cuda_fp8.h>

#include <math.h>

#include "w4_half.cuh"
#include "w4_internal.cuh"
#include "w8a8.h"

namespace w4 {
namespace {

constexpr int kColTile = 256;    // columns per CTA of the column-max pass
constexpr int kChunkRows = 256;  // rows per CTA of the column-max pass

template <int OP>
__device__ __forceinline__ float col_apply(float x, float c) {
    if (OP == W8_COL_MUL) return __fmul_rn(x, c);
    if (OP == W8_COL_DIV) return __fdiv_rn(x, c);
    return x;
}

// v[0..7] = col_apply(A[i*8 + j], col[k0 + j]) for the i-th 8-element word.
template <int XT, int OP>
__device__ __forceinline__ void load_v8(const uint16_t *__restrict__ A,
                                        const float *__restrict__ col, int64_t i, int64_t K,
                                        float v[8]) {
    widen8<XT>(__ldg(reinterpret_cast<const uint4 *>(A) + i), v);
    if (OP != W8_COL_NONE) {
        const int64_t k0 = (i * 8) % K;
        const float4 c0 = __ldg(reinterpret_cast<const float4 *>(col + k0));
        const float4 c1 = __ldg(reinterpret_cast<const float4 *>(col + k0 + 4));
        const float c[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] = col_apply<OP>(v[j], c[j]);
    }
}

__device__ __forceinline__ unsigned block_max_bits(unsigned b, unsigned *red) {
    b = __reduce_max_sync(0xffffffffu, b);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (lane == 0) red[warp] = b;
    __syncthreads();
    unsigned m = 0;
    if (threadIdx.x == 0)
        for (int q = 0; q < static_cast<int>(blockDim.x >> 5); ++q) m = max(m, red[q]);
    return m;  // valid in thread 0
}

// *amax_bits = max(*amax_bits, bits of max |v|) over the tensor (zeroed before).
// Thread (x, y) owns the 8-column word x of the rows y, y + gridDim.y, ... and
// keeps the largest |a| of each of its columns; the column op is applied once
// per column at the end.  That is exact: the correctly rounded product or
// quotient by a fixed factor is monotone in |a|, so the largest |fl(a op c)|
// of a column is fl(max |a| op |c|).
template <int XT, int OP>
__global__ void __launch_bounds__(256) amax_kernel(const uint16_t *__restrict__ A, int64_t rows,
                                                   int64_t K, const float *__restrict__ col,
                                                   unsigned *__restrict__ amax_bits) {
    __shared__ unsigned red[8];
    const int64_t w = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int64_t words = K / 8;
    float m[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) m[j] = 0.0f;
    if (w < words) {
        for (int64_t r = blockIdx.y; r < rows; r += gridDim.y) {
            float f[8];
            widen8<XT>(__ldg(reinterpret_cast<const uint4 *>(A + r * K) + w), f);
#pragma unroll
            for (int j = 0; j < 8; ++j) m[j] = fmaxf(m[j], fabsf(f[j]));
        }
    }
    float best = 0.0f;
    if (w < words) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            float v = m[j];
            if (OP != W8_COL_NONE) v = fabsf(col_apply<OP>(v, fabsf(__ldg(col + 8 * w + j))));
            best = fmaxf(best, v);
        }
    }
    const unsigned b = block_max_bits(__float_as_uint(best), red);
    if (threadIdx.x == 0) atomicMax(amax_bits, b);
}

// q = codes of v / scale, scale = fl32(amax / qmax); scale[1] holds amax,
// CTA 0 writes scale[0].
template <int XT, int OP, int FMT>
__global__ void __launch_bounds__(256) quant8_kernel(const uint16_t *__restrict__ A, int64_t n8,
                                                     int64_t K, const float *__restrict__ col,
                                                     float *__restrict__ scale,
                                                     uint8_t *__restrict__ q) {
    const float amax = scale[1];
    const float sc = __fdiv_rn(amax, FMT == W8_INT8 ? 127.0f : 448.0f);
    if (blockIdx.x == 0 && threadIdx.x == 0) scale[0] = sc;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        uint32_t lo = 0, hi = 0;
        if (sc != 0.0f) {
            float v[8];
            load_v8<XT, OP>(A, col, i, K, v);
            uint32_t b[8];
            if (FMT == W8_INT8) {
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float r = fminf(fmaxf(rintf(__fdiv_rn(v[j], sc)), -127.0f), 127.0f);
                    b[j] = static_cast<uint32_t>(static_cast<int>(r)) & 0xFFu;
                }
            } else {
#pragma unroll
                for (int j = 0; j < 8; j += 2) {
                    const __nv_fp8x2_storage_t p = __nv_cvt_float2_to_fp8x2(
                        make_float2(__fdiv_rn(v[j], sc), __fdiv_rn(v[j + 1], sc)), __NV_SATFINITE,
                        __NV_E4M3);
                    b[j] = p & 0xFFu;
                    b[j + 1] = (p >> 8) & 0xFFu;
                }
            }
            lo = b[0] | (b[1] << 8) | (b[2] << 16) | (b[3] << 24);
            hi = b[4] | (b[5] << 8) | (b[6] << 16) | (b[7] << 24);
        }
        reinterpret_cast<uint2 *>(q)[i] = make_uint2(lo, hi);
    }
}

// colmax[c] = max(colmax[c], bits of max_r |A[r][c]|) (zeroed before).
// Grid (ceil(K / kColTile), ceil(rows / kChunkRows)); lane l of warp q reads
// columns 8l..8l+7 of the tile in rows q, q + 8, ... of the chunk.
template <int XT>
__global__ void __launch_bounds__(256) colmax_kernel(const uint16_t *__restrict__ A, int64_t rows,
                                                     int64_t K, unsigned *__restrict__ colmax) {
    __shared__ float red[8][kColTile];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t c0 = static_cast<int64_t>(blockIdx.x) * kColTile + lane * 8;
    const int64_t r0 = static_cast<int64_t>(blockIdx.y) * kChunkRows;
    const int64_t r1 = min(rows, r0 + kChunkRows);
    float m[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) m[i] = 0.0f;
    if (c0 < K) {
#pragma unroll 4
        for (int64_t r = r0 + warp; r < r1; r += 8) {
            float f[8];
            widen8<XT>(__ldg(reinterpret_cast<const uint4 *>(A + r * K + c0)), f);
#pragma unroll
            for (int i = 0; i < 8; ++i) m[i] = fmaxf(m[i], fabsf(f[i]));
        }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) red[warp][lane * 8 + i] = m[i];
    __syncthreads();
    const int64_t c = static_cast<int64_t>(blockIdx.x) * kColTile + threadIdx.x;
    if (c < K) {
        float v = 0.0f;
#pragma unroll
        for (int q = 0; q < 8; ++q) v = fmaxf(v, red[q][threadIdx.x]);
        atomicMax(colmax + c, __float_as_uint(v));
    }
}

__global__ void smooth_finish(const unsigned *__restrict__ ax, const unsigned *__restrict__ aw,
                              int64_t K, double alpha, float *__restrict__ s) {
    const int64_t c = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (c >= K) return;
    const float a = __uint_as_float(ax[c]), w = __uint_as_float(aw[c]);
    if (a == 0.0f || w == 0.0f) {
        s[c] = 1.0f;
        return;
    }
    const float num = __double2float_rn(pow(static_cast<double>(a), alpha));
    const float den = __double2float_rn(pow(static_cast<double>(w), 1.0 - alpha));
    const float v = __fdiv_rn(num, den);
    s[c] = v < 1e-5f ? 1e-5f : v;
}

template <int XT, int OP, int FMT>
int quantize_t(const uint16_t *A, int64_t rows, int64_t K, const float *col, float *scale,
               uint8_t *q, cudaStream_t stream) {
    DeviceInfo di;
    int st = device_info(&di);
    if (st != W4_OK) return st;
    const int64_t n8 = rows * K / 8;
    const int64_t want = (n8 + 255) / 256, cap = int64_t(4) * di.sm_count;
    const unsigned grid = static_cast<unsigned>(want < cap ? want : cap);
    cudaError_t e = cudaMemsetAsync(scale + 1, 0, sizeof(float), stream);
    if (e != cudaSuccess) return cuda_fail("cudaMemsetAsync(amax)", e);
    const int64_t words = K / 8;
    const unsigned gx = static_cast<unsigned>((words + 255) / 256);
    int64_t gy = cap / gx;
    if (gy < 1) gy = 1;
    if (gy > rows) gy = rows;
    if (gy > 65535) gy = 65535;
    amax_kernel<XT, OP><<<dim3(gx, static_cast<unsigned>(gy)), 256, 0, stream>>>(
        A, rows, K, col, reinterpret_cast<unsigned *>(scale + 1));
    quant8_kernel<XT, OP, FMT><<<grid, 256, 0, stream>>>(A, n8, K, col, scale, q);
    return cuda_status(cudaGetLastError());
}

template <int XT, int OP>
int quantize_fmt(const uint16_t *A, int64_t rows, int64_t K, const float *col, int fmt,
                 float *scale, uint8_t *q, cudaStream_t stream) {
    if (fmt == W8_INT8) return quantize_t<XT, OP, W8_INT8>(A, rows, K, col, scale, q, stream);
    return quantize_t<XT, OP, W8_E4M3>(A, rows, K, col, scale, q, stream);
}

template <int XT>
int quantize_op(const uint16_t *A, int64_t rows, int64_t K, const float *col, int op, int fmt,
                float *scale, uint8_t *q, cudaStream_t stream) {
    if (op == W8_COL_MUL)
        return quantize_fmt<XT, W8_COL_MUL>(A, rows, K, col, fmt, scale, q, stream);
    if (op == W8_COL_DIV)
        return quantize_fmt<XT, W8_COL_DIV>(A, rows, K, col, fmt, scale, q, stream);
    return quantize_fmt<XT, W8_COL_NONE>(A, rows, K, col, fmt, scale, q, stream);
}

int quantize8(const void *A, int at, int64_t rows, int64_t K, const float *col, int op, int fmt,
              float *scale, void *q, cudaStream_t stream) {
    const uint16_t *a = static_cast<const uint16_t *>(A);
    uint8_t *qq = static_cast<uint8_t *>(q);
    if (at == W4_F16) return quantize_op<W4_F16>(a, rows, K, col, op, fmt, scale, qq, stream);
    return quantize_op<W4_BF16>(a, rows, K, col, op, fmt, scale, qq, stream);
}

int reject(int status, const char *fn, const char *why) { return set_error(status, fn, why); }

bool valid_dt(int t) { return t == W4_F16 || t == W4_BF16; }
bool valid_fmt(int f) { return f == W8_INT8 || f == W8_E4M3; }

const char *check_rows_k(int64_t rows, int64_t K) {
    if (rows <= 0 || K <= 0) return "rows and K must be >= 1";
    if (K % 16 != 0) return "K must be a multiple of 16";
    if (rows >= (int64_t(1) << 31) || K >= (int64_t(1) << 31)) return "rows and K must be below 2^31";
    if (rows > (int64_t(1) << 40) / K) return "rows * K too large";
    return nullptr;
}

}  // namespace
}  // namespace w4

using w4::reject;

extern "C" int w8_smooth_scales(const void *X, const void *W, int xt, int64_t Mc, int64_t K,
                                int64_t N, float alpha, float *s, void *workspace,
                                size_t workspace_bytes, void *stream) {
    const char *fn = "w8_smooth_scales";
    if (!w4::valid_dt(xt)) return reject(W4_ERR_INVALID_ARG, fn, "bad dtype");
    if (const char *why = w4::check_rows_k(Mc > N ? Mc : N, K)) return reject(W4_ERR_INVALID_ARG, fn, why);
    if (Mc <= 0 || N <= 0) return reject(W4_ERR_INVALID_ARG, fn, "Mc and N must be >= 1");
    if ((Mc > N ? Mc : N) > int64_t(65535) * w4::kChunkRows)
        return reject(W4_ERR_INVALID_ARG, fn, "Mc and N must be at most 16776960");
    if (!(alpha >= 0.0f && alpha <= 1.0f)) return reject(W4_ERR_INVALID_ARG, fn, "alpha must lie in [0, 1]");
    if (!X || !W || !s || !workspace) return reject(W4_ERR_INVALID_ARG, fn, "null pointer");
    if (workspace_bytes < size_t(8) * size_t(K))
        return reject(W4_ERR_INVALID_ARG, fn, "workspace smaller than 8 * K bytes");
    if (!w4::aligned16(X) || !w4::aligned16(W) || !w4::aligned16(workspace))
        return reject(W4_ERR_UNSUPPORTED, fn, "pointers must be 16-byte aligned");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    unsigned *ax = static_cast<unsigned *>(workspace);
    unsigned *aw = ax + K;
    cudaError_t e = cudaMemsetAsync(workspace, 0, size_t(8) * size_t(K), st);
    if (e != cudaSuccess) return w4::cuda_fail("cudaMemsetAsync(column maxima)", e);
    const unsigned tiles = static_cast<unsigned>((K + w4::kColTile - 1) / w4::kColTile);
    const unsigned cx = static_cast<unsigned>((Mc + w4::kChunkRows - 1) / w4::kChunkRows);
    const unsigned cw = static_cast<unsigned>((N + w4::kChunkRows - 1) / w4::kChunkRows);
    const uint16_t *x = static_cast<const uint16_t *>(X), *w = static_cast<const uint16_t *>(W);
    if (xt == W4_F16) {
        w4::colmax_kernel<W4_F16><<<dim3(tiles, cx), 256, 0, st>>>(x, Mc, K, ax);
        w4::colmax_kernel<W4_F16><<<dim3(tiles, cw), 256, 0, st>>>(w, N, K, aw);
    } else {
        w4::colmax_kernel<W4_BF16><<<dim3(tiles, cx), 256, 0, st>>>(x, Mc, K, ax);
        w4::colmax_kernel<W4_BF16><<<dim3(tiles, cw), 256, 0, st>>>(w, N, K, aw);
    }
    w4::smooth_finish<<<static_cast<unsigned>((K + 255) / 256), 256, 0, st>>>(
        ax, aw, K, static_cast<double>(alpha), s);
    return w4::cuda_status(cudaGetLastError());
}

extern "C" int w8_quantize(const void *A, int at, int64_t rows, int64_t K, const float *col,
                           int col_op, int fmt, void *q, float *scale, void *stream) {
    const char *fn = "w8_quantize";
    if (!w4::valid_dt(at)) return reject(W4_ERR_INVALID_ARG, fn, "bad dtype");
    if (!w4::valid_fmt(fmt)) return reject(W4_ERR_INVALID_ARG, fn, "fmt is not W8_INT8 or W8_E4M3");
    if (col_op < W8_COL_NONE || col_op > W8_COL_DIV) return reject(W4_ERR_INVALID_ARG, fn, "bad col_op");
    if (const char *why = w4::check_rows_k(rows, K)) return reject(W4_ERR_INVALID_ARG, fn, why);
    if (!A || !q || !scale || (col_op != W8_COL_NONE && !col))
        return reject(W4_ERR_INVALID_ARG, fn, "null pointer");
    if (!w4::aligned16(A) || !w4::aligned16(q) ||
        (col_op != W8_COL_NONE && !w4::aligned16(col)) ||
        (reinterpret_cast<uintptr_t>(scale) & 7u) != 0)
        return reject(W4_ERR_UNSUPPORTED, fn,
                      "A, q and col must be 16-byte aligned, scale 8-byte aligned");
    return w4::quantize8(A, at, rows, K, col, col_op, fmt, scale, q,
                         static_cast<cudaStream_t>(stream));
}

extern "C" size_t w8a8_workspace_bytes(int64_t M, int64_t K) {
    if (w4::check_rows_k(M, K)) return 0;
    return (size_t(M) * size_t(K) + 256 + 255) & ~size_t(255);
}

extern "C" int w8a8_linear(const void *X, int xt, int64_t M, int64_t K, const float *s, int fmt,
                           const void *Wq, const float *w_scale, int64_t N, void *Y,
                           void *workspace, size_t workspace_bytes, void *stream) {
    const char *fn = "w8a8_linear";
    if (!w4::valid_dt(xt)) return reject(W4_ERR_INVALID_ARG, fn, "bad dtype");
    if (!w4::valid_fmt(fmt)) return reject(W4_ERR_INVALID_ARG, fn, "fmt is not W8_INT8 or W8_E4M3");
    if (const char *why = w4::check_rows_k(M, K)) return reject(W4_ERR_INVALID_ARG, fn, why);
    if (N <= 0 || N >= (int64_t(1) << 31)) return reject(W4_ERR_INVALID_ARG, fn, "N must be 1 .. 2^31 - 1");
    if (!X || !Wq || !w_scale || !Y || !workspace) return reject(W4_ERR_INVALID_ARG, fn, "null pointer");
    if (workspace_bytes < w8a8_workspace_bytes(M, K))
        return reject(W4_ERR_INVALID_ARG, fn, "workspace smaller than w8a8_workspace_bytes");
    if (!w4::aligned16(X) || !w4::aligned16(Wq) || !w4::aligned16(Y) || (s && !w4::aligned16(s)) ||
        (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return reject(W4_ERR_UNSUPPORTED, fn,
                      "X, Wq, Y and s must be 16-byte aligned, the workspace 256-byte aligned");
    unsigned char *ws = static_cast<unsigned char *>(workspace);
    float *x_scale = reinterpret_cast<float *>(ws);
    void *Xq = ws + 256;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int r = w4::quantize8(X, xt, M, K, s, s ? W8_COL_DIV : W8_COL_NONE, fmt, x_scale, Xq, st);
    if (r != W4_OK) return r;
    return w8_gemm(Xq, x_scale, Wq, w_scale, fmt, M, K, N, Y, xt, stream);
}
