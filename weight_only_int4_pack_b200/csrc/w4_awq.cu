// w4_awq.cu -- AWQ scale search: the per-input-channel factor s = (a / w)^alpha
// that minimises the W4A16 layer's output error on calibration activations.
//
// Method: "LLM quantization methods: principles and implementation"
// (zhiyuanblog.org/blog/llm-quantization) §4.2 AWQ: minimise
// || Q(W * s)(X / s) - W X || over the per-input-channel factor s, with
// s_j = (a_j / w_j)^alpha, a_j = mean_i |X_ij| the activation importance of
// channel j, w_j = mean_n |W_nj| its weight magnitude, and alpha in [0, 1]
// picked by a grid search; "PTQ weight quantization: from GPTQ to AWQ",
// section "AWQ" (XW = (X diag(s)^-1)(diag(s) W)).
//
// One call, all on the caller's stream and without host synchronization:
//   1. column statistics (colabs_partial + colabs_finish): fp64 partial sums
//      of |.| over chunks of kChunkRows rows, summed in chunk order, divided
//      by the row count in fp64 and rounded once to fp32;
//   2. the unquantized layer's output Yref = X W^T in fp32 (cuBLAS through
//      w4_libs.cu, fp32 accumulation; a plain dense GEMM, done once per call);
//   3. per alpha: s (awq_scale); Q(W * s) with the library's quantizer
//      (col_scale = s); X / s rounded to the 16-bit dtype (scale_activations);
//      Yq = the W4A16 layer (decode path for Mc <= 32, tcgen05 path above);
//      err = sum (Yq - Yref)^2 in fp64 (sqerr_partial + sqerr_finish, a fixed
//      reduction order, so repeated calls give identical results);
//   4. awq_select: the first alpha with the smallest err and s at that alpha;
//      optionally Q(W * s_best) into the caller's packed / scales / zeros.
//
// Memory per alpha on a 12288 x 4096 layer with 512 calibration rows: the
// quantizer reads W (100 MB) and writes the codes (25 MB), the layer reads the
// codes and X / s, and the error pass reads Yq (12.6 MB) and Yref (25 MB).

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <math.h>

#include "w4_half.cuh"
#include "w4_internal.cuh"

namespace w4 {
namespace {

constexpr int kColTile = 256;    // columns per CTA of the statistics pass (32 lanes x 8)
constexpr int kChunkRows = 256;  // rows per partial sum of the statistics pass
constexpr int kSqBlocks = 592;   // CTAs of the error pass (fixed: fixes the summation order)
constexpr int kMaxAlphas = 64;

struct AlphaList {
    float v[kMaxAlphas];
};

// s_j = (a_j / w_j)^alpha, ratio and power in fp64, rounded once to fp32;
// a channel with a_j == 0 or w_j == 0 keeps s_j = 1.
__device__ __forceinline__ float channel_scale(float a, float w, double alpha) {
    if (a == 0.0f || w == 0.0f) return 1.0f;
    return __double2float_rn(pow(static_cast<double>(a) / static_cast<double>(w), alpha));
}

// part[chunk][c] = sum over the chunk's rows r of |A[r][c]| (fp64).
// Grid (ceil(K / kColTile), ceil(rows / kChunkRows)), 256 threads: lane l of
// warp q reads columns 8l..8l+7 of the tile in rows q, q + 8, ... of the chunk.
template <int XT>
__global__ void __launch_bounds__(256) colabs_partial(const uint16_t *__restrict__ A,
                                                      int64_t rows, int64_t K,
                                                      double *__restrict__ part) {
    __shared__ double red[8][kColTile];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t c0 = static_cast<int64_t>(blockIdx.x) * kColTile + lane * 8;
    const int64_t r0 = static_cast<int64_t>(blockIdx.y) * kChunkRows;
    const int64_t r1 = min(rows, r0 + kChunkRows);
    double acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.0;
    if (c0 < K) {  // K % 8 == 0: the whole 8-column word is inside the row
#pragma unroll 4
        for (int64_t r = r0 + warp; r < r1; r += 8) {
            const uint4 v = __ldg(reinterpret_cast<const uint4 *>(A + r * K + c0));
            float f[8];
            widen8<XT>(v, f);
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] += fabs(static_cast<double>(f[i]));
        }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) red[warp][lane * 8 + i] = acc[i];
    __syncthreads();
    const int64_t c = static_cast<int64_t>(blockIdx.x) * kColTile + threadIdx.x;
    if (c < K) {
        double s = 0.0;
#pragma unroll
        for (int q = 0; q < 8; ++q) s += red[q][threadIdx.x];
        part[static_cast<int64_t>(blockIdx.y) * K + c] = s;
    }
}

// mean[c] = fl32((sum over chunks of part[chunk][c]) / count).
__global__ void colabs_finish(const double *__restrict__ part, int64_t nchunk, int64_t K,
                              int64_t count, float *__restrict__ mean) {
    const int64_t c = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (c >= K) return;
    double s = 0.0;
    for (int64_t ch = 0; ch < nchunk; ++ch) s += part[ch * K + c];
    mean[c] = __double2float_rn(s / static_cast<double>(count));
}

__global__ void awq_scale(const float *__restrict__ a, const float *__restrict__ w, int64_t K,
                          double alpha, float *__restrict__ s) {
    const int64_t c = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (c < K) s[c] = channel_scale(a[c], w[c], alpha);
}

// Xs[i][k] = 16-bit(fl32(X[i][k]) / s[k]) with IEEE division; 8 elements per
// thread (K % 8 == 0, so the 8 share one row).
template <int XT>
__global__ void __launch_bounds__(256) scale_activations(const uint16_t *__restrict__ X,
                                                         const float *__restrict__ s,
                                                         int64_t n8, int64_t K,
                                                         uint16_t *__restrict__ Xs) {
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t k0 = (i * 8) % K;
        const uint4 v = __ldg(reinterpret_cast<const uint4 *>(X) + i);
        const float4 s0 = __ldg(reinterpret_cast<const float4 *>(s + k0));
        const float4 s1 = __ldg(reinterpret_cast<const float4 *>(s + k0 + 4));
        const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
        float f[8];
        widen8<XT>(v, f);
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j)
            o[j] = static_cast<uint32_t>(narrow1<XT>(__fdiv_rn(f[2 * j], sv[2 * j]))) |
                   (static_cast<uint32_t>(narrow1<XT>(__fdiv_rn(f[2 * j + 1], sv[2 * j + 1])))
                    << 16);
        reinterpret_cast<uint4 *>(Xs)[i] = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

// Deterministic block sum of one double per thread (256 threads).
__device__ __forceinline__ double block_sum(double v, double *red) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (lane == 0) red[warp] = v;
    __syncthreads();
    double s = 0.0;
    if (threadIdx.x == 0)
        for (int q = 0; q < 8; ++q) s += red[q];
    return s;  // valid in thread 0
}

// part[b] = sum over this CTA's elements of (Yq - Yref)^2 (fp64).  Element
// words of 8 are dealt round-robin over the kSqBlocks x 256 threads; block 0
// also takes the last E % 8 elements.
template <int XT>
__global__ void __launch_bounds__(256) sqerr_partial(const uint16_t *__restrict__ Yq,
                                                     const float *__restrict__ Yref, int64_t E,
                                                     double *__restrict__ part) {
    __shared__ double red[8];
    const int64_t E8 = E / 8;
    double acc = 0.0;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x; i < E8;
         i += static_cast<int64_t>(kSqBlocks) * 256) {
        const uint4 q = __ldg(reinterpret_cast<const uint4 *>(Yq) + i);
        const float4 r0 = __ldg(reinterpret_cast<const float4 *>(Yref) + 2 * i);
        const float4 r1 = __ldg(reinterpret_cast<const float4 *>(Yref) + 2 * i + 1);
        const float r[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
        float f[8];
        widen8<XT>(q, f);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const double d = static_cast<double>(f[j]) - static_cast<double>(r[j]);
            acc += d * d;
        }
    }
    if (blockIdx.x == 0)
        for (int64_t e = E8 * 8 + threadIdx.x; e < E; e += 256) {
            const double d = static_cast<double>(widen1<XT>(Yq[e])) - static_cast<double>(Yref[e]);
            acc += d * d;
        }
    const double s = block_sum(acc, red);
    if (threadIdx.x == 0) part[blockIdx.x] = s;
}

__global__ void __launch_bounds__(256) sqerr_finish(const double *__restrict__ part,
                                                    double *__restrict__ err_t) {
    __shared__ double red[8];
    double acc = 0.0;
    for (int b = threadIdx.x; b < kSqBlocks; b += 256) acc += part[b];
    const double s = block_sum(acc, red);
    if (threadIdx.x == 0) *err_t = s;
}

// The first alpha with the smallest err (a NaN err is never chosen; -1 if all
// are NaN) and s at that alpha (all ones when there is none).  One CTA.
__global__ void __launch_bounds__(256) awq_select(const double *__restrict__ err, int n_alpha,
                                                  AlphaList al, const float *__restrict__ a,
                                                  const float *__restrict__ w, int64_t K,
                                                  float *__restrict__ best_scale,
                                                  int *__restrict__ best_index) {
    __shared__ int sb;
    if (threadIdx.x == 0) {
        int b = -1;
        for (int t = 0; t < n_alpha; ++t)
            if (!isnan(err[t]) && (b < 0 || err[t] < err[b])) b = t;
        sb = b;
        *best_index = b;
    }
    __syncthreads();
    const int b = sb;
    const double alpha = b < 0 ? 0.0 : static_cast<double>(al.v[b]);
    for (int64_t c = threadIdx.x; c < K; c += 256)
        best_scale[c] = b < 0 ? 1.0f : channel_scale(a[c], w[c], alpha);
}

// Yref [Mc][N] fp32 = X [Mc][K] * W [N][K]^T (cuBLAS).  Column-major view:
// Yref^T (N x Mc, ld N) = op T of the K x N matrix W (ld K) times the K x Mc
// matrix X (ld K).
int reference_gemm(const void *W, const void *X, int xt, int64_t Mc, int64_t K, int64_t N,
                   float *Yref, cudaStream_t stream) {
    return blas_gemm_f32("w4_awq_search (reference output)", true, false, static_cast<int>(N),
                         static_cast<int>(Mc), static_cast<int>(K), 1.0f, W, xt,
                         static_cast<int>(K), X, xt, static_cast<int>(K), 0.0f, Yref,
                         static_cast<int>(N), stream);
}

// ---- workspace layout -------------------------------------------------------------------

struct Layout {
    size_t dec, part, a, w, s, packed, scales, zeros, xs, yq, yref, sq, total;
    size_t dec_bytes;
    int64_t nchunk;
};

size_t up256(size_t v) { return (v + 255) & ~size_t(255); }

Layout layout(int64_t Mc, int64_t K, int64_t N, int group) {
    Layout L{};
    const int64_t G = K / group;
    L.dec_bytes = Mc <= 32 ? decode_workspace_bytes(Mc, K, N, group) : 0;
    L.nchunk = ((Mc > N ? Mc : N) + kChunkRows - 1) / kChunkRows;
    size_t o = 0;
    auto take = [&o](size_t bytes) {
        const size_t at = o;
        o = up256(o + bytes);
        return at;
    };
    L.dec = take(L.dec_bytes);
    L.part = take(sizeof(double) * size_t(L.nchunk) * size_t(K));
    L.a = take(sizeof(float) * size_t(K));
    L.w = take(sizeof(float) * size_t(K));
    L.s = take(sizeof(float) * size_t(K));
    L.packed = take(size_t(N) * size_t(K) / 2);
    L.scales = take(sizeof(float) * size_t(N) * size_t(G));
    L.zeros = take(sizeof(float) * size_t(N) * size_t(G));
    L.xs = take(2 * size_t(Mc) * size_t(K));
    L.yq = take(2 * size_t(Mc) * size_t(N));
    L.yref = take(sizeof(float) * size_t(Mc) * size_t(N));
    L.sq = take(sizeof(double) * kSqBlocks);
    L.total = o;
    return L;
}

const char *shape_problem(int64_t Mc, int64_t K, int64_t N, int group) {
    if (Mc <= 0 || K <= 0 || N <= 0) return "need Mc, K, N >= 1";
    if (group != 128) return "group must be 128";
    if (K % group != 0) return "K must be a multiple of group";
    if (Mc >= (int64_t(1) << 31) || K >= (int64_t(1) << 31) || N >= (int64_t(1) << 31))
        return "Mc, K and N must be below 2^31";
    if ((Mc > N ? Mc : N) > int64_t(65535) * kChunkRows) return "Mc and N must be at most 16776960";
    if (Mc > (int64_t(1) << 40) / N || N > (int64_t(1) << 40) / K || Mc > (int64_t(1) << 40) / K)
        return "Mc * N, N * K or Mc * K too large";
    return nullptr;
}

template <int XT>
int search_t(const void *W, const void *X, int64_t Mc, int64_t K, int64_t N, int group, int sym,
             const float *alphas, int n_alpha, double *err, float *best_scale, int *best_index,
             uint8_t *packed_out, float *scales_out, float *zeros_out, unsigned char *ws,
             const Layout &L, cudaStream_t stream) {
    const uint16_t *Wh = static_cast<const uint16_t *>(W);
    const uint16_t *Xh = static_cast<const uint16_t *>(X);
    double *part = reinterpret_cast<double *>(ws + L.part);
    float *a = reinterpret_cast<float *>(ws + L.a);
    float *wm = reinterpret_cast<float *>(ws + L.w);
    float *s = reinterpret_cast<float *>(ws + L.s);
    uint8_t *packed = ws + L.packed;
    float *scales = reinterpret_cast<float *>(ws + L.scales);
    float *zeros = reinterpret_cast<float *>(ws + L.zeros);
    uint16_t *Xs = reinterpret_cast<uint16_t *>(ws + L.xs);
    uint16_t *Yq = reinterpret_cast<uint16_t *>(ws + L.yq);
    float *Yref = reinterpret_cast<float *>(ws + L.yref);
    double *sq = reinterpret_cast<double *>(ws + L.sq);
    cudaError_t e;
    int st;

    if (L.dec_bytes > 0) {
        // the decode path's arrival counters must read zero
        const size_t zeroed = decode_counter_bytes();
        e = cudaMemsetAsync(ws + L.dec, 0, L.dec_bytes < zeroed ? L.dec_bytes : zeroed, stream);
        if (e != cudaSuccess) return cuda_fail("cudaMemsetAsync(decode counters)", e);
    }

    // 1. a_j = mean_i |X_ij|, w_j = mean_n |W_nj|
    const unsigned col_tiles = static_cast<unsigned>((K + kColTile - 1) / kColTile);
    const unsigned kblocks = static_cast<unsigned>((K + 255) / 256);
    const int64_t xchunks = (Mc + kChunkRows - 1) / kChunkRows;
    const int64_t wchunks = (N + kChunkRows - 1) / kChunkRows;
    colabs_partial<XT><<<dim3(col_tiles, static_cast<unsigned>(xchunks)), 256, 0, stream>>>(
        Xh, Mc, K, part);
    colabs_finish<<<kblocks, 256, 0, stream>>>(part, xchunks, K, Mc, a);
    colabs_partial<XT><<<dim3(col_tiles, static_cast<unsigned>(wchunks)), 256, 0, stream>>>(
        Wh, N, K, part);
    colabs_finish<<<kblocks, 256, 0, stream>>>(part, wchunks, K, N, wm);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail("column statistics launch", e);

    // 2. the unquantized layer's output
    if ((st = reference_gemm(W, X, XT, Mc, K, N, Yref, stream)) != W4_OK) return st;

    // 3. one pass per alpha
    const int64_t n8 = Mc * K / 8;
    const int64_t xs_blocks = (n8 + 255) / 256 < 4 * 148 ? (n8 + 255) / 256 : 4 * 148;
    const int64_t E = Mc * N;
    for (int t = 0; t < n_alpha; ++t) {
        awq_scale<<<kblocks, 256, 0, stream>>>(a, wm, K, static_cast<double>(alphas[t]), s);
        if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail("awq_scale launch", e);
        if ((st = launch_quantize(W, XT, K, N, group, sym, s, packed, scales, zeros, stream)) !=
            W4_OK)
            return st;
        scale_activations<XT><<<static_cast<unsigned>(xs_blocks), 256, 0, stream>>>(Xh, s, n8, K,
                                                                                   Xs);
        if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail("scale_activations launch", e);
        if (Mc <= 32)
            st = launch_decode(Xs, XT, Mc, packed, scales, zeros, K, N, Yq, ws + L.dec, L.dec_bytes,
                               stream);
        else
            st = launch_prefill(Xs, XT, Mc, packed, scales, zeros, K, N, Yq, stream);
        if (st != W4_OK) return st;
        sqerr_partial<XT><<<kSqBlocks, 256, 0, stream>>>(Yq, Yref, E, sq);
        sqerr_finish<<<1, 256, 0, stream>>>(sq, err + t);
        if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail("error pass launch", e);
    }

    // 4. the best alpha, its s, and optionally Q(W * s_best)
    AlphaList al{};
    for (int t = 0; t < n_alpha; ++t) al.v[t] = alphas[t];
    awq_select<<<1, 256, 0, stream>>>(err, n_alpha, al, a, wm, K, best_scale, best_index);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail("awq_select launch", e);
    if (packed_out)
        return launch_quantize(W, XT, K, N, group, sym, best_scale, packed_out, scales_out,
                               zeros_out, stream);
    return W4_OK;
}

}  // namespace
}  // namespace w4

extern "C" size_t w4_awq_search_workspace_bytes(int64_t Mc, int64_t K, int64_t N, int group) {
    if (w4::shape_problem(Mc, K, N, group)) return 0;
    return w4::layout(Mc, K, N, group).total;
}

extern "C" int w4_awq_search(const void *W, const void *X, int xt, int64_t Mc, int64_t K,
                             int64_t N, int group, int sym, const float *alphas, int n_alpha,
                             double *err, float *best_scale, int *best_index, uint8_t *packed_out,
                             float *scales_out, float *zeros_out, void *workspace,
                             size_t workspace_bytes, void *stream) {
    const char *fn = "w4_awq_search";
    if (xt != W4_F16 && xt != W4_BF16) return w4::set_error(W4_ERR_INVALID_ARG, fn, "bad dtype");
    if (const char *why = w4::shape_problem(Mc, K, N, group))
        return w4::set_error(group != 128 && group > 0 && K > 0 && K % group == 0
                                 ? W4_ERR_UNSUPPORTED
                                 : W4_ERR_INVALID_ARG,
                             fn, why);
    if (n_alpha < 1 || n_alpha > w4::kMaxAlphas)
        return w4::set_error(W4_ERR_INVALID_ARG, fn, "n_alpha must be 1 .. 64");
    if (!W || !X || !alphas || !err || !best_scale || !best_index)
        return w4::set_error(W4_ERR_INVALID_ARG, fn, "null pointer");
    for (int t = 0; t < n_alpha; ++t)
        if (!(alphas[t] >= 0.0f && alphas[t] <= 1.0f))
            return w4::set_error(W4_ERR_INVALID_ARG, fn, "every alpha must lie in [0, 1]");
    const bool want_q = packed_out || scales_out || zeros_out;
    if (want_q && !(packed_out && scales_out && zeros_out))
        return w4::set_error(W4_ERR_INVALID_ARG, fn,
                             "packed_out, scales_out and zeros_out go together");
    if (!w4::aligned16(W) || !w4::aligned16(X) || !w4::aligned16(best_scale) ||
        (want_q && (!w4::aligned16(packed_out) || !w4::aligned16(scales_out) ||
                    !w4::aligned16(zeros_out))))
        return w4::set_error(W4_ERR_UNSUPPORTED, fn, "pointers must be 16-byte aligned");
    const w4::Layout L = w4::layout(Mc, K, N, group);
    if (!workspace || workspace_bytes < L.total ||
        (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return w4::set_error(W4_ERR_INVALID_ARG, fn,
                             "workspace missing, not 256-byte aligned or smaller than "
                             "w4_awq_search_workspace_bytes");
    unsigned char *ws = static_cast<unsigned char *>(workspace);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (xt == W4_F16)
        return w4::search_t<W4_F16>(W, X, Mc, K, N, group, sym, alphas, n_alpha, err, best_scale,
                                    best_index, packed_out, scales_out, zeros_out, ws, L, s);
    return w4::search_t<W4_BF16>(W, X, Mc, K, N, group, sym, alphas, n_alpha, err, best_scale,
                                 best_index, packed_out, scales_out, zeros_out, ws, L, s);
}
