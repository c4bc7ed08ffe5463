// w4_gptq.cu -- GPTQ: per-group INT4 quantization that pushes each column's
// rounding error onto the columns not yet quantized through the inverse
// Hessian of the layer's calibration activations.
//
// Method: "LLM quantization methods: principles and implementation"
// (zhiyuanblog.org/blog/llm-quantization) §4.1: minimise ||WX - W^X||_F^2,
// H = 2 X X^T, quantize column by column, delta_j = (w_j - q_j) / [H^-1]_jj,
// W[:, j+1:] -= delta_j H^-1[j, j+1:], with a Cholesky factor of H^-1 in
// practice; "PTQ weight quantization: from GPTQ to AWQ", section "GPTQ":
// lazy batch updates every 128 columns.  Here the calibration rows are the
// rows of X [Mc][K], so H = 2 X^T X is [K][K].
//
// One call of w4_gptq, on the caller's stream:
//   1. H = 2 X^T X in fp32 (this library's tiled GEMM, w4_linalg.cu);
//   2. damping: H_jj += percdamp * mean(diag H) (one CTA, fixed-order sum);
//   3. U = upper Cholesky factor of H^-1 (w4_linalg.cu: blocked Cholesky of
//      the index-reversed H and a blocked triangular inverse); the stream is
//      synchronized once here to read the factorization status;
//   4. the column loop (also alone as w4_gptq_quantize, given U):
//      gptq_widen: Wf = fp32 copy of W;
//      per 128-column block b (block = group):
//        gptq_block: four lanes per weight row, each holding 32 of the
//          block's columns: the group's scale / zero point from the row's
//          current weights (the RTN quantizer's formulas), then for
//          each column j in order: code, err_j = (w_j - (u_j - z) s) / U_jj,
//          w_k = fma(-err_j, U_jk, w_k) for the block's k > j; writes the
//          packed codes, scale, zero point and err[n][0..127];
//        gptq_lazy: Wf[:, later k] -= err[:, block] U[block, later k], each
//          element as one fp32 fma chain over the block's 128 columns in
//          order followed by one subtraction (a SIMT tile GEMM whose
//          per-element order is fixed, so the result is reproducible bit for
//          bit; 128 x 128 output tiles, 8 x 8 per thread, operand chunks
//          double-buffered in shared memory).
// Rows are independent given U: every decision of row n depends only on W[n]
// and U, so the parallelism is over rows (block step) and over rows x later
// columns (lazy update).  Outputs use the w4_quantize layout, so w4a16_gemm
// consumes them unchanged.

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "w4_half.cuh"
#include "w4_internal.cuh"

namespace w4 {
namespace {

constexpr int kBlock = 128;  // GPTQ block = quantization group
constexpr int kLT = 128;     // lazy update: output tile rows and columns
constexpr int kLJ = 8;       // lazy update: block columns per shared-memory stage

__global__ void __launch_bounds__(256) gptq_widen(const uint16_t *__restrict__ W, int wt,
                                                  int64_t n8, float *__restrict__ Wf) {
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const uint4 v = __ldg(reinterpret_cast<const uint4 *>(W) + i);
        float f[8];
        if (wt == W4_F16)
            widen8<W4_F16>(v, f);
        else
            widen8<W4_BF16>(v, f);
        reinterpret_cast<float4 *>(Wf)[2 * i] = make_float4(f[0], f[1], f[2], f[3]);
        reinterpret_cast<float4 *>(Wf)[2 * i + 1] = make_float4(f[4], f[5], f[6], f[7]);
    }
}

// Stored code of w under (s, z): sym  u = clamp(rne(w / s), -7, 7) + 8;
// asym u = clamp(rne(fl(w / s) + z), 0, 15); a zero scale gives u = z.
template <int SYM>
__device__ __forceinline__ int code_of(float w, float s, float z) {
    if (s == 0.0f) return static_cast<int>(z);
    if (SYM) return static_cast<int>(fminf(fmaxf(rintf(__fdiv_rn(w, s)), -7.0f), 7.0f)) + 8;
    return static_cast<int>(fminf(fmaxf(rintf(__fadd_rn(__fdiv_rn(w, s), z)), 0.0f), 15.0f));
}

// Shared-memory position of U[b0 + j][b0 + c] in gptq_block: rows of kUPitch
// floats, with 4 floats of padding after every 32 columns so that the four
// lane quarters' 16-byte reads of one row fall in different banks.
constexpr int kUPitch = kBlock + 16;
constexpr int kUSmemBytes = kBlock * kUPitch * 4;  // 73728
__device__ __forceinline__ int upos(int j, int c) { return j * kUPitch + c + 4 * (c / 32); }

// Four lanes per weight row (eight rows per warp): lane quarter q of a row
// holds the block's columns 32q .. 32q+31 in registers.  Each column step is
// computed by the row's four lanes only (a warp advances eight rows per
// instruction), the owner of column j broadcasts w_j within its four lanes,
// and the lanes whose quarter reaches column j update all of it; the U values
// of each step come from the CTA's shared copy of the block.  128 threads (32
// rows) per CTA, so that the CTAs spread evenly over the SMs.
template <int SYM>
__global__ void __launch_bounds__(128) gptq_block(float *__restrict__ Wf, const float *__restrict__ U,
                                                  int64_t N, int64_t K, int64_t b0,
                                                  uint8_t *__restrict__ packed,
                                                  float *__restrict__ scales,
                                                  float *__restrict__ zeros,
                                                  float *__restrict__ Err) {
    // the block's 128 x 128 part of U, staged once per CTA (padded rows, see
    // kUPitch), its strict lower triangle as zeros
    extern __shared__ __align__(16) float ush[];
    {
        const float *ublk = U + b0 * K + b0;  // U[b0 + j][b0 + k] = ublk[j * K + k]
        for (int e = threadIdx.x; e < kBlock * kBlock / 4; e += blockDim.x) {
            const int j = e / (kBlock / 4), c = 4 * (e % (kBlock / 4));
            float4 u = __ldg(reinterpret_cast<const float4 *>(ublk + static_cast<int64_t>(j) * K + c));
            if (c < j) u.x = 0.0f;
            if (c + 1 < j) u.y = 0.0f;
            if (c + 2 < j) u.z = 0.0f;
            if (c + 3 < j) u.w = 0.0f;
            *reinterpret_cast<float4 *>(ush + upos(j, c)) = u;
        }
    }
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int q = lane & 3;
    const int base = lane & ~3;  // first lane of this row's four
    const int64_t n = static_cast<int64_t>(blockIdx.x) * (blockDim.x / 4) + (threadIdx.x >> 2);
    const bool active = n < N;  // inactive rows still take part in the shuffles
    const int64_t G = K / kBlock;
    float w[32];
    {
        const float4 *src = reinterpret_cast<const float4 *>(Wf + (active ? n : 0) * K + b0 + 32 * q);
#pragma unroll
        for (int v = 0; v < 8; ++v) {
            const float4 f = active ? src[v] : make_float4(0.f, 0.f, 0.f, 0.f);
            w[4 * v] = f.x; w[4 * v + 1] = f.y; w[4 * v + 2] = f.z; w[4 * v + 3] = f.w;
        }
    }

    // the group's parameters from the current weights (exact min / max)
    float s, z;
    if (SYM) {
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(w[i]));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
        s = __fdiv_rn(amax, 7.0f);
        z = 8.0f;
    } else {
        float mn = w[0], mx = w[0];
#pragma unroll
        for (int i = 1; i < 32; ++i) {
            mn = fminf(mn, w[i]);
            mx = fmaxf(mx, w[i]);
        }
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, 1));
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, 2));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        s = __fdiv_rn(__fsub_rn(mx, mn), 15.0f);
        z = s == 0.0f ? 0.0f
                      : __fadd_rn(fminf(fmaxf(rintf(__fdiv_rn(-mn, s)), 0.0f), 15.0f), 0.0f);
    }

    // nibble of k % 8 inside its 32-bit word: k % 8 = {0,2,4,6,1,3,5,7}[nibble]
    constexpr int kNibble[8] = {0, 4, 1, 5, 2, 6, 3, 7};
    uint32_t word[4] = {0u, 0u, 0u, 0u};
    float my_err[32];
#pragma unroll 1
    for (int owner = 0; owner < 4; ++owner) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const int j = 32 * owner + i;
            const float wj = __shfl_sync(0xffffffffu, w[i], base | owner);
            const int c = code_of<SYM>(wj, s, z);
            const float deq = __fmul_rn(__fsub_rn(static_cast<float>(c), z), s);
            const float e = __fdiv_rn(__fsub_rn(wj, deq), ush[upos(j, j)]);
            if (q == owner) {
                word[i / 8] |= static_cast<uint32_t>(c) << (4 * kNibble[i % 8]);
                my_err[i] = e;
            }
            // this lane's columns k = 32q + i2 >= j (q >= owner), all of them:
            // the staged U[j][k] is 0 for k < j, and w[j] itself is no
            // longer read, so the columns after j get exactly their update
            // and no predicate is needed
            if (q >= owner) {
                const float4 *urow = reinterpret_cast<const float4 *>(ush + upos(j, 32 * q));
#pragma unroll
                for (int v = 0; v < 8; ++v) {
                    const float4 u4 = urow[v];
                    w[4 * v] = __fmaf_rn(-e, u4.x, w[4 * v]);
                    w[4 * v + 1] = __fmaf_rn(-e, u4.y, w[4 * v + 1]);
                    w[4 * v + 2] = __fmaf_rn(-e, u4.z, w[4 * v + 2]);
                    w[4 * v + 3] = __fmaf_rn(-e, u4.w, w[4 * v + 3]);
                }
            }
        }
    }
    if (!active) return;
    reinterpret_cast<uint4 *>(packed + n * (K / 2) + b0 / 2)[q] =
        make_uint4(word[0], word[1], word[2], word[3]);
    float4 *edst = reinterpret_cast<float4 *>(Err + n * kBlock + 32 * q);
#pragma unroll
    for (int v = 0; v < 8; ++v)
        edst[v] = make_float4(my_err[4 * v], my_err[4 * v + 1], my_err[4 * v + 2], my_err[4 * v + 3]);
    if (q == 0) {
        scales[n * G + b0 / kBlock] = s;
        zeros[n * G + b0 / kBlock] = z;
    }
}

// Wf[n][k] -= sum_{j < 128} Err[n][j] * U[b0 + j][k] for k >= b0 + 128: per
// element acc = fma(Err[n][j], U[b0+j][k], acc) for j = 0, 1, ..., 127 from
// acc = 0, then Wf = Wf - acc.  Tile 128 rows x 128 columns, 256 threads,
// thread (ty, tx) owns rows {4ty..4ty+3, 64+4ty..64+4ty+3} and the same
// pattern of columns.  The block's 128 columns go through shared memory in
// chunks of kLJ, double-buffered: the next chunk is loaded into registers
// while the current one is multiplied.
__global__ void __launch_bounds__(256, 2) gptq_lazy(float *__restrict__ Wf, const float *__restrict__ Err,
                                                    const float *__restrict__ U, int64_t N, int64_t K,
                                                    int64_t b0) {
    __shared__ __align__(16) float Es[2][kLJ][kLT];
    __shared__ __align__(16) float Us[2][kLJ][kLT];
    const int t = threadIdx.x, tx = t & 15, ty = t >> 4;
    const int64_t n0 = static_cast<int64_t>(blockIdx.y) * kLT;
    const int64_t k0 = b0 + kBlock + static_cast<int64_t>(blockIdx.x) * kLT;
    // this thread's share of a chunk: Err row er, block columns eh..eh+3 (a
    // warp stores 32 consecutive rows: no bank conflicts); U row uj, columns
    // uc..uc+3
    const int er = t & (kLT - 1), eh = (t >> 7) * 4, uj = t >> 5, uc = (t & 31) * 4;
    const bool erow_ok = n0 + er < N;
    const float4 *esrc = reinterpret_cast<const float4 *>(Err + (n0 + er) * kBlock + eh);
    const float4 *usrc = reinterpret_cast<const float4 *>(U + (b0 + uj) * K + k0 + uc);
    float4 e0, u0;
    auto fetch = [&](int j0) {
        e0 = erow_ok ? esrc[j0 / 4] : make_float4(0.f, 0.f, 0.f, 0.f);
        u0 = usrc[static_cast<int64_t>(j0) * (K / 4)];
    };
    auto stash = [&](int buf) {
        Es[buf][eh + 0][er] = e0.x;
        Es[buf][eh + 1][er] = e0.y;
        Es[buf][eh + 2][er] = e0.z;
        Es[buf][eh + 3][er] = e0.w;
        *reinterpret_cast<float4 *>(&Us[buf][uj][uc]) = u0;
    };
    float acc[8][8];
#pragma unroll
    for (int r = 0; r < 8; ++r)
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[r][c] = 0.0f;

    fetch(0);
    stash(0);
    __syncthreads();
#pragma unroll 1
    for (int ch = 0; ch < kBlock / kLJ; ++ch) {
        const int buf = ch & 1;
        if (ch + 1 < kBlock / kLJ) fetch((ch + 1) * kLJ);
#pragma unroll
        for (int jj = 0; jj < kLJ; ++jj) {
            const float4 a0 = *reinterpret_cast<const float4 *>(&Es[buf][jj][4 * ty]);
            const float4 a1 = *reinterpret_cast<const float4 *>(&Es[buf][jj][64 + 4 * ty]);
            const float4 q0 = *reinterpret_cast<const float4 *>(&Us[buf][jj][4 * tx]);
            const float4 q1 = *reinterpret_cast<const float4 *>(&Us[buf][jj][64 + 4 * tx]);
            const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            const float b[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
#pragma unroll
            for (int r = 0; r < 8; ++r)
#pragma unroll
                for (int c = 0; c < 8; ++c) acc[r][c] = __fmaf_rn(a[r], b[c], acc[r][c]);
        }
        if (ch + 1 < kBlock / kLJ) stash(buf ^ 1);
        __syncthreads();
    }
    // Wf -= acc, two rows at a time: their four reads are issued before the
    // stores (a store to Wf could alias a later read)
#pragma unroll
    for (int rr = 0; rr < 8; rr += 2) {
        float4 v[2][2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int r = rr + u;
            const int64_t n = n0 + (r < 4 ? 4 * ty + r : 64 + 4 * ty + (r - 4));
#pragma unroll
            for (int h = 0; h < 2; ++h)
                v[u][h] = n < N ? *reinterpret_cast<const float4 *>(Wf + n * K + k0 + 64 * h + 4 * tx)
                                : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int r = rr + u;
            const int64_t n = n0 + (r < 4 ? 4 * ty + r : 64 + 4 * ty + (r - 4));
            if (n >= N) continue;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                float4 w = v[u][h];
                w.x = __fsub_rn(w.x, acc[r][4 * h + 0]);
                w.y = __fsub_rn(w.y, acc[r][4 * h + 1]);
                w.z = __fsub_rn(w.z, acc[r][4 * h + 2]);
                w.w = __fsub_rn(w.w, acc[r][4 * h + 3]);
                *reinterpret_cast<float4 *>(Wf + n * K + k0 + 64 * h + 4 * tx) = w;
            }
        }
    }
}

// H[j][j] += percdamp * mean(diag H); one CTA of 1024 threads, fixed-order sum.
__global__ void __launch_bounds__(1024) gptq_damp(float *__restrict__ H, int64_t K, float percdamp) {
    __shared__ double red[32];
    double v = 0.0;
    for (int64_t j = threadIdx.x; j < K; j += 1024) v += static_cast<double>(H[j * K + j]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    __shared__ float lam;
    if (threadIdx.x == 0) {
        double s = 0.0;
        for (int q = 0; q < 32; ++q) s += red[q];
        lam = __fmul_rn(percdamp, __double2float_rn(s / static_cast<double>(K)));
    }
    __syncthreads();
    for (int64_t j = threadIdx.x; j < K; j += 1024) H[j * K + j] = __fadd_rn(H[j * K + j], lam);
}

size_t up256(size_t v) { return (v + 255) & ~size_t(255); }

struct LoopLayout {
    size_t wf, err, total;
};

LoopLayout loop_layout(int64_t K, int64_t N, size_t at) {
    LoopLayout L;
    L.wf = at;
    L.err = up256(L.wf + sizeof(float) * size_t(N) * size_t(K));
    L.total = up256(L.err + sizeof(float) * size_t(N) * kBlock);
    return L;
}

int column_loop(const void *W, int wt, int64_t K, int64_t N, int sym, const float *U,
                uint8_t *packed, float *scales, float *zeros, unsigned char *ws,
                const LoopLayout &L, cudaStream_t stream) {
    DeviceInfo di;
    int st = device_info(&di);
    if (st != W4_OK) return st;
    float *Wf = reinterpret_cast<float *>(ws + L.wf);
    float *Err = reinterpret_cast<float *>(ws + L.err);
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return set_error(W4_ERR_CUDA, "cudaGetDevice", nullptr);
    static bool attr_done[64] = {};
    if (!attr_done[dev]) {
        cudaError_t e = cudaFuncSetAttribute(gptq_block<0>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kUSmemBytes);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(gptq_block<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     kUSmemBytes);
        if (e != cudaSuccess) return cuda_fail("cudaFuncSetAttribute(gptq_block smem)", e);
        attr_done[dev] = true;
    }
    const int64_t n8 = N * K / 8;
    const int64_t want = (n8 + 255) / 256, cap = int64_t(8) * di.sm_count;
    gptq_widen<<<static_cast<unsigned>(want < cap ? want : cap), 256, 0, stream>>>(
        static_cast<const uint16_t *>(W), wt, n8, Wf);
    const unsigned row_ctas = static_cast<unsigned>((N + 31) / 32);  // 32 rows per CTA
    const unsigned tile_rows = static_cast<unsigned>((N + kLT - 1) / kLT);
    for (int64_t b0 = 0; b0 < K; b0 += kBlock) {
        if (sym)
            gptq_block<1><<<row_ctas, 128, kUSmemBytes, stream>>>(Wf, U, N, K, b0, packed, scales,
                                                                 zeros, Err);
        else
            gptq_block<0><<<row_ctas, 128, kUSmemBytes, stream>>>(Wf, U, N, K, b0, packed, scales,
                                                                 zeros, Err);
        const int64_t rest = K - b0 - kBlock;
        if (rest > 0)
            gptq_lazy<<<dim3(static_cast<unsigned>(rest / kLT), tile_rows), 256, 0, stream>>>(
                Wf, Err, U, N, K, b0);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail("GPTQ column loop launch", e);
    }
    return W4_OK;
}

const char *shape_problem(int64_t K, int64_t N, int group) {
    if (K <= 0 || N <= 0) return "need K, N >= 1";
    if (group != kBlock) return "group must be 128";
    if (K % kBlock != 0) return "K must be a multiple of 128";
    if (K > 65536) return "K must be at most 65536";
    if (N > int64_t(65535) * kLT) return "N must be at most 8388480";  // lazy-update grid rows
    if (N > (int64_t(1) << 40) / K) return "N * K too large";
    return nullptr;
}

struct FullLayout {
    size_t h, scratch, info, loop_at, total;
    LoopLayout loop;
};

FullLayout full_layout(int64_t K, int64_t N) {
    FullLayout F;
    F.h = 0;
    F.scratch = up256(sizeof(float) * size_t(K) * size_t(K));
    F.info = up256(F.scratch + sizeof(float) * linalg_scratch_floats(K));
    F.loop_at = up256(F.info + 256);
    F.loop = loop_layout(K, N, F.loop_at);
    F.total = F.loop.total;
    return F;
}

}  // namespace
}  // namespace w4

using w4::set_error;

extern "C" size_t w4_gptq_quantize_workspace_bytes(int64_t K, int64_t N, int group) {
    if (w4::shape_problem(K, N, group)) return 0;
    return w4::loop_layout(K, N, 0).total;
}

extern "C" int w4_gptq_quantize(const void *W, int wt, int64_t K, int64_t N, int group, int sym,
                                const float *U, uint8_t *packed, float *scales, float *zeros,
                                void *workspace, size_t workspace_bytes, void *stream) {
    const char *fn = "w4_gptq_quantize";
    if (wt != W4_F16 && wt != W4_BF16) return set_error(W4_ERR_INVALID_ARG, fn, "bad dtype");
    if (const char *why = w4::shape_problem(K, N, group))
        return set_error(group != 128 && group > 0 ? W4_ERR_UNSUPPORTED : W4_ERR_INVALID_ARG, fn, why);
    if (!W || !U || !packed || !scales || !zeros || !workspace)
        return set_error(W4_ERR_INVALID_ARG, fn, "null pointer");
    const w4::LoopLayout L = w4::loop_layout(K, N, 0);
    if (workspace_bytes < L.total || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return set_error(W4_ERR_INVALID_ARG, fn,
                         "workspace not 256-byte aligned or smaller than "
                         "w4_gptq_quantize_workspace_bytes");
    if (!w4::aligned16(W) || !w4::aligned16(U) || !w4::aligned16(packed) ||
        !w4::aligned16(scales) || !w4::aligned16(zeros))
        return set_error(W4_ERR_UNSUPPORTED, fn, "pointers must be 16-byte aligned");
    return w4::column_loop(W, wt, K, N, sym, U, packed, scales, zeros,
                           static_cast<unsigned char *>(workspace), L,
                           static_cast<cudaStream_t>(stream));
}

extern "C" size_t w4_gptq_workspace_bytes(int64_t Mc, int64_t K, int64_t N, int group) {
    if (Mc <= 0 || Mc >= (int64_t(1) << 31) || w4::shape_problem(K, N, group)) return 0;
    return w4::full_layout(K, N).total;
}

extern "C" int w4_gptq(const void *W, const void *X, int xt, int64_t Mc, int64_t K, int64_t N,
                       int group, int sym, float percdamp, uint8_t *packed, float *scales,
                       float *zeros, float *U_out, void *workspace, size_t workspace_bytes,
                       void *stream) {
    const char *fn = "w4_gptq";
    if (xt != W4_F16 && xt != W4_BF16) return set_error(W4_ERR_INVALID_ARG, fn, "bad dtype");
    if (const char *why = w4::shape_problem(K, N, group))
        return set_error(group != 128 && group > 0 ? W4_ERR_UNSUPPORTED : W4_ERR_INVALID_ARG, fn, why);
    if (Mc <= 0 || Mc >= (int64_t(1) << 31)) return set_error(W4_ERR_INVALID_ARG, fn, "need 1 <= Mc < 2^31");
    if (!(percdamp >= 0.0f && percdamp <= 1.0f))
        return set_error(W4_ERR_INVALID_ARG, fn, "percdamp must lie in [0, 1]");
    if (!W || !X || !packed || !scales || !zeros || !workspace)
        return set_error(W4_ERR_INVALID_ARG, fn, "null pointer");
    const w4::FullLayout F = w4::full_layout(K, N);
    if (workspace_bytes < F.total || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return set_error(W4_ERR_INVALID_ARG, fn,
                         "workspace not 256-byte aligned or smaller than w4_gptq_workspace_bytes");
    if (!w4::aligned16(W) || !w4::aligned16(X) || !w4::aligned16(packed) ||
        !w4::aligned16(scales) || !w4::aligned16(zeros) || (U_out && !w4::aligned16(U_out)))
        return set_error(W4_ERR_UNSUPPORTED, fn, "pointers must be 16-byte aligned");
    unsigned char *ws = static_cast<unsigned char *>(workspace);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    float *H = reinterpret_cast<float *>(ws + F.h);
    // 1. H = 2 X^T X (fp32 accumulation; the tiles on and above the diagonal)
    int st = w4::hessian(X, xt, Mc, K, H, s);
    if (st != W4_OK) return st;
    // 2. damping
    w4::gptq_damp<<<1, 1024, 0, s>>>(H, K, percdamp);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return w4::cuda_fail("gptq_damp launch", e);
    // 3. U, the upper Cholesky factor of H^-1 (in place)
    st = w4::inverse_factor(fn, H, K, reinterpret_cast<float *>(ws + F.scratch),
                            reinterpret_cast<int *>(ws + F.info), s);
    if (st != W4_OK) return st;
    if (U_out) {
        e = cudaMemcpyAsync(U_out, H, sizeof(float) * size_t(K) * size_t(K), cudaMemcpyDeviceToDevice, s);
        if (e != cudaSuccess) return w4::cuda_fail("copy of U", e);
    }
    // 4. the column loop
    return w4::column_loop(W, xt, K, N, sym, H, packed, scales, zeros, ws, F.loop, s);
}
