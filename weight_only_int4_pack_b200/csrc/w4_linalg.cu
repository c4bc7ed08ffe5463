// w4_linalg.cu -- the dense linear algebra of GPTQ on the device: the Hessian
// H = 2 X^T X and the upper Cholesky factor U of the inverse of the damped
// Hessian (U^T U = H^-1), the two steps that "LLM quantization methods:
// principles and implementation" (zhiyuanblog.org/blog/llm-quantization)
// §4.1 and "PTQ weight quantization: from GPTQ to AWQ" (section "GPTQ")
// put in front of the column loop ("Hessian inverse, in practice through a
// Cholesky factorization").
//
// Everything is fp32 on the CUDA cores:
//   * gemm_kernel: a 128 x 128-tiled fp32 GEMM (k steps of 16),
//     C = alpha * sum_k A(m,k) B(n,k)
//     + beta * C, with 16-bit or fp32 operands read in either orientation
//     (widened exactly to fp32), options to compute only the tiles on or
//     above / on or below the diagonal, k-ranges cut to the nonzero part of a
//     triangular operand, and batching over blockIdx.z.  Each thread owns an
//     8 x 8 block of C and sums over k in increasing order with fmaf, so a
//     result is a fixed function of the inputs (run to run identical).
//   * U without forming H^-1: with P the index reversal, P H P = L L^T
//     (lower Cholesky), so H = R R^T with R = P L P upper triangular and
//     H^-1 = R^-T R^-1; U = R^-1 = P L^-1 P is upper triangular with a
//     positive diagonal, hence the Cholesky factor of H^-1.  L comes from a
//     right-looking blocked Cholesky (each 64 x 64 diagonal block factored and
//     inverted together in registers, four columns at a time, fused with the
//     panel L21 = A21 T^T that it feeds, T the inverse of the diagonal block;
//     trailing update with the GEMM), L^-1 from recursive doubling
//     [A 0; B C]^-1 = [A^-1 0; -C^-1 B A^-1, C^-1] starting from the inverted
//     diagonal blocks.
//   * A pivot that is not positive (or not finite) sets an info word that the
//     host reads after the factorization (the damped Hessian is then not
//     positive definite).

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "w4_internal.cuh"

namespace w4 {
namespace {

constexpr int kBM = 128, kBN = 128, kBK = 16;
constexpr int kNB = 64;  // Cholesky block

enum Tri { kAll = 0, kUpper = 1, kLower = 2 };

struct GemmArgs {
    const void *A;
    const void *B;
    float *C;
    int64_t lda, ldb, ldc;
    int64_t sA, sB, sC;  // batch strides (elements)
    int M, N, K;
    float alpha, beta;
    int tri;          // kAll, kUpper (tiles with n0 + BN > m0), kLower (tiles with n0 < m0 + BM)
    int k_from_n;     // B(n, k) = 0 for k < n: start k at the tile's n0
    int k_to_m;       // A(m, k) = 0 for k > m: end k at the tile's m0 + BM
    int pair;         // 0, or 1 / 2: each CTA takes two mirrored tiles along n / m
};

// Four consecutive elements widened exactly to fp32.
template <typename T>
__device__ __forceinline__ float4 load4(const T *p);
template <>
__device__ __forceinline__ float4 load4<float>(const float *p) {
    return *reinterpret_cast<const float4 *>(p);
}
template <>
__device__ __forceinline__ float4 load4<__half>(const __half *p) {
    const uint2 u = *reinterpret_cast<const uint2 *>(p);
    const float2 a = __half22float2(*reinterpret_cast<const __half2 *>(&u.x));
    const float2 b = __half22float2(*reinterpret_cast<const __half2 *>(&u.y));
    return make_float4(a.x, a.y, b.x, b.y);
}
template <>
__device__ __forceinline__ float4 load4<__nv_bfloat16>(const __nv_bfloat16 *p) {
    const uint2 u = *reinterpret_cast<const uint2 *>(p);
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.y));
    return make_float4(a.x, a.y, b.x, b.y);
}

// One 128 (rows r) x 16 (k) operand tile, fetched as 512 groups of four
// consecutive elements (two per thread) and stored k-major (S[k][r]).
// RC: element (r, k) at p[k * ld + r] (r contiguous; a warp reads 512
// consecutive bytes of one k row); else at p[r * ld + k] (k contiguous; a
// warp reads 16 bytes of 32 consecutive rows and stores 32 consecutive r,
// so the transposing stores are bank-conflict free).
template <typename T, bool RC>
struct Tile {
    float4 v[2];
    __device__ __forceinline__ void load(const T *p, int64_t ld, int r0, int R, int k0, int khi, int t) {
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            const int idx = t + 256 * q;
            int r, k;
            if (RC) { k = idx >> 5; r = 4 * (idx & 31); } else { r = idx & 127; k = 4 * (idx >> 7); }
            const bool ok = r0 + r < R && k0 + k < khi;
            v[q] = ok ? load4<T>(p + (RC ? static_cast<int64_t>(k0 + k) * ld + r0 + r
                                         : static_cast<int64_t>(r0 + r) * ld + k0 + k))
                      : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
    __device__ __forceinline__ void store(float (*S)[kBM], int t) const {
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            const int idx = t + 256 * q;
            if (RC) {
                *reinterpret_cast<float4 *>(&S[idx >> 5][4 * (idx & 31)]) = v[q];
            } else {
                const int r = idx & 127, k = 4 * (idx >> 7);
                S[k][r] = v[q].x;
                S[k + 1][r] = v[q].y;
                S[k + 2][r] = v[q].z;
                S[k + 3][r] = v[q].w;
            }
        }
    }
};

// C[m][n] = alpha * sum_k A(m, k) B(n, k) + beta * C[m][n] (beta == 0: C not read).
// A(m, k) = A[m * lda + k] if !AMC, A[k * lda + m] if AMC (m contiguous);
// B(n, k) = B[n * ldb + k] if !BNC, B[k * ldb + n] if BNC (n contiguous).
// 128 x 128 tile per CTA, 256 threads (two CTAs per SM when both operands
// are k-contiguous, one otherwise: the register need), 8 x 8 outputs per
// thread (rows 4 ty + {0..3} and 64 + 4 ty + {0..3}, the same for columns
// with tx, so the float4 reads of a quarter warp are bank-conflict free), k in
// steps of 16 through two shared-memory buffers (the next step's operands are
// fetched into registers while the current one is used).  The host checks
// the alignment the four-element fetches need.
template <typename TA, typename TB, bool AMC, bool BNC>
__device__ __forceinline__ void gemm_tile(const GemmArgs &g, int m0, int n0, float (*As)[kBK][kBM],
                                          float (*Bs)[kBK][kBN]) {
    const TA *A = static_cast<const TA *>(g.A) + blockIdx.z * g.sA;
    const TB *B = static_cast<const TB *>(g.B) + blockIdx.z * g.sB;
    float *C = g.C + blockIdx.z * g.sC;
    const int tid = threadIdx.x;
    const int tx = tid & 15, ty = tid >> 4;
    int k_lo = 0, k_hi = g.K;
    if (g.k_from_n) k_lo = n0;
    if (g.k_to_m) k_hi = min(g.K, m0 + kBM);
    Tile<TA, AMC> ta;
    Tile<TB, BNC> tb;
    float acc[8][8] = {};
    if (k_lo < k_hi) {
        ta.load(A, g.lda, m0, g.M, k_lo, k_hi, tid);
        tb.load(B, g.ldb, n0, g.N, k_lo, k_hi, tid);
        ta.store(As[0], tid);
        tb.store(Bs[0], tid);
        __syncthreads();
        int buf = 0;
        for (int k0 = k_lo; k0 < k_hi; k0 += kBK) {
            const bool more = k0 + kBK < k_hi;
            if (more) {
                ta.load(A, g.lda, m0, g.M, k0 + kBK, k_hi, tid);
                tb.load(B, g.ldb, n0, g.N, k0 + kBK, k_hi, tid);
            }
#pragma unroll
            for (int kk = 0; kk < kBK; ++kk) {
                const float4 a0 = *reinterpret_cast<const float4 *>(&As[buf][kk][4 * ty]);
                const float4 a1 = *reinterpret_cast<const float4 *>(&As[buf][kk][64 + 4 * ty]);
                const float4 b0 = *reinterpret_cast<const float4 *>(&Bs[buf][kk][4 * tx]);
                const float4 b1 = *reinterpret_cast<const float4 *>(&Bs[buf][kk][64 + 4 * tx]);
                const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
                const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
                for (int i = 0; i < 8; ++i)
#pragma unroll
                    for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
            }
            if (more) {
                ta.store(As[buf ^ 1], tid);
                tb.store(Bs[buf ^ 1], tid);
                __syncthreads();
                buf ^= 1;
            }
        }
    }
    // epilogue in four quarters of two rows: the four C reads of a quarter
    // are issued before its stores (stores to C could alias later reads)
#pragma unroll
    for (int qr = 0; qr < 4; ++qr) {
        const int half = qr >> 1;
        float4 o[2][2];
        if (g.beta != 0.f) {
#pragma unroll
            for (int ii = 0; ii < 2; ++ii) {
                const int m = m0 + 64 * half + 4 * ty + 2 * (qr & 1) + ii;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int n = n0 + 4 * tx + 64 * h;
                    o[ii][h] = m < g.M && n < g.N
                                   ? *reinterpret_cast<const float4 *>(C + static_cast<int64_t>(m) * g.ldc + n)
                                   : make_float4(0.f, 0.f, 0.f, 0.f);
                }
            }
        }
#pragma unroll
        for (int ii = 0; ii < 2; ++ii) {
            const int i = 4 * half + 2 * (qr & 1) + ii;
            const int m = m0 + 64 * half + 4 * ty + 2 * (qr & 1) + ii;
            if (m >= g.M) continue;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int n = n0 + 4 * tx + 64 * h;
                if (n >= g.N) continue;
                float4 v = make_float4(g.alpha * acc[i][4 * h], g.alpha * acc[i][4 * h + 1],
                                       g.alpha * acc[i][4 * h + 2], g.alpha * acc[i][4 * h + 3]);
                if (g.beta != 0.f)
                    v = make_float4(fmaf(g.alpha, acc[i][4 * h], g.beta * o[ii][h].x),
                                    fmaf(g.alpha, acc[i][4 * h + 1], g.beta * o[ii][h].y),
                                    fmaf(g.alpha, acc[i][4 * h + 2], g.beta * o[ii][h].z),
                                    fmaf(g.alpha, acc[i][4 * h + 3], g.beta * o[ii][h].w));
                *reinterpret_cast<float4 *>(C + static_cast<int64_t>(m) * g.ldc + n) = v;
            }
        }
    }
}

// One output tile per CTA, or with g.pair two: tile i and its mirror
// (count - 1 - i) along n (pair == 1) or m (pair == 2), so that a CTA's
// k range adds up to the same length for every CTA of a triangular operand.
template <typename TA, typename TB, bool AMC, bool BNC>
__global__ void __launch_bounds__(256, (!AMC && !BNC) ? 2 : 1) gemm_kernel(GemmArgs g) {
    __shared__ __align__(16) float As[2][kBK][kBM];
    __shared__ __align__(16) float Bs[2][kBK][kBN];
    const int nt = (g.N + kBN - 1) / kBN, mt = (g.M + kBM - 1) / kBM;
    const int cnt = g.pair == 0 ? 1 : 2;
#pragma unroll 1
    for (int w = 0; w < cnt; ++w) {
        int bx = blockIdx.x, by = blockIdx.y;
        if (w == 1) {
            if (g.pair == 1) {
                bx = nt - 1 - bx;
                if (bx <= static_cast<int>(blockIdx.x)) break;
            } else {
                by = mt - 1 - by;
                if (by <= static_cast<int>(blockIdx.y)) break;
            }
            __syncthreads();  // the first tile's last reads of As / Bs
        }
        const int m0 = by * kBM, n0 = bx * kBN;
        if (g.tri == kUpper && n0 + kBN <= m0) continue;
        if (g.tri == kLower && n0 >= m0 + kBM) continue;
        gemm_tile<TA, TB, AMC, BNC>(g, m0, n0, As, Bs);
    }
}

template <typename TA, typename TB, bool AMC, bool BNC>
int gemm(const GemmArgs &g, int batch, cudaStream_t s) {
    // four-element fetches and stores: 16-byte aligned rows of whole groups
    auto al = [](const void *p, size_t bytes) { return reinterpret_cast<uintptr_t>(p) % bytes == 0; };
    const bool ok = g.lda % 4 == 0 && g.ldb % 4 == 0 && g.ldc % 4 == 0 && g.sA % 4 == 0 &&
                    g.sB % 4 == 0 && g.sC % 4 == 0 && al(g.A, 4 * sizeof(TA)) &&
                    al(g.B, 4 * sizeof(TB)) && al(g.C, 16) && g.N % 4 == 0 &&
                    (AMC ? g.M % 4 == 0 : g.K % 4 == 0) && (BNC || g.K % 4 == 0);
    if (!ok) return set_error(W4_ERR_UNSUPPORTED, "gemm_kernel", "operand alignment");
    unsigned gx = static_cast<unsigned>((g.N + kBN - 1) / kBN), gy = static_cast<unsigned>((g.M + kBM - 1) / kBM);
    if (g.pair == 1) gx = (gx + 1) / 2;
    if (g.pair == 2) gy = (gy + 1) / 2;
    const dim3 grid(gx, gy, static_cast<unsigned>(batch));
    gemm_kernel<TA, TB, AMC, BNC><<<grid, 256, 0, s>>>(g);
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? W4_OK : cuda_fail("gemm_kernel launch", e);
}

GemmArgs gargs(const void *A, int64_t lda, const void *B, int64_t ldb, float *C, int64_t ldc,
               int M, int N, int K, float alpha, float beta) {
    GemmArgs g = {};
    g.A = A;
    g.B = B;
    g.C = C;
    g.lda = lda;
    g.ldb = ldb;
    g.ldc = ldc;
    g.M = M;
    g.N = N;
    g.K = K;
    g.alpha = alpha;
    g.beta = beta;
    return g;
}

// One step of the blocked Cholesky: factors the 64 x 64 diagonal block D at
// (k0, k0) of the row-major n x n matrix P (only its lower part is read),
// forms T = L_D^-1, and overwrites the panel below it, P[i][k0 .. k0+64) for
// i >= k0 + 64, with L[i][..] = P[i][..] T^T.  Grid: one CTA per 128 panel
// rows (at least one); 256 threads.  Every CTA factors D itself (the factored
// block is not stored: later steps read only T and the panels); CTA 0 writes
// T to Tb and the status.
//
// The block is factored right-looking four columns at a time.  Thread (c, h)
// holds rows 16h .. 16h+15 of column c of D and entries 16h .. 16h+15 of row
// c of the running right-hand side R (R = I at the start; row c of T once
// final).  For columns j .. j+3:
//   1. their owners publish those four columns of D and rows of R;
//   2. every thread factors the 4 x 4 pivot block itself (reciprocal square
//      roots from the hardware, a few ulp) and inverts it, forms row c of the
//      four columns of L by forward substitution, and one entry of rows
//      j .. j+3 of T (the inverse pivot block times the published rows of R;
//      final from then on);
//   3. D[r][c] -= sum_q L[r][j+q] L[c][j+q] and R[c][k] -= sum_q L[c][j+q] T[j+q][k]
//      for the later columns c, each in the order q = 0 .. 3 (a warp skips the
//      rows above the pivot and the entries right of it, which stay as they
//      are); the owners of rows j .. j+3 take them from T.
// A pivot that is not positive or not finite sets *info (first bad pivot + 1).
__global__ void __launch_bounds__(256) chol_panel(float *__restrict__ P, int64_t n, int k0,
                                                  float *__restrict__ Tb, int *info) {
    __shared__ __align__(16) float PC[4][kNB];    // published columns of D
    __shared__ __align__(16) float PR[4][kNB];    // published rows of R
    __shared__ __align__(16) float LT[kNB][kNB];  // LT[j][r] = L[r][j] (0 for r < j)
    __shared__ __align__(16) float TR[kNB][kNB];  // TR[j][k] = T[j][k] (0 for k > j)
    __shared__ int bad;
    const int c = threadIdx.x & (kNB - 1), h = threadIdx.x >> 6, r0 = 16 * h;
    float a[16], t[16];
    {
        const float *col = P + static_cast<int64_t>(k0 + r0) * n + k0 + c;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            a[i] = r0 + i >= c ? col[i * n] : 0.f;
            t[i] = r0 + i == c ? 1.f : 0.f;
        }
    }
    if (threadIdx.x == 0) bad = 0;
#pragma unroll 1
    for (int j = 0; j < kNB; j += 4) {
        const int q = c - j;  // 0 .. 3: one of this step's columns
        const bool own = q >= 0 && q < 4;
        if (own) {
#pragma unroll
            for (int i = 0; i < 16; i += 4) {
                *reinterpret_cast<float4 *>(&PC[q][r0 + i]) = make_float4(a[i], a[i + 1], a[i + 2], a[i + 3]);
                *reinterpret_cast<float4 *>(&PR[q][r0 + i]) = make_float4(t[i], t[i + 1], t[i + 2], t[i + 3]);
            }
        }
        __syncthreads();
        // pivot block p_xy = D[j+x][j+y] (y <= x), factored: L4 with 1 / diagonal i0..i3
        int badq = -1;
        auto rs = [&](float d, int qq) {
            const bool ok = d > 0.f && d <= 3.4e38f;
            if (!ok && badq < 0) badq = qq;
            return ok ? rsqrtf(d) : 1.f;
        };
        const float p00 = PC[0][j], p10 = PC[0][j + 1], p20 = PC[0][j + 2], p30 = PC[0][j + 3];
        const float p11 = PC[1][j + 1], p21 = PC[1][j + 2], p31 = PC[1][j + 3];
        const float p22 = PC[2][j + 2], p32 = PC[2][j + 3], p33 = PC[3][j + 3];
        const float v0 = PC[0][c], v1 = PC[1][c], v2 = PC[2][c], v3 = PC[3][c];
        const float x0 = PR[0][c], x1 = PR[1][c], x2 = PR[2][c], x3 = PR[3][c];
        const float i0 = rs(p00, 0);
        const float L10 = p10 * i0, L20 = p20 * i0, L30 = p30 * i0;
        const float d1 = fmaf(-L10, L10, p11);
        const float i1 = rs(d1, 1);
        const float L21 = fmaf(-L20, L10, p21) * i1, L31 = fmaf(-L30, L10, p31) * i1;
        const float d2 = fmaf(-L21, L21, fmaf(-L20, L20, p22));
        const float i2 = rs(d2, 2);
        const float L32 = fmaf(-L31, L21, fmaf(-L30, L20, p32)) * i2;
        const float d3 = fmaf(-L32, L32, fmaf(-L31, L31, fmaf(-L30, L30, p33)));
        const float i3 = rs(d3, 3);
        if (badq >= 0 && threadIdx.x == 0 && bad == 0) bad = k0 + j + badq + 1;
        // row c of columns j .. j+3 of L (later rows: forward substitution)
        float l0 = 0.f, l1 = 0.f, l2 = 0.f, l3 = 0.f;
        if (c > j + 3) {
            l0 = v0 * i0;
            l1 = fmaf(-l0, L10, v1) * i1;
            l2 = fmaf(-l1, L21, fmaf(-l0, L20, v2)) * i2;
            l3 = fmaf(-l2, L32, fmaf(-l1, L31, fmaf(-l0, L30, v3))) * i3;
        }
        if (h == 0) {
            float w0 = l0, w1 = l1, w2 = l2, w3 = l3;
            if (own) {
                const float L00 = p00 * i0, L11 = d1 * i1, L22 = d2 * i2, L33 = d3 * i3;
                w0 = q == 0 ? L00 : q == 1 ? L10 : q == 2 ? L20 : L30;
                w1 = q == 0 ? 0.f : q == 1 ? L11 : q == 2 ? L21 : L31;
                w2 = q <= 1 ? 0.f : q == 2 ? L22 : L32;
                w3 = q <= 2 ? 0.f : L33;
            }
            LT[j][c] = w0;
            LT[j + 1][c] = w1;
            LT[j + 2][c] = w2;
            LT[j + 3][c] = w3;
        }
        {
            // T[j+h][c] = row h of L4^-1 times column c of the published rows
            const float m10 = -L10 * i0 * i1;
            const float m20 = -fmaf(L21, m10, L20 * i0) * i2, m21 = -L21 * i1 * i2;
            const float m30 = -fmaf(L32, m20, fmaf(L31, m10, L30 * i0)) * i3;
            const float m31 = -fmaf(L32, m21, L31 * i1) * i3, m32 = -L32 * i2 * i3;
            const float w0 = h == 0 ? i0 : h == 1 ? m10 : h == 2 ? m20 : m30;
            const float w1 = h == 0 ? 0.f : h == 1 ? i1 : h == 2 ? m21 : m31;
            const float w2 = h <= 1 ? 0.f : h == 2 ? i2 : m32;
            const float w3 = h <= 2 ? 0.f : i3;
            TR[j + h][c] = fmaf(w3, x3, fmaf(w2, x2, fmaf(w1, x1, w0 * x0)));
        }
        __syncthreads();
        if (c > j + 3) {
            const float lu[4] = {l0, l1, l2, l3};
            if (r0 + 15 >= j + 4) {
#pragma unroll
                for (int i = 0; i < 16; i += 4) {
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const float4 lr = *reinterpret_cast<const float4 *>(&LT[j + u][r0 + i]);
                        a[i] = fmaf(-lr.x, lu[u], a[i]);
                        a[i + 1] = fmaf(-lr.y, lu[u], a[i + 1]);
                        a[i + 2] = fmaf(-lr.z, lu[u], a[i + 2]);
                        a[i + 3] = fmaf(-lr.w, lu[u], a[i + 3]);
                    }
                }
            }
            if (r0 <= j + 3) {
#pragma unroll
                for (int i = 0; i < 16; i += 4) {
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const float4 tj = *reinterpret_cast<const float4 *>(&TR[j + u][r0 + i]);
                        t[i] = fmaf(-lu[u], tj.x, t[i]);
                        t[i + 1] = fmaf(-lu[u], tj.y, t[i + 1]);
                        t[i + 2] = fmaf(-lu[u], tj.z, t[i + 2]);
                        t[i + 3] = fmaf(-lu[u], tj.w, t[i + 3]);
                    }
                }
            }
        } else if (own) {
#pragma unroll
            for (int i = 0; i < 16; i += 4) {
                const float4 tj = *reinterpret_cast<const float4 *>(&TR[j + q][r0 + i]);
                t[i] = tj.x;
                t[i + 1] = tj.y;
                t[i + 2] = tj.z;
                t[i + 3] = tj.w;
            }
        }
    }
    __syncthreads();
    if (blockIdx.x == 0) {
        float *tb = Tb + c * kNB + r0;
#pragma unroll
        for (int i = 0; i < 16; i += 4)
            *reinterpret_cast<float4 *>(tb + i) =
                make_float4(r0 + i <= c ? t[i] : 0.f, r0 + i + 1 <= c ? t[i + 1] : 0.f,
                            r0 + i + 2 <= c ? t[i + 2] : 0.f, r0 + i + 3 <= c ? t[i + 3] : 0.f);
        if (threadIdx.x == 0 && bad && *info == 0) *info = bad;
    }
    // the panel: two threads per row, each 32 of its outputs,
    // L[i][cc] = sum_{k <= cc} P[i][k] T[cc][k]
    const int64_t row = k0 + kNB + 128 * static_cast<int64_t>(blockIdx.x) + (threadIdx.x & 127);
    const bool live = row < n;
    const int half = threadIdx.x >> 7;
    float *pr = P + row * n + k0;
    float x[kNB];
#pragma unroll
    for (int k = 0; k < kNB; k += 4) {
        const float4 v = live ? *reinterpret_cast<const float4 *>(pr + k) : make_float4(0.f, 0.f, 0.f, 0.f);
        x[k] = v.x;
        x[k + 1] = v.y;
        x[k + 2] = v.z;
        x[k + 3] = v.w;
    }
    // both halves of a row have read it before either writes (the row's two
    // threads are in different warps)
    __syncthreads();
    if (!live) return;
#pragma unroll 1
    for (int cc = 32 * half; cc < 32 * half + 32; cc += 8) {
        float o[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int k = 0; k < kNB; k += 4) {
            if (k < cc + 8) {
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const float4 tv = *reinterpret_cast<const float4 *>(&TR[cc + u][k]);
                    o[u] = fmaf(x[k], tv.x, o[u]);
                    o[u] = fmaf(x[k + 1], tv.y, o[u]);
                    o[u] = fmaf(x[k + 2], tv.z, o[u]);
                    o[u] = fmaf(x[k + 3], tv.w, o[u]);
                }
            }
        }
        *reinterpret_cast<float4 *>(pr + cc) = make_float4(o[0], o[1], o[2], o[3]);
        *reinterpret_cast<float4 *>(pr + cc + 4) = make_float4(o[4], o[5], o[6], o[7]);
    }
}

// B[e] = H[n*n - 1 - e]: both indices reversed.
__global__ void reverse_both(const float *__restrict__ H, int64_t n, float *__restrict__ B) {
    const int64_t total = n * n;
    for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < total;
         e += static_cast<int64_t>(gridDim.x) * blockDim.x)
        B[e] = H[total - 1 - e];
}

// U[i][j] = Linv[n-1-i][n-1-j] for j >= i, 0 below the diagonal.
__global__ void reverse_upper(const float *__restrict__ Linv, int64_t n, float *__restrict__ U) {
    const int64_t total = n * n;
    for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < total;
         e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t i = e / n, j = e - i * n;
        U[e] = j >= i ? Linv[total - 1 - e] : 0.f;
    }
}

// Linv's diagonal 64 x 64 blocks from the inverted Cholesky blocks, zero elsewhere
// above them (the strict upper triangle is zero; the lower part is written later).
__global__ void place_diag_inverses(const float *__restrict__ Tb, int64_t n,
                                    float *__restrict__ Linv) {
    const int64_t total = n * n;
    for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < total;
         e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t i = e / n, j = e - i * n;
        float v = 0.f;
        if (i / kNB == j / kNB) v = Tb[(i / kNB) * kNB * kNB + (i % kNB) * kNB + (j % kNB)];
        Linv[e] = v;
    }
}

}  // namespace

size_t linalg_scratch_floats(int64_t n) {
    // L (n x n), the temporary of the inversion (n x n / 4 at most), the
    // inverted diagonal blocks (n x 64)
    return size_t(n) * size_t(n) + size_t(n) * size_t(n) / 4 + size_t(n) * kNB;
}

int hessian(const void *X, int xt, int64_t Mc, int64_t K, float *H, cudaStream_t s) {
    // H[i][j] = 2 sum_m X[m][i] X[m][j]: A(i, m) = X[m * K + i] (i contiguous),
    // B(j, m) = X[m * K + j] (j contiguous); the tiles on and above the
    // diagonal (the factorization reads only those, through the reversal)
    GemmArgs g = gargs(X, K, X, K, H, K, static_cast<int>(K), static_cast<int>(K),
                       static_cast<int>(Mc), 2.0f, 0.0f);
    g.tri = kUpper;
    if (xt == W4_F16) return gemm<__half, __half, true, true>(g, 1, s);
    return gemm<__nv_bfloat16, __nv_bfloat16, true, true>(g, 1, s);
}

int inverse_factor(const char *fn, float *H, int64_t n, float *scratch, int *info_dev,
                   cudaStream_t s) {
    if (n % kNB != 0) return set_error(W4_ERR_UNSUPPORTED, fn, "n must be a multiple of 64");
    float *P = scratch;                       // P H P, factored in place into L
    float *Y = scratch + n * n;               // temporary of the inversion
    float *Tb = Y + n * n / 4;                // inverted diagonal blocks [n/64][64][64]
    cudaError_t e = cudaMemsetAsync(info_dev, 0, sizeof(int), s);
    if (e != cudaSuccess) return cuda_fail("clearing the factorization status", e);
    reverse_both<<<1184, 256, 0, s>>>(H, n, P);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail("reverse_both launch", e);
    // blocked right-looking Cholesky of P (lower)
    const int nb = static_cast<int>(n / kNB);
    for (int kb = 0; kb < nb; ++kb) {
        const int k0 = kb * kNB;
        const int rest = static_cast<int>(n) - k0 - kNB;
        chol_panel<<<max(1, (rest + 127) / 128), 256, 0, s>>>(P, n, k0, Tb + int64_t(kb) * kNB * kNB,
                                                               info_dev);
        if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail("chol_panel launch", e);
        if (rest == 0) break;
        // trailing update of the lower part: P[i][j] -= sum_c L[i][c] L[j][c]
        {
            const float *pan = P + int64_t(k0 + kNB) * n + k0;
            float *tr = P + int64_t(k0 + kNB) * n + k0 + kNB;
            GemmArgs g = gargs(pan, n, pan, n, tr, n, rest, rest, kNB, -1.f, 1.f);
            g.tri = kLower;
            int st = gemm<float, float, false, false>(g, 1, s);
            if (st != W4_OK) return st;
        }
    }
    // L^-1 into H's buffer: diagonal blocks, then recursive doubling
    float *Linv = H;
    place_diag_inverses<<<1184, 256, 0, s>>>(Tb, n, Linv);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail("place_diag_inverses launch", e);
    // level b: blocks [j b, min((j + 1) b, n)); pair p joins blocks 2p (size b)
    // and 2p + 1 (size cs <= b, smaller only for the last block); an unpaired
    // last block is already inverted and carries over to the next level
    for (int64_t b = kNB; b < n; b *= 2) {
        const int64_t nblk = (n + b - 1) / b;
        const int64_t npair = nblk / 2;
        const int64_t last_cs = n - (2 * npair - 1) * b;  // size of block 2(npair-1)+1
        const int64_t full = last_cs >= b ? npair : npair - 1;
        for (int part = 0; part < 2; ++part) {
            const int64_t p0 = part == 0 ? 0 : full;
            const int64_t cnt = part == 0 ? full : npair - full;
            if (cnt <= 0) continue;
            const int cs = static_cast<int>(part == 0 ? b : last_cs), bb = static_cast<int>(b);
            const int64_t off = p0 * (2 * b * n + 2 * b);  // element offset of pair p0's A block
            // Y_p = B_p A_p^-1 (cs x b): B_p = L[(2p+1)b.., 2pb..], A_p^-1 = Linv[2pb.., 2pb..]
            // (lower: A^-1[k][c] = 0 for k < c)
            {
                GemmArgs g = gargs(P + off + b * n, n, Linv + off, n, Y, b, cs, bb, bb, 1.f, 0.f);
                g.sA = 2 * b * n + 2 * b;
                g.sB = 2 * b * n + 2 * b;
                g.sC = b * b;
                g.k_from_n = 1;
                g.pair = 1;
                int st = gemm<float, float, false, true>(g, static_cast<int>(cnt), s);
                if (st != W4_OK) return st;
            }
            // Linv[(2p+1)b.., 2pb..] = -C_p^-1 Y_p (cs x b), C_p^-1 = Linv[(2p+1)b.., (2p+1)b..]
            // (lower: C^-1[r][k] = 0 for k > r)
            {
                GemmArgs g = gargs(Linv + off + b * n + b, n, Y, b, Linv + off + b * n, n, cs, bb, cs,
                                   -1.f, 0.f);
                g.sA = 2 * b * n + 2 * b;
                g.sB = b * b;
                g.sC = 2 * b * n + 2 * b;
                g.k_to_m = 1;
                g.pair = 2;
                int st = gemm<float, float, false, true>(g, static_cast<int>(cnt), s);
                if (st != W4_OK) return st;
            }
        }
    }
    int info = 0;
    e = cudaMemcpyAsync(&info, info_dev, sizeof info, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail("reading the factorization status", e);
    if (info != 0)
        return set_error(W4_ERR_INVALID_ARG, fn,
                         "the damped Hessian is not positive definite (raise the damping)");
    reverse_upper<<<1184, 256, 0, s>>>(Linv, n, P);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail("reverse_upper launch", e);
    e = cudaMemcpyAsync(H, P, sizeof(float) * size_t(n) * size_t(n), cudaMemcpyDeviceToDevice, s);
    if (e != cudaSuccess) return cuda_fail("copy of U", e);
    return W4_OK;
}

}  // namespace w4
