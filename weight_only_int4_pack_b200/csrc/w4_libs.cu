// w4_libs.cu -- the two NVIDIA libraries the calibration entry points call
// for plain dense linear algebra, opened on first use: cuBLAS (a GEMM with
// fp32 output: the unquantized layer's output in the AWQ search, the Hessian
// 2 X^T X of GPTQ) and cuSOLVER (Cholesky factorization and triangular
// inversion for the GPTQ inverse-Hessian factor).
//
// The library does not link them: only these calibration entry points use
// them, and the quantizer and GEMM entry points must load where they are
// absent.  The first use on a device opens libcublas.so.12 /
// libcusolver.so.11 (the process's copy when one is already loaded, e.g. by
// PyTorch) and creates one handle per device, kept for the life of the
// process.  Calls are serialized by a process-wide lock (a handle is bound
// to one stream at a time).

#include <cublas_v2.h>
#include <cusolverDn.h>
#include <dlfcn.h>

#include <mutex>
#include <vector>

#include "w4_internal.cuh"

namespace w4 {
namespace {

using PFN_blas_create = cublasStatus_t (*)(cublasHandle_t *);
using PFN_blas_set_stream = cublasStatus_t (*)(cublasHandle_t, cudaStream_t);
using PFN_gemm_ex = cublasStatus_t (*)(cublasHandle_t, cublasOperation_t, cublasOperation_t, int,
                                       int, int, const void *, const void *, cudaDataType, int,
                                       const void *, cudaDataType, int, const void *, void *,
                                       cudaDataType, int, cublasComputeType_t, cublasGemmAlgo_t);
using PFN_solver_create = cusolverStatus_t (*)(cusolverDnHandle_t *);
using PFN_solver_set_stream = cusolverStatus_t (*)(cusolverDnHandle_t, cudaStream_t);
using PFN_potrf_bufsize = cusolverStatus_t (*)(cusolverDnHandle_t, cublasFillMode_t, int, float *,
                                               int, int *);
using PFN_potrf = cusolverStatus_t (*)(cusolverDnHandle_t, cublasFillMode_t, int, float *, int,
                                       float *, int, int *);
using PFN_trtri_bufsize = cusolverStatus_t (*)(cusolverDnHandle_t, cublasFillMode_t,
                                               cublasDiagType_t, int64_t, cudaDataType, void *,
                                               int64_t, size_t *, size_t *);
using PFN_trtri = cusolverStatus_t (*)(cusolverDnHandle_t, cublasFillMode_t, cublasDiagType_t,
                                       int64_t, cudaDataType, void *, int64_t, void *, size_t,
                                       void *, size_t, int *);

constexpr int kMaxDevices = 64;
std::mutex g_mu;

PFN_blas_create g_blas_create = nullptr;
PFN_blas_set_stream g_blas_set_stream = nullptr;
PFN_gemm_ex g_gemm_ex = nullptr;
cublasHandle_t g_blas[kMaxDevices] = {};

PFN_solver_create g_solver_create = nullptr;
PFN_solver_set_stream g_solver_set_stream = nullptr;
PFN_potrf_bufsize g_potrf_bufsize = nullptr;
PFN_potrf g_potrf = nullptr;
PFN_trtri_bufsize g_trtri_bufsize = nullptr;
PFN_trtri g_trtri = nullptr;
cusolverDnHandle_t g_solver[kMaxDevices] = {};

int current_device(const char *fn, int *dev) {
    cudaError_t e = cudaGetDevice(dev);
    if (e != cudaSuccess) return cuda_fail("cudaGetDevice", e);
    if (*dev < 0 || *dev >= kMaxDevices) return set_error(W4_ERR_CUDA, fn, "device ordinal out of range");
    return W4_OK;
}

// Caller holds g_mu.
int blas_handle(const char *fn, cublasHandle_t *out) {
    int dev = 0, st = current_device(fn, &dev);
    if (st != W4_OK) return st;
    if (!g_gemm_ex) {
        void *h = dlopen("libcublas.so.12", RTLD_NOW | RTLD_LOCAL);
        if (!h) return set_error(W4_ERR_UNSUPPORTED, fn, "libcublas.so.12 could not be loaded");
        g_blas_create = reinterpret_cast<PFN_blas_create>(dlsym(h, "cublasCreate_v2"));
        g_blas_set_stream = reinterpret_cast<PFN_blas_set_stream>(dlsym(h, "cublasSetStream_v2"));
        g_gemm_ex = reinterpret_cast<PFN_gemm_ex>(dlsym(h, "cublasGemmEx"));
        if (!g_blas_create || !g_blas_set_stream || !g_gemm_ex) {
            g_gemm_ex = nullptr;
            return set_error(W4_ERR_UNSUPPORTED, fn, "libcublas.so.12 lacks cublasGemmEx");
        }
    }
    if (!g_blas[dev]) {
        cublasHandle_t h = nullptr;
        if (g_blas_create(&h) != CUBLAS_STATUS_SUCCESS)
            return set_error(W4_ERR_CUDA, fn, "cublasCreate failed");
        g_blas[dev] = h;
    }
    *out = g_blas[dev];
    return W4_OK;
}

// Caller holds g_mu.
int solver_handle(const char *fn, cusolverDnHandle_t *out) {
    int dev = 0, st = current_device(fn, &dev);
    if (st != W4_OK) return st;
    if (!g_trtri) {
        void *h = dlopen("libcusolver.so.11", RTLD_NOW | RTLD_LOCAL);
        if (!h) return set_error(W4_ERR_UNSUPPORTED, fn, "libcusolver.so.11 could not be loaded");
        g_solver_create = reinterpret_cast<PFN_solver_create>(dlsym(h, "cusolverDnCreate"));
        g_solver_set_stream =
            reinterpret_cast<PFN_solver_set_stream>(dlsym(h, "cusolverDnSetStream"));
        g_potrf_bufsize = reinterpret_cast<PFN_potrf_bufsize>(dlsym(h, "cusolverDnSpotrf_bufferSize"));
        g_potrf = reinterpret_cast<PFN_potrf>(dlsym(h, "cusolverDnSpotrf"));
        g_trtri_bufsize = reinterpret_cast<PFN_trtri_bufsize>(dlsym(h, "cusolverDnXtrtri_bufferSize"));
        g_trtri = reinterpret_cast<PFN_trtri>(dlsym(h, "cusolverDnXtrtri"));
        if (!g_solver_create || !g_solver_set_stream || !g_potrf_bufsize || !g_potrf ||
            !g_trtri_bufsize || !g_trtri) {
            g_trtri = nullptr;
            return set_error(W4_ERR_UNSUPPORTED, fn, "libcusolver.so.11 lacks potrf / trtri");
        }
    }
    if (!g_solver[dev]) {
        cusolverDnHandle_t h = nullptr;
        if (g_solver_create(&h) != CUSOLVER_STATUS_SUCCESS)
            return set_error(W4_ERR_CUDA, fn, "cusolverDnCreate failed");
        g_solver[dev] = h;
    }
    *out = g_solver[dev];
    return W4_OK;
}

}  // namespace

int blas_gemm_f32(const char *fn, bool trans_a, bool trans_b, int m, int n, int k, float alpha,
                  const void *A, int at, int lda, const void *B, int bt, int ldb, float beta,
                  float *C, int ldc, cudaStream_t stream) {
    std::lock_guard<std::mutex> lk(g_mu);
    cublasHandle_t h = nullptr;
    int st = blas_handle(fn, &h);
    if (st != W4_OK) return st;
    if (g_blas_set_stream(h, stream) != CUBLAS_STATUS_SUCCESS)
        return set_error(W4_ERR_CUDA, fn, "cublasSetStream failed");
    const cudaDataType ta = at == W4_F16 ? CUDA_R_16F : CUDA_R_16BF;
    const cudaDataType tb = bt == W4_F16 ? CUDA_R_16F : CUDA_R_16BF;
    const cublasStatus_t bs =
        g_gemm_ex(h, trans_a ? CUBLAS_OP_T : CUBLAS_OP_N, trans_b ? CUBLAS_OP_T : CUBLAS_OP_N, m, n,
                  k, &alpha, A, ta, lda, B, tb, ldb, &beta, C, CUDA_R_32F, ldc, CUBLAS_COMPUTE_32F,
                  CUBLAS_GEMM_DEFAULT);
    if (bs != CUBLAS_STATUS_SUCCESS) return set_error(W4_ERR_CUDA, fn, "cublasGemmEx failed");
    return W4_OK;
}

size_t solver_work_bytes(int64_t n) {
    // potrf / trtri of an fp32 n x n matrix ask for far less (a few panel
    // widths times n); the run-time query is checked against this.
    const size_t v = sizeof(float) * size_t(n) * 512;
    return v < (size_t(1) << 22) ? (size_t(1) << 22) : v;
}

namespace {

// B[i][j] = H[n-1-i][n-1-j]: the matrix with its index order reversed
// (grid-stride over the n^2 elements; consecutive threads read consecutive,
// descending addresses).
__global__ void reverse_both(const float *__restrict__ H, int64_t n, float *__restrict__ B) {
    const int64_t total = n * n;
    for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < total;
         e += static_cast<int64_t>(gridDim.x) * blockDim.x)
        B[e] = H[total - 1 - e];
}

// U[i][j] = Linv(n-1-i, n-1-j) for j >= i (0 below), Linv the lower-triangular
// column-major matrix in B (element (r, c) at B[r + c n]), i.e.
// U[i][j] = B[(n-1-j) n + (n-1-i)]: a transpose, done through 32 x 32 shared
// tiles so that both the reads and the writes are coalesced.  Block (32, 8).
__global__ void reverse_transpose_upper(const float *__restrict__ B, int64_t n,
                                        float *__restrict__ U) {
    __shared__ float tile[32][33];
    const int64_t i0 = static_cast<int64_t>(blockIdx.y) * 32, j0 = static_cast<int64_t>(blockIdx.x) * 32;
    const int tx = threadIdx.x;
    for (int ty = threadIdx.y; ty < 32; ty += 8) {
        const int64_t j = j0 + ty, i = i0 + tx;
        if (i < n && j < n) tile[ty][tx] = B[(n - 1 - j) * n + (n - 1 - i)];
    }
    __syncthreads();
    for (int ty = threadIdx.y; ty < 32; ty += 8) {
        const int64_t i = i0 + ty, j = j0 + tx;
        if (i < n && j < n) U[i * n + j] = j >= i ? tile[tx][ty] : 0.0f;
    }
}

}  // namespace

// U, the upper Cholesky factor of H^-1 (H^-1 = U^T U), without forming H^-1:
// with P the index reversal, P H P = Lr Lr^T (lower Cholesky), so
// H = R R^T with R = P Lr P upper triangular and H^-1 = R^-T R^-1; U = R^-1 =
// P Lr^-1 P is upper triangular with a positive diagonal, hence the Cholesky
// factor.  One potrf and one trtri (half the flops of potrf + potri + potrf).
int solver_inverse_factor(const char *fn, float *H, int n, float *scratch, void *work,
                          size_t work_bytes, int *info_dev, cudaStream_t stream) {
    std::lock_guard<std::mutex> lk(g_mu);
    cusolverDnHandle_t h = nullptr;
    int st = solver_handle(fn, &h);
    if (st != W4_OK) return st;
    if (g_solver_set_stream(h, stream) != CUSOLVER_STATUS_SUCCESS)
        return set_error(W4_ERR_CUDA, fn, "cusolverDnSetStream failed");
    reverse_both<<<1184, 256, 0, stream>>>(H, n, scratch);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail("reverse_both launch", e);
    int lwork = 0;
    size_t dev_bytes = 0, host_bytes = 0;
    if (g_potrf_bufsize(h, CUBLAS_FILL_MODE_LOWER, n, scratch, n, &lwork) != CUSOLVER_STATUS_SUCCESS ||
        g_trtri_bufsize(h, CUBLAS_FILL_MODE_LOWER, CUBLAS_DIAG_NON_UNIT, n, CUDA_R_32F, scratch, n,
                        &dev_bytes, &host_bytes) != CUSOLVER_STATUS_SUCCESS)
        return set_error(W4_ERR_CUDA, fn, "cuSOLVER buffer size query failed");
    if (size_t(lwork) * sizeof(float) > work_bytes || dev_bytes > work_bytes)
        return set_error(W4_ERR_UNSUPPORTED, fn, "cuSOLVER asks for more work space than reserved");
    std::vector<unsigned char> host(host_bytes > 0 ? host_bytes : 1);
    if (g_potrf(h, CUBLAS_FILL_MODE_LOWER, n, scratch, n, static_cast<float *>(work), lwork,
                info_dev) != CUSOLVER_STATUS_SUCCESS ||
        g_trtri(h, CUBLAS_FILL_MODE_LOWER, CUBLAS_DIAG_NON_UNIT, n, CUDA_R_32F, scratch, n, work,
                work_bytes, host.data(), host_bytes, info_dev + 1) != CUSOLVER_STATUS_SUCCESS)
        return set_error(W4_ERR_CUDA, fn, "cuSOLVER potrf / trtri failed to launch");
    int info[2] = {0, 0};
    e = cudaMemcpyAsync(info, info_dev, sizeof info, cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return cuda_fail("reading the factorization status", e);
    if (info[0] != 0 || info[1] != 0)
        return set_error(W4_ERR_INVALID_ARG, fn,
                         "the damped Hessian is not positive definite (raise the damping)");
    const dim3 tiles(static_cast<unsigned>((n + 31) / 32), static_cast<unsigned>((n + 31) / 32));
    reverse_transpose_upper<<<tiles, dim3(32, 8), 0, stream>>>(scratch, n, H);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail("reverse_transpose_upper launch", e);
    return W4_OK;
}

}  // namespace w4
